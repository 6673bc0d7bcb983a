// attn_common.cuh - pieces shared by the attention kernels: parameters,
// shared-memory tile geometry, descriptor helpers and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "opr_internal.cuh"
#include "sm100.cuh"

namespace opr {

// 2 s: any pipeline wait longer than this is a hang.  The pipeline waits take their
// limit from AttnParams::wait_ns (this value unless a test lowers it); the drains
// before a CTA exits always use this one.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

#ifdef OPR_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// CTA shape shared by the attention kernels: warp 0 TMA producer, warp 1 TMEM
// owner / MMA issuer, warps 2..9 compute.  Two compute warps share each TMEM
// lane quadrant (warp % 4): warps 2..5 own columns 0..63 of their rows, warps
// 6..9 columns 64..127.
constexpr int kThreads = 320;
constexpr int kComputeThreads = 256;

// Bounded mbarrier wait taken by a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, limit_ns));
}

// A 128-row tile of head_dim D bf16 values is stored as D/64 "chunks", each
// 128 rows x 128 bytes with the 128-byte swizzle TMA writes (box {64, 1, 128}).
constexpr int kChunkBytes = kTile * 128;  // 16 KiB

template <int D>
struct TileGeom {
  static constexpr int kChunks = D / 64;
  static constexpr int kBytes = kChunks * kChunkBytes;
};

// K-major operand (rows x D, D contiguous): the MMA's K step kk (16 elements)
// lies in chunk kk/4 at byte offset 32*(kk%4) inside each 128-byte row.
// Leading byte offset is unused for swizzled K-major layouts (encoded as 16),
// stride byte offset = 1024 (eight 128-byte rows).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_saddr, int kk) {
  return smem_desc_sw128(tile_saddr + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024);
}

// MN-major operand (K rows x N, N contiguous, i.e. a [keys][D] tile used as
// the N x K operand of P V): the K step kk (16 rows) starts 16*128 bytes
// further; along N the 64-element chunks are kChunkBytes apart (leading byte
// offset), eight K rows span 1024 bytes (stride byte offset).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile_saddr, int kk) {
  return smem_desc_sw128(tile_saddr + kk * 2048, kChunkBytes, 1024);
}

// The same descriptors as a base (K step 0) plus a per-step increment of the
// start-address field: the MMA issue loops build the base once per tile and
// add a compile-time constant per step, so each MMA costs one 64-bit add.
// (Shared-memory addresses stay below 2^18 bytes, so the 14-bit start field
// never carries into the next field.)
__device__ __forceinline__ constexpr uint64_t kmajor_step(int kk) {
  return static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
}
__device__ __forceinline__ constexpr uint64_t mnmajor_step(int kk) { return static_cast<uint64_t>((kk * 2048) >> 4); }

// Loads a [128 tokens][D] tile of one head with TMA (D/64 boxes).
template <int D>
__device__ __forceinline__ void tma_tile(const CUtensorMap* map, uint64_t* bar, void* dst, int head, int tok0) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c)
    tma_load_3d(map, bar, static_cast<char*>(dst) + c * kChunkBytes, c * 64, head, tok0);
}

// Dynamic shared memory requested by every TMEM kernel: at least this much so
// that only one CTA fits on an SM (each CTA allocates all 512 TMEM columns).
constexpr size_t kMinSmemOneCtaPerSm = 116 * 1024;

__host__ __device__ constexpr size_t smem_request(size_t need) {
  return need > kMinSmemOneCtaPerSm ? need : kMinSmemOneCtaPerSm;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// ---------------------------------------------------------------- partial tiles
// Set bits [a, b) (0 <= a <= b <= 128) of a 128-bit mask held as two 64-bit words.
__device__ __forceinline__ void set_range128(uint64_t& lo, uint64_t& hi, int a, int b) {
  const int la = min(a, 64), lb = min(b, 64);
  const int ha = max(a, 64) - 64, hb = max(b, 64) - 64;
  const uint64_t lmask = (lb == 64 ? ~0ull : ((1ull << lb) - 1ull)) & ~((la == 64) ? ~0ull : ((1ull << la) - 1ull));
  const uint64_t hmask = (hb == 64 ? ~0ull : ((1ull << hb) - 1ull)) & ~((ha == 64) ? ~0ull : ((1ull << ha) - 1ull));
  if (la < lb) lo |= lmask;
  if (ha < hb) hi |= hmask;
}

// Does a query of meta qmeta see a key of meta kmeta (same conversation, key not after the query)?
__device__ __forceinline__ bool type_rule(int32_t qmeta, int32_t kmeta) { return turn_type_rule(qmeta, kmeta); }

// Mask of the keys kbase + c (c < 128) visible from query qg: one rule test per
// run of the key tile, with the causal limit k <= qg.  m[w] holds columns 32w..32w+31.
__device__ __forceinline__ void query_row_mask(const TileMeta& t, int kbase, int qg, int qconv, int qmeta,
                                               uint32_t (&m)[4]) {
  uint64_t lo = 0ull, hi = 0ull;
  const int lim = min(max(qg - kbase + 1, 0), 128);
  const int nr = min(t.nruns, kTile);  // a record always has 1..128 runs
#pragma unroll 4
  for (int r = 0; r < nr; ++r) {
    const int a = t.bound[r], b = min(t.bound[r + 1], lim);
    if (a < b && t.conv[r] == qconv && type_rule(qmeta, t.meta[r])) set_range128(lo, hi, a, b);
  }
  m[0] = static_cast<uint32_t>(lo);
  m[1] = static_cast<uint32_t>(lo >> 32);
  m[2] = static_cast<uint32_t>(hi);
  m[3] = static_cast<uint32_t>(hi >> 32);
}

// Mask of the queries qbase + c (c < 128) that see key kg (roles swapped: runs of the query tile).
__device__ __forceinline__ void key_row_mask(const TileMeta& t, int qbase, int kg, int kconv, int kmeta,
                                             uint32_t (&m)[4]) {
  uint64_t lo = 0ull, hi = 0ull;
  const int first = min(max(kg - qbase, 0), 128);
  const int nr = min(t.nruns, kTile);  // a record always has 1..128 runs
#pragma unroll 4
  for (int r = 0; r < nr; ++r) {
    const int a = max(t.bound[r], first), b = t.bound[r + 1];
    if (a < b && t.conv[r] == kconv && type_rule(t.meta[r], kmeta)) set_range128(lo, hi, a, b);
  }
  m[0] = static_cast<uint32_t>(lo);
  m[1] = static_cast<uint32_t>(lo >> 32);
  m[2] = static_cast<uint32_t>(hi);
  m[3] = static_cast<uint32_t>(hi >> 32);
}

__device__ __forceinline__ bool mask_bit(const uint32_t (&m)[4], int c) { return (m[c >> 5] >> (c & 31)) & 1u; }

// Debug builds (OPR_DEBUG_CHECKS) check, before their first use, the indices an
// attention CTA takes from the layout tables: its tile id, the sequence bounds of
// the tile, the length of its tile list and each entry of the list (a tile inside
// the sequence, class full or partial).  On a failure every thread of the CTA
// returns false (one block-wide vote, taken before any barrier, TMEM allocation or
// copy) and OPR_DEV_BOUNDS is set; the caller then returns without touching
// memory through those indices.  Release builds compile it to `true`.
template <typename Params>
__device__ __forceinline__ bool debug_tile_ok(const Params& p, int tile_id, const int32_t* cnt_tab,
                                              const int32_t* list_tab) {
  if constexpr (!kDebugChecks) {
    return true;
  } else {
    bool bad = p.T <= 0 || tile_id < 0 || tile_id >= p.n_items;
    int n = 0, seq_len = 0;
    if (!bad) {
      const int s = tile_id / p.T, I = tile_id % p.T;
      const int a = p.cu_seqlens[s], b = p.cu_seqlens[s + 1];
      n = cnt_tab[tile_id];
      seq_len = b - a;
      bad = a < 0 || b < a || b > p.total || n < 0 || n > p.T || (n > 0 && I * kTile >= seq_len);
    }
    if (!bad) {
      const int32_t* list = list_tab + static_cast<size_t>(tile_id) * p.T;
      for (int x = threadIdx.x; x < n && !bad; x += blockDim.x) {
        const int e = list[x];
        const int idx = entry_index(e), cls = entry_class(e);
        bad = idx < 0 || idx >= p.T || idx * kTile >= seq_len || (cls != OPR_TILE_FULL && cls != OPR_TILE_PARTIAL);
      }
    }
    bad = __syncthreads_or(bad) != 0;
    if (bad && threadIdx.x == 0) atomicOr(p.dev_status, OPR_DEV_BOUNDS);
    return !bad;
  }
}

// Tensor maps and buffers of one backward call (built by the entry point).
struct BwdMaps {
  CUtensorMap q, k, v, dout;  // the call's operands (q/k type, bf16 v and dO)
  CUtensorMap v16, dout16;    // fp16 copies of v and dO in the workspace
};

struct BwdBuffers {
  uint32_t* dout_absmax;  // one word: bits of max |dO|
  const void* o;
  int o_fp32;
  const __nv_bfloat16* dout;
  const __nv_bfloat16* v;
  float* row_terms;  // D tiles, then LSE * log2(e) tiles
  __half* dout16;
  __half* v16;
  const int32_t* rope_pos;  // not null: rotate dq and dk back by these positions (base rope_base)
  double rope_base;
};

// Token rows of the attention kernels are attention positions (the layout's
// attention order): q, k and v tiles, conv_idx and tok_meta are in that order;
// stream_of maps a position to the stream row that O, LSE, dO, dQ, dK and dV
// (and v in the backward) use.
struct AttnParams {
  const int32_t* cu_seqlens;
  const int32_t* stream_of;
  const int32_t* conv_idx;
  const int32_t* tok_meta;
  const int32_t* row_cnt;
  const int32_t* row_list;
  const int32_t* col_cnt;
  const int32_t* col_list;
  const int32_t* sched;
  const TileMeta* tile_meta;
  int32_t T;
  int32_t n_items;
  int64_t total;
  int32_t hq, hkv;
  float scale;
  float scale_log2;
  // forward outputs
  void* o;
  int32_t o_fp32;
  float* lse;
  // backward
  const float* lse_in;      // [hq, total]
  const float* d_tiles;     // -2^k D = -2^k rowsum(dO * O), [hq][n_items][128]
  const float* lse2_tiles;  // -LSE * log2(e), [hq][n_items][128]
  const uint32_t* dout_absmax;  // bits of max |dO| (a non-negative float), sets the scale 2^k
  float* dq;
  float* dk;
  float* dv;
  // dK/dV split by q head (small grids): the dK/dV grid has one CTA per (key tile,
  // q head).  A key column of at least split_min_cnt query tiles is split: each CTA
  // writes its head's dK and dV to dk_part / dv_part [hq][total][D], which a second
  // kernel sums per GQA group into dk / dv.  A shorter column is done whole by the
  // CTA of the group's first head, which writes dk / dv itself.
  int32_t dkdv_split;
  int32_t split_min_cnt;
  float* dk_part;
  float* dv_part;
  int32_t* dev_status;
  uint32_t wait_ns;  // limit of the pipeline waits (kWaitLimitNs; 0: a wait not already done times out)
};

// ---------------------------------------------------------------- gradient scale
// The backward is linear in dO, so it runs on 2^k dO and divides the results
// by 2^k (exact: a power of two).  k puts max |2^k dO| in [8, 16): the fp16
// copies of dO and the fp16 dS keep their 11-bit significands for small
// upstream gradients (loss / token count, 1e-5 .. 1e-8), which fp16 would
// otherwise hold as subnormals or zero, and large ones stay inside the fp16
// range.  `bits` is max |dO| as float bits; zero, inf and NaN give k = 0.
__host__ __device__ __forceinline__ int grad_scale_exp(uint32_t bits) {
  const int e = static_cast<int>((bits >> 23) & 0xFFu);  // biased exponent
  if (bits == 0u || e == 0xFF) return 0;
  const int k = e == 0 ? 100 : 130 - e;  // max = 1.f * 2^(e - 127) -> 1.f * 2^(e - 127 + k) in [8, 16)
  return k < -100 ? -100 : (k > 100 ? 100 : k);
}

// 2^x for a pair of fp32 values on the FMA and integer pipes instead of the
// special-function unit (which the softmax otherwise saturates): x = n + f with
// n = rint(x), taken by adding 1.5 * 2^23 (Cody and Waite's additive range
// reduction); 2^f by the degree-3 Chebyshev interpolant of 2^f on [-1/2, 1/2]
// (coefficients from csrc/exp2_poly.py, relative error below 1e-4); n added to
// the exponent field.  Exact 0 for x below -125 (and for -inf), where the
// exponent would leave the normal range (the special-function unit flushes
// there too).
__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x2) {
  constexpr float kShift = 12582912.f;  // 1.5 * 2^23: its ulp is 1
  constexpr float kC0 = 9.999245405e-01f, kC1 = 6.931367517e-01f, kC2 = 2.426394820e-01f, kC3 = 5.583828315e-02f;
  const uint64_t t2 = fadd2(x2, f2(kShift, kShift));      // the low mantissa bits hold rint(x)
  const uint64_t n2 = fadd2(t2, f2(-kShift, -kShift));    // rint(x)
  const uint64_t fr = ffma2(n2, f2(-1.f, -1.f), x2);      // f = x - rint(x) in [-1/2, 1/2]
  uint64_t p = ffma2(f2(kC3, kC3), fr, f2(kC2, kC2));
  p = ffma2(p, fr, f2(kC1, kC1));
  p = ffma2(p, fr, f2(kC0, kC0));
  float xl, xh, pl, ph, tl, th;
  f2_split(x2, xl, xh);
  f2_split(p, pl, ph);
  f2_split(t2, tl, th);
  // bits(t) << 23 is rint(x) << 23 (the shifter's own bits vanish in the shift)
  const float rl = __int_as_float(__float_as_int(pl) + (__float_as_int(tl) << 23));
  const float rh = __int_as_float(__float_as_int(ph) + (__float_as_int(th) << 23));
  return f2(xl >= -125.f ? rl : 0.f, xh >= -125.f ? rh : 0.f);
}

// 2^k as a float, built from its bits (|k| <= 126).
__host__ __device__ __forceinline__ float pow2f(int k) {
  const uint32_t b = static_cast<uint32_t>(127 + k) << 23;
  float f;
  memcpy(&f, &b, sizeof f);
  return f;
}

}  // namespace opr
