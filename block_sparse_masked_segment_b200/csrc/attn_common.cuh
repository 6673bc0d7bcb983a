// attn_common.cuh - pieces shared by the attention kernels: parameters,
// shared-memory tile geometry, descriptor helpers and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "opr_internal.cuh"
#include "sm100.cuh"

namespace opr {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: any pipeline wait longer than this is a hang

// CTA shape shared by the attention kernels: warp 0 TMA producer, warp 1 TMEM
// owner / MMA issuer, warps 2..9 compute.  Two compute warps share each TMEM
// lane quadrant (warp % 4): warps 2..5 own columns 0..63 of their rows, warps
// 6..9 columns 64..127.
constexpr int kThreads = 320;
constexpr int kComputeThreads = 256;

// Bounded mbarrier wait taken by a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kWaitLimitNs));
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
__device__ __forceinline__ bool type_rule(int32_t qmeta, int32_t kmeta) {
  const uint32_t bits = (kmeta < (qmeta & ~3)) ? kPrevTurnBits : ((kSameTurnBits >> ((qmeta & 3) * 4)) & 0xFu);
  return (bits >> (kmeta & 3)) & 1u;
}

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

// Tensor maps and buffers of one backward call (built by the entry point).
struct BwdMaps {
  CUtensorMap q, k, v, dout;  // the call's operands (q/k type, bf16 v and dO)
  CUtensorMap v16, dout16;    // fp16 copies of v and dO in the workspace
};

struct BwdBuffers {
  const void* o;
  int o_fp32;
  const __nv_bfloat16* dout;
  const __nv_bfloat16* v;
  float* row_terms;  // D tiles, then LSE * log2(e) tiles
  __half* dout16;
  __half* v16;
};

struct AttnParams {
  const int32_t* cu_seqlens;
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
  const float* d_tiles;     // -D = -rowsum(dO * O), [hq][n_items][128]
  const float* lse2_tiles;  // -LSE * log2(e), [hq][n_items][128]
  float* dq;
  float* dk;
  float* dv;
  int32_t* dev_status;
};

}  // namespace opr
