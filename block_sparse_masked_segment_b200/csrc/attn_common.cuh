// attn_common.cuh - pieces shared by the attention kernels: parameters,
// shared-memory tile geometry, descriptor helpers and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
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
// The 128 columns of a partial tile split into runs of equal (conversation,
// turn, type).  Warp-wide: lanes have written conv[]/meta[] of the tile; the
// run starts are returned as a 128-bit mask (bit c of starts[c / 32]).
__device__ __forceinline__ void build_run_starts(const int32_t* conv, const int32_t* meta, uint32_t* starts,
                                                 int lane) {
  __syncwarp();
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int c = w * 32 + lane;
    const bool st = (c == 0) || conv[c] != conv[c - 1] || meta[c] != meta[c - 1];
    const uint32_t b = __ballot_sync(0xffffffffu, st);
    if (lane == 0) starts[w] = b;
  }
}

// First run start at or after column x (128 if none).
__device__ __forceinline__ int next_run_start(const uint32_t (&st)[4], int x) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    if (x < 32 * (w + 1)) {
      const int sh = x - 32 * w;
      const uint32_t m = sh <= 0 ? st[w] : (st[w] & (0xffffffffu << sh));
      if (m) return 32 * w + __ffs(m) - 1;
    }
  }
  return 128;
}

// Set bits [a, b) of a 128-bit mask.
__device__ __forceinline__ void set_bit_range(uint32_t (&m)[4], int a, int b) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int lo = max(a, 32 * w), hi = min(b, 32 * w + 32);
    if (lo < hi) {
      const int n = hi - lo;
      const uint32_t bits = n == 32 ? 0xffffffffu : ((1u << n) - 1u);
      m[w] |= bits << (lo - 32 * w);
    }
  }
}

// Does a query of meta qmeta see a key of meta kmeta (same conversation, key not after the query)?
__device__ __forceinline__ bool type_rule(int32_t qmeta, int32_t kmeta) {
  const uint32_t bits = (kmeta < (qmeta & ~3)) ? kPrevTurnBits : ((kSameTurnBits >> ((qmeta & 3) * 4)) & 0xFu);
  return (bits >> (kmeta & 3)) & 1u;
}

// Mask of the keys kbase + c (c < 128) visible from query qg: one rule test per
// column run, with the causal limit k <= qg.
__device__ __forceinline__ void query_row_mask(const uint32_t* starts_smem, const int32_t* kconv, const int32_t* kmeta,
                                               int kbase, int qg, int qconv, int qmeta, uint32_t (&m)[4]) {
  m[0] = m[1] = m[2] = m[3] = 0u;
  const int lim = min(qg - kbase + 1, 128);
  if (lim <= 0) return;
  const uint32_t st[4] = {starts_smem[0], starts_smem[1], starts_smem[2], starts_smem[3]};
  int a = 0;
  while (a < lim) {
    const int b = next_run_start(st, a + 1);
    if (kconv[a] == qconv && type_rule(qmeta, kmeta[a])) set_bit_range(m, a, min(b, lim));
    a = b;
  }
}

// Mask of the queries qbase + c (c < 128) that see key kg (roles of query_row_mask swapped).
__device__ __forceinline__ void key_row_mask(const uint32_t* starts_smem, const int32_t* qconv, const int32_t* qmeta,
                                             int qbase, int kg, int kconv, int kmeta, uint32_t (&m)[4]) {
  m[0] = m[1] = m[2] = m[3] = 0u;
  const int first = max(kg - qbase, 0);
  if (first >= 128) return;
  const uint32_t st[4] = {starts_smem[0], starts_smem[1], starts_smem[2], starts_smem[3]};
  int a = 0;
  while (a < 128) {
    const int b = next_run_start(st, a + 1);
    if (b > first && qconv[a] == kconv && type_rule(qmeta[a], kmeta)) set_bit_range(m, max(a, first), b);
    a = b;
  }
}

__device__ __forceinline__ bool mask_bit(const uint32_t (&m)[4], int c) { return (m[c >> 5] >> (c & 31)) & 1u; }

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
  const float* d_tiles;     // D = rowsum(dO * O), [hq][n_items][128]
  const float* lse2_tiles;  // LSE * log2(e), [hq][n_items][128]
  float* dq;
  float* dk;
  float* dv;
  int32_t* dev_status;
};

}  // namespace opr
