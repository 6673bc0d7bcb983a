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

struct AttnParams {
  const int32_t* cu_seqlens;
  const int32_t* conv_idx;
  const int32_t* tok_meta;
  const int32_t* row_cnt;
  const int32_t* row_list;
  const int32_t* col_cnt;
  const int32_t* col_list;
  const int32_t* sched;
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
  const float* lse_in;
  const float* row_d;  // D = rowsum(dO * O), [hq, total]
  float* dq;
  float* dk;
  float* dv;
  int32_t* dev_status;
};

}  // namespace opr
