// attn_bwd.cu - block-sparse masked attention backward for sm_100a.
//
// Gradients of the One-Pass to Reason attention layer (fine-tuning needs
// them; the mask is the one of "分块稀疏注意力掩码").  With P recomputed from
// the forward's log-sum-exp:
//   D  = rowsum(dO * O)
//   dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D)
//   dQ = scale dS K,   dK = scale dS^T Q   (dK, dV summed over a GQA group)
// Deterministic split into two tcgen05 kernels (no atomics):
//   dq kernel    one CTA per (query tile, q head), loops over the row's
//                non-empty key tiles: S, dP -> dS (TMEM) -> dQ += dS K;
//   dkdv kernel  one CTA per (key tile, kv head), loops over the column's
//                non-empty query tiles and, for each, the q heads of the group:
//                S^T = K Q^T, dP^T = V dO^T -> P^T, dS^T (TMEM) ->
//                dV += P^T dO, dK += dS^T Q.
// Q/K and the dS operand share one 16-bit type (fp16 when QK16, else bf16).
// Both kernels form dP from fp16 copies of 2^k dO and of V, which the row-terms
// stage writes in the attention order; P^T is an fp16 operand of dV = P^T dO
// (bf16 P^T loses too much there).  Q, K, the copies and the tile lists are in
// the attention order; dQ, dK, dV rows go back to their stream rows.
// Warp roles as in the forward: warp 0 TMA producer (+ metadata lanes),
// warp 1 TMEM owner and MMA issuer, warps 2..9 two threads per TMEM lane
// (row), each owning 64 of the tile's 128 columns.
#include <cuda_fp16.h>

#include <algorithm>

#include "attn_common.cuh"

namespace opr {
namespace {

constexpr int kStages = 2;
constexpr int kListSmem = 1024;  // entries of a tile list kept in shared memory
constexpr float kLog2e = 1.4426950408889634f;

// ----------------------------------------------------------------------------
// max |dO| over the whole tensor, as float bits (non-negative floats order
// like their bits), into *absmax (zeroed before the launch).  It fixes the
// gradient scale 2^k of the call (grad_scale_exp).
__global__ void __launch_bounds__(256) dout_absmax_kernel(const __nv_bfloat16* __restrict__ x, int64_t n8,
                                                          uint32_t* __restrict__ absmax) {
  float m = 0.f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // |bf16| of both halves: clear the sign bits, widen to fp32 by a shift
      m = fmax3(m, __uint_as_float((w[k] & 0x7FFFu) << 16), __uint_as_float(w[k] & 0x7FFF0000u));
    }
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wm[w]);
    atomicMax(absmax, __float_as_uint(m));
  }
}

// Row terms, stored negated and per 128-token tile so the kernels can
// bulk-copy them and fold each into one fused multiply-add:
// d_tiles[h][tile][c] = -2^k sum_d dO * O and lse2_tiles[h][tile][c] = -LSE * log2(e)
// of token c of tile (s, J); 0 and -inf past the end of the sequence.  The
// kernel also writes dout16, the fp16 copy of 2^k dO that the dkdv kernel
// reads (exact: 2^k dO lies in fp16's normal range except for entries below
// 2^-10 of max |dO|; an inf or NaN sets OPR_DEV_FP16_RANGE).
__device__ __forceinline__ bool fp16_range_ok(float x) { return fabsf(x) <= 65504.f; }

// One block of 256 threads per (tile, head); each warp walks 16 of the tile's
// tokens, one token row per step with the whole warp (lane l holds elements
// [l D/32, (l+1) D/32) of the row), so every access is a full coalesced row.
template <int D, typename OT>
__global__ void __launch_bounds__(256) row_terms_kernel(const OT* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                                        const float* __restrict__ lse, const int32_t* __restrict__ cu_seqlens,
                                                        const int32_t* __restrict__ stream_of,
                                                        int64_t total, int32_t hq, int32_t T, float* __restrict__ d_tiles,
                                                        float* __restrict__ lse2_tiles, __half* __restrict__ dout16,
                                                        const uint32_t* __restrict__ absmax,
                                                        int32_t* __restrict__ dev_status) {
  constexpr int kE = D / 32;  // elements per lane: 4 (D = 128) or 2 (D = 64)
  const int tile = blockIdx.x, h = blockIdx.y;
  const float gs = pow2f(grad_scale_exp(*absmax));  // 2^k
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = tile / T, J = tile % T;
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  if constexpr (kDebugChecks) {  // the sequence must lie inside the token range
    if (seq0 < 0 || L < 0 || seq0 + L > total) {
      if (threadIdx.x == 0) atomicOr(dev_status, OPR_DEV_BOUNDS);
      return;
    }
  }
  bool in_range = true;
  for (int i = 0; i < kTile / 8; ++i) {
    const int c = warp * (kTile / 8) + i;
    const size_t out = (static_cast<size_t>(h) * gridDim.x + tile) * kTile + c;
    if (J * kTile + c >= L) {
      if (lane == 0) {
        d_tiles[out] = 0.f;
        lse2_tiles[out] = -INFINITY;
      }
      continue;
    }
    const int64_t tok = seq0 + J * kTile + c;  // attention position: tiles and the dO copy
    const int64_t src = stream_of[tok];         // stream row: O, dO and LSE
    if (src < 0 || src >= total) {
      if (lane == 0) {
        d_tiles[out] = 0.f;
        lse2_tiles[out] = -INFINITY;
      }
      continue;
    }
    const size_t base = (static_cast<size_t>(tok) * hq + h) * D + lane * kE;
    const size_t sbase = (static_cast<size_t>(src) * hq + h) * D + lane * kE;
    float df[kE], ov[kE];
    if constexpr (kE == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(dout + sbase);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&u);
      df[0] = __low2float(d2[0]) * gs; df[1] = __high2float(d2[0]) * gs;
      df[2] = __low2float(d2[1]) * gs; df[3] = __high2float(d2[1]) * gs;
      *reinterpret_cast<uint2*>(dout16 + base) = make_uint2(pack_f16x2(df[0], df[1]), pack_f16x2(df[2], df[3]));
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(dout + sbase);
      const __nv_bfloat162 d2 = *reinterpret_cast<const __nv_bfloat162*>(&u);
      df[0] = __low2float(d2) * gs; df[1] = __high2float(d2) * gs;
      *reinterpret_cast<uint32_t*>(dout16 + base) = pack_f16x2(df[0], df[1]);
    }
    if constexpr (sizeof(OT) == 4) {
      if constexpr (kE == 4) {
        const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(o) + sbase);
        ov[0] = f.x; ov[1] = f.y; ov[2] = f.z; ov[3] = f.w;
      } else {
        const float2 f = *reinterpret_cast<const float2*>(static_cast<const float*>(o) + sbase);
        ov[0] = f.x; ov[1] = f.y;
      }
    } else if constexpr (kE == 4) {  // four bf16 values in one 8-byte load
      const uint2 u = *reinterpret_cast<const uint2*>(o + sbase);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&u);
      ov[0] = __low2float(o2[0]); ov[1] = __high2float(o2[0]); ov[2] = __low2float(o2[1]); ov[3] = __high2float(o2[1]);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(o + sbase);
      const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162*>(&u);
      ov[0] = __low2float(o2); ov[1] = __high2float(o2);
    }
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < kE; ++k) {
      acc = fmaf(ov[k], df[k], acc);
      in_range &= fp16_range_ok(df[k]);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) {
      d_tiles[out] = -acc;
      lse2_tiles[out] = -lse[static_cast<size_t>(h) * total + src] * kLog2e;
    }
  }
  if (!in_range) atomicOr(dev_status, OPR_DEV_FP16_RANGE);
}

// fp16 copy of V for the dkdv kernel, eight values per thread (same range rule).
// Row t of y (attention order) is row stream_of[t] of x (stream order); a row
// holds row8 groups of eight values.
__global__ void __launch_bounds__(256) cast_f16_kernel(const __nv_bfloat16* __restrict__ x, __half* __restrict__ y,
                                                       int64_t n8, int64_t row8, int64_t total,
                                                       const int32_t* __restrict__ stream_of,
                                                       int32_t* __restrict__ dev_status) {
  bool in_range = true;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t src_row = stream_of[i / row8];
    if (src_row < 0 || src_row >= total) {
      reinterpret_cast<uint4*>(y)[i] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4 u = reinterpret_cast<const uint4*>(x)[src_row * row8 + i % row8];
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    float f[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __low2float(b2[k]);
      f[2 * k + 1] = __high2float(b2[k]);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) in_range &= fp16_range_ok(f[k]);
    reinterpret_cast<uint4*>(y)[i] =
        make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]), pack_f16x2(f[4], f[5]), pack_f16x2(f[6], f[7]));
  }
  if (!in_range) atomicOr(dev_status, OPR_DEV_FP16_RANGE);
}

// ----------------------------------------------------------------------------
template <int D>
struct DqSmem {
  alignas(1024) uint8_t q[TileGeom<D>::kBytes];
  alignas(1024) uint8_t dout[TileGeom<D>::kBytes];
  alignas(1024) uint8_t k[kStages][TileGeom<D>::kBytes];
  alignas(1024) uint8_t v[kStages][TileGeom<D>::kBytes];
  alignas(16) TileMeta kmeta[kStages];  // key metadata of a partial tile, rides with its K tile
  int32_t list[kListSmem];
  uint64_t bar_qdo;
  uint64_t bar_kfull[kStages], bar_kempty[kStages], bar_vfull[kStages], bar_vempty[kStages];
  uint64_t bar_sfull, bar_sfree, bar_dpfull, bar_dsfull, bar_dqdone, bar_final;
  uint32_t tmem_base;
  int abort_flag;
};

// TMEM columns of the dq kernel: S at 0, dP at 128, dQ accumulator at 256,
// dS (16-bit, 64 columns) at 384.
constexpr uint32_t kDqColS = 0, kDqColDP = 128, kDqColAcc = 256, kDqColDS = 384;

template <int D, bool QK16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const AttnParams p) {
  constexpr uint32_t kTileBytes = TileGeom<D>::kBytes;
  extern __shared__ uint8_t smem_raw[];
  DqSmem<D>& sm = *reinterpret_cast<DqSmem<D>*>(align1024(smem_raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // head-major grid: the CTAs that run together share one kv head's K/V tiles in L2
  const int head = blockIdx.x / p.n_items;
  const int tile_id = p.sched[blockIdx.x % p.n_items];
  if (head >= p.hq) return;
  if (!debug_tile_ok(p, tile_id, p.row_cnt, p.row_list)) return;
  const int n = p.row_cnt[tile_id];
  if (n == 0) return;
  const int s = tile_id / p.T, I = tile_id % p.T;
  const int32_t* list = p.row_list + static_cast<size_t>(tile_id) * p.T;
  const int seq0 = p.cu_seqlens[s];
  const int seq_len = p.cu_seqlens[s + 1] - seq0;
  const int q0 = seq0 + I * kTile;
  const int kvh = head / (p.hq / p.hkv);

  for (int x = threadIdx.x; x < n && x < kListSmem; x += blockDim.x) sm.list[x] = list[x];
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_qdo, 1);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&sm.bar_kfull[st], 1);
      mbar_init(&sm.bar_kempty[st], 1);
      mbar_init(&sm.bar_vfull[st], 1);
      mbar_init(&sm.bar_vempty[st], 1);
    }
    mbar_init(&sm.bar_sfull, 1);
    mbar_init(&sm.bar_sfree, kComputeThreads);
    mbar_init(&sm.bar_dpfull, 1);
    mbar_init(&sm.bar_dsfull, kComputeThreads);
    mbar_init(&sm.bar_dqdone, 1);
    mbar_init(&sm.bar_final, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  const int32_t* lst = sm.list;
  auto entry = [&](int j) { return j < kListSmem ? lst[j] : list[j]; };

  if (warp == 0) {
    // lane 0: Q and dO once, then the K ring (+ key metadata of partial tiles); lane 1: the V ring
    if (lane == 0) {
      const TileMeta* tmeta = p.tile_meta + static_cast<size_t>(s) * p.T;
      mbar_arrive_expect_tx(&sm.bar_qdo, 2 * kTileBytes);
      tma_tile<D>(&tm_q, &sm.bar_qdo, sm.q, head, q0);
      tma_tile<D>(&tm_do, &sm.bar_qdo, sm.dout, head, q0);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        const int e = entry(j);
        const int J = entry_index(e);
        if (j >= kStages && !mbar_wait(&sm.bar_kempty[st], ((j / kStages) + 1) & 1, abort_flag, p.wait_ns))
          break;
        const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
        mbar_arrive_expect_tx(&sm.bar_kfull[st], kTileBytes + (partial ? sizeof(TileMeta) : 0));
        tma_tile<D>(&tm_k, &sm.bar_kfull[st], sm.k[st], kvh, seq0 + J * kTile);
        if (partial) bulk_load(&sm.kmeta[st], tmeta + J, sizeof(TileMeta), &sm.bar_kfull[st]);
        issued = j + 1;
      }
      // every copy issued has landed before the CTA exits (also after an abort, when
      // no consumer waited for the last ones)
      mbar_wait(&sm.bar_qdo, 0, nullptr, kWaitLimitNs);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait(&sm.bar_kfull[j % kStages], (j / kStages) & 1, nullptr, kWaitLimitNs);
    } else if (lane == 1) {
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&sm.bar_vempty[st], ((j / kStages) + 1) & 1, abort_flag, p.wait_ns))
          break;
        mbar_arrive_expect_tx(&sm.bar_vfull[st], kTileBytes);
        tma_tile<D>(&tm_v, &sm.bar_vfull[st], sm.v[st], kvh, seq0 + entry_index(entry(j)) * kTile);
        issued = j + 1;
      }
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait(&sm.bar_vfull[j % kStages], (j / kStages) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // the whole warp runs this loop; elect.sync picks the issuing lane
    // On a partial tile of which no query sees one 64-key half, S and dP are the
    // N = 64 products over the other half (in that half's columns) and dQ takes
    // its 64 keys only.
    constexpr uint32_t idesc_s = idesc_f32acc(128, 128, QK16, 0, 0);   // S = Q K^T (q/k type)
    constexpr uint32_t idesc_s64 = idesc_f32acc(128, 64, QK16, 0, 0);  // S over one key half
    constexpr uint32_t idesc_p = idesc_f32acc(128, 128, true, 0, 0);   // dP = 2^k dO V^T (fp16 copies)
    constexpr uint32_t idesc_p64 = idesc_f32acc(128, 64, true, 0, 0);  // dP over one key half
    constexpr uint32_t idesc_q = idesc_f32acc(128, D, QK16, 0, 1);     // dQ += dS K (K tile MN-major)
    const uint32_t sq = smem_u32(sm.q), sdo = smem_u32(sm.dout);
    // S(j) = Q K(j)^T
    auto issue_s = [&](int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_kfull[st], (j / kStages) & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const int hv = entry_halves(entry(j));
      const uint32_t k0 = hv == 2 ? kKeyHalf : 0;  // first key of the product
      const uint64_t kb = desc_kmajor(smem_u32(sm.k[st]) + k0 * 128, 0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + kDqColS + k0, (desc_kmajor(sq, 0) + kmajor_step(kk)), kb + kmajor_step(kk),
               hv == 3 ? idesc_s : idesc_s64, kk > 0 ? 1u : 0u);
      mma_commit(&sm.bar_sfull);
      return true;
    };
    // dP(j) = dO V(j)^T; releases V(j)
    auto issue_dp = [&](int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_vfull[st], (j / kStages) & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const int hv = entry_halves(entry(j));
      const uint32_t k0 = hv == 2 ? kKeyHalf : 0;
      const uint64_t vb = desc_kmajor(smem_u32(sm.v[st]) + k0 * 128, 0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + kDqColDP + k0, (desc_kmajor(sdo, 0) + kmajor_step(kk)), vb + kmajor_step(kk),
               hv == 3 ? idesc_p : idesc_p64, kk > 0 ? 1u : 0u);
      mma_commit(&sm.bar_dpfull);
      mma_commit(&sm.bar_vempty[st]);
      return true;
    };
    // dQ += dS(j) K(j); releases K(j) and its metadata
    auto issue_dq = [&](int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_dsfull, j & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const int hv = entry_halves(entry(j));
      const uint64_t kb = desc_mnmajor(smem_u32(sm.k[st]), 0);
      uint32_t acc = j > 0 ? 1u : 0u;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (!((hv >> half) & 1)) continue;  // no query of the tile sees these 64 keys
#pragma unroll
        for (int kk = 4 * half; kk < 4 * half + 4; ++kk) {
          mma_ts(tmem + kDqColAcc, tmem + kDqColDS + kk * 8, kb + mnmajor_step(kk), idesc_q, acc);
          acc = 1u;
        }
      }
      mma_commit(&sm.bar_kempty[st]);
      return true;
    };
    // Issue order S(0) dP(0) | S(1) dQ(0) dP(1) | S(2) dQ(1) dP(2) | ...: S(j+1) starts as
    // soon as the compute warps have read S(j), while they still form P(j) and dS(j).
    bool ok = warp_wait(&sm.bar_qdo, 0, abort_flag, p.wait_ns) && issue_s(0) && issue_dp(0);
    for (int j = 0; ok && j < n; ++j) {
      if (j + 1 < n) {
        ok = warp_wait(&sm.bar_sfree, j & 1, abort_flag, p.wait_ns) && issue_s(j + 1);
        if (!ok) break;
      }
      ok = issue_dq(j);
      if (ok && j + 1 < n) ok = issue_dp(j + 1);
    }
    if (ok) mma_commit(&sm.bar_dqdone);
    mma_commit(&sm.bar_final);
    __all_sync(0xffffffffu, mbar_wait(&sm.bar_final, 0, nullptr, kWaitLimitNs));
  } else {
    // two threads per query row: `half` selects key columns [64 half, 64 half + 64)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const bool qv = I * kTile + row < seq_len;
    const int qg = q0 + row;
    const int qconv = qv ? p.conv_idx[qg] : -2;
    const int qmeta = qv ? p.tok_meta[qg] : 0;
    const size_t rt = (static_cast<size_t>(head) * p.n_items + tile_id) * kTile + row;
    const float nlse2 = qv ? p.lse2_tiles[rt] : 0.f;  // -LSE * log2(e)
    const float nd = qv ? p.d_tiles[rt] : 0.f;        // -2^k D
    const int gk = grad_scale_exp(*p.dout_absmax);
    // dP comes from the fp16 copy of 2^k dO, so dS is formed as 2^k P (dP - D)
    const uint64_t sl2x2 = f2(p.scale_log2, p.scale_log2), nlse2x2 = f2(nlse2, nlse2), ndx2 = f2(nd, nd);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int st = j % kStages;
      const int e = entry(j);
      const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
      const int kbase = seq0 + entry_index(e) * kTile;
      if (!((entry_halves(e) >> half) & 1)) {
        // no query of the tile sees this thread's 64 keys: nothing to form, only the
        // hand-offs (each wait orders this thread's arrival after the phase before)
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull, j & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        mbar_arrive(&sm.bar_sfree);
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dpfull, j & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        mbar_arrive(&sm.bar_dsfull);
        continue;
      }
      if (partial &&
          !__all_sync(0xffffffffu, mbar_wait(&sm.bar_kfull[st], (j / kStages) & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      // visibility of this thread's 64 key columns (all set on full tiles)
      uint32_t mm[2] = {0xffffffffu, 0xffffffffu};
      if (partial) {
        uint32_t m[4];
        query_row_mask(sm.kmeta[st], kbase, qg, qconv, qmeta, m);
        mm[0] = half ? m[2] : m[0];
        mm[1] = half ? m[3] : m[1];
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull, j & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float pv[64];
      {
        uint32_t sr[64];
        tmem_ld64(tl + kDqColS + half * 64, sr);
        tc_fence_before();
        mbar_arrive(&sm.bar_sfree);  // S may be overwritten by the next Q K^T
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float a0, a1;
          f2_split(ffma2(f2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, nlse2x2), a0, a1);
          pv[c] = fast_exp2(a0);
          pv[c + 1] = fast_exp2(a1);
        }
      }
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (!((mm[c >> 5] >> (c & 31)) & 1u)) pv[c] = 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dpfull, j & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t r[64];
        tmem_ld64(tl + kDqColDP + half * 64, r);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const uint64_t t = fadd2(f2(__uint_as_float(r[c * 32 + 2 * x]), __uint_as_float(r[c * 32 + 2 * x + 1])), ndx2);
            float d0, d1;
            f2_split(fmul2(f2(pv[c * 32 + 2 * x], pv[c * 32 + 2 * x + 1]), t), d0, d1);
            pk[x] = pack_x2<QK16>(d0, d1);
          }
          tmem_st16(tl + kDqColDS + half * 32 + c * 16, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_dsfull);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&sm.bar_dqdone, 0, abort_flag, p.wait_ns))) {
      tc_fence_after();
      const int srow = qv ? p.stream_of[qg] : -1;  // stream row of this query's dQ
      const bool qw = srow >= 0 && srow < p.total;
      float* dst = p.dq + (static_cast<size_t>(qw ? srow : 0) * p.hq + head) * D;
      const float osc = p.scale * pow2f(-gk);  // undoes the gradient scale 2^k
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        const int oc = half * (D / 2) + c * 32;
        tmem_ld32(tl + kDqColAcc + oc, r);
        if (qw) {
          float4* d4 = reinterpret_cast<float4*>(dst + oc);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = make_float4(__uint_as_float(r[4 * x]) * osc, __uint_as_float(r[4 * x + 1]) * osc,
                                __uint_as_float(r[4 * x + 2]) * osc, __uint_as_float(r[4 * x + 3]) * osc);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sm.abort_flag) atomicOr(p.dev_status, OPR_DEV_WAIT_TIMEOUT);
}

// ----------------------------------------------------------------------------
template <int D>
struct DkdvSmem {
  alignas(1024) uint8_t k[TileGeom<D>::kBytes];
  alignas(1024) uint8_t v[TileGeom<D>::kBytes];              // fp16 copy of V
  alignas(1024) uint8_t q[kStages][TileGeom<D>::kBytes];
  alignas(1024) uint8_t dout[kStages][TileGeom<D>::kBytes];  // fp16 copy of dO
  // column data of a query tile, bulk-copied with its Q tile: LSE * log2(e), D and
  // (for partial tiles) the query metadata
  alignas(16) float qlse2[kStages][kTile];
  alignas(16) float qd[kStages][kTile];
  alignas(16) TileMeta qmeta[kStages];
  int32_t list[kListSmem];
  uint64_t bar_kv;
  uint64_t bar_qfull[kStages], bar_qempty[kStages], bar_dofull[kStages], bar_doempty[kStages];
  uint64_t bar_sfull, bar_dpfull;
  uint64_t bar_pfull[2], bar_dsfull[2];  // one per query half
  uint64_t bar_accdone, bar_final;
  uint32_t tmem_base;
  int abort_flag;
};

// TMEM columns of the dkdv kernel: S^T at 0..127 and dP^T at 128..255 (one
// column per query of the tile), dV accumulator at 256, dK at 256 + D.  The
// compute warps of query half h (columns 64h..64h+63 of each region) write
// the packed fp16 P^T and dS^T of their half over the first 32 of those
// columns, which the dV and dK products read as their A operand.
constexpr uint32_t kKvColS = 0, kKvColDP = 128, kKvColDV = 256;

template <int D, bool QK16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v16, const __grid_constant__ CUtensorMap tm_do16,
                         const AttnParams p) {
  constexpr uint32_t kTileBytes = TileGeom<D>::kBytes;
  constexpr uint32_t kColDK = kKvColDV + D;
  extern __shared__ uint8_t smem_raw[];
  DkdvSmem<D>& sm = *reinterpret_cast<DkdvSmem<D>*>(align1024(smem_raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // kv-head-major grid over a schedule grouped by sequence: the CTAs that run
  // together stream the Q and dO tiles of one kv head group and sequence,
  // which stay in L2.  In split mode (p.dkdv_split) the grid's major index is the
  // q head: a long column (split_col) is walked for that head only, a short one by
  // the group's first head for the whole group, as in the unsplit grid.
  const int group = p.hq / p.hkv;
  const int major = blockIdx.x / p.n_items;
  const int tile_id = p.sched[blockIdx.x % p.n_items];
  if (major >= (p.dkdv_split ? p.hq : p.hkv)) return;
  const int kvh = p.dkdv_split ? major / group : major;
  if (!debug_tile_ok(p, tile_id, p.col_cnt, p.col_list)) return;
  const int cnt = p.col_cnt[tile_id];
  if (cnt == 0) return;
  const bool split_col = p.dkdv_split && cnt >= p.split_min_cnt;
  if (p.dkdv_split && !split_col && major % group != 0) return;
  const int n = split_col ? cnt : cnt * group;
  // Iteration j covers query tile entry(tile_of(j)) of q head head_of(j): a whole
  // column walks its query tiles in order and, for each, the group's q heads in
  // turn.  Against the heads-outermost walk this takes fewer SM cycles (fewer
  // long-scoreboard stalls) at the cost of more L2 misses on Q and dO, which at
  // this kernel's DRAM rate cost no bandwidth.
  auto head_of = [&](int j) { return split_col ? major : kvh * group + j % group; };
  auto tile_of = [&](int j) { return split_col ? j : j / group; };
  const int s = tile_id / p.T, J = tile_id % p.T;
  const int32_t* list = p.col_list + static_cast<size_t>(tile_id) * p.T;
  const int seq0 = p.cu_seqlens[s];
  const int seq_len = p.cu_seqlens[s + 1] - seq0;
  const int k0 = seq0 + J * kTile;

  for (int x = threadIdx.x; x < cnt && x < kListSmem; x += blockDim.x) sm.list[x] = list[x];
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_kv, 1);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&sm.bar_qfull[st], 1);
      mbar_init(&sm.bar_qempty[st], 1);
      mbar_init(&sm.bar_dofull[st], 1);
      mbar_init(&sm.bar_doempty[st], 1);
    }
    mbar_init(&sm.bar_sfull, 1);
    mbar_init(&sm.bar_dpfull, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sm.bar_pfull[h], kComputeThreads / 2);
      mbar_init(&sm.bar_dsfull[h], kComputeThreads / 2);
    }
    mbar_init(&sm.bar_accdone, 1);
    mbar_init(&sm.bar_final, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  const int32_t* lst = sm.list;
  auto entry = [&](int j) { return j < kListSmem ? lst[j] : list[j]; };

  if (warp == 0) {
    // lane 0: K and V once, then the Q ring with each query tile's column data;
    // lane 1: the dO ring.  Iteration j covers q head head_of(j) and query tile
    // entry(tile_of(j)).
    if (lane == 0) {
      const TileMeta* tmeta = p.tile_meta + static_cast<size_t>(s) * p.T;
      mbar_arrive_expect_tx(&sm.bar_kv, 2 * kTileBytes);
      tma_tile<D>(&tm_k, &sm.bar_kv, sm.k, kvh, k0);
      tma_tile<D>(&tm_v16, &sm.bar_kv, sm.v, kvh, k0);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        const int e = entry(tile_of(j));
        const int Iq = entry_index(e);
        const int h = head_of(j);
        if (j >= kStages && !mbar_wait(&sm.bar_qempty[st], ((j / kStages) + 1) & 1, abort_flag, p.wait_ns))
          break;
        const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
        mbar_arrive_expect_tx(&sm.bar_qfull[st],
                              kTileBytes + 2 * kTile * sizeof(float) + (partial ? sizeof(TileMeta) : 0));
        tma_tile<D>(&tm_q, &sm.bar_qfull[st], sm.q[st], h, seq0 + Iq * kTile);
        const size_t rt = (static_cast<size_t>(h) * p.n_items + s * p.T + Iq) * kTile;
        bulk_load(sm.qlse2[st], p.lse2_tiles + rt, kTile * sizeof(float), &sm.bar_qfull[st]);
        bulk_load(sm.qd[st], p.d_tiles + rt, kTile * sizeof(float), &sm.bar_qfull[st]);
        if (partial) bulk_load(&sm.qmeta[st], tmeta + Iq, sizeof(TileMeta), &sm.bar_qfull[st]);
        issued = j + 1;
      }
      // every copy issued has landed before the CTA exits (also after an abort, when
      // no consumer waited for the last ones)
      mbar_wait(&sm.bar_kv, 0, nullptr, kWaitLimitNs);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait(&sm.bar_qfull[j % kStages], (j / kStages) & 1, nullptr, kWaitLimitNs);
    } else if (lane == 1) {
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        const int h = head_of(j);
        if (j >= kStages && !mbar_wait(&sm.bar_doempty[st], ((j / kStages) + 1) & 1, abort_flag, p.wait_ns))
          break;
        mbar_arrive_expect_tx(&sm.bar_dofull[st], kTileBytes);
        tma_tile<D>(&tm_do16, &sm.bar_dofull[st], sm.dout[st], h, seq0 + entry_index(entry(tile_of(j))) * kTile);
        issued = j + 1;
      }
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait(&sm.bar_dofull[j % kStages], (j / kStages) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // the whole warp runs this loop; elect.sync picks the issuing lane
    constexpr uint32_t idesc_s = idesc_f32acc(128, 128, QK16, 0, 0);  // S^T = K Q^T (q/k type)
    constexpr uint32_t idesc_p = idesc_f32acc(128, 128, true, 0, 0);  // dP^T = V dO^T (fp16)
    constexpr uint32_t idesc_v = idesc_f32acc(128, D, true, 0, 1);    // dV += P_h^T dO_h (fp16)
    constexpr uint32_t idesc_k = idesc_f32acc(128, D, QK16, 0, 1);    // dK += dS_h^T Q_h (q/k type)
    const uint64_t dk_base = desc_kmajor(smem_u32(sm.k), 0), dv_base = desc_kmajor(smem_u32(sm.v), 0);
    // S^T(j) = K Q(j)^T.  Full 128-query products: both operands come from shared
    // memory, whose bandwidth a narrower N would spend faster than the tensor core.
    auto issue_s = [&](int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_qfull[st], (j / kStages) & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const uint64_t qb = desc_kmajor(smem_u32(sm.q[st]), 0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + kKvColS, dk_base + kmajor_step(kk), qb + kmajor_step(kk), idesc_s, kk > 0 ? 1u : 0u);
      mma_commit(&sm.bar_sfull);
      return true;
    };
    // dP^T(j) = V dO(j)^T
    auto issue_dp = [&](int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_dofull[st], (j / kStages) & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const uint64_t ob = desc_kmajor(smem_u32(sm.dout[st]), 0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + kKvColDP, dv_base + kmajor_step(kk), ob + kmajor_step(kk), idesc_p, kk > 0 ? 1u : 0u);
      mma_commit(&sm.bar_dpfull);
      return true;
    };
    // dV += P^T(j)[:, half h] dO(j)[half h]; the second half releases dO(j)
    auto issue_dv = [&](int h, int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_pfull[h], j & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const uint64_t ob = desc_mnmajor(smem_u32(sm.dout[st]), 4 * h);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tmem + kKvColDV, tmem + kKvColS + 64 * h + kk * 8, ob + mnmajor_step(kk), idesc_v,
               (j > 0 || h > 0 || kk > 0) ? 1u : 0u);
      if (h == 1) mma_commit(&sm.bar_doempty[st]);
      return true;
    };
    // dK += dS^T(j)[:, half h] Q(j)[half h]; the second half releases Q(j) and its column data
    auto issue_dk = [&](int h, int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(&sm.bar_dsfull[h], j & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const uint64_t qb = desc_mnmajor(smem_u32(sm.q[st]), 4 * h);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tmem + kColDK, tmem + kKvColDP + 64 * h + kk * 8, qb + mnmajor_step(kk), idesc_k,
               (j > 0 || h > 0 || kk > 0) ? 1u : 0u);
      if (h == 1) mma_commit(&sm.bar_qempty[st]);
      return true;
    };
    // Issue order S(0) dP(0) | dV_0(j) dV_1(j) S(j+1) dK_0(j) dK_1(j) dP(j+1) | ...:
    // the next S^T is formed while the compute warps turn dP^T into dS^T, and
    // the next dP^T while they turn S^T into P^T; each half's dV (dK) product
    // starts as soon as that half's P^T (dS^T) is in place.
    bool ok = warp_wait(&sm.bar_kv, 0, abort_flag, p.wait_ns) && issue_s(0) && issue_dp(0);
    for (int j = 0; ok && j < n; ++j) {
      const bool more = j + 1 < n;
      ok = issue_dv(0, j) && issue_dv(1, j);
      if (ok && more) ok = issue_s(j + 1);
      if (ok) ok = issue_dk(0, j) && issue_dk(1, j);
      if (ok && more) ok = issue_dp(j + 1);
    }
    if (ok) mma_commit(&sm.bar_accdone);
    mma_commit(&sm.bar_final);
    __all_sync(0xffffffffu, mbar_wait(&sm.bar_final, 0, nullptr, kWaitLimitNs));
  } else {
    // query half `half`: warps 2..5 own query columns 0..63, warps 6..9 columns
    // 64..127; one key row per thread
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t cs = kKvColS + 64 * half, cdp = kKvColDP + 64 * half;
    const bool kvld = J * kTile + row < seq_len;
    const int kg = k0 + row;
    const int kconv = kvld ? p.conv_idx[kg] : -1;
    const int kmeta = kvld ? p.tok_meta[kg] : 0;
    const uint64_t sl2x2 = f2(p.scale_log2, p.scale_log2);
    const int c0 = half * 64;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int st = j % kStages;
      const int e = entry(tile_of(j));
      const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
      const int qt0 = seq0 + entry_index(e) * kTile;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_qfull[st], (j / kStages) & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      // visibility of this stream's 64 query columns (all set on full tiles)
      uint32_t mm[2] = {0xffffffffu, 0xffffffffu};
      if (partial) {
        uint32_t m[4];
        key_row_mask(sm.qmeta[st], qt0, kg, kconv, kmeta, m);
        mm[0] = half ? m[2] : m[0];
        mm[1] = half ? m[3] : m[1];
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull, j & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // P^T as fp16, two query columns per TMEM column, over this half's own S^T
      // columns; the packed values also serve the dS step below
      uint32_t pp[32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sr[32];
        tmem_ld32(tl + cs + cc * 32, sr);
        const float4* l4 = reinterpret_cast<const float4*>(&sm.qlse2[st][c0 + cc * 32]);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 l = l4[x];  // -LSE * log2(e) of four query columns
          const int c = cc * 32 + 4 * x;
          float a0, a1, a2, a3;
          f2_split(ffma2(f2(__uint_as_float(sr[4 * x]), __uint_as_float(sr[4 * x + 1])), sl2x2, f2(l.x, l.y)), a0, a1);
          f2_split(ffma2(f2(__uint_as_float(sr[4 * x + 2]), __uint_as_float(sr[4 * x + 3])), sl2x2, f2(l.z, l.w)), a2,
                   a3);
          float p0 = fast_exp2(a0);
          float p1 = fast_exp2(a1);
          float p2 = fast_exp2(a2);
          float p3 = fast_exp2(a3);
          if (partial) {
            const uint32_t b = mm[c >> 5] >> (c & 31);
            p0 = (b & 1u) ? p0 : 0.f;
            p1 = (b & 2u) ? p1 : 0.f;
            p2 = (b & 4u) ? p2 : 0.f;
            p3 = (b & 8u) ? p3 : 0.f;
          }
          pp[cc * 16 + 2 * x] = pack_f16x2(p0, p1);
          pp[cc * 16 + 2 * x + 1] = pack_f16x2(p2, p3);
        }
      }
      tmem_st16(tl + cs, reinterpret_cast<const uint32_t(&)[16]>(pp[0]));
      tmem_st16(tl + cs + 16, reinterpret_cast<const uint32_t(&)[16]>(pp[16]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_pfull[half]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dpfull, j & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // dS^T = P^T (dP^T - D) in the q/k type, over this half's own dP^T columns
      {
        const float4* d4 = reinterpret_cast<const float4*>(&sm.qd[st][c0]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(tl + cdp + c * 32, r);
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 nd = d4[c * 8 + x];  // -D of four query columns
            const float2 pa = __half22float2(*reinterpret_cast<const __half2*>(&pp[c * 16 + 2 * x]));
            const float2 pb = __half22float2(*reinterpret_cast<const __half2*>(&pp[c * 16 + 2 * x + 1]));
            float d0, d1, d2, d3;
            f2_split(fmul2(f2(pa.x, pa.y), fadd2(f2(__uint_as_float(r[4 * x]), __uint_as_float(r[4 * x + 1])),
                                                 f2(nd.x, nd.y))),
                     d0, d1);
            f2_split(fmul2(f2(pb.x, pb.y), fadd2(f2(__uint_as_float(r[4 * x + 2]), __uint_as_float(r[4 * x + 3])),
                                                 f2(nd.z, nd.w))),
                     d2, d3);
            pk[2 * x] = pack_x2<QK16>(d0, d1);
            pk[2 * x + 1] = pack_x2<QK16>(d2, d3);
          }
          tmem_st16(tl + cdp + c * 16, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_dsfull[half]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&sm.bar_accdone, 0, abort_flag, p.wait_ns))) {
      tc_fence_after();
      // partials at the attention position, final rows at the stream row
      const int srow = kvld ? p.stream_of[kg] : -1;
      const bool kw = kvld && (split_col || (srow >= 0 && srow < p.total));
      const size_t fin = static_cast<size_t>(srow >= 0 && srow < p.total ? srow : 0);
      float* dvp = split_col ? p.dv_part + (static_cast<size_t>(major) * p.total + kg) * D
                             : p.dv + (fin * p.hkv + kvh) * D;
      float* dkp = split_col ? p.dk_part + (static_cast<size_t>(major) * p.total + kg) * D
                             : p.dk + (fin * p.hkv + kvh) * D;
      const float vsc = pow2f(-grad_scale_exp(*p.dout_absmax));  // undoes the gradient scale 2^k
      const float ksc = p.scale * vsc;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        const int oc = half * (D / 2) + c * 32;
        tmem_ld32(tl + kKvColDV + oc, r);
        if (kw) {
          float4* d4 = reinterpret_cast<float4*>(dvp + oc);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = make_float4(__uint_as_float(r[4 * x]) * vsc, __uint_as_float(r[4 * x + 1]) * vsc,
                                __uint_as_float(r[4 * x + 2]) * vsc, __uint_as_float(r[4 * x + 3]) * vsc);
        }
      }
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        const int oc = half * (D / 2) + c * 32;
        tmem_ld32(tl + kColDK + oc, r);
        if (kw) {
          float4* d4 = reinterpret_cast<float4*>(dkp + oc);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = make_float4(__uint_as_float(r[4 * x]) * ksc, __uint_as_float(r[4 * x + 1]) * ksc,
                                __uint_as_float(r[4 * x + 2]) * ksc, __uint_as_float(r[4 * x + 3]) * ksc);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sm.abort_flag) atomicOr(p.dev_status, OPR_DEV_WAIT_TIMEOUT);
}

// dK, dV [total][hkv][D] (stream rows) of the tokens of split key columns (at
// least min_cnt query tiles) = the sum over the q heads of each GQA group of the
// per-head partials [hq][total][D] (attention positions) the split dK/dV kernel
// wrote (head order kvh * group + 0, 1, ...; one float4 of dK and of dV per
// thread and step).  The tokens of shorter columns were written whole by the
// dK/dV kernel and are left alone.
template <int D>
__global__ void __launch_bounds__(256) gqa_sum_kernel(const float* __restrict__ dk_part,
                                                      const float* __restrict__ dv_part, int64_t total, int32_t hq,
                                                      int32_t hkv, const int32_t* __restrict__ cu_seqlens,
                                                      const int32_t* __restrict__ stream_of,
                                                      int32_t n_seqs, int32_t T, const int32_t* __restrict__ col_cnt,
                                                      int32_t min_cnt, float* __restrict__ dk, float* __restrict__ dv) {
  const int group = hq / hkv;
  const int64_t n4 = total * hkv * (D / 4);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c4 = static_cast<int>(i % (D / 4));
    const int64_t tk = i / (D / 4);  // token * hkv + kv head
    const int kvh = static_cast<int>(tk % hkv);
    const int64_t tok = tk / hkv;
    int lo = 0, hi = n_seqs - 1;  // sequence of tok: the last s with cu_seqlens[s] <= tok
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cu_seqlens[mid] <= tok) lo = mid; else hi = mid - 1;
    }
    const int J = static_cast<int>((tok - cu_seqlens[lo]) / kTile);
    if (J < 0 || J >= T || col_cnt[lo * T + J] < min_cnt) continue;
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
    for (int g = 0; g < group; ++g) {
      const size_t src = ((static_cast<size_t>(kvh) * group + g) * total + tok) * (D / 4) + c4;
      const float4 a = reinterpret_cast<const float4*>(dk_part)[src];
      const float4 b = reinterpret_cast<const float4*>(dv_part)[src];
      sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
      sv.x += b.x; sv.y += b.y; sv.z += b.z; sv.w += b.w;
    }
    const int64_t srow = stream_of[tok];
    if (srow < 0 || srow >= total) continue;
    const int64_t o = (srow * hkv + kvh) * (D / 4) + c4;  // stream row of the attention position tok
    reinterpret_cast<float4*>(dk)[o] = sk;
    reinterpret_cast<float4*>(dv)[o] = sv;
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t smem, int* configured) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && configured[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess && dev < 64) configured[dev] = 1;
  return e;
}

template <int D, bool QK16>
cudaError_t launch_bwd_t(const BwdMaps& m, const BwdBuffers& b, const AttnParams& pq, const AttnParams& pkv,
                         int stages, cudaStream_t stream) {
  static int conf_dq[64] = {0}, conf_kv[64] = {0};
  cudaError_t e = cudaSuccess;
  // 1) row terms D and LSE * log2(e) per 128-token tile, and the fp16 copies of dO and V
  if ((stages & OPR_BWD_ROW_TERMS) && pq.n_items > 0) {
    if ((e = cudaMemsetAsync(b.dout_absmax, 0, sizeof(uint32_t), stream)) != cudaSuccess) return e;
    const int64_t n8_do = pq.total * pq.hq * D / 8;
    if (n8_do > 0) {
      const int64_t blocks = std::min<int64_t>((n8_do + 255) / 256, 148 * 8);
      dout_absmax_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(b.dout, n8_do, b.dout_absmax);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const dim3 grid(pq.n_items, pq.hq);
    float* row_d = b.row_terms;
    float* row_l = b.row_terms + static_cast<size_t>(pq.hq) * pq.n_items * kTile;
    if (b.o_fp32)
      row_terms_kernel<D, float><<<grid, 256, 0, stream>>>(static_cast<const float*>(b.o), b.dout, pq.lse_in,
                                                               pq.cu_seqlens, pq.stream_of, pq.total, pq.hq, pq.T,
                                                               row_d, row_l, b.dout16, b.dout_absmax, pq.dev_status);
    else
      row_terms_kernel<D, __nv_bfloat16><<<grid, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(b.o), b.dout, pq.lse_in, pq.cu_seqlens, pq.stream_of, pq.total, pq.hq,
          pq.T, row_d, row_l, b.dout16, b.dout_absmax, pq.dev_status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t n8 = pq.total * pq.hkv * D / 8;
    if (n8 > 0) {
      const int64_t blocks = std::min<int64_t>((n8 + 255) / 256, 148 * 16);
      cast_f16_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(b.v, b.v16, n8, pq.hkv * D / 8, pq.total,
                                                                         pq.stream_of, pq.dev_status);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  // 2) dQ
  if (stages & OPR_BWD_DQ) {
    const size_t smem_q = smem_request(sizeof(DqSmem<D>) + 1024);
    if ((e = set_smem(attn_bwd_dq_kernel<D, QK16>, smem_q, conf_dq)) != cudaSuccess) return e;
    const int64_t bq = static_cast<int64_t>(pq.n_items) * pq.hq;
    if (bq > 0)
      attn_bwd_dq_kernel<D, QK16><<<static_cast<unsigned>(bq), kThreads, smem_q, stream>>>(m.q, m.k, m.v16, m.dout16,
                                                                                          pq);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (b.rope_pos != nullptr &&  // dq w.r.t. the unrotated q: one pass over the rows
        (e = launch_rope(pq.dq, OPR_DTYPE_FP32, pq.dq, OPR_DTYPE_FP32, b.rope_pos, nullptr, pq.total, pq.hq, D, b.rope_base, 1,
                         pq.dev_status, stream)) != cudaSuccess)
      return e;
  }
  // 3) dK, dV
  if (stages & OPR_BWD_DKDV) {
    const size_t smem_kv = smem_request(sizeof(DkdvSmem<D>) + 1024);
    if ((e = set_smem(attn_bwd_dkdv_kernel<D, QK16>, smem_kv, conf_kv)) != cudaSuccess) return e;
    const int64_t bkv = static_cast<int64_t>(pkv.n_items) * (pkv.dkdv_split ? pkv.hq : pkv.hkv);
    if (bkv > 0)
      attn_bwd_dkdv_kernel<D, QK16>
          <<<static_cast<unsigned>(bkv), kThreads, smem_kv, stream>>>(m.q, m.k, m.v16, m.dout16, pkv);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (pkv.dkdv_split) {  // sum each GQA group's per-head partials, in head order
      const int64_t n4 = pkv.total * pkv.hkv * (D / 4);
      if (n4 > 0) {
        const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, 148 * 16);
        gqa_sum_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            pkv.dk_part, pkv.dv_part, pkv.total, pkv.hq, pkv.hkv, pkv.cu_seqlens, pkv.stream_of, pkv.n_items / pkv.T,
            pkv.T,
            pkv.col_cnt, pkv.split_min_cnt, pkv.dk, pkv.dv);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
      }
    }
    if (b.rope_pos != nullptr)  // dk w.r.t. the unrotated k
      e = launch_rope(pkv.dk, OPR_DTYPE_FP32, pkv.dk, OPR_DTYPE_FP32, b.rope_pos, nullptr, pkv.total, pkv.hkv, D, b.rope_base, 1,
                      pkv.dev_status, stream);
  }
  return e;
}

}  // namespace

cudaError_t launch_attn_bwd(int head_dim, bool qk_f16, const BwdMaps& m, const BwdBuffers& b, const AttnParams& pq,
                            const AttnParams& pkv, int stages, cudaStream_t stream) {
  if (!qk_f16) return cudaErrorNotSupported;  // the entry points accept fp16 q and k only
  if (head_dim == 128) return launch_bwd_t<128, true>(m, b, pq, pkv, stages, stream);
  return launch_bwd_t<64, true>(m, b, pq, pkv, stages, stream);
}

}  // namespace opr
