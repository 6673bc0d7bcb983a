// attn_fwd.cu - block-sparse masked attention forward for sm_100a.
//
// One-Pass to Reason, "分块稀疏注意力掩码": attention restricted by the per-type
// visibility rules, evaluated block-sparsely (the pages use a FlexAttention
// block mask on H100, "实现细节"; this is a hand-written Blackwell kernel).
//
// One CTA per (query tile of 128 rows, q head), 10 warps:
//   warp 0      lane 0 loads Q once, then the K tiles of the row's non-empty
//               tiles (3-stage ring) with TMA, plus, for partial tiles, the
//               tile's precomputed key metadata (one bulk copy); lane 1
//               loads the V tiles (2-stage ring);
//   warp 1      allocates TMEM and issues tcgen05.mma: S = Q K^T into one of
//               two TMEM buffers, then O += P V with P read from TMEM;
//   warps 2..9  two threads per query row, each owning 64 of the tile's 128
//               key columns: read S from TMEM, apply the visibility mask on
//               partial tiles only, online softmax in base 2 (the row max is
//               taken over all 128 columns by both threads, so no exchange is
//               needed), write their half of P (V's type) to TMEM, rescale
//               their half of O in TMEM only when the running max grows by
//               more than 2^8; epilogue O / l and the log-sum-exp.
// TMEM columns: S buffer 0 at 0, buffer 1 at 128, O at 256, P buffers at 384
// and 448 (512 allocated).
// Q and K may be bf16 or fp16 (QK16: the rotated q, k stored in fp16, whose
// 11-bit significand keeps the rounding of the rotation 8x smaller).  V and P
// share one 16-bit type: fp16 (V16; P keeps 11 bits, so O, and the backward's
// D = rowsum(dO * O), are about 8x closer to exact) or bf16.
#include "attn_common.cuh"

namespace opr {
namespace {

constexpr int kStagesK = 3, kStagesV = 2;
constexpr int kListSmem = 1024;  // entries of the row's tile list kept in shared memory
constexpr uint32_t kOCol = 256;
constexpr uint32_t kPCol = 384;  // P buffers (bf16, 64 columns each): never alias S, which both
                                 // threads of a row read for the row max

template <int D>
struct FwdSmem {
  alignas(1024) uint8_t q[TileGeom<D>::kBytes];
  alignas(1024) uint8_t k[kStagesK][TileGeom<D>::kBytes];
  alignas(1024) uint8_t v[kStagesV][TileGeom<D>::kBytes];
  alignas(16) TileMeta kmeta[kStagesK];  // key metadata of a partial tile, rides with its K tile
  int32_t list[kListSmem];
  float lsum[2][kTile];  // row-sum halves, combined in the epilogue
  uint64_t bar_q;
  uint64_t bar_kfull[kStagesK], bar_kempty[kStagesK], bar_vfull[kStagesV], bar_vempty[kStagesV];
  uint64_t bar_sfull[2], bar_pfull[2], bar_odone, bar_final;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool QK16, bool V16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr uint32_t kTileBytes = TileGeom<D>::kBytes;
  extern __shared__ uint8_t smem_raw[];
  FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(align1024(smem_raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // head-major grid: the CTAs that run together share one kv head's K/V tiles in L2
  const int head = blockIdx.x / p.n_items;
  const int tile_id = p.sched[blockIdx.x % p.n_items];
  if (head >= p.hq) return;
  if (!debug_tile_ok(p, tile_id, p.row_cnt, p.row_list)) return;
  const int n = p.row_cnt[tile_id];
  if (n == 0) return;  // tile past the end of its sequence
  const int s = tile_id / p.T, I = tile_id % p.T;
  const int32_t* list = p.row_list + static_cast<size_t>(tile_id) * p.T;
  const int seq0 = p.cu_seqlens[s];
  const int seq_len = p.cu_seqlens[s + 1] - seq0;
  const int q0 = seq0 + I * kTile;
  const int kvh = head / (p.hq / p.hkv);

  for (int x = threadIdx.x; x < n && x < kListSmem; x += blockDim.x) sm.list[x] = list[x];
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int st = 0; st < kStagesK; ++st) {
      mbar_init(&sm.bar_kfull[st], 1);
      // released when S = Q K^T has completed and every compute thread has read the metadata
      mbar_init(&sm.bar_kempty[st], 1 + kComputeThreads);
    }
    for (int st = 0; st < kStagesV; ++st) {
      mbar_init(&sm.bar_vfull[st], 1);
      mbar_init(&sm.bar_vempty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.bar_sfull[b], 1);
      mbar_init(&sm.bar_pfull[b], kComputeThreads);
    }
    mbar_init(&sm.bar_odone, 1);
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
  const TileMeta* tmeta = p.tile_meta + static_cast<size_t>(s) * p.T;

  if (warp == 0) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(&sm.bar_q, kTileBytes);
      tma_tile<D>(&tm_q, &sm.bar_q, sm.q, head, q0);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStagesK;
        const int e = entry(j);
        const int J = entry_index(e);
        if (j >= kStagesK && !mbar_wait(&sm.bar_kempty[st], ((j / kStagesK) + 1) & 1, abort_flag, p.wait_ns))
          break;
        const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
        mbar_arrive_expect_tx(&sm.bar_kfull[st], kTileBytes + (partial ? sizeof(TileMeta) : 0));
        tma_tile<D>(&tm_k, &sm.bar_kfull[st], sm.k[st], kvh, seq0 + J * kTile);
        if (partial) bulk_load(&sm.kmeta[st], tmeta + J, sizeof(TileMeta), &sm.bar_kfull[st]);
        issued = j + 1;
      }
      // every copy issued has landed before the CTA exits (also after an abort, when
      // no consumer waited for the last ones)
      mbar_wait(&sm.bar_q, 0, nullptr, kWaitLimitNs);
      for (int j = (issued > kStagesK ? issued - kStagesK : 0); j < issued; ++j)
        mbar_wait(&sm.bar_kfull[j % kStagesK], (j / kStagesK) & 1, nullptr, kWaitLimitNs);
    } else if (lane == 1) {
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStagesV;
        if (j >= kStagesV && !mbar_wait(&sm.bar_vempty[st], ((j / kStagesV) + 1) & 1, abort_flag, p.wait_ns))
          break;
        mbar_arrive_expect_tx(&sm.bar_vfull[st], kTileBytes);
        tma_tile<D>(&tm_v, &sm.bar_vfull[st], sm.v[st], kvh, seq0 + entry_index(entry(j)) * kTile);
        issued = j + 1;
      }
      for (int j = (issued > kStagesV ? issued - kStagesV : 0); j < issued; ++j)
        mbar_wait(&sm.bar_vfull[j % kStagesV], (j / kStagesV) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // the whole warp runs this loop; elect.sync picks the issuing lane
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_f32acc(128, 128, QK16, 0, 0);  // S = Q K^T in the q/k type
    constexpr uint32_t idesc_o = idesc_f32acc(128, D, V16, 0, 1);  // O += P V, P and V fp16 (V16) or bf16
    const uint32_t sq = smem_u32(sm.q);
    bool ok = warp_wait(&sm.bar_q, 0, abort_flag, p.wait_ns);
    auto issue_pv = [&](int jp) -> bool {
      const int bp = jp & 1, stp = jp % kStagesV;
      if (!warp_wait(&sm.bar_pfull[bp], (jp >> 1) & 1, abort_flag, p.wait_ns)) return false;
      if (!warp_wait(&sm.bar_vfull[stp], (jp / kStagesV) & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const uint32_t sv = smem_u32(sm.v[stp]);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_ts(tmem + kOCol, tmem + kPCol + bp * 64 + kk * 8, (desc_mnmajor(sv, 0) + mnmajor_step(kk)), idesc_o,
               (jp > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&sm.bar_vempty[stp]);
      mma_commit(&sm.bar_odone);
      return true;
    };
    for (int j = 0; ok && j < n; ++j) {
      const int st = j % kStagesK, b = j & 1;
      if (!warp_wait(&sm.bar_kfull[st], (j / kStagesK) & 1, abort_flag, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sk = smem_u32(sm.k[st]);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + b * 128, (desc_kmajor(sq, 0) + kmajor_step(kk)), (desc_kmajor(sk, 0) + kmajor_step(kk)), idesc_s, kk > 0 ? 1u : 0u);
      mma_commit(&sm.bar_sfull[b]);
      mma_commit(&sm.bar_kempty[st]);
      if (j >= 1 && !issue_pv(j - 1)) ok = false;
    }
    if (ok) issue_pv(n - 1);
    // All MMAs issued by this thread must be complete before TMEM is freed.
    mma_commit(&sm.bar_final);
    __all_sync(0xffffffffu, mbar_wait(&sm.bar_final, 0, nullptr, kWaitLimitNs));
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;  // key columns [64 half, 64 half + 64)
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const bool qv = I * kTile + row < seq_len;
    const int qg = q0 + row;
    const int qconv = qv ? p.conv_idx[qg] : -2;
    const int qmeta = qv ? p.tok_meta[qg] : 0;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;  // l_run: this thread's half of the row sum
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int b = j & 1, st = j % kStagesK;
      const int e = entry(j);
      const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
      const int kbase = seq0 + entry_index(e) * kTile;
      // the K stage carries the tile's key metadata; it is released after this read
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_kfull[st], (j / kStagesK) & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      // visibility: own 64 columns in words 0..1, the partner's in 2..3 (all set on full tiles)
      uint32_t mm[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (partial) {
        uint32_t m[4];
        query_row_mask(sm.kmeta[st], kbase, qg, qconv, qmeta, m);
        mm[0] = half ? m[2] : m[0];
        mm[1] = half ? m[3] : m[1];
        mm[2] = half ? m[0] : m[2];
        mm[3] = half ? m[1] : m[3];
      }
      mbar_arrive(&sm.bar_kempty[st]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull[b], (j >> 1) & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // own 64 columns in sv[0..63], the partner thread's 64 in sv[64..127] (max only)
      float sv[kTile];
      {
        uint32_t sr[kTile];
        const uint32_t own = tl + b * 128 + half * 64, oth = tl + b * 128 + (half ^ 1) * 64;
        tmem_ld32x4(own, own + 32, oth, oth + 32, sr);
#pragma unroll
        for (int c = 0; c < kTile; ++c) sv[c] = __uint_as_float(sr[c]);
      }
      if (partial) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (!mask_bit(mm, c)) sv[c] = -INFINITY;
      }
      // row max over all 128 columns (8 independent chains)
      float mx8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) mx8[x] = sv[x];
#pragma unroll
      for (int c = 8; c < kTile; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool need = m_new > m_run + 8.f;  // also true on the first finite max
      const float m_use = need ? m_new : m_run;
      const float mb = (m_use == -INFINITY) ? 0.f : m_use;
      // this thread's 64 columns of P, packed two per TMEM column over S
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float p0 = fast_exp2(fmaf(sv[c * 32 + 2 * x], sl2, -mb));
          const float p1 = fast_exp2(fmaf(sv[c * 32 + 2 * x + 1], sl2, -mb));
          rs8[x & 7] += p0 + p1;
          pk[x] = pack_x2<V16>(p0, p1);
        }
        tmem_st16(tl + kPCol + b * 64 + half * 32 + c * 16, pk);
      }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      tmem_wait_st();
      // O may be rescaled only once the previous P V product has landed.
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_odone, (j - 1) & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      const float factor = need ? fast_exp2(m_run - m_new) : 1.f;
      if (__any_sync(0xffffffffu, need && j >= 1)) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t r[32];
          const uint32_t oc = kOCol + half * (D / 2) + c * 32;
          tmem_ld32(tl + oc, r);
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * factor);
          tmem_st32(tl + oc, r);
        }
        tmem_wait_st();
      }
      l_run = l_run * factor + rs;
      if (need) m_run = m_new;
      tc_fence_before();
      mbar_arrive(&sm.bar_pfull[b]);
    }
    // ------------------------------------------------------------ epilogue
    // Every compute thread reaches this barrier exactly once (also after an abort).
    sm.lsum[half][row] = l_run;
    named_bar_sync(1, kComputeThreads);
    if (ok && __all_sync(0xffffffffu, mbar_wait(&sm.bar_odone, (n - 1) & 1, abort_flag, p.wait_ns))) {
      tc_fence_after();
      const float l_tot = sm.lsum[0][row] + sm.lsum[1][row];
      const float inv = 1.f / l_tot;
      const int srow = qv ? p.stream_of[qg] : -1;  // stream row of this query's O and LSE
      const bool qw = srow >= 0 && srow < p.total;
      const size_t orow = (static_cast<size_t>(qw ? srow : 0) * p.hq + head) * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        const int oc = half * (D / 2) + c * 32;
        tmem_ld32(tl + kOCol + oc, r);
        if (qw) {
          if (p.o_fp32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + oc);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              dst[x] = make_float4(__uint_as_float(r[4 * x]) * inv, __uint_as_float(r[4 * x + 1]) * inv,
                                   __uint_as_float(r[4 * x + 2]) * inv, __uint_as_float(r[4 * x + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + orow + oc);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * x]) * inv, __uint_as_float(r[8 * x + 1]) * inv),
                                  pack_bf16x2(__uint_as_float(r[8 * x + 2]) * inv, __uint_as_float(r[8 * x + 3]) * inv),
                                  pack_bf16x2(__uint_as_float(r[8 * x + 4]) * inv, __uint_as_float(r[8 * x + 5]) * inv),
                                  pack_bf16x2(__uint_as_float(r[8 * x + 6]) * inv, __uint_as_float(r[8 * x + 7]) * inv));
          }
        }
      }
      if (qw && half == 0)
        p.lse[static_cast<size_t>(head) * p.total + srow] = (m_run + __log2f(l_tot)) * 0.69314718055994531f;
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
// Pieces of one thread's row of a tile in the head-pair kernel, for the NC keys
// (128, or the 64 of the one key half that some query of the tile sees) that it
// processes.

// Row max of NC scores (NC a multiple of 16, at least 32): eight chains, each
// over columns x, x + 8, x + 16, ..., mostly with the three-input max.
template <int NC>
__device__ __forceinline__ float row_max(const float (&sv)[NC]) {
  constexpr int W = 8;
  static_assert(NC % (2 * W) == 0 && NC >= 4 * W, "whole blocks of 16 columns");
  constexpr int kPairs = (NC - 3 * W) / (2 * W);  // blocks of 8 taken two at a time
  float mx[W];
#pragma unroll
  for (int x = 0; x < W; ++x) mx[x] = fmax3(sv[x], sv[W + x], sv[2 * W + x]);
#pragma unroll
  for (int b = 0; b < kPairs; ++b)
#pragma unroll
    for (int x = 0; x < W; ++x) mx[x] = fmax3(mx[x], sv[3 * W + 2 * W * b + x], sv[4 * W + 2 * W * b + x]);
#pragma unroll
  for (int x = 0; x < W; ++x) mx[x] = fmaxf(mx[x], sv[NC - W + x]);  // the last block of 8
  return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// P = 2^(S scale log2(e) - mb) of NC scores (the scale-and-shift on fp32 pairs),
// stored two per TMEM column from p_addr, in the type of V (fp16 when V16, else
// bf16); returns the sum of the unrounded P.  One pair
// in kFmaExpEvery takes the FMA-pipe exponential, the others the special-function
// unit, so that the two pipes share the softmax's exponentials.
constexpr int kFmaExpEvery = 3;

template <int NC, bool V16>
__device__ __forceinline__ float exp_pack_row(const float (&sv)[NC], float sl2, float mb, uint32_t p_addr) {
  const uint64_t sl2x2 = f2(sl2, sl2), nmb2 = f2(-mb, -mb);
  float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const uint64_t a2 = ffma2(f2(sv[c * 32 + 2 * x], sv[c * 32 + 2 * x + 1]), sl2x2, nmb2);
      float p0, p1;
      if (x % kFmaExpEvery == kFmaExpEvery - 1) {  // resolved at compile time (unrolled loop)
        f2_split(exp2_fma2(a2), p0, p1);
      } else {
        float a0, a1;
        f2_split(a2, a0, a1);
        p0 = fast_exp2(a0);
        p1 = fast_exp2(a1);
      }
      rs8[x & 7] += p0 + p1;
      pk[x] = pack_x2<V16>(p0, p1);
    }
    tmem_st16(p_addr + c * 16, pk);
  }
  return ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
}

// Running-max decision of a row after a tile whose masked row max is mx (scaled
// to base 2 by sl2): P is taken against the old max unless the max grew by more
// than 8 (a factor of 256), in which case O is rescaled to the new one.
struct MaxStep {
  float m_new;  // running max after the tile
  bool need;    // rescale O and the row sum to m_new
  float mb;     // the max P is taken against (0 while the row has seen nothing)
};
__device__ __forceinline__ MaxStep max_step(float m_run, float mx, float sl2) {
  MaxStep r;
  r.m_new = fmaxf(m_run, mx * sl2);
  r.need = r.m_new > m_run + 8.f;  // also true on the first finite max
  const float m_use = r.need ? r.m_new : m_run;
  r.mb = (m_use == -INFINITY) ? 0.f : m_use;
  return r;
}

// ----------------------------------------------------------------------------
// Head-pair forward: one CTA per (query tile, two q heads of one GQA group).
// Both heads read the same K/V tiles and the same mask, so the two heads are
// two independent softmax streams on one K/V pipeline: while the tensor core
// forms head B's S (or P V) the compute warps of head A work, and vice versa.
//   warp 0      lane 0: both Q tiles, then the K ring (+ key metadata of
//               partial tiles); lane 1: the V ring
//   warp 1      TMEM owner, MMA issuer: S_A(0) S_B(0) | P_A V, S_A(j+1),
//               P_B V, S_B(j+1) | ...
//   warps 2..5  head A, warps 6..9 head B: one query row per thread, P (V's type)
//               written over the first 64 columns of the thread's own row of S
// TMEM columns: S_A 0, S_B 128, O_A 256, O_B 384.
// Full 128x128 products on every non-empty tile: the kernel is bound by its
// softmax, not by the tensor core, and the 64-key half products measured slower
// here (the dQ kernel uses them).
template <int D>
struct FwdPairSmem {
  alignas(1024) uint8_t q[2][TileGeom<D>::kBytes];
  alignas(1024) uint8_t k[kStagesV][TileGeom<D>::kBytes];
  alignas(1024) uint8_t v[kStagesV][TileGeom<D>::kBytes];
  alignas(16) TileMeta kmeta[kStagesV];
  int32_t list[kListSmem];
  uint64_t bar_q;
  uint64_t bar_kfull[kStagesV], bar_kempty[kStagesV], bar_vfull[kStagesV], bar_vempty[kStagesV];
  uint64_t bar_sfull[2], bar_pfull[2], bar_odone[2], bar_final;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool QK16, bool V16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int NS = kStagesV;  // K and V rings share a depth here (two Q tiles resident)
  constexpr uint32_t kTileBytes = TileGeom<D>::kBytes;
  extern __shared__ uint8_t smem_raw[];
  FwdPairSmem<D>& sm = *reinterpret_cast<FwdPairSmem<D>*>(align1024(smem_raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pair-major grid: the CTAs that run together share one kv head's K/V tiles in L2
  const int pair = blockIdx.x / p.n_items;
  const int tile_id = p.sched[blockIdx.x % p.n_items];
  if (pair >= p.hq / 2) return;
  if (!debug_tile_ok(p, tile_id, p.row_cnt, p.row_list)) return;
  const int n = p.row_cnt[tile_id];
  if (n == 0) return;
  const int s = tile_id / p.T, I = tile_id % p.T;
  const int32_t* list = p.row_list + static_cast<size_t>(tile_id) * p.T;
  const int seq0 = p.cu_seqlens[s];
  const int seq_len = p.cu_seqlens[s + 1] - seq0;
  const int q0 = seq0 + I * kTile;
  const int head0 = 2 * pair;
  const int kvh = head0 / (p.hq / p.hkv);  // both heads of the pair share it (even group size)

  for (int x = threadIdx.x; x < n && x < kListSmem; x += blockDim.x) sm.list[x] = list[x];
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int st = 0; st < NS; ++st) {
      mbar_init(&sm.bar_kfull[st], 1);
      // released when both S = Q K^T have completed and every compute thread has read the metadata
      mbar_init(&sm.bar_kempty[st], 1 + kComputeThreads);
      mbar_init(&sm.bar_vfull[st], 1);
      mbar_init(&sm.bar_vempty[st], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sm.bar_sfull[h], 1);
      mbar_init(&sm.bar_pfull[h], 128);
      mbar_init(&sm.bar_odone[h], 1);
    }
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
    if (lane == 0) {
      const TileMeta* tmeta = p.tile_meta + static_cast<size_t>(s) * p.T;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(&sm.bar_q, 2 * kTileBytes);
      tma_tile<D>(&tm_q, &sm.bar_q, sm.q[0], head0, q0);
      tma_tile<D>(&tm_q, &sm.bar_q, sm.q[1], head0 + 1, q0);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % NS;
        const int e = entry(j);
        const int J = entry_index(e);
        if (j >= NS && !mbar_wait(&sm.bar_kempty[st], ((j / NS) + 1) & 1, abort_flag, p.wait_ns)) break;
        const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
        mbar_arrive_expect_tx(&sm.bar_kfull[st], kTileBytes + (partial ? sizeof(TileMeta) : 0));
        tma_tile<D>(&tm_k, &sm.bar_kfull[st], sm.k[st], kvh, seq0 + J * kTile);
        if (partial) bulk_load(&sm.kmeta[st], tmeta + J, sizeof(TileMeta), &sm.bar_kfull[st]);
        issued = j + 1;
      }
      // every copy issued has landed before the CTA exits (also after an abort, when
      // no consumer waited for the last ones)
      mbar_wait(&sm.bar_q, 0, nullptr, kWaitLimitNs);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_wait(&sm.bar_kfull[j % NS], (j / NS) & 1, nullptr, kWaitLimitNs);
    } else if (lane == 1) {
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % NS;
        if (j >= NS && !mbar_wait(&sm.bar_vempty[st], ((j / NS) + 1) & 1, abort_flag, p.wait_ns)) break;
        mbar_arrive_expect_tx(&sm.bar_vfull[st], kTileBytes);
        tma_tile<D>(&tm_v, &sm.bar_vfull[st], sm.v[st], kvh, seq0 + entry_index(entry(j)) * kTile);
        issued = j + 1;
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_wait(&sm.bar_vfull[j % NS], (j / NS) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // the whole warp runs this loop; elect.sync picks the issuing lane
    constexpr uint32_t idesc_s = idesc_f32acc(128, 128, QK16, 0, 0);  // S = Q K^T in the q/k type
    constexpr uint32_t idesc_o = idesc_f32acc(128, D, V16, 0, 1);    // O += P V, P and V fp16 (V16) or bf16
    const uint32_t sq[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
    auto issue_s = [&](int h, int j) {
      const uint32_t sk = smem_u32(sm.k[j % NS]);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + h * 128, (desc_kmajor(sq[h], 0) + kmajor_step(kk)), (desc_kmajor(sk, 0) + kmajor_step(kk)), idesc_s, kk > 0 ? 1u : 0u);
      mma_commit(&sm.bar_sfull[h]);
    };
    auto issue_pv = [&](int h, int j) -> bool {
      if (!warp_wait(&sm.bar_pfull[h], j & 1, abort_flag, p.wait_ns)) return false;
      tc_fence_after();
      const uint32_t sv = smem_u32(sm.v[j % NS]);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_ts(tmem + 256 + h * 128, tmem + h * 128 + kk * 8, (desc_mnmajor(sv, 0) + mnmajor_step(kk)), idesc_o,
               (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&sm.bar_odone[h]);
      return true;
    };
    bool ok = warp_wait(&sm.bar_q, 0, abort_flag, p.wait_ns) &&
              warp_wait(&sm.bar_kfull[0], 0, abort_flag, p.wait_ns);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      issue_s(1, 0);
      mma_commit(&sm.bar_kempty[0]);
    }
    for (int j = 0; ok && j < n; ++j) {
      const bool more = j + 1 < n;
      if (!warp_wait(&sm.bar_vfull[j % NS], (j / NS) & 1, abort_flag, p.wait_ns)) {
        ok = false;
        break;
      }
      if (!(ok = issue_pv(0, j))) break;
      if (more) {
        if (!warp_wait(&sm.bar_kfull[(j + 1) % NS], ((j + 1) / NS) & 1, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(0, j + 1);
      }
      if (!(ok = issue_pv(1, j))) break;
      mma_commit(&sm.bar_vempty[j % NS]);
      if (more) {
        issue_s(1, j + 1);
        mma_commit(&sm.bar_kempty[(j + 1) % NS]);
      }
    }
    mma_commit(&sm.bar_final);
    __all_sync(0xffffffffu, mbar_wait(&sm.bar_final, 0, nullptr, kWaitLimitNs));
  } else {
    const int hx = (warp - 2) >> 2;  // 0: head A (warps 2..5), 1: head B (warps 6..9)
    const int head = head0 + hx;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t scol = hx * 128, ocol = 256 + hx * 128;
    const bool qv = I * kTile + row < seq_len;
    const int qg = q0 + row;
    const int qconv = qv ? p.conv_idx[qg] : -2;
    const int qmeta = qv ? p.tok_meta[qg] : 0;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int st = j % NS;
      const int e = entry(j);
      const bool partial = entry_class(e) == OPR_TILE_PARTIAL;
      const int kbase = seq0 + entry_index(e) * kTile;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_kfull[st], (j / NS) & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      uint32_t mm[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (partial)
        query_row_mask(sm.kmeta[st], kbase, qg, qconv, qmeta, mm);
      mbar_arrive(&sm.bar_kempty[st]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull[hx], j & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kTile];
      {
        uint32_t sr[kTile];
        tmem_ld128(tl + scol, sr);
#pragma unroll
        for (int c = 0; c < kTile; ++c) sv[c] = __uint_as_float(sr[c]);
      }
      if (partial) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (!mask_bit(mm, c)) sv[c] = -INFINITY;
      }
      const MaxStep ms = max_step(m_run, row_max<kTile>(sv), sl2);
      const float rs = exp_pack_row<kTile, V16>(sv, sl2, ms.mb, tl + scol);  // P over S's read columns
      tmem_wait_st();
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_odone[hx], (j - 1) & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      const float factor = ms.need ? fast_exp2(m_run - ms.m_new) : 1.f;
      if (__any_sync(0xffffffffu, ms.need && j >= 1)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tl + ocol + c * 32, r);
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * factor);
          tmem_st32(tl + ocol + c * 32, r);
        }
        tmem_wait_st();
      }
      l_run = l_run * factor + rs;
      if (ms.need) m_run = ms.m_new;
      tc_fence_before();
      mbar_arrive(&sm.bar_pfull[hx]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&sm.bar_odone[hx], (n - 1) & 1, abort_flag, p.wait_ns))) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      const int srow = qv ? p.stream_of[qg] : -1;  // stream row of this query's O and LSE
      const bool qw = srow >= 0 && srow < p.total;
      const size_t orow = (static_cast<size_t>(qw ? srow : 0) * p.hq + head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tl + ocol + c * 32, r);
        if (qw) {
          if (p.o_fp32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              dst[x] = make_float4(__uint_as_float(r[4 * x]) * inv, __uint_as_float(r[4 * x + 1]) * inv,
                                   __uint_as_float(r[4 * x + 2]) * inv, __uint_as_float(r[4 * x + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + orow + c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * x]) * inv, __uint_as_float(r[8 * x + 1]) * inv),
                                  pack_bf16x2(__uint_as_float(r[8 * x + 2]) * inv, __uint_as_float(r[8 * x + 3]) * inv),
                                  pack_bf16x2(__uint_as_float(r[8 * x + 4]) * inv, __uint_as_float(r[8 * x + 5]) * inv),
                                  pack_bf16x2(__uint_as_float(r[8 * x + 6]) * inv, __uint_as_float(r[8 * x + 7]) * inv));
          }
        }
      }
      if (qw) p.lse[static_cast<size_t>(head) * p.total + srow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
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

}  // namespace

template <int D, bool QK16, bool V16>
cudaError_t launch_attn_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const AttnParams& p, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  const bool pairs = (p.hq / p.hkv) % 2 == 0;
  const size_t smem_single = smem_request(sizeof(FwdSmem<D>) + 1024);
  const size_t smem_pair = smem_request(sizeof(FwdPairSmem<D>) + 1024);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, QK16, V16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_single));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_fwd_pair_kernel<D, QK16, V16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_pair));
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  if (pairs) {
    // two q heads of one GQA group per CTA
    const int64_t blocks = static_cast<int64_t>(p.n_items) * (p.hq / 2);
    if (blocks == 0) return cudaSuccess;
    attn_fwd_pair_kernel<D, QK16, V16><<<static_cast<unsigned>(blocks), kThreads, smem_pair, stream>>>(tq, tk, tv, p);
  } else {
    const int64_t blocks = static_cast<int64_t>(p.n_items) * p.hq;
    if (blocks == 0) return cudaSuccess;
    attn_fwd_kernel<D, QK16, V16><<<static_cast<unsigned>(blocks), kThreads, smem_single, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd(int head_dim, bool qk_f16, bool v_f16, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const AttnParams& p, cudaStream_t stream) {
  if (!qk_f16) return cudaErrorNotSupported;  // the entry points accept fp16 q and k only
  if (head_dim == 128)
    return v_f16 ? launch_attn_fwd_t<128, true, true>(tq, tk, tv, p, stream)
                 : launch_attn_fwd_t<128, true, false>(tq, tk, tv, p, stream);
  return v_f16 ? launch_attn_fwd_t<64, true, true>(tq, tk, tv, p, stream)
               : launch_attn_fwd_t<64, true, false>(tq, tk, tv, p, stream);
}

}  // namespace opr
