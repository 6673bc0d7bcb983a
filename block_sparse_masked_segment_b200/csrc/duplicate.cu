// duplicate.cu - the step before the attention layer: token duplication.
//
// One-Pass to Reason wiki note, "Token 复制": each response r_i is stored
// twice, as r_i^in (the context copy) and r_i^out (the copy that is trained
// on), so the one-pass stream of a turn is h_i t_i r_i^in r_i^out while the
// original stream holds h_i t_i r_i once.  Conversations follow each other in
// index order in both streams.
//
//   dup_index_kernel   the map between the streams: src_index[i] = original
//                      token of one-pass token i; copy_index[o] = the one-pass
//                      positions of original token o (second = -1 for h, t);
//   gather_rows_kernel one-pass rows as copies of original rows (token ids,
//                      embeddings or any fixed-width row);
//   fold_rows_kernel   the gradient of that copy: each original row sums its
//                      copies' rows in slot order, in fp32.  A gather over
//                      copy_index, so no atomics and the sum order is fixed;
//   kpass_*            the K-pass arrangement and its token map (below).
#include <cuda_runtime.h>

#include "opr_internal.cuh"

namespace opr {
namespace {

constexpr int kDupThreads = 1024;

// Single block.  Turns are taken kDupThreads at a time: one thread per turn
// loads (h, t, r), a block scan turns them into the turns' offsets in both
// streams, then the whole block writes the indices of those turns' tokens.
// Every write is bounds-checked against the sizes the caller gave; a total
// that disagrees with the lengths sets OPR_DEV_TOTAL_MISMATCH.
__global__ void __launch_bounds__(kDupThreads) dup_index_kernel(const int32_t* __restrict__ turn_lens,
                                                                 const int32_t* __restrict__ conv_turn_ptr,
                                                                 int32_t n_convs, int32_t n_turns, int64_t total,
                                                                 int64_t orig_total, int32_t* __restrict__ src_index,
                                                                 int32_t* __restrict__ copy_index,
                                                                 int32_t* __restrict__ dev_status) {
  __shared__ int64_t one_off[kDupThreads], orig_off[kDupThreads];
  __shared__ int32_t lens[kDupThreads][3];
  __shared__ int64_t warp_one[32], warp_orig[32];
  __shared__ int64_t carry_one, carry_orig;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry_one = 0;
    carry_orig = 0;
    if (conv_turn_ptr[0] != 0 || conv_turn_ptr[n_convs] != n_turns) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
  }
  __syncthreads();
  bool bad = false;
  for (int base = 0; base < n_turns; base += kDupThreads) {
    const int t = base + tid;
    int h = 0, tt = 0, r = 0;
    if (t < n_turns) {
      h = turn_lens[3 * t];
      tt = turn_lens[3 * t + 1];
      r = turn_lens[3 * t + 2];
      if (h < 0 || tt < 0 || r < 0) bad = true;
      h = max(h, 0);
      tt = max(tt, 0);
      r = max(r, 0);
    }
    lens[tid][0] = h;
    lens[tid][1] = tt;
    lens[tid][2] = r;
    // inclusive warp scans of both streams' token counts, then across warps
    int64_t a = static_cast<int64_t>(h) + tt + 2 * static_cast<int64_t>(r);
    int64_t b = static_cast<int64_t>(h) + tt + r;
    int64_t ia = a, ib = b;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int64_t ya = __shfl_up_sync(0xffffffffu, ia, d), yb = __shfl_up_sync(0xffffffffu, ib, d);
      if (lane >= d) {
        ia += ya;
        ib += yb;
      }
    }
    if (lane == 31) {
      warp_one[warp] = ia;
      warp_orig[warp] = ib;
    }
    __syncthreads();
    if (warp == 0) {
      const int64_t wa = warp_one[lane], wb = warp_orig[lane];
      int64_t xa = wa, xb = wb;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int64_t ya = __shfl_up_sync(0xffffffffu, xa, d), yb = __shfl_up_sync(0xffffffffu, xb, d);
        if (lane >= d) {
          xa += ya;
          xb += yb;
        }
      }
      warp_one[lane] = xa - wa;  // exclusive warp offsets
      warp_orig[lane] = xb - wb;
    }
    __syncthreads();
    const int64_t c1 = carry_one, c2 = carry_orig;
    one_off[tid] = c1 + warp_one[warp] + ia - a;
    orig_off[tid] = c2 + warp_orig[warp] + ib - b;
    __syncthreads();
    if (tid == kDupThreads - 1) {
      carry_one = c1 + warp_one[warp] + ia;
      carry_orig = c2 + warp_orig[warp] + ib;
    }
    // the tokens of this chunk's turns, one turn after another, the block across each turn
    const int nt = min(kDupThreads, n_turns - base);
    for (int u = 0; u < nt; ++u) {
      const int hu = lens[u][0], tu = lens[u][1], ru = lens[u][2];
      const int64_t o1 = one_off[u], o2 = orig_off[u];
      const int n = hu + tu + 2 * ru;
      for (int x = tid; x < n; x += kDupThreads) {
        const int64_t i = o1 + x;
        const int xo = x < hu + tu + ru ? x : x - ru;  // r^out copies r^in's originals
        const int64_t o = o2 + xo;
        if (i < total && o < orig_total) src_index[i] = static_cast<int32_t>(o);
        if (x < hu + tu + ru && o < orig_total) {
          const bool is_r = x >= hu + tu;
          const int64_t second = is_r ? i + ru : -1;
          copy_index[2 * o] = i < total ? static_cast<int32_t>(i) : -1;
          copy_index[2 * o + 1] = (is_r && second < total) ? static_cast<int32_t>(second) : -1;
        }
      }
    }
    __syncthreads();
  }
  if (bad) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
  if (tid == 0 && (carry_one != total || carry_orig != orig_total)) atomicOr(dev_status, OPR_DEV_TOTAL_MISMATCH);
}

// y[i] = x[src_index[i]], rows of row_units units of type U (16, 4 or 1 bytes).
// Wide rows: one warp per row, lanes across the row (coalesced); narrow rows
// (fewer than 32 units): one thread per row.
template <typename U>
__global__ void __launch_bounds__(256) gather_rows_kernel(const U* __restrict__ x, int64_t orig_total,
                                                          int64_t row_units, const int32_t* __restrict__ src_index,
                                                          int64_t total, U* __restrict__ y,
                                                          int32_t* __restrict__ dev_status) {
  const bool wide = row_units >= 32;
  const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t first = wide ? gid / 32 : gid, step = wide ? stride / 32 : stride;
  const int64_t c0 = wide ? (threadIdx.x & 31) : 0, cs = wide ? 32 : 1;
  bool bad = false;
  for (int64_t i = first; i < total; i += step) {
    const int32_t o = src_index[i];
    if (o < 0 || o >= orig_total) {
      bad = true;
      continue;
    }
    const U* src = x + static_cast<int64_t>(o) * row_units;
    U* dst = y + i * row_units;
    for (int64_t c = c0; c < row_units; c += cs) dst[c] = src[c];
  }
  if (bad && dev_status != nullptr) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
}

// dx[o] = dy[first] + dy[second] (or dy[first] alone), V = float4 or float;
// rows spread over warps or threads as in gather_rows_kernel.
template <typename V>
__device__ __forceinline__ V add_v(V a, V b);
template <>
__device__ __forceinline__ float add_v<float>(float a, float b) {
  return a + b;
}
template <>
__device__ __forceinline__ float4 add_v<float4>(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

template <typename V>
__global__ void __launch_bounds__(256) fold_rows_kernel(const V* __restrict__ dy, int64_t total, int64_t row_units,
                                                        const int32_t* __restrict__ copy_index, int32_t slots,
                                                        int64_t orig_total, V* __restrict__ dx,
                                                        int32_t* __restrict__ dev_status) {
  const bool wide = row_units >= 32;
  const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t first = wide ? gid / 32 : gid, step = wide ? stride / 32 : stride;
  const int64_t c0 = wide ? (threadIdx.x & 31) : 0, cs = wide ? 32 : 1;
  bool bad = false;
  for (int64_t o = first; o < orig_total; o += step) {
    const int32_t* cp = copy_index + o * slots;
    int n = 0;
    int32_t a0 = -1, a1 = -1;  // the first two valid copies, in slot order
    for (int k = 0; k < slots; ++k) {
      const int32_t a = cp[k];
      if (a >= total) bad = true;
      if (a < 0 || a >= total) continue;
      if (n == 0) a0 = a;
      else if (n == 1) a1 = a;
      ++n;
    }
    if (n == 0) {  // every original token has at least its first copy
      bad = true;
      continue;
    }
    V* dst = dx + o * row_units;
    if (n <= 2) {  // the common case (one response copy more): both source rows known up front
      const V* s0 = dy + static_cast<int64_t>(a0) * row_units;
      const V* s1 = dy + static_cast<int64_t>(n == 2 ? a1 : a0) * row_units;
#pragma unroll 4
      for (int64_t c = c0; c < row_units; c += cs) {
        V v = s0[c];
        if (n == 2) v = add_v(v, s1[c]);
        dst[c] = v;
      }
      continue;
    }
    for (int64_t c = c0; c < row_units; c += cs) {
      bool have = false;
      V acc;
      for (int k = 0; k < slots; ++k) {  // slot order: first copy, then the others in order
        const int32_t a = cp[k];
        if (a < 0 || a >= total) continue;
        const V v = dy[static_cast<int64_t>(a) * row_units + c];
        acc = have ? add_v(acc, v) : v;
        have = true;
      }
      dst[c] = acc;
    }
  }
  if (bad && dev_status != nullptr) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
}

// ---------------------------------------------------------------------------
// K-pass ("K-Pass 中间方案").  Reading: a conversation's N turns fall into
// K' = min(K, N) contiguous groups with bounds b_g = floor(g N / K'); pass g is
// one conversation of the output: the history of the turns before the group,
// each turn j as the single context segment (h_j + r_j, 0, 0), then the
// group's own turns (h, t, r).  The output is an ordinary input of the
// layout, so the attention kernels serve every K unchanged.

__device__ __forceinline__ int kpass_bound(int g, int n, int k) {
  return static_cast<int>((static_cast<int64_t>(g) * n) / k);
}

// Turns of conversation c, or 0 (flagged) when its pointers leave [0, n_turns]
// or run backwards: no turn outside the arrays is ever read.
__device__ __forceinline__ int conv_turns(const int32_t* conv_turn_ptr, int c, int n_turns, int32_t* dev_status) {
  const int t0 = conv_turn_ptr[c], t1 = conv_turn_ptr[c + 1];
  if (t0 < 0 || t1 < t0 || t1 > n_turns) {
    if (dev_status != nullptr) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
    return 0;
  }
  return t1 - t0;
}

// Single block, conversations kDupThreads at a time: one thread per
// conversation counts its output turns (sum of b_{g+1}) and passes (K'), a block
// scan gives their offsets, then the block writes the conversations' output turns.
__global__ void __launch_bounds__(kDupThreads) kpass_plan_kernel(
    const int32_t* __restrict__ turn_lens, const int32_t* __restrict__ conv_turn_ptr,
    const int32_t* __restrict__ seq_conv_ptr, int32_t n_seqs, int32_t n_convs, int32_t n_turns, int32_t K,
    int32_t n_out_turns, int32_t n_out_convs, int32_t* __restrict__ out_turn_lens,
    int32_t* __restrict__ out_conv_turn_ptr, int32_t* __restrict__ out_seq_conv_ptr,
    int32_t* __restrict__ out_turn_src, int32_t* __restrict__ dev_status) {
  __shared__ int64_t turn_off[kDupThreads], conv_off[kDupThreads];
  __shared__ int64_t warp_a[32], warp_b[32];
  __shared__ int64_t carry_a, carry_b;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry_a = 0;
    carry_b = 0;
    if (conv_turn_ptr[0] != 0 || conv_turn_ptr[n_convs] != n_turns) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
  }
  __syncthreads();
  for (int base = 0; base < n_convs; base += kDupThreads) {
    const int c = base + tid;
    int64_t a = 0, b = 0;
    if (c < n_convs) {
      const int n = conv_turns(conv_turn_ptr, c, n_turns, dev_status);
      const int k = min(K, n);
      for (int g = 0; g < k; ++g) a += kpass_bound(g + 1, n, k);
      b = k;
    }
    int64_t ia = a, ib = b;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int64_t ya = __shfl_up_sync(0xffffffffu, ia, d), yb = __shfl_up_sync(0xffffffffu, ib, d);
      if (lane >= d) {
        ia += ya;
        ib += yb;
      }
    }
    if (lane == 31) {
      warp_a[warp] = ia;
      warp_b[warp] = ib;
    }
    __syncthreads();
    if (warp == 0) {
      const int64_t wa = warp_a[lane], wb = warp_b[lane];
      int64_t xa = wa, xb = wb;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int64_t ya = __shfl_up_sync(0xffffffffu, xa, d), yb = __shfl_up_sync(0xffffffffu, xb, d);
        if (lane >= d) {
          xa += ya;
          xb += yb;
        }
      }
      warp_a[lane] = xa - wa;
      warp_b[lane] = xb - wb;
    }
    __syncthreads();
    const int64_t ca = carry_a, cb = carry_b;
    turn_off[tid] = ca + warp_a[warp] + ia - a;
    conv_off[tid] = cb + warp_b[warp] + ib - b;
    __syncthreads();
    if (tid == kDupThreads - 1) {
      carry_a = ca + warp_a[warp] + ia;
      carry_b = cb + warp_b[warp] + ib;
    }
    // sequence pointers that fall in this chunk
    for (int s = tid; s <= n_seqs; s += kDupThreads) {
      const int cs = seq_conv_ptr[s];
      if (cs >= base && cs < base + kDupThreads && cs < n_convs) out_seq_conv_ptr[s] = static_cast<int32_t>(conv_off[cs - base]);
    }
    const int nc = min(kDupThreads, n_convs - base);
    for (int u = 0; u < nc; ++u) {
      const int cu = base + u;
      const int t0 = conv_turn_ptr[cu];
      const int n = conv_turns(conv_turn_ptr, cu, n_turns, nullptr);
      const int k = min(K, n);
      const int64_t to = turn_off[u], co = conv_off[u];
      // pass pointers
      for (int g = tid; g < k; g += kDupThreads) {
        int64_t before = 0;
        for (int q = 0; q < g; ++q) before += kpass_bound(q + 1, n, k);
        if (co + g < n_out_convs) out_conv_turn_ptr[co + g] = static_cast<int32_t>(to + before);
      }
      // output turns: pass g holds the conversation's turns 0 .. b_{g+1}-1, those below b_g as history
      int64_t total_u = 0;
      for (int g = 0; g < k; ++g) total_u += kpass_bound(g + 1, n, k);
      for (int64_t x = tid; x < total_u; x += kDupThreads) {
        int g = 0;
        int64_t start = 0;
        while (g < k && start + kpass_bound(g + 1, n, k) <= x) {
          start += kpass_bound(g + 1, n, k);
          ++g;
        }
        const int j = static_cast<int>(x - start);  // turn index inside the conversation
        const int tj = t0 + j;
        const int64_t ou = to + x;
        if (ou >= n_out_turns) continue;
        const int h = max(turn_lens[3 * tj], 0), tt = max(turn_lens[3 * tj + 1], 0), r = max(turn_lens[3 * tj + 2], 0);
        if (j < kpass_bound(g, n, k)) {  // history turn: group of turn j, then d = g - that group
          int gj = 0;
          while (kpass_bound(gj + 1, n, k) <= j) ++gj;
          out_turn_lens[3 * ou] = h + r;
          out_turn_lens[3 * ou + 1] = 0;
          out_turn_lens[3 * ou + 2] = 0;
          out_turn_src[2 * ou] = tj;
          out_turn_src[2 * ou + 1] = g - gj;
        } else {
          out_turn_lens[3 * ou] = h;
          out_turn_lens[3 * ou + 1] = tt;
          out_turn_lens[3 * ou + 2] = r;
          out_turn_src[2 * ou] = tj;
          out_turn_src[2 * ou + 1] = -1;
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (carry_a != n_out_turns || carry_b != n_out_convs) {
      atomicOr(dev_status, OPR_DEV_TOTAL_MISMATCH);
    } else {
      out_conv_turn_ptr[n_out_convs] = n_out_turns;
    }
    for (int s = 0; s <= n_seqs; ++s)
      if (seq_conv_ptr[s] >= n_convs) out_seq_conv_ptr[s] = static_cast<int32_t>(carry_b);
  }
}

// Single block: exclusive scans of the original turns' token counts (h + t + r)
// and of the output turns' (h + t + 2r), into the workspace.
__global__ void __launch_bounds__(kDupThreads) kpass_offsets_kernel(const int32_t* __restrict__ turn_lens,
                                                                     int32_t n_turns,
                                                                     const int32_t* __restrict__ out_turn_lens,
                                                                     int32_t n_out_turns, int64_t* __restrict__ orig_off,
                                                                     int64_t* __restrict__ out_off) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int pass = 0; pass < 2; ++pass) {
    const int32_t* lens = pass == 0 ? turn_lens : out_turn_lens;
    const int n = pass == 0 ? n_turns : n_out_turns;
    const int rmul = pass == 0 ? 1 : 2;
    int64_t* off = pass == 0 ? orig_off : out_off;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kDupThreads) {
      const int i = base + tid;
      const int64_t v = (i < n) ? static_cast<int64_t>(max(lens[3 * i], 0)) + max(lens[3 * i + 1], 0) +
                                      static_cast<int64_t>(rmul) * max(lens[3 * i + 2], 0)
                                : 0;
      int64_t incl = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
      }
      if (lane == 31) warp_sums[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        const int64_t w = warp_sums[lane];
        int64_t x = w;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int64_t y = __shfl_up_sync(0xffffffffu, x, d);
          if (lane >= d) x += y;
        }
        warp_sums[lane] = x - w;
      }
      __syncthreads();
      const int64_t c0 = carry;
      if (i < n) off[i] = c0 + warp_sums[warp] + incl - v;
      __syncthreads();
      if (tid == kDupThreads - 1) carry = c0 + warp_sums[warp] + incl;
      __syncthreads();
    }
    if (tid == 0) off[n] = carry;
    __syncthreads();
  }
}

// One block per output turn: src_index of its tokens and their copy slots
// (0: own-pass h / t / r^in copy, 1: r^out copy, 1 + d: history copy d groups later).
__global__ void __launch_bounds__(256) kpass_index_kernel(
    const int32_t* __restrict__ turn_lens, const int32_t* __restrict__ out_turn_lens,
    const int32_t* __restrict__ out_turn_src, int32_t n_turns, const int64_t* __restrict__ orig_off,
    const int64_t* __restrict__ out_off, int64_t total, int64_t orig_total, int32_t slots,
    int32_t* __restrict__ src_index, int32_t* __restrict__ copy_index, int32_t* __restrict__ dev_status) {
  const int u = blockIdx.x;
  const int j = out_turn_src[2 * u], d = out_turn_src[2 * u + 1];
  if (j < 0 || j >= n_turns || (d >= 1 && 1 + d >= slots)) {
    if (threadIdx.x == 0) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
    return;
  }
  const int h = max(turn_lens[3 * j], 0), t = max(turn_lens[3 * j + 1], 0), r = max(turn_lens[3 * j + 2], 0);
  const int64_t o = orig_off[j], base = out_off[u];
  const int n = d >= 1 ? h + r : h + t + 2 * r;
  for (int x = threadIdx.x; x < n; x += blockDim.x) {
    int64_t oi;
    int slot;
    if (d >= 1) {
      oi = x < h ? o + x : o + h + t + (x - h);
      slot = 1 + d;
    } else if (x < h + t + r) {
      oi = o + x;
      slot = 0;
    } else {
      oi = o + h + t + (x - h - t - r);
      slot = 1;
    }
    const int64_t i = base + x;
    if (i >= total || oi >= orig_total) continue;
    src_index[i] = static_cast<int32_t>(oi);
    copy_index[oi * slots + slot] = static_cast<int32_t>(i);
  }
}

// Blocks for `rows` rows of `units` units: a warp per wide row, a thread per narrow one;
// at most 148 SMs x max_per_sm blocks (grid-stride beyond).
int64_t grid_for(int64_t rows, int64_t units, int64_t max_per_sm = 16) {
  const int64_t threads = units >= 32 ? rows * 32 : rows;
  const int64_t blocks = (threads + 255) / 256;
  return blocks < 148 * max_per_sm ? (blocks > 0 ? blocks : 1) : 148 * max_per_sm;
}

// The fold's rows differ in cost (one or two source rows), so its grid covers
// more rows at once and the block scheduler evens the load out.
constexpr int64_t kFoldBlocksPerSm = 64;

}  // namespace

cudaError_t launch_dup_index(const int32_t* turn_lens, const int32_t* conv_turn_ptr, int32_t n_convs, int32_t n_turns,
                             int64_t total, int64_t orig_total, int32_t* src_index, int32_t* copy_index,
                             int32_t* dev_status, cudaStream_t stream) {
  dup_index_kernel<<<1, kDupThreads, 0, stream>>>(turn_lens, conv_turn_ptr, n_convs, n_turns, total, orig_total,
                                                  src_index, copy_index, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, int64_t orig_total, int64_t row_bytes, const int32_t* src_index,
                               int64_t total, void* y, int32_t* dev_status, cudaStream_t stream) {
  const bool a16 = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (reinterpret_cast<uintptr_t>(y) % 16 == 0);
  const bool a4 = (reinterpret_cast<uintptr_t>(x) % 4 == 0) && (reinterpret_cast<uintptr_t>(y) % 4 == 0);
  if (row_bytes % 16 == 0 && a16) {
    const int64_t u = row_bytes / 16;
    gather_rows_kernel<uint4><<<static_cast<unsigned>(grid_for(total, u)), 256, 0, stream>>>(
        static_cast<const uint4*>(x), orig_total, u, src_index, total, static_cast<uint4*>(y), dev_status);
  } else if (row_bytes % 4 == 0 && a4) {
    const int64_t u = row_bytes / 4;
    gather_rows_kernel<uint32_t><<<static_cast<unsigned>(grid_for(total, u)), 256, 0, stream>>>(
        static_cast<const uint32_t*>(x), orig_total, u, src_index, total, static_cast<uint32_t*>(y), dev_status);
  } else {
    gather_rows_kernel<uint8_t><<<static_cast<unsigned>(grid_for(total, row_bytes)), 256, 0, stream>>>(
        static_cast<const uint8_t*>(x), orig_total, row_bytes, src_index, total, static_cast<uint8_t*>(y),
        dev_status);
  }
  return cudaGetLastError();
}

cudaError_t launch_fold_rows(const float* dy, int64_t total, int64_t width, const int32_t* copy_index, int32_t slots,
                             int64_t orig_total, float* dx, int32_t* dev_status, cudaStream_t stream) {
  const bool a16 = (reinterpret_cast<uintptr_t>(dy) % 16 == 0) && (reinterpret_cast<uintptr_t>(dx) % 16 == 0);
  if (width % 4 == 0 && a16) {
    const int64_t u = width / 4;
    fold_rows_kernel<float4><<<static_cast<unsigned>(grid_for(orig_total, u, kFoldBlocksPerSm)), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(dy), total, u, copy_index, slots, orig_total, reinterpret_cast<float4*>(dx),
        dev_status);
  } else {
    fold_rows_kernel<float><<<static_cast<unsigned>(grid_for(orig_total, width, kFoldBlocksPerSm)), 256, 0, stream>>>(
        dy, total, width, copy_index, slots, orig_total, dx, dev_status);
  }
  return cudaGetLastError();
}

cudaError_t launch_kpass_plan(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                              int32_t n_seqs, int32_t n_convs, int32_t n_turns, int32_t K, int32_t n_out_turns,
                              int32_t n_out_convs, int32_t* out_turn_lens, int32_t* out_conv_turn_ptr,
                              int32_t* out_seq_conv_ptr, int32_t* out_turn_src, int32_t* dev_status,
                              cudaStream_t stream) {
  kpass_plan_kernel<<<1, kDupThreads, 0, stream>>>(turn_lens, conv_turn_ptr, seq_conv_ptr, n_seqs, n_convs, n_turns, K,
                                                   n_out_turns, n_out_convs, out_turn_lens, out_conv_turn_ptr,
                                                   out_seq_conv_ptr, out_turn_src, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_kpass_index(const int32_t* turn_lens, int32_t n_turns, const int32_t* out_turn_lens,
                               const int32_t* out_turn_src, int32_t n_out_turns, int64_t total, int64_t orig_total,
                               int32_t slots, int32_t* src_index, int32_t* copy_index, int64_t* ws,
                               int32_t* dev_status, cudaStream_t stream) {
  int64_t* orig_off = ws;
  int64_t* out_off = ws + (n_turns + 1);
  cudaError_t e = cudaMemsetAsync(copy_index, 0xFF, sizeof(int32_t) * static_cast<size_t>(orig_total) * slots, stream);
  if (e != cudaSuccess) return e;
  kpass_offsets_kernel<<<1, kDupThreads, 0, stream>>>(turn_lens, n_turns, out_turn_lens, n_out_turns, orig_off, out_off);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (n_out_turns > 0)
    kpass_index_kernel<<<static_cast<unsigned>(n_out_turns), 256, 0, stream>>>(
        turn_lens, out_turn_lens, out_turn_src, n_turns, orig_off, out_off, total, orig_total, slots, src_index,
        copy_index, dev_status);
  return cudaGetLastError();
}

}  // namespace opr
