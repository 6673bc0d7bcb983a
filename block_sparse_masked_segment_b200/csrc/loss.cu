// loss.cu - the step after the attention layer: the one-pass rows that carry
// the N-pass next-token losses, and a fused softmax cross-entropy.
//
// The pages prove that the one-pass loss equals the N-pass loss ("理论保证")
// and train on the r^out copies ("Token 复制").  In N-pass run i the losses
// are the next-token predictions of t_i and r_i: from the last h_i row
// (target: the first t_i token, or r_i[0] when t_i is empty), from each t_i row
// (target: the next t_i token, or r_i[0] after the last t_i token) and from
// each r_i row but the last (target: the next r_i token).  In one pass those
// rows are the last h_i row, the t_i rows and the r_i^out rows.
//
//   loss_rows_kernel       compacted list of those rows, in stream order, with
//                          the original-stream index of each row's target;
//   cross_entropy_kernel   per row: loss = logsumexp(z) - z[target] and, when
//                          asked, dz = scale (softmax(z) - onehot(target)).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "opr_internal.cuh"

namespace opr {
namespace {

constexpr int kLossThreads = 1024;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int turn_loss_rows(int h, int t, int r) {
  return ((h > 0 && t + r > 0) ? 1 : 0) + (r > 0 ? t : (t > 0 ? t - 1 : 0)) + (r > 1 ? r - 1 : 0);
}

// Single block, turns kLossThreads at a time: per-turn row counts and the
// turns' offsets in the one-pass and original streams by block scans, then the
// block writes the rows of those turns.  Writes are bounds-checked; a count
// that disagrees with n_rows (or a total with the lengths) is flagged.
__global__ void __launch_bounds__(kLossThreads) loss_rows_kernel(const int32_t* __restrict__ turn_lens,
                                                                 int32_t n_turns, int64_t total, int64_t orig_total,
                                                                 int64_t n_rows, int32_t* __restrict__ rows,
                                                                 int32_t* __restrict__ targets,
                                                                 int32_t* __restrict__ dev_status) {
  __shared__ int64_t off[3][kLossThreads];
  __shared__ int32_t lens[kLossThreads][3];
  __shared__ int64_t warp_s[3][32];
  __shared__ int64_t carry[3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 3) carry[tid] = 0;
  __syncthreads();
  bool bad = false;
  for (int base = 0; base < n_turns; base += kLossThreads) {
    const int tu = base + tid;
    int h = 0, t = 0, r = 0;
    if (tu < n_turns) {
      h = turn_lens[3 * tu];
      t = turn_lens[3 * tu + 1];
      r = turn_lens[3 * tu + 2];
      if (h < 0 || t < 0 || r < 0) bad = true;
      h = max(h, 0);
      t = max(t, 0);
      r = max(r, 0);
    }
    lens[tid][0] = h;
    lens[tid][1] = t;
    lens[tid][2] = r;
    int64_t v[3] = {static_cast<int64_t>(h) + t + 2 * static_cast<int64_t>(r), static_cast<int64_t>(h) + t + r,
                    turn_loss_rows(h, t, r)};
    int64_t inc[3] = {v[0], v[1], v[2]};
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int64_t y = __shfl_up_sync(0xffffffffu, inc[q], d);
        if (lane >= d) inc[q] += y;
      }
    }
    if (lane == 31)
#pragma unroll
      for (int q = 0; q < 3; ++q) warp_s[q][warp] = inc[q];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int64_t w0 = warp_s[q][lane];
        int64_t x = w0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int64_t y = __shfl_up_sync(0xffffffffu, x, d);
          if (lane >= d) x += y;
        }
        warp_s[q][lane] = x - w0;
      }
    }
    __syncthreads();
    int64_t c0[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      c0[q] = carry[q];
      off[q][tid] = c0[q] + warp_s[q][warp] + inc[q] - v[q];
    }
    __syncthreads();
    if (tid == kLossThreads - 1)
#pragma unroll
      for (int q = 0; q < 3; ++q) carry[q] = c0[q] + warp_s[q][warp] + inc[q];
    const int nt = min(kLossThreads, n_turns - base);
    for (int u = 0; u < nt; ++u) {
      const int hu = lens[u][0], tu2 = lens[u][1], ru = lens[u][2];
      const int64_t one = off[0][u], orig = off[1][u], ro = off[2][u];
      const int hrow = (hu > 0 && tu2 + ru > 0) ? 1 : 0;
      const int trows = ru > 0 ? tu2 : (tu2 > 0 ? tu2 - 1 : 0);
      const int n = turn_loss_rows(hu, tu2, ru);
      for (int x = tid; x < n; x += kLossThreads) {
        int64_t row, tgt;
        if (x < hrow) {
          row = one + hu - 1;
          tgt = orig + hu;
        } else if (x < hrow + trows) {
          const int k = x - hrow;
          row = one + hu + k;
          tgt = orig + hu + k + 1;
        } else {
          const int k = x - hrow - trows;
          row = one + hu + tu2 + ru + k;
          tgt = orig + hu + tu2 + k + 1;
        }
        const int64_t i = ro + x;
        if (i < n_rows && row < total && tgt < orig_total) {
          rows[i] = static_cast<int32_t>(row);
          targets[i] = static_cast<int32_t>(tgt);
        }
      }
    }
    __syncthreads();
  }
  if (bad) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
  if (tid == 0 && (carry[0] != total || carry[1] != orig_total || carry[2] != n_rows))
    atomicOr(dev_status, OPR_DEV_TOTAL_MISMATCH);
}

// Online (max, sum 2^(x - max)) of a thread's values in base 2: a new maximum
// rescales the running sum once, every other value adds one 2^(x - max).
__device__ __forceinline__ void online_add(float& m, float& s, float x2) {
  if (x2 == -INFINITY) return;  // a masked logit adds nothing
  if (x2 > m) {
    s = s * ex2f(m - x2) + 1.f;
    m = x2;
  } else {
    s += ex2f(x2 - m);
  }
}

__device__ __forceinline__ void merge_ms(float& m, float& s, float m2, float s2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  s = s * ex2f(m - mm) + s2 * ex2f(m2 - mm);
  m = mm;
}

// Eight consecutive logits of a row as floats (bf16: one 16-byte load; fp32: two).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]) {
  if constexpr (std::is_same_v<T, float>) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __low2float(b2[k]);
      v[2 * k + 1] = __high2float(b2[k]);
    }
  }
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&v)[8]) {
  if constexpr (std::is_same_v<T, float>) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 u;
    __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) b2[k] = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
}

template <typename T>
__device__ __forceinline__ float to_float(T v) {
  if constexpr (std::is_same_v<T, float>)
    return v;
  else
    return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_float(float v) {
  if constexpr (std::is_same_v<T, float>)
    return v;
  else
    return __float2bfloat16_rn(v);
}

// One block of 256 threads per row; the arithmetic runs in base 2 on the SFU's
// ex2 (scores pre-multiplied by log2 e).  Two reads of the row (statistics,
// then the gradient) and one write.  VEC: the row is 16-byte aligned with
// vocab % 8 == 0, read eight values at a time.
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) cross_entropy_kernel(const T* __restrict__ logits, int64_t n_rows, int32_t V,
                                                            const int32_t* __restrict__ target_ids,
                                                            float* __restrict__ loss, T* __restrict__ dlogits,
                                                            float grad_scale, int32_t* __restrict__ dev_status) {
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.69314718055994531f;
  __shared__ float red_m[8], red_s[8];
  __shared__ float row_lse2;
  const int64_t row = blockIdx.x;
  if (row >= n_rows) return;
  const T* z = logits + row * V;
  const int tgt = target_ids[row];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tgt < 0 || tgt >= V) {  // ignored row (or a bad target, flagged): no loss, no gradient
    if (tgt >= V && tid == 0) atomicOr(dev_status, OPR_DEV_BAD_INPUT);
    if (tid == 0) loss[row] = 0.f;
    if (dlogits != nullptr)
      for (int j = tid; j < V; j += blockDim.x) dlogits[row * V + j] = from_float<T>(0.f);
    return;
  }
  float m = -INFINITY, s = 0.f;
  if constexpr (VEC) {
    for (int j = tid * 8; j < V; j += blockDim.x * 8) {
      float v[8];
      load8(z + j, v);
#pragma unroll
      for (int k = 0; k < 8; ++k) online_add(m, s, v[k] * kLog2e);
    }
  } else {
    for (int j = tid; j < V; j += blockDim.x) online_add(m, s, to_float(z[j]) * kLog2e);
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, d), s2 = __shfl_xor_sync(0xffffffffu, s, d);
    merge_ms(m, s, m2, s2);
  }
  if (lane == 0) {
    red_m[warp] = m;
    red_s[warp] = s;
  }
  __syncthreads();
  if (tid == 0) {
    float mm = red_m[0], ss = red_s[0];
    for (int w = 1; w < 8; ++w) merge_ms(mm, ss, red_m[w], red_s[w]);
    row_lse2 = mm + log2f(ss);
    loss[row] = row_lse2 * kLn2 - to_float(z[tgt]);
  }
  __syncthreads();
  if (dlogits == nullptr) return;
  const float lse2 = row_lse2;
  T* dz = dlogits + row * V;
  if constexpr (VEC) {
    for (int j = tid * 8; j < V; j += blockDim.x * 8) {
      float v[8];
      load8(z + j, v);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        v[k] = grad_scale * (ex2f(fmaf(v[k], kLog2e, -lse2)) - (j + k == tgt ? 1.f : 0.f));
      store8(dz + j, v);
    }
  } else {
    for (int j = tid; j < V; j += blockDim.x)
      dz[j] = from_float<T>(grad_scale * (ex2f(fmaf(to_float(z[j]), kLog2e, -lse2)) - (j == tgt ? 1.f : 0.f)));
  }
}

}  // namespace

cudaError_t launch_loss_rows(const int32_t* turn_lens, int32_t n_turns, int64_t total, int64_t orig_total,
                             int64_t n_rows, int32_t* rows, int32_t* targets, int32_t* dev_status,
                             cudaStream_t stream) {
  loss_rows_kernel<<<1, kLossThreads, 0, stream>>>(turn_lens, n_turns, total, orig_total, n_rows, rows, targets,
                                                   dev_status);
  return cudaGetLastError();
}

cudaError_t launch_cross_entropy(const void* logits, bool bf16, int64_t n_rows, int32_t V, const int32_t* target_ids,
                                 float* loss, void* dlogits, float grad_scale, int32_t* dev_status,
                                 cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(n_rows);
  const bool vec = V % 8 == 0 && reinterpret_cast<uintptr_t>(logits) % 16 == 0 &&
                   (dlogits == nullptr || reinterpret_cast<uintptr_t>(dlogits) % 16 == 0);
  if (bf16) {
    const auto* z = static_cast<const __nv_bfloat16*>(logits);
    auto* dz = static_cast<__nv_bfloat16*>(dlogits);
    if (vec)
      cross_entropy_kernel<__nv_bfloat16, true><<<grid, 256, 0, stream>>>(z, n_rows, V, target_ids, loss, dz,
                                                                          grad_scale, dev_status);
    else
      cross_entropy_kernel<__nv_bfloat16, false><<<grid, 256, 0, stream>>>(z, n_rows, V, target_ids, loss, dz,
                                                                           grad_scale, dev_status);
  } else {
    const auto* z = static_cast<const float*>(logits);
    auto* dz = static_cast<float*>(dlogits);
    if (vec)
      cross_entropy_kernel<float, true><<<grid, 256, 0, stream>>>(z, n_rows, V, target_ids, loss, dz, grad_scale,
                                                                  dev_status);
    else
      cross_entropy_kernel<float, false><<<grid, 256, 0, stream>>>(z, n_rows, V, target_ids, loss, dz, grad_scale,
                                                                   dev_status);
  }
  return cudaGetLastError();
}

}  // namespace opr
