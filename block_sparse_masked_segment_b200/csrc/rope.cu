// rope.cu - rotary position embedding by position id, in place.
//
// The equivalence argument of One-Pass to Reason ("理论保证": position
// encoding equivalence -> attention pattern equivalence -> loss equivalence)
// rests on every token keeping, in the one-pass layout, the rotary position it
// would have in its N-pass sequence.  Convention: rotate-half (Qwen-3), the
// pair (x[j], x[j + d/2]) rotated by pos * base^(-2j/d).
//
// One thread per (token, j < d/2): the angle is formed and reduced in fp64 once
// and applied to every head of the token.  HBM-bound: each element is read and
// written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "opr_internal.cuh"

namespace opr {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(T* __restrict__ x, const int32_t* __restrict__ pos_id, int64_t total,
                                                   int32_t n_heads, int32_t half, double neg_log_base_over_half,
                                                   double sign) {
  const int tokens_per_block = blockDim.x / half;
  const int64_t tok = static_cast<int64_t>(blockIdx.x) * tokens_per_block + threadIdx.x / half;
  const int j = threadIdx.x % half;
  if (threadIdx.x >= tokens_per_block * half || tok >= total) return;
  // theta_j = base^(-2j/d) = exp(-(j/half) * ln(base)); angle in fp64
  const double theta = exp(static_cast<double>(j) * neg_log_base_over_half);
  const double ang = sign * static_cast<double>(pos_id[tok]) * theta;
  double sd, cd;
  sincos(ang, &sd, &cd);
  const float c = static_cast<float>(cd), s = static_cast<float>(sd);
  T* row = x + tok * n_heads * (2 * half);
  for (int h = 0; h < n_heads; ++h) {
    T* p = row + static_cast<int64_t>(h) * 2 * half;
    const float a = to_f(p[j]), b = to_f(p[j + half]);
    p[j] = from_f<T>(a * c - b * s);
    p[j + half] = from_f<T>(b * c + a * s);
  }
}

}  // namespace

cudaError_t launch_rope(void* x, int32_t dtype, const int32_t* pos_id, int64_t total, int32_t n_heads,
                        int32_t head_dim, double base, int32_t inverse, cudaStream_t stream) {
  if (total == 0 || n_heads == 0) return cudaSuccess;
  const int half = head_dim / 2;
  const int threads = 256 / half * half;
  const int tpb = threads / half;
  const int64_t blocks = (total + tpb - 1) / tpb;
  const double nl = -log(base) / static_cast<double>(half);
  const double sign = inverse ? -1.0 : 1.0;
  if (dtype == OPR_DTYPE_BF16)
    rope_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        static_cast<__nv_bfloat16*>(x), pos_id, total, n_heads, half, nl, sign);
  else
    rope_kernel<float><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(static_cast<float*>(x), pos_id, total,
                                                                              n_heads, half, nl, sign);
  return cudaGetLastError();
}

}  // namespace opr
