// rope.cu - rotary position embedding by position id, in place.
//
// The equivalence argument of One-Pass to Reason ("理论保证": position
// encoding equivalence -> attention pattern equivalence -> loss equivalence)
// rests on every token keeping, in the one-pass layout, the rotary position it
// would have in its N-pass sequence.  Convention: rotate-half (Qwen-3), the
// pair (x[j], x[j + d/2]) rotated by pos * base^(-2j/d).
//
// One thread per (token, j < d/2): the angle is formed and reduced in fp64 once
// and applied to every head of the token (general form; aligned tensors with
// d/2 a multiple of 8 take the vectorised form below).  HBM-bound: each element is read and
// written once.  Input and output types may differ (bf16 in, fp16 out for the
// rotated q and k; in place when they are the same buffer and type); an fp16
// output value beyond the fp16 range sets OPR_DEV_FP16_RANGE.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

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
template <>
__device__ __forceinline__ float to_f<__half>(__half v) {
  return __half2float(v);
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
template <>
__device__ __forceinline__ __half from_f<__half>(float v) {
  return __float2half_rn(v);
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) rope_kernel(const TI* x, TO* y, const int32_t* __restrict__ pos_id,
                                                   const int32_t* __restrict__ row_map, int64_t total,
                                                   int32_t n_heads, int32_t half, double neg_log_base_over_half,
                                                   double sign, int32_t* __restrict__ dev_status) {
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
  const int64_t orow_tok = row_map != nullptr ? row_map[tok] : tok;
  if (orow_tok < 0 || orow_tok >= total) return;
  const int64_t row = tok * n_heads * (2 * half), orow = orow_tok * n_heads * (2 * half);
  bool out_of_range = false;
  for (int h = 0; h < n_heads; ++h) {
    const int64_t o = row + static_cast<int64_t>(h) * 2 * half, oo = orow + static_cast<int64_t>(h) * 2 * half;
    const float a = to_f(x[o + j]), b = to_f(x[o + j + half]);
    const float ya = a * c - b * s, yb = b * c + a * s;
    if constexpr (sizeof(TO) == 2 && !std::is_same_v<TO, __nv_bfloat16>)
      out_of_range |= !(fabsf(ya) <= 65504.f) || !(fabsf(yb) <= 65504.f);
    y[oo + j] = from_f<TO>(ya);
    y[oo + j + half] = from_f<TO>(yb);
  }
  if (out_of_range && dev_status != nullptr) atomicOr(dev_status, OPR_DEV_FP16_RANGE);
}

// Eight consecutive elements as floats, with 16-byte accesses (the element
// offset is a multiple of 8 and the tensor 16-byte aligned).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]) {
  if constexpr (std::is_same_v<T, float>) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = to_f(e[k]);
  }
}
template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&v)[8]) {
  if constexpr (std::is_same_v<T, float>) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 u;
    T* e = reinterpret_cast<T*>(&u);
#pragma unroll
    for (int k = 0; k < 8; ++k) e[k] = from_f<T>(v[k]);
    *reinterpret_cast<uint4*>(p) = u;
  }
}

// Vectorised form for 16-byte aligned tensors with d/2 a multiple of 8: a block
// takes kRopeTok tokens, forms their cos/sin once in shared memory (fp64 angle
// as above), and each thread rotates eight consecutive pairs (j .. j+7 with
// j+d/2 .. j+d/2+7) of one head; consecutive threads take consecutive chunks,
// so a warp reads and writes whole 128-byte lines.
constexpr int kRopeTok = 8;

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) rope_vec_kernel(const TI* x, TO* y, const int32_t* __restrict__ pos_id,
                                                       const int32_t* __restrict__ row_map, int64_t total,
                                                       int32_t n_heads, int32_t half, double neg_log_base_over_half,
                                                       double sign, int32_t* __restrict__ dev_status) {
  extern __shared__ float2 cs[];  // [kRopeTok][half]: (cos, sin)
  const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRopeTok;
  const int ntok = static_cast<int>(total - tok0 < kRopeTok ? total - tok0 : kRopeTok);
  for (int i = threadIdx.x; i < ntok * half; i += blockDim.x) {
    const int t = i / half, j = i % half;
    const double theta = exp(static_cast<double>(j) * neg_log_base_over_half);
    const double ang = sign * static_cast<double>(pos_id[tok0 + t]) * theta;
    double sd, cd;
    sincos(ang, &sd, &cd);
    cs[i] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
  }
  __syncthreads();
  const int chunks = half / 8;
  const int items = ntok * n_heads * chunks;
  bool out_of_range = false;
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int c = it % chunks, th = it / chunks;
    const int h = th % n_heads, t = th / n_heads;
    const int64_t otok = row_map != nullptr ? row_map[tok0 + t] : tok0 + t;
    if (otok < 0 || otok >= total) continue;
    const int64_t o = ((tok0 + t) * n_heads + h) * static_cast<int64_t>(2 * half) + 8 * c;
    const int64_t oo = (otok * n_heads + h) * static_cast<int64_t>(2 * half) + 8 * c;
    float a[8], b[8], ya[8], yb[8];
    load8(x + o, a);
    load8(x + o + half, b);
    const float2* w = cs + t * half + 8 * c;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 cw = w[k];
      ya[k] = a[k] * cw.x - b[k] * cw.y;
      yb[k] = b[k] * cw.x + a[k] * cw.y;
      if constexpr (sizeof(TO) == 2 && !std::is_same_v<TO, __nv_bfloat16>)
        out_of_range |= !(fabsf(ya[k]) <= 65504.f) || !(fabsf(yb[k]) <= 65504.f);
    }
    store8(y + oo, ya);
    store8(y + oo + half, yb);
  }
  if (out_of_range && dev_status != nullptr) atomicOr(dev_status, OPR_DEV_FP16_RANGE);
}

// No position ids: the rotation by angle 0, i.e. a plain type conversion (e.g.
// the fp16 copy of v that lets the forward's P V product take P in fp16).  Eight
// elements per thread and step when both tensors are 16-byte aligned and n is a
// multiple of 8 (16-byte accesses), else one.
template <typename TI, typename TO>
__global__ void __launch_bounds__(256) convert_kernel(const TI* x, TO* y, const int32_t* __restrict__ row_map,
                                                      int64_t total, int64_t row_len, bool vec,
                                                      int32_t* __restrict__ dev_status) {
  constexpr bool kF16 = std::is_same<TO, __half>::value;
  bool out_of_range = false;
  const int64_t n = total * row_len;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // output element of input element e (row e / row_len moved to row_map[row])
  auto out_at = [&](int64_t e) -> int64_t {
    if (row_map == nullptr) return e;
    const int64_t r = row_map[e / row_len];
    return (r < 0 || r >= total) ? -1 : r * row_len + e % row_len;
  };
  if (vec) {  // row_len is a multiple of 8: eight elements never straddle two rows
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n / 8; i += stride) {
      const int64_t o = out_at(8 * i);
      if (o < 0) continue;
      float v[8];
      load8(x + 8 * i, v);
      if constexpr (kF16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) out_of_range |= !(fabsf(v[k]) <= 65504.f);
      }
      store8(y + o, v);
    }
  } else {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride) {
      const int64_t o = out_at(i);
      if (o < 0) continue;
      const float v = to_f<TI>(x[i]);
      if constexpr (kF16) out_of_range |= !(fabsf(v) <= 65504.f);
      y[o] = from_f<TO>(v);
    }
  }
  if (out_of_range && dev_status != nullptr) atomicOr(dev_status, OPR_DEV_FP16_RANGE);
}

template <typename TI, typename TO>
cudaError_t launch_t(const void* x, void* y, const int32_t* pos_id, const int32_t* row_map, int64_t total,
                     int32_t n_heads, int32_t half, double nl, double sign, int32_t* dev_status, cudaStream_t stream) {
  if (pos_id == nullptr) {
    const int64_t row_len = static_cast<int64_t>(n_heads) * 2 * half;
    const int64_t n = total * row_len;
    const bool vec = row_len % 8 == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(y) & 15u) == 0;
    const int64_t items = vec ? n / 8 : n;
    const int64_t blocks = std::min<int64_t>((items + 255) / 256, 148 * 16);
    convert_kernel<TI, TO><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const TI*>(x), static_cast<TO*>(y), row_map, total, row_len, vec, dev_status);
    return cudaGetLastError();
  }
  const bool vec = half % 8 == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(y) & 15u) == 0;
  if (vec) {
    const int64_t blocks = (total + kRopeTok - 1) / kRopeTok;
    const size_t smem = sizeof(float2) * kRopeTok * half;
    rope_vec_kernel<TI, TO><<<static_cast<unsigned>(blocks), 256, smem, stream>>>(
        static_cast<const TI*>(x), static_cast<TO*>(y), pos_id, row_map, total, n_heads, half, nl, sign, dev_status);
    return cudaGetLastError();
  }
  const int threads = 256 / half * half;
  const int tpb = threads / half;
  const int64_t blocks = (total + tpb - 1) / tpb;
  rope_kernel<TI, TO><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const TI*>(x), static_cast<TO*>(y), pos_id, row_map, total, n_heads, half, nl, sign, dev_status);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_in(const void* x, int32_t y_dtype, void* y, const int32_t* pos_id, const int32_t* row_map,
                      int64_t total, int32_t n_heads, int32_t half, double nl, double sign, int32_t* dev_status,
                      cudaStream_t stream) {
  if (y_dtype == OPR_DTYPE_BF16)
    return launch_t<TI, __nv_bfloat16>(x, y, pos_id, row_map, total, n_heads, half, nl, sign, dev_status, stream);
  if (y_dtype == OPR_DTYPE_FP16)
    return launch_t<TI, __half>(x, y, pos_id, row_map, total, n_heads, half, nl, sign, dev_status, stream);
  return launch_t<TI, float>(x, y, pos_id, row_map, total, n_heads, half, nl, sign, dev_status, stream);
}

}  // namespace

cudaError_t launch_rope(const void* x, int32_t x_dtype, void* y, int32_t y_dtype, const int32_t* pos_id,
                        const int32_t* row_map, int64_t total, int32_t n_heads, int32_t head_dim, double base,
                        int32_t inverse, int32_t* dev_status, cudaStream_t stream) {
  if (total == 0 || n_heads == 0) return cudaSuccess;
  const int half = head_dim / 2;
  const double nl = -log(base) / static_cast<double>(half);
  const double sign = inverse ? -1.0 : 1.0;
  if (x_dtype == OPR_DTYPE_BF16)
    return launch_in<__nv_bfloat16>(x, y_dtype, y, pos_id, row_map, total, n_heads, half, nl, sign, dev_status, stream);
  if (x_dtype == OPR_DTYPE_FP16)
    return launch_in<__half>(x, y_dtype, y, pos_id, row_map, total, n_heads, half, nl, sign, dev_status, stream);
  return launch_in<float>(x, y_dtype, y, pos_id, row_map, total, n_heads, half, nl, sign, dev_status, stream);
}

}  // namespace opr
