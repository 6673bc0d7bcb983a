// noalloc.cu - opr_attn_bwd_noalloc: the attention backward with its scratch
// in a fixed, library-owned device array instead of caller-provided memory.
//
// Some callers cannot allocate device memory when they call the backward: a
// host framework that owns every device allocation and gives extensions no
// allocator hook, or a latency-critical path that must not call cudaMalloc
// (it can block and synchronize the device).  For them this entry point takes
// the same inputs and outputs as opr_attn_bwd but no workspace: the whole
// backward scratch (max |dO|, the row terms, and the fp16 copies of dO and v)
// lives in the file-scope array below, which every GPU that loads the library
// holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "host_status.h"
#include "opr_internal.cuh"

namespace opr {
namespace {

// Largest backward scratch this entry point serves (OPR_NOALLOC_SCRATCH_BYTES):
// a call is accepted when opr_attn_bwd_min_workspace_bytes(n_seqs, max_seqlen,
// hq, head_dim) -- max |dO|, the row terms and both fp16 copies -- fits.  The
// dK/dV stage is split by q head only when its partials fit as well.
constexpr size_t kNoAllocScratchBytes = OPR_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device, looked up once per device
// (the caller's stream must belong to the current device).
opr_status scratch_on_current_device(void** out) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return OPR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t ea = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (ea != cudaSuccess) return record_cuda_error(ea);
    if (p == nullptr) return record_cuda_error(cudaErrorInvalidSymbol);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return OPR_OK;
}

}  // namespace
}  // namespace opr

extern "C" {

opr_status opr_attn_bwd_noalloc(const void* q, const void* k, const void* v, int32_t qk_dtype, const void* o,
                                int32_t o_dtype, const void* dout, const float* lse, const int32_t* cu_seqlens,
                                const int32_t* conv_idx, const void* layout_ws, int32_t n_seqs, int32_t n_convs,
                                int32_t n_turns, int64_t total_tokens, int32_t max_seqlen, int32_t hq, int32_t hkv,
                                int32_t head_dim, float scale, float* dq, float* dk, float* dv,
                                const int32_t* rope_pos_id, double rope_base, int32_t* dev_status, void* stream) {
  if (!opr::sizes_ok(n_seqs, n_convs, n_turns, total_tokens, max_seqlen) || hq < 0) return OPR_INVALID_ARG;
  if (opr_attn_bwd_min_workspace_bytes(n_seqs, max_seqlen, hq, head_dim) > opr::kNoAllocScratchBytes)
    return OPR_SCRATCH_TOO_LARGE;
  void* scratch = nullptr;
  const opr_status st = opr::scratch_on_current_device(&scratch);
  if (st != OPR_OK) return st;
  // The row-terms kernel writes every scratch entry the other two kernels read,
  // so nothing has to be cleared between calls.
  return opr_attn_bwd(q, k, v, qk_dtype, o, o_dtype, dout, lse, cu_seqlens, conv_idx, layout_ws, n_seqs, n_convs,
                      n_turns, total_tokens, max_seqlen, hq, hkv, head_dim, scale, dq, dk, dv, rope_pos_id, rope_base,
                      scratch, opr::kNoAllocScratchBytes, dev_status, stream);
}

}  // extern "C"
