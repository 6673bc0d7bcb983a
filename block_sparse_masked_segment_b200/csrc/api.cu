// api.cu - the extern "C" entry points of libopr.so declared in include/opr.h:
// host-side argument checks, TMA descriptor encoding and kernel dispatch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include <atomic>

#include "../../include/opr_testing.h"
#include "attn_common.cuh"
#include "host_status.h"
#include "opr_internal.cuh"

namespace opr {
cudaError_t launch_attn_fwd(int head_dim, bool qk_f16, bool v_f16, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_bwd(int head_dim, bool qk_f16, const BwdMaps& m, const BwdBuffers& b, const AttnParams& pq,
                            const AttnParams& pkv, int stages, cudaStream_t stream);
cudaError_t launch_dup_index(const int32_t* turn_lens, const int32_t* conv_turn_ptr, int32_t n_convs, int32_t n_turns,
                             int64_t total, int64_t orig_total, int32_t* src_index, int32_t* copy_index,
                             int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_gather_rows(const void* x, int64_t orig_total, int64_t row_bytes, const int32_t* src_index,
                               int64_t total, void* y, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_fold_rows(const float* dy, int64_t total, int64_t width, const int32_t* copy_index, int32_t slots,
                             int64_t orig_total, float* dx, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_kpass_plan(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                              int32_t n_seqs, int32_t n_convs, int32_t n_turns, int32_t K, int32_t n_out_turns,
                              int32_t n_out_convs, int32_t* out_turn_lens, int32_t* out_conv_turn_ptr,
                              int32_t* out_seq_conv_ptr, int32_t* out_turn_src, int32_t* dev_status,
                              cudaStream_t stream);
cudaError_t launch_loss_rows(const int32_t* turn_lens, int32_t n_turns, int64_t total, int64_t orig_total,
                             int64_t n_rows, int32_t* rows, int32_t* targets, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_cross_entropy(const void* logits, bool bf16, int64_t n_rows, int32_t V, const int32_t* target_ids,
                                 float* loss, void* dlogits, float grad_scale, int32_t* dev_status,
                                 cudaStream_t stream);
cudaError_t launch_kpass_index(const int32_t* turn_lens, int32_t n_turns, const int32_t* out_turn_lens,
                               const int32_t* out_turn_src, int32_t n_out_turns, int64_t total, int64_t orig_total,
                               int32_t slots, int32_t* src_index, int32_t* copy_index, int64_t* ws,
                               int32_t* dev_status, cudaStream_t stream);

// Sizes every attention entry point accepts (declared in host_status.h).
bool sizes_ok(int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total, int32_t max_seqlen) {
  if (n_seqs < 0 || n_convs < 0 || n_turns < 0 || total < 0 || max_seqlen < 0) return false;
  if (total >= (int64_t{1} << 31)) return false;  // token offsets are int32
  if (n_seqs > 65535) return false;
  const int64_t T = (max_seqlen + kTile - 1) / kTile;
  if (T > 65535) return false;
  if (static_cast<int64_t>(n_seqs) * T >= (int64_t{1} << 31)) return false;
  // every sequence is at most max_seqlen long, so the tokens fit n_seqs * T tiles; the
  // workspaces sized from (n_seqs, max_seqlen) rely on it
  if (total > static_cast<int64_t>(n_seqs) * T * kTile) return false;
  return true;
}

namespace {
thread_local const char* g_cuda_error_text = "no error";
std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};  // pipeline-wait limit of the attention kernels
}  // namespace

opr_status record_cuda_error(cudaError_t e) {
  g_cuda_error_text = cudaGetErrorString(e);
  return OPR_CUDA_ERROR;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// One NVTX range per entry-point call (named after the call), so that a
// profiler timeline shows where each library call's launches begin and end.
// Without an attached tool the push and pop cost a branch each.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

opr_status cuda_fail(cudaError_t e) { return record_cuda_error(e); }

opr_status status_of(cudaError_t e) { return e == cudaSuccess ? OPR_OK : cuda_fail(e); }

opr_status map_fail() {
  g_cuda_error_text = "TMA tensor map encoding failed (cuTensorMapEncodeTiled)";
  return OPR_CUDA_ERROR;
}

// [tokens, heads, head_dim] 16-bit tensor (bf16 or fp16) as a 3-D TMA map with
// 128-byte swizzle; a box is 64 head_dim elements x 1 head x 128 tokens (rows
// past the end read 0).
bool make_map(CUtensorMap* map, const void* ptr, int64_t total, int32_t heads, int32_t head_dim,
              bool f16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(total)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2, static_cast<cuuint64_t>(heads) * head_dim * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kTile)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

opr_status device_check() {
  int dev = 0, major = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  return major == 10 ? OPR_OK : OPR_UNSUPPORTED;
}

AttnParams base_params(const int32_t* cu_seqlens, const int32_t* conv_idx, const void* ws, int32_t n_seqs,
                       int32_t n_convs, int32_t n_turns, int64_t total, int32_t max_seqlen, int32_t hq, int32_t hkv,
                       float scale, int32_t* dev_status) {
  const LayoutWs w = layout_ws_map(n_seqs, n_convs, n_turns, total, max_seqlen);
  (void)conv_idx;  // the kernels read the layout's attention-order copy
  AttnParams p{};
  p.cu_seqlens = cu_seqlens;
  p.conv_idx = ws_ptr<int32_t>(ws, w.attn_conv);
  p.tok_meta = ws_ptr<int32_t>(ws, w.attn_meta);
  p.stream_of = ws_ptr<int32_t>(ws, w.stream_of);
  p.row_cnt = ws_ptr<int32_t>(ws, w.row_cnt);
  p.row_list = ws_ptr<int32_t>(ws, w.row_list);
  p.col_cnt = ws_ptr<int32_t>(ws, w.col_cnt);
  p.col_list = ws_ptr<int32_t>(ws, w.col_list);
  p.sched = ws_ptr<int32_t>(ws, w.q_sched);
  p.tile_meta = ws_ptr<TileMeta>(ws, w.tile_meta);
  p.T = w.T;
  p.n_items = w.n_tiles;
  p.total = total;
  p.hq = hq;
  p.hkv = hkv;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.dev_status = dev_status;
  const uint64_t limit = g_wait_limit_ns.load();
  p.wait_ns = limit > 0xFFFFFFFFull ? 0xFFFFFFFFu : static_cast<uint32_t>(limit);
  return p;
}

bool attn_args_ok(const void* q, const void* k, const void* v, int32_t hq, int32_t hkv, int32_t head_dim,
                  float scale) {
  if (!q || !k || !v) return false;
  if (hq <= 0 || hkv <= 0 || hq % hkv != 0) return false;
  if (head_dim != 64 && head_dim != 128) return false;
  if (!(scale > 0.f)) return false;
  return aligned16(q) && aligned16(k) && aligned16(v);
}

}  // namespace
}  // namespace opr

using namespace opr;

extern "C" {

opr_status opr_duplication_index(const int32_t* turn_lens, const int32_t* conv_turn_ptr, int32_t n_convs,
                                 int32_t n_turns, int64_t total_tokens, int64_t orig_tokens, int32_t* src_index,
                                 int32_t* copy_index, int32_t* dev_status, void* stream) {
  CallRange range("opr_duplication_index");
  if (n_convs < 0 || n_turns < 0 || total_tokens < 0 || orig_tokens < 0) return OPR_INVALID_ARG;
  if (total_tokens >= (int64_t{1} << 31) || orig_tokens > total_tokens) return OPR_INVALID_ARG;
  if (!conv_turn_ptr || !dev_status || (n_turns > 0 && !turn_lens) || (total_tokens > 0 && !src_index) ||
      (orig_tokens > 0 && !copy_index))
    return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_dup_index(turn_lens, conv_turn_ptr, n_convs, n_turns, total_tokens, orig_tokens, src_index,
                                    copy_index, dev_status, static_cast<cudaStream_t>(stream)));
}

opr_status opr_gather_rows(const void* x, int64_t orig_tokens, int64_t row_bytes, const int32_t* src_index,
                           int64_t total_tokens, void* y, int32_t* dev_status, void* stream) {
  CallRange range("opr_gather_rows");
  if (orig_tokens < 0 || total_tokens < 0 || row_bytes <= 0) return OPR_INVALID_ARG;
  if (total_tokens == 0) return OPR_OK;
  if (!x || !src_index || !y) return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_gather_rows(x, orig_tokens, row_bytes, src_index, total_tokens, y, dev_status,
                                      static_cast<cudaStream_t>(stream)));
}

opr_status opr_fold_rows(const float* dy, int64_t total_tokens, int64_t width, const int32_t* copy_index,
                         int32_t slots, int64_t orig_tokens, float* dx, int32_t* dev_status, void* stream) {
  CallRange range("opr_fold_rows");
  if (orig_tokens < 0 || total_tokens < 0 || width <= 0 || slots < 1 || slots > 64) return OPR_INVALID_ARG;
  if (orig_tokens == 0) return OPR_OK;
  if (!dy || !copy_index || !dx) return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_fold_rows(dy, total_tokens, width, copy_index, slots, orig_tokens, dx, dev_status,
                                    static_cast<cudaStream_t>(stream)));
}

opr_status opr_kpass_sizes(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                           int32_t n_seqs, int32_t n_convs, int32_t n_turns, int32_t K, int64_t* n_out_turns,
                           int64_t* n_out_convs, int64_t* total_tokens, int64_t* max_seqlen, int64_t* orig_tokens) {
  if (!conv_turn_ptr || !seq_conv_ptr || (n_turns > 0 && !turn_lens) || !n_out_turns || !n_out_convs ||
      !total_tokens || !max_seqlen || !orig_tokens)
    return OPR_INVALID_ARG;
  if (n_seqs < 0 || n_convs < 0 || n_turns < 0 || K < 1) return OPR_INVALID_ARG;
  if (conv_turn_ptr[0] != 0 || conv_turn_ptr[n_convs] != n_turns || seq_conv_ptr[0] != 0 ||
      seq_conv_ptr[n_seqs] != n_convs)
    return OPR_INVALID_ARG;
  for (int i = 0; i < 3 * n_turns; ++i)
    if (turn_lens[i] < 0) return OPR_INVALID_ARG;
  int64_t turns = 0, convs = 0, total = 0, longest = 0, orig = 0;
  for (int i = 0; i < n_turns; ++i) orig += int64_t{turn_lens[3 * i]} + turn_lens[3 * i + 1] + turn_lens[3 * i + 2];
  for (int s = 0; s < n_seqs; ++s) {
    if (seq_conv_ptr[s + 1] < seq_conv_ptr[s]) return OPR_INVALID_ARG;
    int64_t seq_len = 0;
    for (int c = seq_conv_ptr[s]; c < seq_conv_ptr[s + 1]; ++c) {
      const int64_t t0 = conv_turn_ptr[c], n = conv_turn_ptr[c + 1] - t0;
      if (n < 0) return OPR_INVALID_ARG;
      const int64_t k = n < K ? n : K;  // K' = min(K, N) groups, bounds floor(g N / K')
      for (int64_t g = 0; g < k; ++g) {
        const int64_t b0 = (g * n) / k, b1 = ((g + 1) * n) / k;
        for (int64_t j = t0; j < t0 + b0; ++j)  // history: h_j + r_j as one context segment
          seq_len += int64_t{turn_lens[3 * j]} + turn_lens[3 * j + 2];
        for (int64_t j = t0 + b0; j < t0 + b1; ++j)  // the group's own turns, laid out one-pass
          seq_len += int64_t{turn_lens[3 * j]} + turn_lens[3 * j + 1] + 2 * int64_t{turn_lens[3 * j + 2]};
        turns += b1;
      }
      convs += k;
    }
    total += seq_len;
    longest = seq_len > longest ? seq_len : longest;
  }
  if (turns >= (int64_t{1} << 31) || convs >= (int64_t{1} << 31) || total >= (int64_t{1} << 31))
    return OPR_INVALID_ARG;
  *n_out_turns = turns;
  *n_out_convs = convs;
  *total_tokens = total;
  *max_seqlen = longest;
  *orig_tokens = orig;
  return OPR_OK;
}

opr_status opr_kpass_plan(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                          int32_t n_seqs, int32_t n_convs, int32_t n_turns, int32_t K, int32_t n_out_turns,
                          int32_t n_out_convs, int32_t* out_turn_lens, int32_t* out_conv_turn_ptr,
                          int32_t* out_seq_conv_ptr, int32_t* out_turn_src, int32_t* dev_status, void* stream) {
  CallRange range("opr_kpass_plan");
  if (n_seqs < 0 || n_convs < 0 || n_turns < 0 || K < 1 || n_out_turns < 0 || n_out_convs < 0) return OPR_INVALID_ARG;
  if (!conv_turn_ptr || !seq_conv_ptr || !out_conv_turn_ptr || !out_seq_conv_ptr || !dev_status ||
      (n_turns > 0 && !turn_lens) || (n_out_turns > 0 && (!out_turn_lens || !out_turn_src)))
    return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_kpass_plan(turn_lens, conv_turn_ptr, seq_conv_ptr, n_seqs, n_convs, n_turns, K, n_out_turns,
                                     n_out_convs, out_turn_lens, out_conv_turn_ptr, out_seq_conv_ptr, out_turn_src,
                                     dev_status, static_cast<cudaStream_t>(stream)));
}

size_t opr_kpass_index_workspace_bytes(int32_t n_turns, int32_t n_out_turns) {
  if (n_turns < 0 || n_out_turns < 0) return 0;
  return align_up(sizeof(int64_t) * (static_cast<size_t>(n_turns) + 1 + static_cast<size_t>(n_out_turns) + 1), 256);
}

opr_status opr_kpass_index(const int32_t* turn_lens, int32_t n_turns, const int32_t* out_turn_lens,
                           const int32_t* out_turn_src, int32_t n_out_turns, int64_t total_tokens, int64_t orig_tokens,
                           int32_t slots, int32_t* src_index, int32_t* copy_index, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream) {
  CallRange range("opr_kpass_index");
  if (n_turns < 0 || n_out_turns < 0 || total_tokens < 0 || orig_tokens < 0 || slots < 2 || slots > 64)
    return OPR_INVALID_ARG;
  if (total_tokens >= (int64_t{1} << 31)) return OPR_INVALID_ARG;
  if (!workspace || !dev_status || (n_turns > 0 && !turn_lens) || (n_out_turns > 0 && (!out_turn_lens || !out_turn_src)) ||
      (total_tokens > 0 && !src_index) || (orig_tokens > 0 && !copy_index))
    return OPR_INVALID_ARG;
  if (workspace_bytes < opr_kpass_index_workspace_bytes(n_turns, n_out_turns)) return OPR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) % 8 != 0) return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_kpass_index(turn_lens, n_turns, out_turn_lens, out_turn_src, n_out_turns, total_tokens,
                                      orig_tokens, slots, src_index, copy_index, static_cast<int64_t*>(workspace),
                                      dev_status, static_cast<cudaStream_t>(stream)));
}

int64_t opr_loss_row_count(const int32_t* turn_lens, int32_t n_turns) {
  if (n_turns < 0 || (n_turns > 0 && !turn_lens)) return -1;
  int64_t n = 0;
  for (int i = 0; i < n_turns; ++i) {
    const int64_t h = turn_lens[3 * i], t = turn_lens[3 * i + 1], r = turn_lens[3 * i + 2];
    if (h < 0 || t < 0 || r < 0) return -1;
    n += ((h > 0 && t + r > 0) ? 1 : 0) + (r > 0 ? t : (t > 0 ? t - 1 : 0)) + (r > 1 ? r - 1 : 0);
  }
  return n;
}

opr_status opr_loss_rows(const int32_t* turn_lens, int32_t n_turns, int64_t total_tokens, int64_t orig_tokens,
                         int64_t n_rows, int32_t* rows, int32_t* targets, int32_t* dev_status, void* stream) {
  CallRange range("opr_loss_rows");
  if (n_turns < 0 || total_tokens < 0 || orig_tokens < 0 || n_rows < 0) return OPR_INVALID_ARG;
  if (total_tokens >= (int64_t{1} << 31)) return OPR_INVALID_ARG;
  if (!dev_status || (n_turns > 0 && !turn_lens) || (n_rows > 0 && (!rows || !targets))) return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_loss_rows(turn_lens, n_turns, total_tokens, orig_tokens, n_rows, rows, targets, dev_status,
                                    static_cast<cudaStream_t>(stream)));
}

opr_status opr_cross_entropy(const void* logits, int32_t dtype, int64_t n_rows, int32_t vocab,
                             const int32_t* target_ids, float* loss, void* dlogits, float grad_scale,
                             int32_t* dev_status, void* stream) {
  CallRange range("opr_cross_entropy");
  if (n_rows < 0 || vocab <= 0 || n_rows >= (int64_t{1} << 31)) return OPR_INVALID_ARG;
  if (dtype != OPR_DTYPE_BF16 && dtype != OPR_DTYPE_FP32) return OPR_UNSUPPORTED;
  if (n_rows == 0) return OPR_OK;
  if (!logits || !target_ids || !loss || !dev_status) return OPR_INVALID_ARG;
  const opr_status st = device_check();
  if (st != OPR_OK) return st;
  return status_of(launch_cross_entropy(logits, dtype == OPR_DTYPE_BF16, n_rows, vocab, target_ids, loss, dlogits,
                                        grad_scale, dev_status, static_cast<cudaStream_t>(stream)));
}

const char* opr_version(void) {
#ifdef OPR_DEBUG_CHECKS
  return "opr 0.2.0 sm_100a debug-checks";
#else
  return "opr 0.2.0 sm_100a";
#endif
}

uint64_t opr_testing_set_wait_limit_ns(uint64_t limit_ns) { return g_wait_limit_ns.exchange(limit_ns); }

int opr_testing_layout_tables(int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                              int32_t max_seqlen, uint64_t offsets[4]) {
  if (offsets == nullptr || n_seqs < 0 || n_convs < 0 || n_turns < 0 || total_tokens < 0 || max_seqlen < 0)
    return OPR_INVALID_ARG;
  const LayoutWs w = layout_ws_map(n_seqs, n_convs, n_turns, total_tokens, max_seqlen);
  offsets[0] = w.row_cnt;
  offsets[1] = w.row_list;
  offsets[2] = w.col_cnt;
  offsets[3] = w.col_list;
  return OPR_OK;
}

const char* opr_last_error(void) { return g_cuda_error_text; }

size_t opr_layout_workspace_bytes(int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                                  int32_t max_seqlen) {
  if (!sizes_ok(n_seqs, n_convs, n_turns, total_tokens, max_seqlen)) return 0;
  return layout_ws_map(n_seqs, n_convs, n_turns, total_tokens, max_seqlen).bytes;
}

opr_status opr_build_layout(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                            int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                            int32_t max_seqlen, int32_t* cu_seqlens, int8_t* token_type, int32_t* turn_idx,
                            int32_t* conv_idx, int32_t* pos_id, int32_t* attn_pos, uint8_t* block_map,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  CallRange range("opr_build_layout");
  if (!sizes_ok(n_seqs, n_convs, n_turns, total_tokens, max_seqlen)) return OPR_INVALID_ARG;
  if (!conv_turn_ptr || !seq_conv_ptr || !cu_seqlens || !workspace || !dev_status) return OPR_INVALID_ARG;
  if (n_turns > 0 && !turn_lens) return OPR_INVALID_ARG;
  if (total_tokens > 0 && (!token_type || !turn_idx || !conv_idx || !pos_id || !attn_pos)) return OPR_INVALID_ARG;
  if (workspace_bytes < layout_ws_map(n_seqs, n_convs, n_turns, total_tokens, max_seqlen).bytes)
    return OPR_WORKSPACE_TOO_SMALL;
  cudaError_t e = launch_layout(turn_lens, conv_turn_ptr, seq_conv_ptr, n_seqs, n_convs, n_turns, total_tokens,
                                max_seqlen, cu_seqlens, token_type, turn_idx, conv_idx, pos_id, attn_pos, block_map,
                                workspace, dev_status, static_cast<cudaStream_t>(stream));
  return status_of(e);
}

opr_status opr_rope(const void* x, int32_t x_dtype, void* y, int32_t y_dtype, const int32_t* pos_id,
                    const int32_t* row_map, int64_t total_tokens, int32_t n_heads, int32_t head_dim, double base,
                    int32_t inverse, int32_t* dev_status, void* stream) {
  CallRange range("opr_rope");
  if (total_tokens < 0 || n_heads < 0 || head_dim <= 0 || head_dim % 2 != 0 || head_dim > 256) return OPR_INVALID_ARG;
  auto known = [](int32_t t) { return t == OPR_DTYPE_BF16 || t == OPR_DTYPE_FP16 || t == OPR_DTYPE_FP32; };
  if (!known(x_dtype) || !known(y_dtype)) return OPR_UNSUPPORTED;
  if (!(base > 1.0)) return OPR_INVALID_ARG;
  if (total_tokens > 0 && n_heads > 0 && (!x || !y)) return OPR_INVALID_ARG;
  if (x == y && (x_dtype != y_dtype || row_map != nullptr)) return OPR_INVALID_ARG;
  cudaError_t e = launch_rope(x, x_dtype, y, y_dtype, pos_id, row_map, total_tokens, n_heads, head_dim, base,
                              inverse, dev_status, static_cast<cudaStream_t>(stream));
  return status_of(e);
}

opr_status opr_attn_fwd(const void* q, const void* k, const void* v, int32_t qk_dtype, int32_t v_dtype,
                        const int32_t* cu_seqlens,
                        const int32_t* conv_idx, const void* layout_ws, int32_t n_seqs, int32_t n_convs,
                        int32_t n_turns, int64_t total_tokens, int32_t max_seqlen, int32_t hq, int32_t hkv,
                        int32_t head_dim, float scale, void* o, int32_t o_dtype, float* lse, int32_t* dev_status,
                        void* stream) {
  CallRange range("opr_attn_fwd");
  if (!sizes_ok(n_seqs, n_convs, n_turns, total_tokens, max_seqlen)) return OPR_INVALID_ARG;
  if (total_tokens == 0) return OPR_OK;
  if (!attn_args_ok(q, k, v, hq, hkv, head_dim, scale)) return OPR_INVALID_ARG;
  if (!cu_seqlens || !conv_idx || !layout_ws || !o || !lse || !dev_status || !aligned16(o)) return OPR_INVALID_ARG;
  if (o_dtype != OPR_DTYPE_BF16 && o_dtype != OPR_DTYPE_FP32) return OPR_UNSUPPORTED;
  if (qk_dtype != OPR_DTYPE_FP16) return OPR_UNSUPPORTED;
  if (v_dtype != OPR_DTYPE_FP16 && v_dtype != OPR_DTYPE_BF16) return OPR_UNSUPPORTED;
  const bool f16 = qk_dtype == OPR_DTYPE_FP16;
  const bool v16 = v_dtype == OPR_DTYPE_FP16;
  opr_status st = device_check();
  if (st != OPR_OK) return st;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, total_tokens, hq, head_dim, f16) || !make_map(&tk, k, total_tokens, hkv, head_dim, f16) ||
      !make_map(&tv, v, total_tokens, hkv, head_dim, v16))
    return map_fail();
  AttnParams p = base_params(cu_seqlens, conv_idx, layout_ws, n_seqs, n_convs, n_turns, total_tokens, max_seqlen, hq,
                             hkv, scale, dev_status);
  p.o = o;
  p.o_fp32 = o_dtype == OPR_DTYPE_FP32;
  p.lse = lse;
  cudaError_t e = launch_attn_fwd(head_dim, f16, v16, tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  return status_of(e);
}

namespace {
// The dK/dV stage runs one CTA per (key tile, kv head), each walking the whole
// column for every q head of its GQA group.  When that grid is short of a few
// waves of the 148 SMs, the longest columns set the stage's time; the stage is
// then split by q head (one CTA per key tile and q head, per-head partials summed
// afterwards), which needs room for the partials in the workspace.
constexpr int64_t kSplitGridCtas = 4 * 148;         // split below this many (key tile, kv head) CTAs
constexpr int64_t kSplitMaxHeadTiles = 4 * 148 * 8;  // partials reserved while tiles * hq stays at or below
// A key column is split when its whole-group walk (query tiles x group) reaches
// kSplitColumnRatio x T iterations; shorter columns stay whole (one CTA, no partials).
constexpr double kSplitColumnRatio = 2.0;

// Backward scratch: the row terms, then fp16 copies of dO and V (the minimum),
// then, for small problems, the per-q-head dK and dV partials of the split dK/dV
// stage.  Token counts are bounded by n_seqs * ceil(max_seqlen / 128) * 128 and
// the kv heads by hq.
struct BwdWs {
  size_t absmax, row_terms, dout16, v16, min_bytes, dk_part, dv_part, bytes;
};

BwdWs bwd_ws_map(int32_t n_seqs, int32_t max_seqlen, int32_t hq, int32_t head_dim) {
  const size_t T = (static_cast<size_t>(max_seqlen) + kTile - 1) / kTile;
  const size_t tiles = static_cast<size_t>(n_seqs) * T;
  const size_t tokens = tiles * kTile;
  BwdWs w;
  w.absmax = 0;
  w.row_terms = 256;
  w.dout16 = w.row_terms + align_up(2 * sizeof(float) * static_cast<size_t>(hq) * tokens, 256);
  const size_t copy = align_up(sizeof(uint16_t) * tokens * static_cast<size_t>(hq) * static_cast<size_t>(head_dim), 256);
  w.v16 = w.dout16 + copy;
  w.min_bytes = w.v16 + copy;
  const bool reserve = tiles * static_cast<size_t>(hq) <= static_cast<size_t>(kSplitMaxHeadTiles);
  const size_t part = reserve ? 2 * copy : 0;  // fp32 [hq][tokens][head_dim]
  w.dk_part = w.min_bytes;
  w.dv_part = w.dk_part + part;
  w.bytes = w.dv_part + part;
  return w;
}
}  // namespace

size_t opr_attn_bwd_workspace_bytes(int32_t n_seqs, int32_t max_seqlen, int32_t hq, int32_t head_dim) {
  if (n_seqs < 0 || max_seqlen < 0 || hq < 0 || head_dim < 0) return 0;
  return bwd_ws_map(n_seqs, max_seqlen, hq, head_dim).bytes;
}

size_t opr_attn_bwd_min_workspace_bytes(int32_t n_seqs, int32_t max_seqlen, int32_t hq, int32_t head_dim) {
  if (n_seqs < 0 || max_seqlen < 0 || hq < 0 || head_dim < 0) return 0;
  return bwd_ws_map(n_seqs, max_seqlen, hq, head_dim).min_bytes;
}

opr_status opr_attn_bwd_stages(const void* q, const void* k, const void* v, int32_t qk_dtype, const void* o,
                               int32_t o_dtype,
                               const void* dout, const float* lse, const int32_t* cu_seqlens,
                               const int32_t* conv_idx, const void* layout_ws, int32_t n_seqs, int32_t n_convs,
                               int32_t n_turns, int64_t total_tokens, int32_t max_seqlen, int32_t hq, int32_t hkv,
                               int32_t head_dim, float scale, float* dq, float* dk, float* dv,
                               const int32_t* rope_pos_id, double rope_base, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, int32_t stages, void* stream) {
  CallRange range("opr_attn_bwd_stages");
  if (!sizes_ok(n_seqs, n_convs, n_turns, total_tokens, max_seqlen)) return OPR_INVALID_ARG;
  if (stages & ~(OPR_BWD_ROW_TERMS | OPR_BWD_DQ | OPR_BWD_DKDV)) return OPR_INVALID_ARG;
  if (total_tokens == 0 || stages == 0) return OPR_OK;
  if (!attn_args_ok(q, k, v, hq, hkv, head_dim, scale)) return OPR_INVALID_ARG;
  if (!o || !dout || !lse || !cu_seqlens || !conv_idx || !layout_ws || !dq || !dk || !dv || !workspace ||
      !dev_status)
    return OPR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return OPR_INVALID_ARG;
  if (o_dtype != OPR_DTYPE_BF16 && o_dtype != OPR_DTYPE_FP32) return OPR_UNSUPPORTED;
  if (qk_dtype != OPR_DTYPE_FP16) return OPR_UNSUPPORTED;
  if (rope_pos_id != nullptr && !(rope_base > 1.0)) return OPR_INVALID_ARG;
  const bool f16 = qk_dtype == OPR_DTYPE_FP16;
  if (workspace_bytes < opr_attn_bwd_min_workspace_bytes(n_seqs, max_seqlen, hq, head_dim))
    return OPR_WORKSPACE_TOO_SMALL;
  opr_status st = device_check();
  if (st != OPR_OK) return st;
  const BwdWs bw = bwd_ws_map(n_seqs, max_seqlen, hq, head_dim);
  BwdBuffers buf;
  buf.dout_absmax = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + bw.absmax);
  buf.o = o;
  buf.o_fp32 = o_dtype == OPR_DTYPE_FP32;
  buf.dout = static_cast<const __nv_bfloat16*>(dout);
  buf.v = static_cast<const __nv_bfloat16*>(v);
  buf.row_terms = reinterpret_cast<float*>(static_cast<char*>(workspace) + bw.row_terms);
  buf.dout16 = reinterpret_cast<__half*>(static_cast<char*>(workspace) + bw.dout16);
  buf.v16 = reinterpret_cast<__half*>(static_cast<char*>(workspace) + bw.v16);
  buf.rope_pos = rope_pos_id;
  buf.rope_base = rope_base;
  BwdMaps maps;
  if (!make_map(&maps.q, q, total_tokens, hq, head_dim, f16) || !make_map(&maps.k, k, total_tokens, hkv, head_dim, f16) ||
      !make_map(&maps.v, v, total_tokens, hkv, head_dim) || !make_map(&maps.dout, dout, total_tokens, hq, head_dim) ||
      !make_map(&maps.v16, buf.v16, total_tokens, hkv, head_dim, true) ||
      !make_map(&maps.dout16, buf.dout16, total_tokens, hq, head_dim, true))
    return map_fail();
  const LayoutWs w = layout_ws_map(n_seqs, n_convs, n_turns, total_tokens, max_seqlen);
  AttnParams pq = base_params(cu_seqlens, conv_idx, layout_ws, n_seqs, n_convs, n_turns, total_tokens, max_seqlen,
                              hq, hkv, scale, dev_status);
  pq.lse_in = lse;
  pq.dout_absmax = buf.dout_absmax;
  pq.d_tiles = buf.row_terms;
  pq.lse2_tiles = pq.d_tiles + static_cast<size_t>(hq) * pq.n_items * kTile;
  pq.dq = dq;
  pq.dk = dk;
  pq.dv = dv;
  AttnParams pkv = pq;
  pkv.sched = ws_ptr<int32_t>(layout_ws, w.k_sched);
  // dK/dV split by q head: GQA, a grid short of kSplitGridCtas, and room for the partials
  pkv.dkdv_split = hq > hkv && static_cast<int64_t>(w.n_tiles) * hkv < kSplitGridCtas && bw.bytes > bw.min_bytes &&
                   workspace_bytes >= bw.bytes;
  if (pkv.dkdv_split) {
    const int group = hq / hkv;
    const double c = std::ceil(kSplitColumnRatio * w.T / group);
    pkv.split_min_cnt = c < 1.0 ? 1 : static_cast<int32_t>(c);
  }
  pkv.dk_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + bw.dk_part);
  pkv.dv_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + bw.dv_part);
  cudaError_t e = launch_attn_bwd(head_dim, f16, maps, buf, pq, pkv, stages, static_cast<cudaStream_t>(stream));
  return status_of(e);
}

opr_status opr_attn_bwd(const void* q, const void* k, const void* v, int32_t qk_dtype, const void* o,
                        int32_t o_dtype,
                        const void* dout, const float* lse, const int32_t* cu_seqlens, const int32_t* conv_idx,
                        const void* layout_ws, int32_t n_seqs, int32_t n_convs, int32_t n_turns,
                        int64_t total_tokens, int32_t max_seqlen, int32_t hq, int32_t hkv, int32_t head_dim,
                        float scale, float* dq, float* dk, float* dv, const int32_t* rope_pos_id, double rope_base,
                        void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return opr_attn_bwd_stages(q, k, v, qk_dtype, o, o_dtype, dout, lse, cu_seqlens, conv_idx, layout_ws, n_seqs, n_convs,
                             n_turns, total_tokens, max_seqlen, hq, hkv, head_dim, scale, dq, dk, dv, rope_pos_id,
                             rope_base, workspace, workspace_bytes, dev_status,
                             OPR_BWD_ROW_TERMS | OPR_BWD_DQ | OPR_BWD_DKDV, stream);
}

}  // extern "C"
