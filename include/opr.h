/*
 * opr.h - One-Pass to Reason masked attention on NVIDIA B200 (sm_100a).
 *
 * C ABI of libopr.so.  The operation is the attention layer of
 * "One-Pass to Reason: Token Duplication and Block-Sparse Mask for Efficient
 * Fine-Tuning on Multi-Turn Reasoning" (Goru, Mehta, Jain): every turn i of a
 * conversation is packed as h_i, t_i, r_i^in, r_i^out (the response r_i is
 * stored twice), and attention follows per-type visibility rules so that one
 * pass over the conversation gives the same rows as N causal passes.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Array arguments are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or retains device memory; it keeps no state
 *    between calls except cached kernel attributes and the driver entry point
 *    used to encode TMA descriptors.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream).  The return value reports host-side
 *    argument checks and launch errors only.
 *  - Errors found on the device (inconsistent sizes, a pipeline wait that
 *    timed out) are OR-ed as OPR_DEV_* bits into the caller's int32
 *    `dev_status` word, which the caller zeroes before the first call and
 *    reads after synchronising.  No call aborts, traps or throws.
 *  - Token-major tensors are [total_tokens, heads, head_dim], contiguous,
 *    sequences packed back to back (offsets in cu_seqlens).  LSE and the
 *    backward's row terms are [heads, total_tokens].
 *  - Token types: 0 = h (human message), 1 = t (reasoning), 2 = r^in (response,
 *    context copy), 3 = r^out (response, generation copy).
 */
#ifndef OPR_H_
#define OPR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define OPR_API __attribute__((visibility("default")))
#else
#define OPR_API
#endif

typedef int32_t opr_status;

#define OPR_OK 0
#define OPR_INVALID_ARG 1          /* null pointer, negative size, Hq % Hkv != 0, bad head_dim ... */
#define OPR_UNSUPPORTED 2          /* dtype or device (needs compute capability 10.0) not supported */
#define OPR_CUDA_ERROR 3           /* a CUDA runtime/driver call or a kernel launch failed */
#define OPR_WORKSPACE_TOO_SMALL 4  /* workspace_bytes below what the *_workspace_bytes query returns */
#define OPR_SCRATCH_TOO_LARGE 5    /* opr_attn_bwd_noalloc: scratch needed exceeds OPR_NOALLOC_SCRATCH_BYTES */

/* Bits OR-ed into *dev_status by the kernels. */
#define OPR_DEV_BAD_INPUT 1        /* negative length or non-monotone turn/conversation pointers */
#define OPR_DEV_TOTAL_MISMATCH 2   /* sum of h + t + 2r differs from total_tokens */
#define OPR_DEV_SEQ_TOO_LONG 4     /* a sequence is longer than max_seqlen */
#define OPR_DEV_WAIT_TIMEOUT 8     /* a pipeline wait exceeded its time limit; outputs are invalid */
#define OPR_DEV_FP16_RANGE 16      /* an fp16 value beyond +-65504 was written (opr_rope output, or the
                                      backward's fp16 copies of the scaled dO and of v) */
#define OPR_DEV_BOUNDS 32          /* debug library (libopr_debug.so, built with OPR_DEBUG_CHECKS) only:
                                      an index an attention kernel takes from the layout tables (tile id,
                                      sequence bounds, tile-list length or entry) is out of range; the
                                      kernel's CTA for that tile skipped all of its work, so the outputs
                                      are invalid.  Release builds do not check and never set it. */

#define OPR_DTYPE_BF16 0
#define OPR_DTYPE_FP32 1
#define OPR_DTYPE_FP16 2

#define OPR_TILE 128               /* edge of a block-map tile, in tokens */
#define OPR_TILE_EMPTY 0           /* block-map classes (bits 0-1 of a block-map byte) */
#define OPR_TILE_FULL 1
#define OPR_TILE_PARTIAL 2
#define OPR_TILE_KEY_HALF0 4       /* bits 2-3: a query of the tile sees a key of half 0 / half 1 */
#define OPR_TILE_KEY_HALF1 8

/*
 * Bytes of the layout workspace that opr_build_layout fills and the attention
 * calls read (per-tile lists of non-empty tiles, packed per-token type/turn,
 * per-turn offsets and the tile schedule).  Depends only on the sizes.
 */
OPR_API size_t opr_layout_workspace_bytes(int32_t n_seqs, int32_t n_convs, int32_t n_turns,
                                  int64_t total_tokens, int32_t max_seqlen);

/*
 * opr_build_layout - token duplication, position ids and the block map.
 *
 * Defined by the One-Pass to Reason wiki note: "Token 复制" (r_i stored as
 * r_i^in and r_i^out), "位置 ID 策略" (s_t = s_rin = e_h + 1, s_rout = e_t + 1,
 * s_h(i+1) = e_rin + 1; the first position of every conversation is 0) and
 * "分块稀疏注意力掩码" (h_i sees H<i; t_i and r_i^in see H<i and h_i; r_i^out
 * sees H<i, h_i and t_i; H<i = {h_j, r_j^in : j < i}; every segment causal
 * within itself; conversations packed in one sequence never see each other).
 *
 * Inputs (device):
 *   turn_lens      int32 [n_turns][3]  (h, t, r) of each turn, each >= 0
 *   conv_turn_ptr  int32 [n_convs+1]   turns of conversation c are
 *                                      conv_turn_ptr[c] .. conv_turn_ptr[c+1]-1
 *   seq_conv_ptr   int32 [n_seqs+1]    conversations of sequence s
 *   total_tokens   sum over turns of h + t + 2r (host value, checked on device)
 *   max_seqlen     an upper bound of every sequence's length (host value)
 * Outputs (device, caller-allocated):
 *   cu_seqlens     int32 [n_seqs+1]    token offset of each sequence
 *   token_type     int8  [total]       0 h, 1 t, 2 r^in, 3 r^out
 *   turn_idx       int32 [total]       turn index within the conversation (0-based)
 *   conv_idx       int32 [total]       global conversation index
 *   pos_id         int32 [total]       position id
 *   attn_pos       int32 [total]       the token's row in the attention order, the
 *                  order of the q, k and v rows that opr_attn_fwd and opr_attn_bwd
 *                  take (opr_rope writes them there with row_map = attn_pos).  Per
 *                  conversation: the context tokens h_1 r_1^in ... h_N r_N^in, then
 *                  the trained tokens t_1 r_1^out ... t_N r_N^out, each segment in
 *                  stream order, inside the conversation's own rows.  The mask is the
 *                  same in both orders (every visible key comes before its query in
 *                  both), but the context part is one causal block and the trained
 *                  part a staircase, so far fewer 128 x 128 tiles are partly visible
 *                  (a storage choice of this library; the pages state the segments,
 *                  "Token 复制", and pack them, "实现细节")
 *   block_map      NULL, or uint8 [n_seqs][T][T], T = ceil(max_seqlen / 128), in the
 *                  stream order (the attention calls use their own, internal block
 *                  map of the attention order).  Bits 0-1
 *                  of the byte of tile (I, J) of sequence s: 0 empty, 1 full
 *                  (all 128 x 128 pairs visible), 2 partial; indices past the
 *                  sequence count as not visible, so tail tiles are never full.
 *                  Bits 2-3: bit 2 + h set when some query of the tile sees a
 *                  key of its half h (keys 64 h .. 64 h + 63); the dQ kernel,
 *                  from the same bits of its internal map, skips the half that
 *                  no query of a tile sees
 *   workspace      opr_layout_workspace_bytes(...) bytes, read by the attention calls
 *   dev_status     int32 word, OPR_DEV_* bits OR-ed in on inconsistent input
 * Returns OPR_INVALID_ARG for null pointers / negative sizes / n_seqs > n_convs
 * inconsistencies detectable on the host, OPR_WORKSPACE_TOO_SMALL, OPR_CUDA_ERROR.
 */
OPR_API opr_status opr_build_layout(const int32_t* turn_lens, const int32_t* conv_turn_ptr,
                            const int32_t* seq_conv_ptr, int32_t n_seqs, int32_t n_convs,
                            int32_t n_turns, int64_t total_tokens, int32_t max_seqlen,
                            int32_t* cu_seqlens, int8_t* token_type, int32_t* turn_idx,
                            int32_t* conv_idx, int32_t* pos_id, int32_t* attn_pos, uint8_t* block_map,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream);

/*
 * opr_rope - rotary position embedding by position id.
 *
 * The pages' position-equivalence argument ("理论保证") is about the rotary
 * positions of Qwen-3 (rotate-half convention): for j < head_dim/2 the pair
 * (x[j], x[j + head_dim/2]) is rotated by angle pos_id * base^(-2j/head_dim)
 * (by -angle when `inverse` != 0, which maps gradients w.r.t. rotated values
 * back to gradients w.r.t. the unrotated ones).  Angles are formed in fp64,
 * the rotation in fp32, the result rounded once to y's type.
 *   x, y     [total_tokens, n_heads, head_dim]; x_dtype, y_dtype each one of
 *            OPR_DTYPE_BF16 / OPR_DTYPE_FP16 / OPR_DTYPE_FP32.  y may equal x
 *            (in place) only when the two types are the same.
 *   pos_id   int32 [total_tokens]; NULL: no rotation, only the type conversion
 *            (e.g. the fp16 copy of v that opr_attn_fwd takes for an fp16 P V
 *            product)
 *   row_map  NULL (row t of y is row t of x), or int32 [total_tokens]: row t of x
 *            is written to row row_map[t] of y (opr_build_layout's attn_pos puts
 *            q, k and v in the attention order); y must not be x
 *   dev_status  may be NULL; otherwise OPR_DEV_FP16_RANGE is OR-ed in when an
 *            fp16 output overflows (an inf or NaN input included).
 * head_dim must be even and <= 256.  The attention calls take the rotated q
 * and k in fp16 (bf16 in, fp16 out here): same MMA rate as bf16, 8x smaller
 * rounding of the rotation.
 */
OPR_API opr_status opr_rope(const void* x, int32_t x_dtype, void* y, int32_t y_dtype,
                            const int32_t* pos_id, const int32_t* row_map, int64_t total_tokens, int32_t n_heads,
                            int32_t head_dim, double base, int32_t inverse, int32_t* dev_status,
                            void* stream);

/*
 * opr_attn_fwd - block-sparse masked attention forward (tcgen05 / TMEM / TMA).
 *
 * Defined by the One-Pass to Reason wiki note, "分块稀疏注意力掩码" (one mask
 * over the packed conversation: h_i sees H<i; t_i and r_i^in see H<i and h_i;
 * r_i^out sees H<i, h_i and t_i; every segment causal within itself) and
 * "实现细节" (the mask applied block-sparsely inside attention, with sequence
 * packing); the English note's "Method" (items 1-2) states the same rules.
 * The attention itself is softmax attention restricted to the visible keys:
 * O = softmax(scale * Q K^T restricted to visible keys) V for each q head;
 * q head h reads kv head h / (hq / hkv).  Tiles marked empty in the block map
 * are skipped, the visibility predicate is evaluated only on partial tiles.
 *   q            fp16 [total, hq, head_dim]   rotated, rows in the attention order
 *                (opr_rope with row_map = opr_build_layout's attn_pos)
 *   k            fp16 [total, hkv, head_dim]  rotated, attention order
 *   qk_dtype     OPR_DTYPE_FP16 (the type of the S = Q K^T MMA); any other
 *                value returns OPR_UNSUPPORTED
 *   v            [total, hkv, head_dim] in the attention order, v_dtype
 *                OPR_DTYPE_FP16 or OPR_DTYPE_BF16:
 *                the type of the O += P V MMA, whose P is rounded to the same
 *                type.  fp16 (v copied by opr_rope with no position ids) keeps
 *                P to 11 bits: O, and D = rowsum(dO * O) in the backward, are
 *                then about 8x closer to exact than with bf16 P.
 *   cu_seqlens, conv_idx, layout_ws: outputs of opr_build_layout for the same sizes
 *   o            [total, hq, head_dim] in the stream order (row = stream token),
 *                o_dtype OPR_DTYPE_BF16 or OPR_DTYPE_FP32
 *   lse          fp32 [hq, total], stream order: natural-log sum of exp(scale * q.k)
 *                over visible keys
 * head_dim must be 64 or 128; all pointers 16-byte aligned; total_tokens at
 * most n_seqs * ceil(max_seqlen / 128) * 128 (else OPR_INVALID_ARG).  All
 * buffers are the caller's; the call reads q, k, v and the layout and writes
 * o and lse only.  Errors: OPR_INVALID_ARG, OPR_UNSUPPORTED, OPR_CUDA_ERROR
 * (text from opr_last_error); OPR_DEV_WAIT_TIMEOUT in *dev_status.
 */
OPR_API opr_status opr_attn_fwd(const void* q, const void* k, const void* v, int32_t qk_dtype,
                        int32_t v_dtype, const int32_t* cu_seqlens,
                        const int32_t* conv_idx, const void* layout_ws, int32_t n_seqs,
                        int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                        int32_t max_seqlen, int32_t hq, int32_t hkv, int32_t head_dim,
                        float scale, void* o, int32_t o_dtype, float* lse, int32_t* dev_status,
                        void* stream);

/*
 * Bytes of device scratch for opr_attn_bwd.  With N = n_seqs * ceil(max_seqlen
 * / 128) * 128 (a bound on the token count) and n_tiles = N / 128:
 *   opr_attn_bwd_min_workspace_bytes, the least a call accepts:
 *     256 bytes for max |dO| (which sets the gradient scale below);
 *     the row terms D = rowsum(dO * O) and LSE * log2(e), stored per 128-token
 *     tile: 2 * 4 * hq * N bytes;
 *     an fp16 copy of dO: 2 * N * hq * head_dim bytes;
 *     an fp16 copy of v (kv heads bounded by hq): 2 * N * hq * head_dim bytes;
 *   opr_attn_bwd_workspace_bytes, the recommended size: the minimum, plus, when
 *     n_tiles * hq <= 4736, room for per-q-head fp32 dK and dV partials
 *     (2 * 4 * N * hq * head_dim bytes).  With it, a call whose dK/dV grid
 *     (n_tiles * hkv CTAs) is below 4 * 148 and that has more q heads than kv
 *     heads splits the long key columns of the dK/dV stage by q head: a column
 *     seen by at least 2 * T / (hq / hkv) query tiles (T = max_seqlen / 128,
 *     rounded up) gets one CTA per q head, and a pass sums each group's partials
 *     in head order; shorter columns keep one CTA for the group.  Short grids
 *     (short or few sequences) are otherwise bound by their longest key column.
 *     The two forms differ in the order of the group sum, within fp32 rounding;
 *     each is deterministic.
 * each part rounded up to 256 bytes.  Both return 0 for negative arguments.
 */
OPR_API size_t opr_attn_bwd_workspace_bytes(int32_t n_seqs, int32_t max_seqlen, int32_t hq,
                                            int32_t head_dim);
OPR_API size_t opr_attn_bwd_min_workspace_bytes(int32_t n_seqs, int32_t max_seqlen, int32_t hq,
                                                int32_t head_dim);

/*
 * opr_attn_bwd - gradients of opr_attn_fwd w.r.t. q, k (rotated, or unrotated
 * with rope_pos_id) and v.
 *
 * The pages fine-tune through this layer (wiki note, "理论保证": the one-pass
 * loss equals the N-pass loss, so its gradients are the N-pass gradients;
 * the mask is that of "分块稀疏注意力掩码").  These are the analytic gradients
 * of softmax attention under that mask.  With P recomputed from LSE:
 * D = rowsum(dO * O), dV = P^T dO, dS = P * (dO V^T - D), dQ = scale dS K,
 * dK = scale dS^T Q; dK and dV sum over the q heads that share a kv head.
 * Deterministic (no atomics).
 *   q, k              as in opr_attn_fwd (fp16, rotated, attention order)
 *   v                 bf16 [total, hkv, head_dim], stream order
 *   o, dout           stream order, o in o_dtype, dout bf16 [total, hq, head_dim]
 *   lse               fp32 [hq, total] from opr_attn_fwd (stream order)
 *   dq                fp32 [total, hq, head_dim], stream order
 *   dk, dv            fp32 [total, hkv, head_dim], stream order
 *   rope_pos_id       NULL: dq and dk are the gradients w.r.t. the rotated q and k
 *                     given.  Otherwise int32 [total] position ids (those q and k
 *                     were rotated by, e.g. opr_build_layout's pos_id) and
 *                     rope_base > 1 their base: the call rotates dq and dk back
 *                     (one pass over each, right after the kernel that writes it),
 *                     giving the gradients w.r.t. the unrotated q and k, exactly
 *                     as opr_rope(inverse) on the first form
 *   workspace         at least opr_attn_bwd_min_workspace_bytes(...) bytes of device
 *                     scratch (opr_attn_bwd_workspace_bytes(...) recommended),
 *                     16-byte aligned, owned by the caller; the call overwrites it
 * Precision: the tensor-core products take 16-bit operands.  The backward is
 * linear in dO, so it runs on 2^k dO, with k chosen on the device from max |dO|
 * so that max |2^k dO| lies in [8, 16), and divides dq, dk, dv by 2^k (exact).
 * The fp16 copy of 2^k dO and the fp16 dS therefore keep 11 significant bits
 * at any gradient magnitude (a loss divided by the token count, passed back
 * through later layers, is often 1e-5 .. 1e-8).  v is copied to fp16 as it is:
 * a |v| beyond 65504, or an inf or NaN in dO, sets OPR_DEV_FP16_RANGE in
 * *dev_status (the results are then invalid).  Other errors as opr_attn_fwd.
 */
OPR_API opr_status opr_attn_bwd(const void* q, const void* k, const void* v, int32_t qk_dtype,
                        const void* o, int32_t o_dtype, const void* dout, const float* lse,
                        const int32_t* cu_seqlens, const int32_t* conv_idx, const void* layout_ws,
                        int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                        int32_t max_seqlen, int32_t hq, int32_t hkv, int32_t head_dim,
                        float scale, float* dq, float* dk, float* dv, const int32_t* rope_pos_id,
                        double rope_base, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, void* stream);

/*
 * opr_attn_bwd_stages - the same computation as opr_attn_bwd, split into its
 * three kernels so that a caller can order, overlap or time them one by one.
 * `stages` is an OR of:
 *   OPR_BWD_ROW_TERMS  max |dO|, D = rowsum(dO * O) and the fp16 copies of dO
 *                      and v into `workspace` (needed by the other two)
 *   OPR_BWD_DQ         dq   (one CTA per query tile and q head; then, with
 *                      rope_pos_id, the rotation of dq back)
 *   OPR_BWD_DKDV       dk, dv (one CTA per key tile and kv head, GQA group summed
 *                      in the CTA; or, split as opr_attn_bwd_workspace_bytes says,
 *                      one CTA per key tile and q head and a group-sum pass; then,
 *                      with rope_pos_id, the rotation of dk back)
 * Running all three, in this order on one stream, equals opr_attn_bwd.
 * Other arguments and error behaviour as for opr_attn_bwd; unknown bits give
 * OPR_INVALID_ARG.
 */
#define OPR_BWD_ROW_TERMS 1
#define OPR_BWD_DQ 2
#define OPR_BWD_DKDV 4
OPR_API opr_status opr_attn_bwd_stages(const void* q, const void* k, const void* v,
                                       int32_t qk_dtype, const void* o, int32_t o_dtype, const void* dout, const float* lse,
                                       const int32_t* cu_seqlens, const int32_t* conv_idx,
                                       const void* layout_ws, int32_t n_seqs, int32_t n_convs,
                                       int32_t n_turns, int64_t total_tokens, int32_t max_seqlen,
                                       int32_t hq, int32_t hkv, int32_t head_dim, float scale, float* dq,
                                       float* dk, float* dv, const int32_t* rope_pos_id, double rope_base,
                                       void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                       int32_t stages, void* stream);

/*
 * opr_attn_bwd_noalloc - opr_attn_bwd for callers that cannot allocate device
 * memory at the call (no counterpart in the paper; a convenience of this
 * library).  Examples: a host framework that owns every device allocation and
 * offers extensions no allocator hook, or a latency-critical path that must
 * not call cudaMalloc, which can block and synchronize the device.
 *
 * Same inputs, outputs and error behaviour as opr_attn_bwd, without the
 * workspace arguments: the scratch (max |dO|, the row terms and the fp16
 * copies of dO and v) lives in one fixed
 * library-owned device array of OPR_NOALLOC_SCRATCH_BYTES, allocated by the
 * CUDA loader on every GPU that loads the library and held until the process
 * exits.  The call allocates and frees nothing.
 *   - Returns OPR_SCRATCH_TOO_LARGE, before touching the device, when
 *     opr_attn_bwd_min_workspace_bytes(n_seqs, max_seqlen, hq, head_dim) exceeds
 *     OPR_NOALLOC_SCRATCH_BYTES.  The dK/dV stage is split by q head (as in
 *     opr_attn_bwd) only when opr_attn_bwd_workspace_bytes(...) fits too.
 *   - The array is the current device's: `stream` and every pointer must
 *     belong to the device that is current on the calling thread.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents in
 *     it; each call clears (max |dO|) or rewrites every entry it reads.  Calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on the array: order them on one stream.
 */
#define OPR_NOALLOC_SCRATCH_BYTES (32u << 20)
OPR_API opr_status opr_attn_bwd_noalloc(const void* q, const void* k, const void* v, int32_t qk_dtype,
                                        const void* o, int32_t o_dtype, const void* dout,
                                        const float* lse, const int32_t* cu_seqlens,
                                        const int32_t* conv_idx, const void* layout_ws, int32_t n_seqs,
                                        int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                                        int32_t max_seqlen, int32_t hq, int32_t hkv, int32_t head_dim,
                                        float scale, float* dq, float* dk, float* dv,
                                        const int32_t* rope_pos_id, double rope_base,
                                        int32_t* dev_status, void* stream);

/* Library version string, e.g. "opr 0.1.0 sm_100a". */
/*
 * Token duplication, the step before the attention layer (One-Pass to Reason
 * wiki note, "Token 复制"): the one-pass stream of a turn is h, t, r^in,
 * r^out, the original stream h, t, r, and conversations follow each other in
 * index order in both.  The map is what a fine-tuning pipeline needs to build
 * the one-pass input (token ids, or embeddings) from the original one and to
 * take the gradient back.
 *
 * opr_duplication_index - the map between the two streams.
 *   turn_lens       int32 [n_turns][3] (h, t, r), device, as for opr_build_layout
 *   conv_turn_ptr   int32 [n_convs + 1], device
 *   total_tokens    one-pass tokens, sum of h + t + 2r
 *   orig_tokens     original tokens, sum of h + t + r
 *   src_index       int32 [total_tokens] out: the original token each one-pass token copies
 *   copy_index      int32 [orig_tokens][2] out: the one-pass positions of each original
 *                   token; [o][1] = -1 for h and t tokens, the r^out copy for r tokens
 *   dev_status      required; OPR_DEV_BAD_INPUT for a negative length or a conversation
 *                   pointer that does not span the turns, OPR_DEV_TOTAL_MISMATCH when a
 *                   total disagrees with the lengths (then only in-range entries are written)
 * One thread block on `stream`.  OPR_INVALID_ARG for negative sizes or null pointers.
 */
OPR_API opr_status opr_duplication_index(const int32_t* turn_lens, const int32_t* conv_turn_ptr,
                                         int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                                         int64_t orig_tokens, int32_t* src_index, int32_t* copy_index,
                                         int32_t* dev_status, void* stream);

/*
 * opr_gather_rows - y[i] = x[src_index[i]] for i < total_tokens, rows of row_bytes bytes
 * (token ids, embeddings, hidden states: any fixed-width row; 16-byte aligned
 * tensors with row_bytes % 16 == 0 take 16-byte accesses).
 *   x  [orig_tokens] rows, device;  y  [total_tokens] rows, device, caller-owned
 *   dev_status  may be NULL; otherwise OPR_DEV_BAD_INPUT when an index is out of range
 *               (that row is left unwritten)
 */
OPR_API opr_status opr_gather_rows(const void* x, int64_t orig_tokens, int64_t row_bytes,
                                   const int32_t* src_index, int64_t total_tokens, void* y,
                                   int32_t* dev_status, void* stream);

/*
 * opr_fold_rows - the gradient of opr_gather_rows w.r.t. x, fp32 rows of `width` values:
 * dx[o] = sum of dy[copy_index[o][k]] over the slots k < slots with copy_index[o][k] >= 0, added
 * in slot order (copy_index from opr_duplication_index has 2 slots, from opr_kpass_index K + 1).
 * No atomics; deterministic.
 *   dy  fp32 [total_tokens][width];  dx  fp32 [orig_tokens][width], caller-owned
 *   dev_status  may be NULL; otherwise OPR_DEV_BAD_INPUT for an out-of-range index or a row
 *               without any copy (left unwritten)
 */
OPR_API opr_status opr_fold_rows(const float* dy, int64_t total_tokens, int64_t width,
                                 const int32_t* copy_index, int32_t slots, int64_t orig_tokens,
                                 float* dx, int32_t* dev_status, void* stream);

/*
 * K-pass, between N-pass (K = N) and one-pass (K = 1) (wiki note, "K-Pass 中间方案": a
 * speed / memory trade-off).  The pages give only the trade-off; the reading built here:
 * a conversation's N turns fall into K' = min(K, N) contiguous groups with bounds
 * b_g = floor(g N / K'); pass g is one conversation holding the history of the turns
 * before the group, each turn j as the single context segment (h_j + r_j, 0, 0) (h_j
 * then r_j, positions running on, as h_j and r_j^in in one pass), then the group's own
 * turns (h, t, r).  Every t and r^out row lies in exactly one pass, and the output is an
 * ordinary input of opr_build_layout, so the attention calls serve every K unchanged.
 *
 * opr_kpass_sizes - the sizes of the K-pass arrangement, from HOST copies of the one-pass
 * layout inputs (what a caller needs to allocate the outputs of opr_kpass_plan and
 * opr_kpass_index and the buffers of the attention calls that follow):
 *   turn_lens, conv_turn_ptr, seq_conv_ptr  host arrays, as for opr_build_layout
 *   n_out_turns, n_out_convs   turns and conversations (passes) of the arrangement
 *   total_tokens               its one-pass tokens, sum of h + t + 2r over the output turns
 *   max_seqlen                 its longest sequence (the passes of a conversation stay in
 *                              the conversation's sequence)
 *   orig_tokens                tokens of the original stream, sum of h + t + r
 * Returns OPR_INVALID_ARG for null pointers, K < 1, negative lengths, pointers that do not
 * span the turns and conversations, or sizes beyond int32 token offsets.
 */
OPR_API opr_status opr_kpass_sizes(const int32_t* turn_lens, const int32_t* conv_turn_ptr,
                                   const int32_t* seq_conv_ptr, int32_t n_seqs, int32_t n_convs,
                                   int32_t n_turns, int32_t K, int64_t* n_out_turns,
                                   int64_t* n_out_convs, int64_t* total_tokens, int64_t* max_seqlen,
                                   int64_t* orig_tokens);

/*
 * opr_kpass_plan - the K-pass arrangement as layout inputs (device arrays).
 *   turn_lens, conv_turn_ptr, seq_conv_ptr  the one-pass inputs, as for opr_build_layout
 *   n_out_turns, n_out_convs               from opr_kpass_sizes
 *   out_turn_lens      int32 [n_out_turns][3]; out_conv_turn_ptr int32 [n_out_convs + 1];
 *   out_seq_conv_ptr   int32 [n_seqs + 1] (the passes of a conversation stay in its sequence)
 *   out_turn_src       int32 [n_out_turns][2]: (original turn, d) with d = -1 for a turn of
 *                      the pass's own group and d >= 1 for a history turn d groups before
 *   dev_status         required; OPR_DEV_BAD_INPUT, OPR_DEV_TOTAL_MISMATCH (sizes disagree)
 * One thread block on `stream`.
 */
OPR_API opr_status opr_kpass_plan(const int32_t* turn_lens, const int32_t* conv_turn_ptr,
                                  const int32_t* seq_conv_ptr, int32_t n_seqs, int32_t n_convs,
                                  int32_t n_turns, int32_t K, int32_t n_out_turns, int32_t n_out_convs,
                                  int32_t* out_turn_lens, int32_t* out_conv_turn_ptr,
                                  int32_t* out_seq_conv_ptr, int32_t* out_turn_src, int32_t* dev_status,
                                  void* stream);

/* Bytes of device scratch (8-byte aligned) that opr_kpass_index needs: two turn-offset arrays. */
OPR_API size_t opr_kpass_index_workspace_bytes(int32_t n_turns, int32_t n_out_turns);

/*
 * opr_kpass_index - the token map between the original stream (h, t, r per turn) and the
 * K-pass stream of opr_kpass_plan's arrangement.
 *   total_tokens   K-pass tokens (sum of h + t + 2r over the output turns)
 *   orig_tokens    original tokens (sum of h + t + r over the input turns)
 *   slots          K + 1 (or more)
 *   src_index      int32 [total_tokens] out: the original token each K-pass token copies
 *   copy_index     int32 [orig_tokens][slots] out: slot 0 the copy in the token's own pass
 *                  (h, t or r^in), 1 the r^out copy, 1 + d the history copy d groups later;
 *                  -1 where there is none (the call clears it first)
 *   workspace      opr_kpass_index_workspace_bytes(n_turns, n_out_turns) bytes, caller-owned
 * Fold gradients with opr_fold_rows(..., copy_index, slots, ...).
 */
OPR_API opr_status opr_kpass_index(const int32_t* turn_lens, int32_t n_turns, const int32_t* out_turn_lens,
                                   const int32_t* out_turn_src, int32_t n_out_turns, int64_t total_tokens,
                                   int64_t orig_tokens, int32_t slots, int32_t* src_index,
                                   int32_t* copy_index, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, void* stream);

/*
 * The loss side, the step after the attention layer.  The pages prove that the one-pass
 * loss equals the N-pass loss ("理论保证") and train on the r^out copies ("Token 复制").
 * In N-pass run i the losses are the next-token predictions of t_i and r_i: from the last
 * h_i row (target: the first t_i token, or r_i[0] when t_i is empty), from each t_i row
 * (target: the next t_i token, or r_i[0] after the last) and from each r_i row but the last
 * (target: the next r_i token).  In one pass those rows are the last h_i row, the t_i rows
 * and the r_i^out rows.  (When h_i is empty the first assistant token has no loss row.)
 *
 * opr_loss_row_count - number of such rows, from HOST turn lengths; -1 for bad input.
 */
OPR_API int64_t opr_loss_row_count(const int32_t* turn_lens, int32_t n_turns);

/*
 * opr_loss_rows - the loss rows, in one-pass stream order, and the original-stream index of
 * each row's target token (the original stream holds h, t, r once per turn, conversations in
 * index order; a token id array of that stream gives the target ids).
 *   turn_lens     int32 [n_turns][3], device
 *   total_tokens  one-pass tokens; orig_tokens original tokens; n_rows from opr_loss_row_count
 *   rows, targets int32 [n_rows] out
 *   dev_status    required; OPR_DEV_BAD_INPUT, OPR_DEV_TOTAL_MISMATCH (sizes disagree)
 * One thread block on `stream`.
 */
OPR_API opr_status opr_loss_rows(const int32_t* turn_lens, int32_t n_turns, int64_t total_tokens,
                                 int64_t orig_tokens, int64_t n_rows, int32_t* rows, int32_t* targets,
                                 int32_t* dev_status, void* stream);

/*
 * opr_cross_entropy - softmax cross-entropy of n_rows rows of logits, fused with its gradient:
 * loss[i] = logsumexp(z_i) - z_i[target_ids[i]], and when dlogits is not NULL
 * dlogits[i] = grad_scale * (softmax(z_i) - onehot(target_ids[i])).  fp32 arithmetic.
 *   logits    [n_rows][vocab], dtype OPR_DTYPE_BF16 or OPR_DTYPE_FP32, device
 *   target_ids int32 [n_rows]; a negative id marks a row to ignore (loss 0, gradient 0);
 *             an id >= vocab sets OPR_DEV_BAD_INPUT and is ignored the same way
 *   loss      fp32 [n_rows] out;  dlogits  [n_rows][vocab] in the logits' dtype, or NULL
 * One CTA per row.
 */
OPR_API opr_status opr_cross_entropy(const void* logits, int32_t dtype, int64_t n_rows, int32_t vocab,
                                     const int32_t* target_ids, float* loss, void* dlogits,
                                     float grad_scale, int32_t* dev_status, void* stream);

OPR_API const char* opr_version(void);

/*
 * Text of the CUDA error behind the last OPR_CUDA_ERROR that an entry point
 * returned on the calling host thread ("no error" before any).  The string
 * is static; the caller does not free it.
 */
OPR_API const char* opr_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* OPR_H_ */
