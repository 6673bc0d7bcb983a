// layout.cu - token duplication, position ids, block map and tile lists.
//
// One-Pass to Reason wiki note: "Token 复制" (each response r_i stored as
// r_i^in and r_i^out), "位置 ID 策略" (s_t = s_rin = e_h + 1, s_rout = e_t + 1,
// s_h(i+1) = e_rin + 1), "分块稀疏注意力掩码" (per-type visibility) and
// "实现细节" (mask built on the GPU, vectorised, with simplified Boolean logic;
// sequence packing).  Segment order inside a turn: h, t, r^in, r^out.
#include <cuda_runtime.h>

#include "opr_internal.cuh"

namespace opr {
namespace {

// One thread per conversation: walk its turns, record each turn's first
// position id (cursor p), its token offset inside the conversation, the
// conversation's token count (h + t + 2r per turn) and its count of context
// tokens (h + r^in per turn, which is also the final cursor p).
__global__ void conv_walk_kernel(const int32_t* __restrict__ turn_lens, const int32_t* __restrict__ conv_turn_ptr,
                                 int32_t n_convs, int32_t n_turns, int64_t* __restrict__ conv_tokens,
                                 int64_t* __restrict__ turn_off, int32_t* __restrict__ turn_pos0,
                                 int32_t* __restrict__ turn_conv, int32_t* __restrict__ conv_ctx,
                                 int32_t* __restrict__ dev_status) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n_convs) return;
  const int t0 = conv_turn_ptr[c], t1 = conv_turn_ptr[c + 1];
  if (t0 < 0 || t1 < t0 || t1 > n_turns) {
    atomicOr(dev_status, OPR_DEV_BAD_INPUT);
    conv_tokens[c] = 0;
    conv_ctx[c] = 0;
    return;
  }
  int64_t off = 0;
  int64_t p = 0;
  for (int t = t0; t < t1; ++t) {
    int h = turn_lens[3 * t], tt = turn_lens[3 * t + 1], r = turn_lens[3 * t + 2];
    if (h < 0 || tt < 0 || r < 0) {
      atomicOr(dev_status, OPR_DEV_BAD_INPUT);
      h = h < 0 ? 0 : h;
      tt = tt < 0 ? 0 : tt;
      r = r < 0 ? 0 : r;
    }
    turn_pos0[t] = static_cast<int32_t>(p);
    turn_off[t] = off;
    turn_conv[t] = c;
    off += static_cast<int64_t>(h) + tt + 2 * static_cast<int64_t>(r);
    p += static_cast<int64_t>(h) + r;  // next h starts right after r^in ends
  }
  conv_tokens[c] = off;
  conv_ctx[c] = static_cast<int32_t>(p);
}

// Single block: exclusive scan of conversation token counts (in place, with
// the grand total appended), sequence offsets and consistency checks.
__global__ void seq_scan_kernel(int64_t* __restrict__ conv_off, const int32_t* __restrict__ conv_turn_ptr,
                                const int32_t* __restrict__ seq_conv_ptr, int32_t n_seqs, int32_t n_convs,
                                int32_t n_turns, int64_t total, int32_t max_seqlen, int32_t* __restrict__ cu_seqlens,
                                int32_t* __restrict__ dev_status) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_convs; base += blockDim.x) {
    const int i = base + tid;
    int64_t x = (i < n_convs) ? conv_off[i] : 0;
    int64_t incl = x;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int64_t ws = (lane < (blockDim.x >> 5)) ? warp_sums[lane] : 0;
      int64_t wi = ws;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, wi, d);
        if (lane >= d) wi += y;
      }
      if (lane < (blockDim.x >> 5)) warp_sums[lane] = wi - ws;  // exclusive warp offsets
    }
    __syncthreads();
    const int64_t c0 = carry;
    if (i < n_convs) conv_off[i] = c0 + warp_sums[warp] + incl - x;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = c0 + warp_sums[warp] + incl;
    __syncthreads();
  }
  if (tid == 0) {
    conv_off[n_convs] = carry;
    int bad = 0;
    if (conv_turn_ptr[0] != 0 || conv_turn_ptr[n_convs] != n_turns) bad |= OPR_DEV_BAD_INPUT;
    if (seq_conv_ptr[0] != 0 || seq_conv_ptr[n_seqs] != n_convs) bad |= OPR_DEV_BAD_INPUT;
    if (carry != total) bad |= OPR_DEV_TOTAL_MISMATCH;
    if (bad) atomicOr(dev_status, bad);
  }
  __syncthreads();
  for (int s = tid; s <= n_seqs; s += blockDim.x) {
    int c = seq_conv_ptr[s];
    int cn = (s < n_seqs) ? seq_conv_ptr[s + 1] : c;
    if (c < 0 || c > n_convs || cn < c || cn > n_convs) {
      atomicOr(dev_status, OPR_DEV_BAD_INPUT);
      c = c < 0 ? 0 : (c > n_convs ? n_convs : c);
      cn = c;
    }
    const int64_t a = conv_off[c];
    cu_seqlens[s] = static_cast<int32_t>(a < total ? a : total);
    if (s < n_seqs && conv_off[cn] - a > max_seqlen) atomicOr(dev_status, OPR_DEV_SEQ_TOO_LONG);
  }
}

// One block per turn: write type, turn index, conversation and position of
// each of its h + t + 2r tokens (segment order h, t, r^in, r^out), and the
// token's attention position.  The attention order stores each conversation as
// its context tokens h_1 r^in_1 ... h_N r^in_N, then its trained tokens t_1
// r^out_1 ... t_N r^out_N (each segment in stream order): the mask is the same,
// every visible key still comes before its query, and the context part is one
// causal block and the trained part one staircase, which leaves far fewer
// partially visible 128x128 tiles than the interleaved stream order.
__global__ void fill_tokens_kernel(const int32_t* __restrict__ turn_lens, const int32_t* __restrict__ conv_turn_ptr,
                                   const int64_t* __restrict__ conv_off, const int64_t* __restrict__ turn_off,
                                   const int32_t* __restrict__ turn_pos0, const int32_t* __restrict__ turn_conv,
                                   const int32_t* __restrict__ conv_ctx, int32_t n_convs, int64_t total,
                                   int8_t* __restrict__ token_type, int32_t* __restrict__ turn_idx,
                                   int32_t* __restrict__ conv_idx, int32_t* __restrict__ pos_id,
                                   int32_t* __restrict__ tok_meta, int32_t* __restrict__ attn_pos,
                                   int32_t* __restrict__ attn_conv, int32_t* __restrict__ attn_meta,
                                   int32_t* __restrict__ stream_of) {
  const int t = blockIdx.x;
  const int c = turn_conv[t];
  if (c < 0 || c >= n_convs) return;
  const int h = max(turn_lens[3 * t], 0), tt = max(turn_lens[3 * t + 1], 0), r = max(turn_lens[3 * t + 2], 0);
  const int i = t - conv_turn_ptr[c];
  const int p = turn_pos0[t];
  const int64_t base = conv_off[c] + turn_off[t];
  // attention order: this turn's context tokens start at its cursor p (the
  // context tokens of the earlier turns), its trained ones after the
  // conversation's conv_ctx context tokens and the earlier turns' t + r^out
  const int64_t ctx0 = conv_off[c] + p;
  const int64_t trn0 = conv_off[c] + conv_ctx[c] + (turn_off[t] - p);
  const int n = h + tt + 2 * r;
  for (int x = threadIdx.x; x < n; x += blockDim.x) {
    int type, pos;
    int64_t ap;
    if (x < h) {
      type = kTypeH;
      pos = p + x;
      ap = ctx0 + x;
    } else if (x < h + tt) {
      type = kTypeT;
      pos = p + x;  // t starts at p + h
      ap = trn0 + (x - h);
    } else if (x < h + tt + r) {
      type = kTypeRin;
      pos = p + h + (x - h - tt);
      ap = ctx0 + h + (x - h - tt);
    } else {
      type = kTypeRout;
      pos = p + h + tt + (x - h - tt - r);
      ap = trn0 + tt + (x - h - tt - r);
    }
    const int64_t g = base + x;
    if (g < 0 || g >= total || ap < 0 || ap >= total) continue;
    const int meta = (i << 2) | type;
    token_type[g] = static_cast<int8_t>(type);
    turn_idx[g] = i;
    conv_idx[g] = c;
    pos_id[g] = pos;
    tok_meta[g] = meta;
    attn_pos[g] = static_cast<int32_t>(ap);
    attn_conv[ap] = c;
    attn_meta[ap] = meta;
    stream_of[ap] = static_cast<int32_t>(g);
  }
}

// One block of 128 threads per tile (I, J) of sequence s; thread r owns query
// row I*128 + r and counts its visible keys among the tile's 128 columns, per
// key half.  The tile's byte: class (empty / full / partial) | (key halves << 2),
// bit h of the key halves set when some query sees a key of half h.
__global__ void __launch_bounds__(128) block_map_kernel(const int32_t* __restrict__ cu_seqlens,
                                                        const int32_t* __restrict__ conv_idx,
                                                        const int32_t* __restrict__ tok_meta, int32_t T,
                                                        uint8_t* __restrict__ block_map) {
  __shared__ int32_t kconv[kTile], kmeta[kTile];
  __shared__ int32_t warp_cnt[4][2];
  const int J = blockIdx.x, I = blockIdx.y, s = blockIdx.z;
  const int r = threadIdx.x;
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  uint8_t* out = block_map + (static_cast<size_t>(s) * T + I) * T + J;
  if (J > I || I * kTile >= L || J * kTile >= L) {  // above the diagonal or past the end: empty
    if (r == 0) *out = OPR_TILE_EMPTY;
    return;
  }
  const int qi = I * kTile + r, ki = J * kTile + r;
  const bool qv = qi < L, kv = ki < L;
  const int qconv = qv ? conv_idx[seq0 + qi] : -2;
  const int qmeta = qv ? tok_meta[seq0 + qi] : 0;
  kconv[r] = kv ? conv_idx[seq0 + ki] : -1;
  kmeta[r] = kv ? tok_meta[seq0 + ki] : 0;
  // Quick exit: every key of the tile belongs to a conversation that ends
  // before the tile's first query row (conversation ids grow along a sequence).
  const int first_q_conv = conv_idx[seq0 + I * kTile];
  const int last_k = min(L, (J + 1) * kTile) - 1;
  const bool all_before = conv_idx[seq0 + last_k] < first_q_conv;
  __syncthreads();
  if (all_before) {
    if (r == 0) *out = OPR_TILE_EMPTY;
    return;
  }
  int cnt[2] = {0, 0};
  const int qg = seq0 + qi;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll 8
    for (int c = h * kKeyHalf; c < (h + 1) * kKeyHalf; ++c)
      cnt[h] += visible(qg, qconv, qmeta, seq0 + J * kTile + c, kconv[c], kmeta[c]) ? 1 : 0;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) cnt[h] += __shfl_xor_sync(0xffffffffu, cnt[h], d);
    if ((r & 31) == 0) warp_cnt[r >> 5][h] = cnt[h];
  }
  __syncthreads();
  if (r == 0) {
    int half_cnt[2];
    for (int h = 0; h < 2; ++h) half_cnt[h] = warp_cnt[0][h] + warp_cnt[1][h] + warp_cnt[2][h] + warp_cnt[3][h];
    const int tot = half_cnt[0] + half_cnt[1];
    const int cls = tot == 0 ? OPR_TILE_EMPTY : (tot == kTile * kTile ? OPR_TILE_FULL : OPR_TILE_PARTIAL);
    const int halves = (half_cnt[0] > 0 ? 1 : 0) | (half_cnt[1] > 0 ? 2 : 0);
    *out = static_cast<uint8_t>(cls | (halves << 2));
  }
}

// The block map again, from the key tile's run table (tile_meta_kernel): thread
// r owns query row I*128 + r and counts, per key half, its visible keys run by
// run (one rule test per run instead of per key).  Same bytes as
// block_map_kernel; the attention order has few runs per tile.
__global__ void __launch_bounds__(128) block_map_runs_kernel(const int32_t* __restrict__ cu_seqlens,
                                                             const int32_t* __restrict__ conv_idx,
                                                             const int32_t* __restrict__ tok_meta,
                                                             const TileMeta* __restrict__ tmeta, int32_t T,
                                                             uint8_t* __restrict__ block_map) {
  __shared__ TileMeta km;
  __shared__ int32_t warp_cnt[4][2];
  const int J = blockIdx.x, I = blockIdx.y, s = blockIdx.z;
  const int r = threadIdx.x;
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  uint8_t* out = block_map + (static_cast<size_t>(s) * T + I) * T + J;
  if (J > I || I * kTile >= L || J * kTile >= L) {  // above the diagonal or past the end: empty
    if (r == 0) *out = OPR_TILE_EMPTY;
    return;
  }
  // Quick exit: every key of the tile belongs to a conversation that ends
  // before the tile's first query row (conversation ids grow along a sequence).
  const int first_q_conv = conv_idx[seq0 + I * kTile];
  const int last_k = min(L, (J + 1) * kTile) - 1;
  if (conv_idx[seq0 + last_k] < first_q_conv) {
    if (r == 0) *out = OPR_TILE_EMPTY;
    return;
  }
  {
    const int4* src = reinterpret_cast<const int4*>(tmeta + static_cast<size_t>(s) * T + J);
    int4* dst = reinterpret_cast<int4*>(&km);
    for (int x = r; x < static_cast<int>(sizeof(TileMeta) / sizeof(int4)); x += blockDim.x) dst[x] = src[x];
  }
  __syncthreads();
  const int qi = I * kTile + r;
  int cnt[2] = {0, 0};
  if (qi < L) {
    const int qconv = conv_idx[seq0 + qi];
    const int qmeta = tok_meta[seq0 + qi];
    const int lim = min(max(qi - J * kTile + 1, 0), kTile);  // keys not after the query
    const int nr = min(km.nruns, kTile);
    for (int x = 0; x < nr; ++x) {
      const int a = km.bound[x], b = min(km.bound[x + 1], lim);
      if (a >= b || km.conv[x] != qconv || !turn_type_rule(qmeta, km.meta[x])) continue;
      cnt[0] += max(0, min(b, kKeyHalf) - a);
      cnt[1] += max(0, b - max(a, kKeyHalf));
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) cnt[h] += __shfl_xor_sync(0xffffffffu, cnt[h], d);
    if ((r & 31) == 0) warp_cnt[r >> 5][h] = cnt[h];
  }
  __syncthreads();
  if (r == 0) {
    int half_cnt[2];
    for (int h = 0; h < 2; ++h) half_cnt[h] = warp_cnt[0][h] + warp_cnt[1][h] + warp_cnt[2][h] + warp_cnt[3][h];
    const int tot = half_cnt[0] + half_cnt[1];
    const int cls = tot == 0 ? OPR_TILE_EMPTY : (tot == kTile * kTile ? OPR_TILE_FULL : OPR_TILE_PARTIAL);
    const int halves = (half_cnt[0] > 0 ? 1 : 0) | (half_cnt[1] > 0 ? 2 : 0);
    *out = static_cast<uint8_t>(cls | (halves << 2));
  }
}

// One warp per row (blockIdx.y == 0) or column (== 1) of the tile grid of a
// sequence: compact the non-empty tiles, in ascending order, into a list of
// entries (index << 4) | block-map byte.
__global__ void tile_lists_kernel(const uint8_t* __restrict__ block_map, int32_t T, int32_t* __restrict__ row_cnt,
                                  int32_t* __restrict__ row_list, int32_t* __restrict__ col_cnt,
                                  int32_t* __restrict__ col_list) {
  const int line = blockIdx.x;  // s * T + I (rows) or s * T + J (columns)
  const int s = line / T, x = line % T;
  const int lane = threadIdx.x;
  const bool rows = blockIdx.y == 0;
  const uint8_t* base = block_map + static_cast<size_t>(s) * T * T;
  int32_t* list = (rows ? row_list : col_list) + static_cast<size_t>(line) * T;
  int n = 0;
  for (int y0 = 0; y0 < T; y0 += 32) {
    const int y = y0 + lane;
    int byte = 0;  // class | (key halves << 2)
    if (y < T) byte = rows ? base[static_cast<size_t>(x) * T + y] : base[static_cast<size_t>(y) * T + x];
    const bool nonempty = (byte & 3) != OPR_TILE_EMPTY;
    const unsigned m = __ballot_sync(0xffffffffu, nonempty);
    if (nonempty) list[n + __popc(m & ((1u << lane) - 1u))] = (y << 4) | byte;
    n += __popc(m);
  }
  if (lane == 0) (rows ? row_cnt : col_cnt)[line] = n;
}

// One block of 128 threads per tile (s, J): the tile's TileMeta record (runs of
// equal conversation and meta, in token order).
__global__ void __launch_bounds__(128) tile_meta_kernel(const int32_t* __restrict__ cu_seqlens,
                                                        const int32_t* __restrict__ conv_idx,
                                                        const int32_t* __restrict__ tok_meta, int32_t T,
                                                        TileMeta* __restrict__ out) {
  __shared__ int32_t sconv[kTile], smeta[kTile];
  __shared__ int32_t wcount[4];
  const int tile = blockIdx.x;
  const int s = tile / T, J = tile % T;
  const int c = threadIdx.x, lane = c & 31, w = c >> 5;
  const int seq0 = cu_seqlens[s];
  const int L = cu_seqlens[s + 1] - seq0;
  const bool v = J * kTile + c < L;
  sconv[c] = v ? conv_idx[seq0 + J * kTile + c] : -1;
  smeta[c] = v ? tok_meta[seq0 + J * kTile + c] : 0;
  __syncthreads();
  const bool st = (c == 0) || sconv[c] != sconv[c - 1] || smeta[c] != smeta[c - 1];
  const uint32_t b = __ballot_sync(0xffffffffu, st);
  if (lane == 0) wcount[w] = __popc(b);
  __syncthreads();
  int base = 0;
  for (int x = 0; x < w; ++x) base += wcount[x];
  if (st) {
    const int r = base + __popc(b & ((1u << lane) - 1u));
    out[tile].bound[r] = c;
    out[tile].conv[r] = sconv[c];
    out[tile].meta[r] = smeta[c];
  }
  if (c == 0) {
    const int nr = wcount[0] + wcount[1] + wcount[2] + wcount[3];
    out[tile].nruns = nr;
    out[tile].bound[nr] = kTile;
  }
}

// Single block: order tiles by descending number of non-empty tiles in their
// row (q_sched) or column (k_sched), ties by index, so the longest work
// items start first.  With by_seq the tiles are first grouped by sequence
// (k_sched): the dkdv CTAs that run at the same time then stream the query
// tiles of one sequence, which stay in L2.  Bitonic sort in shared memory;
// above kMaxSort items the natural order is kept.
constexpr int kMaxSort = 8192;

__global__ void __launch_bounds__(1024) sched_kernel(const int32_t* __restrict__ cnt, int32_t n, int32_t T,
                                                    int32_t by_seq, int32_t* __restrict__ order) {
  extern __shared__ unsigned long long keys[];
  if (n > kMaxSort) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) order[i] = i;
    return;
  }
  int np = 1;
  while (np < n) np <<= 1;
  for (int i = threadIdx.x; i < np; i += blockDim.x)
    keys[i] = (i < n) ? ((by_seq ? static_cast<unsigned long long>(0xFFFFu - static_cast<unsigned>(i / T)) << 48 : 0ull) |
                         (static_cast<unsigned long long>(cnt[i]) << 32) | (0xFFFFFFFFull - static_cast<unsigned>(i)))
                      : 0ull;
  __syncthreads();
  for (int k = 2; k <= np; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool desc = (i & k) == 0;  // descending overall
          const unsigned long long a = keys[i], b = keys[p];
          if (desc ? (a < b) : (a > b)) {
            keys[i] = b;
            keys[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    order[i] = static_cast<int32_t>(0xFFFFFFFFull - (keys[i] & 0xFFFFFFFFull));
}

}  // namespace

cudaError_t launch_layout(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                          int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total, int32_t max_seqlen,
                          int32_t* cu_seqlens, int8_t* token_type, int32_t* turn_idx, int32_t* conv_idx,
                          int32_t* pos_id, int32_t* attn_pos, uint8_t* block_map, void* ws, int32_t* dev_status,
                          cudaStream_t stream) {
  const LayoutWs w = layout_ws_map(n_seqs, n_convs, n_turns, total, max_seqlen);
  int64_t* conv_off = ws_ptr<int64_t>(ws, w.conv_off);
  int64_t* turn_off = ws_ptr<int64_t>(ws, w.turn_off);
  int32_t* turn_pos0 = ws_ptr<int32_t>(ws, w.turn_pos0);
  int32_t* turn_conv = ws_ptr<int32_t>(ws, w.turn_conv);
  int32_t* conv_ctx = ws_ptr<int32_t>(ws, w.conv_ctx);
  int32_t* tok_meta = ws_ptr<int32_t>(ws, w.tok_meta);
  int32_t* attn_conv = ws_ptr<int32_t>(ws, w.attn_conv);
  int32_t* attn_meta = ws_ptr<int32_t>(ws, w.attn_meta);
  int32_t* stream_of = ws_ptr<int32_t>(ws, w.stream_of);
  uint8_t* attn_bmap = ws_ptr<uint8_t>(ws, w.attn_bmap);

  cudaError_t e = cudaSuccess;
  if (n_turns > 0 && (e = cudaMemsetAsync(turn_conv, 0xFF, sizeof(int32_t) * n_turns, stream)) != cudaSuccess)
    return e;  // -1: no conversation
  if (total > 0) {
    // -1 where an inconsistent input leaves an attention position unwritten: no
    // conversation (never visible), and no stream row (the kernels skip it)
    if ((e = cudaMemsetAsync(attn_conv, 0xFF, sizeof(int32_t) * total, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(stream_of, 0xFF, sizeof(int32_t) * total, stream)) != cudaSuccess) return e;
  }
  if (n_convs > 0)
    conv_walk_kernel<<<(n_convs + 127) / 128, 128, 0, stream>>>(turn_lens, conv_turn_ptr, n_convs, n_turns,
                                                                conv_off, turn_off, turn_pos0, turn_conv, conv_ctx,
                                                                dev_status);
  seq_scan_kernel<<<1, 1024, 0, stream>>>(conv_off, conv_turn_ptr, seq_conv_ptr, n_seqs, n_convs, n_turns, total,
                                          max_seqlen, cu_seqlens, dev_status);
  if (n_turns > 0)
    fill_tokens_kernel<<<n_turns, 256, 0, stream>>>(turn_lens, conv_turn_ptr, conv_off, turn_off, turn_pos0,
                                                    turn_conv, conv_ctx, n_convs, total, token_type, turn_idx,
                                                    conv_idx, pos_id, tok_meta, attn_pos, attn_conv, attn_meta,
                                                    stream_of);
  if (w.n_tiles > 0) {
    dim3 grid(w.T, w.T, n_seqs);
    if (block_map != nullptr)  // the stream-order block map (an output for the caller)
      block_map_kernel<<<grid, 128, 0, stream>>>(cu_seqlens, conv_idx, tok_meta, w.T, block_map);
    // the attention order's run tables, block map and tile lists (the kernels' view)
    tile_meta_kernel<<<w.n_tiles, 128, 0, stream>>>(cu_seqlens, attn_conv, attn_meta, w.T,
                                                    ws_ptr<TileMeta>(ws, w.tile_meta));
    block_map_runs_kernel<<<grid, 128, 0, stream>>>(cu_seqlens, attn_conv, attn_meta,
                                                    ws_ptr<TileMeta>(ws, w.tile_meta), w.T, attn_bmap);
    tile_lists_kernel<<<dim3(w.n_tiles, 2), 32, 0, stream>>>(
        attn_bmap, w.T, ws_ptr<int32_t>(ws, w.row_cnt), ws_ptr<int32_t>(ws, w.row_list),
        ws_ptr<int32_t>(ws, w.col_cnt), ws_ptr<int32_t>(ws, w.col_list));
    int np = 1;
    while (np < w.n_tiles) np <<= 1;
    const size_t smem = (w.n_tiles <= kMaxSort) ? sizeof(unsigned long long) * np : 0;
    static bool attr_set = false;
    if (!attr_set) {
      cudaFuncSetAttribute(sched_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sizeof(unsigned long long) * kMaxSort));
      attr_set = true;
    }
    sched_kernel<<<1, 1024, smem, stream>>>(ws_ptr<int32_t>(ws, w.row_cnt), w.n_tiles, w.T, 0,
                                            ws_ptr<int32_t>(ws, w.q_sched));
    sched_kernel<<<1, 1024, smem, stream>>>(ws_ptr<int32_t>(ws, w.col_cnt), w.n_tiles, w.T, 1,
                                            ws_ptr<int32_t>(ws, w.k_sched));
  }
  return cudaGetLastError();
}

}  // namespace opr
