// opr_internal.cuh - layout workspace map and the visibility predicate shared
// by the CUDA kernels of libopr (never by the oracle).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/opr.h"

namespace opr {

constexpr int kTile = OPR_TILE;

// Token type codes (One-Pass to Reason segment order inside a turn).
constexpr int kTypeH = 0, kTypeT = 1, kTypeRin = 2, kTypeRout = 3;

// Visibility as two 4-bit tables indexed by the key's type (bit order h, t,
// r^in, r^out = bits 0..3), together with "same conversation" and "key not
// after query".  This is the Karnaugh-map style reduction of the four rules
// of the "分块稀疏注意力掩码" section:
//   earlier turn  -> key visible iff it is h or r^in      (H<i)       : 0b0101
//   same turn     -> h row: {h}; t row: {h, t}; r^in row: {h, r^in};
//                    r^out row: {h, t, r^out}                        : nibbles 1, 3, 5, B
// Causality inside a segment comes from "key not after query".  That rule holds
// in the stream order (h < t < r^in < r^out inside a turn) and in the attention
// order the kernels use (per conversation the context tokens h_1 r^in_1 ... h_N
// r^in_N, then the trained tokens t_1 r^out_1 ... t_N r^out_N): in both, every
// visible key comes before its query and each segment keeps its own order.
constexpr uint32_t kPrevTurnBits = 0x5u;
constexpr uint32_t kSameTurnBits = 0xB531u;  // nibble per query type

// meta = (turn << 2) | type.  A key of a later turn is never visible: in the
// stream order it also comes after the query, but in the attention order the
// later turns' context tokens come before the earlier turns' trained ones, so
// the turn is compared explicitly.
__host__ __device__ __forceinline__ bool turn_type_rule(int32_t qmeta, int32_t kmeta) {
  const int32_t qturn = qmeta >> 2, kturn = kmeta >> 2;
  if (kturn > qturn) return false;
  const uint32_t bits = (kturn < qturn) ? kPrevTurnBits : ((kSameTurnBits >> ((qmeta & 3) * 4)) & 0xFu);
  return (bits >> (kmeta & 3)) & 1u;
}

__host__ __device__ __forceinline__ bool visible(int32_t qg, int32_t qconv, int32_t qmeta, int32_t kg,
                                                 int32_t kconv, int32_t kmeta) {
  if (qconv != kconv || kg > qg) return false;
  return turn_type_rule(qmeta, kmeta);
}

__host__ __device__ __forceinline__ size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// A block-map byte is class | (key halves << 2): class OPR_TILE_*, and bit h of the
// key halves set when some query of the tile sees a key of half h (keys 64 h ..
// 64 h + 63).  A tile-list entry is (tile index << 4) | block-map byte.
__host__ __device__ __forceinline__ int entry_index(int e) { return e >> 4; }
__host__ __device__ __forceinline__ int entry_class(int e) { return e & 3; }
__host__ __device__ __forceinline__ int entry_halves(int e) { return (e >> 2) & 3; }
constexpr int kKeyHalf = kTile / 2;

// Key/query metadata of one 128-token tile of a sequence, precomputed by the
// layout so that the attention kernels fetch it with one bulk copy: the tile's
// tokens split into runs of equal (conversation, turn, type); run r covers
// tokens bound[r] .. bound[r + 1] - 1 of the tile and has conversation conv[r]
// (-1 past the sequence end) and meta[r] = (turn << 2) | type.
struct TileMeta {
  int32_t nruns;
  int32_t pad_[3];
  int32_t bound[kTile + 4];  // bound[nruns] = 128
  int32_t conv[kTile];
  int32_t meta[kTile];
};
static_assert(sizeof(TileMeta) % 16 == 0, "bulk copies move multiples of 16 bytes");

// Byte offsets of the arrays inside the layout workspace.  Per-token arrays
// named attn_* are indexed by attention position (see attn_pos of
// opr_build_layout); the tile lists, run tables and schedules describe the
// attention order too.
struct LayoutWs {
  int32_t T;          // tiles per sequence edge
  int32_t n_tiles;    // n_seqs * T
  size_t tok_meta;    // int32 [total]          (turn << 2) | type, stream order
  size_t attn_conv;   // int32 [total]          conversation of each attention position
  size_t attn_meta;   // int32 [total]          (turn << 2) | type of each attention position
  size_t stream_of;   // int32 [total]          stream index of each attention position
  size_t attn_bmap;   // uint8 [n_tiles][T]     block map in the attention order
  size_t row_cnt;     // int32 [n_tiles]        non-empty tiles in row (s, I)
  size_t row_list;    // int32 [n_tiles][T]     (J << 4) | block-map byte, ascending J
  size_t col_cnt;     // int32 [n_tiles]        non-empty tiles in column (s, J)
  size_t col_list;    // int32 [n_tiles][T]     (I << 4) | block-map byte, ascending I
  size_t q_sched;     // int32 [n_tiles]        s * T + I, most tiles first
  size_t k_sched;     // int32 [n_tiles]        s * T + J, most tiles first
  size_t conv_off;    // int64 [n_convs + 1]    token offset of each conversation
  size_t turn_off;    // int64 [n_turns]        token offset of each turn inside its conversation
  size_t turn_pos0;   // int32 [n_turns]        first position id of h_i
  size_t turn_conv;   // int32 [n_turns]        conversation of each turn
  size_t conv_ctx;    // int32 [n_convs]        context tokens (h and r^in) of each conversation
  size_t tile_meta;   // TileMeta [n_tiles]     per 128-token attention tile: run starts, conversations, metas
  size_t bytes;       // total
};

__host__ __device__ inline LayoutWs layout_ws_map(int32_t n_seqs, int32_t n_convs, int32_t n_turns,
                                                  int64_t total, int32_t max_seqlen) {
  LayoutWs w{};
  w.T = (max_seqlen + kTile - 1) / kTile;
  w.n_tiles = n_seqs * w.T;
  const size_t A = 256;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, A);
    return o;
  };
  const size_t nt = static_cast<size_t>(w.n_tiles);
  w.tok_meta = take(sizeof(int32_t) * static_cast<size_t>(total));
  w.attn_conv = take(sizeof(int32_t) * static_cast<size_t>(total));
  w.attn_meta = take(sizeof(int32_t) * static_cast<size_t>(total));
  w.stream_of = take(sizeof(int32_t) * static_cast<size_t>(total));
  w.attn_bmap = take(nt * static_cast<size_t>(w.T));
  w.row_cnt = take(sizeof(int32_t) * nt);
  w.row_list = take(sizeof(int32_t) * nt * static_cast<size_t>(w.T));
  w.col_cnt = take(sizeof(int32_t) * nt);
  w.col_list = take(sizeof(int32_t) * nt * static_cast<size_t>(w.T));
  w.q_sched = take(sizeof(int32_t) * nt);
  w.k_sched = take(sizeof(int32_t) * nt);
  w.conv_off = take(sizeof(int64_t) * (static_cast<size_t>(n_convs) + 1));
  w.turn_off = take(sizeof(int64_t) * static_cast<size_t>(n_turns));
  w.turn_pos0 = take(sizeof(int32_t) * static_cast<size_t>(n_turns));
  w.turn_conv = take(sizeof(int32_t) * static_cast<size_t>(n_turns));
  w.conv_ctx = take(sizeof(int32_t) * static_cast<size_t>(n_convs));
  w.tile_meta = take(sizeof(TileMeta) * nt);
  w.bytes = off;
  return w;
}

template <typename T>
__host__ __device__ __forceinline__ T* ws_ptr(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}
template <typename T>
__host__ __device__ __forceinline__ const T* ws_ptr(const void* base, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(base) + off);
}

// Launchers implemented in the .cu files (all asynchronous on `stream`).
cudaError_t launch_layout(const int32_t* turn_lens, const int32_t* conv_turn_ptr, const int32_t* seq_conv_ptr,
                          int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total, int32_t max_seqlen,
                          int32_t* cu_seqlens, int8_t* token_type, int32_t* turn_idx, int32_t* conv_idx,
                          int32_t* pos_id, int32_t* attn_pos, uint8_t* block_map, void* ws, int32_t* dev_status,
                          cudaStream_t stream);

cudaError_t launch_rope(const void* x, int32_t x_dtype, void* y, int32_t y_dtype, const int32_t* pos_id,
                        const int32_t* row_map, int64_t total, int32_t n_heads, int32_t head_dim, double base,
                        int32_t inverse, int32_t* dev_status, cudaStream_t stream);

}  // namespace opr
