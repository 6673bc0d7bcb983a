"""fp64 CPU oracle for One-Pass to Reason masked attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The CUDA library never calls it, and
it shares no code, table or helper with the CUDA library.

It is the plain definition of what the one-pass attention layer computes,
evaluated densely and slowly in float64 with numpy:

* ``build_layout``   token duplication, segment order and position ids
  (One-Pass to Reason wiki note, sections "Token 复制" and "位置 ID 策略").
* ``mask_row`` /
  ``dense_mask``     the visibility rules of the four token types
  (same note, section "分块稀疏注意力掩码"; English note, "Method").
* ``block_map``      classification of 128 x 128 tiles as empty / full / partial,
  counted from the dense mask; ``key_half_map`` marks which 64-key halves of a
  tile some query of the tile sees.
* ``rope``           rotate-half rotary embedding by position id (the pages'
  "位置编码等价" argument in "理论保证" relies on it; Qwen-3 uses it).
* ``attention_fwd`` / ``attention_bwd``
                     softmax attention under the mask and its analytic gradients.
* ``npass_rows``     the N-pass baseline: one causal run per turn over
  [h_1 r_1 ... h_{i-1} r_{i-1} h_i t_i r_i] with contiguous positions
  ("问题背景" and "理论保证" / Theorem 2.1).
* ``duplication_index`` / ``gather_rows`` / ``fold_rows``
                     the step before the attention layer: the one-pass token
                     stream as copies of the original (h, t, r per turn) stream,
                     and the gradient of that copy, which sums the gradients of
                     r^in and r^out into their original token ("Token 复制").
* ``kpass_plan`` / ``kpass_index``
                     the K-pass arrangement ("K-Pass 中间方案"): each pass is a
                     group of turns behind the history of the earlier turns.
* ``loss_rows`` / ``cross_entropy``
                     the step after the attention layer: the one-pass rows that
                     carry the N-pass next-token losses (t and r^out, "Token 复制"),
                     their targets, and softmax cross-entropy with its gradient.

Pins (checked by the tests that do not need a GPU): a hand-derived worked
example of positions, visibility and the duplication map, closed-form visible-pair counts per turn,
Theorem 2.1 by brute force (one-pass rows equal N-pass rows to 1e-12),
PyTorch's float64 causal scaled_dot_product_attention for the single-segment
case, RoPE invariants, and central finite differences for every gradient.

Readings where the pages are silent (each one listed in the design notes):
segment order h, t, r_in, r_out inside a turn; each segment causal within
itself; positions restart at 0 for every packed conversation; conversations
never see each other; zero-length segments are allowed; softmax scale
1/sqrt(d); rotate-half RoPE with angle pos * base^(-2j/d); LSE in natural log;
q head h reads kv head floor(h / (Hq / Hkv)).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

H, T, RIN, ROUT = 0, 1, 2, 3      # token types
TILE = 128                          # block-map tile edge
EMPTY, FULL, PARTIAL = 0, 1, 2      # block-map classes


@dataclass
class Layout:
    cu_seqlens: np.ndarray   # int64 [n_seqs + 1]
    token_type: np.ndarray   # int8  [total]
    turn_idx: np.ndarray     # int32 [total], 0-based within the conversation
    conv_idx: np.ndarray     # int32 [total], global conversation index
    pos_id: np.ndarray       # int32 [total]
    max_seqlen: int

    @property
    def n_seqs(self) -> int:
        return len(self.cu_seqlens) - 1

    @property
    def total(self) -> int:
        return int(self.cu_seqlens[-1])


def build_layout(turn_lens, conv_turn_ptr, seq_conv_ptr) -> Layout:
    """Lay out every turn as h_i, t_i, r_i^in, r_i^out and assign position ids.

    Position ids follow "位置 ID 策略": t_i and r_i^in both start right after
    h_i ends, r_i^out starts right after t_i ends, and h_{i+1} starts right
    after r_i^in ends.  Written with a cursor p (first position of h_i) this is
    h_i: p..p+h-1, t_i: p+h.., r_i^in: p+h.., r_i^out: p+h+t.., next p = p+h+r,
    which stays defined when a segment is empty.  p starts at 0 for every
    conversation.
    """
    turn_lens = np.asarray(turn_lens, dtype=np.int64).reshape(-1, 3)
    conv_turn_ptr = np.asarray(conv_turn_ptr, dtype=np.int64)
    seq_conv_ptr = np.asarray(seq_conv_ptr, dtype=np.int64)
    types, turns, convs, poss = [], [], [], []
    cu = [0]
    for s in range(len(seq_conv_ptr) - 1):
        for c in range(seq_conv_ptr[s], seq_conv_ptr[s + 1]):
            p = 0
            for i, ti in enumerate(range(conv_turn_ptr[c], conv_turn_ptr[c + 1])):
                h, t, r = (int(x) for x in turn_lens[ti])
                for typ, start, n in ((H, p, h), (T, p + h, t), (RIN, p + h, r), (ROUT, p + h + t, r)):
                    types += [typ] * n
                    turns += [i] * n
                    convs += [c] * n
                    poss += list(range(start, start + n))
                p = p + h + r
        cu.append(len(types))
    cu = np.asarray(cu, dtype=np.int64)
    max_seqlen = int(np.diff(cu).max()) if len(cu) > 1 else 0
    return Layout(cu, np.asarray(types, dtype=np.int8), np.asarray(turns, dtype=np.int32),
                  np.asarray(convs, dtype=np.int32), np.asarray(poss, dtype=np.int32), max_seqlen)


def mask_row(lay: Layout, q: int, lo: int, hi: int) -> np.ndarray:
    """Visibility of keys lo..hi-1 (global token indices) from query token q.

    The four rules of "分块稀疏注意力掩码", with H<i = {h_j, r_j^in : j < i} of
    the same conversation and every segment causal within itself:
      h_i      sees H<i and h_i up to itself
      t_i      sees H<i, h_i and t_i up to itself
      r_i^in   sees H<i, h_i and r_i^in up to itself
      r_i^out  sees H<i, h_i, t_i and r_i^out up to itself
    """
    idx = np.arange(lo, hi)
    ty, tu, cv = lay.token_type[lo:hi], lay.turn_idx[lo:hi], lay.conv_idx[lo:hi]
    c, i, tau = lay.conv_idx[q], lay.turn_idx[q], lay.token_type[q]
    same_conv = cv == c
    history = same_conv & (tu < i) & ((ty == H) | (ty == RIN))
    cur = same_conv & (tu == i)
    own_prefix = cur & (ty == tau) & (idx <= q)
    if tau == H:
        own = own_prefix
    elif tau == T:
        own = (cur & (ty == H)) | own_prefix
    elif tau == RIN:
        own = (cur & (ty == H)) | own_prefix
    else:  # ROUT
        own = (cur & ((ty == H) | (ty == T))) | own_prefix
    return history | own


def dense_mask(lay: Layout, s: int) -> np.ndarray:
    """Dense bool mask [L, L] of sequence s (row = query, column = key)."""
    a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
    m = np.zeros((b - a, b - a), dtype=bool)
    for q in range(a, b):
        m[q - a] = mask_row(lay, q, a, b)
    return m


def block_map(lay: Layout, tile: int = TILE, max_seqlen: int | None = None) -> np.ndarray:
    """uint8 [n_seqs, T, T]: 0 empty, 1 full (tile*tile visible pairs), 2 partial.

    Indices at or past the sequence length count as not visible, so a tail
    tile is never full.  T = ceil(max_seqlen / tile).
    """
    ms = lay.max_seqlen if max_seqlen is None else max_seqlen
    nt = (ms + tile - 1) // tile
    out = np.zeros((lay.n_seqs, nt, nt), dtype=np.uint8)
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        L = b - a
        counts = np.zeros((nt, nt), dtype=np.int64)
        edges = np.arange(0, L, tile)
        for ql in range(L):
            row = mask_row(lay, a + ql, a, b)
            counts[ql // tile, :len(edges)] += np.add.reduceat(row.astype(np.int64), edges)
        cls = np.where(counts == 0, EMPTY, np.where(counts == tile * tile, FULL, PARTIAL))
        out[s] = cls.astype(np.uint8)
    return out


def key_half_map(lay: Layout, tile: int = TILE, max_seqlen: int | None = None) -> np.ndarray:
    """uint8 [n_seqs, T, T]: for each tile, bit h (h = 0, 1) set when some query of the
    tile sees some key of its key half h (keys [h tile/2, (h + 1) tile/2) of the tile).
    A non-empty tile with one bit clear has a key half that no query sees: the part of
    the tile's products that sub-tile skipping leaves out."""
    ms = lay.max_seqlen if max_seqlen is None else max_seqlen
    nt = (ms + tile - 1) // tile
    half = tile // 2
    out = np.zeros((lay.n_seqs, nt, nt), dtype=np.uint8)
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        L = b - a
        seen = np.zeros((nt, 2 * nt), dtype=bool)
        edges = np.arange(0, L, half)
        for ql in range(L):
            row = mask_row(lay, a + ql, a, b)
            seen[ql // tile, :len(edges)] |= np.logical_or.reduceat(row, edges)
        out[s] = (seen[:, 0::2].astype(np.uint8) | (seen[:, 1::2].astype(np.uint8) << 1))
    return out


def rope(x: np.ndarray, pos: np.ndarray, base: float, inverse: bool = False) -> np.ndarray:
    """Rotate-half rotary embedding, float64.

    x: [tokens, heads, d]; pair (x[j], x[j + d/2]) is rotated by
    angle = pos * base^(-2j/d) (by -angle when ``inverse``).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    theta = float(base) ** (-(2.0 * np.arange(half, dtype=np.float64)) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    if inverse:
        ang = -ang
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def _group(hq: int, hkv: int, h: int) -> int:
    return h // (hq // hkv)


def attention_fwd(q, k, v, lay: Layout, scale: float | None = None):
    """Masked softmax attention over every sequence.

    q: [total, Hq, d], k/v: [total, Hkv, d] (already rotated).  Returns
    O [total, Hq, d] and LSE [Hq, total] = ln sum_visible exp(scale * q.k).
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    total, hq, d = q.shape
    hkv = k.shape[1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    o = np.zeros_like(q)
    lse = np.zeros((hq, total))
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        if b == a:
            continue
        m = dense_mask(lay, s)
        for h in range(hq):
            g = _group(hq, hkv, h)
            S = scale * (q[a:b, h] @ k[a:b, g].T)
            S = np.where(m, S, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            P = np.exp(S - mx)
            l = P.sum(axis=1, keepdims=True)
            P = P / l
            o[a:b, h] = P @ v[a:b, g]
            lse[h, a:b] = (mx + np.log(l))[:, 0]
    return o, lse


def attention_bwd(q, k, v, o, do, lse, lay: Layout, scale: float | None = None):
    """Analytic gradients of O = softmax(scale * q k^T masked) v.

    With P recomputed from LSE: dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
    dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q; dK and dV are summed
    over the q heads that share a kv head.
    """
    q, k, v, o, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, o, do))
    total, hq, d = q.shape
    hkv = k.shape[1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        if b == a:
            continue
        m = dense_mask(lay, s)
        for h in range(hq):
            g = _group(hq, hkv, h)
            S = scale * (q[a:b, h] @ k[a:b, g].T)
            P = np.where(m, np.exp(S - lse[h, a:b][:, None]), 0.0)
            dP = do[a:b, h] @ v[a:b, g].T
            D = (do[a:b, h] * o[a:b, h]).sum(axis=1)
            dS = P * (dP - D[:, None])
            dq[a:b, h] = scale * (dS @ k[a:b, g])
            dk[a:b, g] += scale * (dS.T @ q[a:b, h])
            dv[a:b, g] += P.T @ do[a:b, h]
    return dq, dk, dv


def forward(q_pre, k_pre, v, lay: Layout, base: float, scale: float | None = None):
    """RoPE by the layout's position ids, then masked attention."""
    qr = rope(q_pre, lay.pos_id, base)
    kr = rope(k_pre, lay.pos_id, base)
    return attention_fwd(qr, kr, v, lay, scale)


def backward(q_pre, k_pre, v, o, do, lse, lay: Layout, base: float, scale: float | None = None):
    """Gradients w.r.t. the pre-RoPE q and k (inverse rotation of dq, dk) and v."""
    qr = rope(q_pre, lay.pos_id, base)
    kr = rope(k_pre, lay.pos_id, base)
    dq, dk, dv = attention_bwd(qr, kr, v, o, do, lse, lay, scale)
    return rope(dq, lay.pos_id, base, inverse=True), rope(dk, lay.pos_id, base, inverse=True), dv


# --------------------------------------------------------------------------
# Row and column samples, for workloads too large for the dense evaluation.
# --------------------------------------------------------------------------

def _seq_of(lay: Layout, tok: int) -> int:
    return int(np.searchsorted(lay.cu_seqlens, tok, side="right") - 1)


def attention_rows(q, k, v, lay: Layout, rows, heads, do=None, scale: float | None = None):
    """O, LSE (and dQ when ``do`` is given) of selected query rows, computed one row at a time.

    q/k already rotated.  Returns dict with o [n, len(heads), d], lse
    [len(heads), n] and optionally dq [n, len(heads), d] (w.r.t. rotated q).
    """
    q, k, v = (np.asarray(a) for a in (q, k, v))
    hq, d = q.shape[1], q.shape[2]
    hkv = k.shape[1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    rows = np.asarray(rows)
    o = np.zeros((len(rows), len(heads), d))
    lse = np.zeros((len(heads), len(rows)))
    dq = np.zeros((len(rows), len(heads), d)) if do is not None else None
    for n, tok in enumerate(rows):
        s = _seq_of(lay, int(tok))
        a = int(lay.cu_seqlens[s])
        vis = mask_row(lay, int(tok), a, int(tok) + 1)
        cols = a + np.nonzero(vis)[0]
        for j, h in enumerate(heads):
            g = _group(hq, hkv, h)
            kk = k[cols, g].astype(np.float64)
            vv = v[cols, g].astype(np.float64)
            srow = scale * (kk @ q[tok, h].astype(np.float64))
            mx = srow.max()
            p = np.exp(srow - mx)
            l = p.sum()
            p /= l
            o[n, j] = p @ vv
            lse[j, n] = mx + np.log(l)
            if do is not None:
                dor = do[tok, h].astype(np.float64)
                dp = vv @ dor
                Dq = float(dor @ o[n, j])
                ds = p * (dp - Dq)
                dq[n, j] = scale * (ds @ kk)
    out = dict(o=o, lse=lse)
    if dq is not None:
        out["dq"] = dq
    return out


def attention_cols(q, k, v, do, lay: Layout, cols, kv_head: int, scale: float | None = None):
    """dK and dV (w.r.t. rotated k) of selected key tokens for one kv head.

    Every query row that sees one of the keys is evaluated in full (its own
    softmax, O and D), then its contributions are summed into the selected keys.
    """
    q, k, v, do = (np.asarray(a) for a in (q, k, v, do))
    hq, d = q.shape[1], q.shape[2]
    hkv = k.shape[1]
    group = hq // hkv
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    cols = np.asarray(cols)
    dk = np.zeros((len(cols), d))
    dv = np.zeros((len(cols), d))
    # candidate rows: same conversation, at or after the earliest selected key
    cand = set()
    for c in cols:
        s = _seq_of(lay, int(c))
        b = int(lay.cu_seqlens[s + 1])
        same = np.nonzero(lay.conv_idx[int(c):b] == lay.conv_idx[int(c)])[0] + int(c)
        cand.update(int(t) for t in same)
    for tok in sorted(cand):
        s = _seq_of(lay, tok)
        a = int(lay.cu_seqlens[s])
        vis = mask_row(lay, tok, a, tok + 1)
        sel = cols[(cols >= a) & (cols <= tok)]
        if not np.any(vis[sel - a]):
            continue
        vcols = a + np.nonzero(vis)[0]
        # position of each selected key inside vcols, or -1 when not visible
        where = np.searchsorted(vcols, cols)
        hit = [(int(wi), n) for n, (wi, c) in enumerate(zip(where, cols))
               if wi < len(vcols) and vcols[wi] == c]
        kk = k[vcols, kv_head].astype(np.float64)
        vv = v[vcols, kv_head].astype(np.float64)
        for h in range(kv_head * group, (kv_head + 1) * group):
            qr = q[tok, h].astype(np.float64)
            dor = do[tok, h].astype(np.float64)
            srow = scale * (kk @ qr)
            p = np.exp(srow - srow.max())
            p /= p.sum()
            orow = p @ vv
            dp = vv @ dor
            ds = p * (dp - float(dor @ orow))
            for j, n in hit:
                dk[n] += scale * ds[j] * qr
                dv[n] += p[j] * dor
    return dk, dv


# --------------------------------------------------------------------------
# N-pass baseline (Theorem 2.1 brute force)
# --------------------------------------------------------------------------

def npass_token_lists(lay: Layout, turn_lens, conv_turn_ptr):
    """For each (conversation, turn i): one-pass token indices of the N-pass sequence
    [h_1 r_1 ... h_{i-1} r_{i-1} h_i t_i r_i], where the context copies r_j are the
    r_j^in tokens and the current response r_i is the r_i^out tokens."""
    out = []
    conv_turn_ptr = np.asarray(conv_turn_ptr)
    for c in range(len(conv_turn_ptr) - 1):
        sel = np.nonzero(lay.conv_idx == c)[0]
        nt = int(conv_turn_ptr[c + 1] - conv_turn_ptr[c])
        ty, tu = lay.token_type[sel], lay.turn_idx[sel]
        for i in range(nt):
            hist = sel[(tu < i) & ((ty == H) | (ty == RIN))]
            cur = sel[(tu == i) & ((ty == H) | (ty == T) | (ty == ROUT))]
            out.append((c, i, np.concatenate([hist, cur])))
    return out


def causal_attention(q, k, v, scale: float | None = None):
    """Plain causal softmax attention of one sequence: q [n, Hq, d], k/v [n, Hkv, d]."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    n, hq, d = q.shape
    hkv = k.shape[1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    causal = np.tril(np.ones((n, n), dtype=bool))
    o = np.zeros_like(q)
    lse = np.zeros((hq, n))
    for h in range(hq):
        g = _group(hq, hkv, h)
        S = np.where(causal, scale * (q[:, h] @ k[:, g].T), -np.inf)
        mx = S.max(axis=1, keepdims=True)
        P = np.exp(S - mx)
        l = P.sum(axis=1, keepdims=True)
        o[:, h] = (P / l) @ v[:, g]
        lse[h] = (mx + np.log(l))[:, 0]
    return o, lse


def npass_rows(q_pre, k_pre, v, lay: Layout, turn_lens, conv_turn_ptr, base: float,
               scale: float | None = None):
    """Run the N-pass baseline and return, per (conversation, turn), the token
    indices and the causal run's O and LSE (positions 0..n-1, RoPE applied)."""
    res = []
    for c, i, toks in npass_token_lists(lay, turn_lens, conv_turn_ptr):
        pos = np.arange(len(toks))
        qr = rope(np.asarray(q_pre)[toks], pos, base)
        kr = rope(np.asarray(k_pre)[toks], pos, base)
        o, lse = causal_attention(qr, kr, np.asarray(v)[toks], scale)
        res.append((c, i, toks, o, lse))
    return res


def visible_pairs(lay: Layout) -> int:
    """Number of visible (q, k) pairs per head, counted from the mask rows."""
    n = 0
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        for q in range(a, b):
            n += int(mask_row(lay, q, a, q + 1).sum())
    return n


# --------------------------------------------------------------------------
# Token duplication ("Token 复制"): the step before the attention layer.
#
# The original stream holds each conversation's turns once, h_i t_i r_i, and
# conversations back to back in index order; the one-pass stream holds
# h_i t_i r_i^in r_i^out.  Every one-pass token is a copy of one original token.

def duplication_index(turn_lens, conv_turn_ptr):
    """(src, copies): src[i] = original index of one-pass token i; copies[o] = the
    one-pass positions of original token o as [first, second], second = -1 for
    h and t tokens (one copy) and the r^out position for r tokens (two copies)."""
    turn_lens = np.asarray(turn_lens, dtype=np.int64).reshape(-1, 3)
    conv_turn_ptr = np.asarray(conv_turn_ptr, dtype=np.int64)
    src, copies = [], []
    one_pass = 0
    orig = 0
    for c in range(len(conv_turn_ptr) - 1):
        for t in range(conv_turn_ptr[c], conv_turn_ptr[c + 1]):
            h, tt, r = (int(x) for x in turn_lens[t])
            h_orig, t_orig, r_orig = orig, orig + h, orig + h + tt
            h_one, t_one, rin_one, rout_one = one_pass, one_pass + h, one_pass + h + tt, one_pass + h + tt + r
            src += list(range(h_orig, h_orig + h)) + list(range(t_orig, t_orig + tt))
            src += list(range(r_orig, r_orig + r)) + list(range(r_orig, r_orig + r))
            copies += [[h_one + x, -1] for x in range(h)] + [[t_one + x, -1] for x in range(tt)]
            copies += [[rin_one + x, rout_one + x] for x in range(r)]
            one_pass += h + tt + 2 * r
            orig += h + tt + r
    return np.asarray(src, dtype=np.int32), np.asarray(copies, dtype=np.int32).reshape(-1, 2)


def gather_rows(x: np.ndarray, src: np.ndarray) -> np.ndarray:
    """The one-pass stream's rows: row i is a copy of original row src[i]."""
    return np.stack([x[int(o)] for o in src]) if len(src) else x[:0]


def fold_rows(dy: np.ndarray, copies: np.ndarray) -> np.ndarray:
    """Gradient of gather_rows w.r.t. x, in float32: each original row sums the
    rows of its copies (the non-negative entries of its row of `copies`), in
    slot order, one float32 addition after another."""
    dy = np.asarray(dy, dtype=np.float32)
    out = np.zeros((len(copies),) + dy.shape[1:], dtype=np.float32)
    for o, row in enumerate(copies):
        acc = None
        for a in row:
            if a < 0:
                continue
            acc = dy[a].copy() if acc is None else (acc + dy[a]).astype(np.float32)
        out[o] = acc
    return out


# --------------------------------------------------------------------------
# K-pass ("K-Pass 中间方案"): between N-pass (K = N) and one-pass (K = 1).
#
# Reading (the pages give only the trade-off): a conversation's N turns are
# split into K' = min(K, N) contiguous groups, group g holding turns
# [floor(g N / K'), floor((g + 1) N / K')).  Pass g is one sequence-packed
# conversation: first the history of the turns before the group, each turn j
# as h_j followed by r_j in one causal context segment (the turn (h_j + r_j, 0, 0):
# positions run on from h_j into r_j, exactly as h_j and r_j^in do in one pass),
# then the group's turns (h, t, r) laid out one-pass.  Every loss row (t and
# r^out) appears in exactly one pass; K = 1 is the one-pass layout.

def kpass_groups(n: int, K: int):
    """Turn boundaries b_0 = 0 < ... < b_K' = n of the K' = min(K, n) groups."""
    k = min(K, n)
    return [(g * n) // k for g in range(k + 1)] if k > 0 else [0]


def kpass_plan(turn_lens, conv_turn_ptr, seq_conv_ptr, K: int):
    """(turn_lens', conv_turn_ptr', seq_conv_ptr', turn_src): the K-pass
    arrangement as a workload for the one-pass layout, one conversation per
    pass, passes of a conversation back to back in its sequence; turn_src[u] =
    (original turn, pass offset) with pass offset -1 for a turn of the pass's
    own group and, for a history turn, (pass - group of the turn) >= 1."""
    turn_lens = np.asarray(turn_lens, dtype=np.int64).reshape(-1, 3)
    conv_turn_ptr = np.asarray(conv_turn_ptr, dtype=np.int64)
    seq_conv_ptr = np.asarray(seq_conv_ptr, dtype=np.int64)
    out_lens, out_conv, out_seq, src = [], [0], [0], []
    conv_pass0 = []
    n_out_convs = 0
    for c in range(len(conv_turn_ptr) - 1):
        t0, t1 = int(conv_turn_ptr[c]), int(conv_turn_ptr[c + 1])
        b = kpass_groups(t1 - t0, K)
        conv_pass0.append(n_out_convs)
        for g in range(len(b) - 1):
            for j in range(t0, t0 + b[g]):  # history: h_j then r_j as one context segment
                h, _, r = (int(x) for x in turn_lens[j])
                out_lens.append([h + r, 0, 0])
                gj = next(q for q in range(len(b) - 1) if b[q] <= j - t0 < b[q + 1])
                src.append([j, g - gj])
            for j in range(t0 + b[g], t0 + b[g + 1]):
                out_lens.append([int(x) for x in turn_lens[j]])
                src.append([j, -1])
            out_conv.append(len(out_lens))
            n_out_convs += 1
    conv_pass0.append(n_out_convs)
    for s in range(len(seq_conv_ptr) - 1):
        out_seq.append(conv_pass0[int(seq_conv_ptr[s + 1])])
    return (np.asarray(out_lens, dtype=np.int32).reshape(-1, 3), np.asarray(out_conv, dtype=np.int32),
            np.asarray(out_seq, dtype=np.int32), np.asarray(src, dtype=np.int32).reshape(-1, 2))


def kpass_index(turn_lens, conv_turn_ptr, seq_conv_ptr, K: int):
    """(src, copies): src[i] = original token of K-pass token i; copies[o] has K + 1
    slots: 0 = the copy in the token's own pass (h, t or r^in), 1 = the r^out copy
    (r tokens), 1 + d = the history copy in the pass d groups later (h and r tokens);
    -1 where there is none.  The original stream is the one of duplication_index."""
    turn_lens = np.asarray(turn_lens, dtype=np.int64).reshape(-1, 3)
    orig_off = np.concatenate([[0], np.cumsum(turn_lens.sum(axis=1))])
    lens2, _, _, tsrc = kpass_plan(turn_lens, conv_turn_ptr, seq_conv_ptr, K)
    copies = -np.ones((int(orig_off[-1]), K + 1), dtype=np.int32)
    src = []
    pos = 0
    for (n_h, _, _), (j, d) in zip(lens2, tsrc):
        h, t, r = (int(x) for x in turn_lens[j])
        o = int(orig_off[j])
        if d >= 1:  # history turn: originals of h_j, then of r_j
            ids = list(range(o, o + h)) + list(range(o + h + t, o + h + t + r))
            for x, oi in enumerate(ids):
                src.append(oi)
                copies[oi, 1 + d] = pos + x
            pos += len(ids)
        else:
            for x in range(h + t + r):
                src.append(o + x)
                copies[o + x, 0] = pos + x
            for x in range(r):
                src.append(o + h + t + x)
                copies[o + h + t + x, 1] = pos + h + t + r + x
            pos += h + t + 2 * r
    return np.asarray(src, dtype=np.int32), copies


# --------------------------------------------------------------------------
# Loss side: which one-pass rows carry the N-pass next-token losses.
#
# Reading (the pages say the loss is that of the N-pass runs, "理论保证", and
# that r^out is the copy trained on, "Token 复制"): in N-pass run i the
# sequence is [H<i, h_i, t_i, r_i] and the losses are the next-token
# predictions of t_i and r_i: from the last h_i row (target: the first t_i
# token, or the first r_i token when t_i is empty), from each t_i row (target:
# the next t_i token, or the first r_i token after the last), and from each
# r_i row but the last (target: the next r_i token).  In one pass those rows
# are the last h_i row, the t_i rows and the r_i^out rows (Theorem 2.1).

def loss_rows(turn_lens, conv_turn_ptr):
    """(rows, targets): one-pass row indices carrying a loss, in stream order, and the
    original-stream index of each row's target token."""
    turn_lens = np.asarray(turn_lens, dtype=np.int64).reshape(-1, 3)
    conv_turn_ptr = np.asarray(conv_turn_ptr, dtype=np.int64)
    rows, targets = [], []
    one_pass = orig = 0
    for c in range(len(conv_turn_ptr) - 1):
        for t in range(conv_turn_ptr[c], conv_turn_ptr[c + 1]):
            h, tt, r = (int(x) for x in turn_lens[t])
            assistant = list(range(orig + h, orig + h + tt + r))  # original t then r tokens
            if h > 0 and assistant:
                rows.append(one_pass + h - 1)
                targets.append(assistant[0])
            for x in range(tt):  # t rows: the next assistant token
                if x + 1 < len(assistant):
                    rows.append(one_pass + h + x)
                    targets.append(assistant[x + 1])
            for x in range(r - 1):  # r^out rows but the last
                rows.append(one_pass + h + tt + r + x)
                targets.append(orig + h + tt + x + 1)
            one_pass += h + tt + 2 * r
            orig += h + tt + r
    return np.asarray(rows, dtype=np.int32), np.asarray(targets, dtype=np.int32)


def cross_entropy(logits: np.ndarray, target_ids: np.ndarray):
    """Per-row softmax cross-entropy in float64 and its gradient w.r.t. the logits:
    loss = logsumexp(z) - z[target], dz = softmax(z) - onehot(target)."""
    z = np.asarray(logits, dtype=np.float64)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    s = e.sum(axis=1, keepdims=True)
    lse = (np.log(s) + m)[:, 0]
    idx = np.asarray(target_ids, dtype=np.int64)
    loss = lse - z[np.arange(len(idx)), idx]
    dz = e / s
    dz[np.arange(len(idx)), idx] -= 1.0
    return loss, dz
