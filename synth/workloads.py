"""Synthetic multi-turn conversations shaped like the One-Pass to Reason workloads.

The pages fine-tune Qwen-3 4B/8B/32B on multi-turn math dialogues
(One-Pass to Reason wiki note, "实验结果" and "数据集" sections); that dataset is
not available here, so conversations are drawn from uniform length
distributions and packed into sequences with the rule below.

Packing rule (the pages only say that packing is supported, "实现细节"):
turns are drawn one at a time into the current sequence; a conversation ends
after ``n_turns`` turns; when a drawn turn (costing h + t + 2r tokens once the
response is duplicated) would overflow the sequence capacity, the sequence is
closed, its last conversation is cut at that turn boundary and the drawn turn
is discarded.  The next sequence starts a new conversation.  No padding.

Everything here is integer bookkeeping or random number generation.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Workload table.  Length ranges are inclusive integer ranges (lo, hi).
CONFIGS: dict[int, dict] = {
    0: dict(name="tiny: 1 head, d64, N=2 turns, h16 t32 r16 (L=160)",
            batch=1, hq=1, hkv=1, d=64, n_turns=2,
            h=(16, 16), t=(32, 32), r=(16, 16), capacity=None,
            one_conv_per_seq=True, base=1e4, fp32_inputs=True, bwd=True),
    1: dict(name="qwen3-4b-like fwd: 32q/8kv, d128, N=4, packed to 16384",
            batch=1, hq=32, hkv=8, d=128, n_turns=4,
            h=(32, 256), t=(256, 1024), r=(64, 512), capacity=16384,
            one_conv_per_seq=False, base=1e6, fp32_inputs=False, bwd=False),
    2: dict(name="qwen3-8b-like fwd+bwd: 32q/8kv, d128, N=8, 2 x packed to 32768",
            batch=2, hq=32, hkv=8, d=128, n_turns=8,
            h=(32, 256), t=(256, 1024), r=(64, 512), capacity=32768,
            one_conv_per_seq=False, base=1e6, fp32_inputs=False, bwd=True),
    # Depth sweep: fixed h=128, t=512, r=256, one conversation per sequence.
    3: dict(name="depth sweep: 32q/8kv, d128, h128 t512 r256, one conversation",
            batch=1, hq=32, hkv=8, d=128, n_turns=4,
            h=(128, 128), t=(512, 512), r=(256, 256), capacity=None,
            one_conv_per_seq=True, base=1e6, fp32_inputs=False, bwd=True),
    4: dict(name="qwen3-32b-like fwd+bwd: 64q/8kv, d128, N=16, packed to 65536",
            batch=1, hq=64, hkv=8, d=128, n_turns=16,
            h=(64, 512), t=(512, 2048), r=(128, 1024), capacity=65536,
            one_conv_per_seq=False, base=1e6, fp32_inputs=False, bwd=True),
}

DEPTH_SWEEP_TURNS = (2, 4, 8, 12, 16)


@dataclass
class Workload:
    """Per-turn lengths grouped into conversations and sequences (host int32 arrays)."""

    turn_lens: np.ndarray          # int32 [n_turns, 3]: h, t, r of every turn
    conv_turn_ptr: np.ndarray      # int32 [n_convs + 1]: turns of conversation c
    seq_conv_ptr: np.ndarray       # int32 [n_seqs + 1]: conversations of sequence s
    hq: int
    hkv: int
    d: int
    base: float
    name: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def n_turns(self) -> int:
        return int(self.turn_lens.shape[0])

    @property
    def n_convs(self) -> int:
        return int(self.conv_turn_ptr.shape[0] - 1)

    @property
    def n_seqs(self) -> int:
        return int(self.seq_conv_ptr.shape[0] - 1)

    def seq_lengths(self) -> np.ndarray:
        """Token count of each packed sequence, responses counted twice."""
        cost = (self.turn_lens[:, 0].astype(np.int64) + self.turn_lens[:, 1]
                + 2 * self.turn_lens[:, 2].astype(np.int64))
        out = np.zeros(self.n_seqs, dtype=np.int64)
        for s in range(self.n_seqs):
            c0, c1 = self.seq_conv_ptr[s], self.seq_conv_ptr[s + 1]
            t0, t1 = self.conv_turn_ptr[c0], self.conv_turn_ptr[c1]
            out[s] = cost[t0:t1].sum()
        return out

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lengths().sum())

    @property
    def max_seqlen(self) -> int:
        sl = self.seq_lengths()
        return int(sl.max()) if sl.size else 0

    def conversation_tokens(self) -> int:
        """Tokens of the conversations before duplication (h + t + r per turn)."""
        return int(self.turn_lens.astype(np.int64).sum())


def _from_nested(seqs, hq, hkv, d, base, name, extra=None) -> Workload:
    turns, conv_ptr, seq_ptr = [], [0], [0]
    for convs in seqs:
        for conv in convs:
            turns.extend(conv)
            conv_ptr.append(len(turns))
        seq_ptr.append(len(conv_ptr) - 1)
    tl = np.asarray(turns, dtype=np.int32).reshape(-1, 3)
    return Workload(tl, np.asarray(conv_ptr, dtype=np.int32),
                    np.asarray(seq_ptr, dtype=np.int32), hq, hkv, d, base, name,
                    extra or {})


def _draw_turn(rng, cfg):
    return tuple(int(rng.integers(lo, hi + 1)) for lo, hi in (cfg["h"], cfg["t"], cfg["r"]))


def make_workload(index: int, seed: int | None = None, n_turns: int | None = None) -> Workload:
    """Workload ``index`` of the table, drawn with ``default_rng(seed)`` (default 1000 + index)."""
    cfg = dict(CONFIGS[index])
    if n_turns is not None:
        cfg["n_turns"] = n_turns
    rng = np.random.default_rng(1000 + index if seed is None else seed)
    seqs = []
    for _ in range(cfg["batch"]):
        if cfg["one_conv_per_seq"]:
            seqs.append([[_draw_turn(rng, cfg) for _ in range(cfg["n_turns"])]])
            continue
        convs, cur, used = [], [], 0
        while True:
            turn = _draw_turn(rng, cfg)
            cost = turn[0] + turn[1] + 2 * turn[2]
            if used + cost > cfg["capacity"]:
                if cur:
                    convs.append(cur)
                break
            cur.append(turn)
            used += cost
            if len(cur) == cfg["n_turns"]:
                convs.append(cur)
                cur = []
        seqs.append(convs)
    name = cfg["name"] if n_turns is None else f"{cfg['name']} (N={n_turns})"
    return _from_nested(seqs, cfg["hq"], cfg["hkv"], cfg["d"], cfg["base"], name,
                        dict(config=index, fp32_inputs=cfg["fp32_inputs"], bwd=cfg["bwd"]))


def make_custom_workload(seqs, hq=1, hkv=1, d=64, base=1e4, name="custom") -> Workload:
    """Workload from nested lists: seqs[s][c][i] = (h, t, r)."""
    return _from_nested(seqs, hq, hkv, d, base, name)


def random_small_workload(seed: int, n_seqs=2, max_convs=3, max_turns=4,
                          h=(0, 90), t=(0, 200), r=(0, 150), hq=4, hkv=2, d=128,
                          base=1e4) -> Workload:
    """Ragged workload with zero-length segments allowed, for parity tests."""
    rng = np.random.default_rng(seed)
    seqs = []
    for _ in range(n_seqs):
        convs = []
        for _ in range(int(rng.integers(1, max_convs + 1))):
            nt = int(rng.integers(1, max_turns + 1))
            conv = [(int(rng.integers(h[0], h[1] + 1)), int(rng.integers(t[0], t[1] + 1)),
                     int(rng.integers(r[0], r[1] + 1))) for _ in range(nt)]
            convs.append(conv)
        seqs.append(convs)
    return _from_nested(seqs, hq, hkv, d, base, f"random-small seed {seed}")


def npass_workload(w: Workload) -> tuple[Workload, list]:
    """The N-pass arrangement of the same conversations.

    Turn i of a conversation becomes its own sequence of length
    sum_{j<i}(h_j + r_j) + h_i + t_i + r_i, encoded as one turn (n, 0, 0) so
    that its mask is plain causal.  Each N-pass sequence holds one
    conversation.  Returns the workload and, for every N-pass sequence, the
    (conversation, turn) it was built for.
    """
    seqs, origin = [], []
    for c in range(w.n_convs):
        t0, t1 = int(w.conv_turn_ptr[c]), int(w.conv_turn_ptr[c + 1])
        hist = 0
        for i in range(t0, t1):
            h, t, r = (int(x) for x in w.turn_lens[i])
            seqs.append([[(hist + h + t + r, 0, 0)]])
            origin.append((c, i - t0))
            hist += h + r
    nw = _from_nested(seqs, w.hq, w.hkv, w.d, w.base, w.name + " [N-pass]")
    return nw, origin


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32)
    # keep NaN payloads quiet; inputs here are finite Gaussians
    return np.where(np.isnan(x), x, out)


def gaussian(rng: np.random.Generator, shape, bf16: bool = True) -> np.ndarray:
    """N(0, 1) float32 tensor, optionally rounded to bf16 values."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    return round_bf16(x) if bf16 else x
