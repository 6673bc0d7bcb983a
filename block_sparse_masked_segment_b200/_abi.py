"""ctypes marshalling for libopr.so: same names as the C entry points.

Each wrapper checks shapes and dtypes, allocates outputs with PyTorch on the
input's device, passes raw pointers plus the current CUDA stream, and turns a
non-zero ``opr_status`` into :class:`OprError`.  No arithmetic happens here.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# OPR_DEBUG_CHECKS=1 selects the library built with device-side bounds checks
# (same entry points; a failed check sets OPR_DEV_BOUNDS in the status word).
_LIB_PATH = os.path.join(_HERE, "lib", "libopr_debug.so" if os.environ.get("OPR_DEBUG_CHECKS") == "1" else "libopr.so")

OPR_OK, OPR_INVALID_ARG, OPR_UNSUPPORTED, OPR_CUDA_ERROR, OPR_WORKSPACE_TOO_SMALL = 0, 1, 2, 3, 4
DEV_BITS = {1: "bad input", 2: "total mismatch", 4: "sequence longer than max_seqlen", 8: "pipeline wait timeout",
            16: "fp16 range exceeded (rope output or backward fp16 copy)",
            32: "layout-table index out of range (debug checks)"}
DTYPE_BF16, DTYPE_FP32, DTYPE_FP16 = 0, 1, 2
TILE = 128

EXPORTED_SYMBOLS = (
    "opr_version",
    "opr_last_error",
    "opr_layout_workspace_bytes",
    "opr_build_layout",
    "opr_rope",
    "opr_attn_fwd",
    "opr_attn_bwd_workspace_bytes",
    "opr_attn_bwd_min_workspace_bytes",
    "opr_attn_bwd",
    "opr_attn_bwd_stages",
    "opr_attn_bwd_noalloc",
    "opr_duplication_index",
    "opr_gather_rows",
    "opr_fold_rows",
    "opr_kpass_sizes",
    "opr_kpass_plan",
    "opr_kpass_index_workspace_bytes",
    "opr_kpass_index",
    "opr_loss_row_count",
    "opr_loss_rows",
    "opr_cross_entropy",
    "opr_testing_set_wait_limit_ns",
    "opr_testing_layout_tables",
)

BWD_ROW_TERMS, BWD_DQ, BWD_DKDV = 1, 2, 4

_STATUS_NAMES = {1: "OPR_INVALID_ARG", 2: "OPR_UNSUPPORTED", 3: "OPR_CUDA_ERROR", 4: "OPR_WORKSPACE_TOO_SMALL",
                 5: "OPR_SCRATCH_TOO_LARGE"}
OPR_SCRATCH_TOO_LARGE = 5
NOALLOC_SCRATCH_BYTES = 32 << 20


class OprError(RuntimeError):
    pass


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libopr.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise OprError(f"{_LIB_PATH} is missing: build it with `python -m block_sparse_masked_segment_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, I64, SZ, D, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                             ctypes.c_double, ctypes.c_float)
    lib.opr_version.restype = ctypes.c_char_p
    lib.opr_version.argtypes = []
    lib.opr_last_error.restype = ctypes.c_char_p
    lib.opr_last_error.argtypes = []
    lib.opr_duplication_index.restype = ctypes.c_int
    lib.opr_duplication_index.argtypes = [P, P, I32, I32, I64, I64, P, P, P, P]
    lib.opr_gather_rows.restype = ctypes.c_int
    lib.opr_gather_rows.argtypes = [P, I64, I64, P, I64, P, P, P]
    lib.opr_fold_rows.restype = ctypes.c_int
    lib.opr_fold_rows.argtypes = [P, I64, I64, P, I32, I64, P, P, P]
    lib.opr_kpass_sizes.restype = ctypes.c_int
    lib.opr_kpass_sizes.argtypes = [P, P, P, I32, I32, I32, I32, P, P, P, P, P]
    lib.opr_kpass_plan.restype = ctypes.c_int
    lib.opr_kpass_plan.argtypes = [P, P, P, I32, I32, I32, I32, I32, I32, P, P, P, P, P, P]
    lib.opr_kpass_index_workspace_bytes.restype = ctypes.c_size_t
    lib.opr_kpass_index_workspace_bytes.argtypes = [I32, I32]
    lib.opr_loss_row_count.restype = ctypes.c_int64
    lib.opr_loss_row_count.argtypes = [P, I32]
    lib.opr_loss_rows.restype = ctypes.c_int
    lib.opr_loss_rows.argtypes = [P, I32, I64, I64, I64, P, P, P, P]
    lib.opr_cross_entropy.restype = ctypes.c_int
    lib.opr_cross_entropy.argtypes = [P, I32, I64, I32, P, P, P, F, P, P]
    lib.opr_kpass_index.restype = ctypes.c_int
    lib.opr_kpass_index.argtypes = [P, I32, P, P, I32, I64, I64, I32, P, P, P, SZ, P, P]
    lib.opr_layout_workspace_bytes.restype = SZ
    lib.opr_layout_workspace_bytes.argtypes = [I32, I32, I32, I64, I32]
    lib.opr_build_layout.restype = I32
    lib.opr_build_layout.argtypes = [P, P, P, I32, I32, I32, I64, I32, P, P, P, P, P, P, P, P, SZ, P, P]
    lib.opr_rope.restype = I32
    lib.opr_rope.argtypes = [P, I32, P, I32, P, P, I64, I32, I32, D, I32, P, P]
    lib.opr_attn_fwd.restype = I32
    lib.opr_attn_fwd.argtypes = [P, P, P, I32, I32, P, P, P, I32, I32, I32, I64, I32, I32, I32, I32, F, P, I32, P, P, P]
    lib.opr_attn_bwd_workspace_bytes.restype = SZ
    lib.opr_attn_bwd_workspace_bytes.argtypes = [I32, I32, I32, I32]
    lib.opr_attn_bwd_min_workspace_bytes.restype = SZ
    lib.opr_attn_bwd_min_workspace_bytes.argtypes = [I32, I32, I32, I32]
    lib.opr_attn_bwd.restype = I32
    lib.opr_attn_bwd.argtypes = [P, P, P, I32, P, I32, P, P, P, P, P, I32, I32, I32, I64, I32, I32, I32, I32, F,
                                 P, P, P, P, D, P, SZ, P, P]
    lib.opr_attn_bwd_stages.restype = I32
    lib.opr_attn_bwd_stages.argtypes = [P, P, P, I32, P, I32, P, P, P, P, P, I32, I32, I32, I64, I32, I32, I32, I32,
                                        F, P, P, P, P, D, P, SZ, P, I32, P]
    lib.opr_testing_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.opr_testing_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.opr_testing_layout_tables.restype = I32
    lib.opr_testing_layout_tables.argtypes = [I32, I32, I32, I64, I32, P]
    lib.opr_attn_bwd_noalloc.restype = I32
    lib.opr_attn_bwd_noalloc.argtypes = [P, P, P, I32, P, I32, P, P, P, P, P, I32, I32, I32, I64, I32, I32, I32, I32,
                                         F, P, P, P, P, D, P, P]
    _lib = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != OPR_OK:
        detail = f" ({load_library().opr_last_error().decode()})" if status == 3 else ""
        raise OprError(f"{what} returned {_STATUS_NAMES.get(status, status)}{detail}")


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise OprError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise OprError("tensors must be contiguous")


def opr_version() -> str:
    return load_library().opr_version().decode()


def opr_layout_workspace_bytes(n_seqs, n_convs, n_turns, total_tokens, max_seqlen) -> int:
    return int(load_library().opr_layout_workspace_bytes(n_seqs, n_convs, n_turns, total_tokens, max_seqlen))


def opr_attn_bwd_workspace_bytes(n_seqs, max_seqlen, hq, head_dim) -> int:
    return int(load_library().opr_attn_bwd_workspace_bytes(n_seqs, max_seqlen, hq, head_dim))


def opr_attn_bwd_min_workspace_bytes(n_seqs, max_seqlen, hq, head_dim) -> int:
    return int(load_library().opr_attn_bwd_min_workspace_bytes(n_seqs, max_seqlen, hq, head_dim))


@dataclass
class Layout:
    """Device outputs of opr_build_layout plus the sizes the attention calls need."""

    n_seqs: int
    n_convs: int
    n_turns: int
    total: int
    max_seqlen: int
    cu_seqlens: torch.Tensor
    token_type: torch.Tensor
    turn_idx: torch.Tensor
    conv_idx: torch.Tensor
    pos_id: torch.Tensor
    attn_pos: torch.Tensor  # row of each stream token in the attention order (q, k, v of the attention calls)
    block_map: torch.Tensor | None
    workspace: torch.Tensor
    dev_status: torch.Tensor

    @property
    def T(self) -> int:
        return (self.max_seqlen + TILE - 1) // TILE


def layout_table_offsets(lay: "Layout") -> dict[str, int]:
    """Byte offsets of the tile tables inside lay.workspace (test hook of include/opr_testing.h)."""
    out = (ctypes.c_uint64 * 4)()
    st = load_library().opr_testing_layout_tables(lay.n_seqs, lay.n_convs, lay.n_turns, lay.total, lay.max_seqlen,
                                                  ctypes.cast(out, ctypes.c_void_p))
    _check(st, "opr_testing_layout_tables")
    return dict(zip(("row_cnt", "row_list", "col_cnt", "col_list"), (int(x) for x in out)))


def read_status(dev_status: torch.Tensor) -> list[str]:
    """Synchronise and decode the device status word (empty list = no error)."""
    v = int(dev_status.item())
    return [name for bit, name in DEV_BITS.items() if v & bit]


def _lens_host(turn_lens, conv_turn_ptr, seq_conv_ptr):
    tl = np.asarray(turn_lens.cpu() if isinstance(turn_lens, torch.Tensor) else turn_lens, dtype=np.int64)
    cp = np.asarray(conv_turn_ptr.cpu() if isinstance(conv_turn_ptr, torch.Tensor) else conv_turn_ptr, dtype=np.int64)
    sp = np.asarray(seq_conv_ptr.cpu() if isinstance(seq_conv_ptr, torch.Tensor) else seq_conv_ptr, dtype=np.int64)
    return tl.reshape(-1, 3), cp, sp


def sizes_from_lengths(turn_lens, conv_turn_ptr, seq_conv_ptr) -> tuple[int, int]:
    """(total_tokens, max_seqlen) of host length arrays: token counts h + t + 2r."""
    tl, cp, sp = _lens_host(turn_lens, conv_turn_ptr, seq_conv_ptr)
    cost = tl[:, 0] + tl[:, 1] + 2 * tl[:, 2]
    csum = np.concatenate([[0], np.cumsum(cost)])
    seq_len = csum[cp[sp[1:]]] - csum[cp[sp[:-1]]]
    return int(cost.sum()), int(seq_len.max()) if seq_len.size else 0


def opr_build_layout(turn_lens, conv_turn_ptr, seq_conv_ptr, total_tokens=None, max_seqlen=None,
                     device="cuda", block_map: bool = True) -> Layout:
    """Run opr_build_layout.  Length arrays may be host (copied in) or device int32 tensors.
    ``block_map=False`` skips the stream-order block map (the attention calls do not read it)."""
    lib = load_library()
    device = torch.device(device)
    if total_tokens is None or max_seqlen is None:
        tot, ms = sizes_from_lengths(turn_lens, conv_turn_ptr, seq_conv_ptr)
        total_tokens = tot if total_tokens is None else total_tokens
        max_seqlen = ms if max_seqlen is None else max_seqlen

    def dev_i32(x):
        t = x if isinstance(x, torch.Tensor) else torch.as_tensor(np.asarray(x, dtype=np.int32))
        return t.to(device=device, dtype=torch.int32, non_blocking=True).contiguous()

    tl, cp, sp = dev_i32(turn_lens).reshape(-1), dev_i32(conv_turn_ptr), dev_i32(seq_conv_ptr)
    n_turns, n_convs, n_seqs = tl.numel() // 3, cp.numel() - 1, sp.numel() - 1
    T = (max_seqlen + TILE - 1) // TILE
    ws_bytes = opr_layout_workspace_bytes(n_seqs, n_convs, n_turns, total_tokens, max_seqlen)
    if ws_bytes == 0 and total_tokens > 0:
        raise OprError("sizes out of range for opr_build_layout")
    lay = Layout(
        n_seqs, n_convs, n_turns, int(total_tokens), int(max_seqlen),
        cu_seqlens=torch.empty(n_seqs + 1, dtype=torch.int32, device=device),
        token_type=torch.empty(total_tokens, dtype=torch.int8, device=device),
        turn_idx=torch.empty(total_tokens, dtype=torch.int32, device=device),
        conv_idx=torch.empty(total_tokens, dtype=torch.int32, device=device),
        pos_id=torch.empty(total_tokens, dtype=torch.int32, device=device),
        attn_pos=torch.empty(total_tokens, dtype=torch.int32, device=device),
        block_map=torch.empty((n_seqs, T, T), dtype=torch.uint8, device=device) if block_map else None,
        workspace=torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device),
        dev_status=torch.zeros(1, dtype=torch.int32, device=device),
    )
    st = lib.opr_build_layout(
        _ptr(tl), _ptr(cp), _ptr(sp), n_seqs, n_convs, n_turns, total_tokens, max_seqlen,
        _ptr(lay.cu_seqlens), _ptr(lay.token_type), _ptr(lay.turn_idx), _ptr(lay.conv_idx), _ptr(lay.pos_id),
        _ptr(lay.attn_pos), _ptr(lay.block_map), _ptr(lay.workspace), lay.workspace.numel(), _ptr(lay.dev_status),
        _stream(device))
    _check(st, "opr_build_layout")
    lay._inputs = (tl, cp, sp)  # keep the device copies alive until the stream has used them
    return lay


_DT = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_FP16, torch.float32: DTYPE_FP32}


def opr_rope(x: torch.Tensor, pos_id: torch.Tensor | None, base: float, inverse: bool = False,
             out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
             row_map: torch.Tensor | None = None) -> torch.Tensor:
    """Rotate x [total, heads, head_dim] by position id, into ``out`` (default: in place).

    x and out may be bf16, fp16 or fp32 (types may differ when out is not x).  With
    ``pos_id`` None there is no rotation, only the type conversion.  With ``row_map``
    (e.g. a layout's attn_pos) row t of x goes to row row_map[t] of out (out must not be x).
    """
    out = x if out is None else out
    _need_cuda(x, out, *(() if pos_id is None else (pos_id,)), *(() if row_map is None else (row_map,)))
    if row_map is not None and (row_map.dtype != torch.int32 or row_map.numel() != x.shape[0]):
        raise OprError("row_map must be int32 with one entry per row of x")
    if pos_id is not None and (pos_id.dtype != torch.int32 or pos_id.numel() != x.shape[0]):
        raise OprError("pos_id must be int32 with one entry per row of x")
    if out.device != x.device or any(t is not None and t.device != x.device for t in (pos_id, row_map)):
        raise OprError("opr_rope: every tensor must be on x's device")
    if x.dtype not in _DT or out.dtype not in _DT:
        raise OprError("opr_rope takes bf16, fp16 or fp32")
    if out.shape != x.shape:
        raise OprError("opr_rope: out must have the shape of x")
    total, heads, d = x.shape
    st = load_library().opr_rope(_ptr(x), _DT[x.dtype], _ptr(out), _DT[out.dtype], _ptr(pos_id), _ptr(row_map),
                                 total, heads, d,
                                 float(base), int(bool(inverse)), _ptr(dev_status), _stream(x.device))
    _check(st, "opr_rope")
    return out


def _attn_shapes(q, k, v, lay: Layout, v_types=(torch.bfloat16,)):
    _need_cuda(q, k, v)
    if q.dtype != torch.float16 or k.dtype != torch.float16:
        raise OprError("q and k must be fp16 (rotated by opr_rope with an fp16 output)")
    if v.dtype not in v_types:
        raise OprError("v must be " + " or ".join(str(t).replace("torch.", "") for t in v_types))
    total, hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != total or k.shape[2] != d or total != lay.total:
        raise OprError("shape mismatch between q, k, v and the layout")
    return total, hq, k.shape[1], d


def _grad_buffers(out, q, total, hq, hkv, d):
    """(dq, dk, dv): the caller's buffers after checking them, or new fp32 tensors."""
    shapes = ((total, hq, d), (total, hkv, d), (total, hkv, d))
    if out is None:
        return tuple(torch.empty(sh, dtype=torch.float32, device=q.device) for sh in shapes)
    if len(out) != 3:
        raise OprError("out must be (dq, dk, dv)")
    for name, t, sh in zip(("dq", "dk", "dv"), out, shapes):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or tuple(t.shape) != sh:
            raise OprError(f"out {name} must be an fp32 tensor of shape {sh}")
        if t.device != q.device or not t.is_contiguous():
            raise OprError(f"out {name} must be contiguous on {q.device}")
    return tuple(out)


def opr_attn_fwd(q, k, v, lay: Layout, scale: float | None = None, out_dtype=torch.float32):
    """O [total, hq, d] (out_dtype) and LSE [hq, total] fp32.  v is fp16 (P V in fp16, see
    include/opr.h) or bf16."""
    total, hq, hkv, d = _attn_shapes(q, k, v, lay, v_types=(torch.float16, torch.bfloat16))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty((total, hq, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((hq, total), dtype=torch.float32, device=q.device)
    st = load_library().opr_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _DT[v.dtype], _ptr(lay.cu_seqlens), _ptr(lay.conv_idx),
        _ptr(lay.workspace), lay.n_seqs, lay.n_convs, lay.n_turns, total, lay.max_seqlen, hq, hkv, d, float(scale),
        _ptr(o), DTYPE_FP32 if out_dtype == torch.float32 else DTYPE_BF16, _ptr(lse), _ptr(lay.dev_status),
        _stream(q.device))
    _check(st, "opr_attn_fwd")
    return o, lse


def _rope_args(rope_base, lay: Layout):
    """(pos_id pointer, base) of the rotation the backward undoes, or (None, 0)."""
    if rope_base is None:
        return None, 0.0
    return _ptr(lay.pos_id), float(rope_base)


def opr_attn_bwd(q, k, v, o, do, lse, lay: Layout, scale: float | None = None, workspace=None, out=None,
                 stages: int | None = None, rope_base: float | None = None):
    """dQ [total, hq, d], dK and dV [total, hkv, d] (fp32), w.r.t. the rotated q, k and v; with
    ``rope_base``, dQ and dK are rotated back by the layout's position ids (the gradients
    w.r.t. the unrotated q and k).

    ``out`` = (dq, dk, dv) reuses buffers; ``stages`` (OR of BWD_ROW_TERMS,
    BWD_DQ, BWD_DKDV) runs only those kernels through opr_attn_bwd_stages, with
    the row terms kept in ``workspace`` between calls.  A ``workspace`` below
    opr_attn_bwd_min_workspace_bytes is replaced by one of the recommended size;
    one between the two sizes is used as given (the dK/dV stage then runs unsplit).
    """
    total, hq, hkv, d = _attn_shapes(q, k, v, lay)
    _need_cuda(o, do, lse)
    if do.dtype != torch.bfloat16 or lse.dtype != torch.float32:
        raise OprError("dout must be bf16 and lse fp32")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = _grad_buffers(out, q, total, hq, hkv, d)
    wb = opr_attn_bwd_workspace_bytes(lay.n_seqs, lay.max_seqlen, hq, d)
    if workspace is None or workspace.numel() < opr_attn_bwd_min_workspace_bytes(lay.n_seqs, lay.max_seqlen, hq, d):
        workspace = torch.empty(max(wb, 256), dtype=torch.uint8, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(o), DTYPE_FP32 if o.dtype == torch.float32 else DTYPE_BF16, _ptr(do),
            _ptr(lse), _ptr(lay.cu_seqlens), _ptr(lay.conv_idx), _ptr(lay.workspace), lay.n_seqs, lay.n_convs,
            lay.n_turns, total, lay.max_seqlen, hq, hkv, d, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
            *_rope_args(rope_base, lay), _ptr(workspace), workspace.numel(), _ptr(lay.dev_status))
    lib = load_library()
    if stages is None:
        _check(lib.opr_attn_bwd(*args, _stream(q.device)), "opr_attn_bwd")
    else:
        _check(lib.opr_attn_bwd_stages(*args, int(stages), _stream(q.device)), "opr_attn_bwd_stages")
    return dq, dk, dv


def opr_attn_bwd_stages(q, k, v, o, do, lse, lay: Layout, stages: int, workspace, out, scale=None, rope_base=None):
    """Run only the backward kernels selected by ``stages`` (see opr_attn_bwd)."""
    return opr_attn_bwd(q, k, v, o, do, lse, lay, scale, workspace=workspace, out=out, stages=stages,
                        rope_base=rope_base)


def opr_attn_bwd_noalloc(q, k, v, o, do, lse, lay: Layout, scale: float | None = None, out=None,
                         rope_base: float | None = None):
    """opr_attn_bwd with the scratch in the library's fixed device array (no workspace argument).

    For callers that cannot allocate device memory at the call; see the C
    header for the size limit and the sharing rules of the array.  ``out`` =
    (dq, dk, dv) lets the caller provide the output buffers too.
    """
    total, hq, hkv, d = _attn_shapes(q, k, v, lay)
    _need_cuda(o, do, lse)
    if do.dtype != torch.bfloat16 or lse.dtype != torch.float32:
        raise OprError("dout must be bf16 and lse fp32")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = _grad_buffers(out, q, total, hq, hkv, d)
    with torch.cuda.device(q.device):  # the library uses the current device's array
        st = load_library().opr_attn_bwd_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(o), DTYPE_FP32 if o.dtype == torch.float32 else DTYPE_BF16,
            _ptr(do), _ptr(lse), _ptr(lay.cu_seqlens), _ptr(lay.conv_idx), _ptr(lay.workspace), lay.n_seqs,
            lay.n_convs, lay.n_turns, total, lay.max_seqlen, hq, hkv, d, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
            *_rope_args(rope_base, lay), _ptr(lay.dev_status), _stream(q.device))
    _check(st, "opr_attn_bwd_noalloc")
    return dq, dk, dv


# ------------------------------------------------------------------ token duplication
def opr_duplication_index(turn_lens, conv_turn_ptr, total_tokens=None, orig_tokens=None, device="cuda",
                          dev_status: torch.Tensor | None = None):
    """(src_index [total], copy_index [orig, 2]) int32 device tensors: the one-pass stream
    (h, t, r^in, r^out per turn) as copies of the original stream (h, t, r per turn)."""
    lib = load_library()
    device = torch.device(device)

    def dev_i32(x):
        t = x if isinstance(x, torch.Tensor) else torch.as_tensor(np.asarray(x, dtype=np.int32))
        return t.to(device=device, dtype=torch.int32).contiguous()

    tl, cp = dev_i32(turn_lens).reshape(-1), dev_i32(conv_turn_ptr)
    if total_tokens is None or orig_tokens is None:
        lens = np.asarray(turn_lens.cpu() if isinstance(turn_lens, torch.Tensor) else turn_lens,
                          dtype=np.int64).reshape(-1, 3)
        lens = np.maximum(lens, 0)
        total_tokens = int(lens[:, 0].sum() + lens[:, 1].sum() + 2 * lens[:, 2].sum()) \
            if total_tokens is None else total_tokens
        orig_tokens = int(lens.sum()) if orig_tokens is None else orig_tokens
    src = torch.empty(total_tokens, dtype=torch.int32, device=device)
    copies = torch.empty((orig_tokens, 2), dtype=torch.int32, device=device)
    status = dev_status if dev_status is not None else torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib.opr_duplication_index(_ptr(tl), _ptr(cp), cp.numel() - 1, tl.numel() // 3, total_tokens, orig_tokens,
                                     _ptr(src), _ptr(copies), _ptr(status), _stream(device)),
           "opr_duplication_index")
    src._inputs = (tl, cp, status)  # keep the device copies alive until the stream has used them
    return src, copies


def opr_gather_rows(x: torch.Tensor, src_index: torch.Tensor, out: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """out[i] = x[src_index[i]] along the first dimension (any dtype, rows contiguous)."""
    _need_cuda(x, src_index)
    if src_index.dtype != torch.int32 or src_index.device != x.device:
        raise OprError("opr_gather_rows: src_index must be int32 on x's device")
    rows = src_index.numel()
    if out is None:
        out = torch.empty((rows,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    _need_cuda(out)
    if out.shape[0] != rows or out.shape[1:] != x.shape[1:] or out.dtype != x.dtype or out.device != x.device:
        raise OprError("opr_gather_rows: out must be [len(src_index)] rows of x's row shape and dtype, on x's device")
    row_bytes = x[0].numel() * x.element_size() if x.shape[0] > 0 else out[0].numel() * out.element_size()
    _check(lib_call("opr_gather_rows", _ptr(x), x.shape[0], row_bytes, _ptr(src_index), rows, _ptr(out),
                    _ptr(dev_status) if dev_status is not None else None, _stream(x.device)), "opr_gather_rows")
    return out


def opr_fold_rows(dy: torch.Tensor, copy_index: torch.Tensor, out: torch.Tensor | None = None,
                  dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Gradient of opr_gather_rows: out[o] = sum over the slots of copy_index[o] that are >= 0 of
    dy[copy_index[o, k]], in slot order (fp32); copy_index [orig, slots]."""
    _need_cuda(dy, copy_index)
    if dy.dtype != torch.float32:
        raise OprError("opr_fold_rows: dy must be fp32")
    if copy_index.dtype != torch.int32 or copy_index.dim() != 2 or copy_index.device != dy.device:
        raise OprError("opr_fold_rows: copy_index must be int32 [orig, slots] on dy's device")
    rows = copy_index.shape[0]
    if out is None:
        out = torch.empty((rows,) + tuple(dy.shape[1:]), dtype=torch.float32, device=dy.device)
    _need_cuda(out)
    if out.dtype != torch.float32 or tuple(out.shape) != (rows,) + tuple(dy.shape[1:]) or out.device != dy.device:
        raise OprError("opr_fold_rows: out must be fp32 [len(copy_index)] rows of dy's row shape, on dy's device")
    width = int(np.prod(dy.shape[1:])) if dy.dim() > 1 else 1
    _check(lib_call("opr_fold_rows", _ptr(dy), dy.shape[0], width, _ptr(copy_index), copy_index.shape[1], rows, _ptr(out),
                    _ptr(dev_status) if dev_status is not None else None, _stream(dy.device)), "opr_fold_rows")
    return out


def lib_call(name: str, *args) -> int:
    return int(getattr(load_library(), name)(*args))


# ------------------------------------------------------------------ K-pass
@dataclass
class KPass:
    """The K-pass arrangement of a batch as layout inputs, plus its token map."""

    K: int
    turn_lens: torch.Tensor        # int32 [n_out_turns, 3]
    conv_turn_ptr: torch.Tensor    # int32 [n_out_convs + 1]
    seq_conv_ptr: torch.Tensor     # int32 [n_seqs + 1]
    turn_src: torch.Tensor         # int32 [n_out_turns, 2]
    src_index: torch.Tensor        # int32 [total_tokens]
    copy_index: torch.Tensor       # int32 [orig_tokens, K + 1]
    total_tokens: int
    max_seqlen: int
    dev_status: torch.Tensor


def opr_kpass(turn_lens, conv_turn_ptr, seq_conv_ptr, K: int, device="cuda") -> KPass:
    """opr_kpass_sizes, opr_kpass_plan and opr_kpass_index in one call.  Length arrays are host
    arrays (sizes are taken from them before the device work)."""
    lib = load_library()
    device = torch.device(device)
    lens = np.asarray(turn_lens, dtype=np.int32).reshape(-1, 3)
    cp = np.ascontiguousarray(np.asarray(conv_turn_ptr, dtype=np.int32))
    sp = np.ascontiguousarray(np.asarray(seq_conv_ptr, dtype=np.int32))
    n_turns, n_convs, n_seqs = lens.shape[0], cp.size - 1, sp.size - 1
    sizes = [ctypes.c_int64(0) for _ in range(5)]
    lens_flat = np.ascontiguousarray(lens.reshape(-1))
    _check(lib.opr_kpass_sizes(lens_flat.ctypes.data, cp.ctypes.data, sp.ctypes.data, n_seqs, n_convs, n_turns, K,
                               *(ctypes.byref(x) for x in sizes)), "opr_kpass_sizes")
    n_out_turns, n_out_convs, total, max_seqlen, orig = (x.value for x in sizes)
    dev = lambda a: torch.as_tensor(a).to(device=device, dtype=torch.int32).contiguous()  # noqa: E731
    tl, cpd, spd = dev(lens.reshape(-1)), dev(cp), dev(sp)
    out_lens = torch.empty((n_out_turns, 3), dtype=torch.int32, device=device)
    out_cp = torch.empty(n_out_convs + 1, dtype=torch.int32, device=device)
    out_sp = torch.empty(n_seqs + 1, dtype=torch.int32, device=device)
    out_src = torch.empty((n_out_turns, 2), dtype=torch.int32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib.opr_kpass_plan(_ptr(tl), _ptr(cpd), _ptr(spd), n_seqs, n_convs, n_turns, K, n_out_turns, n_out_convs,
                              _ptr(out_lens), _ptr(out_cp), _ptr(out_sp), _ptr(out_src), _ptr(status),
                              _stream(device)), "opr_kpass_plan")
    slots = K + 1
    src = torch.empty(total, dtype=torch.int32, device=device)
    copies = torch.empty((orig, slots), dtype=torch.int32, device=device)
    ws = torch.empty(max(int(lib.opr_kpass_index_workspace_bytes(n_turns, n_out_turns)), 256), dtype=torch.uint8,
                     device=device)
    _check(lib.opr_kpass_index(_ptr(tl), n_turns, _ptr(out_lens), _ptr(out_src), n_out_turns, total, orig, slots,
                               _ptr(src), _ptr(copies), _ptr(ws), ws.numel(), _ptr(status), _stream(device)),
           "opr_kpass_index")
    kp = KPass(K, out_lens, out_cp, out_sp, out_src, src, copies, total, max_seqlen, status)
    kp._keep = (tl, cpd, spd, ws)  # alive until the stream has used them
    return kp


# ------------------------------------------------------------------ loss side
def opr_loss_rows(turn_lens, device="cuda", dev_status: torch.Tensor | None = None):
    """(rows, targets) int32 device tensors: the one-pass rows carrying the N-pass next-token
    losses and the original-stream index of each row's target token."""
    lib = load_library()
    device = torch.device(device)
    lens = np.ascontiguousarray(np.asarray(turn_lens, dtype=np.int32).reshape(-1, 3))
    n_turns = lens.shape[0]
    n_rows = int(lib.opr_loss_row_count(lens.ctypes.data, n_turns))
    if n_rows < 0:
        raise OprError("opr_loss_row_count: negative lengths")
    l64 = np.maximum(lens.astype(np.int64), 0)
    total = int(l64[:, 0].sum() + l64[:, 1].sum() + 2 * l64[:, 2].sum())
    orig = int(l64.sum())
    tl = torch.as_tensor(lens.reshape(-1)).to(device)
    rows = torch.empty(n_rows, dtype=torch.int32, device=device)
    targets = torch.empty(n_rows, dtype=torch.int32, device=device)
    status = dev_status if dev_status is not None else torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib.opr_loss_rows(_ptr(tl), n_turns, total, orig, n_rows, _ptr(rows), _ptr(targets), _ptr(status),
                             _stream(device)), "opr_loss_rows")
    rows._inputs = (tl, status)
    return rows, targets


def opr_cross_entropy(logits: torch.Tensor, target_ids: torch.Tensor, grad_scale: float = 1.0,
                      with_grad: bool = True, dev_status: torch.Tensor | None = None):
    """(loss fp32 [n], dlogits [n, V] in the logits' dtype or None): fused softmax cross-entropy."""
    _need_cuda(logits, target_ids)
    if logits.dtype not in (torch.bfloat16, torch.float32) or logits.dim() != 2:
        raise OprError("opr_cross_entropy: logits must be [n, V] bf16 or fp32")
    n, V = logits.shape
    loss = torch.empty(n, dtype=torch.float32, device=logits.device)
    dl = torch.empty_like(logits) if with_grad else None
    status = dev_status if dev_status is not None else torch.zeros(1, dtype=torch.int32, device=logits.device)
    _check(load_library().opr_cross_entropy(_ptr(logits), _DT[logits.dtype], n, V, _ptr(target_ids), _ptr(loss),
                                            _ptr(dl), grad_scale, _ptr(status), _stream(logits.device)),
           "opr_cross_entropy")
    loss._status = status
    return loss, dl
