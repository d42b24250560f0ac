"""Python binding of libmla_b200.so, the sm_100a absorbed-MLA decode library.

Argument marshalling only: each function checks the torch tensors it is given
(dtype, device, contiguity, shape), turns them into raw pointers and sizes, and
calls the C entry point of the same name (include/mla.h).  Every step of the
decode path runs in the library's CUDA kernels; there is no CPU fallback, and
importing the binding fails loudly when the shared library has not been built.

    import head_latent_attention_07_b200 as mla
    dims = mla.MlaDims(n_heads=128, d_c=512, d_rope=64, qk_nope=128, v_head=128,
                       d_model=7168, page_size=64)
    mla.mla_query_proj(dims, h, w_dq, w_uq, c_q, q)          # q-LoRA query path (optional)
    mla.mla_append_latent(dims, h, w_dkv, seq_idx, pos, page_table, pool)
    mla.mla_absorb_q(dims, q, pos, w_uk, q_lat)
    # or both in one launch: mla.mla_append_absorb(dims, h, w_dkv, seq_idx, pos, page_table, pool, q, w_uk, q_lat)
    mla.mla_decode_attn(dims, q_lat, pool, page_table, seq_lens, w_uv, workspace, out, lse)
    mla.mla_out_proj(dims, out, w_o, y)                       # layer output (optional)

Context split of long sequences over ranks: mla_decode_attn_partial on each
rank's window, then mla_merge_ranks (see context_split.py for the process-group
form).
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_b200.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_MISALIGNED = -3
MLA_ERR_WORKSPACE = -4
MLA_ERR_CUDA = -5
MLA_ERR_TIMEOUT = -6
MLA_ERR_RANGE = -7

# Every entry point declared in include/mla.h, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int32
SIGNATURES = {
    "mla_append_latent": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _I, _I, _P, _P]),
    "mla_absorb_q": (ctypes.c_int, [_P, _P, _P, _P, _P, _I, _P]),
    "mla_append_absorb": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _I, _P, _P]),
    "mla_decode_workspace_bytes": (ctypes.c_size_t, [_P, _I, _I]),
    "mla_decode_attn": (ctypes.c_int, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, ctypes.c_size_t,
                                       _P, _P, _P, _P]),
    "mla_decode_attn_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "mla_decode_attn_partial": (ctypes.c_int, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, ctypes.c_size_t,
                                               _P, _P, _P, _P]),
    "mla_merge_ranks": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p), _I, _I,
                                       _P, _P, _P, _P]),
    "mla_out_proj": (ctypes.c_int, [_P, _P, _P, _P, _I, _P]),
    "mla_query_proj": (ctypes.c_int, [_P, _I, _P, _P, _P, _P, _P, _I, _P]),
    "mla_status_read": (ctypes.c_int, [_P, _P]),
    "mla_status_clear": (ctypes.c_int, [_P, _P]),
    "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_last_cuda_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_char_p)]),
    "mla_version": (ctypes.c_char_p, []),
}


class MlaDims(ctypes.Structure):
    """mirror of `mla_dims` in include/mla.h"""
    _fields_ = [("n_heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("qk_nope", ctypes.c_int32), ("v_head", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("rope_theta", ctypes.c_float)]

    @property
    def row(self) -> int:
        return self.d_c + self.d_rope


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} ({status})"
        if status == MLA_ERR_CUDA:
            name = ctypes.c_char_p()
            code = load_library().mla_last_cuda_error(ctypes.byref(name))
            msg += f" [{name.value.decode() if name.value else '?'} ({code})]"
        super().__init__(msg)


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (once) and declare its signatures.  Raises
    FileNotFoundError when it has not been built: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise FileNotFoundError(
                f"{path} is missing; build it with `python -m head_latent_attention_07_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().mla_status_string(int(status)).decode()


def version() -> str:
    return load_library().mla_version().decode()


# ------------------------------------------------------------------ marshalling helpers

def _torch():
    import torch
    return torch


def _ptr(t, dtype, name, ndim=None):
    torch = _torch()
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != MLA_OK:
        raise MlaError(status, where)


def _shape(t, expect, name):
    if tuple(t.shape) != tuple(expect):
        raise ValueError(f"{name} must have shape {tuple(expect)}, got {tuple(t.shape)}")


# ------------------------------------------------------------------ entry points

def mla_append_latent(dims: MlaDims, h, w_dkv, seq_idx, pos, page_table, pool,
                      dev_status=None, stream=None) -> None:
    """Write [W_DKV h || RoPE(W_KR h, pos)] of each token into its paged cache slot."""
    torch = _torch()
    T = h.shape[0]
    B, max_pages = page_table.shape
    num_pages = pool.shape[0]
    _shape(h, (T, dims.d_model), "h")
    _shape(w_dkv, (dims.row, dims.d_model), "w_dkv")
    _shape(seq_idx, (T,), "seq_idx")
    _shape(pos, (T,), "pos")
    _shape(pool, (num_pages, dims.page_size, dims.row), "pool")
    st = load_library().mla_append_latent(
        ctypes.byref(dims), _ptr(h, torch.bfloat16, "h"), _ptr(w_dkv, torch.bfloat16, "w_dkv"),
        _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(pos, torch.int32, "pos"),
        _ptr(page_table, torch.int32, "page_table"), B, max_pages,
        _ptr(pool, torch.bfloat16, "pool"), num_pages, T,
        _ptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(st, "mla_append_latent")


def mla_absorb_q(dims: MlaDims, q, pos, w_uk, q_lat, stream=None) -> None:
    """q_lat[t, h] = [W_UK,h^T q_nope || RoPE(q_rope, pos[t])]."""
    torch = _torch()
    T = q.shape[0]
    _shape(q, (T, dims.n_heads, dims.qk_nope + dims.d_rope), "q")
    _shape(pos, (T,), "pos")
    _shape(w_uk, (dims.n_heads, dims.qk_nope, dims.d_c), "w_uk")
    _shape(q_lat, (T, dims.n_heads, dims.row), "q_lat")
    st = load_library().mla_absorb_q(
        ctypes.byref(dims), _ptr(q, torch.bfloat16, "q"), _ptr(pos, torch.int32, "pos"),
        _ptr(w_uk, torch.bfloat16, "w_uk"), _ptr(q_lat, torch.bfloat16, "q_lat"), T, _stream(stream))
    _check(st, "mla_absorb_q")


def mla_append_absorb(dims: MlaDims, h, w_dkv, seq_idx, pos, page_table, pool, q, w_uk, q_lat,
                      dev_status=None, stream=None) -> None:
    """mla_append_latent and mla_absorb_q of one decode step (the same tokens and
    positions) in one call."""
    torch = _torch()
    T = h.shape[0]
    B, max_pages = page_table.shape
    num_pages = pool.shape[0]
    _shape(h, (T, dims.d_model), "h")
    _shape(w_dkv, (dims.row, dims.d_model), "w_dkv")
    _shape(seq_idx, (T,), "seq_idx")
    _shape(pos, (T,), "pos")
    _shape(pool, (num_pages, dims.page_size, dims.row), "pool")
    _shape(q, (T, dims.n_heads, dims.qk_nope + dims.d_rope), "q")
    _shape(w_uk, (dims.n_heads, dims.qk_nope, dims.d_c), "w_uk")
    _shape(q_lat, (T, dims.n_heads, dims.row), "q_lat")
    st = load_library().mla_append_absorb(
        ctypes.byref(dims), _ptr(h, torch.bfloat16, "h"), _ptr(w_dkv, torch.bfloat16, "w_dkv"),
        _ptr(seq_idx, torch.int32, "seq_idx"), _ptr(pos, torch.int32, "pos"),
        _ptr(page_table, torch.int32, "page_table"), B, max_pages,
        _ptr(pool, torch.bfloat16, "pool"), num_pages, _ptr(q, torch.bfloat16, "q"),
        _ptr(w_uk, torch.bfloat16, "w_uk"), _ptr(q_lat, torch.bfloat16, "q_lat"), T,
        _ptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(st, "mla_append_absorb")


def mla_decode_workspace_bytes(dims: MlaDims, batch: int, nq: int) -> int:
    n = load_library().mla_decode_workspace_bytes(ctypes.byref(dims), batch, nq)
    if n == 0:
        raise MlaError(MLA_ERR_INVALID_ARG, "mla_decode_workspace_bytes")
    return n


def mla_decode_attn(dims: MlaDims, q_lat, pool, page_table, seq_lens, w_uv, workspace, out,
                    lse=None, dev_status=None, stream=None) -> None:
    """Absorbed attention of q_lat [B, nq, H, d_c+d_rope] over the paged cache,
    split-KV with a log-sum-exp combine, then W_UV: out [B, nq, H, v_head]."""
    torch = _torch()
    B, nq = q_lat.shape[0], q_lat.shape[1]
    _shape(q_lat, (B, nq, dims.n_heads, dims.row), "q_lat")
    num_pages = pool.shape[0]
    _shape(pool, (num_pages, dims.page_size, dims.row), "pool")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    max_pages = page_table.shape[1]
    _shape(seq_lens, (B,), "seq_lens")
    _shape(w_uv, (dims.n_heads, dims.v_head, dims.d_c), "w_uv")
    _shape(out, (B, nq, dims.n_heads, dims.v_head), "out")
    if lse is not None:
        _shape(lse, (B, nq, dims.n_heads), "lse")
    if workspace.dtype != torch.uint8 or workspace.dim() != 1:
        raise TypeError("workspace must be a 1-D uint8 tensor")
    st = load_library().mla_decode_attn(
        ctypes.byref(dims), _ptr(q_lat, torch.bfloat16, "q_lat"), _ptr(pool, torch.bfloat16, "pool"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        B, nq, max_pages, num_pages, _ptr(w_uv, torch.bfloat16, "w_uv"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(st, "mla_decode_attn")


def mla_decode_attn_noalloc(dims: MlaDims, q_lat, pool, page_table, seq_lens, w_uv, out,
                            lse=None, dev_status=None, stream=None) -> None:
    """mla_decode_attn without a caller workspace: the library's own 64 MiB device
    scratch is used instead (see include/mla.h for the sharing rules)."""
    torch = _torch()
    B, nq = q_lat.shape[0], q_lat.shape[1]
    _shape(q_lat, (B, nq, dims.n_heads, dims.row), "q_lat")
    num_pages = pool.shape[0]
    _shape(pool, (num_pages, dims.page_size, dims.row), "pool")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    _shape(seq_lens, (B,), "seq_lens")
    _shape(w_uv, (dims.n_heads, dims.v_head, dims.d_c), "w_uv")
    _shape(out, (B, nq, dims.n_heads, dims.v_head), "out")
    if lse is not None:
        _shape(lse, (B, nq, dims.n_heads), "lse")
    st = load_library().mla_decode_attn_noalloc(
        ctypes.byref(dims), _ptr(q_lat, torch.bfloat16, "q_lat"), _ptr(pool, torch.bfloat16, "pool"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        B, nq, page_table.shape[1], num_pages, _ptr(w_uv, torch.bfloat16, "w_uv"),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(st, "mla_decode_attn_noalloc")


def mla_decode_attn_partial(dims: MlaDims, q_lat, pool, page_table, seq_lens, kv_rank: int, kv_ranks: int,
                            workspace, o_lat, lse, dev_status=None, stream=None) -> None:
    """Rank kv_rank's window of a context-split decode: o_lat [B, nq, H, d_c] (fp32)
    and lse [B, nq, H] over pages [P_b r / R, P_b (r+1) / R) of each sequence."""
    torch = _torch()
    B, nq = q_lat.shape[0], q_lat.shape[1]
    _shape(q_lat, (B, nq, dims.n_heads, dims.row), "q_lat")
    num_pages = pool.shape[0]
    _shape(pool, (num_pages, dims.page_size, dims.row), "pool")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    _shape(seq_lens, (B,), "seq_lens")
    _shape(o_lat, (B, nq, dims.n_heads, dims.d_c), "o_lat")
    _shape(lse, (B, nq, dims.n_heads), "lse")
    if workspace.dtype != torch.uint8 or workspace.dim() != 1:
        raise TypeError("workspace must be a 1-D uint8 tensor")
    st = load_library().mla_decode_attn_partial(
        ctypes.byref(dims), _ptr(q_lat, torch.bfloat16, "q_lat"), _ptr(pool, torch.bfloat16, "pool"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        B, nq, page_table.shape[1], num_pages, kv_rank, kv_ranks,
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _ptr(o_lat, torch.float32, "o_lat"), _ptr(lse, torch.float32, "lse"),
        _ptr(dev_status, torch.int32, "dev_status"), _stream(stream))
    _check(st, "mla_decode_attn_partial")


def mla_merge_ranks(dims: MlaDims, o_lats, lses, w_uv, out, lse=None, stream=None) -> None:
    """Merge the ranks' (o_lat [T, H, d_c], lse [T, H]) partials by log-sum-exp, then
    W_UV: out [T, H, v_head].  o_lats / lses are sequences of tensors (one per rank;
    [B, nq, ...] shapes are accepted as T = B * nq)."""
    torch = _torch()
    R = len(o_lats)
    if R != len(lses) or R < 1:
        raise ValueError("one o_lat and one lse per rank")
    if out.dim() < 3 or tuple(out.shape[-2:]) != (dims.n_heads, dims.v_head):
        raise ValueError(f"out must be [..., {dims.n_heads}, {dims.v_head}], got {tuple(out.shape)}")
    T = out.numel() // (dims.n_heads * dims.v_head)
    _shape(w_uv, (dims.n_heads, dims.v_head, dims.d_c), "w_uv")
    for o, l in zip(o_lats, lses):
        if tuple(o.shape[-2:]) != (dims.n_heads, dims.d_c) or o.numel() != T * dims.n_heads * dims.d_c:
            raise ValueError(f"each o_lat must be [..., {dims.n_heads}, {dims.d_c}] with T = {T} tokens")
        if l.shape[-1] != dims.n_heads or l.numel() != T * dims.n_heads:
            raise ValueError(f"each lse must be [..., {dims.n_heads}] with T = {T} tokens")
    if lse is not None and (lse.shape[-1] != dims.n_heads or lse.numel() != T * dims.n_heads):
        raise ValueError(f"lse must be [..., {dims.n_heads}] with T = {T} tokens")
    po = (ctypes.c_void_p * R)(*[_ptr(o, torch.float32, "o_lat").value for o in o_lats])
    pl = (ctypes.c_void_p * R)(*[_ptr(l, torch.float32, "lse").value for l in lses])
    st = load_library().mla_merge_ranks(
        ctypes.byref(dims), po, pl, R, T, _ptr(w_uv, torch.bfloat16, "w_uv"), _ptr(out, torch.bfloat16, "out"),
        _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(st, "mla_merge_ranks")


def mla_out_proj(dims: MlaDims, o, w_o, y, stream=None) -> None:
    """Layer output y [T, d_model] = W_O concat_h(o[t, h]) for o [T, H, v_head]
    (or the [B, nq, H, v_head] output of mla_decode_attn)."""
    torch = _torch()
    T = o.numel() // (dims.n_heads * dims.v_head) if o.dim() >= 2 else -1
    if o.dim() < 3 or tuple(o.shape[-2:]) != (dims.n_heads, dims.v_head):
        raise ValueError(f"o must be [..., {dims.n_heads}, {dims.v_head}], got {tuple(o.shape)}")
    _shape(w_o, (dims.d_model, dims.n_heads * dims.v_head), "w_o")
    _shape(y, (T, dims.d_model), "y")
    st = load_library().mla_out_proj(
        ctypes.byref(dims), _ptr(o, torch.bfloat16, "o"), _ptr(w_o, torch.bfloat16, "w_o"),
        _ptr(y, torch.bfloat16, "y"), T, _stream(stream))
    _check(st, "mla_out_proj")


def mla_query_proj(dims: MlaDims, h, w_dq, w_uq, c_q, q, stream=None) -> None:
    """c_q [T, q_lora_rank] = W_DQ h, then q [T, H, qk_nope + d_rope] = W_UQ c_q."""
    torch = _torch()
    T = h.shape[0]
    r = w_dq.shape[0]
    _shape(h, (T, dims.d_model), "h")
    _shape(w_dq, (r, dims.d_model), "w_dq")
    _shape(w_uq, (dims.n_heads * (dims.qk_nope + dims.d_rope), r), "w_uq")
    _shape(c_q, (T, r), "c_q")
    _shape(q, (T, dims.n_heads, dims.qk_nope + dims.d_rope), "q")
    st = load_library().mla_query_proj(
        ctypes.byref(dims), r, _ptr(h, torch.bfloat16, "h"), _ptr(w_dq, torch.bfloat16, "w_dq"),
        _ptr(w_uq, torch.bfloat16, "w_uq"), _ptr(c_q, torch.bfloat16, "c_q"), _ptr(q, torch.bfloat16, "q"),
        T, _stream(stream))
    _check(st, "mla_query_proj")


def mla_status_read(dev_status, stream=None) -> int:
    """Synchronise `stream` and return the status recorded on the device."""
    torch = _torch()
    return load_library().mla_status_read(_ptr(dev_status, torch.int32, "dev_status"), _stream(stream))


def mla_status_clear(dev_status, stream=None) -> None:
    torch = _torch()
    _check(load_library().mla_status_clear(_ptr(dev_status, torch.int32, "dev_status"), _stream(stream)),
           "mla_status_clear")
