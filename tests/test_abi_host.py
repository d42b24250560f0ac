"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/mla.h declares, and rejects bad arguments before
launching anything."""
import ctypes
import os
import re

import pytest
import torch

import head_latent_attention_07_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|size_t|char\s*\*|void)\s*\**\s*(mla_\w+)\s*\(",
                                 text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(M.LIB_PATH):
        from head_latent_attention_07_b200 import build
        build.build()
    return M.load_library()


def test_header_declares_the_three_calls():
    names = declared_entry_points()
    for n in ("mla_append_latent", "mla_absorb_q", "mla_decode_attn"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_entry_points()
    assert names, "no entry points parsed from include/mla.h"
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/mla.h but not exported"
    # and the binding declares a signature for every one of them
    assert sorted(M.SIGNATURES) == names


def test_version_and_status_strings(lib):
    assert "sm_100a" in M.version()
    for code in range(0, -8, -1):
        s = M.status_string(code)
        assert s.startswith("MLA_"), s
    assert M.status_string(-99) == "unknown mla_status"


def v3_dims(**kw):
    d = dict(n_heads=128, d_c=512, d_rope=64, qk_nope=128, v_head=128, d_model=7168, page_size=64,
             softmax_scale=0.0, rope_theta=0.0)
    d.update(kw)
    return M.MlaDims(**d)


FAKE = 1 << 20          # 16-byte aligned fake device address (never dereferenced)
FAKE_MIS = FAKE + 2     # misaligned


def absorb(lib, dims, q=FAKE, pos=FAKE, w=FAKE, out=FAKE, n=4):
    return lib.mla_absorb_q(ctypes.byref(dims) if dims is not None else None, q, pos, w, out, n, None)


def test_absorb_argument_checks(lib):
    assert absorb(lib, None) == M.MLA_ERR_INVALID_ARG
    assert absorb(lib, v3_dims(d_rope=0)) == M.MLA_ERR_UNSUPPORTED     # no decoupled RoPE: refuse
    assert absorb(lib, v3_dims(n_heads=129)) == M.MLA_ERR_UNSUPPORTED
    assert absorb(lib, v3_dims(d_c=520 + 8)) == M.MLA_ERR_UNSUPPORTED
    assert absorb(lib, v3_dims(d_c=500)) == M.MLA_ERR_UNSUPPORTED
    assert absorb(lib, v3_dims(n_heads=0)) == M.MLA_ERR_INVALID_ARG
    assert absorb(lib, v3_dims(softmax_scale=float("nan"))) == M.MLA_ERR_INVALID_ARG
    assert absorb(lib, v3_dims(), q=None) == M.MLA_ERR_INVALID_ARG
    assert absorb(lib, v3_dims(), q=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert absorb(lib, v3_dims(), n=-1) == M.MLA_ERR_INVALID_ARG
    assert absorb(lib, v3_dims(), q=None, n=0) == M.MLA_OK              # empty: no-op


def test_append_argument_checks(lib):
    d = v3_dims()
    call = lambda **kw: lib.mla_append_latent(
        ctypes.byref(d), kw.get("h", FAKE), FAKE, FAKE, FAKE, FAKE, kw.get("B", 2), kw.get("mp", 4),
        kw.get("pool", FAKE), kw.get("np_", 8), kw.get("T", 2), kw.get("st", None), None)
    assert call(h=None) == M.MLA_ERR_INVALID_ARG
    assert call(pool=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(st=FAKE + 4) == M.MLA_ERR_MISALIGNED
    assert call(B=0) == M.MLA_ERR_INVALID_ARG
    assert call(np_=0) == M.MLA_ERR_INVALID_ARG
    assert call(T=0, h=None) == M.MLA_OK


def test_append_absorb_argument_checks(lib):
    # the checks of both calls it stands for, before any launch
    d = v3_dims()
    call = lambda dims=d, **kw: lib.mla_append_absorb(
        ctypes.byref(dims) if dims is not None else None, kw.get("h", FAKE), FAKE, FAKE, kw.get("pos", FAKE),
        FAKE, kw.get("B", 2), 4, kw.get("pool", FAKE), 8, kw.get("q", FAKE), FAKE, kw.get("q_lat", FAKE),
        kw.get("T", 2), kw.get("st", None), None)
    assert call(dims=None) == M.MLA_ERR_INVALID_ARG
    assert call(dims=v3_dims(d_rope=0)) == M.MLA_ERR_UNSUPPORTED
    assert call(h=None) == M.MLA_ERR_INVALID_ARG
    assert call(q=None) == M.MLA_ERR_INVALID_ARG
    assert call(q_lat=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(pool=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(pos=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(st=FAKE + 4) == M.MLA_ERR_MISALIGNED
    assert call(B=0) == M.MLA_ERR_INVALID_ARG
    assert call(T=-1) == M.MLA_ERR_INVALID_ARG
    assert call(T=0, h=None, q=None) == M.MLA_OK                      # empty: no-op


def test_decode_argument_checks(lib):
    d = v3_dims()
    def call(**kw):
        return lib.mla_decode_attn(
            ctypes.byref(d), kw.get("q", FAKE), FAKE, FAKE, FAKE, kw.get("B", 2), kw.get("nq", 1),
            kw.get("mp", 4), 8, FAKE, kw.get("ws", FAKE), kw.get("wsb", 1 << 30), kw.get("out", FAKE),
            kw.get("lse", None), None, None)
    assert call(q=None) == M.MLA_ERR_INVALID_ARG
    assert call(ws=None) == M.MLA_ERR_INVALID_ARG
    assert call(B=0) == M.MLA_ERR_INVALID_ARG
    assert call(nq=0) == M.MLA_ERR_INVALID_ARG
    assert call(B=1025) == M.MLA_ERR_UNSUPPORTED
    assert call(nq=1025) == M.MLA_ERR_UNSUPPORTED
    assert call(B=1000, nq=1000) == M.MLA_ERR_UNSUPPORTED     # batch * nq above 2^18
    assert call(mp=1 << 26) == M.MLA_ERR_UNSUPPORTED       # max_pages * page overflows int32
    assert call(out=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(lse=FAKE + 4) == M.MLA_ERR_MISALIGNED


def test_workspace_query_rejects_bad_arguments(lib):
    assert lib.mla_decode_workspace_bytes(ctypes.byref(v3_dims()), 0, 1) == 0
    assert lib.mla_decode_workspace_bytes(ctypes.byref(v3_dims()), 1, 0) == 0
    assert lib.mla_decode_workspace_bytes(ctypes.byref(v3_dims(d_rope=0)), 1, 1) == 0
    assert lib.mla_decode_workspace_bytes(None, 1, 1) == 0


def test_status_calls_reject_null(lib):
    assert lib.mla_status_read(None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_status_clear(None, None) == M.MLA_ERR_INVALID_ARG


def test_out_proj_argument_checks(lib):
    d = v3_dims()
    call = lambda **kw: lib.mla_out_proj(
        ctypes.byref(d) if kw.get("dims", True) else None, kw.get("o", FAKE), kw.get("w", FAKE),
        kw.get("y", FAKE), kw.get("T", 16), None)
    assert call(dims=False) == M.MLA_ERR_INVALID_ARG
    assert call(o=None) == M.MLA_ERR_INVALID_ARG
    assert call(w=None) == M.MLA_ERR_INVALID_ARG
    assert call(y=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(w=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(T=-1) == M.MLA_ERR_INVALID_ARG
    assert call(T=(1 << 20) + 1) == M.MLA_ERR_UNSUPPORTED
    assert call(T=0, o=None, y=None) == M.MLA_OK                      # empty: no-op


def test_query_proj_argument_checks(lib):
    d = v3_dims()
    call = lambda **kw: lib.mla_query_proj(
        ctypes.byref(d), kw.get("r", 1536), kw.get("h", FAKE), kw.get("wdq", FAKE), kw.get("wuq", FAKE),
        kw.get("c", FAKE), kw.get("q", FAKE), kw.get("T", 16), None)
    assert call(h=None) == M.MLA_ERR_INVALID_ARG
    assert call(q=None) == M.MLA_ERR_INVALID_ARG
    assert call(r=0) == M.MLA_ERR_INVALID_ARG
    assert call(r=1540) == M.MLA_ERR_UNSUPPORTED                    # rows of w_uq must stay 16-byte aligned
    assert call(c=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(wuq=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert call(T=-1) == M.MLA_ERR_INVALID_ARG
    assert call(T=0, h=None, q=None) == M.MLA_OK                     # empty: no-op


def test_context_split_argument_checks(lib):
    d = v3_dims()
    part = lambda **kw: lib.mla_decode_attn_partial(
        ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 2, 1, 4, 8, kw.get("r", 0), kw.get("R", 2), FAKE, 1 << 30,
        kw.get("o", FAKE), kw.get("l", FAKE), None, None)
    assert part(r=2) == M.MLA_ERR_INVALID_ARG                      # rank outside [0, R)
    assert part(r=-1) == M.MLA_ERR_INVALID_ARG
    assert part(R=0) == M.MLA_ERR_INVALID_ARG
    assert part(o=None) == M.MLA_ERR_INVALID_ARG
    assert part(l=None) == M.MLA_ERR_INVALID_ARG
    assert part(o=FAKE_MIS) == M.MLA_ERR_MISALIGNED

    def merge(n=2, T=4, o=None, l=None, out=FAKE):
        o = o or [FAKE] * max(n, 1)
        l = l or [FAKE] * max(n, 1)
        po = (ctypes.c_void_p * len(o))(*o)
        pl = (ctypes.c_void_p * len(l))(*l)
        return lib.mla_merge_ranks(ctypes.byref(d), po, pl, n, T, FAKE, out, None, None)
    assert merge(n=0) == M.MLA_ERR_INVALID_ARG
    assert merge(n=17) == M.MLA_ERR_UNSUPPORTED
    assert merge(T=-1) == M.MLA_ERR_INVALID_ARG
    assert merge(T=(1 << 18) + 1) == M.MLA_ERR_UNSUPPORTED
    assert merge(o=[FAKE, None]) == M.MLA_ERR_INVALID_ARG
    assert merge(l=[FAKE, FAKE_MIS]) == M.MLA_ERR_MISALIGNED
    assert merge(out=FAKE_MIS) == M.MLA_ERR_MISALIGNED
    assert merge(T=0) == M.MLA_OK                                   # empty: no-op


def test_merge_binding_rejects_mismatched_shapes():
    # shape checks in the binding run before any pointer is taken (CPU tensors suffice)
    d = v3_dims()
    T, H = 4, d.n_heads
    o = torch.zeros(T, H, d.d_c)
    l = torch.zeros(T, H)
    w_uv = torch.zeros(H, d.v_head, d.d_c, dtype=torch.bfloat16)
    out = torch.zeros(T, H, d.v_head, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        M.mla_merge_ranks(d, [o], [l, l], w_uv, out)                       # one lse too many
    with pytest.raises(ValueError):
        M.mla_merge_ranks(d, [torch.zeros(T, H, d.d_c - 8)], [l], w_uv, out)
    with pytest.raises(ValueError):
        M.mla_merge_ranks(d, [o], [torch.zeros(T + 1, H)], w_uv, out)
    with pytest.raises(ValueError):
        M.mla_merge_ranks(d, [o], [l], w_uv, torch.zeros(T, H, d.v_head + 8, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        M.mla_merge_ranks(d, [o], [l], w_uv[:, :64], out)
