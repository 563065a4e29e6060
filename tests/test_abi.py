"""Host-only checks of the C ABI: the library loads, exports every entry point that
include/gdn.h declares, names its status codes, sizes its workspace, and rejects bad
arguments with the documented codes before any launch (no GPU needed: the pointers
passed here are never dereferenced)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def glib():
    from gated_deltanet_token_b200 import _build, gdn

    _build.build()
    return gdn


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(gdn_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(glib):
    names = declared_functions()
    assert {"gdn_prefill", "gdn_decode", "gdn_prefill_workspace_size", "gdn_status_string",
            "gdn_read_device_status"} <= set(names)
    L = glib.lib()
    for n in names:
        assert hasattr(L, n), f"{n} not exported"


def test_status_strings(glib):
    expect = {0: "GDN_OK", -1: "GDN_ERR_NULL", -2: "GDN_ERR_SHAPE", -3: "GDN_ERR_DTYPE",
              -4: "GDN_ERR_ALIGN", -5: "GDN_ERR_WORKSPACE", -6: "GDN_ERR_CUDA",
              -7: "GDN_ERR_DEVICE_TIMEOUT", -8: "GDN_ERR_INDEX"}
    for c, s in expect.items():
        assert glib.gdn_status_string(c) == s
    assert glib.gdn_status_string(-99) == "GDN_ERR_UNKNOWN"


def test_workspace_size(glib):
    d = glib.make_dims(1, 4096, 16, 32, 1, 1)
    w = glib.gdn_prefill_workspace_size(d)
    assert w > 0 and w % 256 == 0
    d2 = glib.make_dims(1, 8192, 16, 32, 1, 1)
    assert glib.gdn_prefill_workspace_size(d2) > w
    assert glib.gdn_prefill_workspace_size(glib.make_dims(1, 16, 16, 32, 1, 1, d_k=64)) == 0
    assert glib.gdn_prefill_workspace_size(glib.make_dims(1, 16, 3, 32, 1, 1)) == 0


FAKE = 1 << 20  # 16-byte aligned fake device address, never dereferenced


def _prefill(glib, dims, ptrs=None, ws_bytes=1 << 40):
    p = [FAKE] * 14 if ptrs is None else ptrs
    P = [ctypes.c_void_p(x) if x else None for x in p]
    return glib.lib().gdn_prefill(ctypes.byref(dims), *P[:13], P[13], ctypes.c_void_p(FAKE),
                                  ctypes.c_size_t(ws_bytes), None)


def test_prefill_rejects_bad_arguments(glib):
    ok = glib.make_dims(2, 100, 16, 32, 1, 1)
    assert glib.lib().gdn_prefill(None, *([None] * 14), None, 0, None) == -1
    assert _prefill(glib, glib.make_dims(0, 100, 16, 32, 1, 1)) == -2
    assert _prefill(glib, glib.make_dims(1, -1, 16, 32, 1, 1)) == -2
    assert _prefill(glib, glib.make_dims(1, 100, 16, 30, 1, 1)) == -2
    assert _prefill(glib, glib.make_dims(1, 100, 16, 32, 1, 1, d_v=64)) == -2
    assert _prefill(glib, glib.make_dims(1, 100, 1, 16, 1, 1)) == -2  # more than 8 V heads per QK head
    assert _prefill(glib, glib.make_dims(1, 100, 16, 32, 2, 1)) == -3
    assert _prefill(glib, glib.make_dims(1, 100, 16, 32, 1, 7)) == -3
    ptrs = [FAKE] * 14
    ptrs[0] = None  # q
    assert _prefill(glib, ok, ptrs) == -1
    ptrs = [FAKE] * 14
    ptrs[11] = None  # cu_seqlens missing with two sequences
    assert _prefill(glib, ok, ptrs) == -1
    ptrs = [FAKE] * 14
    ptrs[3] = FAKE + 4  # misaligned z
    assert _prefill(glib, ok, ptrs) == -4
    assert _prefill(glib, ok, ws_bytes=16) == -5


def test_decode_rejects_bad_arguments(glib):
    L = glib.lib()

    def call(dims, ptrs):
        return L.gdn_decode(ctypes.byref(dims), *[ctypes.c_void_p(x) if x else None for x in ptrs], None)

    good = [FAKE] * 13
    assert call(glib.make_dims(4, 5, 16, 32, 1, 1), good) == -2  # total_tokens != n_seqs
    bad = list(good)
    bad[11] = None
    assert call(glib.make_dims(4, 4, 16, 32, 1, 1), bad) == -1
    bad = list(good)
    bad[10] = FAKE + 8
    assert call(glib.make_dims(4, 4, 16, 32, 1, 1), bad) == -4
    assert call(glib.make_dims(4, 4, 16, 32, 5, 1), good) == -3


def test_handoff_calls_reject_bad_arguments(glib):
    L = glib.lib()
    V = ctypes.c_void_p

    def conv(dims, q=FAKE, k=FAKE, v=FAKE, cu=FAKE, out=FAKE):
        return L.gdn_prefill_conv_state(None if dims is None else ctypes.byref(dims),
                                        *[V(x) if x else None for x in (q, k, v, cu, out)], None)

    two = glib.make_dims(2, 100, 16, 32, 1, 1)
    assert conv(None) == -1
    assert conv(two, out=None) == -1
    assert conv(two, cu=None) == -1  # two sequences need cu_seqlens
    assert conv(two, q=None) == -1
    assert conv(two, v=FAKE + 4) == -4
    assert conv(glib.make_dims(2, 100, 16, 30, 1, 1)) == -2
    assert conv(glib.make_dims(2, 100, 16, 32, 3, 1)) == -3

    def slots(dims, n_slots=4, ids=FAKE, pool=FAKE):
        ptrs = [FAKE] * 10 + [pool, FAKE]
        return L.gdn_decode_slots(ctypes.byref(dims), *[V(x) for x in ptrs], ctypes.c_int32(n_slots),
                                  V(ids) if ids else None, V(FAKE), None)

    four = glib.make_dims(4, 4, 16, 32, 1, 1)
    assert slots(four, ids=None) == -1
    assert slots(four, ids=FAKE + 4) == -4
    assert slots(four, n_slots=0) == -2
    assert slots(glib.make_dims(4, 5, 16, 32, 1, 1)) == -2  # total_tokens != n_seqs
    assert slots(four, pool=FAKE + 8) == -4


def test_decode_multi_rejects_bad_arguments(glib):
    L = glib.lib()

    def call(dims, K, ptrs=None):
        p = [FAKE] * 13 if ptrs is None else ptrs
        return L.gdn_decode_multi(None if dims is None else ctypes.byref(dims), ctypes.c_int32(K),
                                  *[ctypes.c_void_p(x) if x else None for x in p], None)

    assert call(None, 2) == -1
    assert call(glib.make_dims(4, 8, 16, 32, 1, 1), 0) == -2
    assert call(glib.make_dims(4, 36, 16, 32, 1, 1), 9) == -2  # more than 8 tokens
    assert call(glib.make_dims(4, 7, 16, 32, 1, 1), 2) == -2   # total_tokens != n_seqs * n_tokens
    bad = [FAKE] * 13
    bad[11] = None
    assert call(glib.make_dims(4, 8, 16, 32, 1, 1), 2, bad) == -1
    bad = [FAKE] * 13
    bad[0] = FAKE + 2
    assert call(glib.make_dims(4, 8, 16, 32, 1, 1), 2, bad) == -4


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from gated_deltanet_token_b200 import gdn

    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="libgdn.so not found"):
        gdn.lib()


def test_path_options_round_trip(glib):
    """The path-option word (host only): set returns the previous word, unknown bits are
    dropped, and the previous value is restored."""
    prev = glib.gdn_set_options(0)
    try:
        assert glib.gdn_get_options() == 0
        assert glib.gdn_set_options(0xFF) == 0
        assert glib.gdn_get_options() == (glib.GDN_OPT_FORCE_FP32_PATH | glib.GDN_OPT_SEPARATE_NORM |
                                          glib.GDN_OPT_NO_PDL)
    finally:
        glib.gdn_set_options(prev)
    assert glib.gdn_get_options() == prev


def test_projections_reject_bad_arguments(glib):
    L = glib.lib()
    bf = glib.make_dims(1, 16, 16, 32, glib.GDN_DTYPE_BF16, glib.GDN_DTYPE_BF16)

    def inp(dims, hidden, ptrs=None):
        p = [FAKE] * 8 if ptrs is None else ptrs
        return L.gdn_in_proj(None if dims is None else ctypes.byref(dims), ctypes.c_int32(hidden),
                             *[ctypes.c_void_p(x) if x else None for x in p], None)

    def outp(dims, hidden, ptrs=None):
        p = [FAKE] * 3 if ptrs is None else ptrs
        return L.gdn_out_proj(None if dims is None else ctypes.byref(dims), ctypes.c_int32(hidden),
                              *[ctypes.c_void_p(x) if x else None for x in p], None)

    assert inp(None, 2048) == -1
    assert inp(glib.make_dims(1, 16, 16, 32, glib.GDN_DTYPE_F32, glib.GDN_DTYPE_BF16), 2048) == -3
    assert inp(bf, 2000) == -2  # hidden not a multiple of the 64-wide K block
    assert inp(bf, 0) == -2
    bad = [FAKE] * 8
    bad[6] = None  # a
    assert inp(bf, 2048, bad) == -1
    bad = [FAKE] * 8
    bad[0] = FAKE + 8  # x misaligned
    assert inp(bf, 2048, bad) == -4
    assert outp(None, 2048) == -1
    assert outp(glib.make_dims(1, 16, 16, 32, glib.GDN_DTYPE_BF16, glib.GDN_DTYPE_F32), 2048) == -3
    assert outp(bf, 2047) == -2
    assert outp(bf, 2048, [FAKE, None, FAKE]) == -1
    assert outp(bf, 2048, [FAKE, FAKE, FAKE + 4]) == -4


def test_recurrence_backward_rejects_bad_arguments(glib):
    L = glib.lib()
    dims = glib.make_dims(1, 100, 2, 4, glib.GDN_DTYPE_F32, glib.GDN_DTYPE_F32)
    need = L.gdn_recurrence_backward_workspace_size(ctypes.byref(dims))
    assert need > 0
    # the dims' dtype codes are not read by the fp32 backward
    odd = glib.make_dims(1, 100, 2, 4, 7, 9)
    assert L.gdn_recurrence_backward_workspace_size(ctypes.byref(odd)) == need

    def call(d, ptrs=None, ws=FAKE, nbytes=None):
        p = [FAKE] * 15 if ptrs is None else ptrs
        return L.gdn_recurrence_backward(None if d is None else ctypes.byref(d),
                                         *[ctypes.c_void_p(x) if x else None for x in p],
                                         ctypes.c_void_p(ws) if ws else None,
                                         ctypes.c_size_t(need if nbytes is None else nbytes), None)

    assert call(None) == -1
    assert call(glib.make_dims(1, 100, 3, 4, 1, 1)) == -2  # h_v not a multiple of h_qk
    p = [FAKE] * 15
    p[14] = None  # dS_init
    assert call(dims, p) == -1
    p = [FAKE] * 15
    p[0] = None  # qh with tokens present
    assert call(dims, p) == -1
    p = [FAKE] * 15
    p[6] = None  # no cu_seqlens for two sequences
    assert call(glib.make_dims(2, 100, 2, 4, 1, 1), p) == -1
    p = [FAKE] * 15
    p[3] = FAKE + 4  # g misaligned
    assert call(dims, p) == -4
    assert call(dims, nbytes=need - 1) == -5
    assert call(dims, ws=0) == -5


def test_wait_limit_rejects_zero(glib):
    assert glib.lib().gdn_set_wait_limit_ns(ctypes.c_uint64(0)) == -2


def test_noalloc_token_limits_match_the_header(glib):
    """gdn.h states what fits the allocation-free prefill's 64 MiB scratch at the model shape
    (one sequence, 16 QK / 32 value heads): 960 tokens with bf16 inputs, 740 with fp32."""
    cap = 64 << 20

    def fits(T, dt):
        return glib.gdn_prefill_workspace_size(glib.make_dims(1, T, 16, 32, dt, glib.GDN_DTYPE_F32)) <= cap

    assert fits(960, glib.GDN_DTYPE_BF16) and not fits(961, glib.GDN_DTYPE_BF16)
    assert fits(740, glib.GDN_DTYPE_F32) and not fits(741, glib.GDN_DTYPE_F32)
