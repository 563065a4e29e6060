"""gdn_prefill_noalloc: the prefill on the library's built-in scratch array.

It serves callers that cannot allocate device memory at call time -- code whose device
memory is entirely owned by another allocator, or code that must not take the device-wide
synchronisation of cudaMalloc / cudaFree inside a latency-critical loop.  This file is
collected last on purpose, so a run that stops at the first failure has run everything
else first; it also passes when run alone in a fresh process.

The call goes through the C ABI with raw device pointers and is compared with the
ordinary gdn_prefill (caller workspace), on two calls in a row with different inputs (the
scratch keeps the previous call's contents, so a stale byte would show up in the second
call).  Both run the same kernels on the same inputs with the same workspace layout, so
their outputs must be identical bit for bit; the parity tolerance would let a slightly
perturbed result through.  Both input dtypes are covered: bf16 inputs use the tensor-core
workspace layout, fp32 inputs the fp32 path's.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_deltanet_token_b200 import gdn
from gated_deltanet_token_b200.inputs import make_inputs
from tests._helpers import run_prefill, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(inp):
    names = ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w", "norm_w", "init_state")
    t = {n: to_dev(inp.get(n)) for n in names}
    cu = to_dev(inp["cu_seqlens"].astype(np.int32))
    T, h_qk, _ = t["q"].shape
    h_v = t["v"].shape[1]
    n = cu.numel() - 1
    in_dt = gdn.GDN_DTYPE_BF16 if t["q"].dtype == torch.bfloat16 else gdn.GDN_DTYPE_F32
    dims = gdn.make_dims(n, T, h_qk, h_v, in_dt, gdn.GDN_DTYPE_F32)
    assert gdn.gdn_prefill_workspace_size(dims) <= 64 << 20
    y = torch.full((T, h_v, 128), float("nan"), dtype=torch.float32, device="cuda")
    fs = torch.full((n, h_v, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    P = lambda x: ctypes.c_void_p(x.data_ptr())  # noqa: E731
    rc = gdn.lib().gdn_prefill_noalloc(
        ctypes.byref(dims), *[P(t[nm]) for nm in names], P(cu), P(y), P(fs),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == gdn.GDN_OK, gdn.gdn_status_string(rc)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), fs.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_prefill_on_two_calls(dtype):
    for seed, lens in ((0, [300, 0, 129, 64]), (1, [65, 5, 250])):
        inp = make_inputs("varlen8_prefill_bf16", seed=seed, lengths=lens, dtype=dtype)
        y_ref, S_ref = run_prefill(inp, torch.float32)
        y, S = _noalloc(inp)
        assert np.isfinite(y).all() and np.isfinite(S).all()
        assert np.array_equal(y, y_ref) and np.array_equal(S, S_ref)


def test_noalloc_rejects_dims_beyond_its_scratch():
    inp = make_inputs("varlen8_prefill_bf16", lengths=[4096])
    with pytest.raises(gdn.GdnError) as ei:
        gdn.gdn_prefill_noalloc(*(to_dev(inp[n]) for n in ("q", "k", "v", "z", "a", "b", "A_log",
                                                          "dt_bias", "conv_w", "norm_w")),
                                to_dev(inp["init_state"]), to_dev(inp["cu_seqlens"]))
    assert ei.value.code == -5  # GDN_ERR_WORKSPACE
