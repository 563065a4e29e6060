"""The Python binding checks its arguments before anything reaches the library: CPU tensors,
non-contiguous tensors, wrong index dtypes and mismatched pools raise, with no CUDA call."""
import pytest
import torch

from gated_deltanet_token_b200 import gdn


def _prefill_args(dev="cpu", T=8):
    bf = torch.bfloat16
    q = torch.zeros(T, 2, 128, dtype=bf, device=dev)
    k = torch.zeros(T, 2, 128, dtype=bf, device=dev)
    v = torch.zeros(T, 4, 128, dtype=bf, device=dev)
    z = torch.zeros(T, 4, 128, dtype=bf, device=dev)
    a = torch.zeros(T, 4, device=dev)
    b = torch.zeros(T, 4, device=dev)
    par = [torch.zeros(4, device=dev), torch.zeros(4, device=dev), torch.zeros(768, 4, device=dev),
           torch.ones(128, device=dev)]
    return [q, k, v, z, a, b] + par


def test_prefill_rejects_host_tensors():
    with pytest.raises(ValueError, match="contiguous CUDA tensors"):
        gdn.gdn_prefill(*_prefill_args(), workspace=torch.zeros(16, dtype=torch.uint8))


def test_prefill_rejects_int64_cu_seqlens():
    with pytest.raises(TypeError, match="int32"):
        gdn.gdn_prefill(*_prefill_args(), None, torch.tensor([0, 8], dtype=torch.int64))


def test_conv_state_rejects_int64_cu_seqlens():
    q, k, v = _prefill_args()[:3]
    with pytest.raises(TypeError, match="int32"):
        gdn.gdn_prefill_conv_state(q, k, v, torch.tensor([0, 8], dtype=torch.int64))


def test_decode_slots_checks_ids_and_pools():
    args = _prefill_args(T=3)
    pool_c = torch.zeros(4, 3, 768, dtype=torch.bfloat16)
    pool_s = torch.zeros(4, 4, 128, 128)
    with pytest.raises(TypeError, match="one entry per sequence"):
        gdn.gdn_decode_slots(*args, pool_c, pool_s, torch.zeros(3, dtype=torch.int64))
    with pytest.raises(TypeError, match="one entry per sequence"):
        gdn.gdn_decode_slots(*args, pool_c, pool_s, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="same number of slots"):
        gdn.gdn_decode_slots(*args, pool_c, pool_s[:3], torch.zeros(3, dtype=torch.int32))


def test_unsupported_dtype_is_rejected():
    args = _prefill_args()
    args[0] = args[0].to(torch.float16)
    with pytest.raises(TypeError, match="unsupported dtype"):
        gdn.gdn_prefill(*args)
