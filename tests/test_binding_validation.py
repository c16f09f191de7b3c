"""The Python binding checks its tensors before calling the library: host
tensors, wrong dtypes, wrong ranks and mismatched shapes raise on the CPU,
with no CUDA call (so these run without a GPU)."""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv


def _host(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def test_host_tensors_are_rejected():
    q = _host(1, 1, 4, 128)
    kc = _host(8, 16, 2, 128)
    bt = torch.zeros(1, 8, dtype=torch.int32)
    sl = torch.ones(1, dtype=torch.int32)
    with pytest.raises(TypeError):
        pkv.paged_decode_attn(q, kc, kc, bt, sl, max_seqlen_k=1)
    with pytest.raises(TypeError):
        pkv.paged_prefill_attn(q, kc, kc, bt, sl, max_seqlen_k=1)
    with pytest.raises(TypeError):
        pkv.kv_append(_host(1, 1, 2, 128), _host(1, 1, 2, 128), kc, kc, bt, sl)
    with pytest.raises(TypeError):
        pkv.paged_prefill_attn_bwd(q, kc, kc, bt, sl, q, torch.zeros(1, 4, 1), q)
    with pytest.raises(TypeError):
        pkv.paged_varlen_attn(_host(3, 4, 128), kc, kc, bt, sl, torch.zeros(2, dtype=torch.int32), 3)


def test_packed_calls_want_three_dimensional_tensors():
    with pytest.raises(TypeError):  # host and 4-D: the device check comes first
        pkv.kv_append_varlen(_host(1, 3, 2, 128), _host(1, 3, 2, 128), _host(8, 16, 2, 128),
                             _host(8, 16, 2, 128), torch.zeros(1, 8, dtype=torch.int32),
                             torch.zeros(1, dtype=torch.int32), torch.zeros(2, dtype=torch.int32))


def test_fp32_inputs_are_rejected():
    q = _host(1, 1, 4, 128, dtype=torch.float32)
    kc = _host(8, 16, 2, 128)
    with pytest.raises(TypeError):
        pkv.paged_decode_attn(q, kc, kc, torch.zeros(1, 8, dtype=torch.int32),
                              torch.ones(1, dtype=torch.int32), max_seqlen_k=1)
