"""The Python binding checks its tensors before calling the library: host
tensors, wrong dtypes, wrong ranks and mismatched shapes raise on the CPU,
with no CUDA call (so these run without a GPU)."""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv
from paged_kv_decode_31_b200 import binding


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


def _case(B=2, nb=8, bs=16, Hkv=2, D=128, W=4):
    kc = _host(nb, bs, Hkv, D)
    return kc, kc.clone(), torch.zeros(B, W, dtype=torch.int32), torch.ones(B, dtype=torch.int32)


def test_cache_and_table_checks_accept_consistent_shapes():
    kc, vc, bt, sl = _case()
    binding._need_cache_and_table(2, 2, 128, kc, vc, bt, sl)
    binding._need_cache_and_table(1, None, 128, kc, vc, bt, sl)  # more rows than the batch is fine
    wide = torch.zeros(2, 8, dtype=torch.int32)[:, :4]             # row stride 8, column stride 1
    binding._need_cache_and_table(2, 2, 128, kc, vc, wide, sl)


@pytest.mark.parametrize("bad", ["v_shape", "head_dim", "kv_heads", "table_1d", "table_rows",
                                 "table_cols_strided", "seqlens_short", "seqlens_strided",
                                 "seqlens_2d"])
def test_cache_and_table_checks_reject_what_would_be_read_out_of_bounds(bad):
    kc, vc, bt, sl = _case()
    B, Hkv, D = 2, 2, 128
    if bad == "v_shape":
        vc = _host(8, 16, 2, 64)
    elif bad == "head_dim":
        D = 64
    elif bad == "kv_heads":
        Hkv = 4
    elif bad == "table_1d":
        bt = bt.reshape(-1)
    elif bad == "table_rows":
        bt = bt[:1]
    elif bad == "table_cols_strided":
        bt = torch.zeros(4, 2, dtype=torch.int32).t()
    elif bad == "seqlens_short":
        sl = sl[:1]
    elif bad == "seqlens_strided":
        sl = torch.ones(4, dtype=torch.int32)[::2]
    elif bad == "seqlens_2d":
        sl = sl.reshape(2, 1)
    with pytest.raises(ValueError):
        binding._need_cache_and_table(B, Hkv, D, kc, vc, bt, sl)


def test_output_and_lse_shape_checks():
    binding._need_rows("out", _host(2, 3, 4, 128), (2, 3, 4, 128))
    with pytest.raises(ValueError):
        binding._need_rows("out", _host(2, 3, 4, 64), (2, 3, 4, 128))
    with pytest.raises(ValueError):
        binding._need_rows("out", _host(2, 3, 4, 128, dtype=torch.float32), (2, 3, 4, 128))
    with pytest.raises(ValueError):  # a unit stride on the head_dim axis is required
        binding._need_rows("out", _host(2, 3, 128, 4).transpose(2, 3), (2, 3, 4, 128))
    binding._need_lse("lse", torch.zeros(2, 4, 3), (2, 4, 3))
    with pytest.raises(ValueError):
        binding._need_lse("lse", torch.zeros(2, 3, 4).transpose(1, 2), (2, 4, 3))
    with pytest.raises(ValueError):
        binding._need_lse("lse", torch.zeros(2, 4, 3, dtype=torch.float64), (2, 4, 3))


def test_error_word_and_device_checks():
    binding._need_err(None)
    with pytest.raises(TypeError):  # a host error word would be written by the device
        binding._need_err(torch.zeros(1, dtype=torch.int32))
    binding._need_one_device(_host(1), None, _host(2))
    with pytest.raises(ValueError):
        binding._need_one_device(_host(1), torch.zeros(1, device="meta"))
