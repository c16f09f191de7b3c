"""Host-side logic of bench.py, on the CPU: the packed host/device buffers of
the end-to-end step, and the guard that reports ncu traffic only for the
kernel sources it was measured on."""
import json

import torch

import bench


def _tensors():
    g = torch.Generator().manual_seed(3)
    return (torch.randn(4, 1, 32, 128, generator=g).to(torch.bfloat16),
            torch.randn(4, 1, 8, 128, generator=g).to(torch.bfloat16),
            torch.arange(3, dtype=torch.int32),                 # 12 bytes: the next start pads
            torch.randint(0, 99, (4, 8192), generator=g, dtype=torch.int32),
            torch.zeros(4, 32, 1, dtype=torch.float32))


def test_packed_layout_aligns_every_start_to_16_bytes():
    ts = _tensors()
    offs, total = bench.packed_layout(ts)
    sizes = [t.numel() * t.element_size() for t in ts]
    assert offs[0] == 0 and all(o % 16 == 0 for o in offs)
    for i in range(1, len(ts)):
        assert offs[i] >= offs[i - 1] + sizes[i - 1]       # no overlap
        assert offs[i] - (offs[i - 1] + sizes[i - 1]) < 16  # padding only to the boundary
    assert total == offs[-1] + (sizes[-1] + 15) // 16 * 16


def test_packed_views_round_trip_and_match_dtype_shape():
    ts = _tensors()
    offs, total = bench.packed_layout(ts)
    buf = torch.zeros(total, dtype=torch.uint8)
    views = bench.packed_views(buf, ts, offs)
    for t, v in zip(ts, views):
        v.copy_(t)
    # the views alias the buffer: a second set of views reads the same values
    for t, v in zip(ts, bench.packed_views(buf.clone(), ts, offs)):
        assert v.dtype == t.dtype and tuple(v.shape) == tuple(t.shape) and v.is_contiguous()
        assert torch.equal(v.view(torch.uint8) if v.dtype != torch.uint8 else v,
                           t.contiguous().view(torch.uint8))
    for v, o in zip(views, offs):
        assert v.data_ptr() - buf.data_ptr() == o


def test_traffic_is_reported_only_for_the_measured_sources(monkeypatch, tmp_path):
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({"kernel_digest": "abc", "dram_bytes_per_call": 123}))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(f))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "abc")
    assert bench.profiled_traffic() == 123
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "def")
    assert bench.profiled_traffic() is None


def test_committed_traffic_summary_is_current_or_ignored():
    """The committed ncu figure is reported only while the kernel sources hash
    to the digest it was taken at; when it is reported, the DRAM bytes per
    call sit within 1 % of the workload's algorithmic K/V bytes."""
    with open(bench.PROFILE_TRAFFIC) as fh:
        t = json.load(fh)
    if t["kernel_digest"] != bench.kernel_source_digest():
        assert bench.profiled_traffic() is None
        return
    algorithmic = 4 * 131072 * 8 * 128 * 2 * 2
    assert bench.profiled_traffic() == t["dram_bytes_per_call"]
    assert abs(t["dram_bytes_per_call"] / algorithmic - 1) < 0.01
