"""Host arithmetic of bench.py: the whole-pass roofline counts the bytes the
method must move and the projection flops (per token: the id, the gathered
rows, hidden read, Y written; the weights once per step; in decode also three
V-ring taps read and one V row written)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from hashed_gram_conditional_hash_b200 import workloads as W  # noqa: E402


def test_pass_roofline_model_shaped_counts():
    w = W.CONFIGS["model_bf16"]             # B=4, T=2048, E=1024, H=1024, hc=4, bf16
    tok = 4 * 2048
    r = bench.pass_roofline(w, tok, 100e-6, 1661.2, 6550.4)
    assert r["bytes_per_step"] == tok * (8 + 1024 * 2 + 2 * 4 * 1024 * 2) + 5 * 1024 * 1024 * 2
    assert r["flops_per_step"] == 2 * 1024 * 1024 * 5 * tok
    assert r["bound"] == "tensor"
    assert r["t_tensor_us"] == pytest.approx(2 * 1024 * 1024 * 5 * tok / 1661.2e12 * 1e6)
    assert r["frac"] == pytest.approx(r["t_tensor_us"] / 100.0)


def test_pass_roofline_decode_adds_ring_traffic():
    w = W.CONFIGS["decode_bf16"]            # 1024 sequences x 1 token, E=1536, H=2048, hc=4
    r = bench.pass_roofline(w, 1024, 64e-6, 1661.2, 6550.4)
    per_tok = 8 + 1536 * 2 + 2 * 4 * 2048 * 2 + 4 * 2048 * 2
    assert r["bytes_per_step"] == 1024 * per_tok + 5 * 2048 * 1536 * 2
    assert r["t_hbm_us"] == pytest.approx(r["bytes_per_step"] / 6550.4e9 * 1e6)


@pytest.mark.parametrize("name,tokens,total_bytes,total_flops", [
    # per token 8 + 2E + 4·hc·H bytes, weights (1+hc)·H·E·2 once, 2·E·H·(1+hc) flops
    ("large_table_bf16", 8 * 4096, 1.4824e9, 1.2885e12),
    ("hbm_table_bf16", 16 * 4096, 4.6478e9, 5.4976e12),
])
def test_pass_roofline_large_workloads(name, tokens, total_bytes, total_flops):
    w = W.CONFIGS[name]
    r = bench.pass_roofline(w, tokens, 1e-3, 1661.2, 6550.4)
    assert r["bytes_per_step"] == pytest.approx(total_bytes, rel=1e-3)
    assert r["flops_per_step"] == pytest.approx(total_flops, rel=1e-3)
    assert r["bound"] == "tensor"


def test_device_memory_report_counts_every_buffer():
    # one replica's device memory as the bench reports it: tables, weights,
    # this step's inputs and output, the workspace, and the static scratch
    import torch
    from hashed_gram_conditional_hash_b200 import _lib as L
    w = W.small_workload(B=2, T=16, hidden=256, hc_mult=2)
    p = W.make_params(w, "cpu")
    ws = torch.empty(4096, dtype=torch.uint8)
    y = torch.empty((w.B, w.T, w.hc_mult, w.hidden), dtype=w.torch_dtype)
    m = bench.device_memory(w, p, ws, y)
    nb = lambda t: t.numel() * t.element_size()
    assert m["tables"] == round(nb(p.table) / 1e9, 3)
    assert m["inputs_outputs"] == round((nb(p.ids) + nb(p.hidden) + nb(y)) / 1e9, 3)
    assert m["static_scratch"] == round(L.NO_ALLOC_SCRATCH_BYTES / 1e9, 3) == 0.034
    assert set(m) == {"tables", "weights", "inputs_outputs", "workspace", "static_scratch"}


def test_load_peaks_takes_measured_figures_key_by_key(tmp_path, monkeypatch):
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()                       # no file: the fallback figures
    assert kind == "fallback" and peaks == bench.PEAKS_FALLBACK
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text(json.dumps({"hbm_gbs": 6550.4, "bf16_tflops": 1661.2, "bf16_tflops_sustained": 1396.1,
                             "clocks": {"sm_mhz": 1965}}))
    peaks, kind = bench.load_peaks()
    assert kind == "measured"
    assert peaks == {"hbm_gbs": 6550.4, "bf16_tflops": 1661.2, "bf16_tflops_sustained": 1396.1}
    f.write_text(json.dumps({"hbm_gbs": 6550.4, "bf16_tflops": "n/a"}))   # partial: the rest falls back
    peaks, kind = bench.load_peaks()
    assert peaks["hbm_gbs"] == 6550.4
    assert peaks["bf16_tflops"] == bench.PEAKS_FALLBACK["bf16_tflops"]
    assert kind.startswith("measured (hbm_gbs)")
    f.write_text("not json")
    assert bench.load_peaks() == (bench.PEAKS_FALLBACK, "fallback")
