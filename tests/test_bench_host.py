"""Host logic of bench.py that needs no GPU: the algorithmic byte and flop counts behind the roofline
fractions, and the line both arms print."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from chunk_wise_hierarchical_summary_b200 import workloads as W  # noqa: E402


def test_decode_bytes_single_token_matches_its_parts():
    w = W.DECODE_BF16
    n = bench.window_left(w.L - 1, w.W, w.S) // w.S
    by = bench.decode_bytes(w)
    assert by["summaries"] == w.B * w.Hq * n * (w.d * 2 + 4)
    assert by["chunks"] == w.B * w.Hkv * min(w.topk, n) * w.S * w.d * 2 * 2
    assert by["window"] == w.B * w.Hkv * (w.L - bench.window_left(w.L - 1, w.W, w.S)) * w.d * 2 * 2
    assert by["total"] == by["summaries"] + by["chunks"] + by["window"] + by["io"]


def test_decode_bytes_multi_token_counts_the_union():
    """M queries of a KV group touch each selected chunk once (the union of their selections) and the
    union of their windows; -1 padding is not a chunk."""
    w = W.Workload("m3", B=1, T=3, L=5000, Hq=4, Hkv=2, d=128, S=64, topk=4, W=256, dtype="bf16", recipe="needle",
                   q_pos0=4997)
    idx = torch.tensor([[[[1, 2, 3, 4], [2, 3, 4, 5], [1, 9, -1, -1]],
                         [[7, 7, 8, -1], [8, 10, 11, 12], [0, 1, 2, 3]]]], dtype=torch.int32)
    by = bench.decode_bytes(w, idx)
    tile = w.S * w.d * 2 * 2
    assert by["chunks"] == (6 + 9) * tile  # group 0: {1,2,3,4,5,9}; group 1: {7,8,10,11,12,0,1,2,3}
    l_first = bench.window_left(w.L - 3, w.W, w.S)
    assert by["window"] == w.B * w.Hkv * (w.L - l_first) * w.d * 2 * 2
    # without the selection the per-query sum is an upper bound of the union
    assert bench.decode_bytes(w)["chunks"] >= by["chunks"]


def test_prefill_work_counts_window_and_selected_tokens():
    w = W.Workload("p", B=1, T=300, L=300, Hq=2, Hkv=1, d=64, S=16, topk=3, W=40, dtype="fp32", recipe="tiny")
    work = bench.prefill_work(w)
    attended = 0
    for p in range(300):
        l = bench.window_left(p, 40, 16)
        attended += (p - l + 1) + min(3, l // 16) * 16
    assert work["attn_flops"] == 4 * 64 * attended * 2


def test_both_arms_share_metric_and_base_config():
    w = W.PREFILL_BF16
    c1, c2 = bench.base_config(w, 1), bench.base_config(w, 4)
    assert c1["workload"] == c2["workload"] == w.name and c2["global_batch"] == 4 * c1["global_batch"]
    assert "TC/HBM roofline" in bench.METRIC


def test_decode_summary_carries_the_headline_decode_half():
    """The line's last key holds the decode workload's us/token and HBM fraction (and the sweep's), in a
    few hundred characters, so any tail of the line shows them."""
    import json

    dec = {"workload": "decode_bf16_B8_L524288", "us_per_token": 129.0, "bytes_per_step": {"total": 628_800_000},
           "roofline": {"frac": 0.75, "achieved": 4870.0, "peak": 6452.5}}
    extra = {"decode_sweep": [{"L": L, "us_per_token": 30.0 + L / 1e5, "hbm_frac": 0.1} for L in W.DECODE_SWEEP_L],
             "decode_multi": {"us_per_step": 192.0, "roofline": {"frac": 0.6}}}
    s = bench.decode_summary(dec, extra)
    assert s["us_per_token"] == 129.0 and s["hbm_frac"] == 0.75
    assert [r[0] for r in s["sweep_L_us_frac"]] == list(W.DECODE_SWEEP_L)
    assert len(json.dumps(s)) < 800
    assert "sweep_L_us_frac" not in bench.decode_summary(dec, {})


def test_reference_arm_line_matches_the_gpu_arms_config_and_sample(capsys):
    """--impl reference prints one line whose metric and config are the GPU arm's, and whose cpu_baseline
    sample is the unit the GPU arm's cpu_baseline leg times (one whole (batch, KV group) slice)."""
    import argparse
    import json

    args = argparse.Namespace(gpus=1, steps=1, warmup=0)
    bench.run_reference(args, bench.Dist(1))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["config"] == bench.base_config(W.PREFILL_BF16, 1)
    assert line["cpu_baseline"]["sample"].startswith(bench.oracle_sample_text(W.PREFILL_BF16, 1))
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
