"""Host logic of bench.py that needs no GPU: the algorithmic byte and flop counts behind the roofline
fractions, the attention's packing statistic, the clock summary that decides whether a run is kept, and
the line both arms print."""
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


def test_packing_counts_selected_chunks_per_query_and_distinct_chunks_per_tile():
    # G = 4: a tile packs 32 queries. Tile 0: every query selects chunks {0, 1}. Tile 1: even queries
    # select {2, 3}, odd queries {4} (one id, then -1 padding).
    w = W.Workload("pack", B=1, T=64, L=512, Hq=4, Hkv=1, d=64, S=64, topk=2, W=64, dtype="fp32", recipe="scaled")
    idx = torch.empty((1, 1, 64, 2), dtype=torch.int32)
    idx[0, 0, :32] = torch.tensor([0, 1], dtype=torch.int32)
    idx[0, 0, 32::2] = torch.tensor([2, 3], dtype=torch.int32)
    idx[0, 0, 33::2] = torch.tensor([4, -1], dtype=torch.int32)
    s = bench.packing_stats(w, idx)
    assert s["queries_per_tile"] == 32
    assert s["selected_chunks_per_query"] == (32 * 2 + 16 * 2 + 16 * 1) / 64
    assert s["selected_chunks_per_tile"] == (2 + 3) / 2


def test_clock_summary_reads_median_max_and_active_reasons():
    idle = "0, 1965, 1965, 650.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
    capped = "0, 1950, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
    hot = "0, 1200, 1965, 500.0, 0x0000000000000048, Not Active, Active, Not Active, Not Active\n"
    assert bench.summarise_clocks([idle, capped, idle, "a partial line, 1965\n"]) == {
        "sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    s = bench.summarise_clocks([idle, hot])
    assert s["reasons"] == ["hw_thermal_slowdown"] and s["sm_mhz"] == (1965.0 + 1200.0) / 2
    assert bench.summarise_clocks([]) is None
    na = "0, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]\n"
    assert bench.summarise_clocks([na]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 1}


def test_clock_sampler_watches_the_physical_gpu(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5")
    assert bench.physical_gpu_index(0) == 3 and bench.physical_gpu_index(1) == 5
    assert bench.physical_gpu_index(2) == 2  # past the list: the local rank
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-0a1b2c3d")  # a UUID: the local rank
    assert bench.physical_gpu_index(0) == 0
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.physical_gpu_index(3) == 3


def test_clock_sampler_reads_and_removes_its_csv(monkeypatch):
    class FakeSmi:  # writes two rows to the file nvidia-smi is asked for, then waits to be stopped
        def __init__(self, cmd, stdout=None, stderr=None):
            self.path = cmd[cmd.index("-f") + 1]
            assert cmd[cmd.index("-i") + 1] == "2" and cmd[0] == "nvidia-smi"
            with open(self.path, "w") as f:
                f.write("2, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                        "2, 1935, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")
            self.stopped = False

        def terminate(self):
            self.stopped = True

        def wait(self, timeout=None):
            assert self.stopped
            return 0

    monkeypatch.setattr(bench.subprocess, "Popen", FakeSmi)
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    sampler = bench.ClockSampler(2).start()
    path = sampler.path
    assert sampler.stop() == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}
    assert not os.path.exists(path)

    def no_smi(*a, **k):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "Popen", no_smi)
    sampler = bench.ClockSampler(0).start()
    assert not os.path.exists(sampler.path)  # its temporary file is not left behind
    assert sampler.stop() is None  # no sampler: the line carries no clock record
