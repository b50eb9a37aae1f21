"""The JSON line of bench.py's reference arm (the CPU oracle) carries the keys the benchmark contract
names (CPU only; the oracle timing itself is replaced by a fixed sample so the test is instant)."""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_line(monkeypatch, capsys):
    calls = []

    def fake_sample(cfg, budget, head_iter=None):
        calls.append(budget)
        return 2.0e10, 0.5, "fp64 oracle on 1 head (stub)"

    monkeypatch.setattr(bench, "oracle_prefill_sample", fake_sample)
    monkeypatch.delenv("RANK", raising=False)
    args = argparse.Namespace(gpus=1, steps=4, warmup=3)
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert len(calls) == 7 and all(b > 0 for b in calls)  # warm-up and timed samples, bounded budgets
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["value"] == 2.0e10 / 0.5 / 1e12
    assert line["config"]["workload"] == bench.HEADLINE
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_other_ranks_do_nothing(monkeypatch, capsys):
    monkeypatch.setattr(bench, "oracle_prefill_sample", lambda *a, **k: (_ for _ in ()).throw(AssertionError))
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(argparse.Namespace(gpus=2, steps=2, warmup=3)) == 0
    assert capsys.readouterr().out == ""


def test_workload_flops():
    # 4 B H N^2 D, halved for causal: the headline workload's figure
    assert bench.prefill_flops(4, 16, 8192, 8192, 64, True) == 549755813888.0
    assert bench.prefill_flops(1, 1, 128, 256, 64, False) == 4 * 128 * 256 * 64


def test_prefix_flops_counts_visible_pairs():
    # 4 D FLOPs per visible (query, key) pair; the prefix-LM pair count by brute force
    N, D = 37, 64
    for p in (0, 1, 10, 36, 37):
        pairs = sum(1 for i in range(N) for j in range(N) if j < p or j <= i)
        assert bench.prefix_flops(2, 3, N, D, p) == 2 * 3 * 4 * D * pairs


def test_token_rates():
    line = {"ms_per_step": 2.0, "config": {"B": 4, "N": 8192},
            "decode": {"ms_per_step": 1.0, "config": {"B": 64},
                       "gqa": {"ms_per_step": 0.5, "config": {"B": 64}},
                       "paged": {"ms_per_step": 0.25, "config": {"B": 64}},
                       "sharded": {"ms_per_step": 4.0, "config": {"B": 4}}}}
    bench.add_token_rates(line, 2)
    assert line["tokens_per_s"] == 4 * 8192 * 2 / 2e-3
    assert line["decode"]["tokens_per_s"] == 64 * 2 / 1e-3
    assert line["decode"]["gqa"]["tokens_per_s"] == 64 * 2 / 0.5e-3
    assert line["decode"]["paged"]["tokens_per_s"] == 64 * 2 / 0.25e-3  # every rank its own batch
    assert line["decode"]["sharded"]["tokens_per_s"] == 4 / 4e-3  # one problem over the ranks
    # partial lines (a leg switched off) keep working
    for partial in ({"ms_per_step": None, "config": {}, "decode": None}, {"decode": {"ms_per_step": 1.0}}, {}):
        bench.add_token_rates(partial, 1)


def test_varlen_flops_sum_per_sequence():
    # each packed sequence attends only to itself: 4 H L^2 D per sequence, by brute-force pair count
    lengths, H, D = [3, 1, 7, 0, 5], 2, 64
    pairs = sum(sum(1 for i in range(L) for j in range(L)) for L in lengths)
    assert bench.varlen_flops(lengths, H, D) == 4 * H * D * pairs
    assert bench.varlen_flops(lengths, H, D, causal=True) == 2 * H * D * pairs
    # the varlen workload's figure from its seeded lengths (about 3.9e11)
    import seeded_inputs as si
    c = si.CONFIGS["varlen"]
    f = bench.varlen_flops(si.varlen_lengths(c["seed"], c["nseq"], c["len_lo"], c["len_hi"]), c["H"], c["D"])
    assert 2e11 < f < 6e11
