#!/usr/bin/env python
"""Benchmark of the exact tiled attention forward pass on B200; prints ONE JSON line (rank 0).

Headline: attention forward TFLOPS on the prefill workload B=4, H=16, N=8192, D=64, causal, bf16
(4*B*H*N^2*D FLOPs, halved for causal), inputs resident in HBM.  One step = one fa_fwd call over the
whole batch.  The same line carries
  * roofline  -- the prefill kernel's achieved TFLOP/s against the measured dense bf16 peak;
  * decode    -- split-KV decode (B=64, H=32, D=128, Nk=8192, 16 splits) in HBM GB/s of K+V+Q+O
                 bytes, with its own roofline against the measured HBM copy bandwidth;
  * e2e       -- the same headline metric through the C ABI with host buffers: every step copies
                 Q, K, V from pinned host memory and O, LSE back (the copies of consecutive steps
                 overlap the kernel on separate streams);
  * cpu_baseline -- the fp64 CPU oracle on a bounded sample of the workload (rank 0, N=1 only);
  * clocks    -- SM clocks and throttle reasons sampled (NVML) during the timed region.

--impl reference times the CPU oracle itself as the reference arm (rank 0 only).
Multi-GPU (--gpus N under torchrun): one process per GPU, each rank runs its own batch of the same
workload (independent problems, no data-path collective); value = all ranks' FLOPs / max-over-ranks
time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import seeded_inputs as si  # noqa: E402

MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HEADLINE = "prefill_d64"
METRIC = "attention fwd TFLOPS (and % of B200 dense bf16 peak); decode HBM GB/s"


def peaks():
    try:
        with open(MEASURED_PEAKS) as fh:
            d = json.load(fh)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "fallback"


CSRC = os.path.join(ROOT, "exact_tiled_attention_47_b200", "csrc")
TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def measured_traffic(key, scale=1.0):
    """DRAM bytes per launch from the committed ncu summary, or None if the kernel changed since."""
    import hashlib
    try:
        with open(TRAFFIC) as fh:
            ent = json.load(fh)[key]
        h = hashlib.sha256()
        for f in ent["files"]:
            with open(os.path.join(CSRC, f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest()[:16] != ent["source_sha"]:
            return None
        b = ent.get("dram_bytes", ent.get("dram_bytes_per_batch_item", ent.get("dram_bytes_per_valid_kv_byte")))
        return float(b) * scale
    except (OSError, KeyError, ValueError):
        return None


def prefill_flops(B, H, Nq, Nk, D, causal):
    f = 4.0 * B * H * Nq * Nk * D
    return f / 2 if causal else f


def prefix_flops(B, H, N, D, prefix):
    """Algorithmic FLOPs of the prefix mask, counted per visible (query, key) pair: rows i < prefix
    see prefix keys, rows i >= prefix see i + 1 keys (square self-attention)."""
    p = min(max(prefix, 0), N)
    pairs = p * p + (N * (N + 1) - p * (p + 1)) // 2
    return 4.0 * B * H * D * pairs


def causal_rows_flops(rows_lo, rows_hi, N, D):
    """Algorithmic FLOPs of query rows [lo, hi) of one causal head with Nq = Nk = N."""
    # row i sees i+1 keys: 4 * (i+1) * D
    n = rows_hi - rows_lo
    s = (rows_lo + 1 + rows_hi) * n / 2.0
    return 4.0 * D * s


# ------------------------------------------------------------------------------------------------
# clocks


class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU with NVML every ~2 ms (read-only)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index, period_s=0.002):
        self.index = index
        self.period_s = period_s
        self.samples = []
        self.reasons = set()
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period_s)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# device helpers


def to_dev(bits, dtype, device):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def rank_seed(cfg_seed: int, rank: int) -> int:
    """Each rank processes its own batch of the workload (independent problems, weak scaling)."""
    return cfg_seed + 1000 * rank


def max_over_ranks(ms: float, dist=None, device="cuda") -> float:
    """The job's time is the slowest rank's (all ranks take the same collective steps)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Units of all ranks per second of the slowest rank."""
    return units_per_step_per_rank * world / (ms_per_step_max * 1e-3)


def timed(fn, steps, stream, dist=None):
    """Time `steps` calls of fn on `stream` with CUDA events; returns the max over ranks (ms)."""
    import torch
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist)
    if dist is not None:
        dist.barrier()
    return ms


def sharded_leg(args, kc, vc, dev, rank, world, dist, pk, pk_kind, fa, torch, stream, steps):
    """Long-context decode with the cache cut along the key axis over the ranks (strong scaling).

    The resident decode cache [64, 8192, 32, 128] is read as 4 sequences of 131072 keys; rank r
    holds keys shard_range(131072, world, r) of it, runs the shard kernels, the ranks all-gather the
    fp32 (O, LSE) blocks (no exchange with one rank), and every rank merges them.  Timing only: the
    shards of different ranks come from each rank's own seeded cache.
    """
    from exact_tiled_attention_47_b200.sharded import gather_parts, part_floats, shard_range
    g = si.CONFIGS["decode_long"]
    B, Nk, H, D, S = g["B"], g["Nk"], g["H"], g["D"], g["num_splits"]
    kl, vl = kc.view(B, Nk, H, D), vc.view(B, Nk, H, D)
    off, n = shard_range(Nk, world, rank)
    if world > 1:
        kl = kl[:, off:off + n].contiguous()
        vl = vl[:, off:off + n].contiguous()
    q = to_dev(si.batched(g["seed"], si.Q_ID, B, (1, H, D), "bf16"), "bf16", dev)
    nf = part_floats(B, H, D)
    part = torch.empty(nf, dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_bytes(B, H, D, S), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)

    def step():
        st = fa.fa_decode_splitkv_shard(q, kl, vl, part, B, H, H, n, off, Nk, D, g["scale"], S, None, ws,
                                        stream=stream)
        if st:
            raise fa.FAError(st, "fa_decode_splitkv_shard")
        parts = gather_parts(part, world)
        st = fa.fa_decode_merge(parts, world, B, H, D, o, lse, stream=stream)
        if st:
            raise fa.FAError(st, "fa_decode_merge")

    for _ in range(args.warmup):
        step()
    ms = timed(step, steps, stream, dist)
    if fa.fa_device_status(clear=True) != 0:
        raise RuntimeError("device status set during the timed sharded decode run")
    t = ms / steps * 1e-3
    shard_bytes = 2 * B * n * H * D * 2
    total_bytes = 2 * B * Nk * H * D * 2
    gbs_rank = shard_bytes / t / 1e9
    return {"metric": "key-sharded long-context decode HBM GB/s", "value": total_bytes / t / 1e9, "unit": "GB/s",
            "scaling": "strong", "shards": world, "ms_per_step": ms / steps, "steps": steps,
            "config": {"workload": "decode_long", "B": B, "H": H, "Nk_total": Nk, "Nk_shard": n, "D": D,
                       "num_splits_per_shard": S, "dtype": "bf16",
                       "exchange": "NCCL all-gather of fp32 (O, LSE) blocks" if world > 1 else "none (one shard)",
                       "exchange_bytes_per_rank": 4 * nf * world if world > 1 else 0,
                       "l2": f"K/V shard {shard_bytes / 1e9:.2f} GB vs 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": gbs_rank, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs_rank / pk["hbm_gbs"], "peak_kind": f"{pk_kind} copy",
                         # the same split kernel streams the same cache bytes as the plain decode: its
                         # DRAM bytes per batch item of that cache, scaled to this rank's shard
                         "traffic": measured_traffic("decode", shard_bytes / (2 * 8192 * H * D * 2)),
                         "algorithmic_bytes_per_step": shard_bytes},
            "gpu_launches": 3 * steps}


def add_token_rates(line, world):
    """Tokens per second beside the FLOP and byte rates: prefill B*N query tokens per step, decode one
    token per sequence per step, all ranks together (max-over-ranks step time).  Never raises: a
    missing figure just leaves the key out."""
    def rate(tokens, ms):
        return tokens / (ms * 1e-3) if tokens and ms else None

    try:
        cfg = line.get("config") or {}
        if line.get("ms_per_step"):
            line["tokens_per_s"] = rate(cfg["B"] * cfg["N"] * world, line["ms_per_step"])
        dec = line.get("decode") or {}
        if dec.get("ms_per_step"):
            dec["tokens_per_s"] = rate(dec["config"]["B"] * world, dec["ms_per_step"])
        for key in ("gqa", "paged", "sharded"):
            sub = dec.get(key) or {}
            if sub.get("ms_per_step"):
                # the sharded cache is one problem split over the ranks: its B sequences per step
                n = sub["config"]["B"] * (world if key != "sharded" else 1)
                sub["tokens_per_s"] = rate(n, sub["ms_per_step"])
    except (KeyError, TypeError, ZeroDivisionError):
        pass
    return line


def timed_run(run, steps, stream, dist=None):
    """Time run(steps), which may use other streams but joins them into `stream` before it returns."""
    import torch
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist)
    if dist is not None:
        dist.barrier()
    return ms


# ------------------------------------------------------------------------------------------------
# CPU oracle legs


def oracle_prefill_sample(cfg, budget_s, head_iter=None):
    """Run the fp64 oracle on the last rows of heads of the prefill workload for ~budget_s seconds.

    The last r query rows of a causal head with all N keys are exactly those rows of the full
    problem (bottom-right alignment).  Returns (flops, seconds, description).
    """
    import oracle
    B, N, H, D, dt = cfg["B"], cfg["Nq"], cfg["H"], cfg["D"], cfg["dtype"]
    causal = cfg.get("causal", False)
    # one batch item's tensors on the host (regenerated from the seed, as on the GPU side)
    b = 0
    qb = si.batch_item(cfg["seed"], si.Q_ID, b, (N, H, D), dt)
    kb = si.batch_item(cfg["seed"], si.K_ID, b, (N, H, D), dt)
    vb = si.batch_item(cfg["seed"], si.V_ID, b, (N, H, D), dt)
    rows = 256
    flops = 0.0
    t0 = time.perf_counter()
    heads = 0
    while True:
        h = heads % H
        qf = si.bits_to_float(qb[N - rows:, h], dt)
        kf = si.bits_to_float(kb[:, h], dt)
        vf = si.bits_to_float(vb[:, h], dt)
        oracle.attention_head(qf, kf, vf, cfg["scale"], causal)
        flops += causal_rows_flops(N - rows, N, N, D) if causal else 4.0 * rows * N * D
        heads += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return flops, el, f"fp64 oracle on the last {rows} query rows of {heads} head(s) of batch item 0"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


# ------------------------------------------------------------------------------------------------
# reference arm: the oracle as the program being compared against


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = si.CONFIGS[HEADLINE]
    total_budget = 90.0
    per_step = max(0.05, total_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_prefill_sample(cfg, per_step)
    flops = secs = 0.0
    desc = ""
    for _ in range(args.steps):
        f, s, desc = oracle_prefill_sample(cfg, per_step)
        flops += f
        secs += s
    tflops = flops / secs / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": HEADLINE, "B": cfg["B"], "H": cfg["H"], "N": cfg["Nq"], "D": cfg["D"],
                   "causal": True, "input_dtype": cfg["dtype"]},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# our arm


def varlen_flops(lengths, H, D, causal=False):
    """Sum over packed sequences of 4 * H * L^2 * D (halved for causal)."""
    f = sum(4.0 * H * int(L) * int(L) * D for L in lengths)
    return f / 2 if causal else f


def other_prefill_leg(args, name, dev, rank, world, dist, pk, pk_kind, fa, torch):
    """One more prefill workload (the other head dim, or the packed varlen encoder) timed the same way
    as the headline: CUDA events over the timed steps, inputs larger than L2.  Returns a sub-line."""
    cfg = si.CONFIGS[name]
    stream = torch.cuda.current_stream(dev)
    seed = rank_seed(cfg["seed"], rank)
    dt, H, D, scale = cfg["dtype"], cfg["H"], cfg["D"], cfg["scale"]
    causal = bool(cfg.get("causal", False))
    if name == "varlen":
        lengths = si.varlen_lengths(cfg["seed"], cfg["nseq"], cfg["len_lo"], cfg["len_hi"])
        q, k, v, cu = si.varlen_qkv(seed, lengths, H, D, dt)
        total = int(cu[-1])
        B, Nq = len(lengths), total
        cud = torch.from_numpy(cu).to(dev)
        flops = varlen_flops(lengths, H, D, causal)
        tokens = total
        lse = torch.empty((H, total), dtype=torch.float32, device=dev)
        conf = {"workload": name, "sequences": B, "total_tokens": total,
                "lengths": f"U{{{cfg['len_lo']}..{cfg['len_hi']}}} seeded", "H": H, "D": D, "causal": causal,
                "input_dtype": dt, "output_dtype": dt, "scale": scale}
    else:
        B, Nq = cfg["B"], cfg["Nq"]
        q, k, v = si.dense_qkv(seed, B, Nq, Nq, H, D, dt)
        cud = None
        flops = prefill_flops(B, H, Nq, Nq, D, causal)
        tokens = B * Nq
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
        conf = {"workload": name, "B": B, "H": H, "N": Nq, "D": D, "causal": causal, "input_dtype": dt,
                "output_dtype": dt, "scale": scale}
    qd, kd, vd = (to_dev(t, dt, dev) for t in (q, k, v))
    del q, k, v
    od = torch.empty_like(qd)
    conf["l2"] = f"inputs {3 * qd.numel() * 2 / 2**20:.0f} MiB > 126 MB L2 (no flush needed)"

    def step():
        st = fa.fa_fwd(qd, kd, vd, od, lse, B, H, Nq, Nq, D, scale, causal, cud, stream)
        if st:
            raise fa.FAError(st, "fa_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = max(10, min(args.steps, 50))
    with ClockSampler(dev.index) as clk:
        ms = timed(step, steps, stream, dist)
    if fa.fa_device_status(clear=True) != 0:
        raise RuntimeError(f"device status set during the timed {name} run")
    ms_step = ms / steps
    tf = flops / (ms_step * 1e-3) / 1e12
    dtn = "fp16" if dt == "fp16" else "bf16"
    out = {"metric": "attention fwd TFLOPS", "value": whole_job_rate(flops, ms_step, world) / 1e12,
           "unit": "TFLOP/s", "ms_per_step": ms_step, "steps": steps,
           "tokens_per_s": tokens * world / (ms_step * 1e-3), "config": conf,
           "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": tf / pk["bf16_tflops"], "traffic": measured_traffic(name),
                        "traffic_unit": "bytes per launch (ncu dram read+write)",
                        "kernel": f"fa_fwd_kernel<{D},{dtn},out {dtn}>",
                        "peak_kind": f"{pk_kind} bf16 burst (fp16 has the same dense rate)",
                        "frac_of_sustained": tf / pk["bf16_tflops_sustained"],
                        "algorithmic_flops_per_launch": flops},
           "clocks": clk.summary(), "gpu_launches": steps}
    del qd, kd, vd, od, lse
    torch.cuda.empty_cache()
    return out


def prefill_leg(args, cfg, dev, rank, world, dist, pk, pk_kind, fa, torch):
    """Time the headline prefill workload; returns (value, ms_step, roofline, e2e, clocks, prefix)."""
    B, N, H, D, dt = cfg["B"], cfg["Nq"], cfg["H"], cfg["D"], cfg["dtype"]
    scale = cfg["scale"]
    stream = torch.cuda.current_stream(dev)
    seed = rank_seed(cfg["seed"], rank)
    q, k, v = si.dense_qkv(seed, B, N, N, H, D, dt)
    qd, kd, vd = (to_dev(t, dt, dev) for t in (q, k, v))
    od = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    causal = bool(cfg.get("causal", False))

    def step():
        st = fa.fa_fwd(qd, kd, vd, od, lse, B, H, N, N, D, scale, causal, None, stream)
        if st:
            raise fa.FAError(st, "fa_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        ms = timed(step, args.steps, stream, dist)
    if fa.fa_device_status(clear=True) != 0:
        raise RuntimeError("device status set during the timed prefill run")

    # the same inputs under the prefix mask (a quarter of the keys visible to every query)
    prefix = None
    if causal and not args.no_prefix:
        plen = N // 4

        def pstep():
            st = fa.fa_fwd_prefix(qd, kd, vd, od, lse, B, H, N, N, D, scale, plen, None, stream)
            if st:
                raise fa.FAError(st, "fa_fwd_prefix")

        for _ in range(args.warmup):
            pstep()
        psteps = max(10, min(args.steps, 50))
        ms_p = timed(pstep, psteps, stream, dist)
        if fa.fa_device_status(clear=True) != 0:
            raise RuntimeError("device status set during the timed prefix run")
        pf = prefix_flops(B, H, N, D, plen)
        ptf = pf / (ms_p / psteps * 1e-3) / 1e12
        prefix = {"metric": "prefix-LM attention fwd TFLOPS", "value": whole_job_rate(pf, ms_p / psteps, world) / 1e12,
                  "unit": "TFLOP/s", "ms_per_step": ms_p / psteps, "steps": psteps, "prefix_len": plen,
                  "algorithmic_flops_per_launch": pf,
                  "roofline": {"bound": "tensor", "achieved": ptf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                               "frac": ptf / pk["bf16_tflops"], "peak_kind": f"{pk_kind} bf16 burst"},
                  "gpu_launches": psteps}
    # the backward pass on the same inputs (upstream gradient: seeded, tensor id 3)
    bwd = None
    if not args.no_backward:
        dout = to_dev(si.batched(seed, 3, B, (N, H, D), dt), dt, dev)
        gq, gk, gv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
        wsb = fa.fa_bwd_workspace_bytes(B, H, N)
        wsd = torch.empty(wsb, dtype=torch.uint8, device=dev)
        step()  # od, lse of these inputs

        def bstep():
            st = fa.fa_bwd(qd, kd, vd, od, dout, lse, gq, gk, gv, B, H, N, N, D, scale, causal, wsd, wsb, stream)
            if st:
                raise fa.FAError(st, "fa_bwd")

        for _ in range(args.warmup):
            bstep()
        bsteps = max(10, min(args.steps, 50))
        ms_b = timed(bstep, bsteps, stream, dist)
        if fa.fa_device_status(clear=True) != 0:
            raise RuntimeError("device status set during the timed backward run")
        bf = 2.5 * prefill_flops(B, H, N, N, D, causal)  # dV, dP, dQ, dK and the recomputed S
        btf = bf / (ms_b / bsteps * 1e-3) / 1e12
        bwd = {"metric": "attention bwd TFLOPS", "value": whole_job_rate(bf, ms_b / bsteps, world) / 1e12,
               "unit": "TFLOP/s", "ms_per_step": ms_b / bsteps, "steps": bsteps,
               "algorithmic_flops_per_step": bf,
               "note": "FLOPs counted as 2.5x the forward (five GEMMs); the kernels run seven (S and dP "
                       "are recomputed in both the dQ and the dK/dV kernel)",
               "roofline": {"bound": "tensor", "achieved": btf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                            "frac": btf / pk["bf16_tflops"], "peak_kind": f"{pk_kind} bf16 burst"},
               "gpu_launches": 3 * bsteps}
        del dout, gq, gk, gv, wsd

    flops_step = prefill_flops(B, H, N, N, D, causal)
    ms_step = ms / args.steps
    tflops_rank = flops_step / (ms_step * 1e-3) / 1e12
    value = whole_job_rate(flops_step, ms_step, world) / 1e12
    peak_b, peak_s = pk["bf16_tflops"], pk["bf16_tflops_sustained"]
    roof = {"bound": "tensor", "achieved": tflops_rank, "peak": peak_b, "unit": "TFLOP/s",
            "frac": tflops_rank / peak_b, "traffic": measured_traffic(args.workload),
            "traffic_unit": "bytes per launch (ncu dram read+write)",
            "kernel": f"fa_fwd_kernel<{D},bf16,out bf16>",
            "peak_kind": f"{pk_kind} bf16 burst", "frac_of_sustained": tflops_rank / peak_s,
            "algorithmic_flops_per_launch": flops_step}

    # ---------------- e2e through the C ABI with host buffers ----------------
    # Every step copies its Q, K, V from pinned host memory and reads its O and LSE back.  The copies
    # of consecutive steps overlap the kernel (H2D on one stream, fa_fwd on the launching stream, D2H
    # on a third, two device buffer sets), as a throughput caller would run it; the timed region
    # starts before the first step's H2D and ends after the last step's D2H.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (torch.from_numpy(np.ascontiguousarray(t).view(np.int16)).view(torch.bfloat16).pin_memory()
                      for t in (q, k, v))
        oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
        lh = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
        sets = [(qd, kd, vd, od, lse),
                (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd), torch.empty_like(od),
                 torch.empty_like(lse))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(nsteps):
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(nsteps):
                b = i % 2
                bq, bk, bv, bo, bl = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_done[b])  # the kernel of step i-2 has read these inputs
                    bq.copy_(qh, non_blocking=True)
                    bk.copy_(kh, non_blocking=True)
                    bv.copy_(vh, non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # the D2H of step i-2 has read these outputs
                st = fa.fa_fwd(bq, bk, bv, bo, bl, B, H, N, N, D, scale, causal, None, stream)
                if st:
                    raise fa.FAError(st, "fa_fwd")
                ev_done[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[b])
                    oh.copy_(bo, non_blocking=True)
                    lh.copy_(bl, non_blocking=True)
                    ev_out[b].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)

        e2e_steps = max(3, min(args.steps, 30))
        e2e_run(2)
        ms_e2e = timed_run(e2e_run, e2e_steps, stream, dist)
        if fa.fa_device_status(clear=True) != 0:
            raise RuntimeError("device status set during the timed e2e run")
        h2d = 3 * qh.numel() * 2
        d2h = oh.numel() * 2 + lh.numel() * 4
        e2e = {"value": flops_step * world / (ms_e2e / e2e_steps * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": ms_e2e / e2e_steps,
               "overlap": "H2D, kernel and D2H of consecutive steps on three streams, two device buffer sets"}
        del qh, kh, vh, oh, lh, sets
    del qd, kd, vd, od, lse
    torch.cuda.empty_cache()

    return value, ms_step, roof, e2e, clk, prefix, bwd


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefix", action="store_true", help="skip the prefix-mask timing of the prefill inputs")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing of the prefill inputs")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the timing of the other prefill workloads (the other head dim, varlen)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--only", choices=["all", "prefill", "decode", "varlen", "other"], default="all",
                    help="profiling runs: time only the headline prefill, the decode legs, the varlen leg, "
                         "or the other head dim's prefill leg")
    ap.add_argument("--workload", choices=["prefill_d64", "prefill_d128"], default=HEADLINE,
                    help="prefill workload of the headline leg (default: the D=64 configuration)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="profiling runs: smaller decode batch than the workload's B=64")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import exact_tiled_attention_47_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        dist = tdist
    fa._lib.load()
    pk, pk_kind = peaks()

    # ---------------- prefill headline ----------------
    cfg = si.CONFIGS[args.workload]
    run_prefill = args.only in ("all", "prefill")
    run_decode = args.only in ("all", "decode") and not args.no_decode
    B, N, H, D, dt = cfg["B"], cfg["Nq"], cfg["H"], cfg["D"], cfg["dtype"]
    scale = cfg["scale"]
    stream = torch.cuda.current_stream(dev)
    value = ms_step = None
    roof = e2e = prefix = bwd = None
    clk = ClockSampler(local)
    if run_prefill:
        value, ms_step, roof, e2e, clk, prefix, bwd = prefill_leg(args, cfg, dev, rank, world, dist, pk, pk_kind,
                                                                  fa, torch)

    # ---------------- the other prefill workloads ----------------
    others = {}
    if not args.no_others:
        other = "prefill_d128" if args.workload == "prefill_d64" else "prefill_d64"
        if args.only in ("all", "other"):
            others["p128" if other == "prefill_d128" else "p64"] = other_prefill_leg(
                args, other, dev, rank, world, dist, pk, pk_kind, fa, torch)
        if args.only in ("all", "varlen"):
            others["varlen"] = other_prefill_leg(args, "varlen", dev, rank, world, dist, pk, pk_kind, fa, torch)

    # ---------------- decode (secondary metric) ----------------
    dec = None
    if run_decode:
        c = si.CONFIGS["decode"]
        Bd, Hd, Nk, Dd, S = c["B"], c["H"], c["Nk"], c["D"], c["num_splits"]
        if args.decode_batch:
            Bd = args.decode_batch
        dseed = rank_seed(c["seed"], rank)
        qd_ = to_dev(si.batched(dseed, si.Q_ID, Bd, (1, Hd, Dd), "bf16"), "bf16", dev)
        kc = torch.empty((Bd, Nk, Hd, Dd), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        for b in range(Bd):  # chunked upload keeps host memory bounded
            kc[b].copy_(to_dev(si.batch_item(dseed, si.K_ID, b, (Nk, Hd, Dd), "bf16"), "bf16", dev))
            vc[b].copy_(to_dev(si.batch_item(dseed, si.V_ID, b, (Nk, Hd, Dd), "bf16"), "bf16", dev))
        o_ = torch.empty_like(qd_)
        l_ = torch.empty((Bd, Hd), dtype=torch.float32, device=dev)
        wsb = fa.fa_decode_workspace_bytes(Bd, Hd, Dd, S)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        dscale = c["scale"]

        def dstep():
            st = fa.fa_decode_splitkv(qd_, kc, vc, o_, l_, Bd, Hd, Nk, Dd, dscale, S, ws, wsb, stream)
            if st:
                raise fa.FAError(st, "fa_decode_splitkv")

        for _ in range(args.warmup):
            dstep()
        dsteps = max(10, args.steps // 2)
        ms_d = timed(dstep, dsteps, stream, dist)
        if fa.fa_device_status(clear=True) != 0:
            raise RuntimeError("device status set during the timed decode run")
        kv_bytes = 2 * Bd * Nk * Hd * Dd * 2
        alg_bytes = kv_bytes + 2 * Bd * Hd * Dd * 2 + Bd * Hd * 4
        gbs = alg_bytes / (ms_d / dsteps * 1e-3) / 1e9
        dec = {"metric": "decode HBM GB/s", "value": gbs * world, "unit": "GB/s",
               "ms_per_step": ms_d / dsteps, "steps": dsteps,
               "config": {"workload": "decode", "B": Bd, "H": Hd, "Nk": Nk, "D": Dd, "num_splits": S,
                          "dtype": "bf16", "l2": f"K/V cache {kv_bytes / 1e9:.2f} GB vs 126 MB L2"},
               "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                            "frac": gbs / pk["hbm_gbs"], "traffic": measured_traffic("decode", Bd),
                            "peak_kind": f"{pk_kind} copy", "algorithmic_bytes_per_step": alg_bytes},
               "gpu_launches": 2 * dsteps}
        if Bd == c["B"]:
            dec["sharded"] = sharded_leg(args, kc, vc, dev, rank, world, dist, pk, pk_kind, fa, torch, stream, dsteps)
        del qd_, kc, vc, o_, l_, ws
        torch.cuda.empty_cache()

        # grouped KV heads with per-sequence cache lengths
        g = si.CONFIGS["decode_gqa"]
        Bg, Hq, Hkv, Nkg, Dg, Sg = g["B"], g["H"], g["Hkv"], g["Nk"], g["D"], g["num_splits"]
        if args.decode_batch:
            Bg = args.decode_batch
        gseed = rank_seed(g["seed"], rank)
        lens = si.varlen_lengths(g["seed"], Bg, g["len_lo"], g["len_hi"])
        qg = to_dev(si.batched(gseed, si.Q_ID, Bg, (1, Hq, Dg), "bf16"), "bf16", dev)
        kg = torch.empty((Bg, Nkg, Hkv, Dg), dtype=torch.bfloat16, device=dev)
        vg = torch.empty_like(kg)
        for b in range(Bg):
            kg[b].copy_(to_dev(si.batch_item(gseed, si.K_ID, b, (Nkg, Hkv, Dg), "bf16"), "bf16", dev))
            vg[b].copy_(to_dev(si.batch_item(gseed, si.V_ID, b, (Nkg, Hkv, Dg), "bf16"), "bf16", dev))
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        og = torch.empty_like(qg)
        lg_ = torch.empty((Bg, Hq), dtype=torch.float32, device=dev)
        wsbg = fa.fa_decode_workspace_bytes(Bg, Hq, Dg, Sg)
        wsg = torch.empty(wsbg, dtype=torch.uint8, device=dev)

        def gstep():
            st = fa.fa_decode_splitkv_gqa(qg, kg, vg, og, lg_, Bg, Hq, Hkv, Nkg, Dg, g["scale"], Sg, sl, wsg, wsbg,
                                          stream)
            if st:
                raise fa.FAError(st, "fa_decode_splitkv_gqa")

        for _ in range(args.warmup):
            gstep()
        ms_g = timed(gstep, dsteps, stream, dist)
        if fa.fa_device_status(clear=True) != 0:
            raise RuntimeError("device status set during the timed grouped decode run")
        kv_g = 2 * int(lens.sum()) * Hkv * Dg * 2  # valid K and V rows only
        alg_g = kv_g + 2 * Bg * Hq * Dg * 2 + Bg * Hq * 4
        gbs_g = alg_g / (ms_g / dsteps * 1e-3) / 1e9
        dec["gqa"] = {"metric": "grouped decode HBM GB/s", "value": gbs_g * world, "unit": "GB/s",
                      "ms_per_step": ms_g / dsteps, "steps": dsteps,
                      "config": {"workload": "decode_gqa", "B": Bg, "Hq": Hq, "Hkv": Hkv, "Nk_capacity": Nkg,
                                 "D": Dg, "num_splits": Sg, "lengths": f"U{{{g['len_lo']}..{g['len_hi']}}}",
                                 "valid_kv_bytes": kv_g},
                      "roofline": {"bound": "hbm", "achieved": gbs_g, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                   "frac": gbs_g / pk["hbm_gbs"], "peak_kind": f"{pk_kind} copy",
                                   "traffic": measured_traffic("decode_gqa", kv_g),
                                   "algorithmic_bytes_per_step": alg_g},
                      "gpu_launches": 2 * dsteps}

        # the same workload over a paged cache: the valid rows of each sequence in pages of 16 rows
        # at seeded pool positions (the pool is built on the device from the contiguous cache)
        pc = si.CONFIGS["decode_paged"]
        ps = pc["page_size"]
        need = [(int(L) + ps - 1) // ps for L in lens]
        n_pages = sum(need)
        pps = (Nkg + ps - 1) // ps
        perm = np.random.default_rng(rank_seed(pc["seed"], rank)).permutation(n_pages)
        table = np.full((Bg, pps), -1, dtype=np.int32)
        kp = torch.empty((n_pages, ps, Hkv, Dg), dtype=torch.bfloat16, device=dev)
        vp = torch.empty_like(kp)
        t0 = 0
        for b, n in enumerate(need):
            pages = perm[t0:t0 + n]
            t0 += n
            table[b, :n] = pages
            idx = torch.from_numpy(pages).to(dev)
            kp[idx] = kg[b, :n * ps].view(n, ps, Hkv, Dg)
            vp[idx] = vg[b, :n * ps].view(n, ps, Hkv, Dg)
        del kg, vg
        torch.cuda.empty_cache()
        tbl = torch.from_numpy(table).to(dev)

        def pstep():
            st = fa.fa_decode_splitkv_paged(qg, kp, vp, tbl, og, lg_, Bg, Hq, Hkv, n_pages, ps, pps, Dg, g["scale"],
                                            Sg, sl, wsg, wsbg, stream)
            if st:
                raise fa.FAError(st, "fa_decode_splitkv_paged")

        for _ in range(args.warmup):
            pstep()
        ms_p = timed(pstep, dsteps, stream, dist)
        if fa.fa_device_status(clear=True) != 0:
            raise RuntimeError("device status set during the timed paged decode run")
        alg_p = alg_g + 4 * n_pages  # plus the table entries read
        gbs_p = alg_p / (ms_p / dsteps * 1e-3) / 1e9
        dec["paged"] = {"metric": "paged decode HBM GB/s", "value": gbs_p * world, "unit": "GB/s",
                        "ms_per_step": ms_p / dsteps, "steps": dsteps,
                        "config": {"workload": "decode_paged", "B": Bg, "Hq": Hq, "Hkv": Hkv, "D": Dg,
                                   "num_splits": Sg, "lengths": f"U{{{g['len_lo']}..{g['len_hi']}}}",
                                   "page_size": ps, "pages": n_pages, "pages_per_seq": pps,
                                   "page_order": "seeded permutation of the pool", "valid_kv_bytes": kv_g},
                        "roofline": {"bound": "hbm", "achieved": gbs_p, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs_p / pk["hbm_gbs"], "peak_kind": f"{pk_kind} copy",
                                     "traffic": measured_traffic("decode_paged", kv_g),
                                     "algorithmic_bytes_per_step": alg_p},
                        "gpu_launches": 2 * dsteps}
        del qg, kp, vp, tbl, og, lg_, wsg, sl
        torch.cuda.empty_cache()

    # ---------------- CPU baseline (oracle) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and run_prefill:
        f, s, desc = oracle_prefill_sample(cfg, args.cpu_budget)
        cpu = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc, "seconds": s}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "H": H, "N": N, "D": D,
                   "causal": bool(cfg.get("causal", False)), "input_dtype": dt, "output_dtype": "bf16",
                   "scale": scale,
                   "l2": f"inputs {3 * B * N * H * D * 2 / 2**20:.0f} MiB > 126 MB L2 (no flush needed)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roof, "clocks": clk.summary(), "e2e": e2e,
        "gpu_launches": args.steps if run_prefill else 0,
        "decode": dec, "prefix": prefix, "backward": bwd, "cpu_baseline": cpu,
    }
    line.update(others)
    add_token_rates(line, world)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
