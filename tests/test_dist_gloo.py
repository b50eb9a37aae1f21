"""Multi-process plumbing of bench.py on CPU: two gloo ranks (no GPU).

Each rank gets its own batch (distinct seeded inputs), the job time is the slowest rank's, and the
whole-job rate counts every rank's work over that time.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import seeded_inputs as si
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, dist, device="cpu")
        seed = bench.rank_seed(2, rank)
        q = si.batch_item(seed, si.Q_ID, 0, (4, 2, 8), "bf16")
        digest = int(np.frombuffer(q.tobytes(), dtype=np.uint16).astype(np.int64).sum())
        rate = bench.whole_job_rate(1e9, ms_max, world)
        out.put((rank, ms_max, digest, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, d0, rate0), (r1, ms1, d1, rate1) = res
    assert ms0 == ms1 == 15.0          # max over ranks, seen identically by both
    assert d0 != d1                    # each rank has its own batch
    assert rate0 == rate1 == pytest.approx(2 * 1e9 / 0.015)


def test_single_process_defaults():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.rank_seed(5, 0) == 5
    assert bench.whole_job_rate(10.0, 1000.0, 1) == pytest.approx(10.0)


def _shard_worker(rank, world, port, out):
    """One rank of the key-sharded decode exchange: the shard result comes from the oracle (the
    stand-in for the shard kernel on a CPU), is packed in the library's block layout and gathered
    with the library's exchange step; the merge of the gathered blocks must equal the decode over
    the whole cache."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import seeded_inputs as si
        from exact_tiled_attention_47_b200.sharded import gather_parts, part_floats, shard_range
        B, Hq, Hkv, Nk, D, scale = 3, 4, 2, 37, 64, 0.125
        lens = [37, 18, 0]  # the second ends inside the first shard (2 ranks) or the second (3), the third is empty
        qb, kb, vb = si.decode_gqa_inputs(41, B, Nk, Hq, Hkv, D, "bf16")
        q, k, v = (si.bits_to_float(t, "bf16") for t in (qb, kb, vb))
        off, n = shard_range(Nk, world, rank)
        o_r, l_r = oracle.attention_decode_shard(q, k[:, off:off + n], v[:, off:off + n], scale, off, lens)
        nf = part_floats(B, Hq, D)
        part = torch.full((nf,), float("nan"), dtype=torch.float32)
        part[:B * Hq * D] = torch.from_numpy(o_r.reshape(-1).astype(np.float32))
        part[B * Hq * D:B * Hq * (D + 1)] = torch.from_numpy(l_r.reshape(-1).astype(np.float32))
        gathered = gather_parts(part, world).numpy().astype(np.float64)
        o_ref, lse_ref = oracle.attention_decode_gqa(q, k, v, scale, lens)
        err_o = err_l = 0.0
        for b in range(B):
            for h in range(Hq):
                row = b * Hq + h
                o_parts = [gathered[r * nf + row * D:r * nf + (row + 1) * D] for r in range(world)]
                l_parts = [gathered[r * nf + B * Hq * D + row] for r in range(world)]
                o, lse = oracle.combine_partials(o_parts, l_parts)
                err_o = max(err_o, float(np.abs(o - o_ref[b, 0, h]).max()))
                if lse_ref[b, h] == -np.inf:
                    assert lse == -np.inf
                else:
                    err_l = max(err_l, abs(lse - lse_ref[b, h]))
        mine = gathered[rank * nf:rank * nf + B * Hq * D]
        out.put((rank, (off, n), err_o, err_l, bool(np.array_equal(mine, part[:B * Hq * D].numpy()))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_exchange_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    bounds = [r[1] for r in res]                      # contiguous shards covering the 37 keys
    assert bounds[0][0] == 0 and bounds[-1][0] + bounds[-1][1] == 37
    assert all(a[0] + a[1] == b[0] for a, b in zip(bounds, bounds[1:]))
    if world == 2:
        assert bounds == [(0, 19), (19, 18)]
    for _, _, err_o, err_l, own_block_in_place in res:
        assert own_block_in_place                       # block r of the gather is rank r's
        assert err_o < 1e-6 and err_l < 1e-6            # fp32 packing is the only rounding


def test_shard_ranges_cover_the_cache():
    from exact_tiled_attention_47_b200.sharded import shard_range
    for total in (8, 37, 131072, 131073):
        for world in (1, 2, 3, 8):
            got = [shard_range(total, world, r) for r in range(world)]
            assert got[0][0] == 0
            assert all(a[0] + a[1] == b[0] for a, b in zip(got, got[1:]))
            assert got[-1][0] + got[-1][1] == total
            assert max(n for _, n in got) - min(n for _, n in got) <= 1
    with pytest.raises(ValueError):
        shard_range(3, 4, 0)
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _decode_sharded_worker(rank, world, port, out):
    """One rank calling the public helper decode_sharded on CPU tensors.  Its two library calls are
    replaced by stand-ins computed with the oracle that honour the documented block layout (the
    shard's fp32 O [B,H,D] then LSE [B,H], padded to 16 bytes; blocks in rank order), so what is
    tested is the helper itself: part sizing, layout, the all-gather and the merge call."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import seeded_inputs as si
        import exact_tiled_attention_47_b200 as fa
        from exact_tiled_attention_47_b200.sharded import decode_sharded, shard_range
        B, Hq, Hkv, Nk, D, scale = 2, 4, 2, 50, 64, 0.2
        lens = [50, 23]
        qb, kb, vb = si.decode_gqa_inputs(43, B, Nk, Hq, Hkv, D, "bf16")
        q, k, v = (si.bits_to_float(t, "bf16") for t in (qb, kb, vb))
        calls = {}

        def fake_shard(q_, k_, v_, part, B_, Hq_, Hkv_, Nk_shard, key_offset, Nk_total, D_, scale_, S_, sl, ws,
                       workspace_bytes=None, stream=None, in_dtype=None):
            calls["shard"] = (Nk_shard, key_offset, Nk_total)
            o_r, l_r = oracle.attention_decode_shard(q_.double().numpy(), k_.double().numpy(), v_.double().numpy(),
                                                     scale_, key_offset, None if sl is None else sl.tolist())
            part[:B_ * Hq_ * D_] = torch.from_numpy(o_r.reshape(-1)).float()
            part[B_ * Hq_ * D_:B_ * Hq_ * (D_ + 1)] = torch.from_numpy(l_r.reshape(-1)).float()
            return 0

        def fake_merge(parts, R, B_, H_, D_, o, lse, stream=None, o_dtype=None):
            calls["merge"] = (R, parts.numel())
            nf = parts.numel() // R
            blocks = parts.view(R, nf).double().numpy()
            for row in range(B_ * H_):
                ob, lb = oracle.combine_partials([blk[row * D_:(row + 1) * D_] for blk in blocks],
                                                 [blk[B_ * H_ * D_ + row] for blk in blocks])
                o.view(B_ * H_, D_)[row] = torch.from_numpy(ob).to(o.dtype)
                lse.view(-1)[row] = float(lb)
            return 0

        fa.fa_decode_splitkv_shard = fake_shard
        fa.fa_decode_merge = fake_merge
        off, n = shard_range(Nk, world, rank)
        qt = torch.from_numpy(q).float()
        kt = torch.from_numpy(np.ascontiguousarray(k[:, off:off + n])).float()
        vt = torch.from_numpy(np.ascontiguousarray(v[:, off:off + n])).float()
        o, lse = decode_sharded(qt, kt, vt, off, Nk, scale=scale, num_splits=4,
                                seqlens_k=torch.tensor(lens, dtype=torch.int32), out_dtype=torch.float32)
        o_ref, lse_ref = oracle.attention_decode_gqa(q, k, v, scale, lens)
        out.put((rank, calls["shard"], calls["merge"], float(np.abs(o.numpy() - o_ref).max()),
                 float(np.abs(lse.numpy() - lse_ref).max())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_decode_sharded_helper_gloo():
    from exact_tiled_attention_47_b200 import build
    build.build()  # the helper sizes its buffers through the library's host functions
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_decode_sharded_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from exact_tiled_attention_47_b200.sharded import part_floats
    for rank, shard, merge, err_o, err_l in res:
        assert shard == ((25, 25 * rank, 50))                      # this rank's keys of the 50-key cache
        assert merge == (2, 2 * part_floats(2, 4, 64))             # both ranks' blocks, one merge
        assert err_o < 1e-6 and err_l < 1e-6                       # fp32 blocks are the only rounding
