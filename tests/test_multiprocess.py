"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2).

The decode path shards into independent (sequence, kv-head) groups with no exchange, so the only
collective steps are the barrier and the max-over-ranks reduction of the timed region; whole-job
throughput is the units all ranks processed divided by that max time (weak scaling).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    class A:
        pass

    w, r, _ = bench.dist_setup(A())
    assert (w, r) == (world, rank)
    bench.barrier(w)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    out.put((rank, t))
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def test_weak_scaling_value_formula():
    sys.path.insert(0, ROOT)
    import bench
    # value = units of all ranks / max time: 2 ranks x 10 steps x 32 layers in 0.5 s
    world, steps, layers, ms_max = 2, 10, bench.LAYERS, 500.0
    assert world * steps * layers / (ms_max / 1e3) == pytest.approx(1280.0)


@pytest.mark.slow
def test_reference_arm_under_torchrun_rank0_only():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "layer-steps/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def _shard_worker(rank, world, port, out):
    """A rank of the kv-head split: its shard of one layer through the oracle (the stand-in for
    the rank's GPU step), then the all-gather of o / lse."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    from adaptive_top_sparse_b200.shard import gather_heads, shard_layer
    from oracle import twl_oracle as O
    from workloads import synth

    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = synth.make_decode("tp", 2, 24, 6, [700, 333], seed=17, permute_pages=True,
                           temperature=True)
    k, v, q, hq, hkv = shard_layer(wl.k, wl.v, wl.q, wl.num_q_heads, wl.num_kv_heads, rank, world)
    sub = synth.DecodeWorkload(name=f"tp{rank}", q=np.ascontiguousarray(q),
                               k=np.ascontiguousarray(k), v=np.ascontiguousarray(v),
                               page_table=wl.page_table, seq_lens=wl.seq_lens, num_q_heads=hq,
                               num_kv_heads=hkv, p=wl.p, eps=wl.eps)
    r = O.decode_step(sub)
    g = hq // hkv
    o = torch.zeros((wl.batch, hq, 128), dtype=torch.float64)
    lse = torch.zeros((wl.batch, hq), dtype=torch.float64)
    for (b, kvh), grp in r["groups"].items():
        for h in range(kvh * g, (kvh + 1) * g):
            o[b, h] = torch.from_numpy(np.asarray(grp["o"][h], dtype=np.float64))
            lse[b, h] = float(grp["lse"][h])
    o_all, lse_all = gather_heads(o, lse, wl.num_q_heads, wl.num_kv_heads, world)
    out.put((rank, o_all.numpy(), lse_all.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_kv_head_split_gathers_the_whole_layer(world):
    """Two (and four, uneven) ranks each run their kv-heads' shard of a layer; the all-gather of
    o / lse equals the single-rank result of the whole layer (the oracle stands in for each rank's
    GPU step: the split is host logic and one collective)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    from oracle import twl_oracle as O
    from workloads import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = synth.make_decode("tp", 2, 24, 6, [700, 333], seed=17, permute_pages=True,
                           temperature=True)
    ref = O.decode_step(wl)
    g = wl.num_q_heads // wl.num_kv_heads
    for rank, o_all, lse_all in got:
        for (b, kvh), grp in ref["groups"].items():
            for h in range(kvh * g, (kvh + 1) * g):
                assert np.array_equal(o_all[b, h], np.asarray(grp["o"][h])), (rank, b, h)
                assert lse_all[b, h] == grp["lse"][h], (rank, b, h)


def test_kv_head_ranges_cover_every_head_once():
    sys.path.insert(0, ROOT)
    from adaptive_top_sparse_b200.shard import kv_head_range
    for hkv in (1, 2, 6, 8, 13):
        for world in range(1, hkv + 1):
            owned = []
            for r in range(world):
                lo, hi = kv_head_range(hkv, r, world)
                assert hi - lo in (hkv // world, -(-hkv // world))
                owned += list(range(lo, hi))
            assert owned == list(range(hkv))
    with pytest.raises(ValueError):
        kv_head_range(2, 0, 3)


def test_shard_slices_are_contiguous_for_numpy_and_torch():
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    from adaptive_top_sparse_b200.shard import shard_layer
    k = np.arange(5 * 4 * 16 * 128, dtype=np.float32).reshape(5, 4, 16, 128).astype(np.float16)
    q = np.arange(2 * 12 * 128, dtype=np.float32).reshape(2, 12, 128).astype(np.float16)
    for conv in (lambda x: x, torch.from_numpy):
        ks, vs, qs, hq, hkv = shard_layer(conv(k), conv(k), conv(q), 12, 4, 1, 2)
        assert (hq, hkv) == (6, 2)
        for x in (ks, vs, qs):
            assert x.flags["C_CONTIGUOUS"] if isinstance(x, np.ndarray) else x.is_contiguous()
        assert np.array_equal(np.asarray(qs), q[:, 6:12]) and np.array_equal(np.asarray(ks), k[:, 2:4])
