"""Host-side multi-rank logic of bench.py on CPU: world_size 2 over gloo.

bench.py shards nothing (each rank streams its own layer stack); what needs checking is the
rank plumbing: set-up from the torchrun environment, barriers, the max-over-ranks time and
the sum-over-ranks work that make the whole-job number.
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

from tests.conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


CHILD = textwrap.dedent(
    """
    import os, sys, json
    sys.path.insert(0, {root!r})
    import bench
    rank, world, local = bench.dist_setup()
    bench.barrier(world)
    t = 10.0 + rank            # this rank's "elapsed ms"
    work = 100.0 * (rank + 1)  # this rank's "bytes"
    out = {{"rank": rank, "world": world, "max": bench.max_over_ranks(t, world),
            "sum": bench.sum_over_ranks(work, world)}}
    bench.barrier(world)
    bench.teardown(world)
    print(json.dumps(out))
    """
)


def test_two_gloo_ranks_agree_on_max_time_and_total_work(tmp_path):
    script = tmp_path / "child.py"
    script.write_text(CHILD.format(root=ROOT))
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=180)
        assert p.returncode == 0, e
        outs.append(o.strip().splitlines()[-1])
    import json
    res = sorted((json.loads(o) for o in outs), key=lambda d: d["rank"])
    for d in res:
        assert d["world"] == 2
        assert d["max"] == pytest.approx(11.0)
        assert d["sum"] == pytest.approx(300.0)


def test_single_rank_needs_no_process_group(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_setup() == (0, 1, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(2.0, 1) == 2.0


def test_reference_arm_line_shape(monkeypatch):
    """--impl reference prints one JSON line with the oracle's sample and no GPU use."""
    import bench
    monkeypatch.setattr(bench, "oracle_sample", lambda wl, rows: [])
    monkeypatch.setattr(bench, "oracle_step", lambda s: 1000)
    args = type("A", (), {"workload": "opt-6.7b-decode", "steps": 3, "warmup": 3})()
    line = bench.run_reference(args)
    assert line["impl"] == "reference"
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


FAILING_CHILD = textwrap.dedent(
    """
    import os, sys, time
    sys.path.insert(0, {root!r})
    import bench
    rank, world, local = bench.dist_setup()
    if rank == 1:
        raise RuntimeError("rank 1 fails between steps")
    t0 = time.time()
    try:
        bench.barrier(world)
    except Exception as e:
        print("collective-error after %.1f s: %s" % (time.time() - t0, type(e).__name__))
        sys.exit(3)
    print("no error")
    """
)


def _launch(script, ranks, world, port, timeout_s):
    procs = {}
    for r in ranks:
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="",
                   OWQ_PG_TIMEOUT_S=str(timeout_s))
        procs[r] = subprocess.Popen([sys.executable, str(script)], env=env,
                                    stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
    return procs


def test_a_rank_that_raises_ends_the_others_collective_with_an_error(tmp_path):
    script = tmp_path / "failing.py"
    script.write_text(FAILING_CHILD.format(root=ROOT))
    procs = _launch(script, (0, 1), 2, _free_port(), 10)
    out = {r: p.communicate(timeout=120) for r, p in procs.items()}
    assert procs[1].returncode != 0 and "rank 1 fails" in out[1][1]
    assert procs[0].returncode == 3, out[0]
    assert "collective-error" in out[0][0]


def test_a_rank_that_never_joins_ends_set_up_with_an_error(tmp_path):
    script = tmp_path / "failing.py"
    script.write_text(FAILING_CHILD.format(root=ROOT))
    procs = _launch(script, (0,), 2, _free_port(), 5)   # rank 1 is never started
    o, e = procs[0].communicate(timeout=120)
    assert procs[0].returncode != 0
    assert "no error" not in o


def test_row_ranges_cover_whole_tiles():
    from weight_only_mixed_owq_b200 import shard
    for N in (1, 15, 16, 17, 100, 4096, 4100, 36864):
        for world in (1, 2, 3, 4, 8):
            rs = [shard.row_range(N, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == N
            for (a, b), (c, d) in zip(rs, rs[1:]):
                assert b == c and a <= b
            for lo, hi in rs:
                if hi < N:     # every shard but the one that ends the layer is whole tiles
                    assert lo % 16 == 0 and (hi - lo) % 16 == 0
                else:          # that one, and any empty ones after it, start on a tile boundary
                    assert lo % 16 == 0 or lo == N
            tiles = [-(-(hi - lo) // 16) for lo, hi in rs]
            assert max(tiles) - min(tiles) <= 1


SHARD_CHILD = textwrap.dedent(
    """
    import os, sys, json
    import numpy as np
    sys.path.insert(0, {root!r})
    import torch, torch.distributed as dist
    import oracle, owq_synth
    from weight_only_mixed_owq_b200 import shard
    import bench
    rank, world, local = bench.dist_setup()
    N, K, bits, group, k, M = {N}, 512, 3, 128, 5, 3
    d = owq_synth.draw_small(N, K, M, 64, seed=55, n_outliers=3)
    q = oracle.owq_quantize(d["W"], d["X"], bits, group, k)     # same on every rank (seeded)
    lo, hi = shard.row_range(N, world, rank)
    part = shard.shard_operands(q, lo, hi)
    # this rank's product over its rows (the library's kernel on a GPU; the oracle here)
    W_hat = oracle.dequant(part["codes"], part["scales"], part["zeros"])
    y_local = torch.from_numpy(oracle.matmul(W_hat, part["w_weak"], part["idx"], d["x"]))
    y = shard.all_gather_rows(y_local, N, world).numpy()
    full = oracle.matmul(oracle.dequant(q["codes"], q["scales"], q["zeros"]), q["w_weak"], q["idx"], d["x"])
    out = {{"rank": rank, "lo": lo, "hi": hi, "equal": bool(np.array_equal(y, full)), "shape": list(y.shape)}}
    bench.teardown(world)
    print(json.dumps(out))
    """
)


@pytest.mark.parametrize("N", [96, 100])
def test_row_sharded_product_all_gathers_to_the_single_rank_result(tmp_path, N):
    """Two gloo ranks each own a block of whole 16-row tiles of one layer, compute their rows
    and all-gather y: the result equals the single-rank product exactly (rows are independent,
    so nothing is re-associated).  Not measured on GPU hardware: every call there has one GPU."""
    script = tmp_path / "shard_child.py"
    script.write_text(SHARD_CHILD.format(root=ROOT, N=N))
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    import json
    res = []
    for p in procs:
        o, e = p.communicate(timeout=180)
        assert p.returncode == 0, e
        res.append(json.loads(o.strip().splitlines()[-1]))
    res.sort(key=lambda d: d["rank"])
    assert res[0]["lo"] == 0 and res[0]["hi"] == res[1]["lo"] and res[1]["hi"] == N
    for d in res:
        assert d["equal"] and d["shape"] == [3, N]
