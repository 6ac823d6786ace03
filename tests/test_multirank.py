"""Two ranks of the multi-GPU plumbing, run on CPU with the gloo backend.

Units (one KV head of one layer of one sequence) are independent, so at N
GPUs each rank prunes its own units with no exchange on the data path; the
only collectives are the barrier around the timed region and the max over
ranks of its duration.  These tests start two gloo ranks as processes on
127.0.0.1 and check:

- the bench's process-group setup, barrier and max over ranks;
- that the reference arm runs and prints on rank 0 only;
- that sharding a step by sequence is exact: a rank that prunes only its own
  sequence's units (p_cur of that sequence, the per-layer statistics) gets
  the rows the whole step gets for those units, so no step of the method
  couples units of different sequences.
"""
import argparse
import contextlib
import io
import json
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(rank, port, fn_name, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(WORLD),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      CUDA_VISIBLE_DEVICES="")
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    try:
        ws, r, _ = bench.dist_setup()
        out = globals()[fn_name](bench, ws, r)
        q.put((rank, "ok", out))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, "error", repr(e)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run(fn_name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_child, args=(r, port, fn_name, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(WORLD):
            rank, status, out = q.get(timeout=240)
            assert status == "ok", f"rank {rank}: {out}"
            results[rank] = out
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    return results


# ---------------------------------------------------------------------------
# rank bodies (run in the children)
# ---------------------------------------------------------------------------
def _body_max(bench, ws, rank):
    import torch.distributed as dist

    assert ws == WORLD and dist.get_backend() == "gloo"
    bench.barrier(ws)
    m = bench.max_over_ranks(10.0 + 5.0 * rank, ws)
    m2 = bench.max_over_ranks(-1.0 - rank, ws)
    bench.barrier(ws)
    return (m, m2)


def _body_reference(bench, ws, rank):
    args = argparse.Namespace(workload="c1", steps=1, warmup=3, gpus=ws, impl="reference")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, ws, rank)
    bench.barrier(ws)
    return buf.getvalue()


def _shard_spec():
    import synth

    return synth.Spec("shard", WORLD, 2, 2, 2, 224, 200, 64, "f32", 512, 4096,
                      positions="scattered", stream=7)


def _shard_stats(spec, wl):
    import oracle
    import synth

    return np.stack([oracle.calibrate(synth.host_elems(synth.calib_queries(spec, wl.hp, l, "cpu")))
                     for l in range(spec.n_layers)])


def _body_shard(bench, ws, rank):
    import torch
    import torch.distributed as dist

    import oracle
    import synth

    oracle.set_threads(1)
    spec = _shard_spec()
    wl = synth.make_workload(spec, "cpu")
    st = _shard_stats(spec, wl)
    per = spec.n_layers * spec.n_kvheads            # units of one sequence
    u0 = rank * per
    sl = slice(u0, u0 + per)
    out = oracle.prune(synth.host_elems(wl.k[sl]), synth.host_elems(wl.v[sl]), wl.pos[sl].numpy(),
                       1, spec.n_layers, spec.n_kvheads, spec.G, st,
                       wl.p_cur[rank:rank + 1].numpy(), spec.B, n_valid=wl.n_valid[sl].numpy())
    mine = {k: out[k] for k in ("kept", "n_kept", "final", "k_dst", "v_dst", "pos_dst")}
    gathered = [None] * ws
    dist.all_gather_object(gathered, (rank, mine))
    t = torch.tensor([float(out["n_kept"].sum())])
    dist.all_reduce(t)
    return {"shards": gathered, "total_kept": float(t.item())}


# ---------------------------------------------------------------------------
# tests
# ---------------------------------------------------------------------------
def test_barrier_and_max_over_ranks():
    res = _run("_body_max")
    assert res[0] == res[1] == (15.0, -1.0)


def test_reference_arm_prints_on_rank0_only():
    res = _run("_body_reference")
    lines = [l for l in res[0].splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == WORLD
    assert rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
    assert res[1].strip() == ""


def test_sequence_shards_equal_the_whole_step():
    import oracle
    import synth

    res = _run("_body_shard")
    spec = _shard_spec()
    wl = synth.make_workload(spec, "cpu")
    st = _shard_stats(spec, wl)
    whole = oracle.prune(synth.host_elems(wl.k), synth.host_elems(wl.v), wl.pos.numpy(),
                         spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, st,
                         wl.p_cur.numpy(), spec.B, n_valid=wl.n_valid.numpy())
    per = spec.n_layers * spec.n_kvheads
    for r in range(WORLD):
        shards = dict(res[r]["shards"])
        assert set(shards) == set(range(WORLD))
        for rank, mine in shards.items():
            sl = slice(rank * per, (rank + 1) * per)
            np.testing.assert_array_equal(mine["kept"], whole["kept"][sl])
            np.testing.assert_array_equal(mine["n_kept"], whole["n_kept"][sl])
            np.testing.assert_array_equal(mine["final"], whole["final"][sl])
            np.testing.assert_array_equal(mine["pos_dst"], whole["pos_dst"][sl])
            assert mine["k_dst"].tobytes() == whole["k_dst"][sl].tobytes()
            assert mine["v_dst"].tobytes() == whole["v_dst"][sl].tobytes()
        assert res[r]["total_kept"] == float(whole["n_kept"].sum())
    # the shards really differ (each sequence draws its own keys and positions)
    assert not np.array_equal(whole["kept"][:per], whole["kept"][per:])


if __name__ == "__main__":  # pragma: no cover
    sys.exit(pytest.main([__file__, "-q"]))
