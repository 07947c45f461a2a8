"""The multi-host form (Star Attention across ranks) on CPU: 2 and 3 gloo ranks run
the sharded layer's host logic (block assignment, anchor broadcast, query
broadcast, partial gather, merge on the query host) with the oracle as compute,
and must reproduce the single-host oracle: every rank's Phase-1 rows, the query
tokens' and two decode steps' outputs and LSEs."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBackend:
    """The sharded layer's compute on the CPU oracle (float64 torch tensors)."""

    def __init__(self):
        sys.path.insert(0, ROOT)
        import oracle
        self.oracle = oracle

    @staticmethod
    def _np(t):
        return None if t is None else t.numpy()

    def phase1(self, q, k, v, block_size):
        o, lse = self.oracle.phase1(q.numpy(), k.numpy(), v.numpy(), block_size)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def phase1_anchored(self, q, k, v, k_anchor, v_anchor, block_size):
        # The definition: this host's blocks are blocks i > 0 of a context that starts
        # with the anchor, so their rows are those of Phase 1 over [anchor ; blocks].
        B = block_size
        qa = np.concatenate([np.zeros((q.shape[0], B) + tuple(q.shape[2:])), q.numpy()], axis=1)
        o, lse = self.oracle.phase1(qa, np.concatenate([k_anchor.numpy(), k.numpy()], axis=1),
                                    np.concatenate([v_anchor.numpy(), v.numpy()], axis=1), B)
        return torch.from_numpy(o[:, B:]), torch.from_numpy(lse[..., B:])

    def partial(self, q, block_size, k_ctx, v_ctx, k, v, k_cache, v_cache, cache_len):
        o, lse, kc, vc = self.oracle.phase2_partial(
            q.numpy(), self._np(k_ctx), self._np(v_ctx), self._np(k), self._np(v),
            self._np(k_cache), self._np(v_cache), cache_len)
        if k_cache is not None:
            k_cache.copy_(torch.from_numpy(kc))
            v_cache.copy_(torch.from_numpy(vc))
        return torch.from_numpy(o), torch.from_numpy(lse)

    def lse_merge(self, o_parts, lse_parts):
        # o_parts [S, b, T, H, d] -> the oracle's [S, b, H, T, d]
        o, lse = self.oracle.lse_merge(o_parts.numpy().transpose(0, 1, 3, 2, 4), lse_parts.numpy())
        return torch.from_numpy(o.transpose(0, 2, 1, 3)), torch.from_numpy(lse)


SHAPE = dict(b=1, hq=4, hkv=2, d=8, L=37, B=8, lq=3, T=2)


def _inputs():
    g = torch.Generator().manual_seed(3)
    s = SHAPE
    r = lambda *sh: torch.randn(*sh, generator=g, dtype=torch.float64)
    ctx = (r(s["b"], s["L"], s["hq"], s["d"]), r(s["b"], s["L"], s["hkv"], s["d"]),
           r(s["b"], s["L"], s["hkv"], s["d"]))
    qry = (r(s["b"], s["lq"], s["hq"], s["d"]), r(s["b"], s["lq"], s["hkv"], s["d"]),
           r(s["b"], s["lq"], s["hkv"], s["d"]))
    dec = [(r(s["b"], 1, s["hq"], s["d"]), r(s["b"], 1, s["hkv"], s["d"]),
            r(s["b"], 1, s["hkv"], s["d"])) for _ in range(s["T"])]
    return ctx, qry, dec


def _worker(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    from block_sparse_attention_phase_b200.sharded import ShardedStarAttention
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = SHAPE
        (q, k, v), qry, dec = _inputs()
        att = ShardedStarAttention(s["b"], s["hq"], s["hkv"], s["d"], s["L"], s["B"],
                                   s["lq"] + s["T"], backend=OracleBackend(), device="cpu",
                                   dtype=torch.float64)
        t0, t1 = att.token_range()
        o1, l1 = att.prefill(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1])
        res = {"range": [t0, t1],
               "o1": None if o1 is None else o1.tolist(), "l1": None if l1 is None else l1.tolist()}
        oq, lq = att.query(*qry)
        res["oq"] = None if oq is None else oq.tolist()
        res["lq"] = None if lq is None else lq.tolist()
        res["dec"] = []
        for t in range(s["T"]):
            od, ld = att.decode(*dec[t])
            res["dec"].append(None if od is None else [od.tolist(), ld.tolist()])
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_layer_matches_single_host(tmp_path, world):
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    import oracle
    s = SHAPE
    (q, k, v), (qq, kq, vq), dec = _inputs()
    ro, rl = oracle.phase1(q.numpy(), k.numpy(), v.numpy(), s["B"])
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    covered = []
    for r in res:
        t0, t1 = r["range"]
        covered += list(range(t0, t1))
        if t1 > t0:
            np.testing.assert_allclose(np.array(r["o1"]), ro[:, t0:t1], atol=1e-12)
            np.testing.assert_allclose(np.array(r["l1"]), rl[:, :, t0:t1], atol=1e-12)
    assert covered == list(range(s["L"]))  # every context token on exactly one rank
    host = res[world - 1]
    for r in res[:-1]:
        assert r["oq"] is None and all(d is None for d in r["dec"])
    rq, rql = oracle.phase2_query(qq.numpy(), kq.numpy(), vq.numpy(), k.numpy(), v.numpy())
    np.testing.assert_allclose(np.array(host["oq"]), rq, atol=1e-12)
    np.testing.assert_allclose(np.array(host["lq"]), rql, atol=1e-12)
    cap = s["lq"] + s["T"]
    kc = np.zeros((s["b"], cap, s["hkv"], s["d"]))
    vc = np.zeros_like(kc)
    kc[:, :s["lq"]], vc[:, :s["lq"]] = kq.numpy(), vq.numpy()
    for t in range(s["T"]):
        qd, kd, vd = (x.numpy() for x in dec[t])
        od, ld, kc, vc = oracle.phase2_decode(qd, kd, vd, k.numpy(), v.numpy(), kc, vc, s["lq"] + t)
        np.testing.assert_allclose(np.array(host["dec"][t][0]), od, atol=1e-12)
        np.testing.assert_allclose(np.array(host["dec"][t][1]), ld, atol=1e-12)


def _bench_worker(rank, world, port, out_dir):
    """bench.py's sharded step (the multi-GPU bench form) on gloo ranks with the
    oracle as compute: every phase runs, and the query rank's merged outputs equal
    the single-host oracle."""
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.Workload("bench-sharded", 1, 4, 2, 16, 70, 16, 3, 2, 0, 5)
        x = {k: t.double() for k, t in workloads.make_inputs(w, device="cpu").items()}
        step = bench.ShardedStep(w, x, "cpu", backend=OracleBackend(), dtype=torch.float64)
        step.run()
        step.run()  # a second pass over the same state (the bench's repeated steps)
        res = {"range": [step.t0, step.t1]}
        oq, lq = step.out["qry"]
        res["oq"] = None if oq is None else oq.tolist()
        res["dec"] = [None if od is None else od.tolist() for od, _ in step.out["dec"]]
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_bench_sharded_step_on_gloo_ranks(tmp_path):
    world = 3
    mp.start_processes(_bench_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    import oracle
    import workloads
    w = workloads.Workload("bench-sharded", 1, 4, 2, 16, 70, 16, 3, 2, 0, 5)
    x = {k: t.double().numpy() for k, t in workloads.make_inputs(w, device="cpu").items()}
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["range"] for r in res][0][0] == 0 and res[-1]["range"][1] == w.ctx_len
    host = res[-1]
    rq, _ = oracle.phase2_query(x["q_qry"], x["k_qry"], x["v_qry"], x["k_ctx"], x["v_ctx"])
    np.testing.assert_allclose(np.array(host["oq"]), rq, atol=1e-12)
    cap = w.cache_capacity
    kc = np.zeros((1, cap, w.num_kv_heads, w.head_dim))
    vc = np.zeros_like(kc)
    kc[:, :w.query_len], vc[:, :w.query_len] = x["k_qry"], x["v_qry"]
    for t in range(w.decode_steps):
        od, _, kc, vc = oracle.phase2_decode(x["q_dec"][t], x["k_dec"][t], x["v_dec"][t],
                                             x["k_ctx"], x["v_ctx"], kc, vc, w.query_len + t)
        np.testing.assert_allclose(np.array(host["dec"][t]), od, atol=1e-12)
    assert all(r["oq"] is None for r in res[:-1])


class _HostEvent:
    """Stand-in for torch.cuda.Event on the host: wall-clock stamps."""

    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, stream=None):
        import time
        self.t = time.perf_counter()

    def synchronize(self):
        pass

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


class _Float64Step:
    """bench.ShardedStep with the oracle as compute on float64 copies of the inputs."""

    def __new__(cls, w, x, device):
        import bench
        return bench._RealShardedStep(w, {k: t.double() for k, t in x.items()}, device,
                                      backend=OracleBackend(), dtype=torch.float64)


def _run_sharded_worker(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import contextlib
    import io
    import bench
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the CUDA calls of the timing harness, replaced by host stand-ins
        torch.cuda.Event = _HostEvent
        torch.cuda.synchronize = lambda *a, **k: None
        torch.cuda.set_device = lambda *a, **k: None
        torch.cuda.empty_cache = lambda *a, **k: None
        torch.cuda.current_device = lambda: 0
        torch.Tensor.pin_memory = lambda self: self
        bench._RealShardedStep = bench.ShardedStep
        bench.ShardedStep = _Float64Step
        w = workloads.Workload("bench-sharded", 1, 4, 2, 16, 70, 16, 3, 2, 0, 5)

        class Args:
            steps, warmup, no_e2e = 2, 3, False
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.run_sharded(Args, w, world, rank, rank, device=torch.device("cpu"))
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{rc}\n{buf.getvalue()}")
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_bench_run_sharded_on_gloo_ranks(tmp_path):
    """bench.py's multi-GPU mode end to end on 2 gloo ranks (timing calls on the
    host, the oracle as compute): warm-up, the timed steps with their collectives,
    the max over ranks, the end-to-end pass and rank 0's JSON line."""
    world = 2
    mp.start_processes(_run_sharded_worker, args=(world, _free_port(), str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    outs = [open(tmp_path / f"rank{r}.txt").read().split("\n", 1) for r in range(world)]
    assert all(rc == "0" for rc, _ in outs)
    assert outs[1][1].strip() == ""  # only rank 0 prints
    line = json.loads(outs[0][1].strip().splitlines()[-1])
    assert line["n_gpus"] == 2 and line["scaling"] == "strong" and line["steps"] == 2
    assert line["config"]["parallelism"] == "star-sharded2" and line["value"] > 0
    assert line["e2e"]["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] > 0
    for k in ("phase1", "query", "decode", "roofline", "clocks", "gpu_launches"):
        assert k in line
