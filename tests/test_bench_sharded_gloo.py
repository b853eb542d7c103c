"""The multi-GPU bench loop (bench.run_sharded: the ownership-sharded step,
each rank's own QK batch, the global S_max, the clip) run as two gloo ranks
on the CPU.  The rank's GPU work is stood in for by the fp64 oracle (the
product path is the CUDA step, tested on the GPU); what is checked here is the
loop's plumbing and the JSON line it prints on rank 0."""
import json
import os
import socket
import time

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl

SHAPES = [(64, 96), (96, 64), (48, 48), (32, 80)]
QK = dict(B=1, S=24, D=16, H=2, dh=8, hot_heads=(1,), hot_scale=6.0)


class CpuCtx:
    def __init__(self, rank, world):
        self.device, self.rank, self.world = torch.device("cpu"), rank, world

    def local_step(self, Ws, Gs, Ms, **hp):
        for W, G, M in zip(Ws, Gs, Ms):
            Wn, Mn, _, _ = oracle.muon_step(W.double().numpy(), G.double().numpy(), M.double().numpy(), **hp)
            W.copy_(torch.from_numpy(Wn).to(W.dtype))
            M.copy_(torch.from_numpy(Mn).to(M.dtype))

    def qk_max_logit(self, x, wq, wk, H, dh, smax):
        s = oracle.qk_max_logit(x.double().numpy(), wq.double().numpy(), wk.double().numpy(), H, dh)
        smax.copy_(torch.from_numpy(s).float())

    def qk_clip(self, wq, wk, smax, H, dh, tau, alpha, gamma, mask):
        q, k, g, m = oracle.qk_clip(wq.double().numpy(), wk.double().numpy(), smax.double().numpy(), tau, alpha,
                                    H, dh)
        wq.copy_(torch.from_numpy(q).to(wq.dtype))
        wk.copy_(torch.from_numpy(k).to(wk.dtype))
        gamma.copy_(torch.from_numpy(np.asarray(g)).float())
        mask.copy_(torch.from_numpy(np.asarray(m)).int())

    def sync(self):
        pass

    def start(self):
        return time.perf_counter()

    def stop(self, t0):
        return (time.perf_counter() - t0) * 1e3

    def profile_begin(self):
        pass

    def profile_end(self):
        return {}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def max_over_ranks(v):
            t = torch.tensor([v], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())

        args = bench.parse_args(["--steps", "2", "--warmup", "3"])
        out = bench.run_sharded(args, CpuCtx(rank, world), SHAPES, QK, dict(wl.HPARAMS), dist.barrier,
                                max_over_ranks)
        if rank == 0:
            with open(os.path.join(outdir, "line.json"), "w") as f:
                f.write(json.dumps(out))
        else:
            assert out is None
    finally:
        dist.destroy_process_group()


def test_bench_sharded_loop_prints_a_contract_line(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    line = json.loads(open(tmp_path / "line.json").read())
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches"):
        assert key in line, key
    assert line["n_gpus"] == world and line["steps"] == 2 and line["warmup"] == 3
    assert line["scaling"] == "strong" and line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["mode"] == "sharded" and line["config"]["parallelism"].startswith("dp2")
    assert line["config"]["matrices"] == len(SHAPES)
    want = bench.ns_dense_flops(SHAPES, wl.HPARAMS["ns_steps"]) + world * bench.qk_flops(
        QK["B"], QK["S"], QK["D"], QK["H"], QK["dh"])
    assert line["config"]["flops_per_step"] == want
