"""Multi-process CPU tests (gloo) of the ownership-sharded data-parallel step
and the global S_max.

Each rank holds replicated weights and its own gradients; the sharded step
(reduce-scatter, owner-local Muon step, all-gather) must leave every replica
equal to the single-process step on the summed gradients, and each momentum
on its owner equal to the single-process momentum.  The owner-local Muon step
here is the fp64 oracle (the product's is the CUDA step, tested on the GPU),
so these tests check the plumbing: the plan, the layout, the collectives.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import sharded
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl

SHAPES = [(64, 96), (96, 64), (128, 128), (32, 200), (200, 32), (48, 48), (80, 40), (16, 16), (40, 80)]
HP = dict(wl.HPARAMS)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weights0():
    rng = wl.rng_for(90, 0)
    return [wl.to_dtype(rng.normal(0, 0.02, s), torch.bfloat16) for s in SHAPES]


def _grads(rank):
    # multiples of 2^-12 with small integer numerators: sums over ranks are
    # exact in fp32, whatever order the collective adds them in
    rng = wl.rng_for(91, rank)
    return [torch.from_numpy(np.round(rng.normal(0, 64, s)) / 4096.0).to(torch.float32) for s in SHAPES]


def oracle_local_step(Ws, Gs, Ms, **hp):
    for W, G, M in zip(Ws, Gs, Ms):
        Wn, Mn, _, _ = oracle.muon_step(W.double().numpy(), G.double().numpy(), M.double().numpy(), **hp)
        W.copy_(torch.from_numpy(Wn).to(W.dtype))
        M.copy_(torch.from_numpy(Mn).to(M.dtype))


def _worker(rank, world, port, outdir, steps):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sm = sharded.ShardedMuon(SHAPES, w_dtype=torch.bfloat16, g_dtype=torch.float32, device="cpu",
                                 local_step=oracle_local_step)
        for w, w0 in zip(sm.weights, _weights0()):
            w.copy_(w0)
        for step in range(steps):
            for g, gl in zip(sm.grads, _grads(rank + 17 * step)):
                g.copy_(gl)
            sm.step(**HP)
        out = {f"w{i}": w.float().numpy() for i, w in enumerate(sm.weights)}
        out.update({f"m{i}": m.numpy() for i, m in enumerate(sm.moms) if m is not None})
        out["owner"] = np.array(sm.owner)

        # global S_max: each rank's batch differs; after the all-reduce every
        # rank holds the max over the union of the batches
        H, dh, D = 3, 8, 16
        rng = wl.rng_for(92, 0)
        Wq, Wk = rng.normal(0, 0.5, (H * dh, D)), rng.normal(0, 0.5, (H * dh, D))
        X = wl.rng_for(93, rank).normal(0, 1, (2, 12, D))
        smax = torch.from_numpy(oracle.qk_max_logit(X, Wq, Wk, H, dh)).float()
        sharded.global_smax(smax)
        out["smax"] = smax.numpy()
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), **out)
    finally:
        dist.destroy_process_group()


def _reference(world, steps):
    Ws = [w.double().numpy() for w in _weights0()]
    Ms = [np.zeros(s) for s in SHAPES]
    for step in range(steps):
        G = [sum(_grads(r + 17 * step)[i].double().numpy() for r in range(world)) for i in range(len(SHAPES))]
        for i in range(len(SHAPES)):
            Wn, Mn, _, _ = oracle.muon_step(Ws[i], G[i], Ms[i], **HP)
            Ws[i] = torch.from_numpy(Wn).to(torch.bfloat16).double().numpy()
            Ms[i] = torch.from_numpy(Mn).to(torch.float32).double().numpy()
    return Ws, Ms


@pytest.mark.parametrize("world,steps", [(2, 2), (3, 1), (4, 1)])
def test_sharded_step_equals_single_process_step(tmp_path, world, steps):
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), steps), nprocs=world,
                       start_method="spawn", join=True)
    res = [dict(np.load(tmp_path / f"rank{r}.npz")) for r in range(world)]
    Wref, Mref = _reference(world, steps)
    owner = res[0]["owner"]
    assert all(np.array_equal(r["owner"], owner) for r in res)       # one plan on every rank
    assert sorted(set(owner.tolist())) == list(range(world))           # every rank owns something
    for i in range(len(SHAPES)):
        for r in range(world):
            assert np.array_equal(res[r][f"w{i}"], res[0][f"w{i}"])    # replicas agree bit for bit
        assert np.array_equal(res[0][f"w{i}"].astype(np.float64), Wref[i]), i
        o = int(owner[i])
        assert np.array_equal(res[o][f"m{i}"].astype(np.float64), Mref[i]), i
        for r in range(world):
            if r != o:
                assert f"m{i}" not in res[r]                            # momentum only on the owner
    # global S_max: the max over every rank's batch
    H, dh, D = 3, 8, 16
    rng = wl.rng_for(92, 0)
    Wq, Wk = rng.normal(0, 0.5, (H * dh, D)), rng.normal(0, 0.5, (H * dh, D))
    Xall = np.concatenate([wl.rng_for(93, r).normal(0, 1, (2, 12, D)) for r in range(world)])
    want = oracle.qk_max_logit(Xall, Wq, Wk, H, dh).astype(np.float32)
    for r in range(world):
        assert np.array_equal(res[r]["smax"], want)


def test_single_process_layout_without_a_process_group():
    """world 1 (no process group): every matrix is owned locally, the views
    tile the flat buffers without overlap and at 256-byte alignment."""
    sm = sharded.ShardedMuon(SHAPES, w_dtype=torch.bfloat16, g_dtype=torch.bfloat16, device="cpu",
                             local_step=oracle_local_step)
    assert sm.world == 1 and sm.owned == list(range(len(SHAPES)))
    spans = []
    for w, g in zip(sm.weights, sm.grads):
        assert (w.data_ptr() - sm.w_flat.data_ptr()) % 256 == 0
        assert (g.data_ptr() - sm.g_flat.data_ptr()) % 256 == 0
        spans.append((w.data_ptr(), w.data_ptr() + w.numel() * 2))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    for w, w0 in zip(sm.weights, _weights0()):
        w.copy_(w0)
    for g, gl in zip(sm.grads, _grads(0)):
        g.copy_(gl.to(torch.bfloat16))
    sm.step(**HP)
    for i, (w0, g) in enumerate(zip(_weights0(), _grads(0))):
        Wn, _, _, _ = oracle.muon_step(w0.double().numpy(), g.to(torch.bfloat16).double().numpy(),
                                       np.zeros(SHAPES[i]), **HP)
        assert torch.equal(sm.weights[i], torch.from_numpy(Wn).to(torch.bfloat16))


def test_shard_plan_properties():
    """Every matrix gets one owner, the loads add up, the plan is the
    longest-processing-time rule (within 4/3 - 1/(3P) of the best makespan,
    checked against brute force on small cases) and is deterministic."""
    def cost(s, k=5):
        m, n = min(s), max(s)
        return k * (4.0 * m * m * n + 2.0 * m ** 3)

    for world in (1, 2, 3, 5):
        owner, load = mc.shard_plan(SHAPES, world)
        assert owner == mc.shard_plan(SHAPES, world)[0]
        assert all(0 <= o < world for o in owner)
        for r in range(world):
            assert load[r] == pytest.approx(sum(cost(s) for s, o in zip(SHAPES, owner) if o == r), rel=1e-12)
        # brute-force best makespan over every assignment (9 matrices)
        if world <= 3:
            costs = [cost(s) for s in SHAPES]
            best = float("inf")
            for code in range(world ** len(costs)):
                loads = [0.0] * world
                c = code
                for x in costs:
                    loads[c % world] += x
                    c //= world
                best = min(best, max(loads))
            assert max(load) <= (4 / 3 - 1 / (3 * world)) * best * (1 + 1e-12)
    # the 7B-shaped set splits evenly over 2, 4 and 8 ranks
    for world in (2, 4, 8):
        _, load = mc.shard_plan(wl.cfg2_shapes(), world)
        assert max(load) == pytest.approx(sum(load) / world, rel=1e-12)


def test_shard_plan_argument_errors():
    with pytest.raises(mc.MuonClipError):
        mc.shard_plan([(0, 4)], 2)
    with pytest.raises(mc.MuonClipError):
        mc.shard_plan([(4, 4)], 0)
    with pytest.raises(mc.MuonClipError):
        mc.shard_plan([(4, 4)], 2, ns_steps=0)
    assert mc.shard_plan([], 3) == ([], [0.0, 0.0, 0.0])
