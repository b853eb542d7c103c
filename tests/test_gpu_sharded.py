"""GPU checks behind the ownership-sharded step (one GPU): a matrix's result
does not depend on which other matrices share its mc_muon_step call, so the
owner-local step of a shard equals the single-GPU step bit for bit; and the
sharded step at world size 1 is exactly the plain step."""
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
from matrix_orthogonalising_optimizer_step_b200 import sharded
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
SHAPES = [(256, 768), (768, 256), (512, 512), (512, 512), (300, 520), (520, 300), (64, 1000), (256, 768)]


def _run(mats, hp):
    Ws = [W.to(DEV) for W, _, _ in mats]
    Gs = [G.to(DEV) for _, G, _ in mats]
    Ms = [M.to(DEV) for _, _, M in mats]
    Us = [torch.empty(W.shape, dtype=torch.float32, device=DEV) for W in Ws]
    mc.muon_step(Ws, Gs, Ms, update_outs=Us, **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    return [W.cpu() for W in Ws], [M.cpu() for M in Ms], [U.cpu() for U in Us]


def test_results_do_not_depend_on_the_rest_of_the_batch(hp):
    mats = [wl.generic_matrix(r, c, seed=60 + i) for i, (r, c) in enumerate(SHAPES)]
    full = _run(mats, hp)
    for subset in ([1, 3, 4, 6], [0], [2, 7, 5]):
        part = _run([mats[i] for i in subset], hp)
        for k, i in enumerate(subset):
            for a, b in zip(part, full):
                assert torch.equal(a[k], b[i]), (subset, i)


def test_sharded_world_one_is_the_plain_step(hp):
    mats = [wl.generic_matrix(r, c, seed=70 + i) for i, (r, c) in enumerate(SHAPES)]
    plain_W, plain_M, _ = _run(mats, hp)
    sm = sharded.ShardedMuon(SHAPES, w_dtype=torch.bfloat16, g_dtype=torch.bfloat16, device=DEV)
    assert sm.world == 1
    for i, (W, G, M) in enumerate(mats):
        sm.weights[i].copy_(W.to(DEV))
        sm.grads[i].copy_(G.to(DEV))
        sm.moms[i].copy_(M.to(DEV))
    sm.step(**hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    for i in range(len(SHAPES)):
        assert torch.equal(sm.weights[i].cpu(), plain_W[i])
        assert torch.equal(sm.moms[i].cpu(), plain_M[i])
