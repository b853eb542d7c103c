"""GPU test of mc_qk_max_logit_static, the allocation-free S_max entry point.

Some callers cannot call cudaMalloc: their device memory is entirely held by
another allocator's reserved pool, or they must not risk the implicit device
synchronisation that cudaMalloc/cudaFree may cause.  For them the library
offers one entry point that takes no workspace and allocates nothing, using a
fixed 64 MiB device array built into the library instead.

This test calls that entry point directly through the C ABI (ctypes), twice in
a row per case (the second call must not be disturbed by what the first left
in the shared scratch), and checks its output against the workspace-taking
mc_qk_max_logit within the S_max tolerance of the other tests.  Output buffers
are created before the calls; the calls themselves allocate nothing.  This file
is named so that pytest collects it after every other test file.
"""
import ctypes

import numpy as np
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
from gpu_util import SMAX_TOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def call_static(lib, x, wq, wk, H, dh, causal, out):
    B, S, D = x.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.mc_qk_max_logit_static(x.data_ptr(), wq.data_ptr(), wk.data_ptr(), B, S, D, H, dh,
                                      int(causal), out.data_ptr(), ctypes.c_void_p(stream))


@pytest.mark.parametrize("B,S,D,H,dh,causal", [
    (2, 300, 64, 3, 64, True),       # ragged sequence, several tiles
    (1, 1024, 256, 4, 64, True),
    (2, 520, 128, 2, 128, False),    # unmasked
    (1, 4096, 4096, 32, 128, True),  # one batch of the full MHA layer: B*S*H*dh = 2^24, the limit
])
def test_static_entry_matches_workspace_entry_twice(B, S, D, H, dh, causal):
    lib = mc.load_library()
    X, Wq, Wk = wl.qk_inputs(B, S, D, H, dh, seed=21, hot_heads=(0,), w_std=0.05 if D >= 1024 else 0.2)
    x, wq, wk = X.to(DEV), Wq.to(DEV), Wk.to(DEV)
    want = mc.qk_max_logit(x, wq, wk, H, dh, causal=causal)
    outs = [torch.full((H,), float("nan"), dtype=torch.float32, device=DEV) for _ in range(2)]
    # a first call settles any one-time set-up (the scratch address lookup);
    # after it the two calls checked below must leave device memory as it is
    assert call_static(lib, x, wq, wk, H, dh, causal, outs[0]) == mc.MC_OK, mc.last_error()
    for out in outs:
        out.fill_(float("nan"))
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    for out in outs:
        rc = call_static(lib, x, wq, wk, H, dh, causal, out)
        assert rc == mc.MC_OK, mc.last_error()
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0
    w = want.cpu().double().numpy()
    # the small cases also against the fp64 oracle (Q, K in fp64, as defined)
    ref = (oracle.qk_max_logit(X.double().numpy(), Wq.double().numpy(), Wk.double().numpy(), H, dh, causal=causal)
           if B * S * D <= 2 ** 20 else None)
    for out in outs:
        got = out.cpu().double().numpy()
        assert np.all(np.isfinite(got))
        assert np.all(np.abs(got - w) <= SMAX_TOL * np.abs(w)), (got, w)
        if ref is not None:
            assert np.all(np.abs(got - ref) <= SMAX_TOL * np.abs(ref)), (got, ref)


def test_static_entry_rejects_sizes_beyond_its_scratch():
    lib = mc.load_library()
    B, S, D, H, dh = 2, 4096, 64, 32, 128  # B*S*H*dh = 2^25 > 2^24
    x = torch.zeros((B, S, D), dtype=torch.bfloat16, device=DEV)
    wq = torch.zeros((H * dh, D), dtype=torch.bfloat16, device=DEV)
    out = torch.full((H,), 7.0, dtype=torch.float32, device=DEV)
    rc = call_static(lib, x, wq, wq.clone(), H, dh, True, out)
    assert rc == mc.MC_ERR_NOSPC
    assert "static scratch" in mc.last_error()
    assert torch.all(out == 7.0)  # nothing was enqueued
    # more heads than the scratch's head table, with few elements
    B, S, D, H, dh = 1, 1, 8, 4104, 8
    x = torch.zeros((B, S, D), dtype=torch.bfloat16, device=DEV)
    wq = torch.zeros((H * dh, D), dtype=torch.bfloat16, device=DEV)
    out = torch.full((H,), 7.0, dtype=torch.float32, device=DEV)
    rc = call_static(lib, x, wq, wq.clone(), H, dh, True, out)
    assert rc == mc.MC_ERR_NOSPC
    assert "heads" in mc.last_error()
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
