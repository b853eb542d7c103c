"""A Muon-type call enqueues its work and returns without waiting for the
device: every piece's parameter tables go up at the start of the call inside
the parameters of a small copy kernel, so no host buffer has to outlive the
call ("MuonClip: speed, then stability", §07: the optimizer step is one stage
of a training step, so the host must be free to queue the next stage behind
it).  For the same reason a call can be captured into a CUDA graph and
replayed."""
import time

import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _busy_stream(seconds):
    # keep the stream busy for about `seconds` (cycles at ~2 GHz)
    torch.cuda._sleep(int(seconds * 2e9))


def test_eight_piece_call_returns_while_the_device_is_busy(hp):
    # 4096 x 131072 = 2^29 elements: one matrix per piece, so eight entries
    # make eight pieces (they share one W, G, M: the pieces run in order)
    r, c = 4096, 131072
    g = torch.Generator(device=DEV)
    g.manual_seed(7)
    W = (torch.randn((r, c), device=DEV, generator=g) * 0.02).to(torch.bfloat16)
    G = (torch.randn((r, c), device=DEV, generator=g) * 1e-3).to(torch.bfloat16)
    M = torch.zeros((r, c), device=DEV)
    Ws, Gs, Ms = [W] * 8, [G] * 8, [M] * 8
    mc.muon_step(Ws, Gs, Ms, **hp)          # workspace and first-use set-up
    torch.cuda.synchronize()
    mc.profile_begin()
    _busy_stream(1.0)
    t0 = time.perf_counter()
    mc.muon_step(Ws, Gs, Ms, **hp)
    host_s = time.perf_counter() - t0
    busy = not torch.cuda.current_stream().query()
    torch.cuda.synchronize()
    k = mc.profile_end()
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    assert busy
    assert host_s < 0.3, host_s
    assert k["momentum"]["launches"] == 8          # eight pieces ...
    assert k["table_upload"]["launches"] == 1      # ... one table copy
    del W, G, M, Ws, Gs, Ms
    mc.release_workspaces()
    torch.cuda.empty_cache()


def test_many_calls_queue_without_waiting(hp):
    """Twenty calls behind a stream that stays busy for a second: none of them
    waits on the host for an earlier call's table copy."""
    Ws = [torch.randn((256, 384), device=DEV).to(torch.bfloat16) * 0.02 for _ in range(3)]
    Gs = [torch.randn((256, 384), device=DEV).to(torch.bfloat16) * 1e-3 for _ in range(3)]
    Ms = [torch.zeros((256, 384), device=DEV) for _ in range(3)]
    mc.muon_step(Ws, Gs, Ms, **hp)
    torch.cuda.synchronize()
    _busy_stream(1.0)
    t0 = time.perf_counter()
    for _ in range(20):
        mc.muon_step(Ws, Gs, Ms, **hp)
    host_s = time.perf_counter() - t0
    busy = not torch.cuda.current_stream().query()
    torch.cuda.synchronize()
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    assert busy
    assert host_s < 0.5, host_s


def _workspace_for(Ws, Gs, Ms, hp):
    import ctypes
    lib = mc.load_library()
    arr, n = mc.make_params(Ws, Gs, Ms, None)
    need = int(lib.mc_muon_workspace_size(arr, n, ctypes.byref(mc.make_hparams(**hp))))
    return torch.empty(need, dtype=torch.uint8, device=DEV)


def test_captured_step_replays_like_direct_calls(hp):
    """A step captured into a CUDA graph (with a workspace of its own) and
    replayed twice gives, bit for bit, what two direct calls give: the tables
    travel inside the captured launches, so a replay re-reads nothing from the
    host."""
    g = torch.Generator(device=DEV)
    g.manual_seed(11)
    shapes = [(256, 768), (768, 256), (512, 512), (300, 520)]
    W0 = [(torch.randn(sh, device=DEV, generator=g) * 0.02).to(torch.bfloat16) for sh in shapes]
    Gs = [(torch.randn(sh, device=DEV, generator=g) * 1e-3).to(torch.bfloat16) for sh in shapes]
    M0 = [torch.randn(sh, device=DEV, generator=g) * 1e-4 for sh in shapes]
    WE, ME = [w.clone() for w in W0], [m.clone() for m in M0]
    WC, MC = [w.clone() for w in W0], [m.clone() for m in M0]
    wsE, wsC = _workspace_for(WE, Gs, ME, hp), _workspace_for(WC, Gs, MC, hp)
    for _ in range(2):
        mc.muon_step(WE, Gs, ME, workspace=wsE, **hp)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        mc.muon_step(WC, Gs, MC, workspace=wsC, **hp)
    torch.cuda.synchronize()
    # capturing ran nothing
    for w, w0 in zip(WC, W0):
        assert torch.equal(w, w0)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    for a, b in zip(WC + MC, WE + ME):
        assert torch.equal(a, b)
    del graph


def test_device_learning_rate_under_a_captured_graph(hp):
    """With hparams.lr_wd pointing at a device (lr, wd) pair, the kernels read
    the learning rate when they run: one captured step replayed under a
    changing schedule matches direct calls made with those values on the host,
    bit for bit (GEMM path, thin path and NorMuon's row pass)."""
    g = torch.Generator(device=DEV)
    g.manual_seed(12)
    shapes = [(256, 768), (768, 256), (16, 300), (300, 24)]
    W0 = [(torch.randn(sh, device=DEV, generator=g) * 0.02).to(torch.bfloat16) for sh in shapes]
    Gs = [(torch.randn(sh, device=DEV, generator=g) * 1e-3).to(torch.bfloat16) for sh in shapes]
    M0 = [torch.randn(sh, device=DEV, generator=g) * 1e-4 for sh in shapes]
    base = {k: v for k, v in hp.items() if k not in ("lr", "wd")}
    lr_wd = torch.tensor([0.02, 0.1], device=DEV, dtype=torch.float32)
    dev_hp = mc.make_hparams(lr_wd=lr_wd, **base)
    WE, ME = [w.clone() for w in W0], [m.clone() for m in M0]
    WC, MC = [w.clone() for w in W0], [m.clone() for m in M0]
    wsE, wsC = _workspace_for(WE, Gs, ME, hp), _workspace_for(WC, Gs, MC, hp)
    mc.muon_step([W0[0].clone()], Gs[:1], [M0[0].clone()], **hp)   # set-up call, on copies
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        mc.muon_step(WC, Gs, MC, workspace=wsC, hparams=dev_hp)
    torch.cuda.synchronize()
    for lr in (0.02, 0.01, 0.003):
        lr_wd.copy_(torch.tensor([lr, 0.1], device=DEV))
        graph.replay()
        mc.muon_step(WE, Gs, ME, workspace=wsE, hparams=mc.make_hparams(lr=lr, wd=0.1, **base))
        torch.cuda.synchronize()
        for a, b in zip(WC + MC, WE + ME):
            assert torch.equal(a, b), lr
    del graph
    # NorMuon: the device pair against the host values, directly
    vs0 = [torch.rand(r, device=DEV, generator=g) * 1e-6 for r, _ in shapes]
    W1, M1, V1 = [w.clone() for w in W0], [m.clone() for m in M0], [v.clone() for v in vs0]
    W2, M2, V2 = [w.clone() for w in W0], [m.clone() for m in M0], [v.clone() for v in vs0]
    lr_wd.copy_(torch.tensor([0.007, 0.05], device=DEV))
    mc.normuon_step(W1, Gs, M1, V1, hparams=mc.make_hparams(lr_wd=lr_wd, **base))
    mc.normuon_step(W2, Gs, M2, V2, hparams=mc.make_hparams(lr=0.007, wd=0.05, **base))
    torch.cuda.synchronize()
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    for a, b in zip(W1 + M1 + V1, W2 + M2 + V2):
        assert torch.equal(a, b)
