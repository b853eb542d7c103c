"""A Muon-type call enqueues its work and returns without waiting for the
device: every piece's parameter tables go up in one copy at the start of the
call, through a page-locked staging buffer of its own ("MuonClip: speed, then
stability", §07: the optimizer step is one stage of a training step, so the
host must be free to queue the next stage behind it)."""
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
    """Twenty calls behind a busy stream: each takes a staging buffer of its
    own, so none waits for an earlier call's table copy."""
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


def test_thirty_third_queued_copy_waits_for_the_oldest(hp):
    """The staging pool holds 32 buffers: behind a stream that stays busy for
    a second, 32 calls queue at once and the 33rd waits (on the host) until
    the first call's table copy has run, i.e. until the busy kernel ends."""
    Ws = [torch.randn((128, 192), device=DEV).to(torch.bfloat16) * 0.02]
    Gs = [torch.randn((128, 192), device=DEV).to(torch.bfloat16) * 1e-3]
    Ms = [torch.zeros((128, 192), device=DEV)]
    for _ in range(40):   # the pool reaches its 32 buffers
        mc.muon_step(Ws, Gs, Ms, **hp)
    torch.cuda.synchronize()
    _busy_stream(1.0)
    t0 = time.perf_counter()
    for _ in range(32):
        mc.muon_step(Ws, Gs, Ms, **hp)
    queued_s = time.perf_counter() - t0
    mc.muon_step(Ws, Gs, Ms, **hp)
    waited_s = time.perf_counter() - t0 - queued_s
    torch.cuda.synchronize()
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    assert queued_s < 0.5, queued_s
    assert waited_s > 0.2, waited_s
