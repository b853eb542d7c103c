"""GPU parity of the multi-head latent attention side of QK-Clip (through the
C ABI) against the fp64 oracle: S_max with a content part and a rotary part
whose key is shared by every head, and the slice-map rescale -- content query
and key by gamma^(1/2), rotary query by gamma, shared rotary key untouched
("MuonClip: speed, then stability" §06; "Muon and MuonClip: orthogonalised
updates for LLM training", "MuonClip: QK-clip, per head, adapted to MLA")."""
import numpy as np
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
from gpu_util import GAMMA_TOL, SMAX_TOL, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ("W_qC", "W_kC", "W_qR", "W_kR")


def rel(a, b):
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-30)


def gpu_mla_smax(X, w, H, dc, dr, causal=True):
    d = {k: v.to(DEV) for k, v in w.items()}
    s = mc.mla_max_logit(X.to(DEV), d["W_qC"], d["W_kC"], d["W_qR"], d["W_kR"], H, dc, dr, causal=causal)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    return s.cpu().double().numpy()


def w64(w):
    return {k: to64(v) for k, v in w.items()}


@pytest.mark.parametrize("B,S,D,H,dc,dr", [(2, 300, 64, 3, 64, 32), (1, 129, 40, 2, 128, 64),
                                           (3, 700, 96, 4, 64, 8), (1, 1, 16, 1, 64, 16),
                                           (2, 520, 256, 2, 128, 72), (1, 300, 64, 2, 256, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_mla_smax_small(B, S, D, H, dc, dr, causal):
    X, w = wl.mla_inputs(B, S, D, H, dc, dr, seed=13, w_std=0.2)
    got = gpu_mla_smax(X, w, H, dc, dr, causal)
    ref = oracle.mla_max_logit(to64(X), w64(w), H, dc, dr, causal=causal)
    refb = oracle.mla_max_logit(to64(X), w64(w), H, dc, dr, causal=causal, qk_bf16=True)
    assert np.all(rel(got, ref) <= SMAX_TOL), (got, ref)
    assert np.all(rel(got, refb) <= 2e-3), (got, refb)


def test_mla_rotary_part_counts_and_is_shared():
    """Content weights zero: S_max comes from the rotary part alone, where
    every head meets the same shared key.  Rotary weights zero: it comes from
    the content part alone."""
    B, S, D, H, dc, dr = 1, 260, 64, 3, 64, 64
    X, w = wl.mla_inputs(B, S, D, H, dc, dr, seed=14, w_std=0.3)
    for zero in (("W_qC", "W_kC"), ("W_qR", "W_kR")):
        v = dict(w)
        for k in zero:
            v[k] = torch.zeros_like(w[k])
        got = gpu_mla_smax(X, v, H, dc, dr)
        ref = oracle.mla_max_logit(to64(X), w64(v), H, dc, dr)
        assert np.all(rel(got, ref) <= SMAX_TOL), (zero, got, ref)


def device_factor(smax: float, tau: float, e: float) -> np.float32:
    """gamma^e as the device forms it: an fp32 division and, for e = 1/2, an
    fp32 square root (both correctly rounded, here as on the device)."""
    g = np.float32(tau) / np.float32(smax)
    return np.sqrt(g) if e == 0.5 else g


def _check_scaled(got, orig, factor, dtype):
    """The device's arithmetic exactly: fp32 product, then nearest-even into
    the weight's dtype."""
    want = (orig.to(torch.float32) * torch.tensor(float(factor), dtype=torch.float32)).to(dtype)
    assert torch.equal(got, want)


def test_mla_clip_slice_map_against_oracle():
    H, dc, dr, D = 4, 64, 32, 96
    _, w = wl.mla_inputs(1, 8, D, H, dc, dr, seed=15, w_std=0.5)
    smax = torch.tensor([400.0, 80.0, 100.0, 250.0], dtype=torch.float32)
    d = {k: v.to(DEV) for k, v in w.items()}
    gamma, mask = mc.qk_clip_slices(mc.mla_slices(d["W_qC"], d["W_kC"], d["W_qR"], H, dc, dr), smax.to(DEV), H,
                                    tau=100.0)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    out, og, om = oracle.qk_clip_slices(w64(w), oracle.mla_slices(H, dc, dr), smax.double().numpy(), 100.0)
    mask = mask.cpu().numpy()
    gamma = gamma.cpu().double().numpy()
    assert list(mask) == list(om) == [1, 0, 0, 1]
    assert np.all(np.abs(gamma - og) <= GAMMA_TOL * og)
    assert gamma[0] == pytest.approx(0.25, abs=1e-7)
    res = {k: v.cpu() for k, v in d.items()}
    assert torch.equal(res["W_kR"], w["W_kR"])          # the shared rotary key is never written
    for h in range(H):
        for name, width, e in (("W_qC", dc, 0.5), ("W_kC", dc, 0.5), ("W_qR", dr, 1.0)):
            rows = slice(h * width, (h + 1) * width)
            if om[h]:
                _check_scaled(res[name][rows], w[name][rows], device_factor(float(smax[h]), 100.0, e), torch.bfloat16)
                assert np.allclose(to64(res[name][rows]), out[name][rows], rtol=2 ** -8, atol=0)
            else:
                assert torch.equal(res[name][rows], w[name][rows])
    # the worked example: 400 against tau 100 halves content rows, quarters rotary query rows
    assert np.allclose(to64(res["W_qC"][:dc]), to64(w["W_qC"][:dc]) * 0.5, rtol=0, atol=0)
    assert np.allclose(to64(res["W_qR"][:dr]), to64(w["W_qR"][:dr]) * 0.25, rtol=0, atol=0)


def test_fused_projection_layout_and_fp32_slices():
    """Slices inside fused matrices: a query projection whose head blocks are
    [content | rotary] rows, and a key/value projection whose head blocks are
    [content key | value] rows (values are not in the map and stay untouched);
    plus fp32 weights and a row length that is not a multiple of 8."""
    H, dc, dr, dv, D = 3, 64, 32, 48, 37
    rng = np.random.default_rng(16)
    qf = wl.to_dtype(rng.normal(0, 0.5, (H * (dc + dr), D)), torch.float32)
    kvf = wl.to_dtype(rng.normal(0, 0.5, (H * (dc + dv), D)), torch.bfloat16)
    smax = torch.tensor([150.0, 1000.0, 99.0], dtype=torch.float32)
    q, kv = qf.to(DEV), kvf.to(DEV)
    sl, osl = [], []
    for h in range(H):
        qb, kb = h * (dc + dr), h * (dc + dv)
        for (t, nm, r0, r1, e) in ((q, "q", qb, qb + dc, 0.5), (q, "q", qb + dc, qb + dc + dr, 1.0),
                                   (kv, "kv", kb, kb + dc, 0.5)):
            sl.append((t, h, r0, r1, e))
            osl.append((nm, h, r0, r1, e))
    gamma, mask = mc.qk_clip_slices(sl, smax.to(DEV), H, tau=100.0)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    out, og, om = oracle.qk_clip_slices({"q": to64(qf), "kv": to64(kvf)}, osl, smax.double().numpy(), 100.0)
    assert list(mask.cpu().numpy()) == list(om) == [1, 1, 0]
    qr, kvr = q.cpu(), kv.cpu()
    for h in range(H):
        qb, kb = h * (dc + dr), h * (dc + dv)
        vrows = slice(kb + dc, kb + dc + dv)
        assert torch.equal(kvr[vrows], kvf[vrows])       # values: not in the map
        if om[h]:
            f_half, f_one = device_factor(float(smax[h]), 100.0, 0.5), device_factor(float(smax[h]), 100.0, 1.0)
            _check_scaled(qr[qb:qb + dc], qf[qb:qb + dc], f_half, torch.float32)
            _check_scaled(qr[qb + dc:qb + dc + dr], qf[qb + dc:qb + dc + dr], f_one, torch.float32)
            _check_scaled(kvr[kb:kb + dc], kvf[kb:kb + dc], f_half, torch.bfloat16)
            assert np.allclose(to64(qr[qb:qb + dc + dr]), out["q"][qb:qb + dc + dr], rtol=1e-6, atol=0)
        else:
            assert torch.equal(qr[qb:qb + dc + dr], qf[qb:qb + dc + dr])
            assert torch.equal(kvr[kb:kb + dc], kvf[kb:kb + dc])


def test_many_slices_span_several_launches():
    """More slices than one launch's table holds (48): 40 heads x 3 slices."""
    H, dc, dr, D = 40, 64, 16, 64
    _, w = wl.mla_inputs(1, 4, D, H, dc, dr, seed=17, w_std=0.5)
    smax = torch.linspace(50.0, 400.0, H, dtype=torch.float32)
    d = {k: v.to(DEV) for k, v in w.items()}
    mc.qk_clip_slices(mc.mla_slices(d["W_qC"], d["W_kC"], d["W_qR"], H, dc, dr), smax.to(DEV), H, tau=100.0)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    out, og, om = oracle.qk_clip_slices(w64(w), oracle.mla_slices(H, dc, dr), smax.double().numpy(), 100.0)
    for k in NAMES:
        got = to64(d[k].cpu())
        assert np.allclose(got, out[k], rtol=2 ** -8, atol=0), k
        if k != "W_kR":
            for h in range(H):
                width = dc if k != "W_qR" else dr
                if not om[h]:
                    assert np.array_equal(got[h * width:(h + 1) * width], to64(w[k])[h * width:(h + 1) * width])
    assert torch.equal(d["W_kR"].cpu(), w["W_kR"])


@pytest.fixture(scope="module")
def mla_layer():
    X, w = wl.mla_layer_inputs()
    c = wl.MLA
    ref = oracle.mla_max_logit(to64(X), w64(w), c["H"], c["dc"], c["dr"], causal=True)
    return X, w, ref


def test_mla_layer_smax_clip_and_recheck(mla_layer):
    """Full-size MLA layer (B 4, S 4096, D 4096, H 32, dc 128, dr 64): S_max of
    every head against the oracle, the clipped set, and S_max back at tau after
    the slice-map clip (both score parts scale by gamma)."""
    X, w, ref = mla_layer
    c = wl.MLA
    H, dc, dr = c["H"], c["dc"], c["dr"]
    x = X.to(DEV)
    d = {k: v.to(DEV) for k, v in w.items()}
    smax = mc.mla_max_logit(x, d["W_qC"], d["W_kC"], d["W_qR"], d["W_kR"], H, dc, dr)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    got = smax.cpu().double().numpy()
    assert np.all(rel(got, ref) <= SMAX_TOL), np.max(rel(got, ref))
    gamma, mask = mc.qk_clip_slices(mc.mla_slices(d["W_qC"], d["W_kC"], d["W_qR"], H, dc, dr), smax, H,
                                    tau=wl.QK_TAU)
    _, og, om = oracle.qk_clip_slices(w64(w), oracle.mla_slices(H, dc, dr), ref, wl.QK_TAU)
    mask = mask.cpu().numpy()
    assert sorted(np.nonzero(mask)[0].tolist()) == sorted(np.nonzero(om)[0].tolist()) == list(c["hot_heads"])
    assert np.all(np.abs(gamma.cpu().double().numpy() - og) <= GAMMA_TOL * og)
    assert torch.equal(d["W_kR"].cpu(), w["W_kR"])
    after = mc.mla_max_logit(x, d["W_qC"], d["W_kC"], d["W_qR"], d["W_kR"], H, dc, dr).cpu().double().numpy()
    for h in c["hot_heads"]:
        assert wl.QK_TAU * (1 - 2 ** -6) <= after[h] <= wl.QK_TAU * (1 + 2 ** -7)
    for h in range(H):
        if not mask[h]:
            assert after[h] == got[h]
    del d, x
    mc.release_workspaces()
    torch.cuda.empty_cache()
