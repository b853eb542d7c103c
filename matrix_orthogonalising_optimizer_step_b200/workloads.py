"""Seeded synthetic workloads for the MuonClip step.

This module only *draws inputs*: shapes, seeded random matrices, spectra and
dtype rounding.  It holds none of the optimizer's arithmetic, so that both the
CUDA path and the fp64 oracle can be fed the same bytes from here without
sharing any of the method.

Every draw uses numpy's PCG64 (``default_rng``) seeded from a
``SeedSequence((config, index, ...))`` in fp64, then rounded to the stored dtype
with round-to-nearest-even (via torch's CPU cast).  "N(0, s)" means standard
deviation ``s``.

Workload recipes (the pages print recipe constants, not datasets; these are
the synthetic stand-ins):

* ``cfg0`` -- one fp32 256x512 weight.  Gradient = rank-8 spike with singular
  values linspace(10, 3, 8) plus N(0, 0.01) noise, momentum zero, W ~ N(0, 0.02).
* ``cfg1`` -- 64 bf16 1024x1024 weights.  Gradient U diag(1/i) V^T with Haar
  U, V (sigma_1 = 1); momentum fp32 N(0, 1e-3); W bf16 N(0, 0.02).
* ``cfg2`` -- 7B-shaped dense transformer, d_model 4096, 32 layers, per layer
  Wq, Wk, Wv, Wo 4096x4096, gate/up 14336x4096, down 4096x14336 (rows =
  out-features).  W bf16 N(0, 0.02); gradient bf16 N(0, 1e-3) * exp(z_row)
  with z_row ~ N(0, 1) per stored row; momentum fp32 zero (first step).
* ``cfg3`` -- causal MHA layer: X bf16 N(0, 1) [4, 4096, 4096]; Wq, Wk bf16
  N(0, 0.02) [4096, 4096] except the rows of heads 3, 17, 29, scaled x8.
* ``cfg4`` -- 64 MoE experts, gate/up 2048x7168 and down 7168x2048.  Gradient
  U diag(i^-0.5) V^T (orthonormal factors from QR of Gaussians); W bf16
  N(0, 0.02); momentum fp32 zero.
"""
from __future__ import annotations

import numpy as np
import torch

# Recipe constants printed by the pages (MuonClip: speed, then stability, §02
# and §05; About Muon: Muon At Scale, "What Moonlight, K2, and GLM Ran").
HPARAMS = dict(mu=0.95, nesterov=True, lr=0.02, wd=0.1, ns_steps=5,
               a=3.4445, b=-4.7750, c=2.0315, eps=1e-7, rms_scale=0.2)
QK_TAU = 100.0
QK_ALPHA = 0.5


def rng_for(*key: int) -> np.random.Generator:
    """A PCG64 generator keyed by a tuple of non-negative ints."""
    return np.random.default_rng(np.random.SeedSequence(list(int(k) for k in key)))


def to_dtype(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """Round an fp64 array to the stored dtype (round-to-nearest-even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    if dtype == torch.bfloat16:
        # fp64 -> fp32 is exact-enough here (RNE), fp32 -> bf16 is RNE.
        return t.to(torch.float32).to(torch.bfloat16)
    return t.to(dtype)


def orthonormal_columns(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """n x k matrix with orthonormal columns: Q of a Gaussian's QR, signs fixed
    so that diag(R) > 0 (this makes Q Haar-distributed)."""
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))[None, :]


def spectral_matrix(rng: np.random.Generator, rows: int, cols: int,
                    sigma: np.ndarray) -> np.ndarray:
    """rows x cols matrix U diag(sigma) V^T with random orthonormal U, V."""
    k = len(sigma)
    U = orthonormal_columns(rng, rows, k)
    V = orthonormal_columns(rng, cols, k)
    return (U * sigma[None, :]) @ V.T


# --------------------------------------------------------------------------
# Config shapes
# --------------------------------------------------------------------------
def cfg2_shapes(layers: int = 32, d_model: int = 4096, d_ff: int = 14336):
    """(rows, cols) of every hidden 2D weight of the 7B-shaped model, in
    per-layer order q, k, v, o, gate, up, down."""
    per_layer = [(d_model, d_model)] * 4 + [(d_ff, d_model)] * 2 + [(d_model, d_ff)]
    return [s for _ in range(layers) for s in per_layer]


def cfg4_shapes(experts: int = 64, d_model: int = 2048, d_ff: int = 7168):
    """(rows, cols) of the MoE experts: gate and up d_model x d_ff, down d_ff x d_model."""
    per_expert = [(d_model, d_ff), (d_model, d_ff), (d_ff, d_model)]
    return [s for _ in range(experts) for s in per_expert]


CFG3 = dict(B=4, S=4096, D=4096, H=32, dh=128, hot_heads=(3, 17, 29), hot_scale=8.0)
# Multi-head latent attention layer at the same scale: each head's 192-wide
# query/key split into a 128-wide content part and a 64-wide rotary part (the
# rotary key shared by all heads).
MLA = dict(B=4, S=4096, D=4096, H=32, dc=128, dr=64, hot_heads=(3, 17, 29), hot_scale=8.0)


# --------------------------------------------------------------------------
# Per-matrix draws (host).  Each returns (W, G, M) torch CPU tensors in the
# stored dtypes.
# --------------------------------------------------------------------------
def cfg0_matrix(seed: int = 0):
    rng = rng_for(0, seed)
    r, c = 256, 512
    W = to_dtype(rng.normal(0.0, 0.02, (r, c)), torch.float32)
    spike = spectral_matrix(rng, r, c, np.linspace(10.0, 3.0, 8))
    G = to_dtype(spike + rng.normal(0.0, 0.01, (r, c)), torch.float32)
    M = torch.zeros((r, c), dtype=torch.float32)
    return W, G, M


def cfg1_matrix(idx: int, n: int = 1024, seed: int = 1):
    rng = rng_for(1, seed, idx)
    sigma = 1.0 / np.arange(1, n + 1, dtype=np.float64)
    G = to_dtype(spectral_matrix(rng, n, n, sigma), torch.bfloat16)
    M = to_dtype(rng.normal(0.0, 1e-3, (n, n)), torch.float32)
    W = to_dtype(rng.normal(0.0, 0.02, (n, n)), torch.bfloat16)
    return W, G, M


def rowscaled_gradient(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    z = rng.standard_normal((rows, 1))
    return rng.normal(0.0, 1e-3, (rows, cols)) * np.exp(z)


def cfg2_matrix(idx: int, seed: int = 2):
    r, c = cfg2_shapes()[idx]
    rng = rng_for(2, seed, idx)
    W = to_dtype(rng.normal(0.0, 0.02, (r, c)), torch.bfloat16)
    G = to_dtype(rowscaled_gradient(rng, r, c), torch.bfloat16)
    M = torch.zeros((r, c), dtype=torch.float32)
    return W, G, M


def cfg4_matrix(idx: int, seed: int = 4):
    r, c = cfg4_shapes()[idx]
    rng = rng_for(4, seed, idx)
    m = min(r, c)
    sigma = np.arange(1, m + 1, dtype=np.float64) ** -0.5
    G = to_dtype(spectral_matrix(rng, r, c, sigma), torch.bfloat16)
    W = to_dtype(rng.normal(0.0, 0.02, (r, c)), torch.bfloat16)
    M = torch.zeros((r, c), dtype=torch.float32)
    return W, G, M


def generic_matrix(rows: int, cols: int, seed: int, *, w_dtype=torch.bfloat16,
                   g_dtype=torch.bfloat16, m_std: float = 1e-3, g_std: float = 1e-2):
    """Plain Gaussian W/G/M of any shape (edge-case and ragged-tile tests)."""
    rng = rng_for(9, seed, rows, cols)
    W = to_dtype(rng.normal(0.0, 0.02, (rows, cols)), w_dtype)
    G = to_dtype(rng.normal(0.0, g_std, (rows, cols)), g_dtype)
    M = to_dtype(rng.normal(0.0, m_std, (rows, cols)), torch.float32)
    return W, G, M


# --------------------------------------------------------------------------
# QK workload
# --------------------------------------------------------------------------
def qk_inputs(B: int, S: int, D: int, H: int, dh: int, *, seed: int = 3,
              hot_heads=(), hot_scale: float = 8.0, w_std: float = 0.02):
    """X [B, S, D], Wq and Wk [H*dh, D] (nn.Linear layout), all bf16.
    The rows of every head in ``hot_heads`` are multiplied by ``hot_scale`` in
    both Wq and Wk (before rounding), which multiplies that head's logits by
    hot_scale**2."""
    rng = rng_for(3, seed, B, S, D, H, dh)
    X = rng.standard_normal((B, S, D))
    Wq = rng.normal(0.0, w_std, (H * dh, D))
    Wk = rng.normal(0.0, w_std, (H * dh, D))
    for h in hot_heads:
        Wq[h * dh:(h + 1) * dh] *= hot_scale
        Wk[h * dh:(h + 1) * dh] *= hot_scale
    return (to_dtype(X, torch.bfloat16), to_dtype(Wq, torch.bfloat16),
            to_dtype(Wk, torch.bfloat16))


def mla_inputs(B: int, S: int, D: int, H: int, dc: int, dr: int, *, seed: int = 5,
               hot_heads=(), hot_scale: float = 8.0, w_std: float = 0.02):
    """X [B, S, D] and the MLA projection weights, all bf16 (nn.Linear layout):
    W_qC, W_kC [H*dc, D], W_qR [H*dr, D], W_kR [dr, D].  The head-specific rows
    (W_qC, W_kC, W_qR) of every head in ``hot_heads`` are multiplied by
    ``hot_scale``; the shared W_kR is not."""
    rng = rng_for(5, seed, B, S, D, H, dc, dr)
    X = rng.standard_normal((B, S, D))
    Wqc = rng.normal(0.0, w_std, (H * dc, D))
    Wkc = rng.normal(0.0, w_std, (H * dc, D))
    Wqr = rng.normal(0.0, w_std, (H * dr, D))
    Wkr = rng.normal(0.0, w_std, (dr, D))
    for h in hot_heads:
        Wqc[h * dc:(h + 1) * dc] *= hot_scale
        Wkc[h * dc:(h + 1) * dc] *= hot_scale
        Wqr[h * dr:(h + 1) * dr] *= hot_scale
    bf = torch.bfloat16
    return (to_dtype(X, bf), {"W_qC": to_dtype(Wqc, bf), "W_kC": to_dtype(Wkc, bf),
                              "W_qR": to_dtype(Wqr, bf), "W_kR": to_dtype(Wkr, bf)})


def mla_layer_inputs():
    c = MLA
    return mla_inputs(c["B"], c["S"], c["D"], c["H"], c["dc"], c["dr"], seed=5,
                      hot_heads=c["hot_heads"], hot_scale=c["hot_scale"])


def cfg3_inputs():
    c = CFG3
    return qk_inputs(c["B"], c["S"], c["D"], c["H"], c["dh"], seed=3,
                     hot_heads=c["hot_heads"], hot_scale=c["hot_scale"])


# --------------------------------------------------------------------------
# Device-side bulk draws, for timing only (values are not compared; every
# compared matrix is drawn on the host above and copied in).
# --------------------------------------------------------------------------
def cfg2_device_tensors(device, seed: int = 2, layers: int = 32):
    """W, G, M for the whole 7B-shaped set, drawn on the device with torch's
    seeded generator: same shapes and distributions as ``cfg2_matrix``."""
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 + seed)
    Ws, Gs, Ms = [], [], []
    for (r, c) in cfg2_shapes(layers=layers):
        W = (torch.randn((r, c), device=device, generator=gen) * 0.02).to(torch.bfloat16)
        z = torch.randn((r, 1), device=device, generator=gen)
        G = (torch.randn((r, c), device=device, generator=gen) * 1e-3 * torch.exp(z)).to(torch.bfloat16)
        M = torch.zeros((r, c), device=device, dtype=torch.float32)
        Ws.append(W); Gs.append(G); Ms.append(M)
    return Ws, Gs, Ms
