"""fp64 oracle of QK-Clip -- TEST INFRASTRUCTURE ONLY (see package doc).

Sources (page title, then section):

* [MC] "MuonClip: speed, then stability" -- §05 "QK-Clip" (per-head
  S_max = max over batch and token pairs of the pre-softmax score;
  gamma_h = min(1, tau/S_max); W_q <- gamma^alpha W_q, W_k <- gamma^(1-alpha) W_k;
  worked example 400 -> gamma 0.25, each side x0.5; 80 -> untouched),
  §07 (momentum is not clipped).
* [MV] "Muon and MuonClip: orthogonalised updates for LLM training" --
  "The exploding-logit problem" (S_max^h = (1/sqrt(d)) max_{samples,i,j} q_i.k_j),
  "MuonClip: QK-clip, per head, adapted to MLA" (MHA rule, alpha = 0.5).
* [MS] "About Muon: Muon At Scale" -- "When Softmax Collapses" (same rule).
* Multi-head latent attention: [MC] §06 "Multi-head latent attention changes
  the surgery" and [MV] "MuonClip: QK-clip, per head, adapted to MLA" (the
  head-specific content query q^C and content key k^C scale by sqrt(gamma_h),
  the head-specific rotary query q^R by gamma_h, the shared rotary key k^R is
  left untouched; [MC] §12 asks implementers to name the physical slices).

Readings where the pages are silent:

* The 1/sqrt(d_head) factor is inside S_max ([MV]).
* Causal attention: a query i sees keys j <= i (the diagonal counts).
* The max is signed (the largest softmax input), not over |score|.
* Plain MHA, no positional terms: q = x W_q^T, rows of W are nn.Linear
  out-features, head h owns rows [h*dh, (h+1)*dh).
* S_max == tau does not clip ("when S_max > tau"); this also keeps gamma
  positive when S_max <= 0.
"""
from __future__ import annotations

import numpy as np


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64.

    Used only for the optional "Q and K stored as bf16" mode, which mirrors
    a kernel that keeps its projections in bf16.  Goes through float32 (RNE)
    and then clears the low 16 bits with RNE on the float32 bit pattern.
    """
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    nan = np.isnan(f)
    out = u.astype(np.uint32).view(np.float32).astype(np.float64)
    out[nan] = np.nan
    return out


def qk_max_logit(X, Wq, Wk, H: int, dh: int, causal: bool = True,
                 qk_bf16: bool = False) -> np.ndarray:
    """Per-head S_max = max_{b, i, j (<= i if causal)} (q_{b,i,h} . k_{b,j,h}) / sqrt(dh).

    X is [B, S, D]; Wq, Wk are [H*dh, D].  Q_b = X_b Wq^T and K_b = X_b Wk^T
    in float64 (optionally rounded to bf16 when ``qk_bf16``).  Returns float64 [H].
    """
    X = np.asarray(X, dtype=np.float64)
    Wq = np.asarray(Wq, dtype=np.float64)
    Wk = np.asarray(Wk, dtype=np.float64)
    B, S, _ = X.shape
    smax = np.full(H, -np.inf)
    keep = np.tril(np.ones((S, S), dtype=bool)) if causal else np.ones((S, S), dtype=bool)
    scale = 1.0 / np.sqrt(dh)
    for b in range(B):
        Q = X[b] @ Wq.T
        K = X[b] @ Wk.T
        if qk_bf16:
            Q = round_bf16(Q)
            K = round_bf16(K)
        for h in range(H):
            q = Q[:, h * dh:(h + 1) * dh]
            k = K[:, h * dh:(h + 1) * dh]
            s = (q @ k.T) * scale
            smax[h] = max(smax[h], float(np.max(np.where(keep, s, -np.inf))))
    return smax


def qk_max_logit_bruteforce(X, Wq, Wk, H: int, dh: int, causal: bool = True) -> np.ndarray:
    """The same statistic by explicit loops over every (b, h, i, j) pair and
    every feature -- for tiny inputs only (an independent check of the above)."""
    X = np.asarray(X, dtype=np.float64)
    Wq = np.asarray(Wq, dtype=np.float64)
    Wk = np.asarray(Wk, dtype=np.float64)
    B, S, D = X.shape
    out = [-np.inf] * H
    for b in range(B):
        for h in range(H):
            for i in range(S):
                for j in range(S):
                    if causal and j > i:
                        continue
                    dot = 0.0
                    for e in range(dh):
                        r = h * dh + e
                        qi = sum(X[b, i, t] * Wq[r, t] for t in range(D))
                        kj = sum(X[b, j, t] * Wk[r, t] for t in range(D))
                        dot += qi * kj
                    out[h] = max(out[h], dot / np.sqrt(dh))
    return np.array(out)


def qk_clip(Wq, Wk, smax, tau: float, alpha: float, H: int, dh: int):
    """QK-Clip for MHA ([MC] §05, [MV], [MS]).

    gamma_h = tau / S_max_h if S_max_h > tau else 1; the rows of head h in Wq
    are scaled by gamma_h**alpha and in Wk by gamma_h**(1 - alpha).  Heads that
    are not clipped are returned bit-for-bit unchanged.  Returns
    (Wq', Wk', gamma [H], mask [H] int32).
    """
    Wq = np.array(Wq, dtype=np.float64, copy=True)
    Wk = np.array(Wk, dtype=np.float64, copy=True)
    smax = np.asarray(smax, dtype=np.float64)
    gamma = np.ones(H)
    mask = np.zeros(H, dtype=np.int32)
    for h in range(H):
        if smax[h] > tau:
            gamma[h] = tau / smax[h]
            mask[h] = 1
            Wq[h * dh:(h + 1) * dh] *= gamma[h] ** alpha
            Wk[h * dh:(h + 1) * dh] *= gamma[h] ** (1.0 - alpha)
    return Wq, Wk, gamma, mask


def qk_clip_slices(weights: dict, slices, smax, tau: float):
    """QK-Clip over an explicit map of weight slices ([MC] §06, §12.5).

    ``weights``: name -> 2D array (rows are output features).  ``slices``: list
    of (name, head, row_begin, row_end, exponent); rows [row_begin, row_end) of
    weights[name] are multiplied by gamma_head**exponent when that head clips.
    MHA is the map {W_q rows of h: alpha, W_k rows of h: 1 - alpha}; MLA is
    {q^C rows of h: 1/2, k^C rows of h: 1/2, q^R rows of h: 1} with the shared
    k^R absent.  gamma_h = tau / S_max_h if S_max_h > tau else 1.  Returns
    (new weights dict, gamma [H], mask [H]).
    """
    smax = np.asarray(smax, dtype=np.float64)
    H = len(smax)
    gamma = np.ones(H)
    mask = np.zeros(H, dtype=np.int32)
    for h in range(H):
        if smax[h] > tau:
            gamma[h] = tau / smax[h]
            mask[h] = 1
    out = {k: np.array(v, dtype=np.float64, copy=True) for k, v in weights.items()}
    for (name, h, r0, r1, e) in slices:
        if mask[h]:
            out[name][r0:r1] *= gamma[h] ** e
    return out, gamma, mask


def mla_max_logit(X, w: dict, H: int, dc: int, dr: int, causal: bool = True,
                  qk_bf16: bool = False) -> np.ndarray:
    """Per-head max logit of a (simplified, uncompressed) multi-head latent
    attention score, split into a content and a rotary part:

      s_h(i, j) = (q^C_{h,i} . k^C_{h,j} + q^R_{h,i} . k^R_j) / sqrt(dc + dr)

    with q^C = x W_qC[h], k^C = x W_kC[h], q^R = x W_qR[h] (head-specific rows)
    and k^R = x W_kR (one rotary key shared by every head).  Positional
    rotation is omitted: it does not change how the clip factors enter.
    X is [B, S, D]; W_qC, W_kC are [H*dc, D], W_qR is [H*dr, D], W_kR [dr, D].
    ``qk_bf16`` rounds the four projections to bf16, as ``qk_max_logit`` does.
    """
    X = np.asarray(X, dtype=np.float64)
    B, S, _ = X.shape
    keep = np.tril(np.ones((S, S), dtype=bool)) if causal else np.ones((S, S), dtype=bool)
    scale = 1.0 / np.sqrt(dc + dr)
    out = np.full(H, -np.inf)
    for b in range(B):
        qc = X[b] @ np.asarray(w["W_qC"], dtype=np.float64).T
        kc = X[b] @ np.asarray(w["W_kC"], dtype=np.float64).T
        qr = X[b] @ np.asarray(w["W_qR"], dtype=np.float64).T
        kr = X[b] @ np.asarray(w["W_kR"], dtype=np.float64).T
        if qk_bf16:
            qc, kc, qr, kr = (round_bf16(t) for t in (qc, kc, qr, kr))
        for h in range(H):
            s = (qc[:, h * dc:(h + 1) * dc] @ kc[:, h * dc:(h + 1) * dc].T
                 + qr[:, h * dr:(h + 1) * dr] @ kr.T) * scale
            out[h] = max(out[h], float(np.max(np.where(keep, s, -np.inf))))
    return out


def mla_slices(H: int, dc: int, dr: int):
    """The MLA slice map of [MC] §06: (name, head, row_begin, row_end, exponent)."""
    sl = []
    for h in range(H):
        sl.append(("W_qC", h, h * dc, (h + 1) * dc, 0.5))
        sl.append(("W_kC", h, h * dc, (h + 1) * dc, 0.5))
        sl.append(("W_qR", h, h * dr, (h + 1) * dr, 1.0))
    return sl
