"""fp64 oracle of the Muon step -- TEST INFRASTRUCTURE ONLY (see package doc).

Sources (page title, then section):

* [MC] "MuonClip: speed, then stability" -- §02 "Momentum remembers.
  Orthogonalization redistributes." (momentum, Nesterov, quintic NS step and
  its coefficients, orientation), §03 "Making Muon scale" (0.2*sqrt(max(n,m))
  scale, decoupled decay W <- W - eta*(O + lambda*W)), §07 "One complete
  training step" (step order).
* [MV] "Muon and MuonClip: orthogonalised updates for LLM training" --
  §2 "Newton-Schulz: an odd polynomial on singular values" (X0 = G/||G||_F,
  A = X X^T, X = aX + (bA + cA A)X, phi(x) = ax + bx^3 + cx^5, m <= n cost
  rule), "The Muon optimizer" (M <- mu M + G; Moonlight form of the update).
* [MS] "About Muon: Muon At Scale" -- "Why Not Bernstein's Multiplier?"
  (update snippet: p *= 1 - lr*wd; p += -lr*scale*u, scale = 0.2*sqrt(max)),
  and "Certain Neurons Still Dominate" (NorMuon: one second-moment scalar per
  row, each row of the orthogonalised update divided by the square root of it,
  then the whole matrix rescaled to the Frobenius norm it had before).

Readings where the pages are silent:

* Nesterov lookahead: [MC] §02 only says one "may be applied".  Read as the
  recurrence applied once more with the current gradient, U = G + mu*M_t, in
  the pages' own sum convention M_t = mu*M_{t-1} + G_t.
* Orientation: the NS input is transposed only when rows > cols, so that
  A = X X^T is min(m,n) square; a square matrix is not transposed.
* Normalisation: X0 = U / max(||U||_F, eps) with eps = 1e-7, so that a zero
  matrix gives a zero update ([MV] prints U/||U||_F with no eps).
* Scale: 0.2*sqrt(max(rows, cols)) ([MC] §03, [MV], [MS]); weight decay acts
  on the pre-update W.
* Polar Express ([MS] "Which Norm for Which Layer"): the pages print only its
  effect (ten steps take 1e-4 to 0.994).  The schedule is read as the
  published construction: step t uses the odd quintic that is closest to 1 in
  the max norm on [l_t, u_t] (l_0 = 1e-3, u_0 = 1), then l_{t+1} = p_t(l_t),
  u_{t+1} = 2 - l_{t+1}; once the interval is narrower than 1e-3 the step is
  the limit of that polynomial, 15/8 x - 5/4 x^3 + 3/8 x^5; every polynomial
  but the last is then evaluated at x / 1.01 (a safety factor).
* NorMuon ([MS]): a "row" is an output feature (a row of the stored r x c
  weight); its second moment is an exponential average, v <- beta2*v +
  (1 - beta2)*mean_j(O_ij^2), with no bias correction; the row is divided by
  sqrt(v) + eps_v; the RMS-matching scale and decay then act as in Muon.
"""
from __future__ import annotations

import numpy as np


def phi(x, a: float, b: float, c: float):
    """The scalar odd quintic phi(x) = a x + b x^3 + c x^5 that one NS step
    applies to every singular value ([MV] §2, odd-polynomial identity)."""
    x = np.asarray(x, dtype=np.float64)
    return a * x + b * x ** 3 + c * x ** 5


def phi_iter(x, steps: int, a: float, b: float, c: float):
    """phi applied ``steps`` times."""
    y = np.asarray(x, dtype=np.float64)
    for _ in range(steps):
        y = phi(y, a, b, c)
    return y


def phi_schedule(x, coeffs):
    """phi_{(a_k, b_k, c_k)} applied in order, one step per coefficient triple."""
    y = np.asarray(x, dtype=np.float64)
    for (a, b, c) in coeffs:
        y = phi(y, a, b, c)
    return y


def newton_schulz(U: np.ndarray, steps: int, a: float, b: float, c: float,
                  eps: float = 1e-7, coeffs=None) -> np.ndarray:
    """Approximate polar factor of ``U`` by the quintic Newton-Schulz iteration.

    [MV] §2: X0 = U/||U||_F, then ``steps`` times A = X X^T,
    X = a X + (b A + c A A) X.  [MC] §02: A is formed after choosing the
    cheaper orientation, i.e. the short side first (m <= n); the result is
    transposed back.  ``coeffs``, if given, is a list of ``steps`` triples
    (a_k, b_k, c_k) used in iteration k instead of (a, b, c): the per-step
    coefficient schedules [MV] §2 compares (cubic, simple and tuned quintic)
    and that "About Muon: Muon At Scale" mentions for Polar Express.  Returns
    an array of U's shape.
    """
    U = np.asarray(U, dtype=np.float64)
    transposed = U.shape[0] > U.shape[1]
    X = U.T if transposed else U
    norm = np.sqrt(np.sum(X * X))
    X = X / max(norm, eps)
    for k in range(steps):
        ak, bk, ck = coeffs[k] if coeffs is not None else (a, b, c)
        A = X @ X.T
        B = bk * A + ck * (A @ A)
        X = ak * X + B @ X
    return X.T if transposed else X


def muon_step(W, G, M, *, mu, nesterov, lr, wd, ns_steps, a, b, c, eps, rms_scale, coeffs=None):
    """One Muon step on one hidden 2D weight, in float64.

    Follows [MC] §07's order: momentum, NS, scaled update with decoupled decay.

      M_t   = mu * M_{t-1} + G                          ([MC] §02, [MV])
      U     = G + mu * M_t  if nesterov else M_t         (reading, see module doc)
      O     = NS_steps(U)                                ([MV] §2)
      Upd   = rms_scale * sqrt(max(rows, cols)) * O      ([MC] §03, [MS])
      W_t   = W_{t-1} - lr * (Upd + wd * W_{t-1})        ([MC] §03)

    ``coeffs``: optional per-iteration (a_k, b_k, c_k) list (see newton_schulz).
    Returns (W_t, M_t, Upd, ||U||_F), all float64.
    """
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    M_new = mu * M + G
    U = G + mu * M_new if nesterov else M_new
    O = newton_schulz(U, ns_steps, a, b, c, eps, coeffs)
    upd = rms_scale * np.sqrt(max(W.shape)) * O
    W_new = W - lr * (upd + wd * W)
    return W_new, M_new, upd, float(np.sqrt(np.sum(U * U)))


def muon_step_many(Ws, Gs, Ms, hp: dict, workers: int = 1):
    """``muon_step`` over a list of independent matrices (optionally in a
    spawn-started process pool).  Returns lists (W_t, M_t, Upd, norm)."""
    args = [(W, G, M) for W, G, M in zip(Ws, Gs, Ms)]
    if workers <= 1 or len(args) <= 1:
        outs = [muon_step(W, G, M, **hp) for (W, G, M) in args]
    else:
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        with ctx.Pool(workers) as pool:
            outs = pool.starmap(_muon_step_kw, [(W, G, M, hp) for (W, G, M) in args])
    return [list(t) for t in zip(*outs)]


def _muon_step_kw(W, G, M, hp):
    return muon_step(W, G, M, **hp)


def normuon_rows(O: np.ndarray, v: np.ndarray, beta2: float, eps_v: float):
    """The NorMuon step after orthogonalisation ([MS] "Certain Neurons Still
    Dominate"): per-row second moment, row division, and the rescale back to
    the Frobenius norm of O.  Returns (O_hat, v_new)."""
    O = np.asarray(O, dtype=np.float64)
    rows, cols = O.shape
    v_new = np.empty(rows)
    O_hat = np.empty_like(O)
    for i in range(rows):
        v_new[i] = beta2 * float(v[i]) + (1.0 - beta2) * float(np.sum(O[i] * O[i])) / cols
        O_hat[i] = O[i] / (np.sqrt(v_new[i]) + eps_v)
    n_in = np.sqrt(np.sum(O * O))
    n_out = np.sqrt(np.sum(O_hat * O_hat))
    if n_out > 0:
        O_hat *= n_in / n_out
    return O_hat, v_new


def normuon_step(W, G, M, v, *, beta2, eps_v, mu, nesterov, lr, wd, ns_steps, a, b, c, eps, rms_scale,
                 coeffs=None):
    """One NorMuon step on one hidden 2D weight, in float64: the Muon step of
    ``muon_step`` with ``normuon_rows`` between Newton-Schulz and the scale.
    ``v`` is the per-row state (length rows).  Returns (W_t, M_t, Upd, v_t)."""
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    M_new = mu * M + G
    U = G + mu * M_new if nesterov else M_new
    O = newton_schulz(U, ns_steps, a, b, c, eps, coeffs)
    O_hat, v_new = normuon_rows(O, np.asarray(v, dtype=np.float64), beta2, eps_v)
    upd = rms_scale * np.sqrt(max(W.shape)) * O_hat
    W_new = W - lr * (upd + wd * W)
    return W_new, M_new, upd, v_new


def minimax_odd_quintic(lo: float, hi: float, iters: int = 200):
    """The odd quintic p(x) = a x + b x^3 + c x^5 minimising max |1 - p(x)| on
    [lo, hi] (0 < lo < hi), by the Remez exchange: solve for equal and
    alternating errors at four points, move the points to the extrema of the
    error (the ends and the two interior zeros of p'), repeat.  Returns
    ((a, b, c), E) with E the minimax error."""
    k = np.arange(4)
    xs = lo + (hi - lo) * (1.0 - np.cos(np.pi * k / 3.0)) / 2.0
    a = b = c = E = 0.0
    for _ in range(iters):
        A = np.stack([xs, xs ** 3, xs ** 5, (-1.0) ** k], axis=1)
        a, b, c, E = np.linalg.solve(A, np.ones(4))
        y = np.roots([5.0 * c, 3.0 * b, a])          # p'(x) = 0 with y = x^2
        inner = sorted(float(np.sqrt(r.real)) for r in y
                       if abs(r.imag) < 1e-12 and r.real > 0 and lo < np.sqrt(r.real) < hi)
        if len(inner) != 2:
            break
        new = np.array([lo, inner[0], inner[1], hi])
        if np.max(np.abs(new - xs)) <= 1e-15 * hi:
            break
        xs = new
    return (float(a), float(b), float(c)), float(abs(E))


def polar_express_schedule(steps: int, l0: float = 1e-3, safety: float = 0.01):
    """Per-iteration (a_k, b_k, c_k) of the Polar Express construction (see the
    module readings).  The safety factor maps p(x) to p(x / (1 + safety)) for
    all but the last step."""
    lo, hi = l0, 1.0
    out = []
    for _ in range(steps):
        if hi - lo < 1e-3:
            # the interval has shrunk onto 1, where the exchange is ill-conditioned
            # (and the minimax error below 1e-9): take the limit of the minimax
            # polynomial, the odd quintic with p(1) = 1 and p'(1) = p''(1) = 0
            (a, b, c), E = (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0), 0.0
        else:
            (a, b, c), E = minimax_odd_quintic(lo, hi)
        out.append((a, b, c))
        lo = a * lo + b * lo ** 3 + c * lo ** 5
        hi = 2.0 - lo
    s = 1.0 + safety
    return [(a / s, b / s ** 3, c / s ** 5) for (a, b, c) in out[:-1]] + [out[-1]]
