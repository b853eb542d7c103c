"""Shared helpers for the GPU parity tests (tolerances and comparisons)."""
import numpy as np
import torch

# Tolerances fixed for this path: the relative Frobenius error of the Newton-
# Schulz update (every shape: matrices whose short side is at most 16 run the
# fp32 thin path, the rest bf16 tensor-core GEMMs), the fp32 elementwise
# stages, S_max and the clip factors.
NS_TOL = 2e-2
EW_TOL = 1e-5
SMAX_TOL = 5e-3
GAMMA_TOL = 5e-3


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def to64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def round_like(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Round fp64 values into the storage dtype (RNE), back to fp64."""
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == torch.bfloat16:
        t = t.to(torch.float32).to(torch.bfloat16)
    else:
        t = t.to(dtype)
    return t.to(torch.float64).numpy()


def check_muon_matrix(W0, G, M0, W1, M1, U1, nrm, hp, oracle_out, tag=""):
    """Compare one matrix of a GPU Muon step with the oracle.

    W0, G, M0: inputs (CPU tensors, stored dtypes); W1, M1, U1, nrm: GPU outputs
    (CPU copies; U1 is the applied update); oracle_out: (W, M, update, norm).
    """
    Wo, Mo, Uo, no = oracle_out
    w0 = to64(W0)
    # fp32 elementwise stages: momentum and the norm of the NS input
    assert rel_fro(to64(M1), Mo) <= EW_TOL, f"{tag} momentum"
    assert abs(float(nrm) - no) <= EW_TOL * no + 1e-30, f"{tag} norm {float(nrm)} vs {no}"
    # bf16 Newton-Schulz path: the applied update
    e_upd = rel_fro(to64(U1), Uo)
    tol = NS_TOL
    assert e_upd <= tol, f"{tag} update rel err {e_upd} (bound {tol})"
    # the apply itself (fp32 math, then the weight's dtype)
    lr, wd = hp["lr"], hp["wd"]
    w_exp = (1.0 - lr * wd) * w0 - lr * to64(U1)
    w1 = to64(W1)
    if W0.dtype == torch.float32:
        assert rel_fro(w1 - w0, w_exp - w0) <= EW_TOL, f"{tag} apply"
    else:
        ulp = np.spacing(np.abs(round_like(w_exp, torch.bfloat16)).astype(np.float32)).astype(np.float64) * 65536
        # fp32 evaluation of (1 - lr wd) w + (-lr) u: a few fp32 roundings of
        # the operands, which matter where the two terms nearly cancel
        slack = 4 * 2.0 ** -24 * (np.abs(w0) + lr * np.abs(to64(U1)))
        err = np.abs(w1 - w_exp)
        assert np.all(err <= ulp + slack), f"{tag} apply beyond 1 bf16 ulp: {np.max(err - ulp - slack)}"
        assert np.mean(w1 == round_like(w_exp, W0.dtype)) >= 0.999, f"{tag} apply rounding"
    # end to end against the oracle, both rounded into the weight's dtype
    wo = round_like(Wo, W0.dtype)
    e_dw = rel_fro(w1 - w0, wo - w0)
    if W0.dtype == torch.float32:
        assert e_dw <= tol, f"{tag} dW rel err {e_dw}"
    else:
        # Rounding W_new to bf16 quantises dW in steps of one ulp of W, about
        # 1/30 of dW here.  On large matrices that noise averages out far below
        # NS_TOL; on matrices of a few elements it does not, so there the bound
        # is NS_TOL plus the relative size q of one ulp against dW.
        ulp_o = np.spacing(np.abs(wo).astype(np.float32)).astype(np.float64) * 65536
        q = float(np.sqrt(np.mean(ulp_o ** 2)) / max(np.sqrt(np.mean((wo - w0) ** 2)), 1e-30))
        bound = tol if w1.size >= 10000 else tol + q
        assert e_dw <= bound, f"{tag} dW rel err {e_dw} (bound {bound})"
    return e_upd, e_dw
