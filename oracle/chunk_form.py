"""fp64 numpy restatement of the chunkwise (WY) form of the gated delta rule.

TEST INFRASTRUCTURE ONLY.  It is a second, independent route to the same
result as the token recurrence in ``gdn_oracle.c``: the tests require the two
to agree, which pins the oracle against the blocked algebra and documents the
equations the GPU kernels follow.  It shares no code with the CUDA path.

Source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated
DeltaNet".  The page names the chunkwise algorithm built on the WY
representation but prints no equations for it; the steps below are derived
from the page's first form of the update.  Write the update as
S_r = alpha_r S_{r-1} + k_r u_r^T with u_r = beta_r (v_r - alpha_r S_{r-1}^T k_r)
and unroll it inside a chunk of length L that starts from state S:

    b_r   = sum_{j<=r} log alpha_j              (chunk-local, inclusive)
    gamma_r = exp(b_r),  Gam[r, i] = exp(b_r - b_i) for i <= r, else 0
    S_r   = gamma_r S + sum_{i<=r} Gam[r, i] k_i u_i^T

Substituting S_{r-1} into u_r gives a unit lower-triangular system

    (I + A) U = diag(beta) (V - diag(gamma) K S),
    A[r, i] = beta_r Gam[r, i] (k_r . k_i)  for i < r,

so with Tm = (I + A)^{-1}:  U = Tm diag(beta) V - Tm diag(beta*gamma) K S
= U~ - W S.  The chunk's outputs and end state are then

    O       = diag(gamma) Q S + (Gam o Q K^T) U            (mask keeps i <= r)
    S_next  = gamma_{L-1} S + K~^T U,   K~ = diag(exp(b_{L-1} - b)) K.
"""
import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def chunk_forward(q, k, v, alpha, beta, S0=None, chunk=64):
    """Chunkwise WY evaluation; same shapes and head map as ``oracle.forward``."""
    q, k, v, alpha, beta, S0 = (_f64(a) for a in (q, k, v, alpha, beta, S0))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    g = Hv // Hqk
    o = np.zeros((B, T, Hv, dv))
    S_final = np.zeros((B, Hv, dk, dv))
    for b in range(B):
        for h in range(Hv):
            hq = h // g
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, chunk):
                L = min(chunk, T - c0)
                K = k[b, c0:c0 + L, hq]
                Q = q[b, c0:c0 + L, hq]
                V = v[b, c0:c0 + L, h]
                be = beta[b, c0:c0 + L, h]
                bc = np.cumsum(np.log(alpha[b, c0:c0 + L, h]))
                gamma = np.exp(bc)
                lower = np.tril(np.ones((L, L), dtype=bool))
                Gam = np.where(lower, np.exp(np.where(lower, bc[:, None] - bc[None, :], 0.0)), 0.0)
                A = np.tril(be[:, None] * Gam * (K @ K.T), k=-1)
                Tm = np.linalg.inv(np.eye(L) + A)
                W = Tm @ ((be * gamma)[:, None] * K)
                U_tilde = Tm @ (be[:, None] * V)
                U = U_tilde - W @ S
                o[b, c0:c0 + L, h] = gamma[:, None] * (Q @ S) + (Gam * (Q @ K.T)) @ U
                K_tilde = np.exp(bc[-1] - bc)[:, None] * K
                S = gamma[-1] * S + K_tilde.T @ U
            S_final[b, h] = S
    return o, S_final
