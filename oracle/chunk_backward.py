"""fp64 numpy restatement of the backward pass in the chunkwise (WY) form.

TEST INFRASTRUCTURE ONLY.  A second route to the gradients of ``backward.py``
(the adjoint of the token recurrence): the tests require the two to agree,
which pins the blocked algebra a chunkwise backward kernel needs, gate
gradients included.  It shares no code with the CUDA path.

Source of the forward: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者",
section 2.1 "Gated DeltaNet" (chunkwise WY evaluation; the chunk equations are
the ones ``chunk_form.py`` derives).  Per chunk of length L from state S, with
b = cumsum(log alpha), gamma = exp(b), Gam[r, i] = exp(b_r - b_i) (i <= r),
g = exp(b_{L-1} - b), Tm = (I + A)^-1, A = strict_lower(diag(beta)(Gam o K K^T)):

    W = Tm diag(beta gamma) K,  U~ = Tm diag(beta) V,  U = U~ - W S
    O = diag(gamma) Q S + (Gam o Q K^T) U,  S' = gamma_{L-1} S + (diag(g) K)^T U

The backward below is the chain rule through these equations, chunk by chunk
from the end, given dO and the gradient dS' of the chunk's end state:

    dS   = gamma_{L-1} dS' + Q^T diag(gamma) dO - W^T dU
    dU   = (diag(g) K) dS' + P^T dO              (P = Gam o Q K^T, lower)
    dW   = -dU S^T,   dU~ = dU,   dP = dO U^T
    dT   = dW (diag(beta gamma) K)^T + dU~ (diag(beta) V)^T
    dA   = -Tm^T dT Tm^T  (strictly lower)

then K, Q, V, beta collect their terms from every place they appear, and the
decay factors (gamma, Gam, g, gamma_{L-1}) pass their gradients to b, whose
reverse cumulative sum is d log alpha.
"""
import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def _chunk_terms(K, Q, V, al, be):
    """Decay factors and WY terms of one chunk (everything that does not need S)."""
    L = K.shape[0]
    bc = np.cumsum(np.log(al))
    gamma = np.exp(bc)
    lower = np.tril(np.ones((L, L), dtype=bool))
    Gam = np.where(lower, np.exp(np.where(lower, bc[:, None] - bc[None, :], 0.0)), 0.0)
    KK, QK = K @ K.T, Q @ K.T
    A = np.tril(be[:, None] * Gam * KK, k=-1)
    Tm = np.linalg.inv(np.eye(L) + A)
    W = Tm @ ((be * gamma)[:, None] * K)
    Ut = Tm @ (be[:, None] * V)
    g = np.exp(bc[-1] - bc)
    return dict(gamma=gamma, Gam=Gam, KK=KK, QK=QK, Tm=Tm, W=W, Ut=Ut, g=g)


def chunk_backward(q, k, v, alpha, beta, dO, S0=None, dS_final=None, chunk=64):
    """Gradients (dq, dk, dv, dalpha, dbeta, dS0) through the chunkwise form;
    same arguments, shapes and head map as ``backward.backward``."""
    q, k, v, alpha, beta, dO, S0, dS_final = (_f64(a) for a in (q, k, v, alpha, beta, dO, S0, dS_final))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hqk
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dal, dbe = np.zeros_like(alpha), np.zeros_like(beta)
    dS0 = np.zeros((B, Hv, dk, dv))
    starts = list(range(0, T, chunk))
    for b in range(B):
        for h in range(Hv):
            hq = h // grp
            # forward over the chunks, keeping each chunk's start state
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            S_start = []
            for c0 in starts:
                L = min(chunk, T - c0)
                K, Q, V = k[b, c0:c0 + L, hq], q[b, c0:c0 + L, hq], v[b, c0:c0 + L, h]
                al, be = alpha[b, c0:c0 + L, h], beta[b, c0:c0 + L, h]
                t = _chunk_terms(K, Q, V, al, be)
                S_start.append(S)
                U = t["Ut"] - t["W"] @ S
                S = t["gamma"][-1] * S + (t["g"][:, None] * K).T @ U
            # backward over the chunks
            dSn = np.zeros((dk, dv)) if dS_final is None else dS_final[b, h].copy()
            for ci in range(len(starts) - 1, -1, -1):
                c0 = starts[ci]
                L = min(chunk, T - c0)
                K, Q, V = k[b, c0:c0 + L, hq], q[b, c0:c0 + L, hq], v[b, c0:c0 + L, h]
                al, be = alpha[b, c0:c0 + L, h], beta[b, c0:c0 + L, h]
                dOc = dO[b, c0:c0 + L, h]
                t = _chunk_terms(K, Q, V, al, be)
                S = S_start[ci]
                gamma, Gam, g, Tm, W = t["gamma"], t["Gam"], t["g"], t["Tm"], t["W"]
                U = t["Ut"] - W @ S
                P = Gam * t["QK"]
                Kt = g[:, None] * K
                # end state S' = gamma_{L-1} S + Kt^T U
                dS = gamma[-1] * dSn
                d_gC = np.sum(dSn * S)
                dU = Kt @ dSn
                dKt = U @ dSn.T
                # outputs O = diag(gamma) Q S + P U
                dS += Q.T @ (gamma[:, None] * dOc)
                dQ = gamma[:, None] * (dOc @ S.T)
                dgamma = np.sum((Q @ S) * dOc, axis=1)
                dP = dOc @ U.T
                dU += P.T @ dOc
                # U = U~ - W S
                dW = -dU @ S.T
                dS += -W.T @ dU
                dUt = dU
                # P = Gam o Q K^T (lower, diagonal included)
                dPG = dP * Gam
                dQ += dPG @ K
                dK = dPG.T @ Q
                dGam = dP * t["QK"]
                # Kt = diag(g) K
                dK += g[:, None] * dKt
                dg = np.sum(K * dKt, axis=1)
                # W = Tm diag(beta gamma) K,  U~ = Tm diag(beta) V
                bgK, bV = (be * gamma)[:, None] * K, be[:, None] * V
                dTm = dW @ bgK.T + dUt @ bV.T
                TdW, TdU = Tm.T @ dW, Tm.T @ dUt
                dK += (be * gamma)[:, None] * TdW
                dV = be[:, None] * TdU
                dbg = np.sum(TdW * K, axis=1)
                dbeta = dbg * gamma + np.sum(TdU * V, axis=1)
                dgamma += dbg * be
                # Tm = (I + A)^-1,  A = strict_lower(diag(beta) (Gam o K K^T))
                dA = np.tril(-Tm.T @ dTm @ Tm.T, k=-1)
                dbeta += np.sum(dA * Gam * t["KK"], axis=1)
                dGam += dA * be[:, None] * t["KK"]
                M = be[:, None] * dA * Gam
                dK += (M + M.T) @ K
                # decay factors -> b -> log alpha
                db = dgamma * gamma
                db[-1] += d_gC * gamma[-1]
                GG = dGam * Gam
                db += GG.sum(axis=1) - GG.sum(axis=0)
                gg = dg * g
                db[-1] += gg.sum()
                db -= gg
                dla = np.cumsum(db[::-1])[::-1]
                dq[b, c0:c0 + L, hq] += dQ
                dkk[b, c0:c0 + L, hq] += dK
                dvv[b, c0:c0 + L, h] = dV
                dbe[b, c0:c0 + L, h] = dbeta
                dal[b, c0:c0 + L, h] = dla / al
                dSn = dS
            dS0[b, h] = dSn
    return dq, dkk, dvv, dal, dbe, dS0
