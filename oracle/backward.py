"""fp64 gradients of the gated delta rule: the adjoint of the token recurrence.

TEST INFRASTRUCTURE ONLY: used by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the library's compute path.

Forward (source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
"Gated DeltaNet", second form of the update), per (sequence, V head):

    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t

with V head h reading q and k of QK head h // (Hv / Hqk) (the grouping the
forward oracle documents).  The pages give the forward only; the gradients
below are its reverse-mode derivative, written from the chain rule for the
scalar L = sum_t <dO_t, o_t> + <dS_final, S_T>.  Walking t from T-1 down to 0
with G the gradient with respect to S_t (G = dS_final before the walk):

    G      += q_t dO_t^T                      (o_t = S_t^T q_t)
    dq_t   += S_t dO_t
    x       = G^T k_t,   w = S_{t-1}^T k_t,   r = v_t - alpha_t w
    dv_t    = beta_t x
    dbeta_t = x . r
    dalpha_t= <G, S_{t-1}> - beta_t x . w     (= <G, (I - beta k k^T) S_{t-1}>)
    dk_t   += beta_t G r - alpha_t beta_t S_{t-1} x
    G       = alpha_t (G - beta_t k_t x^T)    (gradient with respect to S_{t-1})

and dS0 = G at the end.  dq and dk of a QK head sum the contributions of the
V heads that read it.  Every state S_t is recomputed in fp64 and kept, so this
is for test sizes (a few hundred tokens per head), or one head group at a time.
"""
import numpy as np


def _f64(x):
    """fp64 host copy of an array or CPU/GPU tensor (bf16 upcasts exactly)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def forward_states(k, v, alpha, beta, S0):
    """States of one (sequence, V head): S[t] is the state after token t and
    S[-1] = S0.  k: [T, dk], v: [T, dv], alpha, beta: [T], S0: [dk, dv]."""
    T = k.shape[0]
    S = np.empty((T + 1,) + S0.shape)
    S[-1] = S0
    for t in range(T):
        P = S[t - 1]
        S[t] = alpha[t] * (P - beta[t] * np.outer(k[t], k[t] @ P)) + beta[t] * np.outer(k[t], v[t])
    return S


def backward(q, k, v, alpha, beta, dO, S0=None, dS_final=None, h_range=None):
    """Gradients of L = sum <dO, o> + <dS_final, S_final> with respect to every input.

    q, k: [B, T, Hqk, dk]; v, dO: [B, T, Hv, dv]; alpha, beta: [B, T, Hv];
    S0, dS_final: [B, Hv, dk, dv] or None (zeros).  ``h_range`` = (h0, h1)
    restricts the V heads (dq, dk then hold only their contributions).
    Returns (dq, dk, dv, dalpha, dbeta, dS0), fp64, in the input layouts.
    """
    q, k, v, alpha, beta, dO, S0, dS_final = (_f64(a) for a in (q, k, v, alpha, beta, dO, S0, dS_final))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    g = Hv // Hqk
    h0, h1 = (0, Hv) if h_range is None else h_range
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dal = np.zeros_like(alpha)
    dbe = np.zeros_like(beta)
    dS0 = np.zeros((B, Hv, dk, dv))
    for b in range(B):
        for h in range(h0, h1):
            hq = h // g
            kk, qq = k[b, :, hq], q[b, :, hq]
            s0 = np.zeros((dk, dv)) if S0 is None else S0[b, h]
            S = forward_states(kk, v[b, :, h], alpha[b, :, h], beta[b, :, h], s0)
            G = np.zeros((dk, dv)) if dS_final is None else dS_final[b, h].copy()
            for t in range(T - 1, -1, -1):
                a, be = alpha[b, t, h], beta[b, t, h]
                kt, do = kk[t], dO[b, t, h]
                P = S[t - 1]
                G += np.outer(qq[t], do)
                dq[b, t, hq] += S[t] @ do
                x = G.T @ kt
                w = P.T @ kt
                r = v[b, t, h] - a * w
                dvv[b, t, h] = be * x
                dbe[b, t, h] = x @ r
                dal[b, t, h] = np.sum(G * P) - be * (x @ w)
                dkk[b, t, hq] += be * (G @ r) - a * be * (P @ x)
                G = a * (G - be * np.outer(kt, x))
            dS0[b, h] = G
    return dq, dkk, dvv, dal, dbe, dS0
