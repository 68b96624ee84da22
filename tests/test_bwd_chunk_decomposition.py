"""The four-launch decomposition of the chunkwise backward (gdn_bwd_chunk), restated
in fp64 numpy, against the backward oracle (CPU).

The CUDA kernels reorganise the chain rule of oracle/chunk_backward.py: a ragged
last chunk is padded with tokens that leave the state alone (k = q = v = dO = 0,
alpha = 1, beta = 0) so that row 63 is always the last row; the gate terms are
gathered as row and column sums (rows of Q o dO S^T, of T^T dW o K, ...); dT is
formed with the gates on its columns.  This test runs exactly that arrangement,
launch by launch, in fp64 and requires the oracle's gradients to rounding, so
any algebraic slip in the arrangement (a dropped term, a wrong side for a gate,
the padding) fails here, with no GPU.  Source of the forward: "Qwen3.8-Flash-Next
技术总结 -- Qwen4 架构的探路者", section 2.1 "Gated DeltaNet".
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_07_b200 import inputs

C = 64


def _pad(x, L, fill=0.0):
    return x if L == C else np.concatenate([x, np.full((C - L,) + x.shape[1:], fill)])


def four_launches(q, k, v, al, be, dO, S0, dSf, mutation=None):
    B, T, Hqk, D = q.shape
    Hv = v.shape[2]
    grp = Hv // Hqk
    NC = (T + C - 1) // C
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dalpha=np.zeros_like(al),
               dbeta=np.zeros_like(be), dS0=np.zeros((B, Hv, D, D)))
    low = np.tril(np.ones((C, C))) > 0
    for b in range(B):
        for h in range(Hv):
            hq = h // grp
            # 1. preparation (per chunk): gates, A, T, W, U~, P
            prep = []
            for n in range(NC):
                t0 = n * C
                L = min(C, T - t0)
                c = dict(L=L, t0=t0, K=_pad(k[b, t0:t0 + L, hq], L), Q=_pad(q[b, t0:t0 + L, hq], L),
                         V=_pad(v[b, t0:t0 + L, h], L), O=_pad(dO[b, t0:t0 + L, h], L),
                         a=_pad(al[b, t0:t0 + L, h], L, 0.5 if mutation == "pad_alpha" else 1.0),
                         bt=_pad(be[b, t0:t0 + L, h], L))
                bb = np.cumsum(np.log(c["a"]))
                c["Gam"] = np.where(low, np.exp(np.minimum(bb[:, None] - bb[None, :], 0.0)), 0.0)
                c["gam"], c["g"] = np.exp(bb), np.exp(bb[-1] - bb)
                c["KK"], c["QK"] = c["K"] @ c["K"].T, c["Q"] @ c["K"].T
                A = np.tril(c["bt"][:, None] * c["Gam"] * c["KK"], -1)
                c["Tm"] = np.linalg.inv(np.eye(C) + A)
                c["W"] = (c["Tm"] * (c["bt"] * c["gam"])[None, :]) @ c["K"]
                c["Ut"] = (c["Tm"] * c["bt"][None, :]) @ c["V"]
                c["P"] = c["Gam"] * c["QK"]
                prep.append(c)
            # 2. forward state chain: chunk start states and U
            S = np.zeros((D, D)) if S0 is None else S0[b, h].copy()
            Ss, Us = [], []
            for c in prep:
                Ss.append(S)
                U = c["Ut"] - c["W"] @ S
                Us.append(U)
                S = c["gam"][-1] * S + c["K"].T @ (c["g"][:, None] * U)
            # 3. gradient chain, from the last chunk: dS', dU, sum(dS' o S), dS0
            dS = np.zeros((D, D)) if dSf is None else dSf[b, h].copy()
            dSp, dUs, gC = [None] * NC, [None] * NC, [None] * NC
            for n in range(NC - 1, -1, -1):
                c = prep[n]
                dSp[n], gC[n] = dS, np.sum(dS * Ss[n])
                dU = c["g"][:, None] * (c["K"] @ dS) + (c["P"] if mutation == "P_untransposed" else c["P"].T) @ c["O"]
                dUs[n] = dU
                dS = c["gam"][-1] * dS + c["Q"].T @ (c["gam"][:, None] * c["O"]) - c["W"].T @ dU
            out["dS0"][b, h] = dS
            # 4. per-chunk gradients, gate terms as row / column sums
            for n, c in enumerate(prep):
                S, U, dU = Ss[n], Us[n], dUs[n]
                K, Q, V, O, bt, gam, g, Gam, Tm = (c[x] for x in ("K", "Q", "V", "O", "bt", "gam", "g", "Gam", "Tm"))
                X1 = O @ S.T
                dq = (g if mutation == "g_for_gamma" else gam)[:, None] * X1
                r_dgam = np.sum(Q * X1, 1)
                dW = -(dU @ S.T)
                dPG = (O @ U.T) * Gam
                GGP = dPG * c["QK"]
                dq += dPG @ K
                dk = dPG.T @ Q
                TdW = Tm.T @ dW
                dk += (bt * gam)[:, None] * TdW
                r_dbg = np.sum(TdW * K, 1)
                TdU = Tm.T @ dU
                dv = bt[:, None] * TdU
                r_db2 = np.sum(TdU * V, 1)
                X3 = U @ dSp[n].T
                dk += g[:, None] * X3
                r_dg = np.sum(K * X3, 1)
                dT = (bt * gam)[None, :] * (dW @ K.T) + bt[None, :] * (dU @ V.T)
                if mutation == "dT_rows":   # the gates on the rows instead of the columns
                    dT = (bt * gam)[:, None] * (dW @ K.T) + bt[:, None] * (dU @ V.T)
                dA = np.tril(-((Tm.T @ dT) @ Tm.T), -1)
                r_db3 = np.sum(dA * Gam * c["KK"], 1)
                GGA = bt[:, None] * dA * Gam * c["KK"]
                M = bt[:, None] * dA * Gam
                dk += (M if mutation == "no_Mt" else M + M.T) @ K
                dgamma = r_dgam + r_dbg * bt
                dbeta = r_dbg * gam + r_db2 + r_db3
                gg = r_dg * g
                db = dgamma * gam + GGP.sum(1) + GGA.sum(1) - GGP.sum(0) - GGA.sum(0) - gg
                if mutation == "col_sum_sign":
                    db += 2 * (GGP.sum(0) + GGA.sum(0))
                db[-1] += (0.0 if mutation == "drop_gC" else gC[n] * gam[-1]) + gg.sum()
                dla = np.cumsum(db[::-1])[::-1]
                L, t0 = c["L"], c["t0"]
                out["dq"][b, t0:t0 + L, hq] += dq[:L]
                out["dk"][b, t0:t0 + L, hq] += dk[:L]
                out["dv"][b, t0:t0 + L, h] = dv[:L]
                out["dbeta"][b, t0:t0 + L, h] = dbeta[:L]
                out["dalpha"][b, t0:t0 + L, h] = dla[:L] / c["a"][:L]
    return out


@pytest.mark.parametrize("T,s0,dsf", [(1, True, True), (64, False, True), (77, True, False), (130, True, True)])
def test_four_launch_arrangement_matches_the_oracle(T, s0, dsf):
    d = inputs.prefill_inputs(1, T, 1, 3, dtype=torch.float32, s0_std=0.3 if s0 else 0.0, seed=900 + T)
    if not s0:
        d["S0"] = None
    g = torch.Generator().manual_seed(T)
    dO = torch.randn(1, T, 3, 128, generator=g)
    dSf = torch.randn(1, 3, 128, 128, generator=g) * 0.1 if dsf else None
    f64 = lambda x: None if x is None else x.double().numpy()
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, d["S0"], dSf)
    got = four_launches(*(f64(x) for x in (d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, d["S0"], dSf)))
    for name, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), ref):
        err = np.abs(got[name] - r).max() / max(np.abs(r).max(), 1e-300)
        assert err < 1e-10, f"{name}: {err:.2e}"


@pytest.mark.parametrize("mutation", ["pad_alpha", "g_for_gamma", "no_Mt", "col_sum_sign", "drop_gC", "dT_rows",
                                      "P_untransposed"])
def test_each_planted_slip_is_caught(mutation):
    """Each plausible slip in the arrangement (padding, a gate on the wrong side, a
    dropped or sign-flipped term, a transposed operand) moves some gradient far past
    rounding: the comparison above would fail."""
    T = 77   # two chunks, the second ragged
    d = inputs.prefill_inputs(1, T, 1, 3, dtype=torch.float32, s0_std=0.3, seed=977)
    g = torch.Generator().manual_seed(5)
    dO = torch.randn(1, T, 3, 128, generator=g)
    dSf = torch.randn(1, 3, 128, 128, generator=g) * 0.1
    f64 = lambda x: None if x is None else x.double().numpy()
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, d["S0"], dSf)
    got = four_launches(*(f64(x) for x in (d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, d["S0"], dSf)),
                        mutation=mutation)
    worst = max(np.abs(got[name] - r).max() / max(np.abs(r).max(), 1e-300)
                for name, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), ref))
    assert worst > 1e-6, f"{mutation} not caught ({worst:.1e})"
