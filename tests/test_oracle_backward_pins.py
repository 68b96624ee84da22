"""Pins of the fp64 backward oracle (oracle/backward.py) to things other than itself.

* its forward states agree with the forward oracle (C, pinned in test_oracle_pins);
* every gradient agrees with central finite differences of the forward (fp64,
  tiny sizes): the derivative is checked against the definition, not against a
  second copy of the adjoint formulas;
* the no-write case (beta = 0, alpha = 1: S_t = S0 for all t) has closed forms
  for every gradient;
* shared QK heads receive the sum of the gradients of the V heads reading them.
"""
import numpy as np
import pytest

import oracle
from oracle.backward import backward, forward_states


def _problem(B, T, Hqk, Hv, dk, dv, seed, s0=True, dsf=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, Hqk, dk)) / np.sqrt(dk)
    k = rng.standard_normal((B, T, Hqk, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, dv))
    alpha = rng.uniform(0.6, 1.0, (B, T, Hv))
    beta = rng.uniform(0.1, 0.9, (B, T, Hv))
    dO = rng.standard_normal((B, T, Hv, dv))
    S0 = rng.standard_normal((B, Hv, dk, dv)) * 0.5 if s0 else None
    dSf = rng.standard_normal((B, Hv, dk, dv)) if dsf else None
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, dO=dO, S0=S0, dS_final=dSf)


def _loss(d):
    """L = sum_t <dO_t, S_t^T q_t> + <dS_final, S_T>, straight from the forward."""
    B, T, Hqk, _ = d["q"].shape
    Hv = d["v"].shape[2]
    g = Hv // Hqk
    L = 0.0
    for b in range(B):
        for h in range(Hv):
            hq = h // g
            s0 = np.zeros((d["k"].shape[-1], d["v"].shape[-1])) if d["S0"] is None else d["S0"][b, h]
            S = forward_states(d["k"][b, :, hq], d["v"][b, :, h], d["alpha"][b, :, h], d["beta"][b, :, h], s0)
            for t in range(T):
                L += d["dO"][b, t, h] @ (S[t].T @ d["q"][b, t, hq])
            if d["dS_final"] is not None:
                L += np.sum(d["dS_final"][b, h] * S[T - 1])
    return L


def test_backward_states_match_forward_oracle():
    d = _problem(2, 9, 1, 3, 5, 4, seed=1)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    # the forward oracle reads fp32 inputs: compare on fp32-rounded copies
    r = {key: (None if a is None else a.astype(np.float32).astype(np.float64)) for key, a in d.items()}
    for b in range(2):
        for h in range(3):
            S = forward_states(r["k"][b, :, 0], r["v"][b, :, h], r["alpha"][b, :, h], r["beta"][b, :, h],
                               r["S0"][b, h])
            np.testing.assert_allclose(S[8], S_ref[b, h], rtol=1e-12, atol=1e-12)
            o = np.einsum("tij,ti->tj", S[:9], r["q"][b, :, 0])
            np.testing.assert_allclose(o, o_ref[b, :, h], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [3, 4])
def test_backward_matches_finite_differences(seed):
    d = _problem(1, 5, 1, 2, 3, 2, seed=seed)
    grads = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    names = ["q", "k", "v", "alpha", "beta", "S0"]
    eps = 1e-6
    for name, grad in zip(names, grads):
        x = d[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = _loss(d)
            x[idx] = keep - eps
            lm = _loss(d)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_closed_form_without_writes():
    """beta = 0, alpha = 1: S_t = S0, o_t = S0^T q_t.  With G_t = dS_final +
    sum_{s >= t} q_s dO_s^T: dq_t = S0 dO_t, dk = dv = 0, dS0 = G_0,
    dbeta_t = k_t^T G_t (v_t - S0^T k_t), dalpha_t = <G_t, S0>."""
    d = _problem(1, 7, 2, 2, 4, 3, seed=9)
    d["alpha"][:] = 1.0
    d["beta"][:] = 0.0
    dq, dk, dv, dal, dbe, dS0 = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"],
                                         d["S0"], d["dS_final"])
    np.testing.assert_array_equal(dk, 0.0)
    np.testing.assert_array_equal(dv, 0.0)
    for h in range(2):
        S0, q, k, v, dO = d["S0"][0, h], d["q"][0, :, h], d["k"][0, :, h], d["v"][0, :, h], d["dO"][0, :, h]
        G = d["dS_final"][0, h].copy()
        for t in range(6, -1, -1):
            G = G + np.outer(q[t], dO[t])
            np.testing.assert_allclose(dq[0, t, h], S0 @ dO[t], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(dbe[0, t, h], k[t] @ G @ (v[t] - S0.T @ k[t]), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(dal[0, t, h], np.sum(G * S0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dS0[0, h], G, rtol=1e-12, atol=1e-12)


def test_backward_shared_heads_sum():
    """Two V heads reading one QK head get, in dq and dk, the sum of what two
    separate QK heads holding the same q, k would get."""
    d = _problem(1, 6, 1, 2, 4, 3, seed=11)
    shared = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    q2, k2 = np.repeat(d["q"], 2, axis=2), np.repeat(d["k"], 2, axis=2)
    split = backward(q2, k2, d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    np.testing.assert_allclose(shared[0][:, :, 0], split[0].sum(axis=2), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(shared[1][:, :, 0], split[1].sum(axis=2), rtol=1e-12, atol=1e-12)
    for a, b in zip(shared[2:], split[2:]):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_backward_head_range_selects_heads():
    d = _problem(1, 5, 1, 3, 3, 2, seed=12)
    full = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    part = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"],
                    h_range=(1, 2))
    np.testing.assert_allclose(part[2][:, :, 1], full[2][:, :, 1], rtol=1e-12)
    np.testing.assert_array_equal(part[2][:, :, 0], 0.0)


@pytest.mark.parametrize("chunk", [4, 7, 64])
def test_chunk_backward_agrees_with_token_adjoint(chunk):
    """The chunkwise-WY backward (the blocked algebra a chunked kernel follows,
    gate gradients through the cumulative log-decays included) gives the token
    adjoint's gradients; several chunks, a ragged tail, shared QK heads."""
    from oracle.chunk_backward import chunk_backward
    d = _problem(2, 29, 1, 2, 6, 5, seed=20 + chunk)
    ref = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    got = chunk_backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"],
                         chunk=chunk)
    for name, g, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-9, atol=1e-11, err_msg=name)


def test_chunk_backward_head_dim_128_and_no_states():
    from oracle.chunk_backward import chunk_backward
    d = _problem(1, 70, 1, 1, 128, 128, seed=33, s0=False, dsf=False)
    ref = backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"])
    got = chunk_backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], chunk=64)
    for name, g, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), got, ref):
        scale = max(np.abs(r).max(), 1e-300)
        assert np.abs(g - r).max() <= 1e-9 * scale, name


# --------------------------------------------------------------------------- mutants
def _adjoint(mistake=None):
    """The adjoint walk with one planted mistake, to check that the pins catch it."""
    def impl(q, k, v, alpha, beta, dO, S0=None, dS_final=None):
        B, T, Hqk, dk = q.shape
        Hv, dv = v.shape[2], v.shape[3]
        g = Hv // Hqk
        dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        dal, dbe = np.zeros_like(alpha), np.zeros_like(beta)
        dS0 = np.zeros((B, Hv, dk, dv))
        for b in range(B):
            for h in range(Hv):
                hq = h // g
                kk, qq = k[b, :, hq], q[b, :, hq]
                s0 = np.zeros((dk, dv)) if S0 is None else S0[b, h]
                S = forward_states(kk, v[b, :, h], alpha[b, :, h], beta[b, :, h], s0)
                G = np.zeros((dk, dv)) if dS_final is None else dS_final[b, h].copy()
                for t in range(T - 1, -1, -1):
                    a, be = alpha[b, t, h], beta[b, t, h]
                    kt, do = kk[t], dO[b, t, h]
                    P = S[t - 1]
                    if mistake != "readout_grad_after_update":
                        G = G + np.outer(qq[t], do)
                    dq[b, t, hq] += (P if mistake == "dq_from_previous_state" else S[t]) @ do
                    x, w = G.T @ kt, P.T @ kt
                    r = v[b, t, h] - a * w
                    dvv[b, t, h] = x if mistake == "dv_without_beta" else be * x
                    dbe[b, t, h] = x @ (v[b, t, h] if mistake == "dbeta_without_correction" else r)
                    dal[b, t, h] = np.sum(G * P) - (0.0 if mistake == "dalpha_without_write_term" else be * (x @ w))
                    sgn = -1.0 if mistake == "dk_sign" else 1.0
                    dkk[b, t, hq] += be * (G @ r) - sgn * a * be * (P @ x)
                    if mistake == "G_without_decay":
                        G = G - be * np.outer(kt, x)
                    else:
                        G = a * (G - be * np.outer(kt, x))
                    if mistake == "readout_grad_after_update":
                        G = G + np.outer(qq[t], do)
                dS0[b, h] = G
        return dq, dkk, dvv, dal, dbe, dS0
    return impl


def _pin_finite_differences(impl):
    d = _problem(1, 4, 1, 2, 3, 2, seed=5)
    grads = impl(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    eps = 1e-6
    for name, grad in zip(["q", "k", "v", "alpha", "beta", "S0"], grads):
        x = d[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = _loss(d)
            x[idx] = keep - eps
            lm = _loss(d)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-7, err_msg=name)


def _pin_closed_form(impl):
    d = _problem(1, 5, 1, 1, 3, 2, seed=6)
    d["alpha"][:] = 1.0
    d["beta"][:] = 0.0
    dq, dk, dv, dal, dbe, dS0 = impl(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"],
                                     d["dS_final"])
    S0, q, k, v, dO = d["S0"][0, 0], d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0], d["dO"][0, :, 0]
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)
    np.testing.assert_allclose(dv, 0.0, atol=1e-12)
    G = d["dS_final"][0, 0].copy()
    for t in range(4, -1, -1):
        G = G + np.outer(q[t], dO[t])
        np.testing.assert_allclose(dq[0, t, 0], S0 @ dO[t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dbe[0, t, 0], k[t] @ G @ (v[t] - S0.T @ k[t]), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dal[0, t, 0], np.sum(G * S0), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dS0[0, 0], G, rtol=1e-10, atol=1e-12)


BACKWARD_PINS = [_pin_finite_differences, _pin_closed_form]
BACKWARD_MUTANTS = ["readout_grad_after_update", "dq_from_previous_state", "dv_without_beta",
                    "dbeta_without_correction", "dalpha_without_write_term", "dk_sign",
                    "G_without_decay"]


def test_backward_oracle_and_unmutated_adjoint_pass_pins():
    for pin in BACKWARD_PINS:
        pin(backward)
        pin(_adjoint(None))


@pytest.mark.parametrize("mistake", BACKWARD_MUTANTS)
def test_backward_pins_catch_mutants(mistake):
    caught = []
    for pin in BACKWARD_PINS:
        try:
            pin(_adjoint(mistake))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {mistake!r}"
