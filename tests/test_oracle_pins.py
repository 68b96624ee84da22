"""Pins of the CPU oracle against what the pages and the mathematics fix.

Source of the method: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section
2.1 "Gated DeltaNet" (two equal forms of the state update; alpha_t in (0, 1) is a
forget gate, beta_t the write strength; the write corrects "new value minus what
memory already predicts").  The page prints no worked example and no read-out, so
each pin below is a closed form, an invariant, a special case or a brute-force
evaluation that a plausible mistake in the oracle (dropped term, wrong sign or
index, transposed operand, wrong head map) would break.  ``test_pins_catch_mutants``
plants such mistakes in copies of the recurrence and checks that the pins reject
every one of them.
"""
import os

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------------- helpers
def c_oracle(q, k, v, alpha, beta, S0=None):
    return oracle.forward(q, k, v, alpha, beta, S0, nthreads=2)


def dyadic(rng, shape, bits=6):
    """Random values that are exact in fp32 (small dyadic rationals)."""
    return (rng.integers(-(2 ** bits), 2 ** bits, size=shape) / 2 ** bits).astype(np.float32)


def random_case(rng, B=1, T=12, Hqk=1, Hv=1, dk=4, dv=3, s0=True, unit_keys=True):
    q = rng.standard_normal((B, T, Hqk, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, Hqk, dk)).astype(np.float32)
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, dv)).astype(np.float32)
    alpha = np.exp(rng.uniform(-0.5, -0.01, (B, T, Hv))).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((B, T, Hv))))).astype(np.float32)
    S0 = rng.standard_normal((B, Hv, dk, dv)).astype(np.float32) if s0 else None
    return q, k, v, alpha, beta, S0


def load_golden(path):
    out = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            name, rhs = (s.strip() for s in line.split("=", 1))
            out[name] = np.array([[float(x) for x in row.split()] for row in rhs.split(";")])
    return out


# --------------------------------------------------------------------------- pins
# Each pin takes an implementation impl(q, k, v, alpha, beta, S0) -> (o, S_final)
# with the oracle's shapes and raises AssertionError when it disagrees.

def pin_hand_example(impl):
    g = load_golden(os.path.join(os.path.dirname(__file__), "golden", "hand_example_2x2.txt"))
    T = 2
    q = g["q"].reshape(1, T, 1, 2)
    k = g["k"].reshape(1, T, 1, 2)
    v = g["v"].reshape(1, T, 1, 2)
    alpha = g["alpha"].reshape(1, T, 1)
    beta = g["beta"].reshape(1, T, 1)
    S0 = g["S0"].reshape(1, 1, 2, 2)
    o, S = impl(q, k, v, alpha, beta, S0)
    assert np.array_equal(o[0, :, 0], g["o"]), (o[0, :, 0], g["o"])
    assert np.array_equal(S[0, 0], g["S_final"]), (S[0, 0], g["S_final"])


def pin_second_form(impl):
    """Form 2 of the page: S_t = a (I - b k k^T) S_{t-1} + b k v^T, evaluated with
    explicit dk x dk matrices, must equal the result (T = 20, several heads)."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(7), B=2, T=20, Hqk=2, Hv=4,
                                           dk=5, dv=3, unit_keys=False)
    o, S = impl(q, k, v, alpha, beta, S0)
    B, T, Hqk, dk = q.shape
    Hv = v.shape[2]
    for b in range(B):
        for h in range(Hv):
            hq = h // (Hv // Hqk)
            St = S0[b, h].astype(np.float64)
            for t in range(T):
                kt = k[b, t, hq].astype(np.float64)[:, None]
                vt = v[b, t, h].astype(np.float64)[:, None]
                a, be = float(alpha[b, t, h]), float(beta[b, t, h])
                St = a * (np.eye(dk) - be * kt @ kt.T) @ St + be * kt @ vt.T
                np.testing.assert_allclose(o[b, t, h], St.T @ q[b, t, hq].astype(np.float64),
                                           rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S[b, h], St, rtol=1e-12, atol=1e-12)


def pin_identity_gate(impl):
    """alpha = 1, beta = 0: nothing is forgotten or written; S stays S0 and
    o_t = S0^T q_t."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(8), T=9, dk=4, dv=3)
    alpha[:] = 1.0
    beta[:] = 0.0
    o, S = impl(q, k, v, alpha, beta, S0)
    np.testing.assert_array_equal(S[0, 0], S0[0, 0].astype(np.float64))
    for t in range(q.shape[1]):
        np.testing.assert_allclose(o[0, t, 0], S0[0, 0].astype(np.float64).T @ q[0, t, 0],
                                   rtol=1e-13, atol=1e-13)


def pin_pure_decay(impl):
    """beta = 0: S_t = (prod_{s<=t} alpha_s) S0, so o_t = (prod alpha) S0^T q_t."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(9), T=11, dk=4, dv=3)
    beta[:] = 0.0
    o, S = impl(q, k, v, alpha, beta, S0)
    decay = np.cumprod(alpha[0, :, 0].astype(np.float64))
    S0d = S0[0, 0].astype(np.float64)
    np.testing.assert_allclose(S[0, 0], decay[-1] * S0d, rtol=1e-13, atol=1e-15)
    for t in range(q.shape[1]):
        np.testing.assert_allclose(o[0, t, 0], decay[t] * (S0d.T @ q[0, t, 0]),
                                   rtol=1e-12, atol=1e-15)


def pin_delta_retrieval(impl):
    """alpha = beta = 1 with a unit key: after writing v_t under k_t the memory
    returns it exactly, S_t^T k_t = v_t, whatever S_{t-1} was.  Read with q_t = k_t.
    Keys are exact unit vectors (signed coordinate axes) so the check is exact."""
    rng = np.random.default_rng(10)
    T, dk, dv = 10, 4, 3
    k = np.zeros((1, T, 1, dk), np.float32)
    axes = rng.integers(0, dk, T)
    k[0, np.arange(T), 0, axes] = rng.choice([-1.0, 1.0], T)
    q = k.copy()
    v = dyadic(rng, (1, T, 1, dv))
    alpha = np.ones((1, T, 1), np.float32)
    beta = np.ones((1, T, 1), np.float32)
    S0 = dyadic(rng, (1, 1, dk, dv))
    o, _ = impl(q, k, v, alpha, beta, S0)
    np.testing.assert_array_equal(o[0, :, 0], v[0, :, 0].astype(np.float64))
    # And with generic (non-axis) unit keys it holds to rounding.
    q2, k2, v2, a2, b2, S02 = random_case(rng, T=10, dk=6, dv=4)
    a2[:] = 1.0
    b2[:] = 1.0
    k64 = k2.astype(np.float64)
    k64 /= np.linalg.norm(k64, axis=-1, keepdims=True)
    k2 = k64.astype(np.float32)
    o2, _ = impl(k2, k2, v2, a2, b2, S02)
    kk = (k2.astype(np.float64) ** 2).sum(-1)  # |k|^2 of the fp32 key, ~1 within 1e-7
    # S_t^T k = S_{t-1}^T k (1 - |k|^2) + v |k|^2 exactly; with |k| = 1 +- 1e-7 -> v.
    np.testing.assert_allclose(o2[0, :, 0], v2[0, :, 0], rtol=0, atol=1e-5)
    assert np.all(np.abs(kk - 1) < 1e-6)


def pin_orthonormal_memory(impl):
    """S0 = 0, alpha = beta = 1 and orthonormal keys: S = sum_i k_i v_i^T
    (associative memory), and reading with beta = 0 returns each stored v_i."""
    rng = np.random.default_rng(11)
    dk, dv, n = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T                                     # n orthonormal rows
    T = 2 * n
    k = np.zeros((1, T, 1, dk), np.float32)
    k[0, :n, 0] = keys
    q = np.zeros_like(k)
    q[0, n:, 0] = keys                                      # read phase queries
    v = np.zeros((1, T, 1, dv), np.float32)
    v[0, :n, 0] = rng.standard_normal((n, dv))
    alpha = np.ones((1, T, 1), np.float32)
    beta = np.zeros((1, T, 1), np.float32)
    beta[0, :n, 0] = 1.0
    o, S = impl(q, k, v, alpha, beta, None)
    k32 = k[0, :n, 0].astype(np.float64)
    expect_S = sum(np.outer(k32[i], v[0, i, 0]) for i in range(n))
    np.testing.assert_allclose(S[0, 0], expect_S, rtol=0, atol=1e-6)
    np.testing.assert_allclose(o[0, n:, 0], v[0, :n, 0], rtol=0, atol=1e-6)


def pin_product_expansion(impl):
    """Brute force on tiny inputs: with A_s = alpha_s (I - beta_s k_s k_s^T),
    S_t = (A_t ... A_1) S0 + sum_{s<=t} (A_t ... A_{s+1}) beta_s k_s v_s^T."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(12), T=16, dk=4, dv=3,
                                           unit_keys=False)
    o, S = impl(q, k, v, alpha, beta, S0)
    T, dk = q.shape[1], q.shape[3]
    K = k[0, :, 0].astype(np.float64)
    A = [alpha[0, s, 0] * (np.eye(dk) - beta[0, s, 0] * np.outer(K[s], K[s])) for s in range(T)]

    def chain(lo, hi):  # A_{hi} ... A_{lo}, identity when lo > hi
        M = np.eye(dk)
        for s in range(lo, hi + 1):
            M = A[s] @ M
        return M

    for t in range(T):
        St = chain(0, t) @ S0[0, 0].astype(np.float64)
        for s in range(t + 1):
            St = St + chain(s + 1, t) @ (beta[0, s, 0] * np.outer(K[s], v[0, s, 0]))
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0].astype(np.float64),
                                   rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-11, atol=1e-12)


def pin_scalar_closed_form(impl):
    """dk = dv = 1 with constant gates: S_t = a S_{t-1} + c with a = alpha (1 - beta k^2),
    c = beta k v, so S_T = a^T S0 + c (1 - a^T) / (1 - a) (geometric series)."""
    T = 40
    kq, vv, al, be, s0 = 0.75, 1.5, 0.875, 0.5, -2.0
    q = np.full((1, T, 1, 1), 1.25, np.float32)
    k = np.full((1, T, 1, 1), kq, np.float32)
    v = np.full((1, T, 1, 1), vv, np.float32)
    alpha = np.full((1, T, 1), al, np.float32)
    beta = np.full((1, T, 1), be, np.float32)
    S0 = np.full((1, 1, 1, 1), s0, np.float32)
    o, S = impl(q, k, v, alpha, beta, S0)
    a = al * (1 - be * kq * kq)
    c = be * kq * vv
    t = np.arange(1, T + 1)
    St = a ** t * s0 + c * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(o[0, :, 0, 0], 1.25 * St, rtol=1e-13)
    np.testing.assert_allclose(S[0, 0, 0, 0], St[-1], rtol=1e-13)


def pin_head_map(impl):
    """V head h reads QK head h // (Hv / Hqk) (contiguous groups); each head's result
    equals a single-head run on that head's own inputs."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(13), B=2, T=6, Hqk=2, Hv=6,
                                           dk=3, dv=2)
    o, S = impl(q, k, v, alpha, beta, S0)
    for b in range(2):
        for h in range(6):
            hq = h // 3
            sl = lambda x: x[b:b + 1, :, hq:hq + 1]  # noqa: E731
            o1, S1 = impl(sl(q), sl(k), v[b:b + 1, :, h:h + 1], alpha[b:b + 1, :, h:h + 1],
                          beta[b:b + 1, :, h:h + 1], S0[b:b + 1, h:h + 1])
            np.testing.assert_array_equal(o[b, :, h], o1[0, :, 0])
            np.testing.assert_array_equal(S[b, h], S1[0, 0])


PINS = [pin_hand_example, pin_second_form, pin_identity_gate, pin_pure_decay,
        pin_delta_retrieval, pin_orthonormal_memory, pin_product_expansion,
        pin_scalar_closed_form, pin_head_map]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(c_oracle)


# --------------------------------------------------------------------------- structure
def test_chunk_form_agrees_with_oracle():
    """The chunkwise WY restatement (an independent derivation) equals the token
    recurrence for chunk sizes 64, 16 and 7, with a partial last chunk."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(14), B=2, T=150, Hqk=2, Hv=6,
                                           dk=16, dv=8)
    o_ref, S_ref = c_oracle(q, k, v, alpha, beta, S0)
    scale = np.abs(o_ref).max()
    for C in (64, 16, 7):
        o_c, S_c = oracle.chunk_forward(q, k, v, alpha, beta, S0, chunk=C)
        assert np.abs(o_c - o_ref).max() <= 1e-12 * scale, C
        assert np.abs(S_c - S_ref).max() <= 1e-12 * np.abs(S_ref).max(), C


def test_chunk_form_agrees_at_head_dim_128():
    rng = np.random.default_rng(15)
    q, k, v, alpha, beta, _ = random_case(rng, T=130, Hqk=1, Hv=2, dk=128, dv=128, s0=False)
    o_ref, S_ref = c_oracle(q, k, v, alpha, beta, None)
    o_c, S_c = oracle.chunk_forward(q, k, v, alpha, beta, None, chunk=64)
    assert np.abs(o_c - o_ref).max() <= 1e-11 * np.abs(o_ref).max()
    assert np.abs(S_c - S_ref).max() <= 1e-11 * np.abs(S_ref).max()


def test_column_equivariance():
    """Each dv column of S evolves on its own: permuting the columns of v and S0
    permutes those of o and S_final."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(16), T=8, dk=4, dv=5)
    perm = np.array([3, 0, 4, 1, 2])
    o, S = c_oracle(q, k, v, alpha, beta, S0)
    o_p, S_p = c_oracle(q, k, v[..., perm], alpha, beta, S0[..., perm])
    np.testing.assert_array_equal(o_p, o[..., perm])
    np.testing.assert_array_equal(S_p, S[..., perm])


def test_split_invariance():
    """Running T1 tokens and then T2 tokens from the saved state equals one run."""
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(17), B=2, T=21, Hqk=1, Hv=2,
                                           dk=4, dv=3)
    o, S = c_oracle(q, k, v, alpha, beta, S0)
    T1 = 8
    o1, S1 = c_oracle(q[:, :T1], k[:, :T1], v[:, :T1], alpha[:, :T1], beta[:, :T1], S0)
    o2, S2 = c_oracle(q[:, T1:], k[:, T1:], v[:, T1:], alpha[:, T1:], beta[:, T1:],
                      S1.astype(np.float32))
    np.testing.assert_array_equal(o[:, :T1], o1)
    # the hand-off rounds S to fp32, the library's state precision
    np.testing.assert_allclose(o[:, T1:], o2, rtol=0, atol=1e-6 * np.abs(o).max())
    np.testing.assert_allclose(S, S2, rtol=0, atol=1e-6 * np.abs(S).max())


def test_decode_step_matches_forward():
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(18), B=3, T=5, Hqk=2, Hv=4,
                                           dk=4, dv=3)
    o, S = c_oracle(q, k, v, alpha, beta, S0)
    St = S0
    for t in range(5):
        ot, St64 = oracle.decode_step(q[:, t], k[:, t], v[:, t], alpha[:, t], beta[:, t], St)
        np.testing.assert_allclose(ot, o[:, t], rtol=0, atol=1e-6 * np.abs(o).max())
        St = St64.astype(np.float32)
    np.testing.assert_allclose(St, S, rtol=0, atol=1e-6 * np.abs(S).max())


def test_head_range_selects_heads():
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(19), B=2, T=7, Hqk=2, Hv=6,
                                           dk=3, dv=2)
    o, S = c_oracle(q, k, v, alpha, beta, S0)
    o_s, S_s = oracle.forward(q, k, v, alpha, beta, S0, h_range=(2, 5), nthreads=3)
    np.testing.assert_array_equal(o_s, o[:, :, 2:5])
    np.testing.assert_array_equal(S_s, S[:, 2:5])


def test_empty_sequence_returns_initial_state():
    q, k, v, alpha, beta, S0 = random_case(np.random.default_rng(20), T=0, dk=3, dv=2)
    o, S = c_oracle(q, k, v, alpha, beta, S0)
    assert o.shape == (1, 0, 1, 2)
    np.testing.assert_array_equal(S, S0.astype(np.float64))


# --------------------------------------------------------------------------- mutants
def _numpy_recurrence(mistake=None):
    """A plain recurrence with one planted mistake, to check the pins catch it."""
    def impl(q, k, v, alpha, beta, S0):
        q, k, v, alpha, beta = (np.asarray(a, np.float64) for a in (q, k, v, alpha, beta))
        B, T, Hqk, dk = q.shape
        Hv, dv = v.shape[2], v.shape[3]
        g = Hv // Hqk
        o = np.zeros((B, T, Hv, dv))
        Sf = np.zeros((B, Hv, dk, dv))
        for b in range(B):
            for h in range(Hv):
                hq = h % Hqk if mistake == "interleaved_heads" else h // g
                S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0[b, h], np.float64).copy()
                for t in range(T):
                    kt, qt, vt = k[b, t, hq], q[b, t, hq], v[b, t, h]
                    a, be = alpha[b, t, h], beta[b, t, h]
                    p = S.T @ kt
                    if mistake == "readout_before_update":
                        o[b, t, h] = S.T @ qt
                    if mistake == "dropped_alpha_in_correction":
                        u = be * (vt - p)
                    elif mistake == "sign_of_correction":
                        u = be * (vt + a * p)
                    elif mistake == "dropped_beta":
                        u = vt - a * p
                    elif mistake == "correction_with_S_not_transposed" and dk == dv:
                        u = be * (vt - a * (S @ kt))
                    else:
                        u = be * (vt - a * p)
                    if mistake == "alpha_on_write_too":
                        S = a * (S + np.outer(kt, u))
                    elif mistake == "outer_product_transposed" and dk == dv:
                        S = a * S + np.outer(u, kt)
                    else:
                        S = a * S + np.outer(kt, u)
                    if mistake == "readout_not_transposed" and dk == dv:
                        o[b, t, h] = S @ qt
                    elif mistake != "readout_before_update":
                        o[b, t, h] = S.T @ qt
                Sf[b, h] = S
        return o, Sf
    return impl


MUTANTS = ["readout_before_update", "dropped_alpha_in_correction", "sign_of_correction",
           "dropped_beta", "correction_with_S_not_transposed", "alpha_on_write_too",
           "outer_product_transposed", "readout_not_transposed", "interleaved_heads"]


def test_unmutated_numpy_recurrence_passes_pins():
    for pin in PINS:
        pin(_numpy_recurrence(None))


@pytest.mark.parametrize("mistake", MUTANTS)
def test_pins_catch_mutants(mistake):
    impl = _numpy_recurrence(mistake)
    caught = []
    for pin in PINS:
        try:
            pin(impl)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {mistake!r}"
