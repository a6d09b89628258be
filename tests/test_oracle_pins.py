"""Pins of the fp64 CPU oracle against what the pages and mathematics fix.

Each test compares an oracle route with a result obtained another way: the
materialised semiseparable matrix, a closed form, a textbook routine (numpy
matmul, convolve, FFT), exact rational arithmetic or a limit case.  The
mutation tests in test_oracle_mutations.py show that these pins catch
plausible mistakes planted in the oracle.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import ssd_oracle as O
from oracle.ssd_oracle import Problem
from tests.oracle_cases import (all_y, causal_conv_direct, causal_conv_fft, causal_linear_attention,
                                exact_rational_brute, free_response, lti_kernel, random_problem, rel_inf)

SHAPES = [
    # B, T, H, P, G, N
    (1, 1, 1, 1, 1, 1),
    (1, 2, 1, 2, 1, 2),
    (1, 3, 2, 1, 1, 3),
    (2, 7, 2, 3, 2, 2),
    (1, 16, 4, 2, 2, 4),
    (2, 24, 3, 4, 1, 5),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("per_state", [False, True])
def test_recurrence_matches_materialised_matrix(shape, per_state):
    """O1 (recurrence) == O2 (M = L o C B^T materialised), llms.blog "The SSD
    Theoretical Equivalence": M_{i,j} = C_i^T (prod_{k=j+1}^{i} a_k) B_j."""
    B, T, H, P, G, N = shape
    rng = np.random.default_rng(hash((shape, per_state)) % (2**32))
    prob = random_problem(rng, B, T, H, P, G, N, per_state=per_state)
    r1 = O.recurrence(prob)
    r2 = O.brute(prob)
    assert rel_inf(r1["y"], r2["y"]) < 1e-12
    assert rel_inf(r1["final"], r2["final"]) < 1e-12


@pytest.mark.parametrize("per_state", [False, True])
@pytest.mark.parametrize("T,chunks", [(16, [1, 2, 4, 8, 16]), (24, [1, 3, 6, 8, 12, 24]),
                                      (64, [4, 16, 32, 64])])
def test_chunked_is_chunk_invariant(per_state, T, chunks):
    """O3(chunk=q) == O1 for every q dividing T ("State Space Duality", "Two
    algorithms for one operator": the chunk boundary separates the quadratic
    and recurrent forms and nothing else).  q=1 is the pure recurrence, q=T
    the pure quadratic form.  Intermediates: the state handed to chunk k is
    the recurrence's h at t=kq-1, and the chunk cumsum is a prefix sum."""
    rng = np.random.default_rng(T + 7 * per_state)
    prob = random_problem(rng, 2, T, 4, 3, 2, 5, per_state=per_state)
    r1 = O.recurrence(prob, chunk=chunks[1])
    for q in chunks:
        r3 = O.chunked(prob, q)
        assert rel_inf(r3["y"], r1["y"]) < 1e-12, q
        assert rel_inf(r3["final"], r1["final"]) < 1e-12, q
    q = chunks[1]
    r3 = O.chunked(prob, q)
    rb = O.recurrence(prob, chunk=q)
    nc = T // q
    # Hin_k = state after chunk k-1 ; Hin_0 = 0
    assert np.all(r3["Hin"][:, 0] == 0)
    assert rel_inf(r3["Hin"][:, 1:], rb["bounds"][:, : nc - 1]) < 1e-12
    # cumsum restarts at each chunk
    a = prob.a if per_state else prob.a[..., None]
    for c, (b, h) in enumerate(r3["chains"]):
        ref = np.cumsum(a[b, :, h, :].reshape(nc, q, -1), axis=1)
        assert np.allclose(r3["cum"][c], ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("G,H", [(1, 1), (1, 3), (2, 4)])
def test_zero_decay_is_causal_linear_attention(G, H):
    """a == 0 makes every mask entry 1: y = tril(C B^T) X + D X ("State Space
    Duality", "Unrolling into a matrix": attention without a softmax)."""
    rng = np.random.default_rng(11 + G + H)
    prob = random_problem(rng, 2, 20, H, 3, G, 4)
    prob.a[...] = 0.0
    ref = causal_linear_attention(prob)
    for route in (O.recurrence(prob), O.brute(prob), O.chunked(prob, 5)):
        assert rel_inf(all_y(route, 2, H), ref) < 1e-12


@pytest.mark.parametrize("per_state", [False, True])
def test_lti_closed_form_convolution(per_state):
    """Time-invariant a, B, C: y = Kbar * x + D x with Kbar_j = sum_n gamma_n
    beta_n e^{alpha_n j} (llms.blog "Global Convolution"; flashpapers "The
    Dual Representations"), checked by direct and FFT convolution."""
    rng = np.random.default_rng(5 + per_state)
    B, T, H, P, G, N = 1, 48, 2, 3, 1, 4
    x = rng.standard_normal((B, T, H, P))
    beta = rng.standard_normal(N)
    gamma = rng.standard_normal(N)
    D = rng.standard_normal(H)
    alphas = [-rng.uniform(0.01, 0.6, size=N) if per_state else np.full(N, -rng.uniform(0.01, 0.6))
              for _ in range(H)]
    a = np.zeros((B, T, H, N)) if per_state else np.zeros((B, T, H))
    for h in range(H):
        if per_state:
            a[0, :, h, :] = alphas[h][None, :]
        else:
            a[0, :, h] = alphas[h][0]
    Bm = np.broadcast_to(beta, (B, T, G, N)).copy()
    Cm = np.broadcast_to(gamma, (B, T, G, N)).copy()
    prob = Problem(x, a, Bm, Cm, D)
    r1 = O.recurrence(prob)
    r3 = O.chunked(prob, 16)
    for h in range(H):
        K = lti_kernel(alphas[h], beta, gamma, T)
        X = x[0, :, h, :]
        ref_d = causal_conv_direct(K, X) + D[h] * X
        ref_f = causal_conv_fft(K, X) + D[h] * X
        assert rel_inf(ref_d, ref_f) < 1e-12
        assert rel_inf(r1["y"][h], ref_d) < 1e-12
        assert rel_inf(r3["y"][h], ref_d) < 1e-12
        # final state: sum_s e^{alpha (T-1-s)} beta x_s^T
        w = np.exp(alphas[h][None, :] * (T - 1 - np.arange(T))[:, None])  # [T,N]
        fin = (w * beta[None, :]).T @ X
        assert rel_inf(r1["final"][h], fin) < 1e-12


def test_diagonal_with_shared_decay_equals_scalar():
    """Per-state decays all equal to the head's scalar decay reduce the
    diagonal SSM to the scalar-identity one ("On Structured State-Space
    Duality", item (i): the scalar case is a special case)."""
    rng = np.random.default_rng(3)
    prob = random_problem(rng, 2, 32, 3, 4, 1, 6)
    N = prob.Bm.shape[3]
    diag = Problem(prob.x, np.repeat(prob.a[..., None], N, axis=-1), prob.Bm, prob.Cm, prob.D)
    for f in (lambda p: O.recurrence(p), lambda p: O.brute(p), lambda p: O.chunked(p, 8)):
        assert rel_inf(f(diag)["y"], f(prob)["y"]) < 1e-13
        assert rel_inf(f(diag)["final"], f(prob)["final"]) < 1e-13


@pytest.mark.parametrize("per_state", [False, True])
def test_grouped_bc_equals_replicated(per_state):
    """G < H (B, C shared by a contiguous group of H/G heads, llms.blog
    "Multi-Head State Space Layers") equals G = H with B, C replicated."""
    rng = np.random.default_rng(17)
    H, G = 6, 2
    prob = random_problem(rng, 2, 20, H, 3, G, 4, per_state=per_state)
    rep = lambda m: np.repeat(m, H // G, axis=2)
    full = Problem(prob.x, prob.a, rep(prob.Bm), rep(prob.Cm), prob.D)
    for f in (lambda p: O.recurrence(p), lambda p: O.chunked(p, 5), lambda p: O.brute(p)):
        assert rel_inf(f(prob)["y"], f(full)["y"]) < 1e-13


def test_memoryless_limit():
    """a -> -inf resets the state every step (llms.blog "The Selection
    Mechanism": Abar -> 0 focuses on the new token): y_t = (C_t.B_t) x_t + D x_t
    and the final state is B_{T-1} x_{T-1}^T."""
    rng = np.random.default_rng(23)
    prob = random_problem(rng, 1, 18, 2, 3, 1, 4)
    prob.a[...] = -1e4
    for route in (O.recurrence(prob), O.brute(prob), O.chunked(prob, 6)):
        for h in range(2):
            X = prob.x[0, :, h, :]
            cb = np.einsum("tn,tn->t", prob.Cm[0, :, 0, :], prob.Bm[0, :, 0, :])
            ref = cb[:, None] * X + prob.D[h] * X
            assert rel_inf(route["y"][h], ref) < 1e-13
            fin = np.outer(prob.Bm[0, -1, 0, :], X[-1])
            assert rel_inf(route["final"][h], fin) < 1e-13


def test_first_decay_irrelevant_causal_and_linear():
    """Index convention and masking (the product over k=j+1..i in M_{i,j}):
    a_0 never multiplies anything; y_t does not depend on x_s for s > t;
    the map is linear in x."""
    rng = np.random.default_rng(29)
    prob = random_problem(rng, 1, 24, 2, 3, 1, 4)
    base = O.recurrence(prob)["y"]
    p2 = Problem(prob.x, prob.a.copy(), prob.Bm, prob.Cm, prob.D)
    p2.a[:, 0] = -7.0
    assert rel_inf(O.recurrence(p2)["y"], base) < 1e-14
    assert rel_inf(O.chunked(p2, 8)["y"], base) < 1e-12
    s = 13
    p3 = Problem(prob.x.copy(), prob.a, prob.Bm, prob.Cm, prob.D)
    p3.x[:, s] += 5.0
    y3 = O.recurrence(p3)["y"]
    assert np.array_equal(y3[:, :s], base[:, :s])
    assert np.max(np.abs(y3[:, s:] - base[:, s:])) > 1e-3
    p4 = Problem(2.5 * prob.x, prob.a, prob.Bm, prob.Cm, prob.D)
    assert rel_inf(O.recurrence(p4)["y"], 2.5 * base) < 1e-14


def test_exact_rational_brute_force():
    """Decays that are powers of two and small-integer B, C, x give an exactly
    representable answer; exact Fraction arithmetic on the definition of M
    matches every route to rounding."""
    rng = np.random.default_rng(31)
    T, P, N = 9, 2, 3
    e = rng.integers(0, 3, size=T)  # lam_t = 2^-e_t
    lam = [Fraction(1, 2 ** int(v)) for v in e]
    Bi = rng.integers(-3, 4, size=(T, N))
    Ci = rng.integers(-3, 4, size=(T, N))
    xi = rng.integers(-4, 5, size=(T, P))
    Dq = Fraction(3, 4)
    exact = exact_rational_brute([[Fraction(int(v)) for v in r] for r in xi], lam,
                                 [[Fraction(int(v)) for v in r] for r in Bi],
                                 [[Fraction(int(v)) for v in r] for r in Ci], Dq)
    exact = np.array([[float(v) for v in r] for r in exact])
    prob = Problem(xi[None, :, None, :].astype(float), (-np.log(2.0) * e)[None, :, None],
                   Bi[None, :, None, :].astype(float), Ci[None, :, None, :].astype(float),
                   np.array([0.75]))
    for route in (O.recurrence(prob), O.brute(prob), O.chunked(prob, 3)):
        assert np.max(np.abs(route["y"][0] - exact)) < 1e-12 * max(1.0, np.max(np.abs(exact)))


def _read_golden(name):
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    rows = []
    meta = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                if line.startswith("# param "):
                    k, v = line[len("# param "):].split("=", 1)
                    meta[k.strip()] = v.strip()
                continue
            rows.append([float(v) for v in line.split()])
    return meta, np.array(rows)


def test_golden_impulse_response_decay_085():
    """Impulse response of the scalar time-invariant SSM with decay Abar = 0.85
    (the value flashpapers "State-Space Models", "Interactive Walkthrough"
    shows) and Bbar = C = 1: by llms.blog "Global Convolution", y_t = 0.85^t.
    The fixture holds 0.85^t from exact rational arithmetic."""
    meta, rows = _read_golden("impulse_decay_085.txt")
    T = rows.shape[0]
    lam = float(meta["decay"])
    x = np.zeros((1, T, 1, 1)); x[0, 0, 0, 0] = 1.0
    a = np.full((1, T, 1), math.log(lam))
    one = np.ones((1, T, 1, 1))
    prob = Problem(x, a, one, one, None)
    for route in (O.recurrence(prob), O.brute(prob), O.chunked(prob, 4)):
        assert np.max(np.abs(route["y"][0, :, 0] - rows[:, 1])) < 1e-14


@pytest.mark.parametrize("per_state", [False, True])
def test_initial_state_resumes_a_split_sequence(per_state):
    """Running the first t1 tokens, then the rest from the state they ended with,
    gives the single run's y and final state: the initial state is exactly the
    h_{-1} the recurrence would have carried (a sequence split across calls)."""
    rng = np.random.default_rng(31 + per_state)
    prob = random_problem(rng, B=2, T=40, H=3, P=4, G=1, N=5, per_state=per_state)
    B, T, H, P = prob.x.shape
    N = prob.Bm.shape[3]
    full = O.recurrence(prob)
    for t1 in (1, 17, 39):
        cut = lambda arr, sl: None if arr is None else arr[:, sl]
        first = O.Problem(prob.x[:, :t1], cut(prob.a, slice(0, t1)), prob.Bm[:, :t1], prob.Cm[:, :t1], prob.D)
        rest = O.Problem(prob.x[:, t1:], cut(prob.a, slice(t1, None)), prob.Bm[:, t1:], prob.Cm[:, t1:], prob.D)
        r1 = O.recurrence(first)
        r2 = O.recurrence(rest, initial=r1["final"].reshape(B, H, N, P))
        y = np.concatenate([all_y(r1, B, H), all_y(r2, B, H)], axis=2)
        assert rel_inf(y, all_y(full, B, H)) < 1e-12
        assert rel_inf(r2["final"], full["final"]) < 1e-12


@pytest.mark.parametrize("per_state", [False, True])
def test_initial_state_free_response(per_state):
    """x == 0: y is the decayed initial state read out by C (closed form)."""
    rng = np.random.default_rng(41 + per_state)
    prob = random_problem(rng, B=1, T=25, H=2, P=3, G=1, N=4, per_state=per_state)
    prob = O.Problem(np.zeros_like(prob.x), prob.a, prob.Bm, prob.Cm, prob.D)
    h0 = rng.standard_normal((1, 2, 4, 3))
    res = O.recurrence(prob, initial=h0)
    y_ref, fin_ref = free_response(prob, h0)
    assert rel_inf(all_y(res, 1, 2), y_ref) < 1e-12
    assert rel_inf(res["final"].reshape(fin_ref.shape), fin_ref) < 1e-12


def pad_problem(prob, Tp):
    """The problem extended to Tp tokens with a = 0 and x = B = C = 0 past T:
    the reading of a partial last chunk (tokens past T decay by 1 and carry no
    input and no readout)."""
    T = prob.x.shape[1]
    def ext(arr):
        w = [(0, 0)] * arr.ndim
        w[1] = (0, Tp - T)
        return np.pad(arr, w)
    return O.Problem(ext(prob.x), ext(prob.a), ext(prob.Bm), ext(prob.Cm), prob.D)


@pytest.mark.parametrize("per_state", [False, True])
@pytest.mark.parametrize("T,q", [(13, 4), (30, 8), (7, 16)])
def test_zero_padding_is_a_partial_last_chunk(per_state, T, q):
    """Padding past T with a = 0 and x = B = C = 0 leaves y[:T] and the final
    state of the recurrence exactly as they were (each padded step multiplies
    the state by e^0 = 1 and adds B x^T = 0), and the chunked form over the
    padded length agrees with the unpadded recurrence: the padded chunk count
    ceil(T / q) with a partial last chunk is the same operator."""
    rng = np.random.default_rng(61 + T + per_state)
    prob = random_problem(rng, B=2, T=T, H=3, P=4, G=1, N=5, per_state=per_state)
    B, _, H, _ = prob.x.shape
    Tp = -(-T // q) * q
    ref = O.recurrence(prob)
    padded = pad_problem(prob, Tp)
    rp = O.recurrence(padded)
    assert np.array_equal(all_y(rp, B, H)[:, :, :T], all_y(ref, B, H))
    assert np.array_equal(rp["final"], ref["final"])
    rc = O.chunked(padded, q)
    assert rel_inf(all_y(rc, B, H)[:, :, :T], all_y(ref, B, H)) < 1e-12
    assert rel_inf(rc["final"], ref["final"]) < 1e-12


def test_zero_initial_state_is_the_default():
    rng = np.random.default_rng(51)
    prob = random_problem(rng, B=2, T=9, H=2, P=3, G=2, N=4)
    a = O.recurrence(prob)
    b = O.recurrence(prob, initial=np.zeros((2, 2, 4, 3)))
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["final"], b["final"])


def test_discretize_softplus_identities():
    """softplus fixed by its definition log(1 + e^z): softplus(z) - softplus(-z)
    = z, softplus(0) = ln 2, softplus(z) -> z for large z and -> e^z for very
    negative z; a = dt * (-exp(A_log)) and xd = dt * x."""
    z = np.array([-40.0, -5.0, -0.3, 0.0, 0.7, 3.0, 25.0, 60.0])
    raw = z.reshape(1, -1, 1)
    _, _, dt_p = O.discretize(raw, None, np.zeros(1), np.ones((1, z.size, 1, 1)))
    _, _, dt_m = O.discretize(-raw, None, np.zeros(1), np.ones((1, z.size, 1, 1)))
    assert np.allclose(dt_p - dt_m, raw, rtol=0, atol=1e-13)
    assert abs(dt_p[0, 3, 0] - math.log(2.0)) < 1e-15
    assert abs(dt_p[0, 7, 0] - 60.0) < 1e-12
    assert abs(dt_p[0, 0, 0] / math.exp(-40.0) - 1.0) < 1e-12
    rng = np.random.default_rng(91)
    raw = rng.standard_normal((2, 5, 3))
    bias = rng.standard_normal(3)
    A_log = rng.uniform(0.0, 2.0, size=3)
    x = rng.standard_normal((2, 5, 3, 4))
    a, xd, dt = O.discretize(raw, bias, A_log, x)
    direct = np.log(1.0 + np.exp(raw + bias))
    assert np.allclose(dt, direct, rtol=1e-14, atol=0)
    assert np.allclose(a, -dt * np.exp(A_log), rtol=1e-15, atol=0)
    assert np.allclose(xd, dt[..., None] * x, rtol=1e-15, atol=0)
    a4, _, _ = O.discretize(raw, bias, np.tile(A_log[:, None], (1, 6)), x)
    assert a4.shape == (2, 5, 3, 6) and np.allclose(a4[..., 2], a, rtol=1e-15, atol=0)


def test_discretize_step_folds_into_the_input():
    """Bbar_t x_t = (Delta_t B_t) x_t: running the operator with the input
    scaled by dt equals running it with B scaled by dt (one group per head),
    and the decays are log(Abar) = dt * A (Abar = exp(Delta A))."""
    rng = np.random.default_rng(92)
    B_, T, H, P, N = 1, 20, 2, 3, 4
    raw = rng.standard_normal((B_, T, H))
    A_log = rng.uniform(-1.0, 1.0, size=H)
    x = rng.standard_normal((B_, T, H, P))
    Bm = rng.standard_normal((B_, T, H, N)) / 2
    Cm = rng.standard_normal((B_, T, H, N)) / 2
    a, xd, dt = O.discretize(raw, None, A_log, x)
    assert np.allclose(np.exp(a), np.exp(dt * -np.exp(A_log)[None, None, :]), rtol=1e-15, atol=0)
    r1 = O.recurrence(Problem(xd, a, Bm, Cm, None))
    Bbar = Bm * dt[..., None]          # G = H: each head's own B, scaled by its step
    r2 = O.recurrence(Problem(x, a, Bbar, Cm, None))
    assert rel_inf(r1["y"], r2["y"]) < 1e-12 and rel_inf(r1["final"], r2["final"]) < 1e-12
