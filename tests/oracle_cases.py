"""Small float64 problems and independent reference computations for pinning
the oracle.  None of these helpers calls the oracle or the CUDA library; each
computes a result that the pages or plain mathematics fix by another route.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from oracle.ssd_oracle import Problem


def random_problem(rng, B=1, T=12, H=2, P=3, G=1, N=4, per_state=False, a_scale=0.5,
                   with_D=True) -> Problem:
    x = rng.standard_normal((B, T, H, P))
    if per_state:
        a = -rng.uniform(0.0, a_scale, size=(B, T, H, N))
    else:
        a = -rng.uniform(0.0, a_scale, size=(B, T, H))
    Bm = rng.standard_normal((B, T, G, N)) / np.sqrt(N)
    Cm = rng.standard_normal((B, T, G, N)) / np.sqrt(N)
    D = rng.standard_normal(H) if with_D else None
    return Problem(x, a, Bm, Cm, D)


def all_y(res, B, H):
    """[C,T,P] per-chain output of the default chain order (b-major) -> [B,H,T,P]."""
    C, T, P = res["y"].shape
    return res["y"].reshape(B, H, T, P)


def rel_inf(a, b):
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


def causal_linear_attention(prob: Problem):
    """a == 0: y = tril(C B^T) X + D X, per (b, h) -- unnormalised causal
    linear attention ("State Space Duality": attention without a softmax)."""
    B, T, H, P = prob.x.shape
    G = prob.Bm.shape[2]
    y = np.zeros((B, H, T, P))
    for b in range(B):
        for h in range(H):
            g = h // (H // G)
            Cg, Bg = prob.Cm[b, :, g, :], prob.Bm[b, :, g, :]
            X = prob.x[b, :, h, :]
            y[b, h] = np.tril(Cg @ Bg.T) @ X
            if prob.D is not None:
                y[b, h] += prob.D[h] * X
    return y


def lti_kernel(alpha, beta, gamma, T):
    """Impulse response of a time-invariant SSM, K_j = sum_n gamma_n beta_n
    e^{alpha_n j} (llms.blog "Global Convolution": Kbar = (C Bbar, C Abar Bbar,
    ...), with Abar = diag(e^alpha))."""
    j = np.arange(T)[:, None]
    return (np.exp(alpha[None, :] * j) * (gamma * beta)[None, :]).sum(axis=1)


def causal_conv_direct(K, x):
    """y_t = sum_{s<=t} K_{t-s} x_s along axis 0 (numpy.convolve, truncated)."""
    T = x.shape[0]
    out = np.zeros_like(x)
    for p in range(x.shape[1]):
        out[:, p] = np.convolve(K, x[:, p])[:T]
    return out


def causal_conv_fft(K, x):
    """Same causal convolution through numpy's FFT (zero-padded to 2T)."""
    T = x.shape[0]
    L = 2 * T
    Kf = np.fft.rfft(K, L)
    Xf = np.fft.rfft(x, L, axis=0)
    return np.fft.irfft(Kf[:, None] * Xf, L, axis=0)[:T]


def exact_rational_brute(xq, lam, Bq, Cq, Dq):
    """Exact y for one chain with multiplicative decays lam_t = e^{a_t} given as
    Fractions: y_t = sum_{s<=t} (C_t . B_s) (prod_{k=s+1..t} lam_k) x_s + D x_t
    (llms.blog "The SSD Theoretical Equivalence", M_{i,j})."""
    T, P = len(xq), len(xq[0])
    N = len(Bq[0])
    y = []
    for t in range(T):
        row = [Dq * xq[t][p] for p in range(P)]
        for s in range(t + 1):
            prod = Fraction(1)
            for k in range(s + 1, t + 1):
                prod *= lam[k]
            cb = sum((Cq[t][n] * Bq[s][n] for n in range(N)), Fraction(0))
            for p in range(P):
                row[p] += cb * prod * xq[s][p]
        y.append(row)
    return y


def free_response(prob: Problem, h0):
    """Zero input (x == 0): the state only decays, h_t = exp(sum_{k<=t} a_k) o h0,
    so y_t[p] = sum_n C_t[n] exp(sum_{k<=t} a_k[n]) h0[n, p] -- the closed form of
    the unforced recurrence (llms.blog "The SSD Theoretical Equivalence", the
    state-space view with B x = 0).  Returns [B,H,T,P] and the final [B,H,N,P]."""
    B, T, H, P = prob.x.shape
    G, N = prob.Bm.shape[2], prob.Bm.shape[3]
    y = np.zeros((B, H, T, P))
    fin = np.zeros((B, H, N, P))
    for b in range(B):
        for h in range(H):
            g = h // (H // G)
            a = prob.a[b, :, h] if prob.a.ndim == 3 else prob.a[b, :, h, :]
            cum = np.cumsum(a, axis=0)  # inclusive: the decay of h0 up to and including t
            dec = np.exp(cum) if prob.a.ndim == 4 else np.exp(cum)[:, None] * np.ones((1, N))
            for t in range(T):
                y[b, h, t] = (prob.Cm[b, t, g, :] * dec[t]) @ h0[b, h]
            fin[b, h] = dec[T - 1][:, None] * h0[b, h]
    return y, fin
