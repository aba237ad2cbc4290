"""Brute-force unrolling of the selective scan, for tiny inputs (pure Python).

Independent of the oracle: instead of stepping the recurrence it writes every
output as the explicit sum over earlier (forward) or later (backward) tokens,

    y^f_t = sum_{s<=t} sum_n C_tn * exp(A_n * sum_{r=s+1..t} Delta_r) * Delta_s B_sn u_s
    y^b_t = sum_{s>=t} sum_n C_tn * exp(A_n * sum_{r=t..s-1}   Delta_r) * Delta_s B_sn u_s

(the products of Abar = exp(Delta A) over the skipped steps, section "Discretization
via Zero-Order Hold (ZOH)" and "2. The Bidirectional Mamba Block" of the page
"Vision Mamba Guide: Efficient Bidirectional SSM & VMamba"), plus D u_t per
direction, each output summed with math.fsum.  Delta is taken as given.
"""
import math


def bidir_ungated(u, delta, B, C, A, D, Bb=None, Cb=None):
    """One batch item.  u, delta: [L][Di]; B, C: [L][N]; A: [2][Di][N]; D: [2][Di].

    Returns y[L][Di] = y^f + y^b (no gate).  Bb/Cb: backward copies (default B, C).
    """
    Bb = B if Bb is None else Bb
    Cb = C if Cb is None else Cb
    L, Di, N = len(u), len(u[0]), len(B[0])
    y = [[0.0] * Di for _ in range(L)]
    for t in range(L):
        for d in range(Di):
            terms = [D[0][d] * u[t][d], D[1][d] * u[t][d]]
            for s in range(t + 1):                      # forward: earlier tokens
                gap = math.fsum(delta[r][d] for r in range(s + 1, t + 1))
                for n in range(N):
                    terms.append(C[t][n] * math.exp(A[0][d][n] * gap) * delta[s][d] * B[s][n] * u[s][d])
            for s in range(t, L):                       # backward: later tokens
                gap = math.fsum(delta[r][d] for r in range(t, s))
                for n in range(N):
                    terms.append(Cb[t][n] * math.exp(A[1][d][n] * gap) * delta[s][d] * Bb[s][n] * u[s][d])
            y[t][d] = math.fsum(terms)
    return y
