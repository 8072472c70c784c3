"""The block-decomposed (chunked) form of the backward, written out in numpy
and checked against the oracle's token-by-token backward (CPU only).  It
fixes the per-chunk formulas a tensor-core backward computes: the reverse
pass over chunks of dL/dh, the masked products for dx, dB and dC, and the
decay gradient taken through the prefix sums; any dropped term, wrong mask
side or mis-scaled decay moves some gradient far off the 1e-12 bound."""
import numpy as np
import pytest

import oracle


def chunked_bwd(x, dt, A, B, C, D, init, dy, dfinal, Q):
    L, P = x.shape; N = B.shape[1]
    T = (L + Q - 1) // Q
    # forward pieces: per-chunk log decays cs (inclusive), entering states
    hs = []  # state entering each chunk
    h = init.copy()
    cs_all = []
    for c in range(T):
        s0, s1 = c * Q, min(L, c * Q + Q)
        cs = np.cumsum(dt[s0:s1] * A)
        cs_all.append(cs)
        hs.append(h.copy())
        S = np.exp(cs[-1]) * h
        for j in range(s0, s1):
            S = S + np.exp(cs[-1] - cs[j - s0]) * dt[j] * np.outer(x[j], B[j])
        h = S
    # (i) per-chunk dstate: sum_k e^{cs_k} dy_k C_k^T ; (ii) reverse pass over chunks
    Gam = [None] * T                     # dL/dh_c (state after chunk c)
    g = dfinal.copy()
    for c in range(T - 1, -1, -1):
        Gam[c] = g.copy()
        s0, s1 = c * Q, min(L, c * Q + Q)
        cs = cs_all[c]
        dstate = sum(np.exp(cs[k - s0]) * np.outer(dy[k], C[k]) for k in range(s0, s1))
        g = np.exp(cs[-1]) * g + dstate
    dinit = g
    dx = np.zeros_like(x); dB = np.zeros_like(B); dC = np.zeros_like(C); ddt = np.zeros_like(dt)
    dA = 0.0; dD = float((dy * x).sum())
    for c in range(T):
        s0, s1 = c * Q, min(L, c * Q + Q)
        cs = cs_all[c]; n = s1 - s0
        X, Y, Bc, Cc, dtc = x[s0:s1], dy[s0:s1], B[s0:s1], C[s0:s1], dt[s0:s1]
        hp, Gc = hs[c], Gam[c]
        # decay matrix E[i, j] = e^{cs_i - cs_j} for j <= i (else 0)
        E = np.where(np.tri(n, dtype=bool), np.exp(cs[:, None] - cs[None, :]), 0.0)
        el = np.exp(cs[-1] - cs)          # decay from token j to the chunk's end
        ei = np.exp(cs)                   # decay from the chunk's start to token i
        CB = Cc @ Bc.T                    # (C_i . B_j)
        # dx_j = D dy_j + dt_j [ el_j (Gam B_j) + sum_{i>=j} (C_i.B_j) E[i,j] dy_i ]
        GB = (Gc @ Bc.T).T                # rows j: Gam B_j  (P)
        dxc = D * Y + dtc[:, None] * (el[:, None] * GB + (CB * E).T @ Y)
        # dB_j = dt_j [ el_j Gam^T x_j + sum_{i>=j} E[i,j] (dy_i . x_j) C_i ]
        YX = Y @ X.T                      # (dy_i . x_j)
        dBc = dtc[:, None] * (el[:, None] * (X @ Gc) + (YX * E).T @ Cc)
        # dC_i = e^{cs_i} h_prev^T dy_i + sum_{j<=i} E[i,j] dt_j (x_j . dy_i) B_j
        dCc = ei[:, None] * (Y @ hp) + (YX * E * dtc[None, :]) @ Bc
        # decay gradients: dL/dcs through every e^{cs} factor.  Per token pair
        # (i, j<=i) the intra term y_i += CB_ij e^{cs_i - cs_j} dt_j x_j gives
        # d/dcs_i += w_ij, d/dcs_j -= w_ij with w_ij = CB_ij E_ij dt_j (dy_i . x_j);
        # the entering state gives d/dcs_i += e^{cs_i} dy_i^T h_prev C_i; the
        # state handed on gives d/dcs_last += <Gam, h_c>, d/dcs_j -= el_j dt_j x_j^T Gam B_j.
        W = CB * E * dtc[None, :] * YX
        dcs = W.sum(axis=1) - W.sum(axis=0)
        dcs += ei * np.einsum('ip,pn,in->i', Y, hp, Cc)
        dcs[-1] += np.sum(Gc * (np.exp(cs[-1]) * hp + sum(el[j] * dtc[j] * np.outer(X[j], Bc[j]) for j in range(n))))
        dcs -= el * dtc * np.einsum('jp,pn,jn->j', X, Gc, Bc)
        # cs_i = sum_{k<=i} dt_k A  =>  dL/d(dt_k A) = sum_{i>=k} dcs_i  (reverse cumsum)
        ddA = np.cumsum(dcs[::-1])[::-1]
        # input scaling by dt_j: dt_j appears in w_ij, in the chunk state term and dx's
        din = (CB * E * YX).sum(axis=0)                        # sum_i CB_ij E_ij (dy_i.x_j)
        din += el * np.einsum('jp,pn,jn->j', X, Gc, Bc)
        ddtc = din + A * ddA
        dA += float((ddA * dtc).sum())
        dx[s0:s1], dB[s0:s1], dC[s0:s1], ddt[s0:s1] = dxc, dBc, dCc, ddtc
    return dict(dx=dx, ddt=ddt, dA=dA, dB=dB, dC=dC, dD=dD, dinit=dinit)



@pytest.mark.parametrize("L,P,N,Q", [(37, 3, 5, 8), (64, 4, 6, 16), (10, 2, 3, 4), (9, 2, 2, 32)])
def test_chunked_backward_equals_the_recurrence_backward(L, P, N, Q):
    rng = np.random.default_rng(L * 7 + Q)
    x = rng.standard_normal((L, P))
    dt = np.log1p(np.exp(rng.normal(-1, .5, L)))
    A, D = -1.3, 0.7
    B = rng.standard_normal((L, N))
    C = rng.standard_normal((L, N))
    init = rng.standard_normal((P, N))
    dy = rng.standard_normal((L, P))
    df = rng.standard_normal((P, N))
    got = chunked_bwd(x, dt, A, B, C, D, init, dy, df, Q)
    ref = oracle.backward(x[None, :, None], dt[None, :, None], np.array([A]), B[None, :, None],
                          C[None, :, None], np.array([D]), init[None, None], dy[None, :, None],
                          df[None, None])
    for k in got:
        r = np.squeeze(ref[k])
        g = np.squeeze(np.asarray(got[k]))
        assert np.abs(g - r).max() <= 1e-12 * max(np.abs(r).max(), 1e-30), k
