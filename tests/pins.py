"""Pins for the fp64 oracle: checks against results fixed by the mathematics,
not by the oracle itself.  Each pin takes a recurrence callable
``rec(x, dt, A, B, C, D, init) -> (y, final)`` (float64 numpy in and out) so
the same pins run against the real oracle and against deliberately broken
copies of it (tests/test_oracle_mutants.py).

Pins and what they fix:
  semiseparable   the duality: y = M x + D x + (decayed initial state) with the
                  1-semiseparable matrix M[i,j] = C_i.B_j exp(sum_{k=j+1..i} dt_k A) dt_j
                  materialised entry by entry (sums taken directly, not as cumsum
                  differences) -- "Transformers are SSMs" (CiteArk), AI research
                  summary and "what this means" (1-semiseparable SSM = structured
                  masked attention); review page, 核心概念 items 2-3.
  a_zero          A = 0 makes every decay 1: the state is a cumulative sum.
  dta_neg_inf     dt*A -> -inf (A = -1e6): no memory, y_t = dt_t (C_t.B_t) x_t + D x_t.
  c_zero          C = 0 leaves only the skip term: y = D x exactly.
  init_only       x = 0, D = 0: y_t = exp(sum_{k<=t} dt_k A) C_t . h0.
  scalar_brute    P = N = 1, L <= 4: products expanded by hand.
  geometric       constant inputs: y_t = c b dt x (1 - a^{t+1}) / (1 - a) + D x.
  group_map       ngroups = 2: heads 0..H/2-1 read group 0, the rest group 1.
  resume          running halves with the first half's final state as the
                  second half's initial state equals one run.
"""
from __future__ import annotations

import math

import numpy as np


def _rand_case(rng, b, L, H, P, N, G, with_init, A_scale=1.0):
    x = rng.standard_normal((b, L, H, P))
    dt = np.log1p(np.exp(rng.normal(-2.0, 0.7, size=(b, L, H))))
    A = -np.exp(rng.uniform(0.0, math.log(16.0), size=H)) * A_scale
    B = rng.standard_normal((b, L, G, N)) / math.sqrt(N)
    C = rng.standard_normal((b, L, G, N)) / math.sqrt(N)
    D = rng.standard_normal(H)
    init = 0.3 * rng.standard_normal((b, H, P, N)) if with_init else None
    return x, dt, A, B, C, D, init


def _rel(a, b):
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def semiseparable_reference(x, dt, A, B, C, D, init):
    """y and final state from the materialised semiseparable matrix (O(L^2))."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros_like(x)
    final = np.zeros((b, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h * G // H
            M = np.zeros((L, L))
            for i in range(L):
                for j in range(i + 1):
                    s = 0.0
                    for k in range(j + 1, i + 1):
                        s += dt[bi, k, h] * A[h]
                    M[i, j] = float(np.dot(C[bi, i, g], B[bi, j, g])) * math.exp(s) * dt[bi, j, h]
            y[bi, :, h, :] = M @ x[bi, :, h, :] + D[h] * x[bi, :, h, :]
            # final state: sum_j exp(sum_{k=j+1..L-1} dt_k A) dt_j x_j B_j^T
            for j in range(L):
                s = 0.0
                for k in range(j + 1, L):
                    s += dt[bi, k, h] * A[h]
                final[bi, h] += math.exp(s) * dt[bi, j, h] * np.outer(x[bi, j, h], B[bi, j, g])
            if init is not None:
                for i in range(L):
                    s = 0.0
                    for k in range(0, i + 1):
                        s += dt[bi, k, h] * A[h]
                    y[bi, i, h] += math.exp(s) * (init[bi, h] @ C[bi, i, g])
                s = float(np.sum(dt[bi, :, h] * A[h]))
                final[bi, h] += math.exp(s) * init[bi, h]
    return y, final


def pin_semiseparable(rec, seed=0):
    rng = np.random.default_rng(seed)
    for (b, L, H, P, N, G, with_init) in [(1, 1, 1, 1, 1, 1, False), (2, 17, 4, 3, 5, 1, False),
                                          (1, 40, 4, 2, 3, 2, True), (2, 9, 2, 4, 4, 2, True)]:
        args = _rand_case(rng, b, L, H, P, N, G, with_init)
        y, f = rec(*args)
        y_ref, f_ref = semiseparable_reference(*args)
        assert _rel(y, y_ref) < 1e-12, ("semiseparable y", b, L, H, P, N, G, _rel(y, y_ref))
        assert _rel(f, f_ref) < 1e-12, ("semiseparable final", _rel(f, f_ref))


def pin_a_zero(rec, seed=1):
    rng = np.random.default_rng(seed)
    x, dt, A, B, C, D, init = _rand_case(rng, 2, 33, 3, 4, 6, 1, True)
    A = np.zeros_like(A)
    y, f = rec(x, dt, A, B, C, D, init)
    # S_t = h0 + sum_{s<=t} dt_s x_s B_s^T  (cumulative sum), y_t = S_t C_t + D x_t
    contrib = np.einsum("blh,blhp,bln->blhpn", dt, x, B[:, :, 0, :])
    S = np.cumsum(contrib, axis=1) + init[:, None]
    y_ref = np.einsum("blhpn,bln->blhp", S, C[:, :, 0, :]) + D[None, None, :, None] * x
    assert _rel(y, y_ref) < 1e-12, ("a_zero y", _rel(y, y_ref))
    assert _rel(f, S[:, -1]) < 1e-12, ("a_zero final", _rel(f, S[:, -1]))


def pin_dta_neg_inf(rec, seed=2):
    rng = np.random.default_rng(seed)
    x, dt, A, B, C, D, init = _rand_case(rng, 2, 21, 3, 4, 5, 1, True)
    A = np.full_like(A, -1.0e6)
    y, f = rec(x, dt, A, B, C, D, init)
    cb = np.einsum("bln,bln->bl", C[:, :, 0, :], B[:, :, 0, :])
    y_ref = (dt * cb[:, :, None])[..., None] * x + D[None, None, :, None] * x
    f_ref = np.einsum("bh,bhp,bn->bhpn", dt[:, -1], x[:, -1], B[:, -1, 0, :])
    assert _rel(y, y_ref) < 1e-13, ("dta_neg_inf y", _rel(y, y_ref))
    assert _rel(f, f_ref) < 1e-13, ("dta_neg_inf final", _rel(f, f_ref))


def pin_c_zero(rec, seed=3):
    rng = np.random.default_rng(seed)
    x, dt, A, B, C, D, init = _rand_case(rng, 1, 19, 2, 3, 4, 1, True)
    C = np.zeros_like(C)
    y, _ = rec(x, dt, A, B, C, D, init)
    assert np.array_equal(y, D[None, None, :, None] * x), "c_zero: y must equal D*x exactly"


def pin_init_only(rec, seed=4):
    rng = np.random.default_rng(seed)
    x, dt, A, B, C, D, init = _rand_case(rng, 2, 25, 3, 2, 3, 1, True)
    x = np.zeros_like(x)
    D = np.zeros_like(D)
    y, f = rec(x, dt, A, B, C, D, init)
    logdecay = np.cumsum(dt * A[None, None, :], axis=1)            # sum_{k<=t} dt_k A
    y_ref = np.exp(logdecay)[..., None] * np.einsum("bhpn,bln->blhp", init, C[:, :, 0, :])
    f_ref = np.exp(logdecay[:, -1])[..., None, None] * init
    assert _rel(y, y_ref) < 1e-12, ("init_only y", _rel(y, y_ref))
    assert _rel(f, f_ref) < 1e-12, ("init_only final", _rel(f, f_ref))


def pin_scalar_brute(rec):
    # P = N = 1, one head, L = 4, written out term by term.
    dt = [0.5, 0.25, 1.0, 0.125]
    xs = [1.0, -2.0, 0.5, 3.0]
    bs = [0.5, 1.5, -1.0, 2.0]
    cs = [2.0, -0.5, 1.0, 0.25]
    A0, D0, h0 = -0.75, 0.3, 0.4
    a = [math.exp(d * A0) for d in dt]
    h1 = a[0] * h0 + dt[0] * xs[0] * bs[0]
    h2 = a[1] * h1 + dt[1] * xs[1] * bs[1]
    h3 = a[2] * h2 + dt[2] * xs[2] * bs[2]
    h4 = a[3] * h3 + dt[3] * xs[3] * bs[3]
    # the same states, fully expanded as sums of decayed inputs
    h4_expanded = (a[0] * a[1] * a[2] * a[3] * h0
                   + a[1] * a[2] * a[3] * dt[0] * xs[0] * bs[0]
                   + a[2] * a[3] * dt[1] * xs[1] * bs[1]
                   + a[3] * dt[2] * xs[2] * bs[2]
                   + dt[3] * xs[3] * bs[3])
    assert abs(h4 - h4_expanded) < 1e-14
    y_ref = np.array([cs[0] * h1, cs[1] * h2, cs[2] * h3, cs[3] * h4]) + D0 * np.array(xs)
    shp = (1, 4, 1, 1)
    y, f = rec(np.array(xs).reshape(shp), np.array(dt).reshape(1, 4, 1), np.array([A0]),
               np.array(bs).reshape(shp), np.array(cs).reshape(shp), np.array([D0]),
               np.array([h0]).reshape(1, 1, 1, 1))
    assert np.max(np.abs(y.reshape(4) - y_ref)) < 1e-14, ("scalar_brute y", y.reshape(4), y_ref)
    assert abs(float(f.reshape(())) - h4_expanded) < 1e-14, "scalar_brute final"


def pin_geometric(rec):
    L, dtv, A0, xv, bv, cv, D0 = 300, 0.05, -2.0, 1.5, 0.7, -1.3, 0.25
    a = math.exp(dtv * A0)
    shp = (1, L, 1, 1)
    y, f = rec(np.full(shp, xv), np.full((1, L, 1), dtv), np.array([A0]), np.full(shp, bv),
               np.full(shp, cv), np.array([D0]), None)
    t = np.arange(L)
    y_ref = cv * bv * dtv * xv * (1.0 - a ** (t + 1)) / (1.0 - a) + D0 * xv
    assert _rel(y.reshape(L), y_ref) < 1e-12, ("geometric", _rel(y.reshape(L), y_ref))
    f_ref = bv * dtv * xv * (1.0 - a ** L) / (1.0 - a)
    assert abs(float(f.reshape(())) - f_ref) < 1e-12 * abs(f_ref)


def pin_group_map(rec, seed=5):
    rng = np.random.default_rng(seed)
    x, dt, A, B, C, D, init = _rand_case(rng, 1, 13, 4, 2, 3, 2, False)
    B[:, :, 1, :] = 0.0          # group 1 has no input path ...
    C[:, :, 1, :] = 0.0          # ... and no readout
    y, _ = rec(x, dt, A, B, C, D, init)
    skip = D[None, None, :, None] * x
    # heads 2,3 (group 1) see only the skip term; heads 0,1 (group 0) see more
    assert np.array_equal(y[:, :, 2:], skip[:, :, 2:]), "group_map: heads 2,3 must read group 1"
    assert np.max(np.abs(y[:, :, :2] - skip[:, :, :2])) > 1e-3, "group_map: heads 0,1 read group 0"


def pin_resume(rec, seed=6):
    rng = np.random.default_rng(seed)
    x, dt, A, B, C, D, init = _rand_case(rng, 2, 30, 3, 4, 5, 1, True)
    y, f = rec(x, dt, A, B, C, D, init)
    h = 11
    y1, f1 = rec(x[:, :h], dt[:, :h], A, B[:, :h], C[:, :h], D, init)
    y2, f2 = rec(x[:, h:], dt[:, h:], A, B[:, h:], C[:, h:], D, f1)
    assert _rel(np.concatenate([y1, y2], axis=1), y) < 1e-13, "resume y"
    assert _rel(f2, f) < 1e-13, "resume final"


ALL_PINS = [pin_semiseparable, pin_a_zero, pin_dta_neg_inf, pin_c_zero, pin_init_only,
            pin_scalar_brute, pin_geometric, pin_group_map, pin_resume]


def run_all(rec):
    """Run every pin; return the list of (name, error) that failed."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(rec)
        except AssertionError as e:  # noqa: PERF203
            failed.append((pin.__name__, repr(e)))
    return failed
