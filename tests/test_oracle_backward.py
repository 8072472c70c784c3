"""Pins of the oracle's backward (the gradients of the recurrence), CPU only.

The reference for every gradient is a central finite difference of the
oracle's *forward* recurrence, which shares none of the backward's formulas:
a dropped term, a wrong sign, a state taken one token late or a gradient not
summed over a group's heads moves some derivative far outside the tolerance
(the mutants below plant exactly such mistakes and must be caught).  The
closed forms fix the skip path and the zero-readout case."""
import os
import subprocess

import numpy as np
import pytest

import oracle

TOL = 1e-6   # relative to the largest finite-difference derivative (observed ~1e-9)


def _inputs(seed, b=2, L=7, H=4, P=3, N=5, G=2, with_init=True):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((b, L, H, P)),
        dt=np.log1p(np.exp(rng.normal(-1.0, 0.5, (b, L, H)))),
        A=-np.exp(rng.uniform(0.0, np.log(4.0), H)),
        B=rng.standard_normal((b, L, G, N)),
        C=rng.standard_normal((b, L, G, N)),
        D=rng.standard_normal(H),
        init=0.3 * rng.standard_normal((b, H, P, N)) if with_init else None,
    ), rng.standard_normal((b, L, H, P)), rng.standard_normal((b, H, P, N))


def _finite_differences(inp, dy, dfinal, names):
    def loss(**kw):
        a = dict(inp)
        a.update(kw)
        y, f = oracle.recurrence(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["init"])
        return float((y * dy).sum() + (0.0 if dfinal is None else (f * dfinal).sum()))

    out = {}
    for name in names:
        arr = inp[name]
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            e = 1e-6 * max(1.0, abs(arr[idx]))
            ap, am = arr.copy(), arr.copy()
            ap[idx] += e
            am[idx] -= e
            num[idx] = (loss(**{name: ap}) - loss(**{name: am})) / (2 * e)
        out[name] = num
    return out


GRAD = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "init": "dinit"}


def _check_fd(bwd, seed, G, with_init, with_dfinal):
    inp, dy, dfinal = _inputs(seed, G=G, with_init=with_init)
    if not with_dfinal:
        dfinal = None
    g = bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"], dy, dfinal)
    names = [n for n in GRAD if inp[n] is not None]
    num = _finite_differences(inp, dy, dfinal, names)
    errs = {}
    for n in names:
        ref = num[n]
        errs[n] = float(np.abs(g[GRAD[n]] - ref).max() / max(np.abs(ref).max(), 1e-30))
    return errs


@pytest.mark.parametrize("G,with_init,with_dfinal", [(1, True, True), (2, True, False),
                                                      (2, False, True), (1, False, False)])
def test_backward_matches_finite_differences(G, with_init, with_dfinal):
    errs = _check_fd(oracle.backward, 11 + G, G, with_init, with_dfinal)
    assert max(errs.values()) < TOL, errs


def test_backward_gradient_of_zero_initial_state():
    # with init=None the returned dinit is the gradient at a zero initial state:
    # the same as passing explicit zeros
    inp, dy, dfinal = _inputs(5, with_init=False)
    a = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], None, dy, dfinal)
    z = np.zeros_like(dfinal)
    b = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], z, dy, dfinal)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])


def test_skip_gradient_closed_form():
    # dL/dD_h = sum over batch, tokens and p of dy * x, whatever the SSM term does
    inp, dy, dfinal = _inputs(7)
    g = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"], dy, dfinal)
    np.testing.assert_allclose(g["dD"], (dy * inp["x"]).sum(axis=(0, 1, 3)), rtol=1e-13, atol=1e-13)


def test_zero_readout_closed_form():
    # C = 0 and no final-state gradient: the state never reaches the loss, so
    # dB, ddt, dA and dinit vanish and dx is the skip term's D_h dy
    inp, dy, _ = _inputs(9)
    inp["C"] = np.zeros_like(inp["C"])
    g = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["init"], dy, None)
    for k in ("dB", "ddt", "dA", "dinit"):
        assert np.abs(g[k]).max() == 0.0, k
    np.testing.assert_allclose(g["dx"], inp["D"][None, None, :, None] * dy, rtol=0, atol=0)


# (name, exact text in ssd_oracle.c's backward, replacement)
SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")
MUTANTS = [
    ("ddt_without_decay_term", "ddt[(b * L + t) * H + h] = xgb + A[h] * at * gs;",
     "ddt[(b * L + t) * H + h] = xgb;"),
    ("state_gradient_not_decayed", "for (int64_t k = 0; k < PN; ++k) Gm[k] *= at;",
     "for (int64_t k = 0; k < PN; ++k) Gm[k] *= 1.0;"),
    ("dB_missing_dt", "dBt[n] += dtv * Gm[p * N + n] * xt[p];", "dBt[n] += Gm[p * N + n] * xt[p];"),
    ("decay_term_uses_current_state", "gs += Gm[p * N + n] * Sp[p * N + n];",
     "gs += Gm[p * N + n] * St[p * N + n];"),
    ("dC_uses_previous_state", "dCt[n] += St[p * N + n] * dyt[p];", "dCt[n] += Sp[p * N + n] * dyt[p];"),
    ("dA_missing_dt", "dA_part[h] += dtv * at * gs;", "dA_part[h] += at * gs;"),
    ("final_gradient_ignored", "    if (dfinal != NULL)\n        memcpy(Gm", "    if (0)\n        memcpy(Gm"),
    ("dx_missing_skip", "dxt[p] = D[h] * dyt[p] + dtv * gb;", "dxt[p] = dtv * gb;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_backward_pins_catch_mutant(tmp_path, name, old, new):
    with open(SRC) as f:
        source = f.read()
    assert source.count(old) == 1, f"mutation site for {name} not unique in ssd_oracle.c"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", str(lib),
                    str(src), "-lm"], check=True)
    bwd = oracle.backward_from(str(lib))
    worst = 0.0
    for G, with_init, with_dfinal in [(2, True, True)]:
        errs = _check_fd(bwd, 11 + G, G, with_init, with_dfinal)
        worst = max(worst, max(errs.values()))
    assert worst > 100 * TOL, f"no pin caught the planted mistake '{name}' (worst error {worst:.2e})"
