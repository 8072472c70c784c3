"""GPU parity of the backward (ssd_chunk_scan_bwd, through the C ABI) with the
oracle's fp64 backward on the same inputs (bf16 inputs rounded once, then
widened for the oracle).  Every gradient element is compared; the metric is
max|g - g_ref| / max|g_ref| per gradient tensor.  The CUDA-core path computes
in fp32 on the inputs as given, so its bound is the fp32 one, 1e-4; the
tensor-core path (bf16 shapes it covers) rounds its operands to bf16, so its
bound is the bf16 one, 5e-3."""
import numpy as np
import pytest
import torch

import oracle
from parity import record
from ssd_chunked_scan_02_b200 import ssd

TOL = 1e-4
TOL_TC = 5e-3
NAMES = ("dx", "ddt", "dA", "dB", "dC", "dD", "dinit")


def _uses_tc(x, B):
    b, L, H, P = x.shape
    dims = ssd.make_dims(b, L, H, P, B.shape[3], B.shape[2])
    return ssd.ssd_chunk_scan_bwd_uses_tensor_cores(dims, x.dtype)


def _inputs(seed, b, L, H, P, N, G, dtype, with_init, with_dfinal):
    g = torch.Generator().manual_seed(seed)
    t = lambda *s: torch.randn(*s, generator=g)
    inp = dict(
        x=t(b, L, H, P).to(dtype), dt=torch.nn.functional.softplus(t(b, L, H) - 1.0),
        A=-torch.exp(torch.rand(H, generator=g) * np.log(8.0)),
        B=(t(b, L, G, N) / np.sqrt(N)).to(dtype), C=(t(b, L, G, N) / np.sqrt(N)).to(dtype),
        D=t(H), init=(0.3 * t(b, H, P, N)) if with_init else None,
        dy=t(b, L, H, P).to(dtype), dfinal=t(b, H, P, N) if with_dfinal else None)
    return inp


def _run(name, seed, b, L, H, P, N, G, dtype, with_init=True, with_dfinal=True, want_tc=None):
    inp = _inputs(seed, b, L, H, P, N, G, dtype, with_init, with_dfinal)
    tc = _uses_tc(inp["x"], inp["B"])
    if want_tc is not None:
        assert tc == want_tc
    dev = {k: (v.cuda().contiguous() if v is not None else None) for k, v in inp.items()}
    out = ssd.ssd_chunk_scan_bwd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                                 dev["dy"], init_states=dev["init"], dfinal_states=dev["dfinal"])
    torch.cuda.synchronize()
    f = lambda v: None if v is None else v.double().numpy()
    ref = oracle.backward(f(inp["x"]), f(inp["dt"]), f(inp["A"]), f(inp["B"]), f(inp["C"]),
                          f(inp["D"]), f(inp["init"]), f(inp["dy"]), f(inp["dfinal"]))
    errs = {}
    for k in NAMES:
        got = out[k].double().cpu().numpy()
        r = ref[k]
        scale = float(np.abs(r).max()) if r.size else 0.0
        errs[k] = float(np.abs(got - r).max() / scale) if scale > 0 else float(np.abs(got).max() if got.size else 0.0)
    record("bwd_" + name, **errs)
    assert max(errs.values()) <= (TOL_TC if tc == 1 else TOL), errs
    return out, ref


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("G,with_init,with_dfinal", [(2, True, True), (1, False, True), (2, True, False)])
def test_backward_small(dtype, G, with_init, with_dfinal):
    # 150 tokens: two whole 64-token checkpoint segments and a ragged third
    _run(f"small_G{G}_{int(with_init)}{int(with_dfinal)}_{str(dtype)[6:]}", 71 + G, 2, 150, 4,
         16, 32, G, dtype, with_init, with_dfinal)


@pytest.mark.gpu
def test_backward_layer_states():
    # the layers' P 64 x N 128 (tensor cores in bf16; in fp32 8 row blocks of
    # 8 rows on the CUDA cores), and P 128 x N 128
    _run("P64_N128", 81, 1, 130, 2, 64, 128, 1, torch.bfloat16, want_tc=1)
    _run("P128_N128", 84, 1, 70, 2, 128, 128, 2, torch.bfloat16, want_tc=1)
    _run("P64_N128_f32", 81, 1, 130, 2, 64, 128, 1, torch.float32, want_tc=0)


# Tensor-core backward: 128-token chunks, ragged tails, groups, odd heads per
# group, headdim 64 k (k heads of 64 sharing dt, A, D), dstate 64 and 128,
# with and without the initial and final states' gradients.
TC_CASES = [
    # name,          seed, b, L,   H, P,   N,   G, init,  dfinal
    ("L300_G1",        91, 2, 300, 4, 64,  128, 1, True,  True),
    ("L256_N64_G2",    92, 2, 256, 4, 64,  64,  2, True,  False),
    ("L130_odd_heads", 93, 1, 130, 3, 64,  128, 1, False, True),
    ("L200_P128",      94, 1, 200, 2, 128, 128, 1, True,  True),
    ("L129_P192_G3",   95, 1, 129, 6, 192, 64,  3, False, False),
    ("L1",             96, 2, 1,   2, 64,  128, 1, True,  True),
    ("L640_H8_G2",     97, 1, 640, 8, 64,  128, 2, True,  True),
    ("L300_P32",       98, 2, 300, 4, 32,  128, 1, True,  True),
    ("L200_P32_N64_G2", 99, 1, 200, 4, 32, 64,  2, False, True),
    ("L260_P256",     100, 1, 260, 2, 256, 128, 1, True,  True),
    ("L300_P128_N64_G2", 102, 2, 300, 4, 128, 64, 2, True, False),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", TC_CASES, ids=[c[0] for c in TC_CASES])
def test_backward_tensor_cores(case):
    name, seed, b, L, H, P, N, G, wi, wf = case
    _run("tc_" + name, seed, b, L, H, P, N, G, torch.bfloat16, wi, wf, want_tc=1)


@pytest.mark.gpu
def test_backward_tensor_cores_130m_layer():
    """The 130M-layer shape (b 8, L 2048, H 24, P 64, N 128), the bench's
    backward workload, on the tensor cores: every gradient element against
    the oracle (about 15 s of fp64 on the host)."""
    _run("tc_130m_layer", 101, 8, 2048, 24, 64, 128, 1, torch.bfloat16, True, True, want_tc=1)


@pytest.mark.gpu
def test_backward_odd_sizes_single_token():
    _run("odd_L1", 82, 3, 1, 3, 5, 7, 1, torch.float32)
    _run("odd_L65", 83, 1, 65, 6, 12, 20, 3, torch.bfloat16)


@pytest.mark.gpu
def test_backward_no_tokens():
    # L = 0: the initial state's gradient is the final state's; the rest is zero
    b, H, P, N, G = 2, 4, 8, 16, 2
    x = torch.zeros(b, 0, H, P, device="cuda", dtype=torch.bfloat16)
    dt = torch.zeros(b, 0, H, device="cuda")
    Bm = torch.zeros(b, 0, G, N, device="cuda", dtype=torch.bfloat16)
    A = -torch.ones(H, device="cuda")
    D = torch.ones(H, device="cuda")
    dfinal = torch.randn(b, H, P, N, device="cuda")
    out = ssd.ssd_chunk_scan_bwd(x, dt, A, Bm, Bm, D, x, dfinal_states=dfinal)
    torch.cuda.synchronize()
    assert torch.equal(out["dinit"], dfinal)
    assert float(out["dA"].abs().max()) == 0.0 and float(out["dD"].abs().max()) == 0.0


@pytest.mark.gpu
def test_backward_rejects_oversized_state():
    x = torch.zeros(1, 4, 1, 64, device="cuda", dtype=torch.bfloat16)
    Bm = torch.zeros(1, 4, 1, 512, device="cuda", dtype=torch.bfloat16)
    dt = torch.zeros(1, 4, 1, device="cuda")
    one = torch.ones(1, device="cuda")
    with pytest.raises(ssd.SSDError) as e:
        ssd.ssd_chunk_scan_bwd(x, dt, one, Bm, Bm, one, x)
    assert e.value.status == ssd.SSD_ERR_UNSUPPORTED
