"""CUDA path vs the fp64 oracle, element by element, on the same seeded inputs.

Error metric (per tensor): max|gpu - oracle| / max|oracle|; bound 5e-3 for
bf16 storage, 1e-4 for fp32.  Small cases compare every element; the full
workload sizes compare sampled (batch, head) pairs, each recomputed by the
oracle over the whole sequence."""

import numpy as np
import pytest
import torch

import oracle
from parity import TOL, gpu_fwd, oracle_fwd, oracle_pairs, record, rel_err, sample_pairs, to_dev
from ssd_chunked_scan_02_b200 import inputs, ssd

pytestmark = pytest.mark.gpu


def _w(name, b, L, H, P, N, G, Q, dtype, init, seed):
    return inputs.Workload(name, b, L, H, P, N, G, Q, dtype, with_init=init, want_final=True,
                           seed=seed)


def _check_full(w, chunk=None, flow=None):
    inp = inputs.make_inputs(w)
    y, f = gpu_fwd(inp, chunk or w.chunk, flow=flow)
    y_ref, f_ref = oracle_fwd(inp)
    tol = TOL[w.dtype]
    ey, ef = rel_err(y, y_ref), rel_err(f, f_ref)
    record(f"{w.name}_Q{chunk or w.chunk}", y=ey, final=ef)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(f))
    assert ey <= tol, f"{w.name} Q={chunk or w.chunk}: y rel err {ey:.3g} > {tol}"
    assert ef <= tol, f"{w.name} Q={chunk or w.chunk}: final rel err {ef:.3g} > {tol}"
    return ey, ef


def test_tiny_f32_workload_full():
    _check_full(inputs.TINY_F32)


SMALL_BF16 = [
    # name,               b,  L,   H,  P,  N,  G,  Q,  init
    ("bf16_ragged_q256", 2, 600, 4, 64, 128, 1, 256, True),
    ("bf16_ragged_q128", 2, 600, 4, 64, 128, 1, 128, True),
    ("bf16_q64", 2, 300, 4, 64, 128, 1, 64, True),
    ("bf16_n64_groups2", 1, 1000, 6, 64, 64, 2, 256, False),
    ("bf16_short_L_lt_Q", 1, 17, 2, 64, 128, 1, 256, True),
    ("bf16_single_token", 2, 1, 2, 64, 128, 1, 256, True),
    ("bf16_odd_dims", 3, 513, 2, 32, 48, 1, 128, True),
    ("bf16_exact_chunks", 2, 1024, 8, 64, 128, 1, 256, True),
]


# shapes the tensor cores cover through virtual heads (headdim 64 k), phantom
# heads (an odd number of heads per group) and 128-token chunks for smaller
# chunk sizes, through both tensor-core data flows
TC_SHAPES = [
    # name,                     b,  L,   H,  P,   N,  G,  Q,  init
    ("tc_p128_three_kernel", 2, 600, 4, 128, 128, 1, 256, True),
    ("tc_p128_walk_n64", 8, 700, 24, 128, 64, 2, 128, True),
    ("tc_p192_odd_virtual", 2, 400, 3, 192, 64, 1, 128, True),
    ("tc_p256", 1, 500, 2, 256, 128, 1, 256, True),
    ("tc_odd_hpg_three_kernel", 2, 600, 6, 64, 128, 2, 256, True),
    ("tc_odd_hpg_n64_three_kernel", 1, 700, 10, 64, 64, 2, 128, True),
    ("tc_odd_hpg_walk", 16, 600, 10, 64, 128, 2, 256, True),
    ("tc_odd_hpg_walk_n64", 48, 300, 3, 64, 64, 1, 128, False),
    ("tc_q32_runs_q128", 2, 333, 4, 64, 128, 1, 32, True),
    ("tc_q16_ragged", 1, 77, 2, 64, 64, 1, 16, True),
    # headdim 32: a head of 64 with 32 zero columns, internal states padded
    ("tc_p32_three_kernel", 2, 600, 4, 32, 128, 1, 256, True),
    ("tc_p32_walk", 16, 500, 12, 32, 128, 2, 128, True),
    ("tc_p32_walk_n64_odd_hpg", 48, 300, 3, 32, 64, 1, 256, True),
    ("tc_p32_n64_groups2_q64", 2, 333, 6, 32, 64, 2, 64, False),
]


@pytest.mark.parametrize("case", TC_SHAPES, ids=[c[0] for c in TC_SHAPES])
def test_tensor_core_shapes(case):
    name, b, L, H, P, N, G, Q, init = case
    dims = ssd.make_dims(b, L, H, P, N, G)
    assert ssd.ssd_chunk_scan_fwd_uses_tensor_cores(dims, Q, torch.bfloat16) == 1
    _check_full(_w(name, b, L, H, P, N, G, Q, "bf16", init, seed=120 + len(name)))


@pytest.mark.parametrize("case", SMALL_BF16, ids=[c[0] for c in SMALL_BF16])
def test_small_bf16(case):
    name, b, L, H, P, N, G, Q, init = case
    _check_full(_w(name, b, L, H, P, N, G, Q, "bf16", init, seed=100 + len(name)))


SMALL_F32 = [
    ("f32_ragged", 2, 333, 3, 16, 16, 1, 64, True),
    ("f32_tiny_dims", 1, 256, 4, 3, 5, 1, 32, True),
    ("f32_big_dims_groups2", 1, 500, 2, 64, 128, 2, 128, True),
    ("f32_q256", 1, 700, 2, 16, 32, 1, 256, False),
]


@pytest.mark.parametrize("case", SMALL_F32, ids=[c[0] for c in SMALL_F32])
def test_small_f32(case):
    name, b, L, H, P, N, G, Q, init = case
    _check_full(_w(name, b, L, H, P, N, G, Q, "f32", init, seed=200 + len(name)))


def _check_sampled(w, k, seed):
    inp = inputs.make_inputs(w, device="cuda")
    d = inp
    out = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], w.chunk,
                                 init_states=d["init"], return_final_states=True)
    y, f = out
    torch.cuda.synchronize()
    pairs = sample_pairs(w.batch, w.nheads, k, seed)
    refs = oracle_pairs(inp, pairs)
    ys = np.stack([y[b, :, h].double().cpu().numpy() for (b, h) in pairs])
    fs = np.stack([f[b, h].double().cpu().numpy() for (b, h) in pairs])
    y_ref = np.stack([r[0] for r in refs])
    f_ref = np.stack([r[1] for r in refs])
    tol = TOL[w.dtype]
    ey, ef = rel_err(ys, y_ref), rel_err(fs, f_ref)
    record(w.name, y=ey, final=ef)
    assert torch.isfinite(y.float()).all().item()
    assert ey <= tol, f"{w.name}: sampled y rel err {ey:.3g} > {tol}"
    assert ef <= tol, f"{w.name}: sampled final rel err {ef:.3g} > {tol}"


def test_layer_130m_sampled():
    _check_sampled(inputs.LAYER_130M, k=8, seed=1)


def test_layer_2p7b_sampled():
    _check_sampled(inputs.LAYER_2P7B, k=8, seed=2)


@pytest.mark.parametrize("w", inputs.SWEEP, ids=[w.name for w in inputs.SWEEP])
def test_sweep_sampled(w):
    _check_sampled(w, k=3 if w.seqlen >= 131072 else 6, seed=3)


def test_decode_1024_steps_sampled():
    """1024 sequential ssd_step calls at b=256, H=80, P=64, N=128 against the
    fp64 step oracle on sampled (batch, head) pairs: y at every step and the
    state after the last step."""
    w = inputs.DECODE_2P7B
    gen, par = inputs.make_decode_params(w)
    state = par["state"].cuda()
    A, D = par["A"].cuda(), par["D"].cuda()
    pairs = sample_pairs(w.batch, w.nheads, 6, seed=4)
    ost = {p: par["state"][p[0], p[1]].double().numpy().copy() for p in pairs}
    num_y = den_y = 0.0
    for _ in range(w.steps):
        tok = inputs.make_decode_token(w, gen)
        td = to_dev(tok)
        y = ssd.ssd_step(state, td["x"], td["dt"], A, td["B"], td["C"], D)
        ycpu = y.double().cpu().numpy()
        for (b, h) in pairs:
            yo, st = oracle.step(ost[(b, h)][None, None], tok["x"][b:b + 1, h:h + 1],
                                 tok["dt"][b:b + 1, h:h + 1], par["A"][h:h + 1],
                                 tok["B"][b:b + 1], tok["C"][b:b + 1], par["D"][h:h + 1])
            ost[(b, h)] = st[0, 0]
            num_y = max(num_y, float(np.max(np.abs(ycpu[b, h] - yo[0, 0]))))
            den_y = max(den_y, float(np.max(np.abs(yo[0, 0]))))
    torch.cuda.synchronize()
    ey = num_y / den_y
    record("decode_1024", y=ey)
    fs = np.stack([state[b, h].double().cpu().numpy() for (b, h) in pairs])
    fr = np.stack([ost[p] for p in pairs])
    es = rel_err(fs, fr)
    assert ey <= TOL["bf16"], f"decode y rel err {ey:.3g}"
    assert es <= TOL["bf16"], f"decode state rel err {es:.3g}"


def test_decode_f32_small_full():
    """fp32 decode, every element, 50 steps, odd sizes (scalar kernel path)."""
    w = inputs.DecodeWorkload("decode_f32_small", 3, 5, 7, 9, 1, 50, "f32", seed=77)
    gen, par = inputs.make_decode_params(w)
    state = par["state"].cuda()
    ost = par["state"].double().numpy().copy()
    for _ in range(w.steps):
        tok = inputs.make_decode_token(w, gen)
        td = to_dev(tok)
        y = ssd.ssd_step(state, td["x"], td["dt"], par["A"].cuda(), td["B"], td["C"],
                         par["D"].cuda())
        yo, ost = oracle.step(ost, tok["x"], tok["dt"], par["A"], tok["B"], tok["C"], par["D"])
        assert rel_err(y.double().cpu().numpy(), yo) <= TOL["f32"]
    assert rel_err(state.double().cpu().numpy(), ost) <= TOL["f32"]


# --- each step of the forward on its own -------------------------------------------------

STAGE_CASES = [("bf16", 2, 600, 4, 64, 128, 1, 256), ("bf16", 1, 512, 4, 64, 64, 2, 128),
               ("f32", 2, 333, 3, 16, 16, 1, 64),
               ("bf16", 2, 300, 6, 64, 64, 2, 128),       # 3 heads a group: phantom heads
               ("bf16", 1, 400, 3, 128, 128, 1, 256)]     # headdim 128: virtual heads


def _oracle_chunk_views(inp, Q):
    """Oracle chunk states (zero start), log-decays and entering states."""
    x, dt, A, B, C, D, init = (inp[k] for k in ("x", "dt", "A", "B", "C", "D", "init"))
    b, L, H, P = x.shape
    N = B.shape[3]
    T = (L + Q - 1) // Q
    S = np.zeros((b, T, H, P, N))
    prev = np.zeros((b, T, H, P, N))
    ld = np.zeros((b, T, H))
    h = np.zeros((b, H, P, N)) if init is None else init.double().numpy()
    for c in range(T):
        sl = slice(c * Q, min(L, (c + 1) * Q))
        _, s0 = oracle.recurrence(x[:, sl], dt[:, sl], A, B[:, sl], C[:, sl], D, None)
        S[:, c] = s0
        prev[:, c] = h
        _, h = oracle.recurrence(x[:, sl], dt[:, sl], A, B[:, sl], C[:, sl], D, h)
        ld[:, c] = (dt[:, sl].double() * A.double()[None, None, :]).sum(dim=1).numpy()
    return S, ld, prev, h


@pytest.mark.parametrize("case", STAGE_CASES, ids=lambda c: "_".join(map(str, c)))
def test_stage_chunk_state(case):
    dtype, b, L, H, P, N, G, Q = case
    inp = inputs.make_inputs(_w("st", b, L, H, P, N, G, Q, dtype, True, seed=31))
    d = to_dev(inp)
    S, ld = ssd.ssd_chunk_state_fwd(d["x"], d["dt"], d["A"], d["B"], Q)
    torch.cuda.synchronize()
    S_ref, ld_ref, _, _ = _oracle_chunk_views(inp, Q)
    assert rel_err(S.double().cpu().numpy(), S_ref) <= TOL[dtype]
    assert np.max(np.abs(ld.double().cpu().numpy() - ld_ref)) <= 1e-4 * max(1.0, np.max(np.abs(ld_ref)))


@pytest.mark.parametrize("case", STAGE_CASES, ids=lambda c: "_".join(map(str, c)))
def test_stage_state_passing(case):
    dtype, b, L, H, P, N, G, Q = case
    inp = inputs.make_inputs(_w("sp", b, L, H, P, N, G, Q, dtype, True, seed=32))
    S_ref, ld_ref, prev_ref, final_ref = _oracle_chunk_views(inp, Q)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    prev, fin = ssd.ssd_state_passing_fwd(torch.from_numpy(S_ref).float().cuda(),
                                          torch.from_numpy(ld_ref).float().cuda(), Q, L, tdt,
                                          init_states=inp["init"].cuda())
    torch.cuda.synchronize()
    assert rel_err(prev.double().cpu().numpy(), prev_ref) <= TOL[dtype]
    assert rel_err(fin.double().cpu().numpy(), final_ref) <= TOL[dtype]


WALK_CASES = [(2, 600, 4, 64, 128, 1, 256, True), (1, 512, 4, 64, 64, 2, 128, False),
              (3, 100, 2, 64, 128, 1, 128, True), (1, 777, 6, 64, 64, 1, 256, True),
              (2, 300, 6, 64, 128, 2, 256, True), (1, 400, 3, 128, 64, 1, 128, True)]


@pytest.mark.parametrize("case", WALK_CASES, ids=lambda c: "_".join(map(str, c)))
def test_stage_state_walk(case):
    """The fused walk (chunk states + recurrence on chip) against the oracle's
    entering states and final state."""
    b, L, H, P, N, G, Q, init = case
    inp = inputs.make_inputs(_w("walk", b, L, H, P, N, G, Q, "bf16", init, seed=34))
    _, _, prev_ref, final_ref = _oracle_chunk_views(inp, Q)
    d = to_dev(inp)
    prev, fin = ssd.ssd_state_walk_fwd(d["x"], d["dt"], d["A"], d["B"], Q, init_states=d["init"])
    torch.cuda.synchronize()
    ep = rel_err(prev.double().cpu().numpy(), prev_ref)
    ef = rel_err(fin.double().cpu().numpy(), final_ref)
    record(f"walk_{'_'.join(map(str, case))}", prev=ep, final=ef)
    assert ep <= TOL["bf16"] and ef <= TOL["bf16"], (ep, ef)


WALK_FWD_CASES = [
    # name,                   b,  L,    H,  P,  N,  G,  Q,  init
    ("walk_fwd_n128_g2_odd", 16, 700, 10, 64, 128, 2, 256, True),  # 5 heads a group, 3 chunks
    ("walk_fwd_n64_q128", 16, 800, 12, 64, 64, 2, 128, True),      # 7 chunks, last one partial
]


@pytest.mark.parametrize("case", WALK_FWD_CASES, ids=[c[0] for c in WALK_FWD_CASES])
def test_walk_path_full_forward_ragged_groups(case):
    """Shapes the forward runs as walk + output in two launches (enough
    (batch, head pair) walkers; dstate 64 or a head count per group that is
    not a multiple of 4), with a ragged last chunk, two groups and initial
    states; every element checked."""
    name, b, L, H, P, N, G, Q, init = case
    dims = ssd.make_dims(b, L, H, P, N, G)
    assert ssd.ssd_chunk_scan_fwd_data_flow(dims, Q, torch.bfloat16) == ssd.SSD_FLOW_WALK_OUTPUT
    _check_full(_w(name, b, L, H, P, N, G, Q, "bf16", init, seed=35))


FUSED_FWD_CASES = [
    # name,                 b,  L,    H,  P,   N,  G,  Q,  init
    ("fused_n128_g2", 8, 900, 40, 64, 128, 2, 256, True),       # 4 chunks, last one partial;
                                                                # tiles of 10, then 5 heads
    ("fused_q128_p128", 8, 1000, 24, 128, 128, 1, 128, True),   # 48 virtual heads, 8 chunks
    ("fused_p32", 8, 600, 48, 32, 128, 1, 256, False),          # headdim 32 (zero-padded)
    ("fused_tile_heads_9", 6, 700, 36, 64, 128, 1, 256, True),  # tiles of 9 heads: a walker's
                                                                # four heads split between tiles
    ("fused_192_walkers", 48, 520, 16, 64, 128, 1, 256, True),  # more walkers than SMs
    ("fused_one_chunk", 4, 200, 8, 64, 128, 1, 256, True),      # a single (partial) chunk
    ("fused_few_walkers", 1, 1300, 4, 64, 128, 1, 256, True),   # a single walker
    ("fused_quad_phantoms", 40, 300, 6, 64, 128, 1, 256, True),  # walkers of four heads, 6 a
                                                                 # group: two phantom heads
    ("fused_three_phantoms", 16, 600, 10, 64, 128, 2, 256, True),  # 5 heads a group: the second
                                                                   # walker has one real head
    ("fused_n64", 16, 1100, 12, 64, 64, 2, 128, True),          # dstate 64 (walkers of two)
    ("fused_tiles_halved", 2, 2300, 32, 64, 128, 1, 256, True),  # 9 chunks, few tiles: heads a
                                                                 # tile halved 32 -> 4
]


@pytest.mark.parametrize("case", FUSED_FWD_CASES, ids=[c[0] for c in FUSED_FWD_CASES])
def test_fused_walk_output_full_forward(case):
    """The one-launch data flow (walkers of two or four heads and output tiles
    side by side, the tiles waiting on the walkers' progress counters), forced
    on small shapes: ragged chunks, two groups, 128-token chunks, headdim 32
    and 128, dstate 64, tiles whose heads straddle walkers, walkers with
    phantom heads, more walkers than the GPU has SMs (so that walkers start
    in waves), a single chunk and a single walker; every element checked."""
    name, b, L, H, P, N, G, Q, init = case
    _check_full(_w(name, b, L, H, P, N, G, Q, "bf16", init, seed=37),
                flow=ssd.SSD_FLOW_WALK_OUTPUT_FUSED)
    ssd.ssd_poll_device_status()       # raises if a bounded wait gave up


def test_fused_flow_without_states_and_workspace_reuse():
    """The one-launch flow with neither initial nor final states (y only),
    then two different inputs through one workspace: the scheduling counters
    are reset before every launch, so the second call starts clean."""
    w = _w("fused_nostates", 8, 1100, 24, 64, 128, 1, 256, "bf16", False, seed=40)
    inp = inputs.make_inputs(w)
    y, f = gpu_fwd(inp, 256, want_final=False, flow=ssd.SSD_FLOW_WALK_OUTPUT_FUSED)
    assert f is None
    y_ref, _ = oracle_fwd(inp)
    assert rel_err(y, y_ref) <= TOL["bf16"]
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
    n = ssd.ssd_chunk_scan_fwd_workspace_size(dims, 256, torch.bfloat16,
                                              flow=ssd.SSD_FLOW_WALK_OUTPUT_FUSED)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    for seed in (41, 42):
        wi = _w("fused_reuse", 8, 1100, 24, 64, 128, 1, 256, "bf16", True, seed=seed)
        inp = inputs.make_inputs(wi)
        d = to_dev(inp)
        y, f = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256,
                                      init_states=d["init"], return_final_states=True,
                                      workspace=ws, flow=ssd.SSD_FLOW_WALK_OUTPUT_FUSED)
        torch.cuda.synchronize()
        y_ref, f_ref = oracle_fwd(inp)
        assert rel_err(y.double().cpu().numpy(), y_ref) <= TOL["bf16"], seed
        assert rel_err(f.double().cpu().numpy(), f_ref) <= TOL["bf16"], seed
    ssd.ssd_poll_device_status()


def test_fused_flow_taken_for_long_sequences():
    """With 8 chunks or more the forward takes the one-launch flow by itself
    (16 chunks, ragged last chunk; every element checked)."""
    w = _w("fused_default", 4, 3900, 48, 64, 128, 2, 256, "bf16", True, seed=38)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
    assert ssd.ssd_chunk_scan_fwd_data_flow(dims, 256, torch.bfloat16) == \
        ssd.SSD_FLOW_WALK_OUTPUT_FUSED
    _check_full(w)


def test_every_flow_agrees_with_the_oracle():
    """One input set through every data flow the sizes allow, each against the
    oracle (the SIMT flow at the fp32 kernels' accuracy on bf16 inputs)."""
    w = _w("all_flows", 8, 1300, 24, 64, 128, 1, 256, "bf16", True, seed=39)
    inp = inputs.make_inputs(w)
    y_ref, f_ref = oracle_fwd(inp)
    for flow in (ssd.SSD_FLOW_SIMT, ssd.SSD_FLOW_TC_THREE_KERNEL, ssd.SSD_FLOW_WALK_OUTPUT,
                 ssd.SSD_FLOW_WALK_OUTPUT_FUSED):
        y, f = gpu_fwd(inp, 256, flow=flow)
        ey, ef = rel_err(y, y_ref), rel_err(f, f_ref)
        record(f"all_flows_{flow}", y=ey, final=ef)
        assert ey <= TOL["bf16"] and ef <= TOL["bf16"], (flow, ey, ef)


def test_walk_and_three_kernel_flows_agree():
    """The same inputs through both tensor-core data flows, driven step by
    step: walk + output against chunk states + state pass + output."""
    w = _w("flows", 4, 1500, 8, 64, 128, 1, 256, "bf16", True, seed=36)
    d = to_dev(inputs.make_inputs(w))
    prev_w, fin_w = ssd.ssd_state_walk_fwd(d["x"], d["dt"], d["A"], d["B"], 256,
                                           init_states=d["init"])
    S, ld = ssd.ssd_chunk_state_fwd(d["x"], d["dt"], d["A"], d["B"], 256)
    prev_t, fin_t = ssd.ssd_state_passing_fwd(S, ld, 256, w.seqlen, torch.bfloat16,
                                              init_states=d["init"])
    y_w = ssd.ssd_chunk_output_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], prev_w, 256)
    y_t = ssd.ssd_chunk_output_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], prev_t, 256)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle_fwd(inputs.make_inputs(w))
    for y in (y_w, y_t):
        assert rel_err(y.double().cpu().numpy(), y_ref) <= TOL["bf16"]
    for f in (fin_w, fin_t):
        assert rel_err(f.double().cpu().numpy(), f_ref) <= TOL["bf16"]
    assert rel_err(prev_w.double().cpu().numpy(), prev_t.double().cpu().numpy()) <= TOL["bf16"]


@pytest.mark.parametrize("case", STAGE_CASES, ids=lambda c: "_".join(map(str, c)))
def test_stage_chunk_output(case):
    dtype, b, L, H, P, N, G, Q = case
    inp = inputs.make_inputs(_w("co", b, L, H, P, N, G, Q, dtype, True, seed=33))
    _, _, prev_ref, _ = _oracle_chunk_views(inp, Q)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    d = to_dev(inp)
    y = ssd.ssd_chunk_output_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"],
                                 torch.from_numpy(prev_ref).to(tdt).cuda(), Q)
    torch.cuda.synchronize()
    y_ref, _ = oracle_fwd(inp)
    assert rel_err(y.double().cpu().numpy(), y_ref) <= TOL[dtype]


# --- invariants across entry points --------------------------------------------------------

def test_steps_equal_forward():
    """L decode steps reproduce the chunked forward (both on the GPU)."""
    w = _w("inv", 2, 300, 4, 64, 128, 1, 128, "bf16", True, seed=41)
    inp = to_dev(inputs.make_inputs(w))
    y_fwd, f_fwd = ssd.ssd_chunk_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                          inp["D"], w.chunk, init_states=inp["init"],
                                          return_final_states=True)
    state = inp["init"].clone()
    ys = []
    for t in range(w.seqlen):
        ys.append(ssd.ssd_step(state, inp["x"][:, t].contiguous(), inp["dt"][:, t].contiguous(),
                               inp["A"], inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(),
                               inp["D"]))
    y_dec = torch.stack(ys, dim=1)
    torch.cuda.synchronize()
    assert rel_err(y_dec.double().cpu().numpy(), y_fwd.double().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(state.double().cpu().numpy(), f_fwd.double().cpu().numpy()) <= TOL["bf16"]


def test_split_sequence_resume():
    w = _w("res", 2, 1024, 4, 64, 128, 1, 256, "bf16", True, seed=42)
    inp = to_dev(inputs.make_inputs(w))
    y, f = ssd.ssd_chunk_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  256, init_states=inp["init"], return_final_states=True)
    cut = 384  # not a chunk multiple of 256: the second call starts mid-chunk
    part = lambda k, s: inp[k][:, s].contiguous()
    y1, f1 = ssd.ssd_chunk_scan_fwd(part("x", slice(0, cut)), part("dt", slice(0, cut)), inp["A"],
                                    part("B", slice(0, cut)), part("C", slice(0, cut)), inp["D"],
                                    256, init_states=inp["init"], return_final_states=True)
    y2, f2 = ssd.ssd_chunk_scan_fwd(part("x", slice(cut, None)), part("dt", slice(cut, None)),
                                    inp["A"], part("B", slice(cut, None)),
                                    part("C", slice(cut, None)), inp["D"], 256, init_states=f1,
                                    return_final_states=True)
    torch.cuda.synchronize()
    ycat = torch.cat([y1, y2], dim=1)
    assert rel_err(ycat.double().cpu().numpy(), y.double().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(f2.double().cpu().numpy(), f.double().cpu().numpy()) <= TOL["bf16"]


def test_chunk_size_invariance():
    w = _w("inv_q", 2, 1024, 4, 64, 128, 1, 256, "bf16", True, seed=43)
    inp = inputs.make_inputs(w)
    y_ref, f_ref = oracle_fwd(inp)
    outs = {}
    for Q in (64, 128, 256):
        y, f = gpu_fwd(inp, Q)
        assert rel_err(y, y_ref) <= TOL["bf16"], Q
        assert rel_err(f, f_ref) <= TOL["bf16"], Q
        outs[Q] = y
    assert rel_err(outs[64], outs[256]) <= TOL["bf16"]
    assert rel_err(outs[128], outs[256]) <= TOL["bf16"]


# --- degenerate cases and memory hygiene --------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_no_memory_closed_form(dtype):
    """dt*A -> -inf: y_t = dt_t (C_t.B_t) x_t + D x_t and the initial state is forgotten."""
    w = _w("nomem", 2, 520, 4, 64, 128, 1, 256, dtype, True, seed=44)
    inp = inputs.make_inputs(w)
    inp["A"] = torch.full_like(inp["A"], -1.0e6)
    y, f = gpu_fwd(inp, 256)
    x = inp["x"].double().numpy()
    cb = np.einsum("bln,bln->bl", inp["C"][:, :, 0].double().numpy(), inp["B"][:, :, 0].double().numpy())
    y_cf = (inp["dt"].double().numpy() * cb[:, :, None])[..., None] * x + inp["D"].double().numpy()[None, None, :, None] * x
    assert rel_err(y, y_cf) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_a_zero_cumulative_sum(dtype):
    w = _w("azero", 1, 700, 3, 64, 64, 1, 128, dtype, True, seed=45)
    inp = inputs.make_inputs(w)
    inp["A"] = torch.zeros_like(inp["A"])
    y, f = gpu_fwd(inp, 128)
    y_ref, f_ref = oracle_fwd(inp)
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(f, f_ref) <= TOL[dtype]


def test_mixed_decay_heads_one_cta():
    """Heads whose 128-token tiles decay by more than 2^120 take the exact
    (per-element mask) path of the tensor-core output kernel, the others the
    factorised one; both kinds share a CTA here, with one head near the bound."""
    w = _w("mixdecay", 2, 600, 8, 64, 128, 1, 256, "bf16", True, seed=47)
    inp = inputs.make_inputs(w)
    A = inp["A"].clone()
    A[0], A[3], A[5], A[6] = -1.0e3, -30.0, -40.0, 0.0
    inp["A"] = A
    y, f = gpu_fwd(inp, 256)
    y_ref, f_ref = oracle_fwd(inp)
    ey, ef = rel_err(y, y_ref), rel_err(f, f_ref)
    record("mixed_decay_heads", y=ey, final=ef)
    assert ey <= TOL["bf16"] and ef <= TOL["bf16"], (ey, ef)
    for h in (0, 3, 5, 6):
        assert rel_err(y[:, :, h], y_ref[:, :, h]) <= TOL["bf16"], h


def test_c_zero_gives_skip_only():
    w = _w("czero", 2, 300, 4, 64, 128, 1, 256, "bf16", True, seed=46)
    inp = inputs.make_inputs(w)
    inp["C"] = torch.zeros_like(inp["C"])
    y, _ = gpu_fwd(inp, 256)
    skip = (inp["D"][None, None, :, None] * inp["x"].float()).to(torch.bfloat16).double().numpy()
    assert np.max(np.abs(y - skip)) <= 2 ** -8 * np.max(np.abs(skip))


def test_empty_sequence_copies_init():
    init = torch.randn(2, 3, 16, 8, device="cuda")
    fin = torch.full_like(init, float("nan"))
    x = torch.empty(2, 0, 3, 16, device="cuda")
    dt = torch.empty(2, 0, 3, device="cuda")
    Bm = torch.empty(2, 0, 1, 8, device="cuda")
    A = -torch.ones(3, device="cuda")
    D = torch.ones(3, device="cuda")
    ssd.ssd_chunk_scan_fwd(x, dt, A, Bm, Bm, D, 64, init_states=init, final_states=fin)
    torch.cuda.synchronize()
    assert torch.equal(fin, init)
    fin2 = torch.full_like(init, float("nan"))
    ssd.ssd_chunk_scan_fwd(x, dt, A, Bm, Bm, D, 64, final_states=fin2)
    torch.cuda.synchronize()
    assert torch.count_nonzero(fin2).item() == 0


def test_guard_bands_and_full_coverage():
    """Outputs are written exactly in bounds: sentinel padding around y and
    the final states stays intact, and a NaN prefill of y is fully replaced."""
    w = _w("guard", 2, 600, 4, 64, 128, 1, 256, "bf16", True, seed=47)
    inp = to_dev(inputs.make_inputs(w))
    pad = 4096
    ny = inp["x"].numel()
    ybuf = torch.full((ny + 2 * pad,), float("nan"), device="cuda", dtype=torch.bfloat16)
    ybuf[:pad] = 7.0
    ybuf[-pad:] = 7.0
    y = ybuf[pad:pad + ny].view_as(inp["x"])
    nf = 2 * 4 * 64 * 128
    fbuf = torch.full((nf + 2 * pad,), 5.0, device="cuda")
    fin = fbuf[pad:pad + nf].view(2, 4, 64, 128)
    need = ssd.ssd_chunk_scan_fwd_workspace_size(ssd.make_dims(2, 600, 4, 64, 128, 1), 256,
                                                 torch.bfloat16)
    wbuf = torch.full((need + 2 * pad,), 0xAB, device="cuda", dtype=torch.uint8)
    ws = wbuf[pad:pad + need]
    ssd.ssd_chunk_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], 256,
                           init_states=inp["init"], y=y, final_states=fin, workspace=ws)
    torch.cuda.synchronize()
    assert torch.all(ybuf[:pad] == 7.0) and torch.all(ybuf[-pad:] == 7.0)
    assert torch.all(fbuf[:pad] == 5.0) and torch.all(fbuf[-pad:] == 5.0)
    assert torch.all(wbuf[:pad] == 0xAB) and torch.all(wbuf[-pad:] == 0xAB)
    assert torch.isfinite(y.float()).all() and torch.isfinite(fin).all()


def test_tensor_core_path_selected_for_layer_shapes():
    """Every bf16 workload of the benchmark runs on the tcgen05 kernels (so the
    sampled full-size parity tests above exercise them), the fp32 one on the
    exact SIMT kernels."""
    for w in (inputs.LAYER_130M, inputs.LAYER_2P7B) + tuple(inputs.SWEEP):
        dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
        assert ssd.ssd_chunk_scan_fwd_uses_tensor_cores(dims, w.chunk, torch.bfloat16) == 1, w.name
        assert ssd.ssd_chunk_scan_fwd_data_flow(dims, w.chunk, torch.bfloat16) in (
            ssd.SSD_FLOW_WALK_OUTPUT_FUSED, ssd.SSD_FLOW_WALK_OUTPUT,
            ssd.SSD_FLOW_TC_THREE_KERNEL), w.name
    for w, flow in ((inputs.LAYER_130M, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),
                    (inputs.LAYER_2P7B, ssd.SSD_FLOW_WALK_OUTPUT_FUSED)):
        dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups)
        assert ssd.ssd_chunk_scan_fwd_data_flow(dims, w.chunk, torch.bfloat16) == flow, w.name
    t = inputs.TINY_F32
    dims = ssd.make_dims(t.batch, t.seqlen, t.nheads, t.headdim, t.dstate, t.ngroups)
    assert ssd.ssd_chunk_scan_fwd_uses_tensor_cores(dims, t.chunk, torch.float32) == 0
    dims = ssd.make_dims(4, 8192, 80, 64, 128, 1)
    assert ssd.ssd_chunk_scan_fwd_uses_tensor_cores(dims, 256, torch.float32) == 0


POSITIVE_A_CASES = [
    # a growing state: A > 0 with a modest growth per chunk, through each data flow
    ("posA_three_kernel", 2, 600, 4, 64, 128, 1, 256, "bf16"),
    ("posA_walk", 8, 1100, 24, 64, 128, 1, 256, "bf16"),
    ("posA_fused", 8, 1100, 24, 64, 128, 1, 256, "bf16"),
    ("posA_simt_f32", 1, 500, 3, 16, 32, 1, 64, "f32"),
]


@pytest.mark.parametrize("case", POSITIVE_A_CASES, ids=[c[0] for c in POSITIVE_A_CASES])
def test_positive_a_growing_state(case):
    name, b, L, H, P, N, G, Q, dtype = case
    w = _w(name, b, L, H, P, N, G, Q, dtype, True, seed=48)
    inp = inputs.make_inputs(w)
    g = torch.Generator().manual_seed(48)
    inp["A"] = 0.1 + 0.9 * torch.rand(H, generator=g)     # A in [0.1, 1.0]: exp(dt A) > 1
    y, f = gpu_fwd(inp, Q, flow=ssd.SSD_FLOW_WALK_OUTPUT_FUSED if name == "posA_fused" else None)
    y_ref, f_ref = oracle_fwd(inp)
    ey, ef = rel_err(y, y_ref), rel_err(f, f_ref)
    record(name, y=ey, final=ef)
    assert np.max(np.abs(f_ref)) > np.max(np.abs(inp["init"].numpy())), "state did not grow"
    assert ey <= TOL[dtype] and ef <= TOL[dtype], (ey, ef)


def test_rejects_memory_not_on_the_current_device():
    """x in (unregistered) host memory: rejected before any launch, with the
    reason; the library stays usable."""
    import ctypes
    import numpy as npx
    w = _w("devchk", 1, 256, 2, 64, 128, 1, 256, "bf16", False, seed=49)
    d = to_dev(inputs.make_inputs(w))
    host = npx.zeros(d["x"].numel() * 2 + 64, dtype=npx.uint8)
    addr = (host.ctypes.data + 15) // 16 * 16
    lib = ssd.load()
    dims = ssd.make_dims(1, 256, 2, 64, 128, 1)
    y = torch.empty_like(d["x"])
    ws = torch.empty(ssd.ssd_chunk_scan_fwd_workspace_size(dims, 256, torch.bfloat16) + 16,
                     device="cuda", dtype=torch.uint8)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.ssd_chunk_scan_fwd(ctypes.c_void_p(addr), P(d["dt"]), P(d["A"]), P(d["B"]),
                                P(d["C"]), P(d["D"]), 256, None, P(y), None, ctypes.byref(dims),
                                ssd.SSD_BF16, P(ws), ws.numel(), None)
    assert st == ssd.SSD_ERR_INVALID_ARG
    assert "not device memory" in lib.ssd_last_error_detail().decode()
    with pytest.raises(ValueError, match="expected cuda"):
        ssd.ssd_chunk_scan_fwd(d["x"], d["dt"].cpu(), d["A"], d["B"], d["C"], d["D"], 256)
    _check_full(w)
