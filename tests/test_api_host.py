"""C-ABI checks that need no GPU: the library loads, exports every symbol its
header declares, sizes its workspace, and rejects bad arguments before
launching anything (so every call here returns without touching a device)."""
import ctypes
import os
import re

import pytest

from ssd_chunked_scan_02_b200 import build as ssd_build
from ssd_chunked_scan_02_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SSD_API\s+[\w\s\*]*?\b(ssd_\w+)\s*\(", text)))


def test_header_declares_the_two_main_calls():
    syms = declared_symbols()
    assert "ssd_chunk_scan_fwd" in syms and "ssd_step" in syms
    assert len(syms) >= 9


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in include/ssd.h but not exported"
    assert set(declared_symbols()) == set(ssd.EXPORTED)


def test_status_strings(lib):
    assert ssd.status_name(0) == "SSD_OK"
    assert ssd.status_name(1) == "SSD_ERR_INVALID_ARG"
    assert ssd.status_name(2) == "SSD_ERR_UNSUPPORTED"
    assert ssd.status_name(3) == "SSD_ERR_CUDA"
    assert ssd.status_name(4) == "SSD_ERR_TIMEOUT"
    assert ssd.status_name(99) == "SSD_ERR_UNKNOWN"


def _ws(dims, q, dt):
    n = ctypes.c_size_t(0)
    st = ssd.load().ssd_chunk_scan_fwd_workspace_size(ctypes.byref(dims), q, dt, ctypes.byref(n))
    return st, n.value


def _round(v):
    return (v + 255) // 256 * 256


@pytest.mark.parametrize("b,L,H,P,N,G,Q,dt", [
    (4, 8192, 80, 64, 128, 1, 256, ssd.SSD_BF16),
    (8, 2048, 24, 64, 128, 1, 128, ssd.SSD_BF16),   # one launch, 128-token chunks
    (4, 8192, 40, 128, 128, 1, 256, ssd.SSD_BF16),  # one launch, headdim 128
    (1024, 512, 32, 64, 64, 1, 256, ssd.SSD_BF16),  # walk + output (dstate 64)
    (1, 256, 4, 16, 16, 1, 64, ssd.SSD_F32),
    (2, 600, 4, 64, 128, 2, 128, ssd.SSD_BF16),   # ragged: 5 chunks, last one partial
    (3, 1, 2, 3, 5, 1, 16, ssd.SSD_F32),
    (2, 300, 4, 64, 128, 1, 64, ssd.SSD_BF16),    # bf16 below 128: runs 128-token chunks
    (2, 300, 4, 32, 128, 1, 64, ssd.SSD_BF16),    # headdim 32: tensor cores, 64 state rows
    (2, 300, 4, 32, 128, 1, 64, ssd.SSD_F32),     # headdim 32 in fp32: SIMT, chunks as asked
])
def test_workspace_size_formula(lib, b, L, H, P, N, G, Q, dt):
    dims = ssd.make_dims(b, L, H, P, N, G)
    st, n = _ws(dims, Q, dt)
    assert st == ssd.SSD_OK
    tc = lib.ssd_chunk_scan_fwd_uses_tensor_cores(ctypes.byref(dims), Q, dt) == 1
    Qe = max(Q, 128) if tc else Q
    T = (L + Qe - 1) // Qe
    elt = 4 if dt == ssd.SSD_F32 else 2
    # the tensor-core flows keep 64 state rows for a head of headdim 32
    ns = b * T * H * (max(P, 64) if tc else P) * N
    flow = lib.ssd_chunk_scan_fwd_data_flow(ctypes.byref(dims), Q, dt)
    if flow == ssd.SSD_FLOW_WALK_OUTPUT:
        # the walk keeps chunk states on chip: only the entering states
        assert n == _round(ns * elt)
    elif flow == ssd.SSD_FLOW_WALK_OUTPUT_FUSED:
        # entering states, then a ticket counter (32 ints with padding) and one
        # progress counter per walker of four virtual heads
        Hv = H * max(P, 64) // 64
        assert n == _round(ns * elt) + _round((32 + b * Hv // 4) * 4)
    else:
        # chunk states (fp32), per-chunk log-decays, entering states
        assert n == _round(ns * 4) + _round(b * T * H * 4) + _round(ns * elt)


@pytest.mark.parametrize("b,L,H,P,N,G,Q,dt,flow", [
    (4, 8192, 80, 64, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),   # 2.7B layer
    (8, 2048, 24, 64, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),   # 130M layer (8 chunks)
    (8, 1024, 24, 64, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT),   # 4 chunks
    (8, 2048, 24, 64, 128, 1, 128, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),   # 16 chunks
    (1024, 512, 32, 64, 64, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT),  # 2 chunks
    (16, 32768, 32, 64, 64, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT),  # 256 walkers: in waves
    (1, 524288, 32, 64, 64, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_TC_THREE_KERNEL),  # 16 walkers
    (4, 131072, 32, 64, 64, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_TC_THREE_KERNEL),  # 64 walkers
    (6, 32768, 32, 64, 64, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),  # 96 walkers of two heads
    (2, 600, 4, 64, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_TC_THREE_KERNEL),
    (4, 8192, 80, 64, 128, 1, 256, ssd.SSD_F32, ssd.SSD_FLOW_SIMT),
    (4, 8192, 80, 32, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),   # headdim 32
    (2, 600, 4, 32, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_TC_THREE_KERNEL),
    (2, 600, 4, 96, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_SIMT),            # headdim 96
    (4, 8192, 40, 128, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT_FUSED),  # 80 virtual heads
    (2, 600, 6, 64, 128, 2, 256, ssd.SSD_BF16, ssd.SSD_FLOW_TC_THREE_KERNEL),  # 3 heads a group
    (16, 600, 10, 64, 128, 2, 256, ssd.SSD_BF16, ssd.SSD_FLOW_WALK_OUTPUT),   # 96 walkers, 5 heads a group
    (2, 300, 4, 64, 128, 1, 64, ssd.SSD_BF16, ssd.SSD_FLOW_TC_THREE_KERNEL),  # chunk 64
    (2, 300, 4, 64, 48, 1, 256, ssd.SSD_BF16, ssd.SSD_FLOW_SIMT),             # dstate 48
])
def test_data_flow_query(lib, b, L, H, P, N, G, Q, dt, flow):
    dims = ssd.make_dims(b, L, H, P, N, G)
    assert lib.ssd_chunk_scan_fwd_data_flow(ctypes.byref(dims), Q, dt) == flow
    tc = lib.ssd_chunk_scan_fwd_uses_tensor_cores(ctypes.byref(dims), Q, dt)
    assert tc == (0 if flow == ssd.SSD_FLOW_SIMT else 1)


def test_forced_flow_workspace_and_rejections(lib):
    """The flow-choosing entry points: each flow's workspace (the default's is
    the chosen flow's), SSD_ERR_UNSUPPORTED for a flow that does not cover the
    sizes, SSD_ERR_INVALID_ARG for an unknown one -- all before any device
    work."""
    n = ctypes.c_size_t(0)

    def ws(dims, Q, flow):
        st = lib.ssd_chunk_scan_fwd_flow_workspace_size(ctypes.byref(dims), Q, ssd.SSD_BF16,
                                                        flow, ctypes.byref(n))
        return st, int(n.value)

    d = ssd.make_dims(8, 2048, 24, 64, 128, 1)
    T, ns = 8, 8 * 8 * 24 * 64 * 128
    assert ws(d, 256, -1) == ws(d, 256, ssd.SSD_FLOW_WALK_OUTPUT_FUSED)
    assert ws(d, 256, ssd.SSD_FLOW_WALK_OUTPUT)[1] == _round(2 * ns)
    three = _round(4 * ns) + _round(8 * T * 24 * 4) + _round(2 * ns)
    assert ws(d, 256, ssd.SSD_FLOW_TC_THREE_KERNEL)[1] == three
    assert ws(d, 256, ssd.SSD_FLOW_SIMT)[1] == three
    # walkers of four heads (dstate 128): 48 walkers, then 32 + 48 counters
    assert ws(d, 256, ssd.SSD_FLOW_WALK_OUTPUT_FUSED)[1] == _round(2 * ns) + _round((32 + 48) * 4)
    odd = ssd.make_dims(16, 600, 10, 64, 128, 2)            # 5 heads a group: 2 walkers a group
    assert ws(odd, 256, ssd.SSD_FLOW_WALK_OUTPUT_FUSED)[1] == \
        _round(16 * 3 * 10 * 64 * 128 * 2) + _round((32 + 16 * 2 * 2) * 4)
    n64 = ssd.make_dims(8, 2048, 24, 64, 48, 1)             # dstate 48: SIMT only
    assert ws(n64, 256, ssd.SSD_FLOW_WALK_OUTPUT_FUSED)[0] == ssd.SSD_ERR_UNSUPPORTED
    p96 = ssd.make_dims(2, 600, 4, 96, 128, 1)              # no tensor cores
    assert ws(p96, 256, ssd.SSD_FLOW_WALK_OUTPUT)[0] == ssd.SSD_ERR_UNSUPPORTED
    assert ws(p96, 256, ssd.SSD_FLOW_SIMT)[0] == ssd.SSD_OK
    assert ws(d, 256, 7)[0] == ssd.SSD_ERR_INVALID_ARG
    st = lib.ssd_chunk_scan_fwd_with_flow(None, None, None, None, None, None, 256, None, None,
                                          None, ctypes.byref(p96), ssd.SSD_BF16, None, 0, None,
                                          ssd.SSD_FLOW_WALK_OUTPUT_FUSED)
    assert st == ssd.SSD_ERR_UNSUPPORTED


def test_data_flow_query_rejects(lib):
    bad = ssd.make_dims(1, 64, 4, 8, 8, 3)
    assert lib.ssd_chunk_scan_fwd_data_flow(ctypes.byref(bad), 64, ssd.SSD_F32) == -1


def test_workspace_zero_for_empty(lib):
    assert _ws(ssd.make_dims(0, 100, 4, 8, 8, 1), 64, ssd.SSD_F32) == (ssd.SSD_OK, 0)
    assert _ws(ssd.make_dims(2, 0, 4, 8, 8, 1), 64, ssd.SSD_F32) == (ssd.SSD_OK, 0)


@pytest.mark.parametrize("dims,q,dt,expect", [
    ((1, 64, 4, 8, 8, 3), 64, ssd.SSD_F32, ssd.SSD_ERR_INVALID_ARG),      # H % G != 0
    ((1, 64, 0, 8, 8, 1), 64, ssd.SSD_F32, ssd.SSD_ERR_INVALID_ARG),      # H = 0
    ((-1, 64, 4, 8, 8, 1), 64, ssd.SSD_F32, ssd.SSD_ERR_INVALID_ARG),     # b < 0
    ((1, 64, 4, 300, 8, 1), 64, ssd.SSD_F32, ssd.SSD_ERR_UNSUPPORTED),    # P > 256
    ((1, 64, 4, 8, 512, 1), 64, ssd.SSD_F32, ssd.SSD_ERR_UNSUPPORTED),    # N > 256
    ((1, 64, 4, 8, 8, 1), 96, ssd.SSD_F32, ssd.SSD_ERR_UNSUPPORTED),      # not a power of two
    ((1, 64, 4, 8, 8, 1), 512, ssd.SSD_F32, ssd.SSD_ERR_UNSUPPORTED),     # chunk too large
    ((1, 64, 4, 8, 8, 1), 8, ssd.SSD_F32, ssd.SSD_ERR_UNSUPPORTED),       # chunk too small
    ((1, 64, 4, 8, 8, 1), 64, 7, ssd.SSD_ERR_INVALID_ARG),                # unknown dtype
])
def test_workspace_rejects(lib, dims, q, dt, expect):
    st, _ = _ws(ssd.make_dims(*dims), q, dt)
    assert st == expect
    assert ssd.load().ssd_last_error_detail().decode() != ""


def test_null_dims_rejected(lib):
    n = ctypes.c_size_t(0)
    assert lib.ssd_chunk_scan_fwd_workspace_size(None, 64, 0, ctypes.byref(n)) == 1


# Fake, never-dereferenced device addresses: the calls below must fail
# validation before any launch.
A16 = 0x7f0000001000


def _fwd(lib, dims, ptrs, q=64, dt=ssd.SSD_F32, ws_bytes=1 << 30, init=None, fin=None):
    x, dtp, A, B, C, D, y, ws = ptrs
    return lib.ssd_chunk_scan_fwd(x, dtp, A, B, C, D, q, init, y, fin, ctypes.byref(dims), dt,
                                  ws, ws_bytes, None)


def _good():
    return [A16 + k * 0x100000 for k in range(8)]


@pytest.mark.parametrize("which", range(8))
def test_fwd_null_pointer_rejected(lib, which):
    p = _good()
    p[which] = None
    st = _fwd(lib, ssd.make_dims(1, 128, 4, 8, 8, 1), p)
    assert st == ssd.SSD_ERR_INVALID_ARG
    assert "NULL" in lib.ssd_last_error_detail().decode()


@pytest.mark.parametrize("which", range(8))
def test_fwd_misaligned_pointer_rejected(lib, which):
    p = _good()
    p[which] += 4
    st = _fwd(lib, ssd.make_dims(1, 128, 4, 8, 8, 1), p)
    assert st == ssd.SSD_ERR_INVALID_ARG
    assert "aligned" in lib.ssd_last_error_detail().decode()


def test_fwd_misaligned_optional_rejected(lib):
    st = _fwd(lib, ssd.make_dims(1, 128, 4, 8, 8, 1), _good(), init=A16 + 8)
    assert st == ssd.SSD_ERR_INVALID_ARG
    st = _fwd(lib, ssd.make_dims(1, 128, 4, 8, 8, 1), _good(), fin=A16 + 8)
    assert st == ssd.SSD_ERR_INVALID_ARG


def test_fwd_small_workspace_rejected(lib):
    dims = ssd.make_dims(2, 600, 4, 64, 128, 1)
    _, need = _ws(dims, 128, ssd.SSD_BF16)
    st = _fwd(lib, dims, _good(), q=128, dt=ssd.SSD_BF16, ws_bytes=need - 1)
    assert st == ssd.SSD_ERR_INVALID_ARG
    assert "workspace" in lib.ssd_last_error_detail().decode()


def test_fwd_bad_chunk_rejected(lib):
    assert _fwd(lib, ssd.make_dims(1, 128, 4, 8, 8, 1), _good(), q=100) == ssd.SSD_ERR_UNSUPPORTED


def test_fwd_empty_batch_is_noop(lib):
    assert _fwd(lib, ssd.make_dims(0, 128, 4, 8, 8, 1), [None] * 8) == ssd.SSD_OK


def test_step_rejects(lib):
    dims = ssd.make_dims(2, 1, 4, 8, 8, 1)
    p = _good()
    assert lib.ssd_step(None, *p[1:8], ctypes.byref(dims), 0, None) == ssd.SSD_ERR_INVALID_ARG
    p2 = list(p)
    p2[3] += 2
    assert lib.ssd_step(*p2, ctypes.byref(dims), 0, None) == ssd.SSD_ERR_INVALID_ARG
    bad = ssd.make_dims(2, 1, 4, 8, 8, 3)
    assert lib.ssd_step(*p, ctypes.byref(bad), 0, None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_step(*p, ctypes.byref(ssd.make_dims(0, 1, 4, 8, 8, 1)), 0, None) == ssd.SSD_OK


def test_stage_entry_points_reject(lib):
    dims = ssd.make_dims(1, 128, 4, 8, 8, 1)
    assert lib.ssd_chunk_state_fwd(None, A16, A16, A16, 64, A16, A16, ctypes.byref(dims), 0,
                                   None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_state_passing_fwd(A16, None, None, A16, None, 64, ctypes.byref(dims), 0,
                                     None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_chunk_output_fwd(A16, A16, A16, A16, A16, A16, None, 64, A16,
                                    ctypes.byref(dims), 0, None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_chunk_output_fwd(A16, A16, A16, A16, A16, A16, A16, 24, A16,
                                    ctypes.byref(dims), 0, None) == ssd.SSD_ERR_UNSUPPORTED


def test_tensor_core_selection_query(lib):
    f = lib.ssd_chunk_scan_fwd_uses_tensor_cores
    assert f(ctypes.byref(ssd.make_dims(1, 64, 4, 8, 8, 3)), 64, 0) == -1
    assert f(ctypes.byref(ssd.make_dims(1, 256, 4, 16, 16, 1)), 64, ssd.SSD_F32) == 0


def test_binding_checks_shapes_and_dtypes_before_calling(lib):
    import torch
    b, L, H, P, N = 1, 64, 2, 8, 4
    args = dict(x=torch.zeros(b, L, H, P), dt=torch.zeros(b, L, H), A=torch.zeros(H),
                B=torch.zeros(b, L, 1, N), C=torch.zeros(b, L, 1, N), D=torch.zeros(H))
    for key, bad, what in [("dt", torch.zeros(b, L, H + 1), "shape"),
                           ("A", torch.zeros(H, dtype=torch.float64), "dtype"),
                           ("C", torch.zeros(b, L, 1, N + 1), "shape"),
                           ("D", torch.zeros(H + 1), "shape")]:
        a = dict(args)
        a[key] = bad
        with pytest.raises(ValueError, match=f"{key}: {what}"):
            ssd.ssd_chunk_scan_fwd(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], 64)
    with pytest.raises(ValueError, match="init_states: shape"):
        ssd.ssd_chunk_scan_fwd(*args.values(), 64, init_states=torch.zeros(b, H, P, N + 1))
    with pytest.raises(ValueError, match="y: dtype"):
        ssd.ssd_chunk_scan_fwd(*args.values(), 64, y=torch.zeros(b, L, H, P,
                                                                   dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="state: shape"):
        ssd.ssd_step(torch.zeros(b, H, P, N + 1), torch.zeros(b, H, P), torch.zeros(b, H),
                     torch.zeros(H), torch.zeros(b, 1, N), torch.zeros(b, 1, N), torch.zeros(H))


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 64, 2, 8)
    with pytest.raises(ValueError, match="CUDA"):
        ssd.ssd_chunk_scan_fwd(x, torch.zeros(1, 64, 2), torch.zeros(2), torch.zeros(1, 64, 1, 8),
                               torch.zeros(1, 64, 1, 8), torch.zeros(2), 64)


# ------------------------------------------------------------------ backward
def _bwd_ws(dims, dt):
    n = ctypes.c_size_t(0)
    st = ssd.load().ssd_chunk_scan_bwd_workspace_size(ctypes.byref(dims), dt, ctypes.byref(n))
    return st, n.value


@pytest.mark.parametrize("b,L,H,P,N,G,dt", [
    (8, 2048, 24, 64, 128, 1, ssd.SSD_F32),     # 8 rows of 128 a CTA, 32 segments
    (2, 150, 4, 16, 32, 2, ssd.SSD_F32),        # 16 rows (all of P) a CTA, 3 segments
    (1, 65, 6, 12, 20, 3, ssd.SSD_BF16),        # 12 rows (P < 1024 / N), 2 segments
    (1, 70, 2, 128, 128, 2, ssd.SSD_F32),       # 8 rows a CTA, 16 row blocks
])
def test_backward_workspace_size_formula(lib, b, L, H, P, N, G, dt):
    # CUDA-core path, per (batch, head, block of R = min(P, 1024 / N) state
    # rows): fp32 checkpoints every 64 tokens plus one 64-token segment of states
    dims = ssd.make_dims(b, L, H, P, N, G)
    assert ssd.load().ssd_chunk_scan_bwd_uses_tensor_cores(ctypes.byref(dims), dt) == 0
    st, n = _bwd_ws(dims, dt)
    assert st == ssd.SSD_OK
    R = min(P, 1024 // N)
    blocks = b * H * ((P + R - 1) // R)
    assert n == blocks * ((L + 63) // 64 + 64) * R * N * 4


@pytest.mark.parametrize("b,L,H,P,N,G", [
    (8, 2048, 24, 64, 128, 1), (1, 70, 2, 128, 128, 2), (2, 300, 4, 64, 64, 2), (1, 1, 3, 192, 128, 1),
    (2, 300, 4, 32, 64, 2),
])
def test_backward_tensor_core_workspace_size_formula(lib, b, L, H, P, N, G):
    # tensor-core path (bf16): per 128-token chunk the entering states and
    # dL/dh, each as two bf16 planes (value and rounding residue), one fp32
    # buffer of the same size and the chunks' log decays, each rounded up to
    # 256 bytes; a head of headdim 32 keeps 64 state rows
    dims = ssd.make_dims(b, L, H, P, N, G)
    assert ssd.load().ssd_chunk_scan_bwd_uses_tensor_cores(ctypes.byref(dims), ssd.SSD_BF16) == 1
    st, n = _bwd_ws(dims, ssd.SSD_BF16)
    assert st == ssd.SSD_OK
    up = lambda v: (v + 255) // 256 * 256
    T = (L + 127) // 128
    e = b * T * H * max(P, 64) * N
    assert n == 4 * up(e * 2) + up(e * 4) + up(b * T * H * 4)


@pytest.mark.parametrize("P,N,dt,want", [
    (64, 128, ssd.SSD_BF16, 1), (256, 64, ssd.SSD_BF16, 1), (64, 128, ssd.SSD_F32, 0),
    (32, 128, ssd.SSD_BF16, 1), (64, 96, ssd.SSD_BF16, 0), (96, 64, ssd.SSD_BF16, 0),
    (320, 64, ssd.SSD_BF16, -1),
    (64, 512, ssd.SSD_BF16, -1),
])
def test_backward_path_query(lib, P, N, dt, want):
    dims = ssd.make_dims(2, 100, 4, P, N, 2)
    assert ssd.load().ssd_chunk_scan_bwd_uses_tensor_cores(ctypes.byref(dims), dt) == want


def test_backward_workspace_zero_for_empty(lib):
    assert _bwd_ws(ssd.make_dims(0, 100, 4, 8, 8, 1), ssd.SSD_F32) == (ssd.SSD_OK, 0)
    assert _bwd_ws(ssd.make_dims(2, 0, 4, 8, 8, 1), ssd.SSD_BF16) == (ssd.SSD_OK, 0)


def test_backward_rejects_bad_arguments_before_launching(lib):
    L = ssd.load()
    dims = ssd.make_dims(1, 64, 4, 8, 8, 1)
    bad = ssd.make_dims(1, 64, 4, 8, 8, 3)          # H % G != 0
    big = ssd.make_dims(1, 64, 4, 8, 512, 1)        # dstate > 256
    null16 = [None] * 16

    def call(d, ws=None, wsb=0, args=null16):
        return L.ssd_chunk_scan_bwd(*args, ctypes.byref(d), ssd.SSD_BF16, ws, wsb, None)
    assert call(bad) == ssd.SSD_ERR_INVALID_ARG
    assert call(big) == ssd.SSD_ERR_UNSUPPORTED
    assert call(dims) == ssd.SSD_ERR_INVALID_ARG     # NULL A, D, dA, dD
    # valid-looking (never dereferenced) aligned addresses, but a short workspace
    fake = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(16)]
    fake[6] = fake[8] = fake[15] = None              # init, dfinal, dinit are optional
    st = call(dims, ctypes.c_void_p(0x1000000), 16, fake)
    assert st == ssd.SSD_ERR_INVALID_ARG
    assert b"workspace_bytes" in L.ssd_last_error_detail()


# ------------------------------------------------------------------ sequence parallelism
def test_seqpar_entries_reject_bad_arguments_before_launching(lib):
    dims = ssd.make_dims(2, 64, 4, 8, 8, 1)
    d = ctypes.byref(dims)
    assert lib.ssd_seq_logdecay(A16, None, A16, d, None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_seq_logdecay(A16 + 4, A16, A16, d, None) == ssd.SSD_ERR_INVALID_ARG
    # rank outside [0, nranks], nranks < 1, missing gathered values for rank > 0
    assert lib.ssd_state_exchange_combine(A16, A16, None, 3, 2, A16, d, None) == \
        ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_state_exchange_combine(A16, A16, None, -1, 2, A16, d, None) == \
        ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_state_exchange_combine(A16, A16, None, 0, 0, A16, d, None) == \
        ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_state_exchange_combine(None, A16, None, 1, 2, A16, d, None) == \
        ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_state_exchange_combine(A16, A16, None, 1, 2, None, d, None) == \
        ssd.SSD_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert lib.ssd_state_correction_workspace_size(d, ssd.SSD_F32, ctypes.byref(n)) == ssd.SSD_OK
    # tile prefixes of 128-token tiles, (b, tiles, H) fp32
    assert n.value == _round(2 * 1 * 4 * 4)
    st = lib.ssd_state_correction_fwd(A16, A16, A16, A16, A16, None, d, ssd.SSD_F32, A16,
                                      n.value - 1, None)
    assert st == ssd.SSD_ERR_INVALID_ARG and "workspace" in lib.ssd_last_error_detail().decode()
    st = lib.ssd_state_correction_fwd(None, A16, A16, A16, A16, None, d, ssd.SSD_F32, A16,
                                      n.value, None)
    assert st == ssd.SSD_ERR_INVALID_ARG


def test_correction_workspace_size_tensor_core_shape(lib):
    """bf16, P 64, N 128: tile prefixes plus h_in rounded to bf16."""
    dims = ssd.make_dims(4, 4096, 80, 64, 128, 1)
    n = ctypes.c_size_t(0)
    assert lib.ssd_state_correction_workspace_size(ctypes.byref(dims), ssd.SSD_BF16,
                                                   ctypes.byref(n)) == ssd.SSD_OK
    assert n.value == _round(4 * 32 * 80 * 4) + _round(4 * 80 * 64 * 128 * 2)
