"""ssd_chunk_scan_fwd_noalloc: the forward for callers that cannot allocate
device memory (for example a plugin inside a runtime that owns the device
heap and offers no allocator, or a path that cannot afford the device-wide
synchronisation of cudaMalloc/cudaFree).  It takes its scratch from a fixed
array inside the library instead of a caller workspace.

This file is named so that pytest collects it last; it builds and loads the
library itself, so it also runs alone in a fresh process."""
import ctypes

import pytest
import torch

from parity import TOL, rel_err
from ssd_chunked_scan_02_b200 import build as ssd_build
from ssd_chunked_scan_02_b200 import inputs, ssd


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.load()


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    """Runs without a GPU: the size check happens before any device work."""
    dims = ssd.make_dims(4, 8192, 80, 64, 128, 1)      # ~0.5 GB of scratch needed
    st = lib.ssd_chunk_scan_fwd_noalloc(None, None, None, None, None, None, 256, None, None, None,
                                        ctypes.byref(dims), ssd.SSD_BF16, None)
    assert st == ssd.SSD_ERR_UNSUPPORTED
    msg = lib.ssd_last_error_detail().decode()
    assert "scratch" in msg and str(ssd.NOALLOC_SCRATCH_BYTES) in msg


def _case(name, b, L, H, P, N, G, Q, dtype, seed):
    return inputs.Workload(name, b, L, H, P, N, G, Q, dtype, with_init=True, want_final=True,
                           seed=seed)


@pytest.mark.gpu
def test_noalloc_matches_workspace_forward_twice_in_a_row(lib):
    """Two consecutive calls (different sizes and dtypes, so the second one
    runs over whatever the first left in the shared scratch) each agree with
    ssd_chunk_scan_fwd given a caller workspace."""
    cases = [_case("noalloc_bf16", 2, 1000, 8, 64, 128, 1, 256, "bf16", 501),
             _case("noalloc_f32", 1, 700, 4, 32, 64, 2, 128, "f32", 502)]
    for w in cases:
        d = {k: (v.cuda() if v is not None else None) for k, v in inputs.make_inputs(w).items()}
        need = ssd.ssd_chunk_scan_fwd_workspace_size(
            ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups), w.chunk,
            d["x"].dtype)
        assert need <= ssd.NOALLOC_SCRATCH_BYTES
        y_ref, f_ref = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"],
                                              w.chunk, init_states=d["init"],
                                              return_final_states=True)
        y = torch.full_like(y_ref, float("nan"))
        f = torch.full_like(f_ref, float("nan"))
        ssd.ssd_chunk_scan_fwd_noalloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], w.chunk,
                                       init_states=d["init"], y=y, final_states=f)
        torch.cuda.synchronize()
        tol = TOL[w.dtype]
        assert rel_err(y.double().cpu().numpy(), y_ref.double().cpu().numpy()) <= tol, w.name
        assert rel_err(f.double().cpu().numpy(), f_ref.double().cpu().numpy()) <= tol, w.name
