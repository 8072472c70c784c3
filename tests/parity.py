"""Helpers for GPU-vs-oracle parity: run the CUDA path through the binding,
run the fp64 oracle on the same inputs (whole tensors, or sampled
(batch, head) pairs at full size), and measure the error."""
from __future__ import annotations

import concurrent.futures as cf
import json
import os

import numpy as np
import torch

import oracle
from ssd_chunked_scan_02_b200 import ssd

TOL = {"f32": 1e-4, "bf16": 5e-3}


def record(name: str, **errs):
    """Append measured errors to $SSD_PARITY_LOG (JSON lines), when set, so
    the margins to the tolerances stay visible."""
    path = os.environ.get("SSD_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **errs}) + "\n")


def rel_err(a, ref) -> float:
    """max |a - ref| / max |ref| over the whole tensor."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 1.0
    if den == 0.0:
        den = 1.0
    return float(np.max(np.abs(a - ref))) / den if ref.size else 0.0


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: (v.to(device) if v is not None else None) for k, v in inp.items()}


def gpu_fwd(inp: dict, chunk: int, want_final=True, flow=None):
    """CUDA path (the library's data flow, or the SSD_FLOW_* given); returns
    (y float64 numpy on host, final or None)."""
    d = to_dev(inp)
    out = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk,
                                 init_states=d["init"], return_final_states=want_final,
                                 flow=flow)
    torch.cuda.synchronize()
    if want_final:
        y, f = out
        return y.double().cpu().numpy(), f.double().cpu().numpy()
    return out.double().cpu().numpy(), None


def oracle_fwd(inp: dict, threads: int = 0):
    return oracle.recurrence(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                             inp["init"], threads=threads)


def _pair_inputs(inp: dict, b: int, h: int):
    H = inp["x"].shape[2]
    G = inp["B"].shape[2]
    g = h // (H // G)
    sl = lambda t: t.detach().to("cpu")
    out = {
        "x": sl(inp["x"][b:b + 1, :, h:h + 1]),
        "dt": sl(inp["dt"][b:b + 1, :, h:h + 1]),
        "A": sl(inp["A"][h:h + 1]),
        "B": sl(inp["B"][b:b + 1, :, g:g + 1]),
        "C": sl(inp["C"][b:b + 1, :, g:g + 1]),
        "D": sl(inp["D"][h:h + 1]),
        "init": sl(inp["init"][b:b + 1, h:h + 1]) if inp.get("init") is not None else None,
    }
    return out


def oracle_pairs(inp: dict, pairs, workers: int = 8):
    """fp64 oracle for each sampled (batch, head) pair; returns a list of
    (y (L, P), final (P, N)).  Pairs run concurrently (the C call releases
    the GIL)."""
    jobs = [_pair_inputs(inp, b, h) for (b, h) in pairs]

    def one(p):
        y, f = oracle.recurrence(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init"],
                                 threads=1)
        return y[0, :, 0, :], f[0, 0]

    with cf.ThreadPoolExecutor(max_workers=max(1, min(workers, len(jobs)))) as ex:
        return list(ex.map(one, jobs))


def sample_pairs(b: int, H: int, k: int, seed: int):
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (b - 1, H - 1)}
    while len(pairs) < min(k, b * H):
        pairs.add((int(rng.integers(b)), int(rng.integers(H))))
    return sorted(pairs)
