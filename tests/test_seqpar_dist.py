"""The sequence-parallel host logic (ssd_chunked_scan_02_b200.seqpar) on two
and three gloo ranks on CPU.  Each rank holds one contiguous piece of every
sequence; its per-rank steps are done here by the fp64 oracle (test code,
written from the recurrence's definitions), so what is checked is the
exchange: one packed all-gather in rank order, the exclusive scan over the
ranks before this one, and the correction of y and of the final state.  The
concatenated outputs must equal the oracle over the whole sequence."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """Per-rank steps from their definitions, in fp64 on the CPU."""

    @staticmethod
    def forward(x, dt, A, B, C, D, chunk_size):
        import oracle
        y, f = oracle.recurrence(x, dt, A, B, C, D, None)
        return torch.from_numpy(y), torch.from_numpy(f)

    @staticmethod
    def logdecay(dt, A):
        return (dt.double() * A.double()[None, None, :]).sum(dim=1)

    @staticmethod
    def combine(local_final, logdecay, init, rank):
        h = torch.zeros_like(local_final[0]) if init is None else init.double().clone()
        for q in range(rank):
            h = torch.exp(logdecay[q])[:, :, None, None] * h + local_final[q]
        return h

    @staticmethod
    def correct(h_in, dt, A, C, y, final):
        # the entering state's own trajectory: the recurrence with x = 0, D = 0
        import oracle
        zx = torch.zeros(y.shape, dtype=torch.float64)
        yc, fc = oracle.recurrence(zx, dt, A, C, C, torch.zeros_like(A), h_in)
        y += torch.from_numpy(yc)
        final.copy_(final + torch.from_numpy(fc))


def _rank(rank, world, port, cuts, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch.distributed as dist

    from ssd_chunked_scan_02_b200 import inputs, seqpar
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = inputs.Workload("seqpar_cpu", 2, cuts[-1], 3, 4, 5, 1, 16, "f32", with_init=True,
                        want_final=True, seed=91)
    inp = inputs.make_inputs(w)
    sl = slice(cuts[rank], cuts[rank + 1])
    part = {k: inp[k][:, sl].contiguous() for k in ("x", "dt", "B", "C")}
    init = inp["init"].double()
    y, fin, g = seqpar.chunk_scan_fwd_seqpar(part["x"], part["dt"], inp["A"], part["B"],
                                             part["C"], inp["D"], 16, init_states=init,
                                             ops=OracleOps)
    out[rank] = (y.numpy(), fin.numpy(), g.numpy())
    dist.destroy_process_group()


def _run(world, cuts):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, cuts, out), nprocs=world, join=True,
                       start_method="spawn")
    sys.path.insert(0, ROOT)
    import oracle
    from ssd_chunked_scan_02_b200 import inputs
    w = inputs.Workload("seqpar_cpu", 2, cuts[-1], 3, 4, 5, 1, 16, "f32", with_init=True,
                        want_final=True, seed=91)
    inp = inputs.make_inputs(w)
    y_ref, f_ref = oracle.recurrence(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                     inp["D"], inp["init"])
    y = np.concatenate([out[r][0] for r in range(world)], axis=1)
    assert np.max(np.abs(y - y_ref)) <= 1e-10 * np.max(np.abs(y_ref))
    # each rank's shard final is the true state after its shard; the global
    # final is the same on every rank and equals the whole sequence's
    _, f_first = oracle.recurrence(inp["x"][:, :cuts[1]], inp["dt"][:, :cuts[1]], inp["A"],
                                   inp["B"][:, :cuts[1]], inp["C"][:, :cuts[1]], inp["D"],
                                   inp["init"])
    assert np.max(np.abs(out[0][1] - f_first)) <= 1e-10 * np.max(np.abs(f_first))
    assert np.max(np.abs(out[world - 1][1] - f_ref)) <= 1e-10 * np.max(np.abs(f_ref))
    for r in range(world):
        assert np.max(np.abs(out[r][2] - f_ref)) <= 1e-10 * np.max(np.abs(f_ref))


def test_two_gloo_ranks_split_sequence_matches_whole():
    _run(2, [0, 53, 120])


def test_three_gloo_ranks_uneven_shards_match_whole():
    _run(3, [0, 7, 71, 100])


def test_pack_unpack_roundtrip():
    sys.path.insert(0, ROOT)
    from ssd_chunked_scan_02_b200 import seqpar
    f = torch.randn(2, 3, 4, 5)
    ld = torch.randn(2, 3)
    g = torch.stack([seqpar.pack(f, ld), seqpar.pack(2 * f, 3 * ld)])
    fs, lds = seqpar.unpack(g, tuple(f.shape), tuple(ld.shape))
    assert torch.equal(fs[0], f) and torch.equal(fs[1], 2 * f)
    assert torch.equal(lds[0], ld) and torch.equal(lds[1], 3 * ld)
