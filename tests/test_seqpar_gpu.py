"""The sequence-parallel entry points on the GPU against the fp64 oracle.

ssd_seq_logdecay against the sum it is defined as; ssd_state_exchange_combine
against the rank-order fold; ssd_state_correction_fwd by the identity it
rests on: a shard run from a zero state and corrected with the state entering
it equals the oracle run of that shard from that state.  Then the whole
split, emulated on one GPU (shards one after another, the gather done by
stacking), against the oracle over the whole sequence -- every element at
small sizes, sampled (batch, head) pairs at the 2.7B-layer size split in two."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, oracle_pairs, record, rel_err, sample_pairs, to_dev
from ssd_chunked_scan_02_b200 import inputs, seqpar, ssd

pytestmark = pytest.mark.gpu


def _w(name, b, L, H, P, N, G, Q, dtype, init, seed):
    return inputs.Workload(name, b, L, H, P, N, G, Q, dtype, with_init=init, want_final=True,
                           seed=seed)


def test_seq_logdecay_is_the_sum():
    w = _w("ld", 3, 3001, 37, 8, 8, 1, 64, "f32", False, seed=61)
    inp = inputs.make_inputs(w)
    ld = ssd.ssd_seq_logdecay(inp["dt"].cuda(), inp["A"].cuda())
    ref = (inp["dt"].double() * inp["A"].double()[None, None, :]).sum(dim=1).numpy()
    assert np.max(np.abs(ld.double().cpu().numpy() - ref)) <= 1e-6 * np.max(np.abs(ref))


@pytest.mark.parametrize("rank", [0, 1, 2, 3])
def test_exchange_combine_folds_ranks_in_order(rank):
    R, b, H, P, N = 3, 2, 5, 7, 9
    g = torch.Generator().manual_seed(62)
    F = torch.randn(R, b, H, P, N, generator=g)
    ld = -torch.rand(R, b, H, generator=g) * 3
    init = torch.randn(b, H, P, N, generator=g)
    h = init.double()
    for q in range(rank):
        h = torch.exp(ld[q].double())[:, :, None, None] * h + F[q].double()
    out = ssd.ssd_state_exchange_combine(F.cuda(), ld.cuda(), rank, init_states=init.cuda())
    assert rel_err(out.double().cpu().numpy(), h.numpy()) <= 1e-6
    out0 = ssd.ssd_state_exchange_combine(F.cuda(), ld.cuda(), rank)
    h0 = torch.zeros_like(h)
    for q in range(rank):
        h0 = torch.exp(ld[q].double())[:, :, None, None] * h0 + F[q].double()
    assert np.max(np.abs(out0.double().cpu().numpy() - h0.numpy())) <= 1e-6 * max(
        1.0, float(h0.abs().max()))


CORR_CASES = [
    # name,            b,  L,   H,  P,  N,  G, dtype,  A
    ("tc_n128", 2, 700, 8, 64, 128, 1, "bf16", "neg"),       # tcgen05 path, ragged tile
    ("tc_n64_g2", 3, 300, 6, 64, 64, 2, "bf16", "neg"),
    ("tc_growing", 2, 500, 4, 64, 128, 1, "bf16", "pos"),    # A > 0: nothing underflows
    ("tc_underflow", 2, 1000, 4, 64, 128, 1, "bf16", "fast"),  # most tiles skipped
    ("simt_f32", 2, 333, 3, 16, 32, 1, "f32", "neg"),       # exact fp32 path
    ("simt_bf16_p32", 2, 260, 4, 32, 48, 2, "bf16", "neg"),  # bf16 outside the tc shapes
]


@pytest.mark.parametrize("case", CORR_CASES, ids=[c[0] for c in CORR_CASES])
def test_correction_completes_a_zero_start_shard(case):
    name, b, L, H, P, N, G, dtype, amode = case
    w = _w(name, b, L, H, P, N, G, 64, dtype, True, seed=63)
    inp = inputs.make_inputs(w)
    if amode == "pos":
        inp["A"] = 0.1 + 0.2 * torch.rand(H, generator=torch.Generator().manual_seed(1))
    elif amode == "fast":
        inp["A"] = torch.full((H,), -60.0)        # decays underflow within ~100 tokens
    d = to_dev(inp)
    h_in = d["init"]                             # the state entering this shard
    y, fin = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 64,
                                    return_final_states=True)
    ssd.ssd_state_correction_fwd(h_in, d["dt"], d["A"], d["C"], y, final_states=fin)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.recurrence(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                     inp["init"])
    ey, ef = rel_err(y.double().cpu().numpy(), y_ref), rel_err(fin.double().cpu().numpy(), f_ref)
    record(f"correction_{name}", y=ey, final=ef)
    assert ey <= TOL[dtype] and ef <= TOL[dtype], (ey, ef)


def test_correction_leaves_underflowed_tokens_untouched():
    """A <= 0 and tokens far past the decay's underflow: y there is bit-for-bit
    the zero-start y (their correction is exactly zero)."""
    w = _w("untouched", 2, 1024, 4, 64, 128, 1, 256, "bf16", True, seed=64)
    d = to_dev(inputs.make_inputs(w))
    d["A"] = torch.full_like(d["A"], -60.0)
    y = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], 256)
    y0 = y.clone()
    ssd.ssd_state_correction_fwd(d["init"], d["dt"], d["A"], d["C"], y)
    torch.cuda.synchronize()
    assert torch.equal(y[:, 512:], y0[:, 512:])
    assert not torch.equal(y[:, :8], y0[:, :8])


def _split_forward(d, cuts, chunk):
    """The sequence-parallel forward emulated on one GPU: each shard's
    zero-start forward and log-decay, the gathered values stacked in rank
    order, then each shard's combine and correction."""
    R = len(cuts) - 1
    parts = []
    for r in range(R):
        sl = slice(cuts[r], cuts[r + 1])
        p = {k: d[k][:, sl].contiguous() for k in ("x", "dt", "B", "C")}
        y, fin = ssd.ssd_chunk_scan_fwd(p["x"], p["dt"], d["A"], p["B"], p["C"], d["D"], chunk,
                                        return_final_states=True)
        parts.append((p, y, fin, ssd.ssd_seq_logdecay(p["dt"], d["A"])))
    buf = torch.stack([seqpar.pack(fin, ld) for (_, _, fin, ld) in parts])
    finals, lds = seqpar.unpack(buf, tuple(parts[0][2].shape), tuple(parts[0][3].shape))
    ys = []
    for r, (p, y, fin, _) in enumerate(parts):
        h_in = ssd.ssd_state_exchange_combine(finals, lds, r, init_states=d["init"])
        ssd.ssd_state_correction_fwd(h_in, p["dt"], d["A"], p["C"], y, final_states=fin)
        ys.append(y)
    g = ssd.ssd_state_exchange_combine(finals, lds, R, init_states=d["init"])
    return torch.cat(ys, dim=1), parts[-1][2], g


@pytest.mark.parametrize("dtype,cuts", [("bf16", [0, 300, 777, 1200]), ("f32", [0, 100, 333])])
def test_split_sequence_emulated_matches_whole(dtype, cuts):
    L = cuts[-1]
    w = (_w("split_bf16", 2, L, 8, 64, 128, 1, 256, "bf16", True, seed=65) if dtype == "bf16"
         else _w("split_f32", 2, L, 3, 16, 32, 1, 64, "f32", True, seed=66))
    inp = inputs.make_inputs(w)
    y, last_fin, g = _split_forward(to_dev(inp), cuts, w.chunk)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.recurrence(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                     inp["init"])
    ey = rel_err(y.double().cpu().numpy(), y_ref)
    ef = rel_err(last_fin.double().cpu().numpy(), f_ref)
    eg = rel_err(g.double().cpu().numpy(), f_ref)
    record(f"split_{dtype}", y=ey, final=ef, global_final=eg)
    assert ey <= TOL[dtype] and ef <= TOL[dtype] and eg <= TOL[dtype], (ey, ef, eg)


def test_split_2p7b_layer_in_two_sampled():
    """The 2.7B-layer workload split in two along L (4096 tokens per shard):
    sampled (batch, head) pairs against the oracle over the whole sequence."""
    w = inputs.LAYER_2P7B
    d = inputs.make_inputs(w, device="cuda")
    y, last_fin, g = _split_forward(d, [0, w.seqlen // 2, w.seqlen], w.chunk)
    torch.cuda.synchronize()
    pairs = sample_pairs(w.batch, w.nheads, 6, seed=5)
    refs = oracle_pairs(d, pairs)
    ys = np.stack([y[b, :, h].double().cpu().numpy() for (b, h) in pairs])
    fs = np.stack([g[b, h].double().cpu().numpy() for (b, h) in pairs])
    ey = rel_err(ys, np.stack([r[0] for r in refs]))
    ef = rel_err(fs, np.stack([r[1] for r in refs]))
    record("split_2p7b", y=ey, final=ef)
    assert ey <= TOL["bf16"] and ef <= TOL["bf16"], (ey, ef)
    # the last shard's corrected final state is the whole sequence's final state
    assert rel_err(last_fin.double().cpu().numpy(), g.double().cpu().numpy()) <= 1e-5
