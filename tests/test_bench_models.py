"""The roofline denominators bench.py reports (algorithmic FLOPs and bytes)
checked against the counts worked out by hand from their definitions, at the
workload shapes (the table of per-configuration counts: 2.7B layer F_alg
130.1 GF, F_dense 173.9 GF, 719.3 MB; 130M layer 19.9 GF, 26.8 GF, 110.6 MB;
each sweep length 559.5 GF, 841.8 GF, 4.50 GB)."""
import bench
from ssd_chunked_scan_02_b200 import inputs


def test_forward_models_at_the_workload_shapes():
    f_alg, f_dense, nbytes = bench.fwd_model(inputs.LAYER_2P7B)
    assert round(f_alg / 1e9, 1) == 130.1 and round(f_dense / 1e9, 1) == 173.9
    # x read + y written (bf16), B and C (bf16), dt (fp32), init and final states (fp32)
    b, L, H, P, N = 4, 8192, 80, 64, 128
    assert nbytes == b * L * (2 * H * P * 2 + 2 * N * 2 + 4 * H) + 2 * 4 * b * H * P * N
    assert round(nbytes / 1e6, 1) == 719.3

    f_alg, f_dense, nbytes = bench.fwd_model(inputs.LAYER_130M)
    assert round(f_alg / 1e9, 1) == 19.9 and round(f_dense / 1e9, 1) == 26.8
    assert round(nbytes / 1e6, 1) == 110.6

    for w in inputs.SWEEP:
        f_alg, f_dense, nbytes = bench.fwd_model(w)
        assert w.batch * w.seqlen == 524288
        assert round(f_alg / 1e9, 1) == 559.5 and round(f_dense / 1e9, 1) == 841.8
        assert round(nbytes / 1e9, 2) == 4.50


def test_kernel_bytes_of_the_three_kernel_forward():
    kb = bench.kernel_bytes(inputs.LAYER_2P7B)
    assert {k: round(v / 1e6, 1) for k, v in kb.items() if k != "decode"} == {
        "chunk_state": 690.0, "state_pass": 524.3, "chunk_out": 866.1}


def test_backward_bytes():
    # 130M layer, bf16, no initial state: x, dy, B, C (bf16) and dt read; dx, ddt,
    # dB, dC (fp32) and the initial state's gradient written
    b, L, H, P, N = 8, 2048, 24, 64, 128
    reads = b * L * (2 * H * P * 2 + 2 * N * 2 + 4 * H)
    writes = b * L * (H * P * 4 + 4 * H + 2 * N * 4)
    assert bench.bwd_bytes(inputs.LAYER_130M) == reads + writes + 4 * b * H * P * N == 235929600
