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


def test_kernel_bytes_of_both_data_flows():
    """io: each kernel's own reads and writes (intermediates included); alg:
    its share of bytes_min (x, y, B, C, dt, init, final; no intermediates)."""
    kb = bench.kernel_bytes(inputs.LAYER_2P7B)
    io = {k: round(v[1] / 1e6, 1) for k, v in kb.items()}
    assert io == {"chunk_state": 690.0, "state_pass": 524.3, "chunk_out": 866.1,
                  "state_walk": 543.2, "walk_out": 1409.3}
    alg = {k: round(v[0] / 1e6, 1) for k, v in kb.items()}
    # chunk_out: x read + y written + B + C + dt = 698.4 MB
    assert alg["chunk_out"] == 698.4
    # the walk: x + B + dt + initial and final states (fp32, 10.5 MB each)
    b, L, H, P, N = 4, 8192, 80, 64, 128
    assert kb["state_walk"][0] == b * L * (H * P * 2 + N * 2 + 4 * H) + 2 * 4 * b * H * P * N
    # the walk + output flow touches every byte of bytes_min; no share exceeds it,
    # and the one-launch flow's kernel has all of it
    _, _, nbytes = bench.fwd_model(inputs.LAYER_2P7B)
    assert max(v[0] for v in kb.values()) <= nbytes
    assert kb["walk_out"][0] == nbytes
    # its own I/O: x and B read by walkers and tiles, C once, dt twice, the
    # entering states written and read (bf16)
    ns = b * (L // 256) * H * P * N
    assert kb["walk_out"][1] == (3 * b * L * H * P * 2 + 3 * b * L * N * 2 + 2 * 4 * b * L * H
                                 + 2 * 4 * b * H * P * N + 2 * 2 * ns)


def test_backward_bytes():
    # 130M layer, bf16, no initial state: x, dy, B, C (bf16) and dt read; dx, ddt,
    # dB, dC (fp32) and the initial state's gradient written
    b, L, H, P, N = 8, 2048, 24, 64, 128
    reads = b * L * (2 * H * P * 2 + 2 * N * 2 + 4 * H)
    writes = b * L * (H * P * 4 + 4 * H + 2 * N * 4)
    assert bench.bwd_bytes(inputs.LAYER_130M) == reads + writes + 4 * b * H * P * N == 235929600


def test_traffic_records_follow_code_not_comments():
    """A recorded DRAM traffic figure stays valid while a kernel's code is
    unchanged: the source hash ignores comments and whitespace, but not code."""
    src = "int f(int a) {\n    // scale\n    return a * 2; /* twice */\n}\n"
    same = "int f(int a) {   return a * 2;\n}  // reworded comment\n"
    other = "int f(int a) {\n    return a * 3;\n}\n"
    assert bench.code_text(src) == bench.code_text(same)
    assert bench.code_text(src) != bench.code_text(other)
