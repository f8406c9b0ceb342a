"""The work and traffic counts behind the benchmark's numbers (CPU only).

The metric counts the causal triangle only: F = 2 * sum_b n_b (n_b + 1) / 2 *
H * (d_qk + d_v), i.e. one multiply-add per (i, j <= i) pair for q_i . k_j and
one per pair and value column for A_ij v_j.  The roofline's algorithmic bytes
read Q, K, V, U, the tables, timestamps and offsets once and write Y once.
"""
import bench
import hstu_inputs as hi


def brute_force_flops(lengths, H, dqk, dv):
    pairs = 0
    for n in lengths:
        for i in range(n):
            for j in range(n):
                if j <= i:
                    pairs += 1
    return pairs * H * (2 * dqk + 2 * dv)


def test_causal_flops_counts_the_triangle():
    for lengths, H, dqk, dv in [((1,), 1, 1, 1), ((5, 0, 3), 2, 4, 6), ((17, 9), 3, 8, 8)]:
        assert hi.causal_flops(lengths, H, dqk, dv) == brute_force_flops(lengths, H, dqk, dv)


def test_dense_workload_flops_closed_form():
    # B dense sequences of n tokens: B * n (n + 1) * H * (d_qk + d_v)
    for name in ("neurarch", "long", "train", "train_time"):
        w = hi.WORKLOADS[name]
        expect = w.batch * w.seq_len * (w.seq_len + 1) * w.heads * (w.d_qk + w.d_v)
        assert hi.causal_flops([w.seq_len] * w.batch, w.heads, w.d_qk, w.d_v) == expect
    assert hi.causal_flops([1024] * 8, 4, 128, 128) == 8_598_323_200
    assert hi.causal_flops([8192] * 4, 4, 128, 128) == 274_911_461_376
    assert hi.causal_flops([2048] * 16, 4, 128, 128) == 68_753_031_168


def test_neurarch_algorithmic_bytes():
    inp = hi.make_inputs(hi.WORKLOADS["neurarch"], seed=0)
    T, H, d = 8 * 1024, 4, 128
    qkv = 3 * T * H * d * 2            # bf16 Q, K, V
    u_y = 2 * T * H * d * 2            # bf16 U in, Y out
    table = H * (2 * 1024 - 1) * 4     # fp32 position table
    offsets = 9 * 4
    assert bench.algorithmic_bytes(inp) == qkv + u_y + table + offsets == 41_975_828


def test_time_bias_bytes_add_table_and_timestamps():
    spec = hi.workload("train_time", batch=2)
    inp = hi.make_inputs(spec, seed=0)
    T, H, d = 2 * 2048, 4, 128
    expect = 5 * T * H * d * 2 + H * (2 * 2048 - 1) * 4 + H * 128 * 4 + T * 8 + 3 * 4
    assert bench.algorithmic_bytes(inp) == expect
