"""The benchmark's roofline numerators: API-level bytes and flops per token of each workload,
checked against counts written out here from the workloads' shapes (one term per tensor the call
reads or writes), and the roofline arithmetic itself.  CPU only."""
import bench
from gated_delta_rule_76_b200.inputs import WORKLOADS

H, D, C = 16, 128, 64
BF16, F32 = 2, 4


def test_gdn2_forward_and_backward_bytes_per_token():
    wl = WORKLOADS["gdn2_fwd_bwd_bf16"]
    row = H * D * BF16                      # one bf16 [H, d] tensor of one token
    state_per_token = H * D * D * F32 / wl.T  # one fp32 state set, amortised over the sequence
    # forward: q, k, v, alpha, b, w read, o written; h0 read, hT written
    fwd = 7 * row + 2 * state_per_token
    assert bench.fwd_bytes_per_token(wl) == fwd == 29184  # the 29.2 KB of the GDN-2 forward row
    # backward: q, k, v, alpha, b, w, dO read; dq, dk, dv, dalpha, db, dw written in the inputs'
    # dtypes; h0 read, dh0 written (the benchmark's step passes no gradient of the final state)
    bwd = 7 * row + 6 * row + 2 * state_per_token
    assert bench.bwd_bytes_per_token(wl) == bwd == 53760
    tokens = wl.B * wl.T
    assert (fwd + bwd) * tokens == 2717908992  # the step's numerator


def test_scalar_gate_forward_bytes_per_token():
    wl = WORKLOADS["gdn_fwd_scalar_bf16"]
    row = H * D * BF16
    # q, k, v read, o written (bf16); alpha and beta: one fp32 scalar per head; hT written (no h0)
    want = 4 * row + 2 * H * F32 + H * D * D * F32 / wl.T
    assert bench.fwd_bytes_per_token(wl) == want == 16768


def test_flops_per_token():
    wl = WORKLOADS["gdn2_fwd_bwd_bf16"]
    fwd_head = 5 * 2 * C * D + 3 * 2 * D * D  # five C x d products and three d x d ones a token
    assert bench.fwd_flops_per_token(wl) == H * fwd_head == H * 180224
    assert bench.bwd_flops_per_token(wl) == H * (2 * fwd_head + 4 * C * C) == H * 376832


def test_decode_bytes_per_sequence_step():
    wl = WORKLOADS["gdn2_decode_bf16"]
    state = H * D * D * F32 * 2                     # the fp32 state read and written
    io = (2 * H * D + 2 * H * D) * BF16 + (H * D + 2 * H * D) * BF16  # q, k, v, o; alpha, b, w
    assert bench.decode_bytes_per_token(wl) == state + io == 2125824  # 2.13 MB a sequence-step
    assert bench.decode_bytes_per_token(wl) * wl.B == 544210944


def test_roofline_arithmetic():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 80.0}
    # 1 GB in 2 ms is 500 GB/s, half the peak; 1 GFLOP would take 10 us at 100 TFLOP/s: HBM-bound
    r = bench.roofline(1e9, 1e9, 2e-3, peaks, "measured", "x", traffic=3e9)
    assert r["bound"] == "hbm" and r["achieved"] == 500.0 and r["frac"] == 0.5
    assert r["traffic"] == 3000000000 and r["algorithmic_bytes"] == 1000000000
    # 1 MB and 10 TFLOP in 0.5 s: tensor-bound at 20 TFLOP/s, a fifth of the burst peak
    r = bench.roofline(1e6, 1e13, 0.5, peaks, "measured", "x")
    assert r["bound"] == "tensor" and r["achieved"] == 20.0 and r["frac"] == 0.2 and r["traffic"] is None
    # the sustained peak for kernels timed inside a long step
    r = bench.roofline(1e6, 1e13, 0.5, peaks, "measured", "x", sustained=True)
    assert r["peak"] == 80.0 and r["frac"] == 0.25
