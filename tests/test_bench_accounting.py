"""The bench's roofline accounting on the host: the algorithmic bytes and FLOPs
it divides by, checked against the workload arithmetic written out by hand for
the mid bf16 layer (T=2048, H=2048, I=1024, E=64, top-6, shared I=1024), and the
tensor peak each type is measured against."""

import bench
import synth

MID = synth.get_config("mid_bf16_shared_T2048")


def test_grouped_mlp_algorithmic_mid():
    # every expert touched: W1, W3, W2 of 64 experts and of the shared expert,
    # 2 bytes each; FLOPs: 2 * 3 * H * I per routed row, and per token for the
    # shared expert
    b, f = bench.grouped_mlp_algorithmic(MID, touched=64)
    assert b == 2 * 3 * 2048 * (64 * 1024 + 1024)
    assert f == 6 * 2048 * (2048 * 6 * 1024 + 2048 * 1024)


def test_layer_algorithmic_mid():
    wb, wf = bench.grouped_mlp_algorithmic(MID, 64)
    b, f = bench.layer_algorithmic(MID, 64)
    # + the router weight, x in and y out (bf16); + the router GEMM
    assert b == wb + 2 * 64 * 2048 + 2 * 2 * 2048 * 2048
    assert f == wf + 2 * 2048 * 2048 * 64


def test_backward_algorithmic_mid():
    b, f = bench.backward_algorithmic(MID, 64)
    w_el = 3 * 2048 * (64 * 1024 + 1024) + 64 * 2048  # expert, shared, router weights
    R = 2048 * 6
    # bf16 weights read once, fp32 gradients written once; x, dy, dx (T rows)
    # and the saved rows and fc2 rows (R rows)
    assert b == 2 * w_el + 4 * w_el + 2 * (3 * 2048 * 2048 + 2 * R * 2048)
    # dh, dX and the three weight gradients: 12 * H * I per routed row (and per
    # token for the shared expert); the router's dx and dW_r: 4 * T * H * E
    assert f == 12 * 2048 * (R * 1024 + 2048 * 1024) + 4 * 2048 * 2048 * 64


def test_touched_experts_scale_the_bytes():
    b_all, _ = bench.grouped_mlp_algorithmic(MID, 64)
    b_half, _ = bench.grouped_mlp_algorithmic(MID, 32)
    assert b_all - b_half == 2 * 3 * 2048 * 32 * 1024


def test_block_scaled_bytes_include_their_scales():
    nv = synth.get_config("dsv4_nvfp4_decode_T128")
    b, _ = bench.grouped_mlp_algorithmic(nv, touched=10)
    # e2m1 codes (half a byte) plus one e4m3 scale per 16 elements
    assert b == int((0.5 + 1 / 16) * 3 * 7168 * 10 * 3072)
    mx = synth.get_config("dsv3_mxfp8_shared_T4096")
    b, _ = bench.grouped_mlp_algorithmic(mx, touched=10)
    assert b == int((1 + 1 / 32) * 3 * 7168 * (10 * 2048 + 2048))


def test_tensor_peaks_are_the_measured_ones():
    # the block-scaled types take the library GEMMs' measured peaks, above the
    # bf16 one; bf16 takes the driver's measurement (not in this table)
    assert set(bench.TENSOR_PEAK) == {"mxfp8", "nvfp4"}
    assert 1700 < bench.TENSOR_PEAK["mxfp8"] < bench.TENSOR_PEAK["nvfp4"]
