"""bench.py's roofline arithmetic on CPU: the algorithmic byte and FLOP counts it divides by
the measured time, against the figures the kernels' documentation derives by hand."""
import bench


def test_prefill_bytes_1p5b_layer():
    # 640 B per token-head (r, k, v, omega in, y out, bf16) + 32 KB state per head + u
    assert bench.prefill_bytes(8, 4096, 32) == 8 * 4096 * 32 * 640 + 256 * 32768 + 32 * 64 * 4
    assert bench.prefill_bytes(8, 4096, 32) == 679_485_440


def test_decode_bytes():
    # 33,408 B per head-step (fp32 state read + written, 5 bf16 vectors) + u
    assert bench.decode_bytes(256, 32) == 256 * 32 * 33_408 + 32 * 64 * 4
    assert bench.decode_bytes(256, 32) == 273_686_528


def test_backward_counts():
    # three recurrences, 5 FLOPs per state entry per token (readout FMA, update mul + FMA)
    assert bench.backward_flops(8, 4096, 32) == 3 * 5 * 64 * 64 * 8 * 4096 * 32
    assert abs(bench.backward_flops(8, 4096, 32) / 1e9 - 64.42) < 0.01
    # 9 bf16 vectors per token-head, 3 fp32 states per head, u and du
    assert bench.backward_bytes(8, 4096, 32) == 9 * 128 * 8 * 4096 * 32 + 3 * 16384 * 256 + 2 * 32 * 256


def test_alu_peak():
    # 148 SMs x 128 FP32 lanes x 2 FLOPs per FMA x 1.965 GHz
    assert abs(bench.ALU_FP32_TFLOPS - 74.45) < 0.01
