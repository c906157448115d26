"""The algorithmic byte counts behind bench.py's roofline fractions, against the numbers
worked out by hand for the benchmark's workloads (CPU only)."""
import bench
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS


def test_prefill_bytes_small_bf16():
    # 4096 tokens x (x, z, y: 3 x 2048 + B, C: 2 x 1024 + dt: 32) bf16 values = 67 371 008 B,
    # plus the final SSM state (2 x 32 x 64 x 128 fp32 = 2 097 152 B) and the final conv
    # state (2 x 4096 x 3 bf16 = 49 152 B)
    w = WORKLOADS["small_bf16"]
    assert bench.path_bytes(w, 2, 2048, False) == 69_517_312
    # initial states read too
    assert bench.path_bytes(w, 2, 2048, True) == 69_517_312 + 2_146_304
    assert bench.kernel_bytes("tc_prefill", w, 2, 2048) == 69_517_312


def test_decode_bytes_decode_bf16():
    # the fp32 state read and written (2 x 256 x 128 x 64 x 128 x 4 = 2 147 483 648 B), the
    # conv state read and written (2 x 256 x 10240 x 3 x 2 = 31 457 280 B), and one token's
    # x, z, B, C, dt in and y out (256 x (3 x 8192 + 2 x 1024 + 128) x 2 = 13 697 024 B)
    w = WORKLOADS["decode_bf16"]
    assert bench.decode_bytes(w, 256) == 2_192_637_952
    assert bench.kernel_bytes("decode_step", w, 256, 1) == 2_192_637_952


def test_backward_bytes_small_bf16():
    # x, z, B, C, dt read and their gradients written (2 x (2 x 2048 + 2 x 1024 + 32)) plus dy
    # read (2048), per token, bf16: 4096 x 14 400 x 2 = 117 964 800 B
    assert bench.backward_bytes(WORKLOADS["small_bf16"], 2, 2048) == 117_964_800


def test_headline_step_bytes_long_bf16():
    # per 16384-token call: 16384 x (3 x 16384 + 2 x 1024 + 256) bf16 values = 1 686 110 208 B,
    # plus the final SSM state (256 x 64 x 128 fp32 = 8 388 608 B) and conv state
    # (18432 x 3 bf16 = 110 592 B); the second call also reads the first call's final states;
    # the decode token moves its state twice plus one token's inputs and y
    w = WORKLOADS["long_bf16"]
    call = 1_686_110_208 + 8_388_608 + 110_592
    assert bench.path_bytes(w, 1, 16384, False) == call
    assert bench.path_bytes(w, 1, 16384, True) == call + 8_388_608 + 110_592
    dec = 2 * 8_388_608 + 2 * 110_592 + (3 * 16384 + 2 * 1024 + 256) * 2
    assert bench.decode_bytes(w, 1) == dec
    assert bench.headline_step_bytes(w) == 2 * call + 8_388_608 + 110_592 + dec
