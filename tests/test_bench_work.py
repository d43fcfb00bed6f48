"""The algorithmic work that every roofline fraction in bench.py divides by,
restated here from its definition for the three bf16 workloads (values worked
out by hand, not by calling the same formula): forward 1,296 bytes and
294,912 flops per token-head at d = 128, C = 64 (q, k, v, o, vtilde in bf16 and
four fp32 gates; 12 C d + 12 d^2), plus 64 KiB per fp32 state matrix per head
(S_T and M_T written, S0 and M0 read when the workload has them); backward
2,592 bytes and 688,128 flops per token-head (q, k, vtilde, d_o in bf16 and four
fp32 gates read, dq, dk, dv and four gate gradients written in fp32;
28 C d + 28 d^2), plus dS0, dM0 written and S0, M0 read when given (the
bench line's 2,656 bytes per token-head at the 400M-layer shape include them)."""
import bench
import mdn_inputs as mi

KIB64 = 128 * 128 * 4


def test_forward_work_layer400m():
    # 4 x 2048 x 8 = 65,536 token-heads, no entering states: S_T, M_T only
    b, f = bench.pass_work(mi.WORKLOADS[1])
    assert b == 65536 * 1296 + 32 * 2 * KIB64 == 89_128_960
    assert f == 65536 * 294_912 == 19_327_352_832


def test_forward_work_layer1p3b():
    # 8 x 4096 x 16 = 524,288 token-heads, entering states given: four matrices per head
    b, f = bench.pass_work(mi.WORKLOADS[2])
    assert b == 524_288 * 1296 + 128 * 4 * KIB64 == 713_031_680
    assert f == 524_288 * 294_912


def test_forward_work_longctx():
    spec = mi.WORKLOADS[3]
    b, f = bench.pass_work(spec)
    heads = spec.B * spec.H
    states = heads * (4 if spec.state_std > 0 else 2) * KIB64
    assert b == 16384 * 16 * 1296 + states
    assert f == 16384 * 16 * 294_912


def test_backward_work_layer400m():
    b, f = bench.bwd_work(mi.WORKLOADS[1])
    assert b == 65536 * 2592 + 32 * 2 * KIB64 == 174_063_616 == 65536 * 2656
    assert f == 65536 * 688_128 == 45_097_156_608
