"""Host-side pieces of bench.py that need no GPU: the committed-profile lookup and the
bounded oracle sample of the reference arm."""
import hashlib
import os

import bench


def test_profile_traffic_follows_the_kernel_source():
    # a summary counts only while its recorded source hash matches the current kernel
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    text = open(os.path.join(root, "profiles", "kv_quant_traffic_kvcache.md")).read()
    src = open(os.path.join(root, "ternary_weight_bit_b200", "csrc", "kv_quant.cu"), "rb").read()
    recorded = text.split("source_sha256 = ")[1].split()[0]
    got = bench.profile_traffic("kv_quant_traffic_kvcache", "kv_quant.cu")
    if recorded == hashlib.sha256(src).hexdigest():
        assert got is not None and got > 0
    else:
        assert got is None
    assert bench.profile_traffic("no_such_profile", "kv_quant.cu") is None
    assert bench.profile_traffic("kv_quant_traffic_kvcache", "gemv.cu") is None  # other source, other hash


def test_algorithmic_bytes():
    act, gemm = bench.algorithmic_bytes(2, 256, 512, "f32")
    assert act == 2 * 512 * 4 + 2 * 512 + 4 * 2
    assert gemm == 256 * 512 // 4 + 2 * 512 + 4 * 2 + 4 * 2 * 256 + 4
    _, gemm16 = bench.algorithmic_bytes(2, 256, 512, "f32", out_bytes=2)
    assert gemm - gemm16 == 2 * 2 * 256


def test_oracle_sample_is_bounded_and_extrapolated():
    cases = [("t", 24, 384, 512, "int8", True, "normal", "f32", 0),
             ("u", 40, 256, 1024, "int4", True, "student_t3", "f32", 3)]
    rate, desc, done, per_step = bench.time_oracle(cases, budget_s=0.5, steps=3)
    assert done == 3 and rate > 0 and per_step > 0
    assert "extrapolated" in desc and "tokens" in desc
    rate_bf16, _, _, _ = bench.time_oracle(cases, budget_s=0.5, steps=2, bf16_out=True)
    assert rate_bf16 > 0


def test_batches_per_step_spans_the_minimum_step():
    assert bench.batches_per_step(0.66, 5.0) == 8        # default workload: 8 passes of 0.66 ms
    assert bench.batches_per_step(0.035, 5.0) == 143     # decode: 143 passes of 35 us
    assert bench.batches_per_step(7.0, 5.0) == 1         # a pass longer than the minimum
    assert bench.batches_per_step(0.0, 5.0) == bench.MAX_BATCHES  # no pass time measured: capped
    for pass_ms in (0.011, 0.2, 1.3, 4.9):
        b = bench.batches_per_step(pass_ms, 5.0)
        assert b * pass_ms >= 5.0 or b == bench.MAX_BATCHES
        assert (b - 1) * pass_ms < 5.0


def test_workloads_satisfy_the_boundary_rules():
    # every bench case passes the ABI's shape rules: K % 128 == 0, K <= 32768, FWHT needs a
    # power-of-two K, and the decode workloads stay on the GEMV (M <= 16)
    for name in ("decode", "decode_tl2", "prefill", "wdown", "wdown_swiglu", "msweep_M8", "msweep_M64",
                 "msweep_M512", "msweep_M4096", "msweep_M8192"):
        for (label, M, N, K, mode, fwht, xk, xdt, outl) in bench.workload_cases(name):
            assert K % 128 == 0 and K <= 32768, (name, label)
            assert not fwht or (K & (K - 1)) == 0, (name, label)
            assert mode in ("int8", "int4") and xdt in ("f32", "bf16") and M >= 1 and N >= 1
            if name.startswith("decode"):
                assert M <= 16
    assert bench.workload_cases(bench.DEFAULT_WORKLOAD) == bench.workload_cases("msweep_M8192")
