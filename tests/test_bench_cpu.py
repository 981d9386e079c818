"""Host-side checks of bench.py: the algorithmic work behind the roofline line and
the reference arm's JSON contract (the fp64 oracle on the host, tiny workload)."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_ffn_expert_b200.metrics import kernel_work, layer_bytes, layer_flops  # noqa: E402
from mixture_experts_ffn_expert_b200.inputs import WORKLOADS  # noqa: E402


def test_kernel_work_of_the_routed_gemms():
    s = WORKLOADS["coarse_t4096_d4096_f14336_e8k2_s0"]
    T, d, f, k = s.T, s.d, s.f, s.top_k
    A = T * k
    fl, by = kernel_work("grouped_gate_up", s, T, 8)
    assert fl == 4 * A * d * f == 1924145348608
    assert by == 8 * 2 * f * d * 2 + 2 * A * d + 2 * A * f == 2181038080
    # variant tags do not change the work
    assert kernel_work("grouped_down[pair512]", s, T, 8) == \
        (2 * A * d * f, 8 * d * f * 2 + 2 * A * f + 2 * A * d)
    # weight bytes count touched experts only
    s4 = WORKLOADS["dsv3_prefill_t4096_d7168_f2048_e256k8_s1"]
    _, by250 = kernel_work("grouped_gate_up", s4, s4.T, 250)
    _, by256 = kernel_work("grouped_gate_up", s4, s4.T, 256)
    assert by256 - by250 == 6 * 4 * s4.d * s4.f


def test_shared_and_merged_work():
    s = WORKLOADS["dsmoe_small_t8192_d2048_f1408_e64k6_s2"]
    nsf = s.n_shared * s.f
    assert kernel_work("shared_gate_up", s, s.T, 64)[0] == 4 * s.T * s.d * nsf
    merged = kernel_work("grouped_gate_up[+shared]", s, s.T, 64)
    plain = kernel_work("grouped_gate_up", s, s.T, 64)
    shared = kernel_work("shared_gate_up", s, s.T, 64)
    assert merged == (plain[0] + shared[0], plain[1] + shared[1])


def test_reference_arm_prints_one_contract_line():
    out = io.StringIO()
    with redirect_stdout(out):
        rc = bench.main(["--impl", "reference", "--workload", "tiny_t256_d128_f64_e31k7_s1",
                         "--steps", "2", "--warmup", "3"])
    assert rc == 0
    lines = [l for l in out.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_t256_d128_f64_e31k7_s1"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_layer_work_matches_the_page_budget():
    # the page's budget rule: an expert costs 3*d*f multiply-adds per token, so the
    # active FLOPs are 2 * T * 3*d*f*(k + N_s) plus the router's 2*T*d*N_r
    from mixture_experts_ffn_expert_b200.inputs import LayerShape
    s = LayerShape("toy", 1, 128, 256, 8, 2, 0, True)
    assert layer_flops(s) - 2 * s.d * s.n_routed == 2 * 196608
    s1 = LayerShape("toy1", 1, 128, 64, 31, 7, 1, True)
    assert layer_flops(s1) - 2 * s1.d * s1.n_routed == 2 * 196608
    # bytes: x in and out, router, shared and touched routed weights, bf16
    assert layer_bytes(s1, 7) == 2 * (2 * 128 + 31 * 128 + 3 * 128 * 64 * (1 + 7))


def test_roofline_uses_the_burst_peak_for_tensor_bound_work():
    peaks = {"hbm_gbs": 6547.2, "bf16_tflops": 1646.1, "bf16_tflops_sustained": 1391.6}
    r = bench.roofline_of(1.0e12, 1.0e9, 1.0e-3, peaks, "measured")
    assert r["bound"] == "tensor" and r["peak"] == 1646.1
    assert abs(r["frac"] - 1000.0 / 1646.1) < 1e-4
    h = bench.roofline_of(1.0e9, 1.0e9, 1.0e-3, peaks, "measured")
    assert h["bound"] == "hbm" and h["unit"] == "GB/s" and abs(h["achieved"] - 1000.0) < 1e-6
