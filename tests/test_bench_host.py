"""Host-side logic of bench.py (no GPU): the accounting the reported numbers
divide by, and the reference arm's JSON line.

* weight bytes per pass = the stored size of the encoding, 4.127 bits per
  weight ("第 04 篇：QLoRA 原理" §5.3: 4-bit codes + 8-bit block scales +
  fp32 second-level scales), equal to the oracle's unpadded storage size;
* encoding bytes = the fp32 weight read once plus the stored encoding;
* the algorithmic flops of the full-backward workloads match the totals the
  layer formulas give (2MKN + 2Mr(K+N) forward, 2MKN + 4Mr(K+N) backward);
* `--impl reference` prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

import pytest

import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("d_out,d_in", [(512, 512), (4096, 4096), (11008, 4096), (8192, 22016)])
def test_weight_bytes_are_the_stored_encoding(d_out, d_in):
    n = d_out * d_in
    assert bench.weight_bytes(d_out, d_in) == pytest.approx(oracle.packed_bytes(n) - 4, abs=4)
    assert 8 * bench.weight_bytes(d_out, d_in) / n == pytest.approx(4 + 1 / 8 + 1 / 512, rel=1e-9)
    assert bench.quantize_bytes(d_out, d_in) == 4 * n + oracle.packed_bytes(n)


def test_full_backward_flops_follow_the_layer_formulas():
    for name in ("llama7b_mlp_r64_m4096", "llama7b_layer_r16_m8192", "llama65b_layer_r64_m2048"):
        wl = workloads.WORKLOADS[name]
        _, flops = bench.step_totals(wl)
        expect = 0
        for mod in wl.modules:
            for m in wl.tokens:
                K, N, r = mod.d_in, mod.d_out, wl.r
                expect += (2 * m * K * N + 2 * m * r * (K + N)) + (2 * m * K * N + 4 * m * r * (K + N))
        assert flops == expect
    # the SwiGLU MLP at 4096 tokens, r = 64: 2.288 TFLOP per step
    assert bench.step_totals(workloads.WORKLOADS["llama7b_mlp_r64_m4096"])[1] == pytest.approx(2.288e12, rel=1e-3)


def test_default_step_is_six_passes_over_the_weight():
    wl = workloads.WORKLOADS["q_proj4096_r64_m1-4-16"]
    plan = bench.step_plan(wl)
    assert [(m, k) for _, _, m, k in plan] == [(1, "fwd"), (1, "dx"), (4, "fwd"), (4, "dx"), (16, "fwd"), (16, "dx")]
    b, _ = bench.step_totals(wl)
    assert b > 6 * bench.weight_bytes(4096, 4096)


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    # the default workload is the LLaMA-65B layer's linears, a tensor-bound step
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"] == bench.workload_config(workloads.WORKLOADS["llama65b_layer_r64_m2048"], 1)


def test_both_arms_time_the_same_oracle_sample():
    """cpu_baseline (GPU arm) and the reference arm describe one sample and
    one config: the same rows of the same module, the same keys."""
    for name, wl in workloads.WORKLOADS.items():
        mod = wl.modules[0]
        rows = bench.oracle_rows(mod)
        assert rows * mod.d_in % (64 * 256) == 0 or rows == mod.d_out
        assert rows <= mod.d_out
        assert bench.oracle_unit(wl) == ("TFLOP/s" if max(wl.tokens) > 16 else "GB/s")
        assert bench.workload_config(wl, 1) == bench.workload_config(wl, 1)


def test_kernel_flops_split_the_pass_flops():
    """The fused forward and input-gradient kernels carry the base product and
    their own rank-r term; with the LoRA-down / V products (2 M r K, 2 M r N)
    they add up to the pass flops of the layer formulas."""
    for K, N, m, r in ((4096, 11008, 4096, 64), (8192, 8192, 2048, 64), (512, 512, 16, 8)):
        fwd = bench.kernel_flops(N, K, m, r, "nf4_gemm_fwd")
        dx = bench.kernel_flops(N, K, m, r, "nf4_gemm_dx")
        assert fwd + 2 * m * r * K == bench.pass_flops(N, K, m, r, "fwd")
        assert dx + 2 * m * r * N == bench.pass_flops(N, K, m, r, "dx")
