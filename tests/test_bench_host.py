"""Host-side checks of bench.py's accounting (no GPU): algorithmic FLOPs per block
against the closed form, the workload shapes, and the clock-sample parser."""
import importlib.util
import os

import pytest

from wan_inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_block_flops_match_closed_form(bench):
    w2 = WORKLOADS["wan13b_480p_block"]
    w4 = WORKLOADS["wan14b_720p_block"]
    # QKV 6LD^2, O 2LD^2, cross q 2LD^2, cross o 2LD^2, kv 4 Lc D^2: 12 L D^2 + 4 Lc D^2 in total
    for w in (w2, w4):
        L, D, F, Lc = w.tokens, w.dim, w.ffn, w.text_len
        expect = 12 * L * D * D + 4 * Lc * D * D + 4 * L * L * D + 4 * L * Lc * D + 4 * L * D * F
        assert bench.block_flops(w) == pytest.approx(expect, rel=1e-12)
    assert bench.block_flops(w2) / 1e12 == pytest.approx(9.433, abs=0.002)
    assert bench.block_flops(w4) / 1e12 == pytest.approx(163.08, abs=0.02)
    wi = WORKLOADS["wan13b_480p_i2v_block"]
    extra = 4 * wi.img_len * wi.dim ** 2 + 4 * wi.tokens * wi.img_len * wi.dim + 2 * wi.tokens * wi.dim ** 2
    assert bench.block_flops(wi) - bench.block_flops(w2) == pytest.approx(extra, rel=1e-12)


def test_attention_share_of_block(bench):
    w = WORKLOADS["wan13b_480p_block"]
    attn = 4 * w.tokens ** 2 * w.dim
    assert 0.69 < attn / bench.block_flops(w) < 0.71


def test_clock_sampler_parses_nvidia_smi_lines(bench):
    class P:
        def __init__(self, out):
            self.out = out

        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return self.out, ""
    s = bench.ClockSampler(0)
    s.proc = P("0, 1800, 1965, 900.1, 0x0, Not Active, Not Active, Not Active, Active\n"
               "0, 1400, 1965, 1000.2, 0x4, Not Active, Not Active, Not Active, Active\n"
               "0, 1500, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    r = s.stop()
    assert r["sm_mhz"] == 1500 and r["sm_max_mhz"] == 1965 and r["reasons"] == ["sw_power_cap"] and r["samples"] == 3


def test_peaks_source(bench):
    peaks, src = bench.load_peaks()
    assert peaks["bf16_tflops_sustained"] > 0 and src in ("measured", "fallback")


def test_peak_rule_burst_for_short_regions(bench):
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    assert bench.choose_peak(peaks, "measured", 0.17)["value"] == 1600.0
    assert bench.choose_peak(peaks, "measured", 2.5)["value"] == 1400.0
    assert "burst" in bench.choose_peak(peaks, "measured", 0.5)["source"]


def test_kernel_report_splits_a_step(bench):
    """A synthetic trace of two steps in the launch order of wan_dit_stack_fwd with one
    block: gather, patchify GEMM, time MLP, LN, QKV, self-attention, O, LN, cross q,
    cross kv, cross-attention, cross o, LN, FFN1, FFN2, head LN, head GEMM."""
    import video_diffusion_transformer_wan_b200 as wan
    w = WORKLOADS["wan13b_480p_block"]
    S, G, A, N = wan.KIND_SMALL, wan.KIND_GEMM, wan.KIND_ATTN, wan.KIND_NORM
    sa, ca = 6.594e12, 0.103e12
    step = [(S, 0.01, 1e6), (G, 0.05, 6.4e9), (S, 0.01, 1e6), (N, 0.05, 3e8), (G, 0.4, 4.6e11), (A, 5.5, sa),
            (G, 0.15, 1.5e11), (N, 0.05, 3e8), (G, 0.13, 1.5e11), (G, 0.01, 4e9), (A, 0.2, ca), (G, 0.15, 1.5e11),
            (N, 0.05, 3e8), (G, 0.7, 9e11), (G, 0.7, 9e11), (N, 0.05, 3e8), (G, 0.03, 6.4e9)]
    recs = step * 2
    k, roof, peak = bench.kernel_report(w, recs, 2, 8.5, {"sm_mhz": 1900})
    assert k["self_attention"]["ms_per_step"] == pytest.approx(5.5)
    assert roof["achieved"] == pytest.approx(sa / 5.5e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / peak["value"])
    assert k["cross_attention"]["tflops"] == pytest.approx(ca / 0.2e-3 / 1e12)
    assert k["patchify_gemm"]["ms_per_step"] == pytest.approx(0.05)
    assert k["head_gemm"]["ms_per_step"] == pytest.approx(0.03)
    L, D = w.tokens, w.dim
    assert k["patchify_gemm"]["gbs"] == pytest.approx((L * 64 * 2 + D * 64 * 2 + D * 2 + L * D * 4) / 0.05e-3 / 1e9)
    assert k["head_gemm"]["gbs"] == pytest.approx((L * D * 2 + 64 * D * 2 + 64 * 2 + L * 64 * 4) / 0.03e-3 / 1e9)
    assert k["gemm"]["ms_per_step"] == pytest.approx(0.4 + 0.15 + 0.13 + 0.01 + 0.15 + 0.7 + 0.7)
    assert k["layernorm"]["gbs"] == pytest.approx(4 * 3e8 / 0.2e-3 / 1e9)
    with pytest.raises(RuntimeError):
        bench.kernel_report(w, recs[:-1], 2, 8.5, {"sm_mhz": 1900})


def test_kernel_report_per_launch_roofline_with_several_blocks(bench):
    """A stack step runs one self-attention per block: the roofline entry is per launch
    (the step's self-attention time divided by the launches), the per-kind entry per step."""
    import video_diffusion_transformer_wan_b200 as wan
    w = WORKLOADS["wan13b_480p_stack30"]
    G, A, N = wan.KIND_GEMM, wan.KIND_ATTN, wan.KIND_NORM
    sa, ca = 6.594e12, 0.103e12
    block = [(N, 0.05, 3e8), (G, 0.4, 4.6e11), (A, 5.5, sa), (G, 0.15, 1.5e11), (A, 0.2, ca), (G, 0.7, 9e11)]
    step = [(G, 0.05, 6.4e9)] + block * 3 + [(G, 0.03, 6.4e9)]
    k, roof, _ = bench.kernel_report(w, step * 2, 2, 20.0, {"sm_mhz": 1900})
    assert k["self_attention"]["ms_per_step"] == pytest.approx(3 * 5.5)
    assert k["self_attention"]["tflops"] == pytest.approx(sa / 5.5e-3 / 1e12)
    assert roof["ms_per_launch"] == pytest.approx(5.5)
    assert roof["achieved"] == pytest.approx(sa / 5.5e-3 / 1e12)


def test_attention_traffic_only_for_the_profiled_launch_shape(bench):
    """The committed ncu traffic is reported for workloads whose self-attention launch
    has the captured shape (batch 1, 32760 tokens, 12 heads) and for no other."""
    t = bench.attn_traffic_per_launch(WORKLOADS["wan13b_480p_block"])
    assert bench.attn_traffic_per_launch(WORKLOADS["wan14b_720p_block"]) is None
    if t is not None:   # None when attn_tc.cu changed since the capture
        assert t > 0
        assert bench.attn_traffic_per_launch(WORKLOADS["wan13b_480p_stack30"]) == t
        assert bench.attn_traffic_per_launch(WORKLOADS["wan13b_480p_i2v_block"]) == t


def test_code_hash_follows_code_not_comments(bench, tmp_path):
    """The profile's traffic stays valid across comment edits and lapses on a code edit."""
    a = tmp_path / "a.cu"
    a.write_text("// header\nint f(int x) {  // trailing\n  return x + 1;\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("// another header\n\nint f(int x) {\n  return x + 1;   // changed comment\n}\n")
    c = tmp_path / "c.cu"
    c.write_text("// header\nint f(int x) {\n  return x + 2;\n}\n")
    assert bench.code_sha256(str(a)) == bench.code_sha256(str(b))
    assert bench.code_sha256(str(a)) != bench.code_sha256(str(c))
