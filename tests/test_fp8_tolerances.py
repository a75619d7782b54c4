"""The FP8 parity bars of the GPU tests are reproducible: the reduced form of the study
that derives them (``fp8_tolerance_study.py``: the oracle's FP8 results with their
quantiser inputs moved by one bf16 rounding step, and the 8-bit attention under the
running base) stays below 1/1.5 of every bar in ``gpu_util``."""
import gpu_util as G
import fp8_tolerance_study as S


def test_bar_rounding():
    assert S.bar(0.033) == 0.05
    assert abs(S.bar(0.021) - 0.032) < 1e-12
    assert abs(S.bar(0.0143) - 0.022) < 1e-12


def test_fp8_bars_cover_the_reduced_study():
    res = S.study(full=False, log=lambda *a: None)
    assert set(res) == {"FP8_TOL", "FP8A_BLOCK_TOL", "FP8_STACK_TOL", "FP8_SAMPLE_TOL", "FP8_ATTN_DEF_GAP",
                        "FP8_ATTN_RB_TOL"}
    assert res["FP8_ATTN_DEF_GAP"][1] > 0.0          # the two bases do differ in the subnormal range
    for name, (worst_max, worst_rms) in res.items():
        if name == "FP8_ATTN_DEF_GAP":
            continue
        assert getattr(G, name + "_MAX") >= 1.5 * worst_max, (name, worst_max)
        assert getattr(G, name + "_RMS") >= 1.5 * worst_rms, (name, worst_rms)
