"""The measurement rules of bench.py on CPU: which roofline a kernel is rated
against, when L2 is flushed between timed decodes, and the output check that
refuses a line whose timed outputs disagree with the oracle rows."""
import numpy as np

import bench
from mla_decode_attention_11_b200 import workloads as W

PEAKS = {"hbm_gbs": 6552.6, "bf16_tflops": 1659.7}


def test_mma_tensor_peak_by_operand_type():
    assert bench.mma_tensor_peak(PEAKS, e4m3_mma=False) == PEAKS["bf16_tflops"]
    # E4M3 operands: twice the bf16 rate (nominal 4.5 vs 2.25 PFLOP/s dense)
    assert bench.mma_tensor_peak(PEAKS, e4m3_mma=True) == 2 * PEAKS["bf16_tflops"]


def test_roofline_point_sides_of_the_ridge():
    # the headline decode in bf16: 235 flop/B, below the ridge of 253 -> HBM
    w = W.WORKLOADS["metric"]
    import torch
    sl = torch.full((w.B,), w.L, dtype=torch.int32)
    flops, nbytes = w.algorithmic_flops(sl), w.algorithmic_bytes(sl)
    bound, achieved, peak, unit = bench.roofline_point(flops, nbytes, 0.150, PEAKS["hbm_gbs"],
                                                       bench.mma_tensor_peak(PEAKS, False))
    assert (bound, peak, unit) == ("hbm", PEAKS["hbm_gbs"], "GB/s")
    assert abs(achieved - nbytes / 150e-6 / 1e9) < 1e-6 * achieved
    # the long split-KV decode (256 query rows per kv row): tensor-bound
    wl = W.WORKLOADS["long"]
    sll = torch.full((wl.B,), wl.L, dtype=torch.int32)
    b2, a2, p2, u2 = bench.roofline_point(wl.algorithmic_flops(sll), wl.algorithmic_bytes(sll), 0.270,
                                          PEAKS["hbm_gbs"], bench.mma_tensor_peak(PEAKS, False))
    assert (b2, p2, u2) == ("tensor", PEAKS["bf16_tflops"], "TFLOP/s")
    assert abs(a2 - wl.algorithmic_flops(sll) / 270e-6 / 1e12) < 1e-6 * a2
    # the headline over an FP8 cache: half the bytes, but the E4M3 peak doubles
    # the ridge (507 flop/B) and 456 flop/B stays below it -> HBM
    fb = w.algorithmic_bytes_fp8(sl)
    b3, _, p3, _ = bench.roofline_point(flops, fb, 0.140, PEAKS["hbm_gbs"], bench.mma_tensor_peak(PEAKS, True))
    assert (b3, p3) == ("hbm", PEAKS["hbm_gbs"])
    # rated against the bf16 peak instead it would have read as tensor-bound
    b4, _, _, _ = bench.roofline_point(flops, fb, 0.140, PEAKS["hbm_gbs"], bench.mma_tensor_peak(PEAKS, False))
    assert b4 == "tensor"


def test_l2_flush_rule():
    l2 = 126.5e6
    assert bench.needs_flush(75e6, l2)          # DeepSeek-V3 shape, bf16 cache
    assert bench.needs_flush(38e6, l2)          # the same over its FP8 cache
    assert not bench.needs_flush(604e6, l2)     # headline, bf16
    assert not bench.needs_flush(302e6, l2)     # headline, FP8: more than twice L2
    assert "flushed" in bench.flush_note(75e6, l2)


def test_output_check_accepts_and_refuses():
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((8, 512))
    lse = rng.standard_normal(8)
    ok = bench.compare_rows(ref.astype(np.float32), lse.astype(np.float32), ref, lse)
    assert ok["ok"] and ok["rows"] == 8
    off = ref.copy()
    off[3, 7] += 0.05  # beyond the 2e-2 max-abs bound
    assert not bench.compare_rows(off, lse, ref, lse)["ok"]
    nan = ref.copy()
    nan[0, 0] = np.nan
    assert not bench.compare_rows(nan, lse, ref, lse)["ok"]
    bad_lse = lse.copy()
    bad_lse[2] += 0.01  # beyond the 1e-3 lse bound
    assert not bench.compare_rows(ref, bad_lse, ref, lse)["ok"]
