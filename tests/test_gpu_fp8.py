"""GPU parity of the FP8-cache entry point (mla_decode_plan_fp8 /
mla_decode_run_fp8) against the fp64 oracle's FP8 definition: E4M3 codes,
value = kv_scale * e4m3(code), q bf16.  The three FP8 kernels (the codes as
kind::f8f6f4 MMA operands on a CTA pair and in the transposed orientation, the
defaults, and the widening kernel), every group size (16, 32 and 128 query
rows), unsplit and split sequences, lengths
around tile edges, empty sequences, sinks, every finite code, full sizes on
sampled rows.  Rows past a length hold the NaN code (NaN to the oracle,
+-480 * kv_scale to the widening kernel, NaN to the operand kernel; both require
finite codes), so a read past a length would break parity.  Tolerances as in test_gpu_parity (the
cache values are exact in both kernels; q carries about 12 significant bits in
the transposed operand kernel, about 8 in the pair kernel, and P about 8, the
precision of the bf16 path's P)."""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_11_b200 import binding as M
from mla_decode_attention_11_b200 import workloads as W
from tests.test_gpu_parity import OUT_MAX_ABS, assert_parity

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


# the FP8 kernels these tests cover: the codes as MMA operands on a CTA pair (the
# default when Sq*H % 128 == 0) and in the transposed orientation (the default
# otherwise), and the widening kernel
FP8_KERNELS = [M.MLA_KERNEL_FP8_PAIR, M.MLA_KERNEL_FP8_MMA, M.MLA_KERNEL_FP8]


def gpu_decode_fp8(q, codes, ks, sl, scale, num_partitions=0, sinks=None, kernel=M.MLA_KERNEL_FP8_MMA):
    if kernel == M.MLA_KERNEL_FP8_PAIR and (q.shape[1] * q.shape[2]) % 128 != 0:
        pytest.skip("the CTA-pair FP8 kernel runs 128-row query groups (Sq*H % 128 == 0)")
    plan = M.mla_decode_plan_fp8(q.shape[0], q.shape[1], q.shape[2], codes.shape[1], device=0,
                                 num_partitions=num_partitions, kernel=kernel)
    assert plan.kernel == kernel
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.full((q.shape[0], q.shape[1], q.shape[2], 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=DEV)
    sk = None if sinks is None else torch.from_numpy(sinks).to(DEV)
    M.mla_decode_run_fp8(plan, q.to(DEV), codes.to(DEV), ks, sl.to(torch.int32).to(DEV), scale, out, lse, ws,
                         sinks=sk)
    M.mla_decode_check(plan, ws)
    return out.cpu(), lse.cpu(), plan


def check_fp8(w, num_partitions=0, lengths=None, sinks=None, out_max_abs=OUT_MAX_ABS, kernel=M.MLA_KERNEL_FP8_MMA):
    q, codes, ks, sl = W.generate_fp8(w, lengths=lengths)
    out, lse, plan = gpu_decode_fp8(q, codes, ks, sl, w.scale, num_partitions, sinks, kernel)
    ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale, sinks=sinks)
    if sinks is not None:
        # rows whose lse is a finite sink logit are not "empty" for assert_parity
        assert np.array_equal(np.isneginf(lse.numpy()), np.isneginf(rl))
    return assert_parity(out, lse, ro, rl, w.name + " fp8", out_max_abs=out_max_abs), plan


SMALL = {
    "tiny": W.WORKLOADS["tiny"],
    "dsv3": W.small_variant(W.WORKLOADS["dsv3"], B=3, L=1000),
    "mixed": W.small_variant(W.WORKLOADS["mixed"], B=6, L=2100, L_lo=100),
    "lowhead": W.small_variant(W.WORKLOADS["lowhead"], B=20, L=3001),
    "long": W.small_variant(W.WORKLOADS["long"], B=1, L=5000),
}


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("name", sorted(SMALL))
def test_fp8_small_workloads(cuda_device, name, kernel):
    _, plan = check_fp8(SMALL[name], kernel=kernel)
    if kernel == M.MLA_KERNEL_FP8_PAIR:
        assert plan.group_rows == 128
    else:
        assert plan.group_rows == (16 if SMALL[name].Sq * SMALL[name].H == 16 else 32)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("parts", [1, 2, 37, 300])
@pytest.mark.parametrize("H", [16, 128])
def test_fp8_forced_partitions(cuda_device, parts, H, kernel):
    check_fp8(W.custom(B=5, Sq=1, H=H, L=1500, L_lo=1, seed=131), num_partitions=parts, kernel=kernel)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 128, 129, 255, 257, 1023])
def test_fp8_lengths_around_tile_edges(cuda_device, L, kernel):
    if kernel == M.MLA_KERNEL_FP8_PAIR:
        check_fp8(W.custom(B=2, Sq=1, H=128, L=L, seed=142 + L), kernel=kernel)
        return
    check_fp8(W.custom(B=2, Sq=1, H=16, L=L, seed=140 + L), kernel=kernel)
    check_fp8(W.custom(B=1, Sq=1, H=64, L=L, seed=141 + L), kernel=kernel)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("H", [16, 128])
def test_fp8_empty_and_mixed_lengths(cuda_device, H, kernel):
    w = W.custom(B=6, Sq=1, H=H, L=700, seed=152)
    lengths = torch.tensor([0, 1, 700, 0, 129, 5], dtype=torch.int32)
    check_fp8(w, lengths=lengths, kernel=kernel)
    check_fp8(w, lengths=lengths, num_partitions=3, kernel=kernel)
    check_fp8(w, lengths=torch.zeros(6, dtype=torch.int32), kernel=kernel)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
def test_fp8_many_short_sequences(cuda_device, kernel):
    """Far more sequences than partitions, about a tenth of them empty: every
    partition walks several whole sequences plus cut pieces at its ends."""
    B, L = 600, 512
    w = W.custom(B=B, Sq=1, H=128, L=L, seed=760)
    g = torch.Generator().manual_seed(761)
    lengths = torch.randint(1, L + 1, (B,), generator=g, dtype=torch.int32)
    lengths[torch.rand(B, generator=g) < 0.1] = 0
    check_fp8(w, lengths=lengths, kernel=kernel)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("H,Sq", [(16, 2), (32, 1), (64, 3), (128, 2)])
def test_fp8_head_and_token_counts(cuda_device, H, Sq, kernel):
    check_fp8(W.custom(B=2, Sq=Sq, H=H, L=600, seed=160 + H + Sq), kernel=kernel)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("H,parts", [(16, 0), (16, 7), (128, 0), (128, 9)])
def test_fp8_sinks(cuda_device, H, parts, kernel):
    g = np.random.default_rng(170 + H)
    s = g.normal(0.0, 2.0, size=H).astype(np.float32)
    s[0], s[1], s[2] = -np.inf, 30.0, -50.0
    w = W.custom(B=4, Sq=1, H=H, L=900, seed=171)
    lengths = torch.tensor([900, 0, 333, 17], dtype=torch.int32)
    check_fp8(w, num_partitions=parts, lengths=lengths, sinks=s, kernel=kernel)


@pytest.mark.parametrize("kernel", FP8_KERNELS)
def test_fp8_every_finite_code(cuda_device, kernel):
    """Uniformly random codes over all 254 finite E4M3 values (subnormals, both
    zeros, +-448) with a power-of-two scale.  Values span 2^-9 .. 448 times the
    scale, so the max-abs bound is scaled by max(1, max|ref|) as in the
    large-score test of test_gpu_parity."""
    for H, seed in ((16, 180), (128, 181)):
        if kernel == M.MLA_KERNEL_FP8_PAIR and H != 128:
            continue
        g = torch.Generator().manual_seed(seed)
        B, L = 2, 700
        codes = torch.randint(0, 256, (B, L, 576), generator=g, dtype=torch.int64).to(torch.uint8)
        codes[(codes == 0x7F) | (codes == 0xFF)] = 0x00
        q = (torch.randn(B, 1, H, 576, generator=g) * 0.05).to(torch.bfloat16)
        sl = torch.tensor([L, 411], dtype=torch.int32)
        codes[1, 411:] = W.E4M3_NAN_CODE
        ks, scale = 2.0 ** -7, W.custom(1, 1, 16, 1).scale
        out, lse, _ = gpu_decode_fp8(q, codes, ks, sl, scale, kernel=kernel)
        ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, scale)
        assert_parity(out, lse, ro, rl, f"all codes H{H}",
                      out_max_abs=OUT_MAX_ABS * max(1.0, float(np.abs(ro).max())))


@pytest.mark.parametrize("kernel", FP8_KERNELS)
def test_fp8_large_scale_and_rescale(cuda_device, kernel):
    """A kv_scale that makes the scaled scores span tens of units: the lazy
    online rescale runs on the FP8 path too."""
    w = W.custom(B=2, Sq=1, H=128 if kernel == M.MLA_KERNEL_FP8_PAIR else 16, L=2000, sigma=3.0, seed=190)
    q, codes, ks, sl = W.generate_fp8(w)
    out, lse, _ = gpu_decode_fp8(q, codes, ks, sl, w.scale, kernel=kernel)
    ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale)
    assert_parity(out, lse, ro, rl, "fp8 sigma 3", out_max_abs=OUT_MAX_ABS * max(1.0, float(np.abs(ro).max())))


@pytest.mark.parametrize("kernel", FP8_KERNELS)
def test_fp8_rising_scores_force_rescale(cuda_device, kernel):
    """Keys whose scores rise along the sequence by ~13.5 (log2 units) per
    128-key tile: every tile outgrows the reference max by more than any lazy
    threshold, so the FP8 kernels rescale O on every tile."""
    H = 128 if kernel == M.MLA_KERNEL_FP8_PAIR else 16
    w = W.custom(B=1, Sq=1, H=H, L=1024, seed=73)
    q, kv, sl = W.generate(w)
    # last rope column: q = 1, key = a ramp of dequantised values 0 .. 1792
    # (codes 0 .. 448 at kv_scale 4), the other values N(0, 1) as codes of kv / 4
    q[..., 575] = 1.0
    ks = 4.0
    vals = kv.float() / ks
    vals[0, :, 575] = torch.linspace(0, 448, 1024)
    codes = vals.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    out, lse, _ = gpu_decode_fp8(q, codes, ks, sl, w.scale, kernel=kernel)
    ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale)
    assert_parity(out, lse, ro, rl, f"fp8 ramp H{H}", out_max_abs=OUT_MAX_ABS * max(1.0, float(np.abs(ro).max())))


@pytest.mark.parametrize("kernel", FP8_KERNELS)
def test_fp8_deterministic_and_split_invariant(cuda_device, kernel):
    w = W.custom(B=4, Sq=1, H=128, L=2500, L_lo=100, seed=195)
    q, codes, ks, sl = W.generate_fp8(w)
    o1, l1, _ = gpu_decode_fp8(q, codes, ks, sl, w.scale, kernel=kernel)
    o2, l2, _ = gpu_decode_fp8(q, codes, ks, sl, w.scale, kernel=kernel)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)
    o3, l3, _ = gpu_decode_fp8(q, codes, ks, sl, w.scale, num_partitions=1, kernel=kernel)
    assert (o1.double() - o3.double()).abs().max().item() <= 1e-2
    # The operand kernels carry P as two E4M3 terms (about 8 significant bits)
    # rounded against the running reference max, which moves at other points
    # when a sequence is cut: its lse may differ between splits by the rounding
    # of P (measured 1.8e-4), bounded here by the lse parity tolerance.  The
    # widening kernel's operands are exact, so only the fp32 merge differs.
    lse_tol = 1e-4 if kernel == M.MLA_KERNEL_FP8 else 1e-3
    assert (l1 - l3).abs().max().item() <= lse_tol


def test_fp8_plan_and_entry_point_must_agree(cuda_device):
    w = W.custom(B=1, Sq=1, H=16, L=256, seed=197)
    q, codes, ks, sl = W.generate_fp8(w)
    bf_plan = M.mla_decode_plan(1, 1, 16, 256, device=0)
    f8_plan = M.mla_decode_plan_fp8(1, 1, 16, 256, device=0)
    ws = M.alloc_workspace(f8_plan)
    out = torch.empty((1, 1, 16, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, 1, 16), dtype=torch.float32, device=DEV)
    kv_bf16 = torch.zeros((1, 256, 576), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_run_fp8(bf_plan, q.to(DEV), codes.to(DEV), ks, sl.to(DEV), w.scale, out, lse, ws)
    assert e.value.code == 1
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_run(f8_plan, q.to(DEV), kv_bf16, sl.to(DEV), w.scale, out, lse, ws)
    assert e.value.code == 1
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(M.MlaError) as e:
            M.mla_decode_run_fp8(f8_plan, q.to(DEV), codes.to(DEV), bad, sl.to(DEV), w.scale, out, lse, ws)
        assert e.value.code == 1


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("H", [16, 128])
def test_fp8_bounded_wait_timeout_reports_and_recovers(cuda_device, H, kernel):
    """Host-side fault injection as in test_gpu_parity: the producer of CTA 0
    skips one load it armed; the bounded waits (converters and MMA issuer)
    run out, MLA_ERR_TIMEOUT is reported, and the next run is clean."""
    if kernel == M.MLA_KERNEL_FP8_PAIR and H % 128 != 0:
        pytest.skip("the CTA-pair FP8 kernel runs 128-row query groups (Sq*H % 128 == 0)")
    w = W.custom(B=2, Sq=1, H=H, L=1000, seed=201)
    q, codes, ks, sl = W.generate_fp8(w)
    plan = M.mla_decode_plan_fp8(2, 1, H, 1000, device=0, kernel=kernel)
    ws = M.alloc_workspace(plan)
    out = torch.empty((2, 1, H, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((2, 1, H), dtype=torch.float32, device=DEV)
    try:
        M.mla_decode_set_debug(wait_timeout_ns=20_000_000, stall_unit=3)
        M.mla_decode_run_fp8(plan, q.to(DEV), codes.to(DEV), ks, sl.to(DEV), w.scale, out, lse, ws)
        with pytest.raises(M.MlaError) as e:
            M.mla_decode_check(plan, ws)
        assert e.value.code == 5
    finally:
        M.mla_decode_set_debug(0, -1)
    M.mla_decode_run_fp8(plan, q.to(DEV), codes.to(DEV), ks, sl.to(DEV), w.scale, out, lse, ws)
    M.mla_decode_check(plan, ws)
    ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale)
    assert_parity(out.cpu(), lse.cpu(), ro, rl, f"fp8 after timeout H{H}")


# ---- full sizes, in the launch configuration bench.py --fp8 times: sampled
# rows against the oracle, and global properties on every row.
FULL = ["lowhead", "metric"]


@pytest.mark.parametrize("kernel", FP8_KERNELS)
@pytest.mark.parametrize("name", FULL)
def test_fp8_full_size_sampled(cuda_device, name, kernel):
    w = W.WORKLOADS[name]
    q, codes, ks, sl = W.generate_fp8(w)
    out, lse, plan = gpu_decode_fp8(q, codes, ks, sl, w.scale, kernel=kernel)
    R = w.Sq * w.H
    rng = np.random.default_rng(8)
    rows = np.unique(np.concatenate([rng.choice(w.B * R, size=min(64, w.B * R), replace=False),
                                     np.arange(0, w.B * R, max(1, w.B * R // 24))]))
    ro, rl = oracle.mla_decode_fp8(q, codes, ks, sl, w.scale, row_ids=rows)
    assert_parity(out.reshape(-1, 512)[torch.from_numpy(rows)], lse.reshape(-1)[torch.from_numpy(rows)], ro, rl,
                  name + " fp8")
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b in range(0, w.B, max(1, w.B // 6)):
        Lb = int(sl[b])
        v = codes[b, :Lb, :512].view(torch.float8_e4m3fn).float() * ks
        lo, hi = v.min(dim=0).values, v.max(dim=0).values
        ob = out[b].float().reshape(-1, 512)
        tol = 1e-2 + 1e-2 * (hi - lo)
        assert (ob >= lo - tol).all() and (ob <= hi + tol).all()
        assert (lse[b] <= (math.log(Lb) + 1e4)).all()
