"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output): on `out`, max-abs
<= 2e-2 and relative L2 <= 5e-3 over all compared elements; on `lse` (fp32,
natural log) max-abs <= 1e-3.  Rows past each sequence's length are NaN in
every kv tensor here, so any read beyond a length poisons the result.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_11_b200 import binding as M
from mla_decode_attention_11_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def gpu_decode(q, kv, sl, scale, num_partitions=0, kernel=0):
    dev = torch.device("cuda:0")
    qd, kvd, sld = q.to(dev), kv.to(dev), sl.to(torch.int32).to(dev)
    plan = M.mla_decode_plan(q.shape[0], q.shape[1], q.shape[2], kv.shape[1], device=0,
                             num_partitions=num_partitions, kernel=kernel)
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.full((q.shape[0], q.shape[1], q.shape[2], 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=dev)
    M.mla_decode_run(plan, qd, kvd, sld, scale, out, lse, ws)
    M.mla_decode_check(plan, ws)
    return out.cpu(), lse.cpu(), plan


def assert_parity(out_gpu, lse_gpu, out_ref, lse_ref, what="", out_max_abs=OUT_MAX_ABS):
    og = out_gpu.to(torch.float64).numpy().reshape(-1, 512)
    orf = np.asarray(out_ref, dtype=np.float64).reshape(-1, 512)
    lg = lse_gpu.to(torch.float64).numpy().reshape(-1)
    lr = np.asarray(lse_ref, dtype=np.float64).reshape(-1)
    assert np.all(np.isfinite(og)), f"{what}: non-finite output"
    diff = og - orf
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(orf))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    empty = np.isneginf(lr)
    assert np.array_equal(np.isneginf(lg), empty), f"{what}: -inf lse pattern differs"
    lmax = float(np.max(np.abs(lg[~empty] - lr[~empty]))) if (~empty).any() else 0.0
    assert max_abs <= out_max_abs, f"{what}: out max-abs {max_abs:.3e}"
    assert rel <= OUT_REL_L2, f"{what}: out rel-L2 {rel:.3e}"
    assert lmax <= LSE_MAX_ABS, f"{what}: lse max-abs {lmax:.3e}"
    return max_abs, rel, lmax


def check_workload(w, num_partitions=0, lengths=None, out_max_abs=OUT_MAX_ABS, kernel=0):
    q, kv, sl = W.generate(w, lengths=lengths)
    out, lse, plan = gpu_decode(q, kv, sl, w.scale, num_partitions, kernel)
    ro, rl = oracle.mla_decode(q, kv, sl, w.scale)
    return assert_parity(out, lse, ro, rl, w.name, out_max_abs=out_max_abs), plan


# ---- the five workloads at sizes the oracle finishes in seconds (several
# tiles, ragged tails, the same head layout and value distribution)
SMALL = {
    "tiny": W.WORKLOADS["tiny"],
    "dsv3": W.small_variant(W.WORKLOADS["dsv3"], B=3, L=1000),
    "mixed": W.small_variant(W.WORKLOADS["mixed"], B=6, L=2100, L_lo=100),
    "lowhead": W.small_variant(W.WORKLOADS["lowhead"], B=20, L=3001),
    "long": W.small_variant(W.WORKLOADS["long"], B=1, L=5000),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_workloads(cuda_device, name):
    check_workload(SMALL[name])


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 64, 300])
@pytest.mark.parametrize("kernel", [M.MLA_KERNEL_TRANSPOSED, M.MLA_KERNEL_PAIR])
def test_forced_partitions(cuda_device, parts, kernel):
    w = W.custom(B=5, Sq=1, H=128, L=1500, L_lo=1, seed=31)
    check_workload(w, num_partitions=parts, kernel=kernel)


@pytest.mark.parametrize("name", ["dsv3", "mixed", "long"])
def test_both_kernels_on_128_head_workloads(cuda_device, name):
    """The pair kernel (auto for 128-row groups) and the transposed kernel
    (forced) each match the oracle on the same inputs."""
    check_workload(SMALL[name], kernel=M.MLA_KERNEL_TRANSPOSED)
    check_workload(SMALL[name], kernel=M.MLA_KERNEL_PAIR)


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 1023])
def test_lengths_around_tile_edges(cuda_device, L):
    check_workload(W.custom(B=2, Sq=1, H=16, L=L, seed=40 + L))
    check_workload(W.custom(B=1, Sq=1, H=128, L=L, seed=41 + L))
    check_workload(W.custom(B=1, Sq=1, H=128, L=L, seed=41 + L), kernel=M.MLA_KERNEL_TRANSPOSED)


@pytest.mark.parametrize("H", [16, 128])
def test_empty_and_mixed_lengths(cuda_device, H):
    w = W.custom(B=6, Sq=1, H=H, L=700, seed=52)
    lengths = torch.tensor([0, 1, 700, 0, 129, 5], dtype=torch.int32)
    check_workload(w, lengths=lengths)
    check_workload(w, lengths=lengths, num_partitions=3)
    check_workload(w, lengths=torch.zeros(6, dtype=torch.int32))


@pytest.mark.parametrize("B,L,H", [(600, 512, 128), (2000, 256, 16)])
def test_many_short_sequences(cuda_device, B, L, H):
    """Far more sequences than partitions, about a tenth of them empty and the
    rest 1..L keys: every partition walks several whole sequences plus cut
    pieces at its ends, the length scans take many passes over the batch, and
    the combine merges the cut ones and writes the empty ones."""
    w = W.custom(B=B, Sq=1, H=H, L=L, seed=700 + H)
    g = torch.Generator().manual_seed(701 + H)
    lengths = torch.randint(1, L + 1, (B,), generator=g, dtype=torch.int32)
    lengths[torch.rand(B, generator=g) < 0.1] = 0
    check_workload(w, lengths=lengths)
    check_workload(w, lengths=lengths, num_partitions=5)


@pytest.mark.parametrize("H,Sq", [(16, 1), (16, 2), (16, 3), (32, 1), (64, 1), (128, 1), (128, 2), (64, 3),
                                  (64, 2), (32, 4), (128, 3)])
def test_head_and_token_counts(cuda_device, H, Sq):
    check_workload(W.custom(B=2, Sq=Sq, H=H, L=600, seed=60 + H + Sq))


def test_large_scores(cuda_device):
    """sigma = 3 makes scaled scores span tens of units: the online max must
    grow and rescale (the lazy-rescale path) without losing accuracy.  Values
    are N(0, 9) here, so outputs reach |out| ~ 12 where one bf16 rounding of
    the output alone is up to 2^-8 * 12 = 0.047: the max-abs bound is scaled
    by max(1, max|ref| / 1) (the relative-L2 bound is unchanged)."""
    for w in (W.custom(B=2, Sq=1, H=16, L=2000, sigma=3.0, seed=70),
              W.custom(B=1, Sq=1, H=128, L=2000, sigma=3.0, seed=71)):
        q, kv, sl = W.generate(w)
        out, lse, _ = gpu_decode(q, kv, sl, w.scale)
        ro, rl = oracle.mla_decode(q, kv, sl, w.scale)
        assert_parity(out, lse, ro, rl, w.name, out_max_abs=OUT_MAX_ABS * max(1.0, float(np.abs(ro).max())))


def test_rising_scores_force_rescale(cuda_device):
    """Keys whose scores rise along the sequence force a rescale on many tiles."""
    w = W.custom(B=1, Sq=1, H=16, L=1024, seed=72)
    q, kv, sl = W.generate(w)
    # last rope column: q = 1, key = a ramp to 1664, so the scaled score rises
    # by ~12 (log2 units) per 128-row tile and every tile must rescale
    q[..., 575] = 1.0
    kv[0, :, 575] = torch.linspace(0, 1664, 1024).to(torch.bfloat16)
    out, lse, _ = gpu_decode(q, kv, sl, w.scale)
    ro, rl = oracle.mla_decode(q, kv, sl, w.scale)
    assert_parity(out, lse, ro, rl, "ramp")


@pytest.mark.parametrize("B,L,H", [(40, 300, 128), (30, 300, 128), (100, 700, 64), (150, 260, 16)])
def test_uniform_batches_either_schedule(cuda_device, B, L, H):
    """Equal lengths with enough sequences to fill at least half the
    partitions switch the device schedule to one piece per sequence (no cuts);
    fewer sequences keep the balanced split.  Both must match the oracle."""
    w = W.custom(B=B, Sq=1, H=H, L=L, seed=600 + B)
    check_workload(w)


def test_split_matches_unsplit(cuda_device):
    w = W.custom(B=3, Sq=1, H=128, L=3000, seed=80)
    q, kv, sl = W.generate(w)
    o1, l1, _ = gpu_decode(q, kv, sl, w.scale, num_partitions=1)
    o2, l2, _ = gpu_decode(q, kv, sl, w.scale, num_partitions=37)
    d = (o1.double() - o2.double()).abs().max().item()
    assert d <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_two_tokens_equal_two_single_token_calls(cuda_device):
    w = W.custom(B=2, Sq=2, H=16, L=900, seed=90)
    q, kv, sl = W.generate(w)
    o, l, _ = gpu_decode(q, kv, sl, w.scale)
    for t in range(2):
        ot, lt, _ = gpu_decode(q[:, t:t + 1].contiguous(), kv, sl, w.scale)
        assert (ot.double() - o[:, t:t + 1].double()).abs().max().item() <= 1e-2
        assert (lt - l[:, t:t + 1]).abs().max().item() <= 1e-4


def test_deterministic(cuda_device):
    w = W.custom(B=4, Sq=1, H=128, L=2500, L_lo=100, seed=95)
    q, kv, sl = W.generate(w)
    o1, l1, _ = gpu_decode(q, kv, sl, w.scale)
    o2, l2, _ = gpu_decode(q, kv, sl, w.scale)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_seqlen_out_of_range_is_flagged(cuda_device):
    w = W.custom(B=2, Sq=1, H=16, L=300, seed=99)
    q, kv, sl = W.generate(w, tail_fill=0.0)
    bad = torch.tensor([300, 305], dtype=torch.int32)  # second one > L_max
    dev = torch.device("cuda:0")
    plan = M.mla_decode_plan(2, 1, 16, 300, device=0)
    ws = M.alloc_workspace(plan)
    out = torch.empty((2, 1, 16, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((2, 1, 16), dtype=torch.float32, device=dev)
    M.mla_decode_run(plan, q.to(dev), kv.to(dev), bad.to(dev), w.scale, out, lse, ws)
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_check(plan, ws)
    assert e.value.code == 7
    ro, rl = oracle.mla_decode(q, kv, torch.tensor([300, 300], dtype=torch.int32), w.scale)
    assert_parity(out.cpu(), lse.cpu(), ro, rl, "clamped")
    M.mla_decode_check(plan, ws)  # cleared after the read


@pytest.mark.parametrize("H,unit,parts", [(16, 3, 0), (128, 3, 0), (16, 30, 1), (128, 40, 1)])
def test_bounded_wait_timeout_reports_and_recovers(cuda_device, H, unit, parts):
    """A host-side fault injection: the producer of CTA 0 arms a barrier but
    skips a load (an early one, or one deep in the stream with several loads
    of both CTAs still in flight), so the consumer's bounded wait runs out and
    every role unwinds, draining what it armed.  The run must report
    MLA_ERR_TIMEOUT, and the context must stay usable."""
    w = W.custom(B=2, Sq=1, H=H, L=1000, seed=101)
    q, kv, sl = W.generate(w)
    try:
        M.mla_decode_set_debug(wait_timeout_ns=20_000_000, stall_unit=unit)
        dev = torch.device("cuda:0")
        # one partition: CTA 0 streams all 16 tiles, so a late unit lies mid-stream
        plan = M.mla_decode_plan(2, 1, H, 1000, device=0, num_partitions=parts)
        ws = M.alloc_workspace(plan)
        out = torch.empty((2, 1, H, 512), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((2, 1, H), dtype=torch.float32, device=dev)
        M.mla_decode_run(plan, q.to(dev), kv.to(dev), sl.to(dev), w.scale, out, lse, ws)
        with pytest.raises(M.MlaError) as e:
            M.mla_decode_check(plan, ws)
        assert e.value.code == 5
    finally:
        M.mla_decode_set_debug(0, -1)
    # the next run on the same workspace is clean: the check cleared the
    # status words the abandoned run left behind
    M.mla_decode_run(plan, q.to(dev), kv.to(dev), sl.to(dev), w.scale, out, lse, ws)
    M.mla_decode_check(plan, ws)
    ro, rl = oracle.mla_decode(q, kv, sl, w.scale)
    assert_parity(out.cpu(), lse.cpu(), ro, rl, f"after timeout H{H} unit {unit}")
    check_workload(w)


# ---- full sizes, in the launch configuration bench.py times: sampled rows
# against the oracle row by row, and global properties on every row.
FULL = ["tiny", "dsv3", "mixed", "lowhead", "long", "metric"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(cuda_device, name):
    w = W.WORKLOADS[name]
    q, kv, sl = W.generate(w)
    out, lse, plan = gpu_decode(q, kv, sl, w.scale)
    R = w.Sq * w.H
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.choice(w.B * R, size=min(96, w.B * R), replace=False),
                                     np.arange(0, w.B * R, max(1, w.B * R // 32))]))
    ro, rl = oracle.mla_decode_rows(q, kv, sl, w.scale, rows)
    assert_parity(out.reshape(-1, 512)[torch.from_numpy(rows)], lse.reshape(-1)[torch.from_numpy(rows)], ro, rl,
                  name)
    # every row: finite, and each output row is a convex combination of value
    # rows, so it lies inside the per-column range of that sequence's values
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b in range(0, w.B, max(1, w.B // 8)):
        Lb = int(sl[b])
        v = kv[b, :Lb, :512].float()
        lo, hi = v.min(dim=0).values, v.max(dim=0).values
        ob = out[b].float().reshape(-1, 512)
        tol = 1e-2 + 1e-2 * (hi - lo)
        assert (ob >= lo - tol).all() and (ob <= hi + tol).all()
        assert (lse[b] <= (math.log(Lb) + 1e4)).all()
