"""GPU parity of the attention-sink entry point (mla_decode_run_sinks)
against the fp64 oracle's sink definition: one extra softmax term per head,
without a value.  Both kernels, unsplit and split sequences (the sink is folded
in by the main kernel for whole sequences and by the combine kernel for cut
ones), empty sequences (lse = the sink), a head whose sink is switched off
(-inf) and one that dominates the row.  Tolerances as in test_gpu_parity."""
import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_11_b200 import binding as M
from mla_decode_attention_11_b200 import workloads as W
from tests.test_gpu_parity import assert_parity

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _sinks(H, seed):
    g = np.random.default_rng(seed)
    s = g.normal(0.0, 2.0, size=H)
    s[0] = -np.inf      # this head has no sink
    s[1] = 30.0         # far above every score: the sink takes almost all the weight
    s[2] = -50.0        # far below: no visible effect
    return s.astype(np.float32)


def run_sinks(q, kv, sl, scale, sinks, num_partitions=0, kernel=0):
    plan = M.mla_decode_plan(q.shape[0], q.shape[1], q.shape[2], kv.shape[1], device=0,
                             num_partitions=num_partitions, kernel=kernel)
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.full((q.shape[0], q.shape[1], q.shape[2], 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=DEV)
    sk = None if sinks is None else torch.from_numpy(sinks).to(DEV)
    M.mla_decode_run_sinks(plan, q.to(DEV), kv.to(DEV), sl.to(torch.int32).to(DEV), scale, sk, out, lse, ws)
    M.mla_decode_check(plan, ws)
    return out.cpu(), lse.cpu(), plan


CASES = [  # (B, Sq, H, L, L_lo, kernel)
    (4, 1, 128, 1500, 1, M.MLA_KERNEL_PAIR),
    (3, 2, 128, 900, 100, M.MLA_KERNEL_PAIR),
    (5, 1, 16, 1300, 1, M.MLA_KERNEL_TRANSPOSED),
    (4, 1, 64, 700, 1, M.MLA_KERNEL_TRANSPOSED),
    (3, 1, 128, 600, 1, M.MLA_KERNEL_TRANSPOSED),
]


@pytest.mark.parametrize("parts", [0, 1, 7])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Sq{c[1]}_H{c[2]}_L{c[3]}_k{c[5]}")
def test_sinks_match_oracle(cuda_device, case, parts):
    B, Sq, H, L, L_lo, kernel = case
    w = W.custom(B=B, Sq=Sq, H=H, L=L, L_lo=L_lo, seed=200 + H + L)
    lengths = torch.tensor([L] + [max(0, L // (i + 2)) for i in range(B - 2)] + [0], dtype=torch.int32)
    q, kv, sl = W.generate(w, lengths=lengths)
    sinks = _sinks(H, seed=H + L)
    out, lse, plan = run_sinks(q, kv, sl, w.scale, sinks, parts, kernel)
    assert plan.kernel == kernel
    ro, rl = oracle.mla_decode(q, kv, sl, w.scale, sinks=sinks.astype(np.float64))
    assert_parity(out, lse, ro, rl, f"sinks {case} P={plan.num_partitions}")
    # the empty sequence: out = 0, lse = the sink (-inf where a head has none)
    assert torch.count_nonzero(out[-1].float()) == 0
    np.testing.assert_allclose(lse[-1].numpy(), np.broadcast_to(sinks, lse[-1].shape), rtol=0, atol=1e-6)


def test_no_sinks_equals_plain_run(cuda_device):
    w = W.custom(B=3, Sq=1, H=128, L=1000, L_lo=1, seed=301)
    q, kv, sl = W.generate(w)
    out_s, lse_s, plan = run_sinks(q, kv, sl, w.scale, None, 5)
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.empty((w.B, 1, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((w.B, 1, 128), dtype=torch.float32, device=DEV)
    M.mla_decode_run(plan, q.to(DEV), kv.to(DEV), sl.to(DEV), w.scale, out, lse, ws)
    M.mla_decode_check(plan, ws)
    assert torch.equal(out.cpu(), out_s) and torch.equal(lse.cpu(), lse_s)


@pytest.mark.parametrize("name", ["metric", "lowhead"])
def test_sinks_full_size_sampled(cuda_device, name):
    """Full size in the launch configuration bench.py times, sampled rows."""
    w = W.WORKLOADS[name]
    q, kv, sl = W.generate(w)
    sinks = _sinks(w.H, seed=7)
    out, lse, plan = run_sinks(q, kv, sl, w.scale, sinks)
    R = w.Sq * w.H
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([rng.choice(w.B * R, size=64, replace=False),
                                     np.arange(0, w.B * R, max(1, w.B * R // 16))]))
    ro, rl = oracle.mla_decode_rows(q, kv, sl, w.scale, rows, sinks=sinks.astype(np.float64))
    assert_parity(out.reshape(-1, 512)[torch.from_numpy(rows)], lse.reshape(-1)[torch.from_numpy(rows)], ro, rl,
                  f"{name} sinks")
