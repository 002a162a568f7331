"""Batch-invariant plans (mla_decode_plan_batch_invariant): parity with the
fp64 oracle, and bitwise independence of a sequence's result from the rest of
the batch (which other sequences, how many, and at which position), for both
kernels, with and without attention sinks.  Tolerances as in
test_gpu_parity."""
import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_11_b200 import binding as M
from mla_decode_attention_11_b200 import workloads as W
from tests.test_gpu_parity import assert_parity

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def run_inv(q, kv, sl, scale, split_tiles, sinks=None):
    B, Sq, H, _ = q.shape
    plan = M.mla_decode_plan_batch_invariant(B, Sq, H, kv.shape[1], device=0, split_tiles=split_tiles)
    assert plan.split_tiles == (split_tiles or plan.split_tiles) and plan.split_tiles > 0
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.full((B, Sq, H, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Sq, H), float("nan"), dtype=torch.float32, device=DEV)
    sk = None if sinks is None else torch.from_numpy(sinks).to(DEV)
    M.mla_decode_run_sinks(plan, q.to(DEV), kv.to(DEV), sl.to(torch.int32).to(DEV), scale, sk, out, lse, ws)
    M.mla_decode_check(plan, ws)
    return out.cpu(), lse.cpu(), plan


@pytest.mark.parametrize("split_tiles", [1, 3, 0])
@pytest.mark.parametrize("H,Sq", [(128, 1), (16, 1), (64, 2)])
def test_invariant_plan_matches_oracle(cuda_device, H, Sq, split_tiles):
    w = W.custom(B=5, Sq=Sq, H=H, L=2500, L_lo=1, seed=400 + H + split_tiles)
    lengths = torch.tensor([2500, 1, 128, 0, 2049], dtype=torch.int32)
    q, kv, sl = W.generate(w, lengths=lengths)
    sinks = None if split_tiles == 3 else np.linspace(-2.0, 2.0, H).astype(np.float32)
    out, lse, plan = run_inv(q, kv, sl, w.scale, split_tiles, sinks)
    ro, rl = oracle.mla_decode(q, kv, sl, w.scale, sinks=None if sinks is None else sinks.astype(np.float64))
    assert_parity(out, lse, ro, rl, f"invariant H{H} Sq{Sq} S{plan.split_tiles}")


@pytest.mark.parametrize("H", [128, 16])
def test_result_independent_of_batch(cuda_device, H):
    """Sequence X (3000 keys) alone, and inside two different batches at
    different positions: its out and lse rows are bitwise identical."""
    split_tiles = 4
    L = 4096
    big = W.custom(B=9, Sq=1, H=H, L=L, L_lo=1, seed=500 + H)
    q, kv, _ = W.generate(big, lengths=torch.full((9,), L, dtype=torch.int32), tail_fill=0.0)
    x = 4                      # sequence X is row 4 of the big tensors
    Lx = 3000
    sinks = np.linspace(-1.0, 1.0, H).astype(np.float32)

    def run_batch(idx, lens):
        sl = torch.tensor(lens, dtype=torch.int32)
        return run_inv(q[idx].contiguous(), kv[idx].contiguous(), sl, big.scale, split_tiles, sinks)

    alone_o, alone_l, _ = run_batch([x], [Lx])
    a_o, a_l, _ = run_batch([0, 1, x, 2, 3, 5, 6, 7, 8], [4096, 77, Lx, 0, 1500, 4096, 128, 2600, 999])
    b_o, b_l, _ = run_batch([x, 8, 8, 6], [Lx, 4096, 30, 4096])
    for o, l, pos in ((a_o, a_l, 2), (b_o, b_l, 0)):
        assert torch.equal(o[pos], alone_o[0]), "out differs with the batch"
        assert torch.equal(l[pos], alone_l[0]), "lse differs with the batch"
    ro, rl = oracle.mla_decode(q[[x]], kv[[x]], torch.tensor([Lx], dtype=torch.int32), big.scale,
                               sinks=sinks.astype(np.float64))
    assert_parity(alone_o, alone_l, ro, rl, f"X alone H{H}")
