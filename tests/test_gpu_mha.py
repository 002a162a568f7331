"""GPU parity of MHA decode (mha_decode_plan / mha_decode_run: 128-wide
heads, grouped kv heads, separate K and V) against the fp64 MHA oracle on
the same seeded inputs: several head groupings (query rows per kv head from
1 to 32, padded to 16 or 32 columns), ragged and empty sequences, forced
split counts, attention sinks, and the full-size grouped-query batch.
Tolerances as in test_gpu_parity; rows past each length are NaN."""
import numpy as np
import pytest
import torch

import oracle
from mla_decode_attention_11_b200 import binding as M
from mla_decode_attention_11_b200 import workloads as W
from tests.test_gpu_parity import assert_parity

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def run_mha(q, k, v, sl, scale, parts=0, sinks=None):
    B, Sq, H, _ = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    plan = M.mha_decode_plan(B, Sq, H, Hkv, L, device=0, num_partitions=parts)
    assert plan.kernel == M.MLA_KERNEL_MHA
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out = torch.full((B, Sq, H, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Sq, H), float("nan"), dtype=torch.float32, device=DEV)
    sk = None if sinks is None else torch.from_numpy(sinks).to(DEV)
    M.mha_decode_run(plan, q.to(DEV), k.to(DEV), v.to(DEV), sl.to(torch.int32).to(DEV), scale, out, lse, ws, sinks=sk)
    M.mla_decode_check(plan, ws)
    return out.cpu(), lse.cpu(), plan


SHAPES = [  # (B, Sq, H, Hkv, L)
    (4, 1, 32, 8, 1500),    # 4 query rows per kv head (padded to 16)
    (3, 2, 16, 2, 900),     # 16 rows per kv head
    (2, 1, 32, 1, 700),     # one kv head: 32 rows
    (5, 1, 8, 8, 1100),     # one row per kv head
    (3, 4, 24, 3, 640),     # 32 rows per kv head over 4 tokens
]


@pytest.mark.parametrize("parts", [0, 1, 7])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_Sq{}_H{}_Hkv{}_L{}".format(*s))
def test_mha_matches_oracle(cuda_device, shape, parts):
    B, Sq, H, Hkv, L = shape
    w = W.MhaWorkload("mha_case", B=B, Sq=Sq, H=H, Hkv=Hkv, L=L, L_lo=1, seed=3000 + H + L)
    lengths = torch.tensor([L] + [max(1, L // (i + 3)) for i in range(B - 2)] + [0], dtype=torch.int32)
    q, k, v, sl = W.generate_mha(w, lengths=lengths)
    out, lse, plan = run_mha(q, k, v, sl, w.scale, parts)
    ro, rl = oracle.mha_decode(q, k, v, sl, w.scale)
    assert_parity(out, lse, ro, rl, f"mha {shape} P={plan.num_partitions}")


def test_mha_many_short_sequences(cuda_device):
    """Far more sequences than partitions (each partition walks several whole
    sequences plus cut pieces), about a tenth of them empty."""
    B, L = 500, 384
    w = W.MhaWorkload("mha_many", B=B, Sq=1, H=32, Hkv=8, L=L, L_lo=1, seed=3100)
    g = torch.Generator().manual_seed(3101)
    lengths = torch.randint(1, L + 1, (B,), generator=g, dtype=torch.int32)
    lengths[torch.rand(B, generator=g) < 0.1] = 0
    q, k, v, sl = W.generate_mha(w, lengths=lengths)
    out, lse, plan = run_mha(q, k, v, sl, w.scale)
    ro, rl = oracle.mha_decode(q, k, v, sl, w.scale)
    assert_parity(out, lse, ro, rl, f"mha many short P={plan.num_partitions}")


def test_mha_sinks(cuda_device):
    w = W.MHA_WORKLOADS["mha_small"]
    q, k, v, sl = W.generate_mha(w)
    sinks = np.linspace(-3.0, 3.0, w.H).astype(np.float32)
    out, lse, _ = run_mha(q, k, v, sl, w.scale, 5, sinks)
    ro, rl = oracle.mha_decode(q, k, v, sl, w.scale, sinks=sinks.astype(np.float64))
    assert_parity(out, lse, ro, rl, "mha sinks")


def test_mha_full_size(cuda_device):
    w = W.MHA_WORKLOADS["mha_gqa"]
    q, k, v, sl = W.generate_mha(w)
    out, lse, _ = run_mha(q, k, v, sl, w.scale)
    ro, rl = oracle.mha_decode(q, k, v, sl, w.scale)
    assert_parity(out, lse, ro, rl, "mha_gqa full size")
