"""mla_decode_run_noalloc: the decode entry point for callers that must not
allocate device memory while decoding (a serving engine that gave almost all
HBM to its KV cache at start-up, a C host without a device allocator).  It
keeps its split-KV partials in the library's static scratch array instead of
a caller workspace.

Each case runs the call twice in a row, on different inputs, and compares
both results with the fp64 oracle and with mla_decode_run (caller workspace)
on the same inputs, within the parity tolerances of the GPU suite.  A call
that the library rejects must enqueue nothing (checked by capturing it into a
CUDA graph), so it cannot disturb an earlier call still running on the
shared scratch.  The file is collected last so it also
runs after every other GPU test has used the library in the same process; it
passes alone in a fresh process too.
"""
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

DEV = torch.device("cuda:0")


def _inputs(w):
    q, kv, sl = W.generate(w)
    return q.to(DEV), kv.to(DEV), sl.to(torch.int32).to(DEV)


def _oracle(w):
    q, kv, sl = W.generate(w)
    ro, rl = oracle.mla_decode(q, kv, sl, w.scale)
    return torch.from_numpy(ro), torch.from_numpy(rl)


def _outputs(plan):
    out = torch.full((plan.B, plan.Sq, plan.H, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((plan.B, plan.Sq, plan.H), float("nan"), dtype=torch.float32, device=DEV)
    return out, lse


def _with_workspace(plan, q, kv, sl, scale):
    ws = M.alloc_workspace(plan)
    M.mla_decode_workspace_init(plan, ws)
    out, lse = _outputs(plan)
    M.mla_decode_run(plan, q, kv, sl, scale, out, lse, ws)
    M.mla_decode_check(plan, ws)
    return out.cpu(), lse.cpu()


def _close(out, lse, out_ref, lse_ref, what):
    o = out.to(torch.float64).numpy().reshape(-1, 512)
    r = out_ref.to(torch.float64).numpy().reshape(-1, 512)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    d = o - r
    assert float(np.max(np.abs(d))) <= OUT_MAX_ABS, f"{what}: out max-abs {np.max(np.abs(d)):.3e}"
    denom = float(np.linalg.norm(r))
    assert float(np.linalg.norm(d)) <= OUT_REL_L2 * max(denom, 1e-30), f"{what}: out rel-L2"
    lg, lr = lse.to(torch.float64).numpy().reshape(-1), lse_ref.to(torch.float64).numpy().reshape(-1)
    empty = np.isneginf(lr)
    assert np.array_equal(np.isneginf(lg), empty), f"{what}: -inf lse pattern differs"
    if (~empty).any():
        assert float(np.max(np.abs(lg[~empty] - lr[~empty]))) <= LSE_MAX_ABS, f"{what}: lse"


# (workload, kernel): the CTA-pair kernel for 128 query rows per group and
# the single-CTA kernel for 16 heads, each with ragged lengths and split KV
CASES = {
    "pair_H128": (W.small_variant(W.WORKLOADS["mixed"], B=5, L=1500, L_lo=1), M.MLA_KERNEL_PAIR),
    "transposed_H16": (W.small_variant(W.WORKLOADS["lowhead"], B=7, L=1300), M.MLA_KERNEL_TRANSPOSED),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_two_calls_match_workspace_run(cuda_device, name):
    w, kernel = CASES[name]
    w2 = W.small_variant(w, seed_offset=17)
    plan = M.mla_decode_plan(w.B, w.Sq, w.H, w.L, device=0, kernel=kernel)
    assert plan.kernel == kernel
    assert plan.workspace_bytes <= M.MLA_NOALLOC_SCRATCH_BYTES
    a, b = _inputs(w), _inputs(w2)
    ref_a = _with_workspace(plan, *a, w.scale)
    ref_b = _with_workspace(plan, *b, w.scale)

    out1, lse1 = _outputs(plan)
    M.mla_decode_run_noalloc(plan, *a, w.scale, out1, lse1)  # enqueue only
    out2, lse2 = _outputs(plan)
    M.mla_decode_run_noalloc(plan, *b, w.scale, out2, lse2, wait_and_check=True)
    _close(out1.cpu(), lse1.cpu(), *ref_a, f"{name} call 1")
    _close(out2.cpu(), lse2.cpu(), *ref_b, f"{name} call 2")
    _close(out1.cpu(), lse1.cpu(), *_oracle(w), f"{name} call 1 vs oracle")
    _close(out2.cpu(), lse2.cpu(), *_oracle(w2), f"{name} call 2 vs oracle")

    # once set up on this device, a call leaves free device memory unchanged
    out3, lse3 = _outputs(plan)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info(DEV)
    M.mla_decode_run_noalloc(plan, *a, w.scale, out3, lse3, wait_and_check=True)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info(DEV)
    assert free_after == free_before
    _close(out3.cpu(), lse3.cpu(), *ref_a, f"{name} call 3")


def test_noalloc_status_cleared_between_calls(cuda_device):
    w, _ = CASES["pair_H128"]
    plan = M.mla_decode_plan(w.B, w.Sq, w.H, w.L, device=0)
    q, kv, sl = _inputs(w)
    bad = sl.clone()
    bad[1] = w.L + 5  # out of range: clamped and flagged
    out, lse = _outputs(plan)
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_run_noalloc(plan, q, kv, bad, w.scale, out, lse, wait_and_check=True)
    assert e.value.code == 7
    # the next call starts from cleared status words
    out, lse = _outputs(plan)
    M.mla_decode_run_noalloc(plan, q, kv, sl, w.scale, out, lse, wait_and_check=True)
    _close(out.cpu(), lse.cpu(), *_with_workspace(plan, q, kv, sl, w.scale), "after flagged call")


def test_noalloc_rejects_plan_beyond_scratch(cuda_device):
    w, _ = CASES["pair_H128"]
    plan = M.mla_decode_plan(w.B, w.Sq, w.H, w.L, device=0, num_partitions=4096)
    assert plan.workspace_bytes > M.MLA_NOALLOC_SCRATCH_BYTES
    q, kv, sl = _inputs(w)
    out, lse = _outputs(plan)
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_run_noalloc(plan, q, kv, sl, w.scale, out, lse, wait_and_check=True)
    assert e.value.code == 6
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all() and torch.isnan(lse).all()  # nothing was enqueued


def test_noalloc_rejected_call_enqueues_nothing(cuda_device):
    """A rejected call (here: an output pointer that is not 16-byte aligned,
    and an FP8 plan on the bf16 entry point) returns its error before it
    enqueues anything, in particular not the clearing of the shared status
    words: captured into a CUDA graph between two torch kernels, it adds no
    node."""
    from cuda.bindings import runtime as rt
    w, _ = CASES["pair_H128"]
    plan = M.mla_decode_plan(w.B, w.Sq, w.H, w.L, device=0)
    q, kv, sl = _inputs(w)
    out, lse = _outputs(plan)
    M.mla_decode_run_noalloc(plan, q, kv, sl, w.scale, out, lse, wait_and_check=True)  # device set-up
    lib = M.load_library()
    f8 = M.mla_decode_plan_fp8(w.B, w.Sq, 16, w.L, device=0)
    x = torch.zeros(16, device=DEV)
    side = torch.cuda.Stream(DEV)
    g = torch.cuda.CUDAGraph(keep_graph=True)
    codes = []
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            x.add_(1.0)
            h = side.cuda_stream
            codes.append(lib.mla_decode_run_noalloc(M.ctypes.byref(plan), q.data_ptr(), kv.data_ptr(),
                                                    sl.data_ptr(), M.ctypes.c_float(w.scale), out.data_ptr() + 8,
                                                    lse.data_ptr(), 0, h))
            codes.append(lib.mla_decode_run_noalloc(M.ctypes.byref(f8), q.data_ptr(), kv.data_ptr(),
                                                    sl.data_ptr(), M.ctypes.c_float(w.scale), out.data_ptr(),
                                                    lse.data_ptr(), 0, h))
            x.add_(1.0)
    assert codes == [2, 1]
    err, _, n = rt.cudaGraphGetNodes(g.raw_cuda_graph(), 0)
    assert err == rt.cudaError_t.cudaSuccess
    assert n == 2, f"the rejected calls added {n - 2} node(s) to the capture"
    g.replay()
    torch.cuda.synchronize()
    assert float(x[0]) == 2.0
