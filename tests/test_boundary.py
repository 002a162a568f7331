"""C-ABI boundary on the CPU: the library builds, loads without a GPU driver,
exports every symbol include/mla_decode.h declares, and validates arguments
(without launching anything)."""
import ctypes
import os
import re

import pytest
import torch

from mla_decode_attention_11_b200 import build as B
from mla_decode_attention_11_b200 import binding as M
from mla_decode_attention_11_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                            text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "mla_decode_plan" in names and "mla_decode_run" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(M.EXPORTED_SYMBOLS) <= set(names)


def test_library_links_no_driver(lib):
    """The .so must not need libcuda.so at load time: it reaches the driver
    through the statically linked runtime, so it loads on a GPU-less host."""
    import subprocess
    needed = subprocess.run(["readelf", "-d", B.LIB_PATH], capture_output=True, text=True, check=True).stdout
    assert "libcuda.so" not in needed
    assert "libcudart.so" not in needed
    assert lib.mla_decode_abi_version() == 10000


def test_status_strings(lib):
    for code in range(0, 8):
        s = M.status_string(code)
        assert isinstance(s, str) and s
    assert M.status_string(0) == "ok"


@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_plan_for_each_workload(lib, name):
    w = W.WORKLOADS[name]
    p = M.mla_decode_plan(w.B, w.Sq, w.H, w.L, device=-1)
    R = w.Sq * w.H
    assert p.group_rows * p.num_groups == R
    assert p.num_partitions >= 1
    assert p.num_partitions * p.num_groups <= 148
    assert p.smem_bytes <= 232448
    assert p.workspace_bytes >= 256 + 2 * p.num_partitions * R * (512 + 1) * 4


def test_plan_override_and_clamp(lib):
    p = M.mla_decode_plan(4, 1, 16, 100, device=-1, num_partitions=1)
    assert p.num_partitions == 1
    p = M.mla_decode_plan(4, 1, 16, 100, device=-1, num_partitions=100000)
    assert p.num_partitions == 4096


@pytest.mark.parametrize("args,code", [
    ((0, 1, 16, 128), 1), ((70000, 1, 16, 128), 1), ((1, 0, 16, 128), 1), ((1, 17, 16, 128), 1),
    ((1, 1, 16, 0), 1), ((1, 1, 16, (1 << 24) + 1), 1), ((1, 1, 48, 128), 3), ((1, 1, 8, 128), 3),
])
def test_plan_rejects(lib, args, code):
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_plan(*args, device=-1)
    assert e.value.code == code


def test_run_rejects_without_launching(lib):
    """Null pointers, misalignment and a short workspace are refused on the
    host (no device is touched before these checks)."""
    p = M.mla_decode_plan(2, 1, 16, 256, device=-1)
    run = lib.mla_decode_run
    null = None
    rc = run(ctypes.byref(p), null, 16, 16, ctypes.c_float(0.04), 16, 16, 256, p.workspace_bytes, null)
    assert rc == 1
    rc = run(ctypes.byref(p), 16 + 8, 16, 16, ctypes.c_float(0.04), 16, 16, 256, p.workspace_bytes, null)
    assert rc == 2
    rc = run(ctypes.byref(p), 16, 16, 16, ctypes.c_float(0.04), 16, 16, 256, p.workspace_bytes - 1, null)
    assert rc == 6
    rc = run(ctypes.byref(p), 16, 16, 16, ctypes.c_float(0.04), 16, 16, 0, p.workspace_bytes, null)
    assert rc == 6
    rc = run(ctypes.byref(p), 16, 16, 16, ctypes.c_float(float("nan")), 16, 16, 256, p.workspace_bytes, null)
    assert rc == 1
    rc = run(None, 16, 16, 16, ctypes.c_float(0.04), 16, 16, 256, p.workspace_bytes, null)
    assert rc == 1


def test_check_rejects_null(lib):
    assert lib.mla_decode_check(None, None, None) == 1


def test_batch_invariant_plan_without_gpu():
    p = M.mla_decode_plan_batch_invariant(64, 1, 128, 8192, device=-1)
    assert p.split_tiles == 16 and p.kernel == M.MLA_KERNEL_PAIR
    # one fp32 partial (512 values + lse) per 16-tile chunk of every sequence at L_max
    slots = 64 * (8192 // 128 // 16)
    assert p.workspace_bytes >= slots * 128 * 513 * 4
    q = M.mla_decode_plan_batch_invariant(64, 1, 16, 8192, device=-1, split_tiles=5)
    assert q.split_tiles == 5 and q.kernel == M.MLA_KERNEL_TRANSPOSED
    b = M.mla_decode_plan(64, 1, 128, 8192, device=-1)
    assert b.split_tiles == 0
    with pytest.raises(M.MlaError):
        M.mla_decode_plan_batch_invariant(64, 1, 128, 8192, device=-1, split_tiles=-1)


def test_fp8_plan_without_gpu():
    p = M.mla_decode_plan_fp8(132, 1, 16, 16384, device=-1, kernel=M.MLA_KERNEL_FP8)
    assert p.kernel == M.MLA_KERNEL_FP8 and p.group_rows == 16 and p.cta_threads == 320
    assert p.num_partitions == 148 and p.smem_bytes <= 232448
    p = M.mla_decode_plan_fp8(64, 1, 128, 8192, device=-1, kernel=M.MLA_KERNEL_FP8)
    assert p.kernel == M.MLA_KERNEL_FP8 and p.group_rows == 32 and p.num_groups == 4 and p.cta_threads == 256
    assert p.workspace_bytes == M.mla_decode_plan(64, 1, 128, 8192, device=-1,
                                                  kernel=M.MLA_KERNEL_TRANSPOSED).workspace_bytes
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_plan_fp8(64, 1, 24, 8192, device=-1)
    assert e.value.code == 3


def test_fp8_run_rejects_without_launching(lib):
    """A plan of the other kind, a kv_scale that is not finite and positive,
    null pointers and misalignment are refused on the host."""
    f8 = M.mla_decode_plan_fp8(2, 1, 16, 256, device=-1)
    bf = M.mla_decode_plan(2, 1, 16, 256, device=-1)
    run8 = lib.mla_decode_run_fp8
    ok_scale, sc = ctypes.c_float(0.01), ctypes.c_float(0.04)
    rc = run8(ctypes.byref(bf), 16, 16, ok_scale, 16, sc, None, 16, 16, 256, bf.workspace_bytes, None)
    assert rc == 1
    for bad in (0.0, -0.5, float("nan"), float("inf")):
        rc = run8(ctypes.byref(f8), 16, 16, ctypes.c_float(bad), 16, sc, None, 16, 16, 256, f8.workspace_bytes, None)
        assert rc == 1
    rc = run8(ctypes.byref(f8), 16, None, ok_scale, 16, sc, None, 16, 16, 256, f8.workspace_bytes, None)
    assert rc == 1
    rc = run8(ctypes.byref(f8), 16, 16 + 4, ok_scale, 16, sc, None, 16, 16, 256, f8.workspace_bytes, None)
    assert rc == 2
    rc = run8(ctypes.byref(f8), 16, 16, ok_scale, 16, sc, None, 16, 16, 256, f8.workspace_bytes - 1, None)
    assert rc == 6
    # the bf16 entry points refuse an FP8 plan
    rc = lib.mla_decode_run(ctypes.byref(f8), 16, 16, 16, sc, 16, 16, 256, f8.workspace_bytes, None)
    assert rc == 1
    rc = lib.mla_decode_run_fp8_phase(ctypes.byref(f8), 16, 16, ok_scale, 16, sc, 16, 16, 256, f8.workspace_bytes,
                                      None, 3)
    assert rc == 1


def test_fp8_operand_kernel_plan_without_gpu():
    """The FP8 operand kernels are the default FP8 plans: on a CTA pair when
    Sq*H is a multiple of 128, else the transposed one; the others are chosen
    explicitly; other kinds are refused, the pair kernel for shapes it cannot run."""
    for H, G in ((16, 16), (128, 32)):
        o = M.mla_decode_plan_fp8(8, 1, H, 4096, device=-1, kernel=M.MLA_KERNEL_FP8_MMA)
        assert o.kernel == M.MLA_KERNEL_FP8_MMA and o.group_rows == G and o.cta_threads == 192
        assert o.smem_bytes <= 232448
        w = M.mla_decode_plan_fp8(8, 1, H, 4096, device=-1, kernel=M.MLA_KERNEL_FP8)
        assert w.kernel == M.MLA_KERNEL_FP8 and w.group_rows == G
    assert M.mla_decode_plan_fp8(8, 1, 16, 4096, device=-1).kernel == M.MLA_KERNEL_FP8_MMA
    for Sq, H in ((1, 128), (2, 64), (2, 128)):
        p = M.mla_decode_plan_fp8(8, Sq, H, 4096, device=-1)
        bf = M.mla_decode_plan(8, Sq, H, 4096, device=-1)
        assert p.kernel == M.MLA_KERNEL_FP8_PAIR and p.group_rows == 128 and p.cta_threads == 256
        assert p.num_groups == bf.num_groups and p.num_partitions == bf.num_partitions
        assert p.workspace_bytes == bf.workspace_bytes and p.smem_bytes <= 232448
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_plan_fp8(8, 1, 16, 4096, device=-1, kernel=M.MLA_KERNEL_FP8_PAIR)
    assert e.value.code == 3
    for bad in (1, 2, 3, 7):
        with pytest.raises(M.MlaError) as e:
            M.mla_decode_plan_fp8(8, 1, 16, 4096, device=-1, kernel=bad)
        assert e.value.code == 1


def test_fp8_input_generator():
    """generate_fp8: kv_scale = max|kv| / 448 over the used rows (fp32), codes
    are torch's E4M3 rounding of kv / kv_scale, and rows past a length hold
    the NaN code; q and lengths are those of the bf16 generator."""
    from mla_decode_attention_11_b200 import workloads as W
    w = W.custom(B=3, Sq=1, H=16, L=300, L_lo=10, seed=77)
    q, codes, ks, sl = W.generate_fp8(w)
    q0, kv, sl0 = W.generate(w, tail_fill=0.0)
    assert torch.equal(q, q0) and torch.equal(sl, sl0) and codes.dtype == torch.uint8
    used = torch.cat([kv[b, :int(sl[b])] for b in range(w.B)]).float()
    assert ks == float(torch.tensor(float(used.abs().max()) / 448.0, dtype=torch.float32))
    for b in range(w.B):
        L = int(sl[b])
        vals = codes[b, :L].view(torch.float8_e4m3fn).float()
        assert torch.isfinite(vals).all() and vals.abs().max() <= 448
        ref = (kv[b, :L].float() / ks).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        assert torch.equal(codes[b, :L], ref)
        assert (codes[b, L:] == W.E4M3_NAN_CODE).all()


def test_mha_plan_without_gpu():
    p = M.mha_decode_plan(64, 1, 32, 8, 8192, device=-1)
    assert p.kernel == M.MLA_KERNEL_MHA and p.group_rows == 16 and p.num_groups == 8 and p.Hkv == 8
    assert p.head_dim == M.MHA_D and p.num_partitions == 148 // 8
    p = M.mha_decode_plan(2, 4, 32, 4, 1000, device=-1)  # Sq * H/Hkv = 32 query rows per kv head
    assert p.group_rows == 32
    for args, code in (((2, 1, 12, 5, 100), 1),      # H not a multiple of Hkv
                       ((2, 1, 8, 0, 100), 1),       # no kv heads
                       ((2, 3, 64, 4, 100), 3),      # 3 * 16 = 48 query rows per kv head > 32
                       ((0, 1, 8, 2, 100), 1)):
        with pytest.raises(M.MlaError) as e:
            M.mha_decode_plan(*args, device=-1)
        assert e.value.code == code, args


def test_mha_and_sink_runs_reject_without_launching(lib):
    """Plan kinds that do not match the entry point, misaligned pointers
    (sinks included) and short workspaces are refused on the host."""
    mha = M.mha_decode_plan(2, 1, 8, 2, 256, device=-1)
    mla = M.mla_decode_plan(2, 1, 16, 256, device=-1)
    sc = ctypes.c_float(0.09)
    run = lib.mha_decode_run
    assert run(ctypes.byref(mla), 16, 16, 16, 16, sc, None, 16, 16, 256, mla.workspace_bytes, None) == 1
    assert run(ctypes.byref(mha), 16, 16 + 2, 16, 16, sc, None, 16, 16, 256, mha.workspace_bytes, None) == 2
    assert run(ctypes.byref(mha), 16, 16, 16, 16, sc, 16 + 2, 16, 16, 256, mha.workspace_bytes, None) == 2
    assert run(ctypes.byref(mha), 16, 16, 16, 16, sc, None, 16, 16, 256, mha.workspace_bytes - 1, None) == 6
    assert lib.mla_decode_run(ctypes.byref(mha), 16, 16, 16, sc, 16, 16, 256, mha.workspace_bytes, None) == 1
    sinks_run = lib.mla_decode_run_sinks
    assert sinks_run(ctypes.byref(mla), 16, 16, 16, sc, 16 + 1, 16, 16, 256, mla.workspace_bytes, None) == 2


def test_noalloc_refuses_plans_larger_than_its_scratch(lib):
    """A plan whose workspace exceeds the library's static scratch is refused
    before any device call."""
    big = M.mla_decode_plan(4096, 1, 128, 65536, device=-1, num_partitions=4096)
    assert big.workspace_bytes > M.MLA_NOALLOC_SCRATCH_BYTES
    rc = lib.mla_decode_run_noalloc(ctypes.byref(big), 16, 16, 16, ctypes.c_float(0.04), 16, 16, 0, None)
    assert rc == 6


def test_noalloc_rejects_before_touching_the_device(lib):
    """Every argument check of the no-allocation call comes before it touches a
    device or enqueues the clearing of its status words, so a rejected call
    cannot disturb an earlier call still running on the shared scratch.  On a
    machine without a GPU the rejections therefore still name the argument
    (a device access would have returned MLA_ERR_CUDA)."""
    sc = ctypes.c_float(576 ** -0.5)
    ok = M.mla_decode_plan(4, 1, 128, 1024, device=-1)
    f8 = M.mla_decode_plan_fp8(4, 1, 16, 1024, device=-1)
    mha = M.mha_decode_plan(4, 1, 8, 2, 1024, device=-1)
    run = lib.mla_decode_run_noalloc
    assert run(ctypes.byref(f8), 16, 16, 16, sc, 16, 16, 0, None) == 1     # FP8 plan on the bf16 call
    assert run(ctypes.byref(mha), 16, 16, 16, sc, 16, 16, 0, None) == 1    # MHA plan
    assert run(ctypes.byref(ok), 16, 16, 16, ctypes.c_float(float("nan")), 16, 16, 0, None) == 1
    assert run(ctypes.byref(ok), 16, 16, 0, sc, 16, 16, 0, None) == 1      # no lengths
    assert run(ctypes.byref(ok), 16 + 2, 16, 16, sc, 16, 16, 0, None) == 2  # q not 16-byte aligned
    assert run(ctypes.byref(ok), 16, 16, 16, sc, 16 + 8, 16, 1, None) == 2  # out not 16-byte aligned
    bad = M.mla_decode_plan(4, 1, 128, 1024, device=-1)
    bad.group_rows = 64
    assert run(ctypes.byref(bad), 16, 16, 16, sc, 16, 16, 0, None) == 1
