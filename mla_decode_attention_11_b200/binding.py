"""Python binding of libmla_decode.so (ctypes; argument marshalling only).

Every step of MLA decode runs in the library's CUDA kernels.  PyTorch is used
here only to hold device memory, to name the current stream and to read
tensor pointers.  There is no fallback: if the library is missing or the
device is not an sm_100 GPU, the calls raise.

Entry points mirror include/mla_decode.h:
    mla_decode_plan, mla_decode_workspace_init, mla_decode_run,
    mla_decode_check, mla_status_string, mla_decode_set_debug,
    mla_decode_run_noalloc, mla_decode_run_sinks
plus the convenience wrappers ``mla_decode`` (device tensors in, device
tensors out) and ``mla_decode_host`` (host tensors in and out, with the
copies done here around the library call).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

from . import build as _build

D_QK = 576
D_V = 512

MLA_OK = 0
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_ALIGNMENT", 3: "MLA_ERR_UNSUPPORTED",
                4: "MLA_ERR_CUDA", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_WORKSPACE", 7: "MLA_ERR_SEQLEN"}
MLA_KERNEL_TRANSPOSED = 1
MLA_KERNEL_PAIR = 2
MLA_KERNEL_MHA = 3
MLA_KERNEL_FP8 = 4
MLA_KERNEL_FP8_MMA = 5
MLA_KERNEL_FP8_PAIR = 6
MHA_D = 128
MLA_NOALLOC_SCRATCH_BYTES = 40 * 1024 * 1024

EXPORTED_SYMBOLS = ("mla_decode_plan", "mla_decode_plan_kernel", "mla_decode_plan_batch_invariant", "mla_decode_workspace_init", "mla_decode_run", "mla_decode_run_phase",
                    "mla_decode_check", "mla_decode_run_noalloc", "mla_decode_run_sinks",
                    "mla_status_string", "mla_decode_abi_version", "mla_decode_set_debug",
                    "mha_decode_plan", "mha_decode_run", "mha_decode_run_phase",
                    "mla_decode_plan_fp8", "mla_decode_plan_fp8_kernel", "mla_decode_run_fp8",
                    "mla_decode_run_fp8_phase")


class MlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class mla_plan(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Sq", ctypes.c_int32), ("H", ctypes.c_int32), ("L_max", ctypes.c_int32),
                ("device", ctypes.c_int32), ("num_sms", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("group_rows", ctypes.c_int32), ("num_groups", ctypes.c_int32),
                ("num_partitions", ctypes.c_int32), ("tile_kv", ctypes.c_int32), ("cta_threads", ctypes.c_int32),
                ("smem_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
                ("l2_prefetch_tiles", ctypes.c_int32), ("split_tiles", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("reserved", ctypes.c_uint64 * 4)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_ if not k.startswith("reserved")}


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def load_library(build_if_missing: bool = True):
    """Load (building first if needed) libmla_decode.so; raises if it cannot."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.LIB_PATH
        if not os.path.exists(path):
            if not build_if_missing:
                raise OSError(f"libmla_decode.so not built ({path}); run python -m mla_decode_attention_11_b200.build")
            _build.build()
        lib = ctypes.CDLL(path)
        c_i32, c_sz, c_vp, c_f = ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
        lib.mla_decode_plan.restype = c_i32
        lib.mla_decode_plan.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.POINTER(mla_plan),
                                        ctypes.POINTER(c_sz)]
        lib.mla_decode_plan_kernel.restype = c_i32
        lib.mla_decode_plan_kernel.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                               ctypes.POINTER(mla_plan), ctypes.POINTER(c_sz)]
        lib.mla_decode_plan_batch_invariant.restype = c_i32
        lib.mla_decode_plan_batch_invariant.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                                        ctypes.POINTER(mla_plan), ctypes.POINTER(c_sz)]
        lib.mla_decode_workspace_init.restype = c_i32
        lib.mla_decode_workspace_init.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_sz, c_vp]
        lib.mla_decode_run.restype = c_i32
        lib.mla_decode_run.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_vp, c_f, c_vp, c_vp, c_vp, c_sz,
                                       c_vp]
        lib.mla_decode_run_sinks.restype = c_i32
        lib.mla_decode_run_sinks.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_vp, c_f, c_vp, c_vp, c_vp, c_vp,
                                             c_sz, c_vp]
        lib.mla_decode_run_phase.restype = c_i32
        lib.mla_decode_run_phase.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_vp, c_f, c_vp, c_vp, c_vp,
                                             c_sz, c_vp, c_i32]
        lib.mla_decode_run_noalloc.restype = c_i32
        lib.mla_decode_run_noalloc.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_vp, c_f, c_vp, c_vp, c_i32,
                                               c_vp]
        lib.mha_decode_plan.restype = c_i32
        lib.mha_decode_plan.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.POINTER(mla_plan),
                                        ctypes.POINTER(c_sz)]
        lib.mha_decode_run.restype = c_i32
        lib.mha_decode_run.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_vp, c_vp, c_f, c_vp, c_vp, c_vp, c_vp,
                                       c_sz, c_vp]
        lib.mha_decode_run_phase.restype = c_i32
        lib.mha_decode_run_phase.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_vp, c_vp, c_f, c_vp, c_vp, c_vp,
                                             c_vp, c_sz, c_vp, c_i32]
        lib.mla_decode_plan_fp8.restype = c_i32
        lib.mla_decode_plan_fp8.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.POINTER(mla_plan),
                                            ctypes.POINTER(c_sz)]
        lib.mla_decode_plan_fp8_kernel.restype = c_i32
        lib.mla_decode_plan_fp8_kernel.argtypes = [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                                   ctypes.POINTER(mla_plan), ctypes.POINTER(c_sz)]
        lib.mla_decode_run_fp8.restype = c_i32
        lib.mla_decode_run_fp8.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_f, c_vp, c_f, c_vp, c_vp, c_vp,
                                           c_vp, c_sz, c_vp]
        lib.mla_decode_run_fp8_phase.restype = c_i32
        lib.mla_decode_run_fp8_phase.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp, c_f, c_vp, c_f, c_vp, c_vp,
                                                 c_vp, c_sz, c_vp, c_i32]
        lib.mla_decode_check.restype = c_i32
        lib.mla_decode_check.argtypes = [ctypes.POINTER(mla_plan), c_vp, c_vp]
        lib.mla_status_string.restype = ctypes.c_char_p
        lib.mla_status_string.argtypes = [c_i32]
        lib.mla_decode_abi_version.restype = c_i32
        lib.mla_decode_abi_version.argtypes = []
        lib.mla_decode_set_debug.restype = c_i32
        lib.mla_decode_set_debug.argtypes = [ctypes.c_uint64, c_i32]
        _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().mla_status_string(int(code)).decode()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def mla_decode_plan(B: int, Sq: int, H: int, L_max: int, device: Optional[int] = None,
                    num_partitions: int = 0, kernel: int = 0) -> mla_plan:
    """Validate a shape and choose kernel / grid / workspace size.  device=None
    means the current CUDA device; device=-1 plans for a B200 without a GPU.
    kernel: 0 = automatic, MLA_KERNEL_TRANSPOSED or MLA_KERNEL_PAIR
    (mla_decode_plan_kernel)."""
    if device is None:
        device = torch.cuda.current_device()
    p = mla_plan()
    ws = ctypes.c_size_t(0)
    lib = load_library()
    if kernel:
        rc = lib.mla_decode_plan_kernel(int(B), int(Sq), int(H), int(L_max), int(device), int(num_partitions),
                                        int(kernel), ctypes.byref(p), ctypes.byref(ws))
    else:
        rc = lib.mla_decode_plan(int(B), int(Sq), int(H), int(L_max), int(device), int(num_partitions),
                                 ctypes.byref(p), ctypes.byref(ws))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_plan")
    return p


def mla_decode_plan_batch_invariant(B: int, Sq: int, H: int, L_max: int, device: Optional[int] = None,
                                    split_tiles: int = 0) -> mla_plan:
    """A plan whose per-sequence results are bitwise independent of the rest of
    the batch: every sequence is cut into chunks of split_tiles KV tiles
    (0 = the library default) at fixed offsets (mla_decode_plan_batch_invariant)."""
    if device is None:
        device = torch.cuda.current_device()
    p = mla_plan()
    ws = ctypes.c_size_t(0)
    rc = load_library().mla_decode_plan_batch_invariant(int(B), int(Sq), int(H), int(L_max), int(device),
                                                        int(split_tiles), ctypes.byref(p), ctypes.byref(ws))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_plan_batch_invariant")
    return p


def alloc_workspace(plan: mla_plan, device=None) -> torch.Tensor:
    """A zeroed uint8 device buffer of plan.workspace_bytes (torch allocates;
    the library never does)."""
    dev = torch.device("cuda", plan.device if plan.device >= 0 else torch.cuda.current_device())
    ws = torch.zeros(int(plan.workspace_bytes), dtype=torch.uint8, device=dev if device is None else device)
    return ws


def mla_decode_workspace_init(plan: mla_plan, workspace: torch.Tensor, stream=None) -> None:
    rc = load_library().mla_decode_workspace_init(ctypes.byref(plan), workspace.data_ptr(), workspace.numel(),
                                                  _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_workspace_init")


def _check_tensor(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def mla_decode_run(plan: mla_plan, q: torch.Tensor, kv: torch.Tensor, seqlens: torch.Tensor, softmax_scale: float,
                   out: torch.Tensor, lse: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """Enqueue one decode on `stream` (default: torch's current stream)."""
    B, Sq, H, L = plan.B, plan.Sq, plan.H, plan.L_max
    _check_tensor(q, "q", torch.bfloat16, (B, Sq, H, D_QK))
    _check_tensor(kv, "kv", torch.bfloat16, (B, L, D_QK))
    _check_tensor(seqlens, "seqlens", torch.int32, (B,))
    _check_tensor(out, "out", torch.bfloat16, (B, Sq, H, D_V))
    _check_tensor(lse, "lse", torch.float32, (B, Sq, H))
    rc = load_library().mla_decode_run(ctypes.byref(plan), q.data_ptr(), kv.data_ptr(), seqlens.data_ptr(),
                                       float(softmax_scale), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                       workspace.numel(), _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_run")


def mla_decode_run_sinks(plan: mla_plan, q: torch.Tensor, kv: torch.Tensor, seqlens: torch.Tensor,
                         softmax_scale: float, sinks: Optional[torch.Tensor], out: torch.Tensor, lse: torch.Tensor,
                         workspace: torch.Tensor, stream=None) -> None:
    """mla_decode_run with per-head attention-sink logits: sinks is a CUDA
    fp32 tensor [H] (units of the scaled scores) or None for no sinks."""
    B, Sq, H, L = plan.B, plan.Sq, plan.H, plan.L_max
    _check_tensor(q, "q", torch.bfloat16, (B, Sq, H, D_QK))
    _check_tensor(kv, "kv", torch.bfloat16, (B, L, D_QK))
    _check_tensor(seqlens, "seqlens", torch.int32, (B,))
    _check_tensor(out, "out", torch.bfloat16, (B, Sq, H, D_V))
    _check_tensor(lse, "lse", torch.float32, (B, Sq, H))
    if sinks is not None:
        _check_tensor(sinks, "sinks", torch.float32, (H,))
    rc = load_library().mla_decode_run_sinks(ctypes.byref(plan), q.data_ptr(), kv.data_ptr(), seqlens.data_ptr(),
                                             float(softmax_scale), sinks.data_ptr() if sinks is not None else None,
                                             out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                             workspace.numel(), _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_run_sinks")


def mla_decode_run_phase(plan: mla_plan, q: torch.Tensor, kv: torch.Tensor, seqlens: torch.Tensor,
                         softmax_scale: float, out: torch.Tensor, lse: torch.Tensor, workspace: torch.Tensor,
                         phase: int, stream=None) -> None:
    """One of the two launches of mla_decode_run (1 = main kernel, 2 = combine)."""
    rc = load_library().mla_decode_run_phase(ctypes.byref(plan), q.data_ptr(), kv.data_ptr(), seqlens.data_ptr(),
                                             float(softmax_scale), out.data_ptr(), lse.data_ptr(),
                                             workspace.data_ptr(), workspace.numel(), _stream_handle(stream),
                                             int(phase))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_run_phase")


def mla_decode_run_noalloc(plan: mla_plan, q: torch.Tensor, kv: torch.Tensor, seqlens: torch.Tensor,
                           softmax_scale: float, out: torch.Tensor, lse: torch.Tensor, wait_and_check: bool = False,
                           stream=None) -> None:
    """mla_decode_run for callers that may not allocate device memory while
    decoding (an engine whose KV cache took nearly all HBM at start-up, a C host
    without a device allocator): the library's own static scratch array of
    MLA_NOALLOC_SCRATCH_BYTES per device stands in for the workspace.  Calls on
    one device share that array, so calls that may overlap on the GPU race;
    make the first call on a device outside stream capture.  With
    wait_and_check the stream is synchronised and a recorded device fault
    raises, as mla_decode_check does."""
    B, Sq, H, L = plan.B, plan.Sq, plan.H, plan.L_max
    _check_tensor(q, "q", torch.bfloat16, (B, Sq, H, D_QK))
    _check_tensor(kv, "kv", torch.bfloat16, (B, L, D_QK))
    _check_tensor(seqlens, "seqlens", torch.int32, (B,))
    _check_tensor(out, "out", torch.bfloat16, (B, Sq, H, D_V))
    _check_tensor(lse, "lse", torch.float32, (B, Sq, H))
    rc = load_library().mla_decode_run_noalloc(ctypes.byref(plan), q.data_ptr(), kv.data_ptr(), seqlens.data_ptr(),
                                               float(softmax_scale), out.data_ptr(), lse.data_ptr(),
                                               int(bool(wait_and_check)), _stream_handle(stream))
    if rc != MLA_OK:
        what = "mla_decode_run_noalloc"
        if rc == 6:
            what += f" (plan needs more than the {MLA_NOALLOC_SCRATCH_BYTES} bytes of static scratch)"
        raise MlaError(rc, what)


def mla_decode_check(plan: mla_plan, workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the device status; raise on a recorded fault."""
    rc = load_library().mla_decode_check(ctypes.byref(plan), workspace.data_ptr(), _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_check")
    return rc


def mla_decode_set_debug(wait_timeout_ns: int = 0, stall_unit: int = -1) -> None:
    load_library().mla_decode_set_debug(int(wait_timeout_ns), int(stall_unit))


def mla_decode(q: torch.Tensor, kv: torch.Tensor, seqlens: torch.Tensor, softmax_scale: Optional[float] = None,
               num_partitions: int = 0, plan: Optional[mla_plan] = None,
               workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Device tensors in, (out bf16 [B,Sq,H,512], lse fp32 [B,Sq,H]) out."""
    B, Sq, H, _ = q.shape
    L = kv.shape[1]
    if softmax_scale is None:
        softmax_scale = D_QK ** -0.5
    if plan is None:
        plan = mla_decode_plan(B, Sq, H, L, device=q.device.index, num_partitions=num_partitions)
    if workspace is None:
        workspace = alloc_workspace(plan, device=q.device)
    out = torch.empty((B, Sq, H, D_V), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Sq, H), dtype=torch.float32, device=q.device)
    mla_decode_run(plan, q, kv, seqlens, softmax_scale, out, lse, workspace)
    return out, lse


def mla_decode_host(q_host: torch.Tensor, kv_host: torch.Tensor, seqlens_host: torch.Tensor,
                    softmax_scale: float, plan: mla_plan, workspace: torch.Tensor,
                    dev_bufs: Optional[dict] = None, out_host: Optional[torch.Tensor] = None,
                    lse_host: Optional[torch.Tensor] = None, stream=None):
    """End-to-end call with HOST tensors: copy q / kv / seqlens to the device,
    run, copy out / lse back (pinned host buffers make the copies async)."""
    dev = workspace.device
    if dev_bufs is None:
        dev_bufs = {}
    B, Sq, H, L = plan.B, plan.Sq, plan.H, plan.L_max
    if "q" not in dev_bufs:
        dev_bufs["q"] = torch.empty((B, Sq, H, D_QK), dtype=torch.bfloat16, device=dev)
        dev_bufs["kv"] = torch.empty((B, L, D_QK), dtype=torch.bfloat16, device=dev)
        dev_bufs["seqlens"] = torch.empty((B,), dtype=torch.int32, device=dev)
        dev_bufs["out"] = torch.empty((B, Sq, H, D_V), dtype=torch.bfloat16, device=dev)
        dev_bufs["lse"] = torch.empty((B, Sq, H), dtype=torch.float32, device=dev)
    if out_host is None:
        out_host = torch.empty((B, Sq, H, D_V), dtype=torch.bfloat16, pin_memory=True)
    if lse_host is None:
        lse_host = torch.empty((B, Sq, H), dtype=torch.float32, pin_memory=True)
    dev_bufs["q"].copy_(q_host, non_blocking=True)
    dev_bufs["kv"].copy_(kv_host, non_blocking=True)
    dev_bufs["seqlens"].copy_(seqlens_host, non_blocking=True)
    mla_decode_run(plan, dev_bufs["q"], dev_bufs["kv"], dev_bufs["seqlens"], softmax_scale, dev_bufs["out"],
                   dev_bufs["lse"], workspace, stream=stream)
    out_host.copy_(dev_bufs["out"], non_blocking=True)
    lse_host.copy_(dev_bufs["lse"], non_blocking=True)
    return out_host, lse_host


# ---------------------------------------------------------------- MHA decode

def mha_decode_plan(B: int, Sq: int, H: int, Hkv: int, L_max: int, device: Optional[int] = None,
                    num_partitions: int = 0) -> mla_plan:
    """Plan an MHA decode (128-wide heads, H query heads over Hkv kv heads)."""
    if device is None:
        device = torch.cuda.current_device()
    p = mla_plan()
    ws = ctypes.c_size_t(0)
    rc = load_library().mha_decode_plan(int(B), int(Sq), int(H), int(Hkv), int(L_max), int(device),
                                        int(num_partitions), ctypes.byref(p), ctypes.byref(ws))
    if rc != MLA_OK:
        raise MlaError(rc, "mha_decode_plan")
    return p


def mha_decode_run(plan: mla_plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seqlens: torch.Tensor,
                   softmax_scale: float, out: torch.Tensor, lse: torch.Tensor, workspace: torch.Tensor,
                   sinks: Optional[torch.Tensor] = None, stream=None) -> None:
    """Enqueue one MHA decode: q [B,Sq,H,128], k and v [B,L_max,Hkv,128] (bf16)."""
    B, Sq, H, L, Hkv = plan.B, plan.Sq, plan.H, plan.L_max, plan.Hkv
    _check_tensor(q, "q", torch.bfloat16, (B, Sq, H, MHA_D))
    _check_tensor(k, "k", torch.bfloat16, (B, L, Hkv, MHA_D))
    _check_tensor(v, "v", torch.bfloat16, (B, L, Hkv, MHA_D))
    _check_tensor(seqlens, "seqlens", torch.int32, (B,))
    _check_tensor(out, "out", torch.bfloat16, (B, Sq, H, MHA_D))
    _check_tensor(lse, "lse", torch.float32, (B, Sq, H))
    if sinks is not None:
        _check_tensor(sinks, "sinks", torch.float32, (H,))
    rc = load_library().mha_decode_run(ctypes.byref(plan), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       seqlens.data_ptr(), float(softmax_scale),
                                       sinks.data_ptr() if sinks is not None else None, out.data_ptr(),
                                       lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                       _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mha_decode_run")


def mha_decode_run_phase(plan: mla_plan, q, k, v, seqlens, softmax_scale: float, out, lse, workspace, phase: int,
                         sinks=None, stream=None) -> None:
    """One launch of mha_decode_run (1 = main kernel, 2 = combine)."""
    rc = load_library().mha_decode_run_phase(ctypes.byref(plan), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             seqlens.data_ptr(), float(softmax_scale),
                                             sinks.data_ptr() if sinks is not None else None, out.data_ptr(),
                                             lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                             _stream_handle(stream), int(phase))
    if rc != MLA_OK:
        raise MlaError(rc, "mha_decode_run_phase")


# ---------------------------------------------------------------- FP8 latent cache

def mla_decode_plan_fp8(B: int, Sq: int, H: int, L_max: int, device: Optional[int] = None,
                        num_partitions: int = 0, kernel: int = 0) -> mla_plan:
    """A plan for a cache of E4M3 codes (mla_decode_plan_fp8_kernel).  kernel = 0
    picks the default: the codes as kind::f8f6f4 MMA operands on CTA pairs
    (MLA_KERNEL_FP8_PAIR) when Sq*H is a multiple of 128, else in the
    transposed orientation (MLA_KERNEL_FP8_MMA); MLA_KERNEL_FP8 selects the
    kernel that widens the codes to f16 in shared memory."""
    if device is None:
        device = torch.cuda.current_device()
    p = mla_plan()
    ws = ctypes.c_size_t(0)
    rc = load_library().mla_decode_plan_fp8_kernel(int(B), int(Sq), int(H), int(L_max), int(device),
                                                   int(num_partitions), int(kernel), ctypes.byref(p),
                                                   ctypes.byref(ws))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_plan_fp8_kernel")
    return p


def _fp8_codes(kv_fp8: torch.Tensor) -> torch.Tensor:
    return kv_fp8.view(torch.uint8) if kv_fp8.dtype == torch.float8_e4m3fn else kv_fp8


def mla_decode_run_fp8(plan: mla_plan, q: torch.Tensor, kv_fp8: torch.Tensor, kv_scale: float,
                       seqlens: torch.Tensor, softmax_scale: float, out: torch.Tensor, lse: torch.Tensor,
                       workspace: torch.Tensor, sinks: Optional[torch.Tensor] = None, stream=None) -> None:
    """Enqueue one decode over an FP8 cache: kv_fp8 is a CUDA tensor of E4M3
    codes [B, L_max, 576] (torch.uint8 or torch.float8_e4m3fn), kv_value =
    kv_scale * e4m3(code); sinks as in mla_decode_run_sinks."""
    B, Sq, H, L = plan.B, plan.Sq, plan.H, plan.L_max
    codes = _fp8_codes(kv_fp8)
    _check_tensor(q, "q", torch.bfloat16, (B, Sq, H, D_QK))
    _check_tensor(codes, "kv_fp8", torch.uint8, (B, L, D_QK))
    _check_tensor(seqlens, "seqlens", torch.int32, (B,))
    _check_tensor(out, "out", torch.bfloat16, (B, Sq, H, D_V))
    _check_tensor(lse, "lse", torch.float32, (B, Sq, H))
    if sinks is not None:
        _check_tensor(sinks, "sinks", torch.float32, (H,))
    rc = load_library().mla_decode_run_fp8(ctypes.byref(plan), q.data_ptr(), codes.data_ptr(), float(kv_scale),
                                           seqlens.data_ptr(), float(softmax_scale),
                                           sinks.data_ptr() if sinks is not None else None, out.data_ptr(),
                                           lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                           _stream_handle(stream))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_run_fp8")


def mla_decode_run_fp8_phase(plan: mla_plan, q: torch.Tensor, kv_fp8: torch.Tensor, kv_scale: float,
                             seqlens: torch.Tensor, softmax_scale: float, out: torch.Tensor, lse: torch.Tensor,
                             workspace: torch.Tensor, phase: int, stream=None) -> None:
    """One of the two launches of mla_decode_run_fp8 (1 = main kernel, 2 = combine)."""
    codes = _fp8_codes(kv_fp8)
    rc = load_library().mla_decode_run_fp8_phase(ctypes.byref(plan), q.data_ptr(), codes.data_ptr(),
                                                 float(kv_scale), seqlens.data_ptr(), float(softmax_scale),
                                                 out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                                 workspace.numel(), _stream_handle(stream), int(phase))
    if rc != MLA_OK:
        raise MlaError(rc, "mla_decode_run_fp8_phase")
