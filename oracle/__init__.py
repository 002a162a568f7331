"""fp64 CPU oracle for MLA decode -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library (``mla_decode_attention_11_b200``) never imports it, and it imports
nothing from that library: the two share no code.  The arithmetic lives in
``mla_oracle.c`` (plain C, double precision, OpenMP over output rows); this
module only compiles it with gcc and marshals numpy/torch arrays through ctypes.

The computation (textbook scaled-dot-product attention over one shared latent
cache, keys = 576-wide rows, values = their first 512 columns, natural-log LSE)
is the one the TileLang pages use as their running example ("TileLang: Bridging
Programmability and Performance in Modern Neural Kernels", papernotes.org,
section "一个完整示例：FlashMLA 的两阶段优化"); the C file's header states it.
``mla_decode_fp8`` is the same definition over a cache of E4M3 codes with one
dequantization scale (the C file's FP8 section states the reading).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle_mla.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile mla_oracle.c into _build/liboracle_mla.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, dbl, ptr = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.oracle_mla_decode.restype = ctypes.c_int
            lib.oracle_mla_decode.argtypes = [ptr, ptr, ptr, i64, i64, i64, i64, i64, i64,
                                              dbl, ptr, ptr, ctypes.c_int]
            lib.oracle_mla_decode_rows.restype = ctypes.c_int
            lib.oracle_mla_decode_rows.argtypes = [ptr, ptr, ptr, i64, i64, i64, i64, i64, i64,
                                                   dbl, ptr, i64, ptr, ptr, ctypes.c_int]
            lib.oracle_mla_decode_sinks.restype = ctypes.c_int
            lib.oracle_mla_decode_sinks.argtypes = [ptr, ptr, ptr, i64, i64, i64, i64, i64, i64,
                                                    dbl, ptr, ptr, ptr, ctypes.c_int]
            lib.oracle_mla_decode_rows_sinks.restype = ctypes.c_int
            lib.oracle_mla_decode_rows_sinks.argtypes = [ptr, ptr, ptr, i64, i64, i64, i64, i64, i64,
                                                         dbl, ptr, ptr, i64, ptr, ptr, ctypes.c_int]
            lib.oracle_mha_decode.restype = ctypes.c_int
            lib.oracle_mha_decode.argtypes = [ptr, ptr, ptr, ptr, i64, i64, i64, i64, i64, i64, i64,
                                              dbl, ptr, ptr, ctypes.c_int]
            lib.oracle_mha_decode_sinks.restype = ctypes.c_int
            lib.oracle_mha_decode_sinks.argtypes = [ptr, ptr, ptr, ptr, i64, i64, i64, i64, i64, i64, i64,
                                                    dbl, ptr, ptr, ptr, ctypes.c_int]
            lib.oracle_mla_decode_fp8_rows.restype = ctypes.c_int
            lib.oracle_mla_decode_fp8_rows.argtypes = [ptr, ptr, dbl, ptr, i64, i64, i64, i64, i64, i64,
                                                       dbl, ptr, ptr, i64, ptr, ptr, ctypes.c_int]
            lib.oracle_e4m3_to_double.restype = dbl
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_max_threads.restype = ctypes.c_int
            lib.oracle_max_threads.argtypes = []
            _lib = lib
    return _lib


def _as_bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor (CPU) or uint16 numpy array -> C-contiguous uint16 bits."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must hold bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected a bfloat16 tensor, got {x.dtype}")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _sinks_arg(sinks, H):
    """None -> (None, NULL); else a C-contiguous float64 [H] array and its address."""
    if sinks is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(-1))
    if a.shape[0] != H:
        raise ValueError("sinks must have H entries")
    return a, a.ctypes.data


def mla_decode(q, kv, seqlens, scale: float, d_v: int = 512, num_threads: int = 0, sinks=None):
    """Oracle for every row.  q [B,Sq,H,d_qk] bf16, kv [B,L_max,d_qk] bf16,
    seqlens int [B], sinks None or [H] sink logits (one extra, value-free
    softmax term per head).  Returns (out float64 [B,Sq,H,d_v], lse float64 [B,Sq,H])."""
    qb = _as_bf16_bits(q)
    kvb = _as_bf16_bits(kv)
    if qb.ndim != 4 or kvb.ndim != 3:
        raise ValueError("q must be [B,Sq,H,d_qk] and kv [B,L_max,d_qk]")
    B, Sq, H, d_qk = qb.shape
    if kvb.shape[0] != B or kvb.shape[2] != d_qk:
        raise ValueError("q and kv disagree on B or d_qk")
    L_max = kvb.shape[1]
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    if sl.shape[0] != B:
        raise ValueError("seqlens must have B entries")
    out = np.empty((B, Sq, H, d_v), dtype=np.float64)
    lse = np.empty((B, Sq, H), dtype=np.float64)
    keep, sp = _sinks_arg(sinks, H)
    rc = _load().oracle_mla_decode_sinks(qb.ctypes.data, kvb.ctypes.data, sl.ctypes.data,
                                         B, Sq, H, L_max, d_qk, d_v, float(scale), sp,
                                         out.ctypes.data, lse.ctypes.data, int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_mla_decode failed with code {rc}")
    return out, lse


def mla_decode_rows(q, kv, seqlens, scale: float, row_ids, d_v: int = 512, num_threads: int = 0, sinks=None):
    """Oracle for selected flattened rows r = (b*Sq + t)*H + h (sinks as in
    mla_decode).  Returns (out float64 [n, d_v], lse float64 [n])."""
    qb = _as_bf16_bits(q)
    kvb = _as_bf16_bits(kv)
    B, Sq, H, d_qk = qb.shape
    L_max = kvb.shape[1]
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    rows = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64).reshape(-1))
    out = np.empty((rows.shape[0], d_v), dtype=np.float64)
    lse = np.empty((rows.shape[0],), dtype=np.float64)
    keep, sp = _sinks_arg(sinks, H)
    rc = _load().oracle_mla_decode_rows_sinks(qb.ctypes.data, kvb.ctypes.data, sl.ctypes.data,
                                              B, Sq, H, L_max, d_qk, d_v, float(scale), sp,
                                              rows.ctypes.data, rows.shape[0],
                                              out.ctypes.data, lse.ctypes.data, int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_mla_decode_rows failed with code {rc}")
    return out, lse


def mha_decode(q, k, v, seqlens, scale: float, num_threads: int = 0, sinks=None):
    """MHA decode oracle: q [B,Sq,H,D], k [B,L_max,Hkv,D], v [B,L_max,Hkv,Dv]
    (bf16), seqlens int [B]; head h reads kv head h // (H // Hkv).  sinks None
    or [H] per-head sink logits (one extra, value-free softmax term per head,
    as in mla_decode).  Returns (out float64 [B,Sq,H,Dv], lse float64 [B,Sq,H])."""
    qb, kb, vb = _as_bf16_bits(q), _as_bf16_bits(k), _as_bf16_bits(v)
    if qb.ndim != 4 or kb.ndim != 4 or vb.ndim != 4:
        raise ValueError("q must be [B,Sq,H,D], k [B,L_max,Hkv,D] and v [B,L_max,Hkv,Dv]")
    B, Sq, H, D = qb.shape
    _, L_max, Hkv, Dk = kb.shape
    Dv = vb.shape[3]
    if Dk != D or kb.shape[0] != B or vb.shape[:3] != kb.shape[:3]:
        raise ValueError("q, k and v disagree on B, L_max, Hkv or D")
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    if sl.shape[0] != B:
        raise ValueError("seqlens must have B entries")
    out = np.empty((B, Sq, H, Dv), dtype=np.float64)
    lse = np.empty((B, Sq, H), dtype=np.float64)
    keep, sp = _sinks_arg(sinks, H)
    rc = _load().oracle_mha_decode_sinks(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, sl.ctypes.data,
                                         B, Sq, H, Hkv, L_max, D, Dv, float(scale), sp,
                                         out.ctypes.data, lse.ctypes.data, int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_mha_decode failed with code {rc}")
    return out, lse


def _as_u8_codes(x) -> np.ndarray:
    """E4M3 codes: a uint8 numpy array, or a torch uint8 / float8_e4m3fn tensor."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint8:
            raise TypeError("numpy FP8 caches must hold E4M3 codes as uint8")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype == torch.float8_e4m3fn:
        x = x.view(torch.uint8)
    if x.dtype != torch.uint8:
        raise TypeError(f"expected uint8 E4M3 codes, got {x.dtype}")
    return np.ascontiguousarray(x.detach().cpu().contiguous().numpy())


def e4m3_decode(codes) -> np.ndarray:
    """Exact value of every E4M3 code (uint8 array-like), as float64."""
    c = np.asarray(codes, dtype=np.uint8)
    f = _load().oracle_e4m3_to_double
    return np.array([f(int(v)) for v in c.reshape(-1)], dtype=np.float64).reshape(c.shape)


def mla_decode_fp8(q, kv_codes, kv_scale: float, seqlens, scale: float, d_v: int = 512, num_threads: int = 0,
                   sinks=None, row_ids=None):
    """Oracle over an FP8 latent cache: kv value = kv_scale * e4m3(code).
    q [B,Sq,H,d_qk] bf16, kv_codes [B,L_max,d_qk] uint8 (or float8_e4m3fn),
    seqlens int [B], sinks None or [H].  row_ids None: every row, shapes
    ([B,Sq,H,d_v], [B,Sq,H]); else the listed flattened rows r = (b*Sq + t)*H + h,
    shapes ([n, d_v], [n])."""
    qb = _as_bf16_bits(q)
    kvc = _as_u8_codes(kv_codes)
    if qb.ndim != 4 or kvc.ndim != 3:
        raise ValueError("q must be [B,Sq,H,d_qk] and kv_codes [B,L_max,d_qk]")
    B, Sq, H, d_qk = qb.shape
    if kvc.shape[0] != B or kvc.shape[2] != d_qk:
        raise ValueError("q and kv_codes disagree on B or d_qk")
    L_max = kvc.shape[1]
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
    if sl.shape[0] != B:
        raise ValueError("seqlens must have B entries")
    if row_ids is None:
        rows, rp, n = None, None, B * Sq * H
        out = np.empty((B, Sq, H, d_v), dtype=np.float64)
        lse = np.empty((B, Sq, H), dtype=np.float64)
    else:
        rows = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64).reshape(-1))
        rp, n = rows.ctypes.data, rows.shape[0]
        out = np.empty((n, d_v), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
    keep, sp = _sinks_arg(sinks, H)
    rc = _load().oracle_mla_decode_fp8_rows(qb.ctypes.data, kvc.ctypes.data, float(kv_scale), sl.ctypes.data,
                                            B, Sq, H, L_max, d_qk, d_v, float(scale), sp, rp, n,
                                            out.ctypes.data, lse.ctypes.data, int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_mla_decode_fp8_rows failed with code {rc}")
    return out, lse
