"""ctypes binding of the CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.oracle_e2m1.restype = ctypes.c_double
        _lib.oracle_e2m1.argtypes = [ctypes.c_uint]
        _lib.oracle_ue8m0.restype = ctypes.c_double
        _lib.oracle_ue8m0.argtypes = [ctypes.c_uint]
        _lib.oracle_bf16_rne.restype = ctypes.c_uint16
        _lib.oracle_bf16_rne.argtypes = [ctypes.c_double]
        _lib.oracle_bf16_to_double.restype = ctypes.c_double
        _lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        _lib.oracle_expert_bytes.restype = ctypes.c_longlong
        _lib.oracle_expert_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
        _lib.oracle_dequant.restype = None
        _lib.oracle_dequant.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P]
        _lib.oracle_route.restype = ctypes.c_int
        _lib.oracle_route.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        _lib.oracle_permute.restype = None
        _lib.oracle_permute.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
        _lib.oracle_expert_ffn.restype = None
        _lib.oracle_expert_ffn.argtypes = [P, ctypes.c_int, ctypes.c_int] + [P] * 8
        _lib.oracle_moe_forward.restype = ctypes.c_int
        _lib.oracle_moe_forward.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, P, P, P,
                                            ctypes.c_int, P]
        _lib.oracle_moe_saliency.restype = ctypes.c_int
        _lib.oracle_moe_saliency.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, P, P, P,
                                            ctypes.c_int, P]
        _lib.oracle_residual.restype = None
        _lib.oracle_residual.argtypes = [P, P, ctypes.c_size_t]
        _lib.oracle_max_threads.restype = ctypes.c_int
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def e2m1(code: int) -> float:
    return lib().oracle_e2m1(code)


def ue8m0(e: int) -> float:
    return lib().oracle_ue8m0(e)


def bf16_rne(v: float) -> int:
    return lib().oracle_bf16_rne(float(v))


def bf16_to_double(b: int) -> float:
    return lib().oracle_bf16_to_double(b)


def expert_bytes(hidden: int, inter: int) -> int:
    return lib().oracle_expert_bytes(hidden, inter)


def dequant(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    lib().oracle_dequant(_p(codes), _p(scales), rows, K, _p(out))
    return out


def route(logits: np.ndarray, k: int, keep: np.ndarray | None = None):
    """-> (ids int32 [T,k], w float64 [T,k]); raises ValueError on bad input."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    kp = None
    if keep is not None:
        keep = np.ascontiguousarray(keep, dtype=np.uint8)
        kp = _p(keep)
    rc = lib().oracle_route(_p(logits), kp, T, E, k, _p(ids), _p(w))
    if rc != 0:
        raise ValueError(f"oracle_route failed ({rc})")
    return ids, w


def permute(ids: np.ndarray, n_experts: int):
    """-> (counts [E], offsets [E+1], perm [T*k]) int32."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(n_experts, dtype=np.int32)
    offsets = np.empty(n_experts + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    lib().oracle_permute(_p(ids), T, k, n_experts, _p(counts), _p(offsets), _p(perm))
    return counts, offsets, perm


def expert_ffn(x: np.ndarray, t: dict):
    """One token through one expert: -> (h bf16 bits [I], o float64 [H])."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    H = x.shape[0]
    I = t["w1"].shape[0]
    h = np.empty(I, dtype=np.uint16)
    o = np.empty(H, dtype=np.float64)
    a = [np.ascontiguousarray(t[n], dtype=np.uint8) for n in ("w1", "s1", "w3", "s3", "w2", "s2")]
    lib().oracle_expert_ffn(_p(x), H, I, *[_p(v) for v in a], _p(h), _p(o))
    return h, o


def moe_forward(x: np.ndarray, ids: np.ndarray, w: np.ndarray, objs: dict, n_experts: int,
                hidden: int, inter: int, n_threads: int = 0) -> np.ndarray:
    """y float64 [T,H].  ``objs`` maps expert id -> contiguous expert object."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, k = ids.shape
    keep = [np.ascontiguousarray(objs[e], dtype=np.uint8) if e in objs else None
            for e in range(n_experts)]
    ptrs = (ctypes.c_void_p * n_experts)(*[(v.ctypes.data if v is not None else None)
                                           for v in keep])
    y = np.empty((T, hidden), dtype=np.float64)
    rc = lib().oracle_moe_forward(_p(x), T, hidden, inter, n_experts, k, _p(ids), _p(w),
                                  ctypes.cast(ptrs, ctypes.c_void_p), n_threads, _p(y))
    if rc != 0:
        raise ValueError(f"oracle_moe_forward failed ({rc})")
    return y


def saliency(x: np.ndarray, ids: np.ndarray, w: np.ndarray, objs: dict, n_experts: int, hidden: int, inter: int,
             n_threads: int = 0) -> np.ndarray:
    """Per-expert saliency float64 [E]: sum of w[t,j] * ||o_{t,j}||_2 over the
    entries routed to each expert (zero for experts nobody chose)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, k = ids.shape
    keep = [np.ascontiguousarray(objs[e], dtype=np.uint8) if e in objs else None
            for e in range(n_experts)]
    ptrs = (ctypes.c_void_p * n_experts)(*[(v.ctypes.data if v is not None else None)
                                           for v in keep])
    sal = np.zeros(n_experts, dtype=np.float64)
    rc = lib().oracle_moe_saliency(_p(x), T, hidden, inter, n_experts, k, _p(ids), _p(w),
                                   ctypes.cast(ptrs, ctypes.c_void_p), n_threads, _p(sal))
    if rc != 0:
        raise ValueError(f"oracle_moe_saliency failed ({rc})")
    return sal


def residual(x: np.ndarray, y: np.ndarray) -> np.ndarray:
    x = np.array(x, dtype=np.uint16, copy=True, order="C")
    y = np.ascontiguousarray(y, dtype=np.float64)
    lib().oracle_residual(_p(x), _p(y), x.size)
    return x


def max_threads() -> int:
    return lib().oracle_max_threads()
