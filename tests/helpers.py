"""Independent helpers for the oracle pins: decoding from the golden E2M1
table, exact bf16 rounding with Python fractions, brute-force routing."""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def e2m1_table() -> np.ndarray:
    vals = np.empty(16, dtype=np.float64)
    with open(os.path.join(GOLDEN_DIR, "e2m1_table.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, value = line.split()
            vals[int(code, 16)] = float(value)
    return vals


def golden_kv(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN_DIR, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            out[parts[0]] = int(parts[1])
    return out


def dense_from_table(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dense fp64 matrix: table value of each nibble (low nibble first along K)
    times 2**(scale-127), one scale per 32 consecutive K."""
    tab = e2m1_table()
    lo = tab[codes & 0xF]
    hi = tab[codes >> 4]
    vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], codes.shape[1] * 2)
    sc = np.repeat(np.exp2(scales.astype(np.float64) - 127.0), 32, axis=1)
    return vals * sc


def bf16_exact_round(v: float) -> float:
    """Nearest bfloat16 to ``v`` (ties to even), decided with exact rationals."""
    if v == 0.0 or math.isnan(v):
        return v
    a = Fraction(abs(v))
    # quantum: 8 significant bits, floor at the subnormal quantum 2^-133
    e = math.frexp(abs(v))[1]
    q = max(e - 8, -133)
    step = Fraction(2) ** q
    n = a / step
    fl = math.floor(n)
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = float(fl * step)
    return -r if v < 0 else r


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def brute_route(logits: np.ndarray, k: int, keep=None):
    """Sort every routable expert by (-logit, index); softmax of the first k."""
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        cand = [e for e in range(E) if keep is None or keep[e]]
        cand.sort(key=lambda e: (-float(logits[t, e]), e))
        sel = cand[:k]
        ids[t] = sel
        ls = np.array([float(logits[t, e]) for e in sel])
        p = np.exp(ls - ls.max())
        w[t] = p / p.sum()
    return ids, w
