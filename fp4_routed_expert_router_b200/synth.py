"""Seeded synthetic inputs for the routed-expert FP4 FFN.

This module is the one place both the CUDA path and the CPU oracle get their
inputs from.  It holds none of the method's arithmetic: it only draws bytes,
exponents, activations and logits with the shapes and distributions of the
DeepSeek-V4.1-Flash routed-expert layer (10100.com article 151357339, section
"moe专家的容量瓶颈": w1/w3 codes [2304,2560] + UE8M0 scales [2304,160], w2 codes
[5120,1152] + scales [5120,72], 384 routed experts, 6 per token).

Generators
----------
* Expert weights come from a counter-based generator, splitmix64 (Steele, Lea
  and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014;
  the 64-bit finaliser constants are Stafford's "Mix13").  Output i of a
  stream with key K is ``mix(K + (i+1)*0x9E3779B97F4A7C15)``.  Because output i
  depends only on (K, i), the library's device-side generator
  (``csrc/synth_fill.cu``) produces the same bytes for the same key without any
  state, which is what lets a 115 GB arena be filled on the GPU while the oracle
  regenerates only the experts it needs on the host.
* Activations and logits are small, so they are drawn on the host with numpy's
  PCG64 and copied to the device.

Expert byte layout (the "checkpoint layout"): one contiguous object per expert
with w1 codes, w3 codes, w2 codes, then s1, s3, s2 scales, each row-major
[out_features, in_features/2] (codes) or [out_features, in_features/32]
(scales); the low nibble of a code byte is the even K index.  Codes first and
scales after, each contiguous, as the article describes the on-disk object
(section "SSD读取性能").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1

# tensor ids inside one expert object (also the splitmix64 stream ids)
W1, S1, W3, S3, W2, S2 = 0, 1, 2, 3, 4, 5
TENSOR_NAMES = ("w1", "s1", "w3", "s3", "w2", "s2")


# ----------------------------------------------------------------------------
# splitmix64 (scalar and vector forms)
# ----------------------------------------------------------------------------
def mix64(z: int) -> int:
    """splitmix64 output function applied to one 64-bit integer."""
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def stream_key(seed: int, layer: int, expert: int, tensor: int) -> int:
    """Key of the splitmix64 stream for one tensor of one expert."""
    sid = ((layer & 0xFFFF) << 20) | ((expert & 0xFFFF) << 4) | (tensor & 0xF)
    return mix64((mix64(seed) + (sid + 1) * GOLDEN) & _M64)


def splitmix64_stream(key: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs start..start+n-1 of the splitmix64 stream with state ``key``."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_bytes(key: int, nbytes: int) -> np.ndarray:
    """``nbytes`` uniform bytes: the little-endian bytes of consecutive outputs."""
    n64 = (nbytes + 7) // 8
    return splitmix64_stream(key, n64).view(np.uint8)[:nbytes].copy()


def stream_exponents(key: int, n: int, lo: int, hi: int) -> np.ndarray:
    """``n`` UE8M0 exponents uniform on [lo, hi]: one output per exponent,
    ``lo + ((u >> 32) * (hi - lo + 1)) >> 32`` (multiply-shift range reduction)."""
    u = splitmix64_stream(key, n)
    span = np.uint64(hi - lo + 1)
    with np.errstate(over="ignore"):
        e = ((u >> np.uint64(32)) * span) >> np.uint64(32)
    return (e + np.uint64(lo)).astype(np.uint8)


# ----------------------------------------------------------------------------
# expert objects
# ----------------------------------------------------------------------------
def expert_layout(hidden: int, inter: int) -> dict:
    """Byte offset and shape of each tensor inside one expert object."""
    shapes = {
        "w1": (inter, hidden // 2),
        "w3": (inter, hidden // 2),
        "w2": (hidden, inter // 2),
        "s1": (inter, hidden // 32),
        "s3": (inter, hidden // 32),
        "s2": (hidden, inter // 32),
    }
    off = 0
    out = {}
    for name in ("w1", "w3", "w2", "s1", "s3", "s2"):
        r, c = shapes[name]
        out[name] = (off, (r, c))
        off += r * c
    out["total"] = off
    return out


def gen_expert(seed: int, layer: int, expert: int, hidden: int, inter: int,
               scale_lo: int, scale_hi: int) -> dict:
    """One expert's six tensors (checkpoint layout) as numpy uint8 arrays."""
    lay = expert_layout(hidden, inter)
    out = {}
    for tid, name in enumerate(TENSOR_NAMES):
        _, (r, c) = lay[name]
        key = stream_key(seed, layer, expert, tid)
        if name.startswith("w"):
            out[name] = stream_bytes(key, r * c).reshape(r, c)
        else:
            out[name] = stream_exponents(key, r * c, scale_lo, scale_hi).reshape(r, c)
    return out


def expert_object(tensors: dict, hidden: int, inter: int) -> np.ndarray:
    """Concatenate the six tensors into one contiguous expert object."""
    lay = expert_layout(hidden, inter)
    buf = np.empty(lay["total"], dtype=np.uint8)
    for name in ("w1", "w3", "w2", "s1", "s3", "s2"):
        off, (r, c) = lay[name]
        buf[off:off + r * c] = tensors[name].reshape(-1)
    return buf


# ----------------------------------------------------------------------------
# activations, logits, popularity bias
# ----------------------------------------------------------------------------
def _rng(seed: int, *tags: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed & _M64, *tags])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def gen_x(seed: int, tokens: int, hidden: int, step: int = 0) -> np.ndarray:
    """Activations: bf16(N(0,1)), rounded to nearest even.  uint16 bits [T, H]."""
    z = _rng(seed, 101, step).standard_normal((tokens, hidden), dtype=np.float32)
    return f32_to_bf16_bits(z)


def zipf_rank(seed: int, layer: int, n_experts: int) -> np.ndarray:
    """Popularity rank (1 = most popular) of each expert: a seeded permutation."""
    perm = _rng(seed, 202, layer).permutation(n_experts)
    rank = np.empty(n_experts, dtype=np.int64)
    rank[perm] = np.arange(1, n_experts + 1)
    return rank


def zipf_bias(seed: int, layer: int, n_experts: int, alpha: float, s: float = 1.1) -> np.ndarray:
    """Per-expert logit bias alpha*(ln p_rank(e) - mean_r ln p_r), p_r ~ r^-s.

    Centred log-popularity of a Zipf(s) law over a seeded ranking; alpha sets
    how strongly the router concentrates on the popular experts."""
    if alpha == 0.0:
        return np.zeros(n_experts, dtype=np.float32)
    r = np.arange(1, n_experts + 1, dtype=np.float64)
    lnp = -s * np.log(r)
    lnp -= np.log(np.exp(lnp).sum())
    rank = zipf_rank(seed, layer, n_experts)
    return (alpha * (lnp[rank - 1] - lnp.mean())).astype(np.float32)


def gen_logits(seed: int, layer: int, tokens: int, n_experts: int, alpha: float,
               step: int = 0) -> np.ndarray:
    """Router logits: fp32 N(0,1) plus the layer's popularity bias.  [T, E]."""
    z = _rng(seed, 303, layer, step).standard_normal((tokens, n_experts), dtype=np.float32)
    return (z + zipf_bias(seed, layer, n_experts, alpha)[None, :]).astype(np.float32)


def keep_mask(seed: int, layer: int, n_experts: int, n_keep: int) -> np.ndarray:
    """uint8 [E]: 1 for the ``n_keep`` most popular experts of the layer's ranking."""
    return (zipf_rank(seed, layer, n_experts) <= n_keep).astype(np.uint8)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    tokens: int
    n_layers: int = 1
    scale_lo: int = 118
    scale_hi: int = 124
    zipf_alpha: float = 0.0
    n_keep: int = 0          # 0: no mask (all experts routable)
    seed: int = 20260917
    notes: str = field(default="", compare=False)

    @property
    def n_slots(self) -> int:
        kept = self.n_keep if self.n_keep else self.n_experts
        return kept * self.n_layers

    @property
    def expert_bytes(self) -> int:
        return expert_layout(self.hidden, self.inter)["total"]


WORKLOADS = {
    "tiny": Workload("tiny", 256, 128, 16, 2, 4, scale_lo=120, scale_hi=126,
                     notes="hidden 256, inter 128, 16 experts, top-2, 4 tokens"),
    "decode_b1": Workload("decode_b1", 5120, 2304, 384, 6, 1, zipf_alpha=0.5,
                          notes="one V4.1-Flash layer, 384 experts resident, batch 1"),
    "decode_b64": Workload("decode_b64", 5120, 2304, 384, 6, 64, zipf_alpha=0.5,
                           notes="one V4.1-Flash layer, 384 experts resident, batch 64"),
    "prefill_2048": Workload("prefill_2048", 5120, 2304, 384, 6, 2048, zipf_alpha=0.47,
                             notes="one V4.1-Flash layer, 2048-token prefill chunk"),
    "drafter_b1": Workload("drafter_b1", 5120, 2304, 128, 3, 1, zipf_alpha=0.5,
                           notes="drafter-shaped MoE (128 experts, top-3) at the layer's hidden/inter, batch 1"),
    "drafter_b256": Workload("drafter_b256", 5120, 2304, 128, 3, 256, zipf_alpha=0.5,
                             notes="drafter-shaped MoE (128 experts, top-3), batch 256"),
    "stack40_b1": Workload("stack40_b1", 5120, 2304, 384, 6, 1, n_layers=40, zipf_alpha=0.5,
                           n_keep=154, notes="40 layers x 154 kept experts, batch 1"),
    "stack40_b8": Workload("stack40_b8", 5120, 2304, 384, 6, 8, n_layers=40, zipf_alpha=0.5,
                           n_keep=154, notes="40 layers x 154 kept experts, batch 8"),
}


def layer_inputs(wl: Workload, layer: int = 0, step: int = 0, tokens: int | None = None):
    """(logits [T,E] f32, keep mask [E] u8 or None) for one layer of a workload."""
    t = wl.tokens if tokens is None else tokens
    logits = gen_logits(wl.seed, layer, t, wl.n_experts, wl.zipf_alpha, step)
    mask = keep_mask(wl.seed, layer, wl.n_experts, wl.n_keep) if wl.n_keep else None
    return logits, mask


def resident_experts(wl: Workload, layer: int) -> np.ndarray:
    """Experts of ``layer`` that own an arena slot (all, or the kept set)."""
    if wl.n_keep:
        return np.nonzero(keep_mask(wl.seed, layer, wl.n_experts, wl.n_keep))[0]
    return np.arange(wl.n_experts)
