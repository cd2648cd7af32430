"""Thin ctypes binding of libmoe_fp4 (include/moe_fp4.h).

Argument marshalling only: torch provides device memory and streams, every
step of the layer runs in the library's CUDA kernels.  Loading fails loudly
when the library is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libmoe_fp4.so")
SYNTH_PATH = os.path.join(_PKG, "lib", "libmoe_synth.so")

OK, EINVAL, ENOMEM, ECUDA, ESLOT, ETIMEOUT = 0, 1, 2, 3, 4, 5
STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ENOMEM", 3: "ECUDA", 4: "ESLOT", 5: "ETIMEOUT"}
PATH_AUTO, PATH_GEMV, PATH_TC = 0, 1, 2
OPT_PATH, OPT_PROFILE, OPT_WAIT_LIMIT_US = 1, 2, 3

# every symbol include/moe_fp4.h declares
EXPORTS = ("moe_fp4_slot_bytes", "moe_fp4_create", "moe_fp4_destroy", "moe_fp4_arena",
           "moe_fp4_set_option", "moe_fp4_profile_read", "moe_fp4_load_expert_slot", "moe_fp4_route",
           "moe_fp4_forward", "moe_fp4_route_forward", "moe_fp4_last_error", "moe_fp4_forward_noalloc",
           "moe_fp4_saliency", "moe_fp4_stream_experts", "moe_fp4_residency_stats", "moe_fp4_expert_outputs",
           "moe_fp4_combine")


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_slots", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32)]


_lib = None
_synth = None


def load(path: str = LIB_PATH):
    """Load libmoe_fp4.so (raises if it is missing: no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} not built: run python -m fp4_routed_expert_router_b200.build")
        L = ctypes.CDLL(path)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.moe_fp4_slot_bytes.restype = SZ
        L.moe_fp4_slot_bytes.argtypes = [ctypes.POINTER(Config)]
        L.moe_fp4_create.restype = I32
        L.moe_fp4_create.argtypes = [ctypes.POINTER(Config), I32, P, SZ, ctypes.POINTER(P)]
        L.moe_fp4_destroy.restype = None
        L.moe_fp4_destroy.argtypes = [P]
        L.moe_fp4_arena.restype = P
        L.moe_fp4_arena.argtypes = [P]
        L.moe_fp4_set_option.restype = I32
        L.moe_fp4_set_option.argtypes = [P, I32, I32]
        L.moe_fp4_profile_read.restype = I32
        L.moe_fp4_profile_read.argtypes = [P, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float), I32]
        L.moe_fp4_load_expert_slot.restype = I32
        L.moe_fp4_load_expert_slot.argtypes = [P, I32, I32, I32, P, P, P, P, P, P, P]
        L.moe_fp4_route.restype = I32
        L.moe_fp4_route.argtypes = [P, I32, P, P, I32, P, P, P, P, P, P]
        L.moe_fp4_forward.restype = I32
        L.moe_fp4_forward.argtypes = [P, I32, P, I32, P, P, P, P, P, P, P, P]
        L.moe_fp4_route_forward.restype = I32
        L.moe_fp4_route_forward.argtypes = [P, I32, P, P, P, I32, P, P, P, P, P, P, P, P]
        L.moe_fp4_saliency.restype = I32
        L.moe_fp4_saliency.argtypes = [P, I32, P, P, P, P, P]
        L.moe_fp4_stream_experts.restype = I32
        L.moe_fp4_stream_experts.argtypes = [P, I32, P, I32, P, P, P]
        L.moe_fp4_residency_stats.restype = I32
        L.moe_fp4_residency_stats.argtypes = [P, P]
        L.moe_fp4_expert_outputs.restype = I32
        L.moe_fp4_expert_outputs.argtypes = [P, I32, P, I32, P, P, P]
        L.moe_fp4_combine.restype = I32
        L.moe_fp4_combine.argtypes = [P, I32, P, P, P, P, P, P]
        L.moe_fp4_last_error.restype = I32
        L.moe_fp4_last_error.argtypes = [P, ctypes.c_char_p, SZ]
        L.moe_fp4_forward_noalloc.restype = I32
        L.moe_fp4_forward_noalloc.argtypes = [ctypes.POINTER(Config), P, P, I32, P, I32, P, P, P, P, P, P, P]
        _lib = L
    return _lib


def load_synth(path: str = SYNTH_PATH):
    global _synth
    if _synth is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} not built")
        S = ctypes.CDLL(path)
        S.moe_synth_expert_bytes.restype = ctypes.c_size_t
        S.moe_synth_expert_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
        S.moe_synth_l2_discard.restype = ctypes.c_int
        S.moe_synth_l2_discard.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        S.moe_synth_fill_expert.restype = ctypes.c_int
        S.moe_synth_fill_expert.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_void_p]
        _synth = S
    return _synth


def _ptr(t) -> ctypes.c_void_p | None:
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def synth_fill_expert(dst: torch.Tensor, seed: int, layer: int, expert: int, hidden: int, inter: int,
                      scale_lo: int, scale_hi: int, stream=None) -> None:
    """Write the synthetic expert (seed, layer, expert) into ``dst`` (uint8, device)
    in checkpoint layout, bit-identical to ``synth.expert_object``."""
    rc = load_synth().moe_synth_fill_expert(_ptr(dst), seed & ((1 << 64) - 1), layer, expert, hidden, inter,
                                            scale_lo, scale_hi, _stream(stream))
    if rc != 0:
        raise RuntimeError(f"moe_synth_fill_expert failed: cuda error {rc}")


def l2_flush(buf: torch.Tensor, value: float = 0.0, stream=None) -> None:
    """Push every earlier line out of L2 by writing ``buf`` (larger than L2),
    then drop ``buf``'s own lines without write-back: the next kernel starts
    with a cold, clean L2."""
    if stream is None:
        buf.fill_(value)
    else:
        with torch.cuda.stream(stream):
            buf.fill_(value)
    n = buf.numel() * buf.element_size() // 128 * 128
    rc = load_synth().moe_synth_l2_discard(_ptr(buf), n, _stream(stream))
    if rc != 0:
        raise RuntimeError(f"moe_synth_l2_discard failed: cuda error {rc}")


@dataclass
class Routing:
    ids: torch.Tensor       # int32 [T, k]
    weights: torch.Tensor   # fp32 [T, k]
    counts: torch.Tensor    # int32 [E]
    offsets: torch.Tensor   # int32 [E+1]
    perm: torch.Tensor      # int32 [T*k]


class Context:
    """One moe_fp4 context: arena + slot table + workspace on one device."""

    def __init__(self, hidden: int, inter: int, n_experts: int, top_k: int, n_layers: int, n_slots: int,
                 max_tokens: int, device: int = 0, arena: torch.Tensor | None = None):
        self.lib = load()
        self.cfg = Config(hidden, inter, n_experts, top_k, n_layers, n_slots, max_tokens)
        self.device = device
        self._arena_ref = arena
        h = ctypes.c_void_p()
        nbytes = arena.numel() * arena.element_size() if arena is not None else 0
        rc = self.lib.moe_fp4_create(ctypes.byref(self.cfg), device, _ptr(arena), nbytes, ctypes.byref(h))
        if rc != OK:
            raise MoeError(rc, "moe_fp4_create failed")
        self.h = h

    # ------------------------------------------------------------------ basics
    @property
    def slot_bytes(self) -> int:
        return self.lib.moe_fp4_slot_bytes(ctypes.byref(self.cfg))

    def arena_ptr(self) -> int:
        return self.lib.moe_fp4_arena(self.h)

    def close(self) -> None:
        if getattr(self, "h", None):
            self.lib.moe_fp4_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, rc: int, what: str) -> None:
        if rc != OK:
            buf = ctypes.create_string_buffer(256)
            self.lib.moe_fp4_last_error(self.h, buf, 256)
            raise MoeError(rc, f"{what}: {buf.value.decode()}")

    def last_error(self) -> tuple[int, str]:
        buf = ctypes.create_string_buffer(256)
        rc = self.lib.moe_fp4_last_error(self.h, buf, 256)
        return rc, buf.value.decode()

    def set_path(self, path: int) -> None:
        self._check(self.lib.moe_fp4_set_option(self.h, OPT_PATH, path), "set_option")

    def set_wait_limit_us(self, us: int) -> None:
        """Limit of every bounded device-side wait (0 restores the default, 1 s)."""
        self._check(self.lib.moe_fp4_set_option(self.h, OPT_WAIT_LIMIT_US, int(us)), "set_option")

    def set_profile(self, on: bool) -> None:
        self._check(self.lib.moe_fp4_set_option(self.h, OPT_PROFILE, 1 if on else 0), "set_option")

    def profile_read(self, max_records: int = 65536) -> list[tuple[str, float]]:
        """[(kernel name, device ms)] of the profiled launches since the last read."""
        names = (ctypes.c_char_p * max_records)()
        ms = (ctypes.c_float * max_records)()
        n = self.lib.moe_fp4_profile_read(self.h, names, ms, max_records)
        if n < 0:
            raise MoeError(ECUDA, "moe_fp4_profile_read failed")
        return [(names[i].decode(), float(ms[i])) for i in range(n)]

    # ------------------------------------------------------------------ calls
    def load_expert_slot(self, layer: int, expert: int, slot: int, t: dict | None, stream=None) -> None:
        """``t``: w1, s1, w3, s3, w2, s2 tensors in checkpoint layout (host or device),
        or None with slot = -1 to unmap."""
        if t is None:
            ptrs = [None] * 6
        else:
            ptrs = [ctypes.c_void_p(_data_ptr(t[n])) for n in ("w1", "s1", "w3", "s3", "w2", "s2")]
        rc = self.lib.moe_fp4_load_expert_slot(self.h, layer, expert, slot, *ptrs, _stream(stream))
        self._check(rc, "load_expert_slot")

    def load_expert_object(self, layer: int, expert: int, slot: int, obj: torch.Tensor, stream=None) -> None:
        """Load from one contiguous expert object (w1, w3, w2 codes, s1, s3, s2 scales)."""
        H, I = self.cfg.hidden, self.cfg.inter
        c13, c2, s13 = I * H // 2, H * I // 2, I * H // 32
        base = obj.data_ptr()
        offs = {"w1": 0, "w3": c13, "w2": 2 * c13, "s1": 2 * c13 + c2, "s3": 2 * c13 + c2 + s13,
                "s2": 2 * c13 + c2 + 2 * s13}
        ptrs = [ctypes.c_void_p(base + offs[n]) for n in ("w1", "s1", "w3", "s3", "w2", "s2")]
        rc = self.lib.moe_fp4_load_expert_slot(self.h, layer, expert, slot, *ptrs, _stream(stream))
        self._check(rc, "load_expert_slot")

    def alloc_routing(self, T: int) -> Routing:
        dev = torch.device("cuda", self.device)
        k, E = self.cfg.top_k, self.cfg.n_experts
        return Routing(torch.empty((T, k), dtype=torch.int32, device=dev),
                       torch.empty((T, k), dtype=torch.float32, device=dev),
                       torch.empty(E, dtype=torch.int32, device=dev),
                       torch.empty(E + 1, dtype=torch.int32, device=dev),
                       torch.empty(T * k, dtype=torch.int32, device=dev))

    def route(self, layer: int, logits: torch.Tensor, keep: torch.Tensor | None = None,
              out: Routing | None = None, stream=None) -> Routing:
        T = logits.shape[0]
        r = out if out is not None else self.alloc_routing(T)
        rc = self.lib.moe_fp4_route(self.h, layer, _ptr(logits), _ptr(keep), T, _ptr(r.ids), _ptr(r.weights),
                                    _ptr(r.counts), _ptr(r.offsets), _ptr(r.perm), _stream(stream))
        self._check(rc, "route")
        return r

    def forward(self, layer: int, x: torch.Tensor, r: Routing, y: torch.Tensor | None = None,
                x_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """x: uint16/bf16 [T, H] bf16 bits.  Returns y fp32 [T, H]."""
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.hidden), dtype=torch.float32, device=x.device)
        rc = self.lib.moe_fp4_forward(self.h, layer, _ptr(x), T, _ptr(r.ids), _ptr(r.weights), _ptr(r.counts),
                                      _ptr(r.offsets), _ptr(r.perm), _ptr(y), _ptr(x_out), _stream(stream))
        self._check(rc, "forward")
        return y

    def route_forward(self, layer: int, logits: torch.Tensor, x: torch.Tensor, keep: torch.Tensor | None = None,
                      out: Routing | None = None, y: torch.Tensor | None = None,
                      x_out: torch.Tensor | None = None, stream=None) -> tuple[Routing, torch.Tensor]:
        """Route + forward in one call (one kernel for decode batches)."""
        T = x.shape[0]
        r = out if out is not None else self.alloc_routing(T)
        if y is None:
            y = torch.empty((T, self.cfg.hidden), dtype=torch.float32, device=x.device)
        rc = self.lib.moe_fp4_route_forward(self.h, layer, _ptr(logits), _ptr(keep), _ptr(x), T, _ptr(r.ids),
                                            _ptr(r.weights), _ptr(r.counts), _ptr(r.offsets), _ptr(r.perm),
                                            _ptr(y), _ptr(x_out), _stream(stream))
        self._check(rc, "route_forward")
        return r, y

    def expert_outputs(self, layer: int, x: torch.Tensor, experts: torch.Tensor, o: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
        """o[i] = expert experts[i] applied to x[i] (fp32 [n, H]); x bf16 bits [n, H]."""
        n = x.shape[0]
        if o is None:
            o = torch.empty((n, self.cfg.hidden), dtype=torch.float32, device=x.device)
        rc = self.lib.moe_fp4_expert_outputs(self.h, layer, _ptr(x), n, _ptr(experts), _ptr(o), _stream(stream))
        self._check(rc, "expert_outputs")
        return o

    def combine(self, o: torch.Tensor, weights: torch.Tensor, x: torch.Tensor | None = None,
                y: torch.Tensor | None = None, x_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """y[t] = sum_j weights[t, j] * o[t*k + j] (+ x_out = bf16(x + y))."""
        T = weights.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.hidden), dtype=torch.float32, device=o.device)
        rc = self.lib.moe_fp4_combine(self.h, T, _ptr(o), _ptr(weights), _ptr(x), _ptr(y), _ptr(x_out),
                                      _stream(stream))
        self._check(rc, "combine")
        return y

    def stream_experts(self, layer: int, experts, objects, stream=None) -> list[int]:
        """Make the listed distinct experts of ``layer`` resident (LRU slots).
        ``objects``: per expert a contiguous checkpoint-layout object (pinned
        host or device uint8 tensor, or numpy array), or None if resident.
        Returns the slot of each expert."""
        n = len(experts)
        ids = (ctypes.c_int32 * n)(*[int(e) for e in experts])
        ptrs = (ctypes.c_void_p * n)(*[(_data_ptr(o) if o is not None else None) for o in objects])
        slots = (ctypes.c_int32 * n)()
        rc = self.lib.moe_fp4_stream_experts(self.h, layer, ids, n, ptrs, slots, _stream(stream))
        self._check(rc, "stream_experts")
        return list(slots)

    def residency_stats(self) -> tuple[int, int, int]:
        """(hits, misses, bytes copied) of stream_experts since create."""
        out = (ctypes.c_int64 * 3)()
        rc = self.lib.moe_fp4_residency_stats(self.h, out)
        self._check(rc, "residency_stats")
        return out[0], out[1], out[2]

    def saliency(self, r: Routing, sal: torch.Tensor, stream=None) -> torch.Tensor:
        """Accumulate per-expert saliency (fp64 [E] device tensor) of the last
        forward on this context: sal[e] += sum of weight * ||expert output||_2
        over the entries routed to e.  Call after forward, same stream."""
        T = r.ids.shape[0]
        rc = self.lib.moe_fp4_saliency(self.h, T, _ptr(r.weights), _ptr(r.offsets), _ptr(r.perm), _ptr(sal),
                                       _stream(stream))
        self._check(rc, "saliency")
        return sal


def _data_ptr(t) -> int:
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return t.ctypes.data   # numpy array (host memory)


def forward_noalloc(cfg: Config, arena_ptr: int, slot_table: torch.Tensor, layer: int, x: torch.Tensor,
                    r: Routing, y: torch.Tensor, x_out: torch.Tensor | None = None,
                    err: torch.Tensor | None = None, stream=None) -> int:
    """moe_fp4_forward_noalloc: the decode forward with library-owned static
    scratch, for callers that may not allocate device memory.  Returns the
    status code (EINVAL when T exceeds the scratch limit)."""
    return load().moe_fp4_forward_noalloc(ctypes.byref(cfg), ctypes.c_void_p(arena_ptr), _ptr(slot_table), layer,
                                          _ptr(x), x.shape[0], _ptr(r.weights), _ptr(r.offsets), _ptr(r.perm),
                                          _ptr(y), _ptr(x_out), _ptr(err), _stream(stream))
