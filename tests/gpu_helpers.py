"""Shared set-up for the GPU tests: contexts filled from the seeded generators,
oracle references for sampled tokens, and the parity bar."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from fp4_routed_expert_router_b200 import moe, synth

# Parity bar for fp32 outputs: per token, max_n |y - y_ref| <= 1e-2 * rms_n(y_ref).
REL_RMS_TOL = 1e-2


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, tol: float = REL_RMS_TOL) -> float:
    """Assert the per-token bar; returns the worst ratio max|dy| / rms(y_ref)."""
    worst = 0.0
    for t in range(y_ref.shape[0]):
        rms = float(np.sqrt(np.mean(y_ref[t] ** 2)))
        err = float(np.max(np.abs(y_gpu[t].astype(np.float64) - y_ref[t])))
        ratio = err / rms if rms > 0 else err
        worst = max(worst, ratio)
        assert ratio <= tol, f"token {t}: max|dy| = {err:.3e}, rms = {rms:.3e}, ratio {ratio:.3e}"
    return worst


class Filled:
    """A context whose arena holds the workload's resident experts."""

    def __init__(self, wl: synth.Workload, max_tokens: int | None = None, layers: int | None = None,
                 from_host: bool = False):
        self.wl = wl
        L = layers if layers is not None else wl.n_layers
        self.L = L
        kept = wl.n_keep if wl.n_keep else wl.n_experts
        self.ctx = moe.Context(wl.hidden, wl.inter, wl.n_experts, wl.top_k, L, kept * L,
                               max_tokens if max_tokens is not None else max(wl.tokens, 8))
        self.slot_of = {}
        staging = torch.empty(wl.expert_bytes, dtype=torch.uint8, device="cuda")
        slot = 0
        for layer in range(L):
            for e in synth.resident_experts(wl, layer):
                e = int(e)
                if from_host:
                    t = synth.gen_expert(wl.seed, layer, e, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
                    self.ctx.load_expert_slot(layer, e, slot, t)
                else:
                    moe.synth_fill_expert(staging, wl.seed, layer, e, wl.hidden, wl.inter, wl.scale_lo,
                                          wl.scale_hi)
                    self.ctx.load_expert_object(layer, e, slot, staging)
                self.slot_of[(layer, e)] = slot
                slot += 1
        torch.cuda.synchronize()
        rc, msg = self.ctx.last_error()
        assert rc == moe.OK, msg
        self._host_cache = {}

    def host_object(self, layer: int, e: int) -> np.ndarray:
        key = (layer, e)
        if key not in self._host_cache:
            wl = self.wl
            t = synth.gen_expert(wl.seed, layer, e, wl.hidden, wl.inter, wl.scale_lo, wl.scale_hi)
            self._host_cache[key] = synth.expert_object(t, wl.hidden, wl.inter)
        return self._host_cache[key]

    def oracle_y(self, layer: int, x: np.ndarray, ids: np.ndarray, w: np.ndarray, tokens) -> np.ndarray:
        """Oracle y for the listed token rows (x, ids, w are full [T, .] arrays)."""
        tokens = list(tokens)
        need = sorted({int(e) for t in tokens for e in ids[t]})
        objs = {e: self.host_object(layer, e) for e in need}
        wl = self.wl
        return oracle.moe_forward(x[tokens], ids[tokens], w[tokens], objs, wl.n_experts, wl.hidden, wl.inter)

    def close(self):
        self.ctx.close()


def to_dev(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if t.dtype == torch.uint16:
        t = t.view(torch.int16)
    return t.cuda()


def routing_to_host(r: moe.Routing):
    return (r.ids.cpu().numpy(), r.weights.cpu().numpy(), r.counts.cpu().numpy(), r.offsets.cpu().numpy(),
            r.perm.cpu().numpy())


def check_routing(r: moe.Routing, logits: np.ndarray, k: int, E: int, keep=None):
    """Routing bit-exact against the oracle; weights to fp32 rounding."""
    ids, w, counts, offsets, perm = routing_to_host(r)
    rid, rw = oracle.route(logits, k, keep)
    rc, ro, rp = oracle.permute(rid, E)
    assert np.array_equal(ids, rid), "router ids differ"
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro), "counts/offsets differ"
    assert np.array_equal(perm, rp), "perm differs"
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=1e-7)
    return rid, rw
