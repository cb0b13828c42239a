"""Shared pieces of the GPU parity tests: device setup of a seeded workload,
calls through the C ABI, and the comparison rules.

Comparison rules (the layer's output contract):
  * top-k indices, permutation, offsets and histograms: bit-exact;
  * gate weights: |w_gpu - w_oracle| <= 1e-4 (oracle in fp64);
  * outputs (bf16): per element |g - r| <= 2e-2 * max(|r|, rms of r's row),
    r the oracle's fp64 value before its final rounding.
"""
from __future__ import annotations

import numpy as np

import moe_synth as S
import oracle as O

OUT_RTOL = 2e-2
W_ATOL = 1e-4
# Per-pair expert outputs w * y of the prefill path are intermediates, not layer
# outputs: the weights, h and the stored value are each rounded once to bf16
# and there is no residual to dominate the row.  A CPU emulation of exactly
# those roundings (tests/test_tolerance_model.py) reaches 2.1e-2 elementwise
# (relative to max(|r|, row rms)) about once in 10^6 elements and 0.5e-2
# normwise; the checks on them use 3e-2 elementwise and 1e-2 normwise.  A
# prefill layer run with the residual off returns the MoE part alone, a
# weighted sum of those intermediates, and is checked the same way; layer
# outputs with the residual keep OUT_RTOL.
PAIR_RTOL = 3e-2
PAIR_NORM_RTOL = 1e-2


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def assert_out_close(got_bits: np.ndarray, ref_f64: np.ndarray, rows=None, tol=OUT_RTOL):
    g = bits_to_f32(got_bits).astype(np.float64)
    r = np.asarray(ref_f64, np.float64)
    if rows is not None:
        g, r = g[rows], r[rows]
    rms = np.sqrt(np.mean(r * r, axis=1, keepdims=True))
    lim = tol * np.maximum(np.abs(r), rms)
    bad = ~(np.abs(g - r) <= lim)  # a NaN on either side counts as out of tolerance
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} / {bad.size} outputs out of tolerance; first at {tuple(i)}: "
                             f"gpu {g[tuple(i)]} oracle {r[tuple(i)]} limit {lim[tuple(i)]}")
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))


class Workload:
    """A seeded layer (or stack) on the device, plus what the oracle needs."""

    def __init__(self, cfg: S.LayerConfig, device_arena: bool | None = None, T: int | None = None):
        import torch
        self.cfg = cfg
        self.T = cfg.T if T is None else T
        self.desc = cfg.desc()
        big = self.desc.slot_bytes * self.desc.n_slots > 2_000_000_000
        self.device_arena = big if device_arena is None else device_arena
        if self.device_arena:
            self.arena = S.gen_arena_device(cfg)
            self.arena_host = None
        else:
            self.arena_host = S.gen_arena_host(cfg)
            self.arena = torch.from_numpy(self.arena_host).cuda()
        self.slot_table_host = S.gen_slot_table(cfg)
        self.slot_table = torch.from_numpy(self.slot_table_host).cuda()
        self.W_host = [S.gen_router(cfg, l) for l in range(cfg.L)]
        self.b_host = [S.gen_bias(cfg, l) for l in range(cfg.L)]
        self.W = [torch.from_numpy(w).cuda() for w in self.W_host]
        self.b = [None if b is None else torch.from_numpy(b).cuda() for b in self.b_host]

    def x_host(self, stream_offset=0):
        return S.gen_x(self.cfg, self.T, stream_offset)

    def slot_bytes_of(self, s: int) -> np.ndarray:
        sb = self.desc.slot_bytes
        if self.arena_host is not None:
            return self.arena_host[s * sb:(s + 1) * sb]
        return self.arena[s * sb:(s + 1) * sb].cpu().numpy()

    def mini_arena(self, layer: int, experts) -> tuple:
        """Host arena holding only the listed experts of `layer`, with a slot
        table that maps them (and -1 elsewhere, which the oracle never reads)."""
        cfg = self.cfg
        experts = sorted(set(int(e) for e in experts))
        sb = self.desc.slot_bytes
        mini = np.zeros(len(experts) * sb, np.uint8)
        table = np.full(cfg.L * cfg.E, -1, np.int32)
        for i, e in enumerate(experts):
            s = int(self.slot_table_host[layer * cfg.E + e])
            mini[i * sb:(i + 1) * sb] = self.slot_bytes_of(s)
            table[layer * cfg.E + e] = i
        d = S.make_desc(cfg.H, cfg.I, cfg.bits, n_slots=max(1, len(experts)))
        return d, mini, table

    def oracle_layer(self, layer: int, x_bits: np.ndarray, tokens=None, residual=True, steer=None):
        """Oracle output for `layer` on x_bits (all tokens or the listed ones)."""
        cfg = self.cfg
        xs = x_bits if tokens is None else x_bits[np.asarray(tokens)]
        lg = O.router_logits(xs, self.W_host[layer], self.b_host[layer])
        idx, _ = O.topk(lg, cfg.top_k)
        d, mini, table = self.mini_arena(layer, np.unique(idx))
        return O.moe_layer(d, mini, table, cfg.L, layer, x_bits, self.W_host[layer], self.b_host[layer],
                           cfg.top_k, residual=residual, tokens=tokens, steer=steer)


def route_buffers(T, k, E):
    import torch
    dev = "cuda"
    return {
        "topk_idx": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "topk_w": torch.zeros(T * k, dtype=torch.float32, device=dev),
        "expert_offsets": torch.zeros(E + 1, dtype=torch.int32, device=dev),
        "perm": torch.full((T * k,), -1, dtype=torch.int32, device=dev),
        "n_rechecked": torch.zeros(1, dtype=torch.int32, device=dev),
    }


def run_layer(wl: Workload, layer: int, x_bits: np.ndarray, prefill: bool, residual=True, hist=None, steer=None):
    """Call the library for one layer; returns (out bits, routing dict of numpy arrays)."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = wl.cfg
    T = x_bits.shape[0]
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    out = torch.zeros_like(x)
    ws = torch.empty(M.moe_workspace_bytes(T, cfg.E, cfg.top_k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    ro = route_buffers(T, cfg.top_k, cfg.E)
    fn = M.moe_forward_prefill if prefill else M.moe_forward_decode
    sv = None if steer is None else torch.from_numpy(np.ascontiguousarray(steer, np.float32)).cuda()
    fn(wl.desc, wl.arena, wl.slot_table, cfg.L, layer, x, wl.W[layer], wl.b[layer], cfg.top_k, residual, out,
       hist=hist, route_out=ro, ws=ws, steer=sv)
    torch.cuda.synchronize()
    st = M.moe_last_device_error()
    assert st == 0, f"device status {st}: {M.strerror(st)}"
    res = {k: v.cpu().numpy() for k, v in ro.items()}
    res["topk_idx"] = res["topk_idx"].reshape(T, cfg.top_k)
    res["topk_w"] = res["topk_w"].reshape(T, cfg.top_k)
    return out.cpu().numpy().view(np.uint16), res


def check_routing(res: dict, idx_ref: np.ndarray, w_ref: np.ndarray, E: int):
    """Bit-exact indices, offsets and permutation; weights within W_ATOL."""
    assert np.array_equal(res["topk_idx"], idx_ref), "top-k indices differ"
    counts, offsets, perm, inv = O.permutation(idx_ref, E)
    assert np.array_equal(res["expert_offsets"], offsets), "expert offsets differ"
    assert np.array_equal(res["perm"], perm), "permutation differs"
    assert np.max(np.abs(res["topk_w"] - w_ref)) <= W_ATOL, "gate weights differ"
    return counts
