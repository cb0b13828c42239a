"""Seeded synthetic inputs for the quantized top-10 MoE layer.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It draws random numbers and lays bytes out in the expert-arena format; it holds
none of the layer's arithmetic (no dequantisation, routing, softmax or FFN).

Workload shapes follow the engine described on the source pages ("Strata Coder
deep-dive" page, section 1: 48 layers x 512 experts, 10 routed per token;
section 2: the pruned 256-expert variant; "Coder benchmark record" page,
test-environment section: prefill chunks of up to 8,192 tokens and a 4-draft
speculative verify window).  Model dimensions H = 2048 and I = 512 are the
stated workload; the pages do not give them.

Arena format (the pages name only ggml quant types; this block-32 format is the
stated stand-in):

* each expert has three matrices: gate W_g [I, H], up W_u [I, H], down W_d [H, I],
  stored row-major by output row, quant blocks of 32 along the reduction axis;
* codes: row r of a b-bit matrix with reduction length K occupies K*b/8 bytes;
  element c sits at byte c*b//8 of that row, bit offset (c*b) % 8, least
  significant bits first;
* scales: fp16 array [rows, K/32] per matrix;
* a slot holds gate codes | up codes | down codes | gate scales | up scales |
  down scales, each section starting on a 128-byte boundary, and the slot
  stride is rounded up to 256 bytes;
* expert (layer, e) lives in slot ``slot_table[layer * E + e]``.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass, field

import numpy as np

GATE, UP, DOWN = 0, 1, 2
BLOCK = 32


def _align(v: int, a: int) -> int:
    return (v + a - 1) // a * a


class ArenaDesc(ctypes.Structure):
    """Mirror of the C struct ``moe_arena_desc`` (include/moe.h)."""

    _fields_ = [
        ("H", ctypes.c_int32),
        ("I", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("bits_gate", ctypes.c_int32),
        ("bits_up", ctypes.c_int32),
        ("bits_down", ctypes.c_int32),
        ("slot_bytes", ctypes.c_int64),
        ("off_codes", ctypes.c_int64 * 3),
        ("off_scales", ctypes.c_int64 * 3),
        ("n_slots", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]

    def bits(self, m: int) -> int:
        return (self.bits_gate, self.bits_up, self.bits_down)[m]

    def as_dict(self) -> dict:
        return {
            "H": self.H, "I": self.I, "block": self.block,
            "bits": [self.bits_gate, self.bits_up, self.bits_down],
            "slot_bytes": self.slot_bytes,
            "off_codes": list(self.off_codes), "off_scales": list(self.off_scales),
            "n_slots": self.n_slots,
        }


def matrix_shape(H: int, I: int, m: int) -> tuple[int, int]:
    """(rows, K) of matrix m: gate/up are [I, H], down is [H, I]."""
    return (I, H) if m in (GATE, UP) else (H, I)


def make_desc(H: int, I: int, bits=(4, 4, 4), n_slots: int = 1) -> ArenaDesc:
    """Lay out one expert slot in the arena format described in the module doc."""
    d = ArenaDesc()
    d.H, d.I, d.block = H, I, BLOCK
    d.bits_gate, d.bits_up, d.bits_down = bits
    off = 0
    for m in range(3):
        rows, K = matrix_shape(H, I, m)
        d.off_codes[m] = off
        off = _align(off + rows * K * bits[m] // 8, 128)
    for m in range(3):
        rows, K = matrix_shape(H, I, m)
        d.off_scales[m] = off
        off = _align(off + rows * (K // BLOCK) * 2, 128)
    d.slot_bytes = _align(off, 256)
    d.n_slots = n_slots
    d.reserved = 0
    return d


# ----------------------------------------------------------------------------
# workload recipes
# ----------------------------------------------------------------------------

@dataclass
class LayerConfig:
    """One synthetic workload.  ``zipf_s`` > 0 adds a per-expert router bias
    b_e = -s * ln(rank_e) with a seeded rank permutation per layer."""

    name: str
    L: int
    E: int
    top_k: int
    H: int
    I: int
    T: int
    bits: tuple = (4, 4, 4)
    router_std: float | None = None       # None -> 1/sqrt(H) (logits ~ N(0,1))
    zipf_s: float = 0.0
    residual: bool = True
    seed: int = 0
    scale_lo: float = 0.001
    scale_hi: float = 0.01
    extra: dict = field(default_factory=dict)

    @property
    def std(self) -> float:
        return self.router_std if self.router_std is not None else 1.0 / math.sqrt(self.H)

    def desc(self) -> ArenaDesc:
        return make_desc(self.H, self.I, self.bits, n_slots=self.L * self.E)


# Expert scales of the two 48-layer stacks.  The layer is x + MoE(x) with no
# normalisation, and a SwiGLU expert grows with |x|^2, so a chain of random
# layers diverges unless the MoE part stays small: with the tiny workload's
# U(0.001, 0.01) a token's residual stream overflows within about 10 layers.
# U(0.0002, 0.002) keeps every token bounded over 48 layers.
STACK_SCALE = (0.0002, 0.002)


def config(name: str, **over) -> LayerConfig:
    """The named workloads.

    tiny        : L=1, E=8, k=2, H=64, I=32, T=4, router std 0.02, seed 0
    decode      : L=1, E=512, k=10, H=2048, I=512, T=5 (T=1 via override), seed 1
    decode_stack: L=48, E=256, k=10, T=5, gate/up 2-bit, down 4-bit, Zipf 1.1, seed 2,
                  scales STACK_SCALE
    prefill     : L=1, E=512, k=10, T=8192, 4-bit, no bias, seed 3
    prefill_stack: L=48, E=512, k=10, T=8192, 2/2/4-bit, Zipf 1.1, seed 4, scales STACK_SCALE
    """
    base = {
        "tiny": LayerConfig("tiny", 1, 8, 2, 64, 32, 4, router_std=0.02, seed=0),
        "decode": LayerConfig("decode", 1, 512, 10, 2048, 512, 5, seed=1),
        "decode_stack": LayerConfig("decode_stack", 48, 256, 10, 2048, 512, 5,
                                    bits=(2, 2, 4), zipf_s=1.1, seed=2, scale_lo=STACK_SCALE[0],
                                    scale_hi=STACK_SCALE[1]),
        "prefill": LayerConfig("prefill", 1, 512, 10, 2048, 512, 8192, seed=3),
        "prefill_stack": LayerConfig("prefill_stack", 48, 512, 10, 2048, 512, 8192,
                                     bits=(2, 2, 4), zipf_s=1.1, seed=4, scale_lo=STACK_SCALE[0],
                                     scale_hi=STACK_SCALE[1]),
    }[name]
    for k, v in over.items():
        setattr(base, k, v)
    return base


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, stream]))


STREAM_X, STREAM_ROUTER, STREAM_BIAS, STREAM_ARENA, STREAM_SLOTS = 1, 2, 3, 4, 5


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even) and return the raw bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def gen_x(cfg: LayerConfig, T: int | None = None, stream_offset: int = 0) -> np.ndarray:
    """Hidden states [T, H] ~ N(0, 1), stored as bf16 bits (uint16)."""
    T = cfg.T if T is None else T
    r = _rng(cfg.seed, STREAM_X + 100 * stream_offset)
    return f32_to_bf16_bits(r.standard_normal((T, cfg.H), dtype=np.float32))


def gen_router(cfg: LayerConfig, layer: int = 0) -> np.ndarray:
    """Router weight [E, H] float32 ~ N(0, std^2)."""
    r = _rng(cfg.seed, STREAM_ROUTER * 1000 + layer)
    return (r.standard_normal((cfg.E, cfg.H), dtype=np.float32) * np.float32(cfg.std)).astype(np.float32)


def gen_bias(cfg: LayerConfig, layer: int = 0) -> np.ndarray | None:
    """Zipf logit bias [E] float32, or None when the workload has none."""
    if cfg.zipf_s <= 0:
        return None
    r = _rng(cfg.seed, STREAM_BIAS * 1000 + layer)
    rank = r.permutation(cfg.E) + 1
    return (-cfg.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32)


def gen_slot_table(cfg: LayerConfig) -> np.ndarray:
    """(layer, expert) -> slot, a seeded permutation of range(L*E) (int32)."""
    r = _rng(cfg.seed, STREAM_SLOTS)
    return r.permutation(cfg.L * cfg.E).astype(np.int32)


def _fill_slot(buf: np.ndarray, desc: ArenaDesc, rng: np.random.Generator,
               lo: float, hi: float) -> None:
    """Random code bytes (uniform codes) and fp16 scales ~ U(lo, hi) in one slot."""
    H, I = desc.H, desc.I
    for m in range(3):
        rows, K = matrix_shape(H, I, m)
        nb = rows * K * desc.bits(m) // 8
        o = desc.off_codes[m]
        buf[o:o + nb] = rng.integers(0, 256, nb, dtype=np.uint8)
    for m in range(3):
        rows, K = matrix_shape(H, I, m)
        ns = rows * (K // BLOCK)
        s = rng.uniform(lo, hi, ns).astype(np.float16)
        o = desc.off_scales[m]
        buf[o:o + 2 * ns] = s.view(np.uint8)


def gen_arena_host(cfg: LayerConfig, n_slots: int | None = None) -> np.ndarray:
    """Whole arena on the host as uint8 [n_slots * slot_bytes]; slot s is
    filled from its own seeded stream so any slot can be regenerated alone."""
    desc = cfg.desc()
    n = desc.n_slots if n_slots is None else n_slots
    out = np.zeros(n * desc.slot_bytes, dtype=np.uint8)
    for s in range(n):
        slot = out[s * desc.slot_bytes:(s + 1) * desc.slot_bytes]
        _fill_slot(slot, desc, _rng(cfg.seed, STREAM_ARENA * 1_000_000 + s),
                   cfg.scale_lo, cfg.scale_hi)
    return out


def gen_slot_host(cfg: LayerConfig, s: int) -> np.ndarray:
    """Slot s alone, byte-identical to slot s of gen_arena_host."""
    desc = cfg.desc()
    out = np.zeros(desc.slot_bytes, dtype=np.uint8)
    _fill_slot(out, desc, _rng(cfg.seed, STREAM_ARENA * 1_000_000 + s), cfg.scale_lo, cfg.scale_hi)
    return out


def gen_arena_device(cfg: LayerConfig, device="cuda", n_slots: int | None = None):
    """Large arenas generated on the device with torch's seeded generator.

    Returns a uint8 tensor [n_slots * slot_bytes].  Codes are uniform bytes;
    each scale section holds fp16 ~ U(lo, hi).  Callers that need slot s on the
    host copy it back (``arena[s*sb:(s+1)*sb].cpu()``).
    """
    import torch
    desc = cfg.desc()
    n = desc.n_slots if n_slots is None else n_slots
    sb = desc.slot_bytes
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 7919 + STREAM_ARENA)
    arena = torch.randint(0, 256, (n, sb), dtype=torch.uint8, device=device, generator=g)
    H, I = desc.H, desc.I
    for m in range(3):
        rows, K = matrix_shape(H, I, m)
        ns = rows * (K // BLOCK)
        o = desc.off_scales[m]
        sc = torch.empty((n, ns), dtype=torch.float32, device=device)
        sc.uniform_(cfg.scale_lo, cfg.scale_hi, generator=g)
        arena[:, o:o + 2 * ns] = sc.to(torch.float16).view(torch.uint8)
        # bytes between sections stay random: nothing may read them
    return arena.view(-1)
