"""CPU oracle for the quantized top-k MoE layer (ctypes wrapper over moe_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The library path never
imports this package and the two share no code.

Functions mirror the C file one for one; see its header for what each step
computes and which passage of the source pages it follows.  Parity of the
fp64 output values themselves is pinned only through closed forms, special
cases and invariants (tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

ORC_OK, ORC_ERR_ARG, ORC_ERR_SLOT = 0, -1, -6


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (plain -O2, no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call([
            "gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
            "-shared", "-o", _LIB, _SRC, "-lm",
        ])
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_half_to_double.restype = ctypes.c_double
        L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_code.restype = ctypes.c_int
        L.oracle_code.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.oracle_dequant.restype = ctypes.c_double
        L.oracle_dequant.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.oracle_silu.restype = ctypes.c_double
        L.oracle_silu.argtypes = [ctypes.c_double]
        L.oracle_expert_ffn.restype = None
        L.oracle_expert_ffn.argtypes = [P, P, P, P, P]
        L.oracle_router_logits.restype = None
        L.oracle_router_logits.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, P]
        L.oracle_topk.restype = None
        L.oracle_topk.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_permutation.restype = None
        L.oracle_permutation.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.oracle_hist_add.restype = None
        L.oracle_hist_add.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_rank.restype = None
        L.oracle_rank.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_moe_layer.restype = ctypes.c_int
        L.oracle_moe_layer.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, P,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P,
                                       ctypes.c_int]
        L.oracle_steer.restype = None
        L.oracle_steer.argtypes = [P, P, ctypes.c_int]
        L.oracle_set_threads.restype = None
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_max_threads.restype = ctypes.c_int
        L.oracle_max_threads.argtypes = []
        del i32, i64
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return None if a is None else np.ascontiguousarray(a, dtype=dt)


# --------------------------------------------------------------- scalars

def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits) & 0xFFFF)


def half_to_double(bits: int) -> float:
    return lib().oracle_half_to_double(int(bits) & 0xFFFF)


def double_to_bf16(v: float) -> int:
    return int(lib().oracle_double_to_bf16(float(v)))


def silu(g: float) -> float:
    return lib().oracle_silu(float(g))


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    f = np.vectorize(bf16_to_double, otypes=[np.float64])
    return f(np.asarray(a, dtype=np.uint16))


# --------------------------------------------------------------- arena

def code(slot: np.ndarray, desc, m: int, row: int, c: int) -> int:
    slot = _c(slot, np.uint8)
    return lib().oracle_code(_p(slot), ctypes.byref(desc), m, row, c)


def dequant(slot: np.ndarray, desc, m: int, row: int, c: int) -> float:
    slot = _c(slot, np.uint8)
    return lib().oracle_dequant(_p(slot), ctypes.byref(desc), m, row, c)


def expert_ffn(slot: np.ndarray, desc, x: np.ndarray):
    """(y [H], h [I]) of one expert for one fp64 token vector."""
    slot = _c(slot, np.uint8)
    x = _c(x, np.float64)
    y = np.zeros(desc.H, np.float64)
    h = np.zeros(desc.I, np.float64)
    lib().oracle_expert_ffn(_p(slot), ctypes.byref(desc), _p(x), _p(y), _p(h))
    return y, h


def dequant_matrix(slot: np.ndarray, desc, m: int) -> np.ndarray:
    """Matrix m (0 gate [I, H], 1 up [I, H], 2 down [H, I]) of one slot, fp64:
    W[r, c] = scale[r, c // 32] * (code[r, c] - 2^(bits - 1)), codes packed
    LSB first along each row.  The same definition as oracle_dequant (the
    block-32 reading of the "Strata Coder deep-dive" page, sections 2-3),
    unpacked for a whole matrix at once."""
    slot = np.asarray(slot, np.uint8)
    rows, K = (desc.I, desc.H) if m < 2 else (desc.H, desc.I)
    b = (desc.bits_gate, desc.bits_up, desc.bits_down)[m]
    o = desc.off_codes[m]
    raw = slot[o:o + rows * K * b // 8].astype(np.int64)
    per = 8 // b
    codes = np.empty((raw.size, per), np.int64)
    for i in range(per):                       # element i of a byte sits at bits i*b .. i*b + b - 1
        codes[:, i] = (raw >> (i * b)) & ((1 << b) - 1)
    codes = codes.reshape(rows, K)
    so = desc.off_scales[m]
    sc = slot[so:so + rows * (K // 32) * 2].view("<f2").astype(np.float64).reshape(rows, K // 32)
    return np.repeat(sc, 32, axis=1) * (codes - (1 << (b - 1))).astype(np.float64)


def expert_ffn_rows(slot: np.ndarray, desc, X: np.ndarray):
    """(y [n, H], h [n, I]) of one expert for n fp64 token rows X [n, H]:
    g = W_g x, u = W_u x, h = silu(g) u, y = W_d h - the definition of
    oracle_expert_ffn (SwiGLU reading of the gate/up/down projections of the
    "Strata Coder deep-dive" page, section 3), with each matrix dequantised
    once and the sums taken by numpy's fp64 matrix product, so that thousands
    of rows of one expert take seconds."""
    X = np.asarray(X, np.float64)
    Wg, Wu, Wd = (dequant_matrix(slot, desc, m) for m in range(3))
    g = X @ Wg.T
    u = X @ Wu.T
    h = g / (1.0 + np.exp(-g)) * u
    return h @ Wd.T, h


# --------------------------------------------------------------- routing

def router_logits(x_bits: np.ndarray, W: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    x_bits = _c(x_bits, np.uint16)
    W = _c(W, np.float32)
    b = _c(b, np.float32)
    T, H = x_bits.shape
    E = W.shape[0]
    out = np.zeros((T, E), np.float64)
    lib().oracle_router_logits(_p(x_bits), T, H, _p(W), _p(b), E, _p(out))
    return out


def topk(logits: np.ndarray, k: int):
    logits = _c(logits, np.float64)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    lib().oracle_topk(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def permutation(idx: np.ndarray, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    inv = np.zeros(T * k, np.int32)
    lib().oracle_permutation(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm, inv


def hist_add(counts: np.ndarray, layer: int, hist: np.ndarray) -> None:
    """hist (uint32 [L, E], updated in place) += counts on `layer`."""
    counts = _c(counts, np.int32)
    assert hist.dtype == np.uint32 and hist.flags.c_contiguous
    lib().oracle_hist_add(_p(counts), counts.shape[0], layer, _p(hist))


def rank(hist: np.ndarray) -> np.ndarray:
    """uint16 [L*E, 2] (layer, expert) pairs, most routed first."""
    hist = _c(hist, np.uint32)
    L, E = hist.shape
    pairs = np.zeros((L * E, 2), np.uint16)
    lib().oracle_rank(_p(hist), L, E, _p(pairs))
    return pairs


# --------------------------------------------------------------- layer

def steer(h: np.ndarray, v: np.ndarray) -> np.ndarray:
    """h - (h . v) v for one row (fp64), the C oracle_steer."""
    h = _c(h, np.float64).copy()
    v = _c(v, np.float32)
    lib().oracle_steer(_p(h), _p(v), h.shape[0])
    return h


def moe_layer(desc, arena: np.ndarray, slot_table: np.ndarray, L: int, layer: int,
              x_bits: np.ndarray, W: np.ndarray, b: np.ndarray | None, k: int,
              residual: bool = True, tokens: np.ndarray | None = None, steer: np.ndarray | None = None):
    """Run the layer for all tokens (or the listed ones); `steer` [H] fp32
    removes that direction from every output row before its rounding.

    Returns dict(out=bf16 bits [T,H], out_f64=[T,H], idx=[T,k], w=[T,k], rc=int);
    rows of unlisted tokens are left zero."""
    arena = _c(arena, np.uint8)
    slot_table = _c(slot_table, np.int32)
    x_bits = _c(x_bits, np.uint16)
    W = _c(W, np.float32)
    b = _c(b, np.float32)
    T, H = x_bits.shape
    E = W.shape[0]
    out = np.zeros((T, H), np.uint16)
    out64 = np.zeros((T, H), np.float64)
    idx = np.full((T, k), -1, np.int32)
    w = np.zeros((T, k), np.float64)
    tok = _c(tokens, np.int32)
    nt = 0 if tok is None else tok.shape[0]
    sv = _c(steer, np.float32)
    rc = lib().oracle_moe_layer(ctypes.byref(desc), _p(arena), _p(slot_table), L, layer,
                                _p(x_bits), T, _p(W), _p(b), E, k, int(bool(residual)), _p(sv),
                                _p(out), _p(out64), _p(idx), _p(w), _p(tok), nt)
    return {"out": out, "out_f64": out64, "idx": idx, "w": w, "rc": rc}


# --------------------------------------------------------------- timing control

def set_threads(n: int) -> None:
    """Threads of the oracle's parallel loops (results do not depend on it)."""
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())
