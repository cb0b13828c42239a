"""The C ABI without a GPU: every declared symbol is exported, host-side
argument checks return their codes before any CUDA call, and the host-only
entry points agree with the oracle."""
import ctypes
import re

import numpy as np
import pytest

import moe_synth as S
import oracle as O
import quantized_expert_ffn_top10_b200 as M
from quantized_expert_ffn_top10_b200 import build as B

FAKE = 1 << 20  # an aligned address that is never dereferenced: every call below fails a host check first


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.lib()


def test_every_declared_function_is_exported(lib):
    hdr = open(B.sources()[-1]).read()
    names = set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(moe_\w+)\s*\(", hdr, re.M))
    assert names == set(M.EXPORTS)
    so = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(so, n), n


def test_binding_constants_match_the_header():
    """Every integer #define MOE_* of the header has the same value in the
    binding (the ones the binding names)."""
    hdr = open(B.sources()[-1]).read()
    defs = {n: int(v.strip("()").replace(" ", "").split("*")[0]) * (
        int(v.strip("()").replace(" ", "").split("*")[1]) if "*" in v else 1)
        for n, v in re.findall(r"^#define\s+(MOE_\w+)\s+(\(?-?\d+(?:\s*\*\s*\d+)?\)?)", hdr, re.M)}
    assert {"MOE_DECODE_MAX_T", "MOE_ROUTER_F64_MAX_T", "MOE_SLOT_REMOTE", "MOE_ERR_TIMEOUT"} <= set(defs)
    checked = 0
    for n, v in defs.items():
        if hasattr(M, n):
            assert getattr(M, n) == v, n
            checked += 1
    assert checked >= 10


def test_workspace_bytes_grows_with_T(lib):
    a = M.moe_workspace_bytes(5, 512, 10, 2048, 512)
    b = M.moe_workspace_bytes(8192, 512, 10, 2048, 512)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    assert M.moe_workspace_bytes(-1, 512, 10, 2048, 512) == 0


@pytest.mark.parametrize("shape", [(512, 10, 2048, 512), (256, 10, 2048, 512), (16, 4, 256, 128), (8, 2, 64, 32)])
def test_workspace_bytes_never_shrinks_with_T(lib, shape):
    """A workspace sized for T serves every shorter call: the size is
    non-decreasing in T, also across the router regimes' limits (8 and 128
    tokens, where the layout itself shrinks)."""
    E, k, H, I = shape
    Ts = list(range(0, 300)) + [511, 512, 4095, 4096, 8191, 8192]
    sizes = [M.moe_workspace_bytes(T, E, k, H, I) for T in Ts]
    assert all(b >= a for a, b in zip(sizes, sizes[1:]))
    assert all(b % 256 == 0 for b in sizes)


def _fwd(fn, desc, T=5, E=512, k=10, L=1, layer=0, x=FAKE, out=FAKE + (1 << 16), ws=FAKE * 64,
         ws_bytes=None, arena=FAKE * 128, W=FAKE * 4, steer=None):
    d = M.as_desc(desc) if desc is not None else None
    if ws_bytes is None:
        ws_bytes = 1 << 40
    return fn(ctypes.byref(d) if d is not None else None, arena, FAKE * 8, L, layer, x, T, W, None, E, k, 1, steer,
              out, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("which", ["decode", "prefill"])
def test_host_checks(lib, which):
    fn = lib.moe_forward_decode if which == "decode" else lib.moe_forward_prefill
    d = S.make_desc(2048, 512, (4, 4, 4), n_slots=512)
    assert _fwd(fn, None) == M.MOE_ERR_ARG
    bad = S.make_desc(2048, 512, (3, 4, 4))
    assert _fwd(fn, bad) == M.MOE_ERR_SHAPE
    bad = S.make_desc(2048, 512, (4, 4, 4)); bad.block = 16
    assert _fwd(fn, bad) == M.MOE_ERR_SHAPE
    bad = S.make_desc(2048, 512, (4, 4, 4)); bad.off_scales[2] = bad.slot_bytes
    assert _fwd(fn, bad) == M.MOE_ERR_SHAPE
    bad = S.make_desc(2048, 512, (4, 4, 4)); bad.slot_bytes += 128
    assert _fwd(fn, bad) == M.MOE_ERR_SHAPE
    maxT = 8 if which == "decode" else 8192
    assert _fwd(fn, d, T=maxT + 1) == M.MOE_ERR_RANGE
    assert _fwd(fn, d, T=-1) == M.MOE_ERR_RANGE
    assert _fwd(fn, d, E=513) == M.MOE_ERR_RANGE
    assert _fwd(fn, d, k=33, E=512) == M.MOE_ERR_RANGE
    assert _fwd(fn, d, k=9, E=8) == M.MOE_ERR_RANGE
    assert _fwd(fn, d, layer=1, L=1) == M.MOE_ERR_RANGE
    assert _fwd(fn, d, x=FAKE + 2) == M.MOE_ERR_ARG          # misaligned
    assert _fwd(fn, d, x=0) == M.MOE_ERR_ARG
    assert _fwd(fn, d, arena=FAKE * 128 + 16) == M.MOE_ERR_ARG
    assert _fwd(fn, d, out=FAKE + 64) == M.MOE_ERR_ARG       # overlaps x
    assert _fwd(fn, d, ws_bytes=1024) == M.MOE_ERR_WS
    assert _fwd(fn, d, steer=FAKE * 2 + 4) == M.MOE_ERR_ARG  # steering vector not 16-byte aligned


def test_prefill_needs_tile_multiples(lib):
    d = S.make_desc(64, 32, (4, 4, 4), n_slots=8)
    assert _fwd(lib.moe_forward_prefill, d, E=8, k=2) == M.MOE_ERR_SHAPE
    # the decode path takes the same small shape (it stops at the workspace check here)
    assert _fwd(lib.moe_forward_decode, d, E=8, k=2, ws_bytes=16) == M.MOE_ERR_WS


def test_route_and_histogram_checks(lib):
    assert lib.moe_route(FAKE, 9000, 2048, FAKE, None, 512, 10, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) \
        == M.MOE_ERR_RANGE
    assert lib.moe_route(FAKE, 5, 2048, FAKE, None, 512, 10, None, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) \
        == M.MOE_ERR_ARG
    assert lib.moe_route(FAKE, 5, 2048, FAKE, None, 512, 10, FAKE, FAKE, FAKE, FAKE, FAKE, 100, None) \
        == M.MOE_ERR_WS
    assert lib.moe_route(FAKE, 0, 2048, FAKE, None, 512, 10, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) \
        == M.MOE_OK
    assert lib.moe_route_histogram(None, 512, 1, 0, FAKE, None) == M.MOE_ERR_ARG
    assert lib.moe_route_histogram(FAKE, 512, 1, 1, FAKE, None) == M.MOE_ERR_RANGE


def test_t_zero_is_a_noop(lib):
    d = S.make_desc(2048, 512, (4, 4, 4), n_slots=512)
    assert _fwd(lib.moe_forward_decode, d, T=0) == M.MOE_OK
    assert _fwd(lib.moe_forward_prefill, d, T=0) == M.MOE_OK


def test_rank_experts_matches_oracle(lib):
    rng = np.random.default_rng(0)
    for L, E in [(1, 8), (48, 256), (48, 512), (3, 5)]:
        hist = rng.integers(0, 20, (L, E)).astype(np.uint32)
        assert np.array_equal(M.moe_rank_experts(hist), O.rank(hist))


def test_strerror_covers_codes(lib):
    msgs = {M.strerror(c) for c in range(-7, 1)}
    assert len(msgs) == 8 and "unknown" in M.strerror(-99)


def test_route_static_checks(lib):
    # beyond the fixed scratch: rejected before any CUDA call, with its own code
    assert lib.moe_route_static(FAKE, M.MOE_ROUTE_STATIC_MAX_T + 1, 2048, FAKE, None, 512, 10, FAKE, FAKE, FAKE,
                                FAKE, None) == M.MOE_ERR_STATIC
    assert "MOE_ROUTE_STATIC_MAX_T" in M.strerror(M.MOE_ERR_STATIC)
    assert lib.moe_route_static(FAKE, 5, 2048, FAKE, None, 513, 10, FAKE, FAKE, FAKE, FAKE, None) == M.MOE_ERR_RANGE
    assert lib.moe_route_static(FAKE, 5, 2048, FAKE, None, 512, 10, None, FAKE, FAKE, FAKE, None) == M.MOE_ERR_ARG
    assert lib.moe_route_static(FAKE + 2, 5, 2048, FAKE, None, 512, 10, FAKE, FAKE, FAKE, FAKE, None) \
        == M.MOE_ERR_ARG
    assert lib.moe_route_static(FAKE, 0, 2048, FAKE, None, 512, 10, FAKE, FAKE, FAKE, FAKE, None) == M.MOE_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without libmoe.so the binding raises; there is no CPU fallback."""
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "LIB_PATH", str(tmp_path / "libmoe.so"))
    with pytest.raises(ImportError):
        M.moe_workspace_bytes(5, 512, 10, 2048, 512)


@pytest.mark.parametrize("T", [1, 5, 8, 9, 64, 128, 129, 300, 8192])
def test_workspace_fields_are_aligned_and_inside(lib, T):
    """The workspace fields the tests read sit on 256-byte boundaries inside
    the workspace, and the fast logits' region holds T x E values of the
    router's dtype (fp64 up to MOE_ROUTER_F64_MAX_T tokens, fp32 above)."""
    E, k, H, I = 512, 10, 2048, 512
    total = M.moe_workspace_bytes(T, E, k, H, I)
    offs = {f: M.moe_workspace_offset(T, E, k, H, I, f)
            for f in (M.MOE_WS_FAST_LOGITS, M.MOE_WS_PAIR_OUT, M.MOE_WS_SLOW_COUNT)}
    for f, o in offs.items():
        assert o % 256 == 0 and o < total, (f, o, total)
    nb = T * E * (8 if T <= M.MOE_ROUTER_F64_MAX_T else 4)
    later = [o for o in offs.values() if o > offs[M.MOE_WS_FAST_LOGITS]]
    assert offs[M.MOE_WS_FAST_LOGITS] + nb <= min(later + [total])
    with pytest.raises(M.MoeError):
        M.moe_workspace_offset(T, E, k, H, I, 99)  # unknown field
