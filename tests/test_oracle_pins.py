"""Pins for the CPU oracle, each against something other than the oracle itself:
closed forms, library routines on special cases, hand-built blocks, brute
force and invariants.  CPU only."""
import json
import math
import os

import numpy as np
import pytest

import moe_synth as S
import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ numbers

def test_bf16_decode_matches_torch():
    import torch
    bits = np.arange(0, 65536, 97, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([O.bf16_to_double(b) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])


def test_bf16_round_nearest_even_hand_cases():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even pattern 0x3F80
    assert O.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 lies halfway between 0x3F81 and 0x3F82: even is 0x3F82
    assert O.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # a hair above the midpoint rounds up
    assert O.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert O.double_to_bf16(-2.0) == 0xC000
    assert O.double_to_bf16(0.0) == 0x0000
    assert O.double_to_bf16(2.0 ** -130) == 0x0008          # bf16 subnormal, exact
    assert O.double_to_bf16(1e39) == 0x7F80                   # overflow to +inf


def test_bf16_round_matches_torch_on_float32_values():
    import torch
    r = np.random.default_rng(5)
    v = (r.standard_normal(20000) * np.exp(r.uniform(-20, 20, 20000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.double_to_bf16(float(a)) for a in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_half_decode_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([O.half_to_double(b) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.all(np.isinf(got[np.isinf(ref)]))


def test_silu_closed_form():
    assert O.silu(0.0) == 0.0
    assert O.silu(1.0) == pytest.approx(1.0 / (1.0 + math.e ** -1), rel=1e-15)
    assert O.silu(-1.0) == pytest.approx(-1.0 / (1.0 + math.e), rel=1e-15)
    assert O.silu(60.0) == pytest.approx(60.0, rel=1e-20 + 1e-15)


# ------------------------------------------------------------------ arena

def _blank_slot(H=64, I=32, bits=(4, 4, 4), code_byte=None):
    d = S.make_desc(H, I, bits)
    slot = np.zeros(d.slot_bytes, np.uint8)
    for m in range(3):
        rows, K = S.matrix_shape(H, I, m)
        nb = rows * K * bits[m] // 8
        if code_byte is not None:
            slot[d.off_codes[m]:d.off_codes[m] + nb] = code_byte[m] if isinstance(code_byte, tuple) else code_byte
    return d, slot


def _set_scales(d, slot, m, values):
    rows, K = S.matrix_shape(d.H, d.I, m)
    v = np.broadcast_to(np.asarray(values, np.float16), (rows, K // 32)).astype(np.float16)
    o = d.off_scales[m]
    slot[o:o + v.nbytes] = v.reshape(-1).view(np.uint8)


def test_desc_layout_sizes_match_stated_expert_bytes():
    assert S.make_desc(2048, 512, (4, 4, 4)).slot_bytes == 1_769_472
    assert S.make_desc(2048, 512, (2, 2, 4)).slot_bytes == 1_245_184
    d = S.make_desc(64, 32, (4, 4, 4))
    offs = sorted(list(d.off_codes) + list(d.off_scales))
    assert all(o % 128 == 0 for o in offs) and d.slot_bytes % 256 == 0


def test_code_packing_lsb_first_4bit_and_2bit():
    d, slot = _blank_slot(bits=(4, 2, 4))
    o = d.off_codes[0]
    slot[o:o + 2] = [0x21, 0x43]                     # gate row 0: codes 1, 2, 3, 4
    assert [O.code(slot, d, 0, 0, c) for c in range(4)] == [1, 2, 3, 4]
    row_bytes = d.H // 2
    slot[o + row_bytes] = 0xF0                        # gate row 1: codes 0, 15
    assert [O.code(slot, d, 0, 1, c) for c in range(2)] == [0, 15]
    o = d.off_codes[1]
    slot[o] = 0xE4                                    # 2-bit up row 0: 0b11_10_01_00
    assert [O.code(slot, d, 1, 0, c) for c in range(4)] == [0, 1, 2, 3]
    slot[o + d.H // 4] = 0x1B                         # up row 1: 0b00_01_10_11
    assert [O.code(slot, d, 1, 1, c) for c in range(4)] == [3, 2, 1, 0]


def test_dequant_closed_forms():
    d, slot = _blank_slot(bits=(4, 2, 4), code_byte=(0x88, 0xAA, 0x88))
    for m in range(3):
        _set_scales(d, slot, m, 0.5)
    # all codes at the offset (8 for 4-bit, 2 for 2-bit) dequantise to zero
    assert O.dequant(slot, d, 0, 3, 17) == 0.0
    assert O.dequant(slot, d, 1, 5, 40) == 0.0
    o = d.off_codes[0]
    slot[o] = 0x0F                                    # gate row 0: c0 = 15, c1 = 0
    assert O.dequant(slot, d, 0, 0, 0) == 3.5         # 0.5 * (15 - 8)
    assert O.dequant(slot, d, 0, 0, 1) == -4.0        # 0.5 * (0 - 8)
    o = d.off_codes[1]
    slot[o] = 0b00000011                              # up row 0: c0 = 3, c1 = 0
    assert O.dequant(slot, d, 1, 0, 0) == 0.5         # 0.5 * (3 - 2)
    assert O.dequant(slot, d, 1, 0, 1) == -1.0        # 0.5 * (0 - 2)
    # the scale is per (row, block of 32): block 1 of gate row 0 gets 0.25
    rows, K = S.matrix_shape(d.H, d.I, 0)
    sc = np.full((rows, K // 32), 0.5, np.float16)
    sc[0, 1] = 0.25
    slot[d.off_scales[0]:d.off_scales[0] + sc.nbytes] = sc.view(np.uint8).reshape(-1)
    slot[d.off_codes[0] + 16] = 0x0F                  # gate row 0, element 32 = 15
    assert O.dequant(slot, d, 0, 0, 32) == 1.75       # 0.25 * 7
    assert O.dequant(slot, d, 0, 0, 31) == 0.0


# ------------------------------------------------------------------ expert FFN

def test_zero_scale_expert_gives_zero():
    cfg = S.config("tiny")
    slot = S.gen_slot_host(cfg, 0)
    d = cfg.desc()
    for m in range(3):
        _set_scales(d, slot, m, 0.0)
    x = np.random.default_rng(1).standard_normal(d.H)
    y, h = O.expert_ffn(slot, d, x)
    assert np.all(y == 0.0) and np.all(h == 0.0)


def test_ffn_one_hot_input_selects_gate_up_column_and_down_row():
    """x = e_j picks column j of W_g and W_u; a W_d with a single nonzero entry
    (c0, r0) makes y = W_d[c0, r0] * h[r0] at c0 and 0 elsewhere."""
    d, slot = _blank_slot(code_byte=0x88)
    H, I = d.H, d.I
    rng = np.random.default_rng(2)
    for m in range(3):
        rows, K = S.matrix_shape(H, I, m)
        sc = rng.uniform(0.1, 1.0, (rows, K // 32)).astype(np.float16)
        slot[d.off_scales[m]:d.off_scales[m] + sc.nbytes] = sc.view(np.uint8).reshape(-1)
    # gate/up: random codes so every (row, column) differs
    for m in (0, 1):
        rows, K = S.matrix_shape(H, I, m)
        slot[d.off_codes[m]:d.off_codes[m] + rows * K // 2] = rng.integers(0, 256, rows * K // 2)
    j = 45
    x = np.zeros(H)
    x[j] = 1.0
    # down: only element (c0, r0) nonzero: code 15 -> (15 - 8) * scale
    c0, r0 = 37, 19
    byte = d.off_codes[2] + c0 * (I // 2) + r0 // 2
    slot[byte] = (0x8 | (15 << 4)) if r0 % 2 else (0x80 | 15)
    y, h = O.expert_ffn(slot, d, x)
    for r in range(I):
        g = O.dequant(slot, d, 0, r, j)
        u = O.dequant(slot, d, 1, r, j)
        assert h[r] == pytest.approx(g / (1 + math.exp(-g)) * u, rel=1e-14, abs=1e-300)
    sc_d = np.frombuffer(slot[d.off_scales[2]:d.off_scales[2] + H * (I // 32) * 2].tobytes(),
                         np.float16).reshape(H, I // 32)
    expect = float(sc_d[c0, r0 // 32]) * 7.0 * h[r0]
    assert y[c0] == pytest.approx(expect, rel=1e-14)
    assert np.count_nonzero(y) == (1 if expect != 0 else 0)


def test_ffn_rank_one_closed_form():
    """Constant codes with per-row scales: W_g[r, c] = a_r, W_u[r, c] = b_r,
    W_d[c, r] = s_c.  Then g_r = a_r S, u_r = b_r S with S = sum(x), and
    y_c = s_c * sum_r silu(a_r S) b_r S."""
    d, slot = _blank_slot(code_byte=(0x99, 0xAA, 0x99))    # codes 9, 10, 9 -> (1, 2, 1) after offset
    H, I = d.H, d.I
    rng = np.random.default_rng(3)
    sg = rng.uniform(0.01, 0.1, I).astype(np.float16)
    su = rng.uniform(0.01, 0.1, I).astype(np.float16)
    sd = rng.uniform(0.01, 0.1, H).astype(np.float16)
    _set_scales(d, slot, 0, np.repeat(sg[:, None], H // 32, 1))
    _set_scales(d, slot, 1, np.repeat(su[:, None], H // 32, 1))
    _set_scales(d, slot, 2, np.repeat(sd[:, None], I // 32, 1))
    x = rng.standard_normal(H)
    Ssum = math.fsum(x)
    a = sg.astype(np.float64) * 1
    b = su.astype(np.float64) * 2
    hh = [a[r] * Ssum / (1 + math.exp(-a[r] * Ssum)) * b[r] * Ssum for r in range(I)]
    expect = sd.astype(np.float64) * 1 * math.fsum(hh)
    y, _ = O.expert_ffn(slot, d, x)
    assert np.allclose(y, expect, rtol=1e-12, atol=0)


# ------------------------------------------------------------------ routing

def _bf16(v):
    return S.f32_to_bf16_bits(np.asarray(v, np.float32))


def test_router_one_hot_input_reads_one_column():
    """x = e_h gives logits W[:, h] + b exactly (one exact product each)."""
    rng = np.random.default_rng(4)
    E, H = 8, 64
    W = rng.standard_normal((E, H)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32)
    x = np.zeros((3, H), np.float32)
    x[0, 5] = 1.0
    x[1, 63] = -2.0
    x[2, 0] = 0.5
    lg = O.router_logits(_bf16(x), W, b)
    assert np.array_equal(lg[0], W[:, 5].astype(np.float64) + b)
    assert np.array_equal(lg[1], -2.0 * W[:, 63].astype(np.float64) + b)
    assert np.array_equal(lg[2], 0.5 * W[:, 0].astype(np.float64) + b)
    assert np.array_equal(O.router_logits(_bf16(x), W, None)[0], W[:, 5].astype(np.float64))


def test_topk_hand_case_with_exact_tie():
    lg = np.array([[0.5, 2.0, -1.0, 2.0, 1.0, 2.0, 0.0, -3.0]])
    idx, w = O.topk(lg, 4)
    assert idx.tolist() == [[1, 3, 5, 4]]         # three-way tie at 2.0: lower index first
    e1 = math.exp(-1.0)
    z = 3 + e1
    assert np.allclose(w[0], [1 / z, 1 / z, 1 / z, e1 / z], rtol=1e-15)


def test_topk_two_way_softmax_closed_form():
    lg = np.array([[0.0, math.log(3.0), -50.0]])
    idx, w = O.topk(lg, 2)
    assert idx.tolist() == [[1, 0]]
    assert w[0, 0] == pytest.approx(0.75, rel=1e-15) and w[0, 1] == pytest.approx(0.25, rel=1e-15)


def test_topk_equals_full_stable_sort_brute_force():
    rng = np.random.default_rng(6)
    T, E, k = 300, 64, 10
    lg = np.round(rng.standard_normal((T, E)), 1)          # many exact ties
    idx, w = O.topk(lg, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-lg[t, e], e))[:k]
        assert idx[t].tolist() == order
    assert np.allclose(w.sum(1), 1.0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 1e-15) and np.all(w > 0) and np.all(w <= 1)


def test_topk_k_equals_E_is_the_dense_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((20, 16)) * 3
    idx, w = O.topk(lg, 16)
    for t in range(20):
        dense = softmax(lg[t])
        assert np.allclose(w[t], dense[idx[t]], rtol=1e-13)
        assert sorted(idx[t].tolist()) == list(range(16))


def test_permutation_equals_stable_argsort():
    rng = np.random.default_rng(8)
    for T, k, E in [(4, 2, 8), (37, 10, 512), (1000, 10, 64), (0, 10, 16)]:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32) \
            if T else np.zeros((0, k), np.int32)
        counts, offsets, perm, inv = O.permutation(idx, E)
        flat = idx.reshape(-1)
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert offsets[0] == 0 and offsets[E] == T * k
        assert np.array_equal(perm, np.argsort(flat, kind="stable"))
        assert np.array_equal(inv[perm], np.arange(T * k))


def test_histogram_totals_and_accumulation():
    rng = np.random.default_rng(9)
    L, E, T, k = 3, 32, 50, 10
    hist = np.zeros((L, E), np.uint32)
    for n in range(1, 5):
        for layer in range(L):
            idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
            counts, *_ = O.permutation(idx, E)
            O.hist_add(counts, layer, hist)
        assert np.all(hist.sum(1) == n * T * k)


def test_rank_hand_case_and_tie_order():
    hist = np.array([[5, 0, 7, 5], [7, 1, 0, 5]], np.uint32)
    pairs = O.rank(hist)
    assert pairs.tolist() == [[0, 2], [1, 0], [0, 0], [0, 3], [1, 3], [1, 1], [0, 1], [1, 2]]


def test_rank_full_pruned_profile_shape():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    L, E = facts["layers"]["value"], facts["experts_pruned"]["value"]
    rng = np.random.default_rng(10)
    hist = rng.integers(0, 50, (L, E)).astype(np.uint32)
    pairs = O.rank(hist)
    assert pairs.shape[0] == facts["profile_pairs_pruned"]["value"]
    key = pairs[:, 0].astype(np.int64) * E + pairs[:, 1]
    assert np.array_equal(np.sort(key), np.arange(L * E))
    c = hist[pairs[:, 0], pairs[:, 1]]
    assert np.all(np.diff(c.astype(np.int64)) <= 0)
    ref = np.lexsort((np.arange(L * E), -hist.reshape(-1).astype(np.int64)))
    assert np.array_equal(key, ref)


def test_page_shapes_match_workloads():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    assert facts["layers"]["value"] * facts["experts_full"]["value"] == facts["experts_total_full"]["value"]
    assert facts["layers"]["value"] * facts["experts_pruned"]["value"] == facts["experts_total_pruned"]["value"]
    for name in ("decode", "prefill", "decode_stack", "prefill_stack"):
        c = S.config(name)
        assert c.top_k == facts["top_k"]["value"]
        assert c.E in (facts["experts_full"]["value"], facts["experts_pruned"]["value"])
    assert S.config("prefill").T == facts["prefill_chunk_max"]["value"]
    assert S.config("decode").T == 1 + facts["spec_drafts"]["value"]
    assert round(facts["vram_slots_12gb"]["value"] / facts["experts_total_pruned"]["value"], 2) == \
        facts["random_hit_rate"]["value"]


# ------------------------------------------------------------------ pins added with the bulk expert check

def test_router_two_term_hand_case():
    """x = (1.5, -0.25) on two coordinates: l_e = 1.5 W[e, 3] - 0.25 W[e, 9] + b_e,
    written out by hand for chosen exactly representable weights."""
    E, H = 3, 16
    W = np.zeros((E, H), np.float32)
    W[0, 3], W[0, 9] = 2.0, 4.0          # 3 - 1 = 2
    W[1, 3], W[1, 9] = -1.0, 0.5         # -1.5 - 0.125 = -1.625
    W[2, 3], W[2, 9] = 0.125, -8.0       # 0.1875 + 2 = 2.1875
    b = np.array([0.5, 0.0, -0.25], np.float32)
    x = np.zeros((1, H), np.float32)
    x[0, 3], x[0, 9] = 1.5, -0.25
    lg = O.router_logits(_bf16(x), W, b)
    assert lg[0].tolist() == [2.5, -1.625, 1.9375]
    assert O.topk(lg, 2)[0].tolist() == [[0, 2]]


def test_histogram_per_expert_hand_case():
    """Counts land on their own (layer, expert) cell: a count moved to another
    expert of the same layer keeps the per-layer total but fails here."""
    hist = np.zeros((2, 4), np.uint32)
    O.hist_add(np.array([3, 0, 1, 6], np.int32), 1, hist)
    O.hist_add(np.array([0, 2, 0, 0], np.int32), 0, hist)
    O.hist_add(np.array([1, 1, 1, 1], np.int32), 1, hist)
    assert hist.tolist() == [[0, 2, 0, 0], [4, 1, 2, 7]]
    idx = np.array([[2, 0], [2, 3], [3, 2]], np.int32)   # 3 tokens, k = 2, E = 4
    counts, *_ = O.permutation(idx, 4)
    assert counts.tolist() == [1, 0, 3, 2]


def test_fp64_router_decides_a_tie_that_fp32_sums_lose():
    """The oracle's logits are fp64 sums of exact products.  Two router rows
    that differ by one fp32 ulp in one weight give fp64 logits that differ by
    that product exactly, while fp32 sequential sums of the same products round
    the difference away: the fp64 order (the higher index first here) is the
    one the oracle - and the GPU, which certifies against it - reports."""
    rng = np.random.default_rng(41)
    H = 2048
    x = _bf16(rng.standard_normal((1, H)).astype(np.float32))
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    W = np.zeros((2, H), np.float32)
    W[0] = (rng.standard_normal(H) / np.sqrt(H)).astype(np.float32)
    W[1] = W[0]
    h = int(np.argmin(np.abs(xf[0])))                  # the smallest |x_h|: a tiny difference
    if xf[0, h] == 0:
        h = int(np.argsort(np.abs(xf[0]))[np.count_nonzero(xf[0] == 0)])
    W[1, h] = np.nextafter(W[0, h], np.float32(np.inf) if xf[0, h] > 0 else np.float32(-np.inf))
    lg = O.router_logits(x, W, None)
    assert lg[0, 1] > lg[0, 0]                         # fp64: row 1 strictly ahead
    assert lg[0, 1] - lg[0, 0] == pytest.approx(float(xf[0, h]) * (float(W[1, h]) - float(W[0, h])), rel=1e-6)
    f32 = np.zeros(2, np.float32)
    for e in range(2):                                  # fp32 sums in index order
        s = np.float32(0)
        for i in range(H):
            s = np.float32(s + np.float32(xf[0, i] * W[e, i]))
        f32[e] = s
    assert f32[0] == f32[1]                             # fp32: an exact tie (row 0 would win)
    assert O.topk(lg, 1)[0].tolist() == [[1]]


def test_expert_ffn_rows_matches_per_element_oracle():
    """The whole-matrix restatement against the per-element C oracle (itself
    pinned above by closed forms) on random slots of each bit layout."""
    rng = np.random.default_rng(42)
    for bits in [(4, 4, 4), (2, 2, 4), (2, 4, 2)]:
        cfg = S.config("tiny", H=128, I=64, bits=bits, seed=43)
        d = cfg.desc()
        slot = S.gen_slot_host(cfg, 3)
        X = rng.standard_normal((5, cfg.H))
        Y, Hh = O.expert_ffn_rows(slot, d, X)
        for t in range(5):
            y, h = O.expert_ffn(slot, d, X[t])
            assert np.allclose(Y[t], y, rtol=1e-12, atol=1e-14)
            assert np.allclose(Hh[t], h, rtol=1e-12, atol=1e-14)
        for m in range(3):
            rows, K = S.matrix_shape(cfg.H, cfg.I, m)
            Wm = O.dequant_matrix(slot, d, m)
            for r, c in [(0, 0), (rows - 1, K - 1), (rows // 2, 33), (1, K // 2 + 7)]:
                assert Wm[r, c] == O.dequant(slot, d, m, r, c)


def test_topk_non_finite_logits_total_order():
    """NaN logits rank as -inf (below every number, ties by lower index) and
    weigh 0 when selected next to a finite maximum; +inf ranks first."""
    nan, inf = float("nan"), float("inf")
    lg = np.array([[nan, 1.0, -inf, 0.5, nan, 2.0],
                   [nan, nan, nan, nan, nan, nan],
                   [0.0, inf, 1.0, inf, -1.0, nan]])
    idx, w = O.topk(lg, 4)
    assert idx[0].tolist() == [5, 1, 3, 0]            # the NaN at 0 ties -inf at 2 and wins by index
    assert w[0, 3] == 0.0 and np.isclose(w[0, :3].sum(), 1.0)
    assert idx[1].tolist() == [0, 1, 2, 3]            # all NaN: the lowest indices
    assert np.all(np.isnan(w[1]))
    assert idx[2].tolist() == [1, 3, 2, 0]
    assert np.all(np.isnan(w[2]))                     # exp(inf - inf)
