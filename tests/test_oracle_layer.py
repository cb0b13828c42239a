"""Layer-level pins for the CPU oracle: special cases with known outputs and
an independent vectorised restatement on the tiny workload.  CPU only."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O


def _tiny():
    cfg = S.config("tiny")
    d = cfg.desc()
    arena = S.gen_arena_host(cfg)
    st = S.gen_slot_table(cfg)
    x = S.gen_x(cfg)
    W = S.gen_router(cfg)
    return cfg, d, arena, st, x, W


def _bits_to_f64(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def _dense(d, slot):
    """Dequantised matrices of one slot with numpy bit ops (independent unpacking)."""
    mats = []
    for m in range(3):
        rows, K = S.matrix_shape(d.H, d.I, m)
        b = d.bits(m)
        raw = np.frombuffer(slot[d.off_codes[m]:d.off_codes[m] + rows * K * b // 8].tobytes(), np.uint8)
        per = 8 // b
        shifts = (np.arange(per) * b).astype(np.uint8)
        codes = ((raw[:, None] >> shifts[None, :]) & ((1 << b) - 1)).reshape(rows, K).astype(np.float64)
        sc = np.frombuffer(slot[d.off_scales[m]:d.off_scales[m] + rows * (K // 32) * 2].tobytes(),
                           np.float16).astype(np.float64).reshape(rows, K // 32)
        mats.append(np.repeat(sc, 32, axis=1) * (codes - 2 ** (b - 1)))
    return mats


def test_tiny_layer_matches_vectorised_restatement():
    cfg, d, arena, st, x, W = _tiny()
    res = O.moe_layer(d, arena, st, 1, 0, x, W, None, cfg.top_k)
    assert res["rc"] == 0
    xf = _bits_to_f64(x)
    lg = xf @ W.astype(np.float64).T
    for t in range(cfg.T):
        order = np.lexsort((np.arange(cfg.E), -lg[t]))[:cfg.top_k]
        assert res["idx"][t].tolist() == order.tolist()
        z = np.exp(lg[t, order] - lg[t, order[0]])
        w = z / z.sum()
        assert np.allclose(res["w"][t], w, rtol=1e-12)
        acc = np.zeros(cfg.H)
        for j, e in enumerate(order):
            slot = arena[st[e] * d.slot_bytes:(st[e] + 1) * d.slot_bytes]
            Wg, Wu, Wd = _dense(d, slot)
            g, u = Wg @ xf[t], Wu @ xf[t]
            acc += w[j] * (Wd @ (g / (1 + np.exp(-g)) * u))
        assert np.allclose(res["out_f64"][t], xf[t] + acc, rtol=1e-10, atol=1e-12)


def test_all_zero_scales_give_residual_exactly():
    cfg, d, arena, st, x, W = _tiny()
    a = arena.copy()
    for s in range(d.n_slots):
        for m in range(3):
            rows, K = S.matrix_shape(d.H, d.I, m)
            o = s * d.slot_bytes + d.off_scales[m]
            a[o:o + rows * (K // 32) * 2] = 0
    res = O.moe_layer(d, a, st, 1, 0, x, W, None, cfg.top_k, residual=True)
    assert np.array_equal(res["out"], x)
    res = O.moe_layer(d, a, st, 1, 0, x, W, None, cfg.top_k, residual=False)
    assert np.all(res["out_f64"] == 0.0)


def test_identical_experts_make_output_independent_of_routing():
    cfg, d, arena, st, x, W = _tiny()
    one = arena[:d.slot_bytes]
    a = np.tile(one, d.n_slots)
    r1 = O.moe_layer(d, a, st, 1, 0, x, W, None, cfg.top_k)
    W2 = np.random.default_rng(11).standard_normal(W.shape).astype(np.float32)
    r2 = O.moe_layer(d, a, st, 1, 0, x, W2, None, cfg.top_k)
    assert not np.array_equal(r1["idx"], r2["idx"])
    assert np.allclose(r1["out_f64"], r2["out_f64"], rtol=1e-12, atol=1e-12)
    # weights sum to one, so the mixture of one expert is that expert's output
    xf = _bits_to_f64(x)
    for t in range(cfg.T):
        y, _ = O.expert_ffn(one, d, xf[t])
        assert np.allclose(r1["out_f64"][t], xf[t] + y, rtol=1e-12, atol=1e-12)


def test_missing_slot_contributes_zero_and_is_reported():
    cfg, d, arena, st, x, W = _tiny()
    ref = O.moe_layer(d, arena, st, 1, 0, x, W, None, cfg.top_k)
    e_bad = int(ref["idx"][0, 0])
    st2 = st.copy()
    st2[e_bad] = -1
    res = O.moe_layer(d, arena, st2, 1, 0, x, W, None, cfg.top_k)
    assert res["rc"] == O.ORC_ERR_SLOT
    assert np.array_equal(res["idx"], ref["idx"])
    # zeroing that expert's scales gives the same result as dropping its slot
    a = arena.copy()
    s = st[e_bad]
    for m in range(3):
        rows, K = S.matrix_shape(d.H, d.I, m)
        o = s * d.slot_bytes + d.off_scales[m]
        a[o:o + rows * (K // 32) * 2] = 0
    res0 = O.moe_layer(d, a, st, 1, 0, x, W, None, cfg.top_k)
    assert np.array_equal(res0["out_f64"], res["out_f64"])


def test_token_subset_matches_full_run():
    cfg, d, arena, st, x, W = _tiny()
    full = O.moe_layer(d, arena, st, 1, 0, x, W, None, cfg.top_k)
    sub = O.moe_layer(d, arena, st, 1, 0, x, W, None, cfg.top_k, tokens=np.array([2, 0]))
    for t in (0, 2):
        assert np.array_equal(sub["out"][t], full["out"][t])
        assert np.array_equal(sub["idx"][t], full["idx"][t])
    assert np.all(sub["out"][1] == 0)


def _steer_setup():
    cfg, d, arena, st, x, W = _tiny()
    rng = np.random.default_rng(71)
    v = rng.standard_normal(cfg.H)
    v = (v / np.linalg.norm(v)).astype(np.float32)
    return cfg, d, arena, st, x, W, v


def test_steer_parallel_and_orthogonal_rows_closed_form():
    """With every expert at zero scale the layer output is x itself; for the
    unit direction e_5, a row equal to a multiple of e_5 projects to exactly 0
    and a row with a zero 5th entry is unchanged."""
    cfg, d, arena, st, x, W = _tiny()
    z = arena.copy()
    for s in range(d.n_slots):
        base = s * d.slot_bytes
        for m in range(3):
            rows, K = S.matrix_shape(d.H, d.I, m)
            z[base + d.off_scales[m]:base + d.off_scales[m] + rows * (K // 32) * 2] = 0
    v = np.zeros(cfg.H, np.float32)
    v[5] = 1.0
    xs = np.zeros_like(x)
    xs[0, 5] = S.f32_to_bf16_bits(np.array([-3.25], np.float32))[0]           # parallel to v
    xs[1] = x[1]
    xs[1, 5] = 0                                                              # orthogonal to v
    xs[2:] = x[2:]
    res = O.moe_layer(d, z, st, 1, 0, xs, W, None, cfg.top_k, steer=v)
    assert np.all(res["out_f64"][0] == 0.0)
    assert np.array_equal(res["out"][1], xs[1])


def test_steer_invariants_on_the_tiny_layer():
    """Against the unsteered layer output h, with s = h . v and n = v . v (v is
    an fp32 rounding of a unit vector, so n = 1 only to ~1e-7):
    out . v = s (1 - n), ||out||^2 = ||h||^2 - 2 s^2 + s^2 n, and a second
    projection moves the row only by s (1 - n) v."""
    cfg, d, arena, st, x, W, v = _steer_setup()
    h = O.moe_layer(d, arena, st, 1, 0, x, W, None, cfg.top_k)["out_f64"]
    out = O.moe_layer(d, arena, st, 1, 0, x, W, None, cfg.top_k, steer=v)["out_f64"]
    vd = v.astype(np.float64)
    n = vd @ vd
    assert abs(n - 1) < 1e-6
    for t in range(cfg.T):
        s = h[t] @ vd
        tol = 1e-13 * np.linalg.norm(h[t]) ** 2
        assert abs(out[t] @ vd - s * (1 - n)) <= 1e-13 * np.linalg.norm(h[t])
        assert abs(out[t] @ out[t] - (h[t] @ h[t] - 2 * s * s + s * s * n)) <= tol
        assert np.allclose(O.steer(out[t], v), out[t] - s * (1 - n) * vd, rtol=0, atol=1e-13 * np.linalg.norm(h[t]))
