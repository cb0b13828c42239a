"""The seeded input recipe: every generator is deterministic, its streams are
independent, and the workloads have the distributions and loads the design
states for them (logits ~ N(0, 1), the Zipf bias law, uniform codes, scales in
their ranges, about 160 tokens per expert in the prefill chunk, loads from
zero to thousands under the Zipf bias, the mid-T distinct-expert counts).  The
routing statistics use a plain fp32 matrix product and a partial sort: they
measure the inputs, not the method, so near-ties do not matter."""
import numpy as np
import pytest

import moe_synth as S


def _routing_counts(x_bits, W, b, k):
    xf = (x_bits.astype(np.uint32) << 16).view(np.float32)
    lg = xf @ W.T
    if b is not None:
        lg = lg + b
    idx = np.argpartition(-lg, k - 1, axis=1)[:, :k]
    return np.bincount(idx.ravel(), minlength=W.shape[0]), lg


def test_generators_are_deterministic_and_streams_independent():
    cfg = S.config("tiny", E=16, top_k=4, H=128, I=64, T=6, zipf_s=1.1, seed=5)
    for fn in (lambda: S.gen_x(cfg), lambda: S.gen_router(cfg), lambda: S.gen_bias(cfg),
               lambda: S.gen_slot_table(cfg), lambda: S.gen_arena_host(cfg)):
        assert np.array_equal(fn(), fn())
    assert not np.array_equal(S.gen_x(cfg), S.gen_x(cfg, stream_offset=1))
    assert not np.array_equal(S.gen_router(cfg, 0), S.gen_router(cfg, 1))
    other = S.config("tiny", E=16, top_k=4, H=128, I=64, T=6, zipf_s=1.1, seed=6)
    assert not np.array_equal(S.gen_x(cfg), S.gen_x(other))
    # a shorter window is the first rows of a longer one from the same stream
    assert np.array_equal(S.gen_x(cfg, T=3), S.gen_x(cfg)[:3])


def test_hidden_states_and_router_give_unit_logits():
    """x ~ N(0, 1) in bf16 and W_r ~ N(0, 1/H): logits ~ N(0, 1) (decode)."""
    cfg = S.config("decode")
    x = S.gen_x(cfg, T=64)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    assert abs(xf.mean()) < 0.01 and abs(xf.std() - 1.0) < 0.01
    W = S.gen_router(cfg)
    assert abs(W.std() * np.sqrt(cfg.H) - 1.0) < 0.01
    _, lg = _routing_counts(x, W, None, cfg.top_k)
    assert abs(lg.mean()) < 0.02 and abs(lg.std() - 1.0) < 0.02


def test_zipf_bias_is_the_stated_law():
    """b_e = -1.1 ln r(e), r a seeded permutation of 1..E, per layer."""
    cfg = S.config("decode_stack")
    b0, b1 = S.gen_bias(cfg, 0), S.gen_bias(cfg, 1)
    law = (-1.1 * np.log(np.arange(1, cfg.E + 1, dtype=np.float64))).astype(np.float32)
    assert np.array_equal(np.sort(b0)[::-1], law)
    assert not np.array_equal(b0, b1)
    assert S.gen_bias(S.config("decode")) is None


def test_slot_table_is_a_permutation():
    cfg = S.config("decode_stack")
    t = S.gen_slot_table(cfg)
    assert t.dtype == np.int32 and np.array_equal(np.sort(t), np.arange(cfg.L * cfg.E))


@pytest.mark.parametrize("bits,lo,hi", [((4, 4, 4), 0.001, 0.01), ((2, 2, 4), *S.STACK_SCALE)])
def test_codes_are_uniform_and_scales_in_range(bits, lo, hi):
    cfg = S.config("tiny", E=4, top_k=2, H=256, I=128, bits=bits, scale_lo=lo, scale_hi=hi, seed=9)
    d = cfg.desc()
    arena = S.gen_arena_host(cfg)
    for s in range(d.n_slots):
        slot = arena[s * d.slot_bytes:(s + 1) * d.slot_bytes]
        for m in range(3):
            rows, K = S.matrix_shape(d.H, d.I, m)
            b = d.bits(m)
            raw = slot[d.off_codes[m]:d.off_codes[m] + rows * K * b // 8]
            codes = np.unpackbits(raw[:, None], axis=1, bitorder="little").reshape(-1, b)
            vals = (codes * (1 << np.arange(b))).sum(1)
            cnt = np.bincount(vals, minlength=1 << b)
            expect = vals.size / (1 << b)
            assert np.all(np.abs(cnt - expect) < 5 * np.sqrt(expect)), (s, m, cnt)
            sc = slot[d.off_scales[m]:d.off_scales[m] + rows * (K // 32) * 2].view(np.float16).astype(np.float64)
            assert sc.min() >= lo * (1 - 2 ** -10) and sc.max() <= hi * (1 + 2 ** -10)
            assert sc.max() - sc.min() > 0.9 * (hi - lo)


def test_one_slot_regenerates_alone():
    cfg = S.config("tiny", E=6, top_k=2, H=128, I=64, seed=4)
    d = cfg.desc()
    arena = S.gen_arena_host(cfg)
    for s in (0, 3, 5):
        assert np.array_equal(S.gen_slot_host(cfg, s), arena[s * d.slot_bytes:(s + 1) * d.slot_bytes])


def test_device_generator_scales_in_range_on_cpu():
    """gen_arena_device draws the large arenas; run on the CPU here, the scale
    sections hold fp16 in [lo, hi] and the draw is repeatable."""
    cfg = S.config("tiny", E=3, top_k=2, H=256, I=128, bits=(2, 2, 4), seed=8)
    d = cfg.desc()
    a = S.gen_arena_device(cfg, device="cpu").numpy()
    assert np.array_equal(a, S.gen_arena_device(cfg, device="cpu").numpy())
    for s in range(d.n_slots):
        slot = a[s * d.slot_bytes:(s + 1) * d.slot_bytes]
        for m in range(3):
            rows, K = S.matrix_shape(d.H, d.I, m)
            sc = slot[d.off_scales[m]:d.off_scales[m] + rows * (K // 32) * 2].view(np.float16).astype(np.float64)
            assert sc.min() >= cfg.scale_lo * (1 - 2 ** -10) and sc.max() <= cfg.scale_hi * (1 + 2 ** -10)


def test_prefill_chunk_loads():
    """T = 8192, k = 10, E = 512, no bias: 160 pairs per expert on average,
    every expert loaded (113 to 214 in this draw)."""
    cfg = S.config("prefill")
    cnt, _ = _routing_counts(S.gen_x(cfg), S.gen_router(cfg), None, cfg.top_k)
    assert cnt.sum() == cfg.T * cfg.top_k and cnt.mean() == 160
    assert 90 <= cnt.min() and cnt.max() <= 240


def test_prefill_stack_loads_span_zero_to_thousands():
    """The Zipf bias of the 48 x 512 stack: many experts get no token of the
    chunk while the top-ranked ones get thousands."""
    cfg = S.config("prefill_stack")
    cnt, _ = _routing_counts(S.gen_x(cfg), S.gen_router(cfg, 0), S.gen_bias(cfg, 0), cfg.top_k)
    assert (cnt == 0).sum() > 100 and cnt.max() > 4000


@pytest.mark.parametrize("T,lo,hi", [(16, 120, 150), (64, 340, 380), (256, 495, 512)])
def test_mid_T_distinct_experts(T, lo, hi):
    """Mid-T chunks at the model's shape select a distinct expert for most
    pairs: about 131, 356 and 509 distinct experts at T = 16, 64, 256 in
    layer 0's draw, 1 to 13 pairs each."""
    cfg = S.config("prefill", T=T)
    cnt, _ = _routing_counts(S.gen_x(cfg), S.gen_router(cfg), None, cfg.top_k)
    nz = cnt[cnt > 0]
    assert lo <= nz.size <= hi and nz.max() <= 14


def test_pruned_stack_traffic_is_concentrated():
    """The 48 x 256 stack under its Zipf bias, 20 windows of 5 tokens per
    layer: the 300 most routed of the 12,288 (layer, expert) pairs take about
    half of the routed reads (48% in this draw) and the first 2,537 nearly all
    (98%): a few hundred experts carry much of the traffic."""
    cfg = S.config("decode_stack")
    tot = np.zeros((cfg.L, cfg.E))
    for layer in range(cfg.L):
        W, b = S.gen_router(cfg, layer), S.gen_bias(cfg, layer)
        x = np.concatenate([S.gen_x(cfg, 5, stream_offset=o) for o in range(20)])
        cnt, _ = _routing_counts(x, W, b, cfg.top_k)
        tot[layer] = cnt
    f = np.sort(tot.ravel())[::-1]
    assert f.sum() == cfg.L * 20 * 5 * cfg.top_k
    assert 0.40 < f[:300].sum() / f.sum() < 0.56
    assert f[:2537].sum() / f.sum() > 0.95
