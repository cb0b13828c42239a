"""Expert profile (STRP v1) and the slot-budget hit-rate simulator: the
library's host code and the oracle's restatement against a hand-assembled file,
the page's shapes, malformed files, and the page's own correctness check that
a ranked profile hits far more often than a wrong index mapping (about
S / (L * E)).  CPU only."""
import json
import os

import numpy as np
import pytest

import moe_synth as S
import oracle as O
from oracle import profile as OP
import quantized_expert_ffn_top10_b200 as M

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand():
    g = json.load(open(os.path.join(GOLDEN, "strp_hand_case.json")))
    return g, bytes.fromhex(g["hex"].replace(" ", ""))


def test_hand_case_bytes():
    g, ref = _hand()
    pairs = np.array(g["pairs"], np.uint16)
    assert OP.profile_bytes(g["pairs"], g["L"], g["E"]) == ref
    assert M.moe_profile_write(pairs, g["L"], g["E"]) == ref
    L, E, pr, inv = M.moe_profile_read(ref)
    assert (L, E) == (2, 3) and pr.tolist() == g["pairs"]
    assert inv.tolist() == [[1, -1, -1], [2, -1, 0]]
    assert OP.parse_profile(ref)[3] == inv.tolist()


def test_hand_case_hit_rates():
    g, _ = _hand()
    hist = np.array(g["hist"], np.uint32)
    for slots, v in g["hit_rate_slots"].items():
        assert OP.hit_rate(g["pairs"], int(slots), hist) == pytest.approx(v, abs=1e-15)
        assert M.moe_profile_hit_rate(np.array(g["pairs"], np.uint16), 2, 3, int(slots), hist) == \
            pytest.approx(v, abs=1e-15)


def test_full_pruned_profile_shape_and_round_trip():
    """48 x 256 = 12,288 ranked pairs (the Coder profile of the page): the
    library's file equals the oracle's, and reads back to the same ranking."""
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    L, E = facts["layers"]["value"], facts["experts_pruned"]["value"]
    rng = np.random.default_rng(61)
    hist = rng.integers(0, 40, (L, E)).astype(np.uint32)
    pairs = O.rank(hist)
    data = M.moe_profile_write(pairs, L, E)
    assert len(data) == 24 + 4 * L * E * 2 == M.lib().moe_profile_bytes(L * E, L, E)
    assert data == OP.profile_bytes(pairs.tolist(), L, E)
    L2, E2, pr, inv = M.moe_profile_read(data)
    assert (L2, E2) == (L, E) and np.array_equal(pr, pairs)
    assert np.array_equal(inv.reshape(-1)[pairs[:, 0].astype(int) * E + pairs[:, 1]], np.arange(L * E))


def test_partial_profile_marks_unranked():
    rng = np.random.default_rng(62)
    L, E = 4, 16
    pairs = O.rank(rng.integers(0, 9, (L, E)).astype(np.uint32))[:20]
    data = M.moe_profile_write(pairs, L, E)
    assert data == OP.profile_bytes(pairs.tolist(), L, E)
    _, _, pr, inv = M.moe_profile_read(data)
    assert (inv == -1).sum() == L * E - 20 and sorted(inv[inv >= 0].tolist()) == list(range(20))


def test_malformed_files_are_rejected():
    g, ref = _hand()
    bad = [b"STRQ" + ref[4:], ref[:4] + (2).to_bytes(4, "little") + ref[8:], ref[:-4], ref + b"\0\0\0\0",
           ref[:24] + (5).to_bytes(2, "little") + ref[26:]]  # a pair's layer out of range
    for b in bad:
        with pytest.raises(M.MoeError):
            M.moe_profile_read(b)
    with pytest.raises(M.MoeError):
        M.moe_profile_write(np.array([[0, 1], [0, 1]], np.uint16), 2, 3)  # ranked twice
    with pytest.raises(M.MoeError):
        M.moe_profile_write(np.array([[2, 0]], np.uint16), 2, 3)          # layer out of range


def test_hit_rate_bounds_and_random_ranking_baseline():
    rng = np.random.default_rng(63)
    L, E = 8, 32
    hist = rng.integers(0, 100, (L, E)).astype(np.uint32)
    pairs = O.rank(hist)
    rates = [M.moe_profile_hit_rate(pairs, L, E, s, hist) for s in range(0, L * E + 1, 16)]
    assert rates[0] == 0.0 and rates[-1] == pytest.approx(1.0) and np.all(np.diff(rates) >= 0)
    S_ = 64
    rnd = [M.moe_profile_hit_rate(pairs[rng.permutation(L * E)], L, E, S_, hist) for _ in range(400)]
    assert np.mean(rnd) == pytest.approx(S_ / (L * E), abs=0.01)


def test_ranked_profile_beats_a_wrong_index_map():
    """The page's check, on the pruned 48 x 256 stack with its Zipf-skewed
    router: a profile ranked from one run's routing counts, evaluated on a
    held-out run at the page's 2,537 slots, hits far more often than the
    slot share 2,537 / 12,288 that a wrong index map (here: each layer's
    expert ids scrambled) falls back to."""
    cfg = S.config("decode_stack")
    L, E, k = cfg.L, cfg.E, cfg.top_k
    slots = 2537
    train = np.zeros((L, E), np.uint32)
    test = np.zeros((L, E), np.uint32)
    for layer in range(L):
        W, b = S.gen_router(cfg, layer), S.gen_bias(cfg, layer)
        for h, off in ((train, 0), (test, 1)):
            idx, _ = O.topk(O.router_logits(S.gen_x(cfg, 40, stream_offset=100 + off), W, b), k)
            counts, *_ = O.permutation(idx, E)
            O.hist_add(counts, layer, h)
    pairs = M.moe_rank_experts(train)
    ranked = M.moe_profile_hit_rate(pairs, L, E, slots, test)
    assert ranked == pytest.approx(OP.hit_rate(pairs.tolist(), slots, test), abs=1e-12)
    rng = np.random.default_rng(64)
    wrong = pairs.copy()
    wrong[:, 1] = np.array([rng.permutation(E) for _ in range(L)])[wrong[:, 0].astype(int), wrong[:, 1].astype(int)]
    scrambled = M.moe_profile_hit_rate(wrong, L, E, slots, test)
    share = slots / (L * E)
    print(f"\n[profile hit rate] ranked {ranked:.3f}, wrong index map {scrambled:.3f}, slot share {share:.3f}")
    assert ranked > 2.5 * share and abs(scrambled - share) < 0.08
