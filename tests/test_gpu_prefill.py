"""Prefill path (tensor-core grouped GEMMs) through the C ABI against the CPU oracle."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O
from helpers import Workload, assert_out_close, check_routing, run_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 37, 300])
def test_prefill_small_shapes(cuda_ok, T):
    """E = 8, H = 256, I = 128: one to several N tiles per expert, ragged tails."""
    cfg = S.config("tiny", H=256, I=128, T=T, seed=11)
    wl = Workload(cfg)
    x = wl.x_host()
    out, res = run_layer(wl, 0, x, prefill=True)
    ref = wl.oracle_layer(0, x)
    check_routing(res, ref["idx"], ref["w"], cfg.E)
    assert_out_close(out, ref["out_f64"])


def test_prefill_skewed_mixed_bits(cuda_ok):
    """Zipf-biased router: loads from 0 to several 256-row tiles per expert."""
    cfg = S.config("tiny", E=64, top_k=10, H=512, I=256, T=700, bits=(2, 2, 4), zipf_s=1.1,
                   router_std=None, seed=12)
    wl = Workload(cfg)
    x = wl.x_host()
    out, res = run_layer(wl, 0, x, prefill=True)
    ref = wl.oracle_layer(0, x)
    counts = check_routing(res, ref["idx"], ref["w"], cfg.E)
    assert counts.max() > 2 * counts.mean()
    assert_out_close(out, ref["out_f64"])


def test_prefill_no_residual(cuda_ok):
    cfg = S.config("tiny", E=16, top_k=4, H=128, I=128, T=64, seed=13)
    wl = Workload(cfg)
    x = wl.x_host()
    out, res = run_layer(wl, 0, x, prefill=True, residual=False)
    ref = wl.oracle_layer(0, x, residual=False)
    check_routing(res, ref["idx"], ref["w"], cfg.E)
    assert_out_close(out, ref["out_f64"])


def test_prefill_matches_decode_on_same_window(cuda_ok):
    cfg = S.config("decode", seed=14)
    wl = Workload(cfg)
    x = S.gen_x(cfg, 5)
    o_dec, r_dec = run_layer(wl, 0, x, prefill=False)
    o_pre, r_pre = run_layer(wl, 0, x, prefill=True)
    assert np.array_equal(r_dec["topk_idx"], r_pre["topk_idx"])
    assert np.array_equal(r_dec["perm"], r_pre["perm"])
    ref = wl.oracle_layer(0, x)
    assert_out_close(o_dec, ref["out_f64"])
    assert_out_close(o_pre, ref["out_f64"])


def _sample_tokens(T, idx, E, rng, n=48):
    """n random tokens plus every token of the 2 most and 2 least loaded experts."""
    counts = np.bincount(idx.reshape(-1), minlength=E)
    used = np.nonzero(counts)[0]
    order = used[np.argsort(counts[used], kind="stable")]
    pick = set(rng.choice(T, n, replace=False).tolist())
    for e in list(order[:2]) + list(order[-2:]):
        toks = np.nonzero((idx == e).any(1))[0]
        pick.update(toks[:64].tolist())
    return np.array(sorted(pick), np.int32)


def _full_size(cfg, layer=0):
    import torch
    wl = Workload(cfg)
    x = wl.x_host()
    hist = torch.zeros((cfg.L, cfg.E), dtype=torch.int32, device="cuda")
    out, res = run_layer(wl, layer, x, prefill=True, hist=hist)
    # routing of every token: fp64 router in the oracle
    lg = O.router_logits(x, wl.W_host[layer], wl.b_host[layer])
    idx, w = O.topk(lg, cfg.top_k)
    counts = check_routing(res, idx, w, cfg.E)
    ref_hist = np.zeros((cfg.L, cfg.E), np.uint32)
    O.hist_add(counts, layer, ref_hist)
    assert np.array_equal(hist.cpu().numpy().view(np.uint32), ref_hist)
    toks = _sample_tokens(cfg.T, idx, cfg.E, np.random.default_rng(cfg.seed))
    ref = wl.oracle_layer(layer, x, tokens=toks)
    assert np.array_equal(ref["idx"][toks], idx[toks])
    assert_out_close(out, ref["out_f64"], rows=toks)
    return counts


def test_prefill_full_chunk_uniform(cuda_ok):
    """8,192 tokens, E = 512, 4-bit, Gaussian router (about 160 tokens per expert)."""
    counts = _full_size(S.config("prefill"))
    assert counts.sum() == 8192 * 10


def test_prefill_stack_layer_zipf(cuda_ok):
    """One layer of the 48 x 512, 2/2/4-bit, Zipf-routed stack at full size."""
    counts = _full_size(S.config("prefill_stack"), layer=7)
    assert counts.max() > 1000 and counts.min() < 50
