"""Prefill path (tensor-core grouped GEMMs) through the C ABI against the CPU oracle."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O
from helpers import PAIR_NORM_RTOL, PAIR_RTOL, Workload, assert_out_close, check_routing, run_layer

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


def _full_size(cfg, layer=0, all_tokens=False):
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
    if all_tokens:
        toks = np.arange(cfg.T, dtype=np.int32)
    else:
        toks = _sample_tokens(cfg.T, idx, cfg.E, np.random.default_rng(cfg.seed), n=min(48, cfg.T))
    ref = wl.oracle_layer(layer, x, tokens=toks)
    assert np.array_equal(ref["idx"][toks], idx[toks])
    assert_out_close(out, ref["out_f64"], rows=toks)
    return counts


def test_prefill_full_chunk_uniform(cuda_ok):
    """8,192 tokens, E = 512, 4-bit, Gaussian router (about 160 tokens per expert)."""
    counts = _full_size(S.config("prefill"))
    assert counts.sum() == 8192 * 10


@pytest.mark.parametrize("T", [16, 64, 256])
def test_prefill_mid_T_model_shape(cuda_ok, T):
    """Mid-T chunks (batched verify windows, short prompts) at the model's shape:
    E = 512, H = 2048, I = 512, 4-bit, Gaussian router.  With 160 to 2,560 pairs
    over 512 experts most experts get 0 to 5 pairs, so nearly every grouped-GEMM
    tile is a single ragged column block.  Routing of every token bit-exact, the
    histogram bit-exact, and the outputs of every token (T <= 64) or of 48
    sampled tokens plus every token of the two most and two least loaded experts."""
    counts = _full_size(S.config("prefill", T=T, seed=70 + T), all_tokens=T <= 64)
    assert counts.sum() == T * 10
    used = counts[counts > 0]
    assert used.max() <= 40 and used.min() >= 1
    assert (counts > 0).sum() >= min(T * 10 // 2, 300)


def _pair_outputs(ws, cfg, T, sel):
    """Rows `sel` (pair positions) of the per-pair expert outputs w * y (bf16)
    the prefill call left in its workspace."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    off = M.moe_workspace_offset(T, cfg.E, cfg.top_k, cfg.H, cfg.I, M.MOE_WS_PAIR_OUT)
    Y = ws[off:off + T * cfg.top_k * cfg.H * 2].view(torch.int16).view(T * cfg.top_k, cfg.H)
    return Y[torch.from_numpy(np.asarray(sel, np.int64)).cuda()].cpu().numpy().view(np.uint16)


def test_prefill_stack_48_layers_teacher_forced(cuda_ok):
    """The 48 x 512, 2/2/4-bit, Zipf-routed stack at full size (T = 8,192),
    the library chaining its own bf16 outputs layer to layer; at every layer the
    oracle takes the library's input to that layer (teacher forcing) and checks:
      - the routing of all 8,192 tokens (indices, offsets, permutation) bit-exact;
      - the layer output of 64 sampled tokens;
      - every routed pair of the 3 most- and the 3 least-loaded experts, on the
        per-pair expert outputs w * y (bf16 intermediates: PAIR_RTOL);
    and at the end the 48 x 512 histogram bit-exact and its ranking equal to the
    oracle's."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config("prefill_stack")
    wl = Workload(cfg)
    T, E, k = cfg.T, cfg.E, cfg.top_k
    x = wl.x_host()
    hist = torch.zeros((cfg.L, E), dtype=torch.int32, device="cuda")
    ref_hist = np.zeros((cfg.L, E), np.uint32)
    ws = torch.empty(M.moe_workspace_bytes(T, E, k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(cfg.seed)
    loads = []
    for layer in range(cfg.L):
        xt = torch.from_numpy(x.view(np.int16)).cuda()
        out = torch.zeros_like(xt)
        from helpers import route_buffers
        ro = route_buffers(T, k, E)
        M.moe_forward_prefill(wl.desc, wl.arena, wl.slot_table, cfg.L, layer, xt, wl.W[layer], wl.b[layer], k,
                              True, out, hist=hist, route_out=ro, ws=ws)
        torch.cuda.synchronize()
        assert M.moe_last_device_error() == 0
        res = {key: v.cpu().numpy() for key, v in ro.items()}
        res["topk_idx"] = res["topk_idx"].reshape(T, k)
        res["topk_w"] = res["topk_w"].reshape(T, k)
        lg = O.router_logits(x, wl.W_host[layer], wl.b_host[layer])
        idx, w = O.topk(lg, k)
        counts = check_routing(res, idx, w, E)
        O.hist_add(counts, layer, ref_hist)
        loads.append((int(counts.max()), int(counts[counts > 0].min())))
        ob = out.cpu().numpy().view(np.uint16)
        moe = torch.zeros_like(xt)  # the same layer without the residual: its MoE part alone
        M.moe_forward_prefill(wl.desc, wl.arena, wl.slot_table, cfg.L, layer, xt, wl.W[layer], wl.b[layer], k,
                              False, moe, ws=ws)
        toks = np.sort(rng.choice(T, 64, replace=False)).astype(np.int32)
        ref = wl.oracle_layer(layer, x, tokens=toks, residual=False)
        # without the residual the row is the MoE part alone, a sum of bf16 intermediates: PAIR_RTOL
        rel = assert_out_close(moe.cpu().numpy().view(np.uint16), ref["out_f64"], rows=toks, tol=PAIR_RTOL)
        assert rel <= PAIR_NORM_RTOL
        xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert_out_close(ob, xf + ref["out_f64"], rows=toks)
        assert np.all(np.isfinite((ob.astype(np.uint32) << 16).view(np.float32)))
        # every pair of the 3 most- and 3 least-loaded (nonzero) experts
        _, offsets, perm, _ = O.permutation(idx, E)
        used = np.nonzero(counts)[0]
        order = used[np.argsort(counts[used], kind="stable")]
        for e in list(order[:3]) + list(order[-3:]):
            pos = np.arange(offsets[e], offsets[e + 1])
            pairs = perm[pos]
            s = int(wl.slot_table_host[layer * E + e])
            y, _ = O.expert_ffn_rows(wl.slot_bytes_of(s), wl.desc, xf[pairs // k])
            r = w.reshape(-1)[pairs][:, None] * y
            rel = assert_out_close(_pair_outputs(ws, cfg, T, pos), r, tol=PAIR_RTOL)
            assert rel <= PAIR_NORM_RTOL
        x = ob
    got = hist.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref_hist)
    assert np.array_equal(M.moe_rank_experts(got), O.rank(ref_hist))
    assert max(m for m, _ in loads) > 1000 and min(n for _, n in loads) < 50
