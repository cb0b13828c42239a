"""The chunk routers - fp64 tensor-core logits for 8 < T <= 128, bf16-plane
tensor-core logits above (E % 128 == 0 and H % 64 == 0), each with a certified
top-k - on exact ties, near ties, a zero token and a huge-norm token; the
measured slack of their error bounds; and moe_route_histogram through the C
ABI."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O
from helpers import Workload, assert_out_close, check_routing, route_buffers, run_layer

pytestmark = pytest.mark.gpu


def _route(x_bits, W, b, k, want_logits=False):
    """moe_route on host inputs; returns the routing (and the fast logits:
    fp64 up to MOE_ROUTER_F64_MAX_T tokens, fp32 above)."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    T, H = x_bits.shape
    E = W.shape[0]
    x = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()
    Wd = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    bd = None if b is None else torch.from_numpy(np.ascontiguousarray(b)).cuda()
    ro = route_buffers(T, k, E)
    ws = torch.empty(M.moe_workspace_bytes(T, E, k, H, 32), dtype=torch.uint8, device="cuda")
    M.moe_route(x, Wd, bd, k, ro["topk_idx"], ro["topk_w"], ro["expert_offsets"], ro["perm"], ws)
    torch.cuda.synchronize()
    assert M.moe_last_device_error() == 0
    res = {key: v.cpu().numpy() for key, v in ro.items()}
    res["topk_idx"] = res["topk_idx"].reshape(T, k)
    res["topk_w"] = res["topk_w"].reshape(T, k)
    if want_logits:
        off = M.moe_workspace_offset(T, E, k, H, 32, M.MOE_WS_FAST_LOGITS)
        f64 = T <= M.MOE_ROUTER_F64_MAX_T
        nb = T * E * (8 if f64 else 4)
        res["fast"] = ws[off:off + nb].view(torch.float64 if f64 else torch.float32).reshape(T, E).cpu().numpy()
    return res


def _ranks(x_bits, W, b):
    """fp64 logits by a plain matrix product: only used to choose rows to edit."""
    xf = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    lg = xf @ W.astype(np.float64).T
    if b is not None:
        lg = lg + b
    return lg


def _tie_workload(T=256):
    """E = 512, H = 2048: rows edited so that exact ties and 1-ulp near ties
    fall inside chosen tokens' top 10 and on their 10th / 11th boundary."""
    cfg = S.config("prefill", T=T, seed=31)
    x = S.gen_x(cfg)
    W = S.gen_router(cfg)
    W[:8] *= 3.0                                   # hot rows: in most tokens' top 10
    W[1] = W[0]                                    # exact tie, every token
    W[3] = W[2]
    W[3, 17] = np.nextafter(W[2, 17], np.float32(np.inf))    # 1-ulp near tie
    W[5] = W[4]
    W[5, 100] = np.nextafter(W[4, 100], np.float32(-np.inf))
    x[0] = 0                                       # all logits 0: the 10 lowest indices
    big = (x[1].astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** 20)
    x[1] = S.f32_to_bf16_bits(big)                 # huge norm, exact power-of-two scaling
    edited = set(range(8))
    boundary = []
    for t in range(2, 40, 3):                      # ties exactly on the 10th / 11th boundary
        lg = _ranks(x, W, None)[t]
        order = np.lexsort((np.arange(cfg.E), -lg))
        e10, e11 = int(order[9]), int(order[10])
        if e10 in edited or e11 in edited:
            continue
        xf = (x[t].astype(np.uint32) << 16).view(np.float32)
        W[e11] = W[e10]
        if len(boundary) % 2:                      # every other one: 1 ulp apart on a nonzero x_h
            h = int(np.argmax(np.abs(xf)))
            W[e11, h] = np.nextafter(W[e10, h], np.float32(np.inf) if len(boundary) % 4 == 1 else
                                     np.float32(-np.inf))
        edited.update((e10, e11))
        boundary.append((t, e10, e11))
    return cfg, x, W, boundary


@pytest.mark.parametrize("T", [64, 256])  # fp64 tensor-core router; bf16-plane tensor-core router
def test_chunk_router_exact_and_near_ties(cuda_ok, T):
    cfg, x, W, boundary = _tie_workload(T)
    k, E = cfg.top_k, cfg.E
    assert len(boundary) >= 6
    res = _route(x, W, None, k)
    lg = O.router_logits(x, W, None)
    idx, w = O.topk(lg, k)
    check_routing(res, idx, w, E)
    assert res["topk_idx"][0].tolist() == list(range(10))
    assert np.allclose(res["topk_w"][0], 0.1, atol=1e-7)
    # the exact ties put the lower index first wherever both rows are selected
    for t in range(cfg.T):
        row = res["topk_idx"][t].tolist()
        if 0 in row and 1 in row:
            assert row.index(0) + 1 == row.index(1)
    # every constructed boundary tie was decided as the fp64 definition decides it
    for t, e10, e11 in boundary:
        assert (e10 in idx[t]) == (e10 in res["topk_idx"][t]) and (e11 in idx[t]) == (e11 in res["topk_idx"][t])


@pytest.mark.parametrize("T", [64, 256])
def test_chunk_router_ties_through_the_layer(cuda_ok, T):
    """The same edited router in a full prefill call: routing of all tokens,
    outputs of the edited tokens and a sample."""
    import torch
    cfg, x, W, boundary = _tie_workload(T)
    wl = Workload(cfg, device_arena=True)
    wl.W_host[0] = W
    wl.W[0] = torch.from_numpy(W).cuda()
    out, res = run_layer(wl, 0, x, prefill=True)
    lg = O.router_logits(x, W, None)
    idx, w = O.topk(lg, cfg.top_k)
    check_routing(res, idx, w, cfg.E)
    toks = sorted(t for t in {0, 1, *[t for t, _, _ in boundary], 50, 100, 200, T - 1} if t < T)
    ref = wl.oracle_layer(0, x, tokens=np.array(toks, np.int32))
    assert_out_close(out, ref["out_f64"], rows=toks)


@pytest.mark.parametrize("name,layer", [("prefill", 0), ("prefill_stack", 5)])
def test_chunk_router_bound_slack(cuda_ok, name, layer):
    """|fast logit - fp64 logit| against the bound the certification uses,
    gamma * (||x_t|| ||W_r[e]|| + |b_e|), over every (token, expert) of a full
    8,192-token chunk: the bound must hold everywhere (ratio < 1); the ratio
    and the error in units of 2^-23 sum |x w| are printed as the measured slack."""
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config(name)
    x = S.gen_x(cfg)
    W = S.gen_router(cfg, layer)
    b = S.gen_bias(cfg, layer)
    res = _route(x, W, b, cfg.top_k, want_logits=True)
    exact = O.router_logits(x, W, b)
    gamma = M.moe_router_gamma(cfg.T, cfg.E, cfg.H)
    assert 0 < gamma < 1e-4
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Wf = W.astype(np.float64)
    babs = np.zeros(cfg.E) if b is None else np.abs(b.astype(np.float64))
    bound = gamma * (np.linalg.norm(xf, axis=1)[:, None] * np.linalg.norm(Wf, axis=1)[None, :] + babs[None, :])
    err = np.abs(res["fast"].astype(np.float64) - exact)
    ratio = float((err / bound).max())
    ulps = float((err / (2.0 ** -23 * (np.abs(xf) @ np.abs(Wf).T + babs[None, :]))).max())
    print(f"\n[router bound slack] {name}: max |fast - exact| / bound = {ratio:.4f}; "
          f"max error = {ulps:.3f} x 2^-23 sum|x w|; gamma = {gamma:.3e}")
    assert ratio < 1.0
    idx, w = O.topk(exact, cfg.top_k)
    check_routing(res, idx, w, cfg.E)


@pytest.mark.parametrize("name,layer,T", [("prefill", 0, 128), ("prefill_stack", 5, 100)])
def test_short_chunk_router_bound_slack(cuda_ok, name, layer, T):
    """The fp64 tensor-core logits of short chunks against the fp64 definition:
    |fast - exact| <= gamma (||x_t|| ||W_r[e]|| + |b_e|) for every (token,
    expert), gamma = moe_router_gamma's gamma_(H+32); the ratio is printed as
    the measured slack.  The routing is the definition's."""
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config(name, T=T)
    x = S.gen_x(cfg)
    W = S.gen_router(cfg, layer)
    b = S.gen_bias(cfg, layer)
    res = _route(x, W, b, cfg.top_k, want_logits=True)
    exact = O.router_logits(x, W, b)
    gamma = M.moe_router_gamma(T, cfg.E, cfg.H)
    assert 0 < gamma < 1e-12
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Wf = W.astype(np.float64)
    babs = np.zeros(cfg.E) if b is None else np.abs(b.astype(np.float64))
    bound = gamma * (np.linalg.norm(xf, axis=1)[:, None] * np.linalg.norm(Wf, axis=1)[None, :] + babs[None, :])
    err = np.abs(res["fast"] - exact)
    ratio = float((err / bound).max())
    print(f"\n[short-chunk router bound slack] {name}: max |fast - exact| / bound = {ratio:.2e}; gamma = {gamma:.3e}")
    assert ratio < 1.0
    idx, w = O.topk(exact, cfg.top_k)
    check_routing(res, idx, w, cfg.E)


def test_route_histogram_entry_point(cuda_ok):
    """moe_route_histogram adds each call's per-expert pair counts to its layer's
    row of a persistent histogram, bit-exact against the oracle's counts."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config("decode_stack")
    L, E, k = 3, cfg.E, cfg.top_k
    hist = torch.zeros((L, E), dtype=torch.int32, device="cuda")
    ref = np.zeros((L, E), np.uint32)
    calls = [(0, 5, 0), (2, 5, 1), (0, 1, 2), (1, 300, 3), (2, 8, 4), (0, 300, 5)]
    for layer, T, off in calls:
        x = S.gen_x(cfg, T, stream_offset=off)
        W = S.gen_router(cfg, layer)
        b = S.gen_bias(cfg, layer)
        res = _route(x, W, b, k)
        offs = torch.from_numpy(res["expert_offsets"]).cuda()
        M.moe_route_histogram(offs, E, L, layer, hist)
        idx, _ = O.topk(O.router_logits(x, W, b), k)
        counts, *_ = O.permutation(idx, E)
        O.hist_add(counts, layer, ref)
    torch.cuda.synchronize()
    got = hist.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref)
    assert got.sum() == k * sum(T for _, T, _ in calls)


def test_profile_from_device_histogram(cuda_ok):
    """The expert-profile pipeline on the device: routing counts of 3 windows
    per layer of the 48 x 256 stack accumulated by moe_route_histogram, ranked
    by moe_rank_experts and written as STRP v1 - byte-identical to the
    oracle's file from its own counts."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    from oracle import profile as OP
    cfg = S.config("decode_stack")
    L, E, k = cfg.L, cfg.E, cfg.top_k
    hist = torch.zeros((L, E), dtype=torch.int32, device="cuda")
    ref = np.zeros((L, E), np.uint32)
    for layer in range(L):
        W, b = S.gen_router(cfg, layer), S.gen_bias(cfg, layer)
        for off in range(3):
            x = S.gen_x(cfg, 5, stream_offset=200 + 3 * layer + off)
            res = _route(x, W, b, k)
            M.moe_route_histogram(torch.from_numpy(res["expert_offsets"]).cuda(), E, L, layer, hist)
            idx, _ = O.topk(O.router_logits(x, W, b), k)
            counts, *_ = O.permutation(idx, E)
            O.hist_add(counts, layer, ref)
    torch.cuda.synchronize()
    got = hist.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref)
    pairs = M.moe_rank_experts(got)
    assert M.moe_profile_write(pairs, L, E) == OP.profile_bytes(O.rank(ref).tolist(), L, E)
