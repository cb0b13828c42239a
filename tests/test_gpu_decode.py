"""Decode path (T <= 8) through the C ABI against the CPU oracle."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O
from helpers import Workload, assert_out_close, check_routing, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def decode_wl(cuda_ok):
    return Workload(S.config("decode"))


def _compare(wl, layer, x, prefill=False, tokens=None):
    out, res = run_layer(wl, layer, x, prefill=prefill)
    ref = wl.oracle_layer(layer, x)
    check_routing(res, ref["idx"], ref["w"], wl.cfg.E)
    rel = assert_out_close(out, ref["out_f64"])
    return out, res, ref, rel


def test_tiny_decode(cuda_ok):
    wl = Workload(S.config("tiny"))
    _compare(wl, 0, wl.x_host())


@pytest.mark.parametrize("T", [1, 5])
def test_decode_full_layer(decode_wl, T):
    wl = decode_wl
    x = S.gen_x(wl.cfg, T)
    _compare(wl, 0, x)


@pytest.mark.parametrize("T", [2, 8])
def test_decode_other_window_sizes(decode_wl, T):
    wl = decode_wl
    _compare(wl, 0, S.gen_x(wl.cfg, T, stream_offset=T))


def test_decode_mixed_bits_and_bias(cuda_ok):
    cfg = S.config("tiny", E=32, top_k=10, H=256, I=96, T=6, bits=(2, 4, 2), zipf_s=1.1, router_std=None)
    wl = Workload(cfg)
    _compare(wl, 0, wl.x_host())


def test_decode_exact_ties_pick_lower_index(cuda_ok):
    """Duplicate router rows give exactly equal logits: the lower index wins
    and its slot comes first; a zero token ties every expert."""
    import torch
    cfg = S.config("tiny", E=16, top_k=4, H=128, I=64, T=3)
    wl = Workload(cfg)
    W = wl.W_host[0].copy()
    W[9] = W[2]
    W[12] = W[2]
    W[5] = W[7]
    wl.W_host[0] = W
    wl.W[0] = torch.from_numpy(W).cuda()
    x = wl.x_host()
    x[2] = 0  # all logits 0: the k lowest indices, equal weights
    out, res, ref, _ = _compare(wl, 0, x)
    assert res["topk_idx"][2].tolist() == [0, 1, 2, 3]
    assert np.allclose(res["topk_w"][2], 0.25)
    assert res["n_rechecked"][0] >= 1


def test_decode_histogram_accumulates(decode_wl):
    import torch
    wl = decode_wl
    cfg = wl.cfg
    hist = torch.zeros((1, cfg.E), dtype=torch.int32, device="cuda")
    ref = np.zeros((1, cfg.E), np.uint32)
    for i in range(3):
        x = S.gen_x(cfg, 5, stream_offset=10 + i)
        out, res = run_layer(wl, 0, x, prefill=False, hist=hist)
        counts, *_ = O.permutation(res["topk_idx"], cfg.E)
        O.hist_add(counts, 0, ref)
    got = hist.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref)
    assert got.sum() == 3 * 5 * cfg.top_k


def test_decode_missing_slot_contributes_zero(cuda_ok):
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config("tiny", E=16, top_k=4, H=128, I=64, T=3)
    wl = Workload(cfg)
    x = wl.x_host()
    ref = wl.oracle_layer(0, x)
    e_bad = int(ref["idx"][1, 0])
    table = wl.slot_table_host.copy()
    table[e_bad] = -1
    wl.slot_table = torch.from_numpy(table).cuda()
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.zeros_like(xt)
    ws = torch.empty(M.moe_workspace_bytes(3, cfg.E, cfg.top_k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    M.moe_forward_decode(wl.desc, wl.arena, wl.slot_table, 1, 0, xt, wl.W[0], None, cfg.top_k, True, out, ws=ws)
    assert M.moe_last_device_error() == M.MOE_ERR_SLOT
    assert M.moe_last_device_error() == 0  # read clears
    d, mini, t2 = wl.mini_arena(0, np.unique(ref["idx"]))
    t2[e_bad] = -1
    r2 = O.moe_layer(d, mini, t2, 1, 0, x, wl.W_host[0], None, cfg.top_k)
    assert r2["rc"] == O.ORC_ERR_SLOT
    assert_out_close(out.cpu().numpy().view(np.uint16), r2["out_f64"])


def test_decode_stack_teacher_forced(cuda_ok):
    """48 layers x 256 experts, 2/2/4-bit, Zipf bias: the oracle chains its own
    bf16 outputs; every layer of the library gets the oracle's input.  Each
    layer runs twice: with the residual (the chain) and without it, so that the
    MoE part, a small fraction of x in this stable chain, is checked on its own."""
    import torch
    cfg = S.config("decode_stack")
    wl = Workload(cfg)
    x = wl.x_host()
    hist = torch.zeros((cfg.L, cfg.E), dtype=torch.int32, device="cuda")
    ref_hist = np.zeros((cfg.L, cfg.E), np.uint32)
    distinct = []
    for layer in range(cfg.L):
        out, res = run_layer(wl, layer, x, prefill=False, hist=hist)
        moe, _ = run_layer(wl, layer, x, prefill=False, residual=False)
        ref = wl.oracle_layer(layer, x, residual=False)
        counts = check_routing(res, ref["idx"], ref["w"], cfg.E)
        O.hist_add(counts, layer, ref_hist)
        assert_out_close(moe, ref["out_f64"])
        xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert_out_close(out, xf + ref["out_f64"])  # the oracle's residual form: x + sum_j w_j y_j
        distinct.append(int((counts > 0).sum()))
        x = np.array([[O.double_to_bf16(v) for v in row] for row in xf + ref["out_f64"]], np.uint16)
    assert np.array_equal(hist.cpu().numpy().view(np.uint32), ref_hist)
    assert max(distinct) <= cfg.T * cfg.top_k


# ---------------------------------------------------------------- the fused (one-kernel) decode layer
# Windows whose gate and up share a bit width, with H % 256 == 0 (H % 512 at
# 2 bits), I % 256 == 0, W_d rows of one or two 128-byte boxes and a shared-
# memory plan that fits, take the persistent kernel; these cases pin it at
# sizes the oracle runs fast.  (2, 4, 4) takes the multi-kernel path.

@pytest.mark.parametrize("T,bits,zipf,I", [(1, (4, 4, 4), 0.0, 256), (3, (2, 2, 4), 1.1, 256),
                                           (8, (4, 4, 4), 1.1, 256), (5, (2, 2, 2), 0.0, 512),
                                           (5, (2, 4, 4), 0.0, 256)])
def test_fused_decode_small(cuda_ok, T, bits, zipf, I):
    cfg = S.config("tiny", E=16, top_k=4, H=1024, I=I, T=T, bits=bits, zipf_s=zipf, router_std=None, seed=21)
    wl = Workload(cfg)
    _compare(wl, 0, wl.x_host())


def test_fused_decode_ties_and_zero_token(cuda_ok):
    import torch
    cfg = S.config("tiny", E=16, top_k=4, H=1024, I=256, T=4, router_std=None, seed=22)
    wl = Workload(cfg)
    W = wl.W_host[0].copy()
    W[11] = W[3]
    W[14] = W[3]
    wl.W_host[0] = W
    wl.W[0] = torch.from_numpy(W).cuda()
    x = wl.x_host()
    x[1] = 0
    out, res, ref, _ = _compare(wl, 0, x)
    assert res["topk_idx"][1].tolist() == [0, 1, 2, 3]


def test_fused_decode_missing_slot(cuda_ok):
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config("tiny", E=16, top_k=4, H=1024, I=256, T=3, router_std=None, seed=23)
    wl = Workload(cfg)
    x = wl.x_host()
    ref = wl.oracle_layer(0, x)
    e_bad = int(ref["idx"][0, 1])
    table = wl.slot_table_host.copy()
    table[e_bad] = -1
    wl.slot_table = torch.from_numpy(table).cuda()
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.zeros_like(xt)
    ws = torch.empty(M.moe_workspace_bytes(3, cfg.E, cfg.top_k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    M.moe_forward_decode(wl.desc, wl.arena, wl.slot_table, 1, 0, xt, wl.W[0], None, cfg.top_k, True, out, ws=ws)
    assert M.moe_last_device_error() == M.MOE_ERR_SLOT
    d, mini, t2 = wl.mini_arena(0, np.unique(ref["idx"]))
    t2[e_bad] = -1
    r2 = O.moe_layer(d, mini, t2, 1, 0, x, wl.W_host[0], None, cfg.top_k)
    assert_out_close(out.cpu().numpy().view(np.uint16), r2["out_f64"])


def test_fused_decode_repeated_calls_are_identical(decode_wl):
    """Same inputs twice: bit-identical outputs (no order-dependent reductions)."""
    x = S.gen_x(decode_wl.cfg, 5, stream_offset=40)
    o1, r1 = run_layer(decode_wl, 0, x, prefill=False)
    o2, r2 = run_layer(decode_wl, 0, x, prefill=False)
    assert np.array_equal(o1, o2) and np.array_equal(r1["perm"], r2["perm"])


def test_fused_decode_wait_expiry_reports_timeout(cuda_ok):
    """A bounded wait that runs out: with the test hooks, the fused kernel's
    first grid barrier waits for an arrival that never comes and gives up
    after a few thousand polls.  At that barrier no CTA has a copy in flight
    or tensor memory allocated, so every CTA leaves cleanly; the call reports
    MOE_ERR_TIMEOUT at site 1, and the next normal call is correct."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config("tiny", E=16, top_k=4, H=1024, I=256, T=3, router_std=None, seed=24)
    wl = Workload(cfg)
    x = wl.x_host()
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.zeros_like(xt)
    ws = torch.empty(M.moe_workspace_bytes(3, cfg.E, cfg.top_k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    assert M.moe_last_device_error() == 0 and M.moe_timeout_site() == 0
    n0 = M.moe_launch_count()
    try:
        M.moe_debug_set(M.MOE_DBG_SPIN_LIMIT, 2000)
        M.moe_debug_set(M.MOE_DBG_BARRIER_EXTRA, 1)
        M.moe_forward_decode(wl.desc, wl.arena, wl.slot_table, 1, 0, xt, wl.W[0], None, cfg.top_k, True, out,
                             ws=ws)
        torch.cuda.synchronize()
    finally:
        M.moe_debug_set(M.MOE_DBG_SPIN_LIMIT, 0)
        M.moe_debug_set(M.MOE_DBG_BARRIER_EXTRA, 0)
    assert M.moe_launch_count() - n0 == 1, "the fused kernel (not the multi-kernel path) must have run"
    assert M.moe_last_device_error() == M.MOE_ERR_TIMEOUT
    site = M.moe_timeout_site()
    assert site // 1000000 == 1, f"timeout site {site}"
    assert M.moe_last_device_error() == 0 and M.moe_timeout_site() == 0  # both read-and-clear
    _compare(wl, 0, x)
