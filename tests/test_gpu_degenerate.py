"""Non-finite inputs, the layer's degenerate case: a token whose hidden state
holds a NaN (every logit NaN), one holding +inf (logits of +-inf and NaN), and
a router row holding a NaN (that expert's logit NaN for every token).  The
selection order is total (a NaN logit ranks as -inf, ties by the lower index),
so every path must return k valid, distinct experts per token, exactly the
oracle's, never touch memory outside its buffers, and produce NaN outputs only
where the oracle does."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O
from helpers import OUT_RTOL, Workload, assert_out_close, route_buffers

pytestmark = pytest.mark.gpu


def _poison(x, W):
    x = x.copy()
    W = W.copy()
    x[0, 7] = 0x7FC0                   # NaN
    x[1, 3] = 0x7F80                   # +inf
    W[3, 11] = np.float32("nan")       # expert 3: NaN logit for every token
    return x, W


def _check(out_bits, res, x, W, b, wl, layer, k, E):
    lg = O.router_logits(x, W, b)
    idx, w = O.topk(lg, k)
    got = res["topk_idx"]
    assert np.array_equal(got, idx), "top-k indices differ"
    assert all(len(set(r.tolist())) == k and r.min() >= 0 and r.max() < E for r in got)
    _, offsets, perm, _ = O.permutation(idx, E)
    assert np.array_equal(res["expert_offsets"], offsets) and np.array_equal(res["perm"], perm)
    assert np.array_equal(np.isnan(res["topk_w"]), np.isnan(w))
    fin = ~np.isnan(w)
    assert np.max(np.abs(res["topk_w"][fin] - w[fin])) <= 1e-4
    assert not np.isin(3, idx[2:]), "a NaN logit must rank last"
    wl.W_host[layer] = W
    ref = wl.oracle_layer(layer, x)
    g = (out_bits.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(np.isnan(g), np.isnan(ref["out_f64"]))
    ok_rows = [t for t in range(x.shape[0]) if np.all(np.isfinite(ref["out_f64"][t]))]
    assert len(ok_rows) >= x.shape[0] - 2
    assert_out_close(out_bits, ref["out_f64"], rows=ok_rows, tol=OUT_RTOL)


def _run(wl, x, W, prefill):
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = wl.cfg
    T = x.shape[0]
    Wd = torch.from_numpy(W).cuda()
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.zeros_like(xt)
    ws = torch.empty(M.moe_workspace_bytes(T, cfg.E, cfg.top_k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    ro = route_buffers(T, cfg.top_k, cfg.E)
    fn = M.moe_forward_prefill if prefill else M.moe_forward_decode
    fn(wl.desc, wl.arena, wl.slot_table, cfg.L, 0, xt, Wd, wl.b[0], cfg.top_k, True, out, route_out=ro, ws=ws)
    torch.cuda.synchronize()
    st = M.moe_last_device_error()
    assert st == 0, f"device status {st}: {M.strerror(st)}"
    res = {key: v.cpu().numpy() for key, v in ro.items()}
    res["topk_idx"] = res["topk_idx"].reshape(T, cfg.top_k)
    res["topk_w"] = res["topk_w"].reshape(T, cfg.top_k)
    return out.cpu().numpy().view(np.uint16), res


@pytest.mark.parametrize("case", ["fused_decode", "multi_kernel_decode", "prefill_small", "prefill_tc_router"])
def test_non_finite_inputs(cuda_ok, case):
    if case == "fused_decode":
        cfg, prefill = S.config("tiny", E=16, top_k=4, H=1024, I=256, T=4, router_std=None, seed=51), False
    elif case == "multi_kernel_decode":
        cfg, prefill = S.config("tiny", E=32, top_k=10, H=256, I=96, T=6, bits=(2, 4, 2), zipf_s=1.1,
                                router_std=None, seed=52), False
    elif case == "prefill_small":
        cfg, prefill = S.config("tiny", E=16, top_k=4, H=256, I=128, T=40, seed=53), True
    else:
        cfg, prefill = S.config("prefill", T=256, seed=54), True
    wl = Workload(cfg, device_arena=case == "prefill_tc_router")
    x, W = _poison(wl.x_host(), wl.W_host[0])
    out, res = _run(wl, x, W, prefill)
    _check(out, res, x, W, wl.b_host[0], wl, 0, cfg.top_k, cfg.E)
