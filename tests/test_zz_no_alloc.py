"""moe_route_static, the routing entry point that runs on the library's fixed
device scratch instead of a caller workspace, against moe_route on the same
inputs.  The file name sorts last so that pytest collects it after every other
test: it must pass both in a fresh process and after the rest of the suite
has used the device."""
import numpy as np
import pytest

import moe_synth as S
import oracle as O
import quantized_expert_ffn_top10_b200 as M
from helpers import W_ATOL, check_routing, route_buffers


def _inputs(cfg, T, offset):
    import torch
    x = torch.from_numpy(S.gen_x(cfg, T=T, stream_offset=offset).view(np.int16)).cuda()
    W = torch.from_numpy(S.gen_router(cfg)).cuda()
    b = S.gen_bias(cfg)
    return x, W, (torch.from_numpy(b).cuda() if b is not None else None)


def _route(fn_static, x, W, b, k, E):
    import torch
    T, H = x.shape
    ro = route_buffers(T, k, E)
    if fn_static:
        M.moe_route_static(x, W, b, k, ro["topk_idx"], ro["topk_w"], ro["expert_offsets"], ro["perm"])
    else:
        ws = torch.empty(M.moe_workspace_bytes(T, E, k, H, 32), dtype=torch.uint8, device="cuda")
        M.moe_route(x, W, b, k, ro["topk_idx"], ro["topk_w"], ro["expert_offsets"], ro["perm"], ws)
    torch.cuda.synchronize()
    st = M.moe_last_device_error()
    assert st == 0, f"device status {st}: {M.strerror(st)}"
    res = {key: v.cpu().numpy() for key, v in ro.items()}
    res["topk_idx"] = res["topk_idx"].reshape(T, k)
    res["topk_w"] = res["topk_w"].reshape(T, k)
    return res


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", [("decode", 5), ("decode", 1), ("decode_stack", 8), ("tiny", 4)])
def test_static_route_matches_workspace_route(cuda_ok, name, T):
    cfg = S.config(name)
    k, E = cfg.top_k, cfg.E
    for call in range(2):  # two calls in a row on the same scratch, different tokens
        x, W, b = _inputs(cfg, T, offset=call)
        got = _route(True, x, W, b, k, E)
        ref = _route(False, x, W, b, k, E)
        assert np.array_equal(got["topk_idx"], ref["topk_idx"]), f"call {call}: top-k indices differ"
        assert np.array_equal(got["expert_offsets"], ref["expert_offsets"]), f"call {call}: offsets differ"
        assert np.array_equal(got["perm"], ref["perm"]), f"call {call}: permutation differs"
        assert np.max(np.abs(got["topk_w"] - ref["topk_w"])) <= W_ATOL, f"call {call}: gate weights differ"
        # and both against the oracle's routing
        xb = x.cpu().numpy().view(np.uint16)
        logits = O.router_logits(xb, W.cpu().numpy(), None if b is None else b.cpu().numpy())
        idx_ref, w_ref = O.topk(logits, k)
        check_routing(got, idx_ref, w_ref, E)


@pytest.mark.gpu
def test_static_route_rejects_T_beyond_limit(cuda_ok):
    import torch
    cfg = S.config("decode")
    T = M.MOE_ROUTE_STATIC_MAX_T + 1
    x, W, b = _inputs(cfg, T, offset=0)
    ro = route_buffers(T, cfg.top_k, cfg.E)
    rc = M.moe_route_static(x, W, b, cfg.top_k, ro["topk_idx"], ro["topk_w"], ro["expert_offsets"], ro["perm"],
                            raise_on_error=False)
    assert rc == M.MOE_ERR_STATIC
    torch.cuda.synchronize()
    assert int((ro["topk_idx"] != -1).sum()) == 0  # nothing was launched


_FRESH = r"""
import sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import moe_synth as S
import quantized_expert_ffn_top10_b200 as M
cfg = S.config("decode_stack")
T, k, E = 8, cfg.top_k, cfg.E
outs = []
for call in range(2):
    x = torch.from_numpy(S.gen_x(cfg, T=T, stream_offset=call).view(np.int16)).cuda()
    W = torch.from_numpy(S.gen_router(cfg)).cuda()
    b = torch.from_numpy(S.gen_bias(cfg)).cuda()
    res = []
    for static in (True, False):  # the no-workspace call first: nothing else has run in this process
        idx = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros(T * k, dtype=torch.float32, device="cuda")
        off = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
        perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        if static:
            M.moe_route_static(x, W, b, k, idx, w, off, perm)
        else:
            ws = torch.empty(M.moe_workspace_bytes(T, E, k, cfg.H, 32), dtype=torch.uint8, device="cuda")
            M.moe_route(x, W, b, k, idx, w, off, perm, ws)
        torch.cuda.synchronize()
        assert M.moe_last_device_error() == 0
        res.append([t.cpu().numpy() for t in (idx, w, off, perm)])
    (i1, w1, o1, p1), (i2, w2, o2, p2) = res
    assert np.array_equal(i1, i2) and np.array_equal(o1, o2) and np.array_equal(p1, p2)
    assert np.max(np.abs(w1 - w2)) <= 1e-4
print("fresh-process static route ok")
"""


@pytest.mark.gpu
def test_static_route_in_a_fresh_process(cuda_ok):
    """The same comparison in a new Python process whose first library call is
    moe_route_static (T = 8, the limit), so that the scratch address lookup
    runs with nothing initialised before it."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FRESH, root], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "fresh-process static route ok" in r.stdout
