"""Expert parallelism on one GPU: the G ranks' library calls run one after the
other on the same device (no collective; the test sums the partials itself).
Each rank's moe_forward_partial sees the whole token set with the experts it
does not hold marked MOE_SLOT_REMOTE; the partials' sum finished by
moe_finish_rows must be the layer (oracle, residual included), the routing
must be the full routing on every rank, and no rank may report a missing slot.
With every expert local the partial is the residual-free layer before its
rounding, bit for bit."""
import numpy as np
import pytest

import moe_synth as S
from helpers import Workload, assert_out_close, bits_to_f32, route_buffers, run_layer

pytestmark = pytest.mark.gpu


def _partial(wl, table, x, prefill, route_out=None):
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = wl.cfg
    T = x.shape[0]
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    part = torch.empty((T, cfg.H), dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_workspace_bytes(T, cfg.E, cfg.top_k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    M.moe_forward_partial(prefill, wl.desc, wl.arena, table, cfg.L, 0, xt, wl.W[0], wl.b[0], cfg.top_k, part,
                          route_out=route_out, ws=ws)
    torch.cuda.synchronize()
    st = M.moe_last_device_error()
    assert st == 0, f"device status {st}: {M.strerror(st)}"
    return part


@pytest.mark.parametrize("case,G", [("fused_decode", 2), ("fused_decode", 3), ("multi_kernel_decode", 2),
                                    ("prefill_small", 2), ("prefill_model_shape", 4)])
def test_expert_parallel_partials_sum_to_the_layer(cuda_ok, case, G):
    import torch
    import quantized_expert_ffn_top10_b200 as M
    from quantized_expert_ffn_top10_b200.ep import ep_slot_table
    if case == "fused_decode":
        cfg, prefill = S.config("decode", seed=91), False
    elif case == "multi_kernel_decode":
        cfg, prefill = S.config("tiny", E=32, top_k=10, H=256, I=96, T=6, bits=(2, 4, 2), router_std=None,
                                seed=92), False
    elif case == "prefill_small":
        cfg, prefill = S.config("tiny", E=16, top_k=4, H=256, I=128, T=40, seed=93), True
    else:
        cfg, prefill = S.config("prefill", T=64, seed=94), True
    wl = Workload(cfg)
    x = wl.x_host()
    T, k, E = x.shape[0], cfg.top_k, cfg.E
    total = torch.zeros((T, cfg.H), dtype=torch.float32, device="cuda")
    routing = []
    for r in range(G):
        table = ep_slot_table(wl.slot_table, cfg.L, E, r, G)
        ro = route_buffers(T, k, E)
        total += _partial(wl, table, x, prefill, route_out=ro)
        routing.append(ro["topk_idx"].cpu().numpy())
    for r in range(1, G):
        assert np.array_equal(routing[r], routing[0]), "every rank routes every token the same way"
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.zeros_like(xt)
    M.moe_finish_rows(xt, total, True, out)
    torch.cuda.synchronize()
    ref = wl.oracle_layer(0, x)
    assert np.array_equal(routing[0].reshape(T, k), ref["idx"])
    assert_out_close(out.cpu().numpy().view(np.uint16), ref["out_f64"])


@pytest.mark.parametrize("case", ["fused_decode", "multi_kernel_decode", "prefill_small"])
def test_all_local_partial_is_the_unrounded_layer(cuda_ok, case):
    if case == "fused_decode":
        cfg, prefill = S.config("decode", seed=95), False
    elif case == "multi_kernel_decode":
        cfg, prefill = S.config("tiny", E=32, top_k=10, H=256, I=96, T=6, bits=(2, 4, 2), router_std=None,
                                seed=96), False
    else:
        cfg, prefill = S.config("tiny", E=16, top_k=4, H=256, I=128, T=40, seed=97), True
    wl = Workload(cfg)
    x = wl.x_host()
    part = _partial(wl, wl.slot_table, x, prefill).cpu().numpy()
    out, _ = run_layer(wl, 0, x, prefill=prefill, residual=False)
    rounded = (part.view(np.uint32) + 0x7FFF + ((part.view(np.uint32) >> 16) & 1)) >> 16  # RNE to bf16
    assert np.array_equal(rounded.astype(np.uint16), out), "the partial is the combine before its rounding"
    assert np.all(np.isfinite(bits_to_f32(out)))


def test_finish_rows_with_steering_matches_the_steered_layer(cuda_ok):
    """moe_finish_rows(x, partial, steer) equals the forward with the same
    steering vector (one token block, the same fp32 arithmetic)."""
    import torch
    import quantized_expert_ffn_top10_b200 as M
    cfg = S.config("decode", seed=98)
    wl = Workload(cfg)
    x = wl.x_host()
    rng = np.random.default_rng(5)
    v = rng.standard_normal(cfg.H).astype(np.float32)
    v /= np.float32(np.linalg.norm(v))
    vt = torch.from_numpy(v).cuda()
    part = _partial(wl, wl.slot_table, x, False)
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.zeros_like(xt)
    M.moe_finish_rows(xt, part, True, out, steer=vt)
    torch.cuda.synchronize()
    ref, _ = run_layer(wl, 0, x, prefill=False, residual=True, steer=v)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)


@pytest.mark.parametrize("case,max_chunk", [("fused_decode", 8192), ("prefill_small", 16)])
def test_forward_ep_on_one_nccl_rank_is_the_layer(cuda_ok, case, max_chunk):
    """moe_forward_ep through a one-rank NCCL group: the gather and the
    reduce-scatter are identities, so the call is the layer (oracle), also when
    the gathered rows go through the library in several chunks (40 tokens in
    chunks of 16, 16 and 8: the chunk path twice, then the decode path)."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    import quantized_expert_ffn_top10_b200 as M
    from quantized_expert_ffn_top10_b200.ep import ep_slot_table, moe_forward_ep
    if case == "fused_decode":
        cfg = S.config("decode", seed=99)
    else:
        cfg = S.config("tiny", E=16, top_k=4, H=256, I=128, T=40, seed=100)
    wl = Workload(cfg)
    x = wl.x_host()
    T = x.shape[0]
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        table = ep_slot_table(wl.slot_table, cfg.L, cfg.E, 0, 1)
        xt = torch.from_numpy(x.view(np.int16)).cuda()
        out = torch.zeros_like(xt)
        ws = torch.empty(M.moe_workspace_bytes(min(T, max_chunk), cfg.E, cfg.top_k, cfg.H, cfg.I),
                         dtype=torch.uint8, device="cuda")
        moe_forward_ep(wl.desc, wl.arena, table, cfg.L, 0, xt, wl.W[0], wl.b[0], cfg.top_k, True, out, ws=ws,
                       max_chunk=max_chunk)
        torch.cuda.synchronize()
        st = M.moe_last_device_error()
        assert st == 0, f"device status {st}: {M.strerror(st)}"
    finally:
        dist.destroy_process_group()
    ref = wl.oracle_layer(0, x)
    assert_out_close(out.cpu().numpy().view(np.uint16), ref["out_f64"])
