"""The steering projection h - (h . v) v ("Coder benchmark record" page,
steering vector section) on every path: the fused decode kernel (rows leave it
in fp32 and a second kernel projects them), the multi-kernel decode combine,
and the prefill combine; against the oracle's layer with the same v."""
import numpy as np
import pytest

import moe_synth as S
from helpers import Workload, assert_out_close, check_routing, run_layer

pytestmark = pytest.mark.gpu


def _unit(H, seed):
    v = np.random.default_rng(seed).standard_normal(H)
    return (v / np.linalg.norm(v)).astype(np.float32)


@pytest.mark.parametrize("case", ["fused_decode", "decode_full", "multi_kernel_decode", "prefill_small",
                                  "prefill_no_residual"])
def test_steered_layer_matches_oracle(cuda_ok, case):
    residual = case != "prefill_no_residual"
    if case == "fused_decode":
        cfg, prefill = S.config("tiny", E=16, top_k=4, H=1024, I=256, T=5, router_std=None, seed=81), False
    elif case == "decode_full":
        cfg, prefill = S.config("decode", seed=82), False
    elif case == "multi_kernel_decode":
        cfg, prefill = S.config("tiny", E=32, top_k=10, H=256, I=96, T=6, bits=(2, 4, 2), zipf_s=1.1,
                                router_std=None, seed=83), False
    else:
        cfg, prefill = S.config("tiny", E=16, top_k=4, H=256, I=128, T=70, seed=84), True
    wl = Workload(cfg)
    x = wl.x_host()
    v = _unit(cfg.H, 85)
    out, res = run_layer(wl, 0, x, prefill=prefill, residual=residual, steer=v)
    ref = wl.oracle_layer(0, x, residual=residual, steer=v)
    check_routing(res, ref["idx"], ref["w"], cfg.E)
    assert_out_close(out, ref["out_f64"])
    g = (out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = ref["out_f64"]
    # the projected rows are orthogonal to v up to their bf16 rounding
    assert np.all(np.abs(g @ v.astype(np.float64)) <= 4 * 2.0 ** -8 * np.abs(g) @ np.abs(v.astype(np.float64)) + 1e-6)
    # and steering changed them: the unsteered layer differs along v
    plain, _ = run_layer(wl, 0, x, prefill=prefill, residual=residual)
    p = (plain.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.abs(p @ v).max() > 10 * np.abs(r @ v).max()
