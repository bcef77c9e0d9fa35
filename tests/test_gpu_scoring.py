"""GPU parity of the router scoring rules in which the per-expert bias steers
only the selection (selection-only-bias softmax, sigmoid), against the CPU
oracle: every router implementation, lane layouts of 2 to 32 experts per
lane, k above 32 (slot values kept in a second register per lane), one
token with k = 1, no bias, and the whole layer under every tile policy
that routes (the few-token one-launch router and the one-launch layer
included).  Routing ids and the permutation must match bit for bit; weights
within W_ABS; y within the layer's tolerance."""
import numpy as np
import pytest

import oracle
import routed_expert_ffn_prefix_b200 as moe
import synth
from synth import Config

from helpers import W_ABS, assert_close_output, dev_bf16, dev_f32, host_f64

pytestmark = pytest.mark.gpu

SCORINGS = {"softmax_select_bias": moe.SCORE_SOFTMAX_SELECT_BIAS, "sigmoid": moe.SCORE_SIGMOID}

# bias scale s of zipf:s (bias_e = -s ln(e+1)) comparable to the spread of
# the sigmoid scores, so the bias changes some selections but not all
CASES = {
    c.name: c for c in [
        Config("sc_e64", T=200, H=512, E=64, I=256, k=6, bias="zipf:0.05"),      # 2 experts per lane
        Config("sc_e256", T=40, H=1024, E=256, I=128, k=8, bias="zipf:0.05"),    # 16-byte lane layout
        Config("sc_e40_few", T=9, H=512, E=40, I=128, k=5, bias="zipf:0.3"),     # few tokens, E % 8 == 0
        Config("sc_k40", T=20, H=256, E=128, I=128, k=40, bias="zipf:0.05"),     # k > 32
        Config("sc_k36_few", T=3, H=256, E=64, I=128, k=36, bias="zipf:0.05"),   # k > 32, few tokens
        Config("sc_one", T=1, H=512, E=32, I=256, k=1, bias="zipf:0.05"),        # one token, k = 1
        Config("sc_nobias", T=64, H=256, E=16, I=128, k=3),                      # no bias
        Config("sc_e36", T=50, H=256, E=36, I=128, k=4, bias="zipf:0.1"),        # E % 8 != 0
        Config("sc_fused", T=4, H=512, E=16, I=256, k=4, I_s=256, bias="zipf:0.05"),
    ]
}
ROUTE_ONLY = {"sc_e1024": Config("sc_e1024", T=24, H=256, E=1024, I=128, k=8, bias="zipf:0.02")}
# k > 32 needs k adjacent gaps per token among closely spaced sigmoid
# scores; these cases take a 2e-5 gap, still ~100x the fp32 error of a
# 256-term logit (~1e-7) scaled by the sigmoid's slope (<= 1/4).
CASE_GAP = {"sc_k40": 2e-5, "sc_k36_few": 2e-5}

_cache = {}


def case(name, scoring):
    key = (name, scoring)
    if key not in _cache:
        cfg = CASES.get(name) or ROUTE_ONLY[name]
        inp = synth.make_inputs(cfg)
        oracle.enforce_logit_gap(inp, gap=CASE_GAP.get(name), scoring=scoring)
        if name in ROUTE_ONLY:
            l = oracle.router_logits(inp.x, inp.w_router, None)
            ids, w = oracle.route_scored(l, inp.bias, cfg.k, scoring)
            ref = dict(ids=ids, w=w)
        else:
            ref = oracle.layer_forward(inp.x, inp.w_router, inp.bias, inp.w_gate_up, inp.w_down, cfg.k,
                                       inp.w_sh_gate_up, inp.w_sh_down, scoring=scoring)
        _cache[key] = (cfg, inp, ref)
    return _cache[key]


def assert_ok(ws):
    st = moe.device_status(ws)
    assert st == 0, moe.STATUS.get(st, st)


def check_weights(w, ref_w, k):
    wg = host_f64(w)
    assert np.abs(wg - ref_w).max() <= W_ABS
    assert np.abs(wg.sum(1) - 1).max() <= 1e-6
    if k == 1:
        assert np.all(wg == 1.0)


@pytest.mark.parametrize("impl", [moe.ROUTER_FMA, moe.ROUTER_TC, moe.ROUTER_SMALL])
@pytest.mark.parametrize("scoring", list(SCORINGS))
@pytest.mark.parametrize("name", list(CASES) + list(ROUTE_ONLY))
def test_route_scoring_matches_oracle(name, scoring, impl):
    cfg, inp, ref = case(name, scoring)
    if impl == moe.ROUTER_TC and cfg.E % 8:
        pytest.skip("tensor-core router needs E % 8 == 0")
    if impl == moe.ROUTER_SMALL and (cfg.T > 16 or cfg.E % 4):
        pytest.skip("few-token router needs T <= 16 and E % 4 == 0")
    ws = moe.alloc_workspace(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    bias = None if inp.bias is None else dev_f32(inp.bias)
    ids, w = moe.route(dev_bf16(inp.x), dev_f32(inp.w_router), bias, cfg.k, ws, impl=impl,
                       scoring=SCORINGS[scoring])
    assert_ok(ws)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref["ids"])
    check_weights(w, ref["w"], cfg.k)


def _tile_policies(cfg):
    out = [moe.TILES_AUTO, moe.TILES_SMALL]
    if cfg.T <= 16 and cfg.E % 4 == 0 and cfg.I_s == 0:  # the persistent one-launch layer
        out.append(moe.TILES_PERSISTENT)
    return out


@pytest.mark.parametrize("scoring", list(SCORINGS))
@pytest.mark.parametrize("name", list(CASES))
def test_forward_scoring_matches_oracle(name, scoring):
    cfg, inp, ref = case(name, scoring)
    import torch
    bias = None if inp.bias is None else dev_f32(inp.bias)
    sh = (dev_bf16(inp.w_sh_gate_up), dev_bf16(inp.w_sh_down)) if cfg.I_s else (None, None)
    x, wr, wgu, wd = dev_bf16(inp.x), dev_f32(inp.w_router), dev_bf16(inp.w_gate_up), dev_bf16(inp.w_down)
    for tiles in _tile_policies(cfg):
        ws = moe.alloc_workspace(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
        y = moe.forward(x, wr, bias, wgu, wd, cfg.k, ws, *sh, tiles=tiles, scoring=SCORINGS[scoring])
        torch.cuda.synchronize()
        assert_ok(ws)
        view = moe.workspace_view(ws, cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
        np.testing.assert_array_equal(view["topk_ids"].cpu().numpy(), ref["ids"], err_msg=f"tiles={tiles}")
        np.testing.assert_array_equal(view["sorted_token_ids"].cpu().numpy(), ref["sorted_token_ids"])
        np.testing.assert_array_equal(view["inv_perm"].cpu().numpy(), ref["inv_perm"])
        check_weights(view["topk_w"], ref["w"], cfg.k)
        assert_close_output(host_f64(y), ref["y"], f"y (tiles={tiles})")


def test_bias_changes_selection_under_both_rules():
    """The cases exercise what they claim: with the bias, selections differ
    from the unbiased ones for some tokens, and sigmoid weights differ from
    selection-only-bias softmax weights."""
    cfg, inp, ref_sig = case("sc_e64", "sigmoid")
    l = oracle.router_logits(inp.x, inp.w_router, None)
    ids_nb, _ = oracle.route_scored(l, None, cfg.k, "sigmoid")
    assert (ids_nb != ref_sig["ids"]).any(axis=1).mean() > 0.05
    ids_sb, w_sb = oracle.route_scored(l, inp.bias, cfg.k, "softmax_select_bias")
    assert np.abs(w_sb - oracle.route_scored(l, inp.bias, cfg.k, "sigmoid")[1]).max() > 1e-2
