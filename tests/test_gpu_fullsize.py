"""Parity at the full sizes of the benchmark workloads, in the launch
configuration bench.py times (automatic tile and router choice).

Routing is checked on every token (ids, weights, counts, offsets, the
permutation and its inverse, bit for bit against the float64 oracle); the
SwiGLU rows h of every slot of a sample of tokens, and the layer output on
those tokens, which the oracle computes one by one: the
first and last token, tokens that use the most and the least loaded
expert, and a seeded random draw.  Expert weights for the oracle are drawn
again on the host from the same counter keys, one expert at a time."""
import numpy as np
import pytest

import oracle
import routed_expert_ffn_prefix_b200 as moe
import synth

from helpers import W_ABS, assert_close_output, dev_bf16, dev_f32, host_f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["qwen_decode_t512", "qwen_prefill_t8192", "ling_skewed_t4096",
        "sweep_decode_t1", "sweep_decode_t4", "sweep_decode_t16", "sweep_decode_t64"]

_weights = {}


def device_weights(cfg):
    import torch
    key = (cfg.H, cfg.E, cfg.I, cfg.seed, cfg.w_std)
    if key not in _weights:
        _weights.clear()
        torch.cuda.empty_cache()
        wgu = torch.empty(cfg.E, cfg.H, 2 * cfg.I, dtype=torch.bfloat16, device="cuda")
        wd = torch.empty(cfg.E, cfg.I, cfg.H, dtype=torch.bfloat16, device="cuda")
        chunk = 32
        for e0 in range(0, cfg.E, chunk):
            e1 = min(cfg.E, e0 + chunk)
            hgu = np.stack([synth.expert_gate_up(cfg, e) for e in range(e0, e1)])
            hd = np.stack([synth.expert_down(cfg, e) for e in range(e0, e1)])
            wgu[e0:e1].copy_(torch.from_numpy(hgu.view(np.int16)).view(torch.bfloat16))
            wd[e0:e1].copy_(torch.from_numpy(hd.view(np.int16)).view(torch.bfloat16))
        _weights[key] = (wgu, wd)
    return _weights[key]


def sample_tokens(cfg, counts, ids, n_random=12):
    rng = np.random.default_rng(1234)
    toks = {0, cfg.T - 1}
    hot, cold = int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
    for e in (hot, cold):
        hit = np.nonzero((ids == e).any(1))[0]
        toks.update(hit[:2].tolist())
    toks.update(rng.choice(cfg.T, size=min(n_random, cfg.T), replace=False).tolist())
    return np.array(sorted(toks))


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, experts=False)
    oracle.enforce_logit_gap(inp)
    wgu, wd = device_weights(cfg)
    sgu = None if inp.w_sh_gate_up is None else dev_bf16(inp.w_sh_gate_up)
    sd = None if inp.w_sh_down is None else dev_bf16(inp.w_sh_down)
    ws = moe.alloc_workspace(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    y = moe.forward(dev_bf16(inp.x), dev_f32(inp.w_router), None if inp.bias is None else dev_f32(inp.bias),
                    wgu, wd, cfg.k, ws, sgu, sd)
    st = moe.device_status(ws)
    assert st == 0, moe.STATUS.get(st, st)

    ids, w = oracle.topk_route(oracle.router_logits(inp.x, inp.w_router, inp.bias), cfg.k)
    counts, offsets, sids, inv = oracle.permute(ids, cfg.E)
    assert counts.sum() == cfg.T * cfg.k
    v = moe.workspace_view(ws, cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ids)
    assert np.abs(host_f64(v["topk_w"]) - w).max() <= W_ABS
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), sids)
    np.testing.assert_array_equal(v["inv_perm"].cpu().numpy(), inv)

    toks = sample_tokens(cfg, counts, ids)
    # h on every permuted row of the sampled tokens (one expert's rows at a time)
    h_dev = v["h"]
    for e in np.unique(ids[toks]):
        tt, jj = np.nonzero(ids[toks] == e)
        rows = inv[toks[tt], jj]
        want_h = oracle.swiglu_ffn_rows(oracle.bf16_to_f64(inp.x[toks[tt]]), synth.expert_gate_up(cfg, int(e)))
        got_h = host_f64(h_dev[torch_index(rows.astype(np.int64))])
        assert_close_output(got_h, want_h, what=f"h of expert {int(e)}")
    want = oracle.layer_forward_tokens(inp.x, toks, ids, w, lambda e: synth.expert_gate_up(cfg, e),
                                       lambda e: synth.expert_down(cfg, e), inp.w_sh_gate_up, inp.w_sh_down)
    got = host_f64(y[torch_index(toks)])
    assert_close_output(got, want)


def torch_index(toks):
    import torch
    return torch.from_numpy(toks).cuda()
