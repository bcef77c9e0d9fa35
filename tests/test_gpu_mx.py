"""GPU parity of the layer on block-scaled FP8 expert weights
(moe_forward_mx): OCP E4M3 codes with one E8M0 scale per 32 weights along
the reduction dimension.  Every such weight is an exact bf16 value, so:

  * routing is bit-exact against the float64 oracle and y, h match the
    oracle's layer on the dequantised weights within the layer's tolerance;
  * with the same tile policy the FP8 kernel runs the same MMAs in the same
    order as the bf16 kernel on the dequantised weights, so y is bitwise
    equal to moe_forward_ex on those bf16 weights.

Cases: ragged counts, a shared expert with a skewed router, one token (the
few-token router and the K split of both GEMMs), k = 1, E not a multiple of
8 (CUDA-core router), 128-row and 256-row passes, and scale codes above 134
(the decode's two-multiply form)."""
import numpy as np
import pytest

import oracle
import routed_expert_ffn_prefix_b200 as moe
import synth
from synth import Config

from helpers import W_ABS, assert_close_output, dev_bf16, dev_f32, host_f64

pytestmark = pytest.mark.gpu

CASES = {
    c.name: c for c in [
        Config("mx_tiny", T=64, H=256, E=8, I=128, k=2),
        Config("mx_ragged", T=300, H=512, E=16, I=256, k=3),
        Config("mx_shared", T=200, H=512, E=8, I=256, k=2, I_s=256, bias="zipf:1.2"),
        Config("mx_one_token", T=1, H=1024, E=64, I=512, k=8),       # K split of both GEMMs
        Config("mx_top1", T=50, H=256, E=8, I=128, k=1),
        Config("mx_e20", T=12, H=512, E=20, I=256, k=5),             # E % 8 != 0
        Config("mx_multipass", T=700, H=256, E=4, I=128, k=2),       # several 256-row passes per expert
        # scale codes up to 140 (factors 2^(code - 7) beyond fp32 for codes above 134): the decode takes
        # its two-multiply form in the k-steps that hold one
        Config("mx_bigscale", T=64, H=512, E=8, I=256, k=2),
    ]
}
BIG_SCALE = {"mx_bigscale": (128, 140)}

_cache = {}


def case(name):
    if name not in _cache:
        cfg = CASES[name]
        inp = synth.make_inputs(cfg, experts=False)
        oracle.enforce_logit_gap(inp)
        gu = [synth.mx_expert_weights(cfg, e, "gate_up") for e in range(cfg.E)]
        dn = [synth.mx_expert_weights(cfg, e, "down") for e in range(cfg.E)]
        if name in BIG_SCALE:  # odd experts get scale codes drawn from a higher range
            lo, hi = BIG_SCALE[name]
            for e in range(1, cfg.E, 2):
                gu[e] = (gu[e][0], synth.e8m0_scale_codes(cfg.seed, synth.TID["misc"], 100 + e, gu[e][1].shape, lo, hi))
                dn[e] = (dn[e][0], synth.e8m0_scale_codes(cfg.seed, synth.TID["misc"], 200 + e, dn[e][1].shape, lo, hi))
        wgu = np.stack([oracle.mx.mx_dequant(c, s) for c, s in gu])   # float64 [E, H, 2I]
        wd = np.stack([oracle.mx.mx_dequant(c, s) for c, s in dn])    # float64 [E, I, H]
        ref = oracle.layer_forward(inp.x, inp.w_router, inp.bias, wgu, wd, cfg.k, inp.w_sh_gate_up, inp.w_sh_down)
        # the library takes the codes of W^T [E, N, K] (K contiguous)
        mx = (np.stack([c.T for c, _ in gu]), np.stack([s for _, s in gu]),
              np.stack([c.T for c, _ in dn]), np.stack([s for _, s in dn]))
        _cache[name] = (cfg, inp, ref, mx, wgu, wd)
    return _cache[name]


def dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def bf16_bits_exact(w64):
    """bf16 bit patterns of values that are exact in bf16 (checked)."""
    f32 = np.asarray(w64, np.float32)
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_to_f64(bits), w64)
    return bits


def run_mx(cfg, inp, mx, tiles, combine=moe.COMBINE_AUTO, info=None):
    ws = moe.alloc_workspace(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    sh = (None, None) if inp.w_sh_gate_up is None else (dev_bf16(inp.w_sh_gate_up), dev_bf16(inp.w_sh_down))
    y = moe.forward_mx(dev_bf16(inp.x), dev_f32(inp.w_router), None if inp.bias is None else dev_f32(inp.bias),
                       *[dev_u8(a) for a in mx], cfg.k, ws, *sh, tiles=tiles, combine=combine, info=info)
    st = moe.device_status(ws)
    assert st == 0, moe.STATUS.get(st, st)
    return y, ws


@pytest.mark.parametrize("tiles", [moe.TILES_AUTO, moe.TILES_SMALL, moe.TILES_LARGE])
@pytest.mark.parametrize("name", list(CASES))
def test_mx_forward_matches_oracle(name, tiles):
    cfg, inp, ref, mx, _, _ = case(name)
    y, ws = run_mx(cfg, inp, mx, tiles)
    v = moe.workspace_view(ws, cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["ids"])
    assert np.abs(host_f64(v["topk_w"]) - ref["w"]).max() <= W_ABS
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), ref["sorted_token_ids"])
    assert_close_output(host_f64(v["h"]), ref["h"], "h")
    assert_close_output(host_f64(y), ref["y"])


@pytest.mark.parametrize("tiles", [moe.TILES_SMALL, moe.TILES_LARGE])
@pytest.mark.parametrize("name", list(CASES))
def test_mx_forward_bitwise_equals_bf16_kernel_on_dequantised_weights(name, tiles):
    import torch
    cfg, inp, ref, mx, wgu, wd = case(name)
    y_mx, _ = run_mx(cfg, inp, mx, tiles)
    ws = moe.alloc_workspace(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    sh = (None, None) if inp.w_sh_gate_up is None else (dev_bf16(inp.w_sh_gate_up), dev_bf16(inp.w_sh_down))
    y_bf = moe.forward(dev_bf16(inp.x), dev_f32(inp.w_router), None if inp.bias is None else dev_f32(inp.bias),
                       dev_bf16(bf16_bits_exact(wgu)), dev_bf16(bf16_bits_exact(wd)), cfg.k, ws, *sh, tiles=tiles)
    assert moe.device_status(ws) == 0
    assert torch.equal(y_mx.cpu(), y_bf.cpu())


def test_mx_split_slab_sum_in_epilogue_equals_reduce_kernel_and_repeats():
    """One token: the K-split gate/up slabs summed in the epilogue of the last
    slab to land (the default) and by the separate reduce kernel give the
    same bits, call after call."""
    import torch
    cfg, inp, ref, mx, _, _ = case("mx_one_token")
    info = {}
    ys = [run_mx(cfg, inp, mx, moe.TILES_AUTO, info=info)[0].cpu() for _ in range(2)]
    assert info["launches"] == 4  # route+permute, gate/up (slab sum + SwiGLU in its epilogue), down, combine
    sep, _ = run_mx(cfg, inp, mx, moe.TILES_AUTO, combine=moe.COMBINE_SEPARATE, info=info)
    assert info["launches"] == 5
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], sep.cpu())
    assert_close_output(host_f64(ys[0]), ref["y"])


def test_mx_rejects_unsupported_options():
    cfg, inp, ref, mx, _, _ = case("mx_one_token")
    for kw in (dict(tiles=moe.TILES_PERSISTENT), dict(combine=moe.COMBINE_FUSED)):
        with pytest.raises(moe.MoEError):
            run_mx(cfg, inp, mx, **{"tiles": moe.TILES_AUTO, **kw})


@pytest.mark.slow
def test_mx_full_size_decode():
    """The 512-expert decode shape (T = 512, H = 4096, I = 1024, top-10) on
    block-scaled FP8 weights, in the launch configuration bench.py times
    (automatic tiles): routing bit-exact on every token, h on every permuted
    row of a sample of tokens and y on those tokens against the oracle on the
    dequantised weights, one expert at a time."""
    import torch
    from test_gpu_fullsize import sample_tokens, torch_index
    cfg = synth.CONFIGS["qwen_decode_t512"]
    inp = synth.make_inputs(cfg, experts=False)
    oracle.enforce_logit_gap(inp)
    E, H, I = cfg.E, cfg.H, cfg.I
    gu_c = torch.empty(E, 2 * I, H, dtype=torch.uint8, device="cuda")   # codes of W^T
    gu_s = torch.empty(E, H // 32, 2 * I, dtype=torch.uint8, device="cuda")
    dn_c = torch.empty(E, H, I, dtype=torch.uint8, device="cuda")
    dn_s = torch.empty(E, I // 32, H, dtype=torch.uint8, device="cuda")
    from concurrent.futures import ThreadPoolExecutor

    def draw(e):
        cg, sg = synth.mx_expert_weights(cfg, e, "gate_up")
        cd, sd = synth.mx_expert_weights(cfg, e, "down")
        return np.ascontiguousarray(cg.T), sg, np.ascontiguousarray(cd.T), sd

    with ThreadPoolExecutor(16) as ex:
        for e0 in range(0, E, 32):
            for e, (cg, sg, cd, sd) in zip(range(e0, e0 + 32), ex.map(draw, range(e0, min(E, e0 + 32)))):
                gu_c[e].copy_(torch.from_numpy(cg))
                gu_s[e].copy_(torch.from_numpy(sg))
                dn_c[e].copy_(torch.from_numpy(cd))
                dn_s[e].copy_(torch.from_numpy(sd))
    ws = moe.alloc_workspace(cfg.T, H, E, I, cfg.k)
    y = moe.forward_mx(dev_bf16(inp.x), dev_f32(inp.w_router), None, gu_c, gu_s, dn_c, dn_s, cfg.k, ws)
    st = moe.device_status(ws)
    assert st == 0, moe.STATUS.get(st, st)

    ids, w = oracle.topk_route(oracle.router_logits(inp.x, inp.w_router, inp.bias), cfg.k)
    counts, offsets, sids, inv = oracle.permute(ids, E)
    v = moe.workspace_view(ws, cfg.T, H, E, I, cfg.k)
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ids)
    assert np.abs(host_f64(v["topk_w"]) - w).max() <= W_ABS
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), sids)
    np.testing.assert_array_equal(v["inv_perm"].cpu().numpy(), inv)

    def gate_up(e):
        return oracle.mx.mx_dequant(*synth.mx_expert_weights(cfg, int(e), "gate_up"))

    def down(e):
        return oracle.mx.mx_dequant(*synth.mx_expert_weights(cfg, int(e), "down"))

    toks = sample_tokens(cfg, counts, ids, n_random=4)
    for e in np.unique(ids[toks]):
        tt, jj = np.nonzero(ids[toks] == e)
        rows = inv[toks[tt], jj]
        want_h = oracle.swiglu_ffn_rows(oracle.bf16_to_f64(inp.x[toks[tt]]), gate_up(e))
        got_h = host_f64(v["h"][torch_index(rows.astype(np.int64))])
        assert_close_output(got_h, want_h, what=f"h of expert {int(e)}")
    want = oracle.layer_forward_tokens(inp.x, toks, ids, w, gate_up, down)
    assert_close_output(host_f64(y[torch_index(toks)]), want)
