"""GPU parity of every stage and of the whole layer against the CPU oracle,
at sizes the oracle finishes in seconds: several tiles per expert, ragged
per-expert row counts, empty experts, one token, k = E, a shared expert,
experts with more rows than one tile pass, every tile policy, every router
implementation, the K-split of the expert GEMMs for a few tokens, E not a
multiple of 4, the largest k (64) and k = 1.  Routing (ids, counts, offsets,
permutation) must match bit for bit; floating-point outputs within the
layer's tolerance."""
import numpy as np
import pytest

import oracle
import routed_expert_ffn_prefix_b200 as moe
import synth
from synth import Config

from helpers import (W_ABS, assert_close_output, dev_bf16, dev_f32, dev_i32, host_f64)

pytestmark = pytest.mark.gpu

CASES = {
    c.name: c for c in [
        synth.CONFIGS["tiny"],
        Config("ragged", T=300, H=512, E=16, I=256, k=3),          # ragged counts, tails not /16
        Config("multipass", T=700, H=256, E=4, I=128, k=2),        # ~350 rows/expert: several row passes
        Config("shared_zipf", T=200, H=512, E=8, I=256, k=2, I_s=256, bias="zipf:1.2"),
        Config("k_eq_E", T=33, H=256, E=4, I=128, k=4),
        Config("one_token", T=1, H=512, E=16, I=256, k=4),
        Config("sparse", T=5, H=256, E=64, I=128, k=2),            # most experts empty
        Config("wide", T=96, H=1024, E=32, I=384, k=6, I_s=128),   # I not a power of two
        # few tokens: the one-launch router and K-split expert GEMMs
        Config("decode_split", T=1, H=1024, E=64, I=512, k=8),      # gate/up 4 K slices, down 2
        Config("few_e20", T=12, H=512, E=20, I=256, k=5),           # E % 8 != 0: ragged column slice
        Config("three_shared", T=3, H=768, E=32, I=128, k=4, I_s=128),
        Config("few_bias", T=7, H=1024, E=128, I=256, k=6, bias="zipf:1.2"),  # biased few-token routing
        # the one-launch layer: shared expert, biased routing, experts chosen by several tokens
        Config("few_shared", T=4, H=512, E=16, I=256, k=4, I_s=256, bias="zipf:1.2"),
        # edge cases: E % 4 != 0 above 128 experts (scalar 8-per-lane top-k), the largest k
        # (k = E = 64: every token takes every expert), and k = 1 (every weight exactly 1)
        Config("odd_e130", T=40, H=256, E=130, I=128, k=5),
        Config("k64", T=8, H=2048, E=64, I=128, k=64),
        Config("top1", T=50, H=256, E=8, I=128, k=1),
    ]
}

_cache = {}


def case(name):
    if name not in _cache:
        cfg = CASES[name]
        inp = synth.make_inputs(cfg)
        oracle.enforce_logit_gap(inp)
        ref = oracle.layer_forward(inp.x, inp.w_router, inp.bias, inp.w_gate_up, inp.w_down, cfg.k,
                                   inp.w_sh_gate_up, inp.w_sh_down)
        _cache[name] = (cfg, inp, ref)
    return _cache[name]


def dev_inputs(inp):
    d = dict(x=dev_bf16(inp.x), w_router=dev_f32(inp.w_router),
             bias=None if inp.bias is None else dev_f32(inp.bias),
             w_gate_up=dev_bf16(inp.w_gate_up), w_down=dev_bf16(inp.w_down))
    d["w_sh_gate_up"] = None if inp.w_sh_gate_up is None else dev_bf16(inp.w_sh_gate_up)
    d["w_sh_down"] = None if inp.w_sh_down is None else dev_bf16(inp.w_sh_down)
    return d


def workspace(cfg):
    return moe.alloc_workspace(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)


def assert_ok(ws):
    st = moe.device_status(ws)
    assert st == 0, moe.STATUS.get(st, st)


def router_skip(cfg, impl):
    if impl == moe.ROUTER_TC and cfg.E % 8:
        pytest.skip("tensor-core router needs E % 8 == 0")
    if impl == moe.ROUTER_SMALL and (cfg.T > 16 or cfg.E % 4):
        pytest.skip("few-token router needs T <= 16 and E % 4 == 0")


@pytest.mark.parametrize("impl", [moe.ROUTER_FMA, moe.ROUTER_TC, moe.ROUTER_SMALL])
@pytest.mark.parametrize("name", list(CASES))
def test_route_matches_oracle(name, impl):
    cfg, inp, ref = case(name)
    router_skip(cfg, impl)
    d = dev_inputs(inp)
    ws = workspace(cfg)
    ids, w = moe.route(d["x"], d["w_router"], d["bias"], cfg.k, ws, impl=impl)
    assert_ok(ws)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref["ids"])
    wg = host_f64(w)
    assert np.abs(wg - ref["w"]).max() <= W_ABS
    assert np.abs(wg.sum(1) - 1).max() <= 1e-6


@pytest.mark.parametrize("name", list(CASES))
def test_permute_bit_exact(name):
    cfg, inp, ref = case(name)
    ws = workspace(cfg)
    counts, offsets, sids, inv = moe.permute(dev_i32(ref["ids"]), cfg.E, ws)
    assert_ok(ws)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(offsets.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(sids.cpu().numpy(), ref["sorted_token_ids"])
    np.testing.assert_array_equal(inv.cpu().numpy(), ref["inv_perm"])


def test_permute_random_ids_large():
    """81,920 slots (the prefill shape's permuted row count) over 512 experts."""
    rng = np.random.default_rng(3)
    T, E, k = 8192, 512, 10
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    want = oracle.permute(ids, E)
    ws = moe.alloc_workspace(T, 256, E, 128, k)
    got = moe.permute(dev_i32(ids), E, ws)
    assert_ok(ws)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g.cpu().numpy().reshape(w.shape), w)


@pytest.mark.parametrize("tiles", [moe.TILES_SMALL, moe.TILES_LARGE, moe.TILES_PAIR])
@pytest.mark.parametrize("name", list(CASES))
def test_grouped_swiglu_matches_oracle(name, tiles):
    cfg, inp, ref = case(name)
    d = dev_inputs(inp)
    ws = workspace(cfg)
    h = moe.grouped_swiglu(d["x"], d["w_gate_up"], dev_i32(ref["offsets"]), dev_i32(ref["sorted_token_ids"]),
                           cfg.k, ws, tiles=tiles)
    assert_ok(ws)
    assert_close_output(host_f64(h), ref["h"], "h")


@pytest.mark.parametrize("tiles", [moe.TILES_SMALL, moe.TILES_LARGE, moe.TILES_PAIR])
@pytest.mark.parametrize("name", list(CASES))
def test_down_combine_matches_oracle(name, tiles):
    """Fed a synthetic h (not the GPU's): y = sum_j w o[inv_perm] + shared."""
    cfg, inp, ref = case(name)
    R = cfg.T * cfg.k
    h_bits = synth.normal_bf16(cfg.seed, synth.TID["h_stage"], 0, (R, cfg.I), 0.5)
    shared = synth.normal_f32(cfg.seed, synth.TID["misc"], 1, (cfg.T, cfg.H), 0.1) if cfg.I_s else None
    ws = workspace(cfg)
    y = moe.down_combine(dev_bf16(h_bits), dev_bf16(inp.w_down), dev_f32(ref["w"]), dev_i32(ref["inv_perm"]),
                         dev_i32(ref["offsets"]), None if shared is None else dev_f32(shared), ws, tiles=tiles)
    assert_ok(ws)
    want = oracle.down_combine(oracle.bf16_to_f64(h_bits), ref["offsets"], ref["inv_perm"], ref["w"],
                               lambda e: inp.w_down[e], None if shared is None else shared.astype(np.float64))
    assert_close_output(host_f64(y), want)


def test_grouped_down_single_group():
    cfg = CASES["wide"]
    rng_bits = synth.normal_bf16(1, synth.TID["misc"], 2, (77, cfg.I), 0.5)
    w = synth.normal_bf16(1, synth.TID["misc"], 3, (1, cfg.I, cfg.H), 0.05)
    ws = workspace(cfg)
    o = moe.grouped_down(dev_bf16(rng_bits), dev_bf16(w), None, ws)
    assert_ok(ws)
    want = oracle.bf16_to_f64(rng_bits) @ oracle.bf16_to_f64(w[0])
    assert_close_output(host_f64(o), want, "o")


def persistent_ok(cfg):
    return cfg.T <= 16 and cfg.E % 4 == 0 and cfg.I_s == 0


@pytest.mark.parametrize("router", [moe.ROUTER_FMA, moe.ROUTER_TC, moe.ROUTER_SMALL])
@pytest.mark.parametrize("tiles", [moe.TILES_SMALL, moe.TILES_LARGE, moe.TILES_PAIR, moe.TILES_PERSISTENT])
@pytest.mark.parametrize("name", list(CASES))
def test_forward_matches_oracle(name, tiles, router):
    cfg, inp, ref = case(name)
    router_skip(cfg, router)
    if tiles == moe.TILES_PERSISTENT and (router != moe.ROUTER_SMALL or not persistent_ok(cfg)):
        pytest.skip("persistent layer: T <= 16, E % 4 == 0, no shared expert (its router is the few-token one)")
    d = dev_inputs(inp)
    ws = workspace(cfg)
    y = moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
                    d["w_sh_gate_up"], d["w_sh_down"], tiles=tiles, router=router)
    assert_ok(ws)
    v = moe.workspace_view(ws, cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["ids"])
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), ref["sorted_token_ids"])
    np.testing.assert_array_equal(v["inv_perm"].cpu().numpy(), ref["inv_perm"])
    assert_close_output(host_f64(y), ref["y"])


def test_forward_bitwise_deterministic():
    """The combine sums each token's slots in a fixed order: repeated runs
    (with other work in between) give identical bits."""
    import torch
    cfg, inp, ref = case("ragged")
    d = dev_inputs(inp)
    ws = workspace(cfg)
    ys = []
    for i in range(4):
        ys.append(moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
                              tiles=moe.TILES_LARGE if i < 2 else moe.TILES_PAIR).cpu())
        moe.forward(d["x"][:7], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k,
                    moe.alloc_workspace(7, cfg.H, cfg.E, cfg.I, cfg.k))
    assert_ok(ws)
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[2], ys[3])


def arrivals_zero(ws, cfg):
    import torch
    lay = moe.workspace_layout(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    torch.cuda.synchronize()
    return bool((ws[lay["arrivals"]:lay["total"]] == 0).all().item())


@pytest.mark.parametrize("tiles", [moe.TILES_AUTO, moe.TILES_SMALL, moe.TILES_LARGE, moe.TILES_PAIR])
@pytest.mark.parametrize("name", list(CASES))
def test_fused_combine_bitwise_equals_separate_kernels(name, tiles):
    """The combine in the down GEMM's epilogue (and, for a K split, the slab
    sum + SwiGLU in the gate/up GEMM's) sums in the same order as the
    separate kernels, so y is bitwise the same whichever warp finishes a
    token; two fused calls in a row agree, and the arrival counters are
    back at zero after each call."""
    import torch
    cfg, inp, ref = case(name)
    d = dev_inputs(inp)
    ws = workspace(cfg)
    args = (d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
            d["w_sh_gate_up"], d["w_sh_down"])
    sep = moe.forward(*args, tiles=tiles, combine=moe.COMBINE_SEPARATE).cpu()
    assert_ok(ws)
    fused = []
    for _ in range(2):
        info = {}
        fused.append(moe.forward(*args, tiles=tiles, combine=moe.COMBINE_FUSED, info=info).cpu())
        assert_ok(ws)
        assert arrivals_zero(ws, cfg)
    assert torch.equal(fused[0], sep) and torch.equal(fused[1], sep)
    assert_close_output(host_f64(fused[0]), ref["y"])


def test_few_token_router_repeated_calls():
    """The one-launch router's last-block counter returns to zero after each
    launch: back-to-back calls (also through the whole layer) stay correct
    and leave the workspace's status block all zero."""
    import torch
    for name in ("decode_split", "few_e20", "three_shared", "few_bias"):
        cfg, inp, ref = case(name)
        d = dev_inputs(inp)
        ws = workspace(cfg)
        for _ in range(3):
            ids, w = moe.route(d["x"], d["w_router"], d["bias"], cfg.k, ws, impl=moe.ROUTER_SMALL)
            np.testing.assert_array_equal(ids.cpu().numpy(), ref["ids"])
            y = moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
                            d["w_sh_gate_up"], d["w_sh_down"])
            assert_close_output(host_f64(y), ref["y"])
        torch.cuda.synchronize()
        assert ws[:32].view(torch.int32).cpu().tolist() == [0] * 8


def test_split_k_forward_bitwise_deterministic():
    """K-split partial slabs are summed in slab order: repeated runs give
    identical bits, and the layout reserves the slabs."""
    import torch
    cfg, inp, ref = case("decode_split")
    lay = moe.workspace_layout(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, 0)
    assert lay["total"] - lay["split"] >= 4 * 4 * cfg.T * cfg.k * 2 * cfg.I  # 4 gate/up slices
    d = dev_inputs(inp)
    ws = workspace(cfg)
    info = {}
    ys = [moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
                      tiles=moe.TILES_SMALL, info=info).cpu() for _ in range(3)]
    assert_ok(ws)
    assert info["launches"] == 4  # route+permute, gate/up (slab sum + SwiGLU in its epilogue), down, combine
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    assert_close_output(host_f64(ys[0]), ref["y"])
    moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
                tiles=moe.TILES_SMALL, info=info, combine=moe.COMBINE_FUSED)
    assert info["launches"] == 3  # route+permute, gate/up, down + combine in its epilogue
    moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws,
                tiles=moe.TILES_SMALL, info=info, combine=moe.COMBINE_SEPARATE)
    assert info["launches"] == 5  # route+permute, gate/up, SwiGLU reduce, down, combine


@pytest.mark.parametrize("name", [n for n, c in CASES.items() if persistent_ok(c)])
def test_persistent_layer_bitwise_equals_kernel_sequence(name):
    """The persistent layer runs the same tiles, K split, epilogue arithmetic
    and router as the multi-kernel path with SMALL tiles and the few-token
    router, so y is bitwise the same; three calls in a row agree, the
    routing is bit-exact against the oracle, and the status block (router,
    plan and exit words) is all zero afterwards."""
    import torch
    cfg, inp, ref = case(name)
    d = dev_inputs(inp)
    ws = workspace(cfg)
    args = (d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws)
    want = moe.forward(*args, tiles=moe.TILES_SMALL, router=moe.ROUTER_SMALL).cpu()
    assert_ok(ws)
    info = {}
    for _ in range(3):
        got = moe.forward(*args, tiles=moe.TILES_PERSISTENT, info=info).cpu()
        assert_ok(ws)
        assert info["launches"] == 1
        assert torch.equal(got, want)
        torch.cuda.synchronize()
        assert ws[:32].view(torch.int32).cpu().tolist() == [0] * 8
    v = moe.workspace_view(ws, cfg.T, cfg.H, cfg.E, cfg.I, cfg.k, cfg.I_s)
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["ids"])
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), ref["sorted_token_ids"])
    np.testing.assert_array_equal(v["inv_perm"].cpu().numpy(), ref["inv_perm"])
    assert_close_output(host_f64(got), ref["y"])


def test_persistent_layer_rejects_unsupported_shapes():
    for name in ("tiny", "three_shared"):  # 64 tokens; a shared expert
        cfg, inp, ref = case(name)
        d = dev_inputs(inp)
        with pytest.raises(moe.MoEError):
            moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, workspace(cfg),
                        d["w_sh_gate_up"], d["w_sh_down"], tiles=moe.TILES_PERSISTENT)


def test_all_tokens_to_the_same_experts():
    """A bias far above the logits' spread sends every token to experts 0..k-1."""
    cfg = Config("hot", T=300, H=256, E=8, I=128, k=2)
    inp = synth.make_inputs(cfg)
    inp.bias = np.array([30.0, 20.0] + [0.0] * 6, np.float32)
    ref = oracle.layer_forward(inp.x, inp.w_router, inp.bias, inp.w_gate_up, inp.w_down, cfg.k)
    assert ref["counts"].tolist() == [300, 300, 0, 0, 0, 0, 0, 0]
    d = dev_inputs(inp)
    for tiles in (moe.TILES_SMALL, moe.TILES_LARGE, moe.TILES_PAIR):
        ws = workspace(cfg)
        y = moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws, tiles=tiles)
        assert_ok(ws)
        assert_close_output(host_f64(y), ref["y"])


# ---------------------------------------------------------------- failure detection (no GPU fault)

def test_bounded_wait_times_out_and_context_stays_usable():
    cfg, inp, ref = case("tiny")
    ws = workspace(cfg)
    moe.selftest_timeout(ws, 50_000_000)  # 50 ms on a barrier nothing completes
    assert moe.device_status(ws) == 5     # MOE_ERR_DEVICE_TIMEOUT
    moe.clear_device_status(ws)
    d = dev_inputs(inp)
    y = moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws)
    assert_ok(ws)
    assert_close_output(host_f64(y), ref["y"])


def test_corrupt_offsets_are_reported_not_followed():
    cfg, inp, ref = case("ragged")
    d = dev_inputs(inp)
    ws = workspace(cfg)
    bad = ref["offsets"].copy()
    bad[5] = cfg.T * cfg.k + 1000  # past the end of h and of sorted_token_ids
    h = moe.grouped_swiglu(d["x"], d["w_gate_up"], dev_i32(bad), dev_i32(ref["sorted_token_ids"]), cfg.k, ws)
    assert moe.device_status(ws) == 7  # MOE_ERR_DEVICE_BOUNDS
    moe.clear_device_status(ws)
    bad_ids = ref["sorted_token_ids"].copy()
    bad_ids[7] = cfg.T + 5  # a token that does not exist
    moe.grouped_swiglu(d["x"], d["w_gate_up"], dev_i32(ref["offsets"]), dev_i32(bad_ids), cfg.k, ws, out=h)
    assert moe.device_status(ws) == 7
    moe.clear_device_status(ws)
    ids = ref["ids"].copy()
    ids[3, 1] = cfg.E + 2
    moe.permute(dev_i32(ids), cfg.E, ws)
    assert moe.device_status(ws) == 7
    moe.clear_device_status(ws)
    # the library still works afterwards
    y = moe.forward(d["x"], d["w_router"], d["bias"], d["w_gate_up"], d["w_down"], cfg.k, ws)
    assert_ok(ws)
    assert_close_output(host_f64(y), ref["y"])
