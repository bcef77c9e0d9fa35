"""The Python binding checks every tensor argument before the library sees a
pointer (CPU): the call patterns the GPU tests and the bench use pass the
shape and dtype checks and stop only at the device check (these tensors are
on the CPU), and wrong shapes, dtypes, layouts, workspaces or a half-given
shared expert are refused with a clear error.  Nothing here reaches a CUDA
call."""
import pytest
import torch

import routed_expert_ffn_prefix_b200 as moe

bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
T, H, E, I, k, I_s = 300, 512, 16, 256, 3, 256


def t(*shape, dtype=bf):
    return torch.zeros(*shape, dtype=dtype)


def ws():
    return torch.zeros(4096, dtype=torch.uint8)


def only_device_error(fn, *a, **kw):
    with pytest.raises(TypeError, match="must be a CUDA tensor"):
        fn(*a, **kw)


def test_valid_call_patterns_stop_at_the_device_check():
    x, wr, b = t(T, H), t(H, E, dtype=f32), t(E, dtype=f32)
    wgu, wd = t(E, H, 2 * I), t(E, I, H)
    only_device_error(moe.forward, x, wr, None, wgu, wd, k, ws())
    only_device_error(moe.forward, x, wr, b, wgu, wd, k, ws(), t(H, 2 * I_s), t(I_s, H), tiles=moe.TILES_PAIR,
                      out=t(T, H), scoring=moe.SCORE_SIGMOID)
    only_device_error(moe.forward, x[:7], wr, b, wgu, wd, k, ws())
    only_device_error(moe.route, x, wr, b, k, ws(), impl=moe.ROUTER_SMALL)
    only_device_error(moe.route, x, wr, None, k, ws(), out=(t(T, k, dtype=i32), t(T, k, dtype=f32)))
    only_device_error(moe.permute, t(T, k, dtype=i32), E, ws())
    only_device_error(moe.grouped_swiglu, x, wgu, t(E + 1, dtype=i32), t(T * k, dtype=i32), k, ws())
    only_device_error(moe.grouped_swiglu, x, wgu, t(E + 1, dtype=i32), t(T * k, dtype=i32), k, ws(),
                      out=t(T * k, I))
    only_device_error(moe.grouped_down, t(77, I), t(1, I, H), None, ws())
    only_device_error(moe.grouped_down, t(T * k, I), wd, t(E + 1, dtype=i32), ws(), out=t(T * k, H, dtype=f32))
    only_device_error(moe.down_combine, t(T * k, I), wd, t(T, k, dtype=f32), t(T, k, dtype=i32),
                      t(E + 1, dtype=i32), t(T, H, dtype=f32), ws())
    only_device_error(moe.down_combine, t(T * k, I), wd, t(T, k, dtype=f32), t(T, k, dtype=i32),
                      t(E + 1, dtype=i32), None, ws(), out=t(T, H))
    only_device_error(moe.device_status, ws())
    only_device_error(moe.selftest_timeout, ws(), 1000)


@pytest.mark.parametrize("what", [
    "w_down_wrong_H", "bias_wrong_E", "router_wrong_E", "router_wrong_H", "out_wrong_shape",
    "shared_wrong_H", "x_rank",
])
def test_forward_refuses_inconsistent_shapes(what):
    a = dict(x=t(T, H), w_router=t(H, E, dtype=f32), bias=t(E, dtype=f32), w_gate_up=t(E, H, 2 * I),
             w_down=t(E, I, H), w_sh_gate_up=None, w_sh_down=None, out=None)
    if what == "w_down_wrong_H":
        a["w_down"] = t(E, I, H - 256)
    elif what == "bias_wrong_E":
        a["bias"] = t(E + 1, dtype=f32)
    elif what == "router_wrong_E":
        a["w_router"] = t(H, E - 1, dtype=f32)
    elif what == "router_wrong_H":
        a["w_router"] = t(H + 256, E, dtype=f32)
    elif what == "out_wrong_shape":
        a["out"] = t(T + 1, H)
    elif what == "shared_wrong_H":
        a["w_sh_gate_up"], a["w_sh_down"] = t(H, 2 * I_s), t(I_s, H + 256)
    elif what == "x_rank":
        a["x"] = t(T, H, 1)
    with pytest.raises(ValueError):
        moe.forward(a["x"], a["w_router"], a["bias"], a["w_gate_up"], a["w_down"], k, ws(),
                    a["w_sh_gate_up"], a["w_sh_down"], out=a["out"])


def test_stage_calls_refuse_inconsistent_shapes():
    x, wgu, wd = t(T, H), t(E, H, 2 * I), t(E, I, H)
    with pytest.raises(ValueError):   # offsets must have E + 1 entries
        moe.grouped_swiglu(x, wgu, t(E, dtype=i32), t(T * k, dtype=i32), k, ws())
    with pytest.raises(ValueError):   # one sorted token id per slot
        moe.grouped_swiglu(x, wgu, t(E + 1, dtype=i32), t(T * k - 1, dtype=i32), k, ws())
    with pytest.raises(ValueError):   # h's width is the experts' I
        moe.grouped_down(t(T * k, I + 128), wd, t(E + 1, dtype=i32), ws())
    with pytest.raises(ValueError):   # h holds T*k rows
        moe.down_combine(t(T * k - 3, I), wd, t(T, k, dtype=f32), t(T, k, dtype=i32), t(E + 1, dtype=i32),
                         None, ws())
    with pytest.raises(ValueError):   # inv_perm is [T, k]
        moe.down_combine(t(T * k, I), wd, t(T, k, dtype=f32), t(T, k + 1, dtype=i32), t(E + 1, dtype=i32),
                         None, ws())
    with pytest.raises(ValueError):
        moe.route(x, t(H, E, dtype=f32), None, k, ws(), out=(t(T, k + 1, dtype=i32), t(T, k, dtype=f32)))


def test_dtype_layout_workspace_and_shared_expert_errors():
    x, wr, wgu, wd = t(T, H), t(H, E, dtype=f32), t(E, H, 2 * I), t(E, I, H)
    with pytest.raises(TypeError, match="must be torch.bfloat16"):
        moe.forward(x.float(), wr, None, wgu, wd, k, ws())
    with pytest.raises(TypeError, match="must be torch.float32"):
        moe.forward(x, wr.to(bf), None, wgu, wd, k, ws())
    with pytest.raises(ValueError, match="contiguous"):
        moe.forward(t(H, T).t(), wr, None, wgu, wd, k, ws())
    with pytest.raises(TypeError, match="workspace"):
        moe.forward(x, wr, None, wgu, wd, k, torch.zeros(64, dtype=torch.int32))
    with pytest.raises(TypeError, match="shared expert"):
        moe.forward(x, wr, None, wgu, wd, k, ws(), t(H, 2 * I_s), None)
    with pytest.raises(TypeError, match="torch.Tensor"):
        moe.route([[0.0]], wr, None, k, ws())


MH, MI = 512, 128  # H != 2I, so a [E, K, N] code tensor cannot pass for [E, N, K]


def mx_args():
    """Block-scaled FP8 weights in the library's layout: codes of W^T [E, N, K]
    (K contiguous), scales [E, K/32, N]."""
    u8 = torch.uint8
    return dict(x=t(T, MH), w_router=t(MH, E, dtype=f32), bias=None,
                gu_codes=t(E, 2 * MI, MH, dtype=u8), gu_scales=t(E, MH // 32, 2 * MI, dtype=u8),
                dn_codes=t(E, MH, MI, dtype=u8), dn_scales=t(E, MI // 32, MH, dtype=u8))


def call_mx(a, **kw):
    return moe.forward_mx(a["x"], a["w_router"], a["bias"], a["gu_codes"], a["gu_scales"], a["dn_codes"],
                          a["dn_scales"], k, ws(), **kw)


def test_forward_mx_valid_calls_stop_at_the_device_check():
    only_device_error(call_mx, mx_args())
    only_device_error(call_mx, mx_args(), tiles=moe.TILES_SMALL, combine=moe.COMBINE_SEPARATE)
    a = mx_args()
    only_device_error(moe.forward_mx, a["x"], a["w_router"], t(E, dtype=f32), a["gu_codes"], a["gu_scales"],
                      a["dn_codes"], a["dn_scales"], k, ws(), t(MH, 2 * I_s), t(I_s, MH))


@pytest.mark.parametrize("what", [
    "gu_codes_not_transposed", "dn_codes_not_transposed", "gu_scales_transposed", "dn_scales_wrong_blocks",
])
def test_forward_mx_refuses_wrong_weight_layouts(what):
    a = mx_args()
    u8 = torch.uint8
    if what == "gu_codes_not_transposed":      # [E, K, N] is the bf16 layout, not the FP8 one
        a["gu_codes"] = t(E, MH, 2 * MI, dtype=u8)
    elif what == "dn_codes_not_transposed":
        a["dn_codes"] = t(E, MI, MH, dtype=u8)
    elif what == "gu_scales_transposed":
        a["gu_scales"] = t(E, 2 * MI, MH // 32, dtype=u8)
    elif what == "dn_scales_wrong_blocks":
        a["dn_scales"] = t(E, MI // 16, MH, dtype=u8)
    with pytest.raises(ValueError):
        call_mx(a)


@pytest.mark.parametrize("which", ["gu_codes", "dn_scales"])
def test_forward_mx_refuses_non_byte_weights(which):
    a = mx_args()
    a[which] = a[which].to(torch.int8 if which == "gu_codes" else bf)
    with pytest.raises(TypeError, match="must be torch.uint8"):
        call_mx(a)
