"""The C-ABI library builds, loads and exports every function include/moe.h
declares; host-side argument checks return the documented status before
anything touches a device (every call here is invalid on purpose, so none
of them reaches a CUDA call)."""
import ctypes
import os
import re

import pytest

import routed_expert_ffn_prefix_b200 as moe
from routed_expert_ffn_prefix_b200 import build as moe_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_layer_calls():
    names = declared_functions()
    for n in ["moe_route", "moe_permute", "moe_grouped_swiglu", "moe_down_combine", "moe_forward",
              "moe_workspace_size", "moe_status_string", "moe_get_device_status"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(lib):
    assert lib.moe_abi_version() == 2
    for code, name in moe.STATUS.items():
        assert lib.moe_status_string(code).decode().startswith(name)


def test_workspace_layout_is_ordered_and_aligned(lib):
    L = moe.workspace_layout(8192, 4096, 512, 1024, 10)
    offs = [L[n] for n in ("status", "topk_ids", "topk_w", "counts", "offsets", "sorted_token_ids",
                           "inv_perm", "block_hist", "logits", "router_split", "h", "o", "h_shared",
                           "o_shared", "split", "arrivals", "total")]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L["o"] - L["h"] >= 81920 * 1024 * 2          # h: [T*k, I] bf16
    assert L["h_shared"] - L["o"] >= 81920 * 4096 * 4   # o: [T*k, H] f32
    assert moe.workspace_size(8192, 4096, 512, 1024, 10) == L["total"]
    Ls = moe.workspace_layout(4096, 8192, 256, 2048, 8, 2048)
    assert Ls["split"] - Ls["o_shared"] >= 4096 * 8192 * 4
    # many tokens: no K split, so no partial slabs
    assert L["arrivals"] == L["split"] and Ls["arrivals"] == Ls["split"]
    # arrival counters of the combine in the down GEMM (one per token and 64 output columns) and one
    # done-counter per expert and 128-column gate/up block, rounded up to 256 bytes
    assert L["total"] - L["arrivals"] == (8192 * (4096 // 64) + 512 * 8 + 63) // 64 * 256
    assert Ls["total"] - Ls["arrivals"] == (4096 * (8192 // 64) + 256 * 16 + 63) // 64 * 256


def test_workspace_layout_reserves_k_split_slabs_for_one_token(lib):
    """One token, 8 of 256 experts, H = 4096, I = 1536: 8 active experts give
    96 gate/up units (-> 3 K slices) and 128 down units (-> 2 slices) for
    148 SMs.  The split region holds both: 3 x 8 rows x 3072 and 2 x 8 rows x 4096 f32."""
    L = moe.workspace_layout(1, 4096, 256, 1536, 8)
    # gate/up slabs, then down slabs (the persistent few-token layer holds both)
    assert L["arrivals"] - L["split"] == (3 * 8 * 3072 + 2 * 8 * 4096) * 4
    # arrival counters: the K-split gate/up's (8 rows x 1536/32 chunks), the down's (1 x 4096/64) and one
    # per expert and 128-column gate/up block, side by side, rounded up to 256 bytes
    assert L["total"] - L["arrivals"] == (8 * 1536 // 32 + 4096 // 64 + 256 * 12 + 63) // 64 * 256
    # the router's partial slabs: one per H slice of the few-token router
    assert L["router_split"] - L["logits"] >= 4 * 1 * 256 * 4


FAKE = 0x100000  # never dereferenced: every call below fails its host-side checks first


def p(v=FAKE):
    return ctypes.c_void_p(v)


@pytest.mark.parametrize("T,H,E,I,k,Is,code", [
    (0, 256, 8, 128, 2, 0, 1),       # no tokens
    (4, 256, 8, 128, 9, 0, 1),       # k > E
    (4, 256, 8, 128, 0, 0, 1),       # k < 1
    (4, 256, 2000, 128, 2, 0, 1),    # E above the supported maximum
    (4, 200, 8, 128, 2, 0, 2),       # H not a multiple of 256
    (4, 256, 8, 96, 2, 0, 2),        # I not a multiple of 128
    (4, 256, 8, 128, 2, 100, 2),     # I_s not a multiple of 128
    (4, 256, 100, 128, 65, 0, 1),    # k above 64
])
def test_layout_rejects_bad_shapes(lib, T, H, E, I, k, Is, code):
    n = ctypes.c_size_t()
    assert lib.moe_workspace_size(T, H, E, I, k, Is, ctypes.byref(n)) == code


def test_forward_options_scoring_is_checked(lib):
    """An unknown scoring rule in the options is refused on the host; the
    options struct keeps its size (the field took a reserved slot)."""
    ws = moe.workspace_size(64, 256, 8, 128, 2)
    assert ctypes.sizeof(moe._Options) == 4 * 2 + 8 * 7 + 4 * 6
    for bad_scoring in (-1, 3):
        opt = moe._Options(0, 0)
        opt.scoring = bad_scoring
        assert lib.moe_forward_ex(p(), p(), None, p(), p(), None, None, 0, 64, 256, 8, 128, 2, p(), p(), ws,
                                  ctypes.byref(opt), None) == 1


def test_forward_options_tiles_and_combine_are_checked(lib):
    """Tile policies run 0..4 (4 = the persistent one-launch layer) and
    combine placements 0..2; anything else is refused on the host, and so
    are the options the FP8-weight layer does not take (the persistent
    layer, the combine in the down epilogue)."""
    ws = moe.workspace_size(64, 256, 8, 128, 2)
    assert (moe.TILES_AUTO, moe.TILES_SMALL, moe.TILES_LARGE, moe.TILES_PAIR, moe.TILES_PERSISTENT) == (0, 1, 2, 3, 4)
    for tiles, combine in ((-1, 0), (5, 0), (0, -1), (0, 3)):
        opt = moe._Options(tiles, 0)
        opt.combine = combine
        assert lib.moe_forward_ex(p(), p(), None, p(), p(), None, None, 0, 64, 256, 8, 128, 2, p(), p(), ws,
                                  ctypes.byref(opt), None) == 1, (tiles, combine)
    for tiles, combine in ((moe.TILES_PERSISTENT, 0), (0, moe.COMBINE_FUSED)):
        opt = moe._Options(tiles, 0)
        opt.combine = combine
        assert lib.moe_forward_mx(p(), p(), None, p(), p(), p(), p(), None, None, 0, 64, 256, 8, 128, 2, p(), p(),
                                  ws, ctypes.byref(opt), None) == 1, (tiles, combine)


def test_forward_argument_errors_before_any_launch(lib):
    f = lib.moe_forward
    ws = moe.workspace_size(64, 256, 8, 128, 2)
    good = [p(), p(), None, p(), p(), None, None, 0, 64, 256, 8, 128, 2, p(), p(), ws, None]
    cases = []
    bad = list(good); bad[0] = None; cases.append((bad, 1))           # x missing
    bad = list(good); bad[13] = None; cases.append((bad, 1))          # y missing
    bad = list(good); bad[12] = 9; cases.append((bad, 1))             # k > E
    bad = list(good); bad[9] = 300; cases.append((bad, 2))            # H misaligned
    bad = list(good); bad[14] = None; cases.append((bad, 3))          # no workspace
    bad = list(good); bad[15] = ws - 1; cases.append((bad, 3))        # workspace too small
    bad = list(good); bad[14] = p(FAKE + 128); cases.append((bad, 2))  # workspace not 256-aligned
    bad = list(good); bad[0] = p(FAKE + 2); cases.append((bad, 2))    # x not 16-aligned
    bad = list(good); bad[5] = p(); cases.append((bad, 1))            # shared gate/up without down
    for args, code in cases:
        assert f(*args) == code, (args, code)


def test_stage_argument_errors(lib):
    ws = moe.workspace_size(64, 256, 8, 128, 2)
    assert lib.moe_route(None, p(), None, 64, 256, 8, 2, p(), p(), p(), ws, None) == 1
    assert lib.moe_route_ex(p(), p(), None, 64, 256, 8, 2, p(), p(), 7, p(), ws, None) == 1
    for bad_scoring in (-1, 3):
        assert lib.moe_route_scored(p(), p(), None, 64, 256, 8, 2, bad_scoring, p(), p(), 0, p(), ws, None) == 1
    assert lib.moe_route_scored(p(), p(), p(FAKE + 4), 64, 256, 8, 2, 2, p(), p(), 0, p(), ws, None) == 2
    assert lib.moe_permute(p(), 64, 8, 2, p(), p(), p(), None, p(), ws, None) == 1
    assert lib.moe_permute(p(), 64, 8, 2, p(), p(), p(), p(), p(), 16, None) == 3
    assert lib.moe_grouped_swiglu(p(), p(), p(), p(), 64, 256, 8, 100, 2, 0, p(), p(), ws, None) == 2
    assert lib.moe_grouped_swiglu(p(), p(), p(), p(), 64, 256, 8, 128, 2, 5, p(), p(), ws, None) == 1
    assert lib.moe_grouped_down(p(), p(), None, 10, 256, 4, 128, 0, p(), p(), ws, None) == 1
    assert lib.moe_down_combine(p(), p(), p(), p(), p(), p(FAKE + 4), 64, 256, 8, 128, 2, 0, p(), p(), ws,
                                None) == 2
    assert lib.moe_selftest_timeout(None, 0, 1000, None) == 3
    assert lib.moe_get_device_status(None, None, None) == 1
