"""Pins for the CPU oracle: each check compares it with something other than
itself -- brute force on tiny inputs, closed forms, library routines for
special cases, and invariants -- chosen so that a plausible slip (dropped
renormalisation, wrong sort direction, swapped gate/up halves, wrong slot
index, shared expert weighted wrongly) fails at least one of them."""
import itertools
import math

import numpy as np
import pytest
import scipy.special

import oracle
import synth
from oracle import moe_oracle as om


def bits(a):
    return synth.bf16_from_f32(np.asarray(a, np.float32))


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


# ---------------------------------------------------------------- bf16 decode

def test_bf16_decode_known_patterns():
    b = np.array([0x3F80, 0xC000, 0x3F00, 0x4049, 0x0000, 0x8000, 0x3C00], np.uint16)
    want = [1.0, -2.0, 0.5, 3.140625, 0.0, -0.0, 2.0 ** -7]
    assert om.bf16_to_f64(b).tolist() == want


# ---------------------------------------------------------------- routing

def test_topk_matches_best_subset_bruteforce():
    """Top-k is the k-subset with the largest logit sum, listed by descending logit."""
    rng = np.random.default_rng(1)
    for E, k in [(5, 2), (6, 3), (7, 1), (6, 6)]:
        l = rng.standard_normal((30, E))
        ids, _ = om.topk_route(l, k)
        for t in range(30):
            best = max(itertools.combinations(range(E), k), key=lambda s: sum(l[t, i] for i in s))
            want = sorted(best, key=lambda i: -l[t, i])
            assert ids[t].tolist() == want


def test_weights_k2_closed_form_is_logistic_of_gap():
    """k=2: w_0 = 1/(1+exp(l_1-l_0)) -- independent of every other logit."""
    rng = np.random.default_rng(2)
    l = rng.standard_normal((50, 9)) * 2
    ids, w = om.topk_route(l, 2)
    for t in range(50):
        d = l[t, ids[t, 1]] - l[t, ids[t, 0]]
        assert w[t, 0] == pytest.approx(1.0 / (1.0 + math.exp(d)), rel=1e-14)
        assert w[t, 1] == pytest.approx(1.0 / (1.0 + math.exp(-d)), rel=1e-14)


def test_weights_equal_full_softmax_when_k_is_E():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((20, 8)) * 3
    ids, w = om.topk_route(l, 8)
    p = scipy.special.softmax(l, axis=1)
    for t in range(20):
        np.testing.assert_allclose(w[t], p[t, ids[t]], rtol=1e-13)


def test_weights_literal_softmax_topk_renormalise():
    """The literal reading -- softmax over all E, pick the k largest
    probabilities, divide by their sum -- written with pure-Python math."""
    rng = np.random.default_rng(4)
    for E, k in [(8, 2), (12, 5), (16, 10)]:
        l = rng.standard_normal((25, E)) * 1.5
        ids, w = om.topk_route(l, k)
        for t in range(25):
            z = [math.exp(v) for v in l[t]]
            s = sum(z)
            p = [v / s for v in z]
            top = sorted(range(E), key=lambda i: (-p[i], i))[:k]
            ps = sum(p[i] for i in top)
            assert ids[t].tolist() == top
            for j, i in enumerate(top):
                assert w[t, j] == pytest.approx(p[i] / ps, rel=1e-12)


def test_k1_weight_exactly_one_and_rows_sum_to_one():
    rng = np.random.default_rng(5)
    l = rng.standard_normal((40, 16))
    _, w1 = om.topk_route(l, 1)
    assert np.all(w1 == 1.0)
    _, w4 = om.topk_route(l, 4)
    np.testing.assert_allclose(w4.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.all(np.diff(w4, axis=1) <= 0)  # descending logits -> descending weights


def test_ties_go_to_lower_expert_id():
    l = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]])
    ids, w = om.topk_route(l, 3)
    assert ids[0].tolist() == [1, 2, 4]
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-15)


def test_router_logits_bias_and_orientation():
    """l[t,e] = sum_h x[t,h] W[h,e] + b[e]: one-hot x picks row h of W."""
    H, E = 4, 3
    W = np.arange(H * E, dtype=np.float32).reshape(H, E) / 8
    x = np.zeros((H, H), np.float32)
    np.fill_diagonal(x, 1.0)
    b = np.array([0.5, -1.0, 2.0], np.float32)
    l = om.router_logits(bits(x), W, b)
    np.testing.assert_array_equal(l, W.astype(np.float64) + b)


# ---------------------------------------------------------------- scoring variants

def test_scored_routing_without_bias_selects_like_softmax():
    """exp and sigmoid are monotone: with no bias every scoring picks the
    same experts in the same order, and select-only-bias weights are the
    plain softmax ones."""
    rng = np.random.default_rng(21)
    l = rng.standard_normal((40, 12)) * 2
    ids0, w0 = om.topk_route(l, 4)
    for scoring in om.SCORINGS:
        ids, w = om.route_scored(l, None, 4, scoring)
        np.testing.assert_array_equal(ids, ids0)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
    _, w1 = om.route_scored(l, None, 4, "softmax_select_bias")
    np.testing.assert_allclose(w1, w0, rtol=1e-14)


def test_select_bias_picks_best_biased_subset_and_weights_ignore_bias():
    """Selection: the k-subset with the largest sum of l + b, by descending
    l + b.  Weights: scipy's softmax over the selected unbiased logits."""
    rng = np.random.default_rng(22)
    for E, k in [(6, 2), (7, 3), (5, 5)]:
        l = rng.standard_normal((25, E))
        b = rng.standard_normal(E) * 1.5
        ids, w = om.route_scored(l, b, k, "softmax_select_bias")
        for t in range(25):
            key = [l[t, i] + b[i] for i in range(E)]
            best = max(itertools.combinations(range(E), k), key=lambda s: sum(key[i] for i in s))
            assert ids[t].tolist() == sorted(best, key=lambda i: -key[i])
            np.testing.assert_allclose(w[t], scipy.special.softmax(l[t, ids[t]]), rtol=1e-13)


def test_select_bias_forces_expert_without_changing_its_share():
    """A large bias on expert 3 makes it slot 0 of every token; the weights
    are those of softmax over the same experts with no bias."""
    rng = np.random.default_rng(23)
    l = rng.standard_normal((30, 8))
    b = np.zeros(8)
    b[3] = 50.0
    ids, w = om.route_scored(l, b, 3, "softmax_select_bias")
    assert np.all(ids[:, 0] == 3)
    ids_sm, w_sm = om.route_scored(l, b, 3, "softmax")
    np.testing.assert_array_equal(ids, ids_sm)
    assert np.all(w_sm[:, 0] > 1 - 1e-15)         # bias inside the softmax swamps the rest
    assert np.all(w[:, 0] < 0.999)                # ... but not under select-only bias
    # shifting every bias by a constant changes nothing
    ids2, w2 = om.route_scored(l, b - 7.25, 3, "softmax_select_bias")
    np.testing.assert_array_equal(ids2, ids)
    np.testing.assert_allclose(w2, w, rtol=1e-15)


def test_sigmoid_weights_worked_by_hand():
    """l = [ln 3, 0, -ln 3] has sigmoids [3/4, 1/2, 1/4]: top-2 weights
    (3/5, 2/5), all three (1/2, 1/3, 1/6), top-1 exactly 1."""
    l = np.array([[math.log(3.0), 0.0, -math.log(3.0)]])
    ids, w = om.route_scored(l, None, 2, "sigmoid")
    assert ids[0].tolist() == [0, 1]
    np.testing.assert_allclose(w[0], [3 / 5, 2 / 5], rtol=1e-15)
    ids, w = om.route_scored(l, None, 3, "sigmoid")
    np.testing.assert_allclose(w[0], [1 / 2, 1 / 3, 1 / 6], rtol=1e-15)
    _, w = om.route_scored(l[:, ::-1].copy(), None, 1, "sigmoid")
    assert w[0, 0] == 1.0


def test_sigmoid_bias_is_added_after_the_sigmoid():
    """l = [2, 0], b = [0, 0.5]: sigmoid keys 0.881 < 1.0 pick expert 1,
    while l + b = [2, 0.5] picks expert 0.  Weights never see the bias."""
    l = np.array([[2.0, 0.0]])
    b = np.array([0.0, 0.5])
    ids, w = om.route_scored(l, b, 1, "sigmoid")
    assert ids[0].tolist() == [1] and w[0, 0] == 1.0
    ids, _ = om.route_scored(l, b, 1, "softmax_select_bias")
    assert ids[0].tolist() == [0]
    ids, w = om.route_scored(l, b, 2, "sigmoid")
    assert ids[0].tolist() == [1, 0]
    np.testing.assert_allclose(w[0], [0.5 / (0.5 + sig(2)), sig(2) / (0.5 + sig(2))], rtol=1e-14)


def test_sigmoid_picks_best_subset_and_matches_expit():
    rng = np.random.default_rng(24)
    for E, k in [(6, 2), (7, 4), (4, 4)]:
        l = rng.standard_normal((25, E)) * 2
        b = rng.standard_normal(E) * 0.2
        ids, w = om.route_scored(l, b, k, "sigmoid")
        for t in range(25):
            key = [sig(l[t, i]) + b[i] for i in range(E)]
            best = max(itertools.combinations(range(E), k), key=lambda s: sum(key[i] for i in s))
            assert ids[t].tolist() == sorted(best, key=lambda i: -key[i])
            s = scipy.special.expit(l[t, ids[t]])
            np.testing.assert_allclose(w[t], s / s.sum(), rtol=1e-14)


def test_sigmoid_extreme_logits_stay_finite():
    l = np.array([[800.0, -800.0, 0.0, -30.0]])
    ids, w = om.route_scored(l, None, 4, "sigmoid")
    assert ids[0].tolist() == [0, 2, 3, 1]
    assert np.all(np.isfinite(w)) and w[0, 3] == 0.0
    np.testing.assert_allclose(w[0, :2], [2 / 3, 1 / 3], rtol=1e-12)
    with pytest.raises(ValueError):
        om.route_scored(l, None, 2, "tanh")


def test_identical_experts_give_dense_ffn_under_every_scoring():
    rng = np.random.default_rng(25)
    T, H, E, I, k = 10, 16, 6, 8, 3
    x = _bf(rng, (T, H), 1)
    gu1, d1 = _bf(rng, (H, 2 * I), 0.3), _bf(rng, (I, H), 0.3)
    Wgu, Wd = np.stack([gu1] * E), np.stack([d1] * E)
    Wr = rng.standard_normal((H, E)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32)
    dense = om.dense_swiglu_ffn(x, gu1, d1)
    for scoring in om.SCORINGS:
        out = om.layer_forward(x, Wr, b, Wgu, Wd, k, scoring=scoring)
        np.testing.assert_allclose(out["y"], dense, rtol=1e-12, atol=1e-14)
        ids, _ = om.route_scored(om.router_logits(x, Wr, None), b, k, scoring)
        np.testing.assert_array_equal(out["ids"], ids)


def test_gap_guarantee_holds_on_sigmoid_keys():
    cfg = synth.Config("gap_sig", T=64, H=256, E=16, I=128, k=4, bias="zipf:0.05")
    inp = synth.make_inputs(cfg)
    oracle.enforce_logit_gap(inp, scoring="sigmoid")
    keys = om.selection_keys(om.router_logits(inp.x, inp.w_router, None), inp.bias, "sigmoid")
    top = -np.sort(-keys, axis=1)[:, :cfg.k + 1]
    assert np.all(top[:, :-1] - top[:, 1:] >= synth.gap_target())


# ---------------------------------------------------------------- permutation

def _random_ids(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


def test_permutation_invariants_and_stable_order():
    rng = np.random.default_rng(6)
    for T, E, k in [(1, 4, 2), (37, 8, 3), (64, 5, 5), (100, 16, 1)]:
        ids = _random_ids(rng, T, E, k)
        counts, offsets, sids, inv = om.permute(ids, E)
        assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
        assert np.all(np.diff(offsets) == counts)
        # brute force: sort (expert, token) pairs
        want = [t for e, t in sorted((int(ids[t, j]), t) for t in range(T) for j in range(k))]
        assert sids.tolist() == want
        # each slot exactly once; permute then un-permute is the identity
        assert sorted(inv.reshape(-1).tolist()) == list(range(T * k))
        vals = rng.standard_normal((T, k))
        permuted = np.empty(T * k)
        permuted[inv.reshape(-1)] = vals.reshape(-1)
        np.testing.assert_array_equal(permuted[inv], vals)
        for t in range(T):
            for j in range(k):
                r = inv[t, j]
                assert sids[r] == t and offsets[ids[t, j]] <= r < offsets[ids[t, j] + 1]


def test_permutation_empty_experts_and_single_hot_expert():
    ids = np.full((10, 1), 3, np.int32)
    counts, offsets, sids, inv = om.permute(ids, 6)
    assert counts.tolist() == [0, 0, 0, 10, 0, 0]
    assert offsets.tolist() == [0, 0, 0, 0, 10, 10, 10]
    assert sids.tolist() == list(range(10)) and inv[:, 0].tolist() == list(range(10))


# ---------------------------------------------------------------- FFN, combine

def _worked_example():
    """Two tokens, H=2, E=3, I=1, k=2; every input exact in bf16.

    x0 = [1,0] -> logits [2,1,0]: experts (0,1), weights (sig(1), sig(-1)).
    x1 = [0,1] -> logits [0,.5,1]: experts (2,1), weights (sig(.5), sig(-.5)).
    Expert 0: g = x0, u = 2 x0, down [1,-1].  Expert 1: g = -x0 + 2 x1,
    u = x0 + x1, down [.5, 2].  Expert 2: g = x1, u = -3 x1, down [1, 1].
    """
    x = np.array([[1, 0], [0, 1]], np.float32)
    Wr = np.array([[2, 1, 0], [0, 0.5, 1]], np.float32)
    Wgu = np.array([[[1, 2], [0, 0]],
                    [[-1, 1], [2, 1]],
                    [[0, 0], [1, -3]]], np.float32)      # [E, H, 2I]: col 0 gate, col 1 up
    Wd = np.array([[[1, -1]], [[0.5, 2]], [[1, 1]]], np.float32)  # [E, I, H]
    # closed forms: silu(1) = sig(1); silu(-1) = -sig(-1); silu(2) = 2 sig(2)
    h00 = 2 * sig(1)            # token 0, expert 0: silu(1) * 2
    h01 = -sig(-1)              # token 0, expert 1: silu(-1) * 1
    h11 = 2 * sig(2)            # token 1, expert 1: silu(2) * 1
    h12 = -3 * sig(1)           # token 1, expert 2: silu(1) * -3
    y0 = [sig(1) * h00 * 1 + sig(-1) * h01 * 0.5, sig(1) * h00 * -1 + sig(-1) * h01 * 2]
    y1 = [sig(0.5) * h12 * 1 + sig(-0.5) * h11 * 0.5, sig(0.5) * h12 * 1 + sig(-0.5) * h11 * 2]
    return x, Wr, Wgu, Wd, np.array([y0, y1])


def test_worked_example_closed_form():
    x, Wr, Wgu, Wd, y = _worked_example()
    out = om.layer_forward(bits(x), Wr, None, bits(Wgu), bits(Wd), 2)
    assert out["ids"].tolist() == [[0, 1], [2, 1]]
    np.testing.assert_allclose(out["w"], [[sig(1), sig(-1)], [sig(0.5), sig(-0.5)]], rtol=1e-14)
    np.testing.assert_allclose(out["y"], y, rtol=1e-13)


def test_worked_example_shared_expert_added_with_weight_one():
    x, Wr, Wgu, Wd, y = _worked_example()
    Wsgu = np.array([[1, 1], [1, 1]], np.float32)   # g = u = x0 + x1 = 1 for both tokens
    Wsd = np.array([[2, -4]], np.float32)
    s = sig(1) * 1                                  # silu(1) * 1
    out = om.layer_forward(bits(x), Wr, None, bits(Wgu), bits(Wd), 2, bits(Wsgu), bits(Wsd))
    np.testing.assert_allclose(out["y"], y + np.array([[2 * s, -4 * s]] * 2), rtol=1e-13)


def _bf(rng, shape, std):
    return bits(rng.standard_normal(shape) * std)


def _bruteforce_layer(x, Wr, b, Wgu, Wd, k, Wsgu=None, Wsd=None):
    """Pure-Python loops: literal softmax -> top-k -> renormalise, then per
    token and slot the SwiGLU FFN, then the weighted sum."""
    dec = om.bf16_to_f64
    xf, gu, dn = dec(x).tolist(), dec(Wgu).tolist(), dec(Wd).tolist()
    T, H = len(xf), len(xf[0])
    E = Wr.shape[1]
    I = len(gu[0][0]) // 2
    y = []
    for t in range(T):
        l = [sum(xf[t][h] * float(Wr[h, e]) for h in range(H)) + (float(b[e]) if b is not None else 0.0)
             for e in range(E)]
        z = [math.exp(v - max(l)) for v in l]
        p = [v / sum(z) for v in z]
        top = sorted(range(E), key=lambda i: (-p[i], i))[:k]
        ps = sum(p[i] for i in top)
        acc = [0.0] * H
        for e in top:
            g = [sum(xf[t][h] * gu[e][h][i] for h in range(H)) for i in range(I)]
            u = [sum(xf[t][h] * gu[e][h][I + i] for h in range(H)) for i in range(I)]
            hh = [g[i] / (1 + math.exp(-g[i])) * u[i] for i in range(I)]
            for c in range(H):
                acc[c] += p[e] / ps * sum(hh[i] * dn[e][i][c] for i in range(I))
        if Wsgu is not None:
            sg, sd = dec(Wsgu).tolist(), dec(Wsd).tolist()
            Is = len(sg[0]) // 2
            g = [sum(xf[t][h] * sg[h][i] for h in range(H)) for i in range(Is)]
            u = [sum(xf[t][h] * sg[h][Is + i] for h in range(H)) for i in range(Is)]
            hh = [g[i] / (1 + math.exp(-g[i])) * u[i] for i in range(Is)]
            for c in range(H):
                acc[c] += sum(hh[i] * sd[i][c] for i in range(Is))
        y.append(acc)
    return np.array(y)


@pytest.mark.parametrize("T,H,E,I,k,Is,bias", [(5, 8, 4, 3, 2, 0, False), (4, 6, 5, 2, 3, 4, True),
                                              (3, 4, 3, 2, 3, 0, False), (6, 5, 6, 4, 1, 0, True)])
def test_layer_matches_bruteforce_loops(T, H, E, I, k, Is, bias):
    rng = np.random.default_rng(7 + T)
    x = _bf(rng, (T, H), 1.0)
    Wr = (rng.standard_normal((H, E)) * 0.5).astype(np.float32)
    b = synth.zipf_bias(E, 1.2) if bias else None
    Wgu, Wd = _bf(rng, (E, H, 2 * I), 0.5), _bf(rng, (E, I, H), 0.5)
    Ws = (_bf(rng, (H, 2 * Is), 0.5), _bf(rng, (Is, H), 0.5)) if Is else (None, None)
    want = _bruteforce_layer(x, Wr, b, Wgu, Wd, k, *Ws)
    got = om.layer_forward(x, Wr, b, Wgu, Wd, k, *Ws)["y"]
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_single_expert_top1_is_dense_swiglu_ffn():
    rng = np.random.default_rng(8)
    T, H, I = 7, 16, 8
    x, Wgu, Wd = _bf(rng, (T, H), 1), _bf(rng, (1, H, 2 * I), 0.3), _bf(rng, (1, I, H), 0.3)
    Wr = rng.standard_normal((H, 1)).astype(np.float32)
    y = om.layer_forward(x, Wr, None, Wgu, Wd, 1)["y"]
    dec = om.bf16_to_f64
    g = dec(x) @ dec(Wgu[0])[:, :I]
    u = dec(x) @ dec(Wgu[0])[:, I:]
    dense = (g * scipy.special.expit(g) * u) @ dec(Wd[0])
    np.testing.assert_allclose(y, dense, rtol=1e-12)


def test_identical_experts_give_dense_ffn_for_any_routing():
    """Weights sum to 1, so identical experts make routing irrelevant."""
    rng = np.random.default_rng(9)
    T, H, E, I, k = 12, 16, 6, 8, 3
    x = _bf(rng, (T, H), 1)
    gu1, d1 = _bf(rng, (H, 2 * I), 0.3), _bf(rng, (I, H), 0.3)
    Wgu, Wd = np.stack([gu1] * E), np.stack([d1] * E)
    Wr = rng.standard_normal((H, E)).astype(np.float32)
    y = om.layer_forward(x, Wr, None, Wgu, Wd, k)["y"]
    np.testing.assert_allclose(y, om.dense_swiglu_ffn(x, gu1, d1), rtol=1e-12, atol=1e-14)
    # and with the shared expert equal to them, the output doubles
    y2 = om.layer_forward(x, Wr, None, Wgu, Wd, k, gu1, d1)["y"]
    np.testing.assert_allclose(y2, 2 * y, rtol=1e-12, atol=1e-14)


def test_zero_routed_down_leaves_only_shared_expert():
    rng = np.random.default_rng(10)
    T, H, E, I, k, Is = 9, 16, 5, 8, 2, 12
    x = _bf(rng, (T, H), 1)
    Wgu, Wd = _bf(rng, (E, H, 2 * I), 0.3), np.zeros((E, I, H), np.uint16)
    sgu, sd = _bf(rng, (H, 2 * Is), 0.3), _bf(rng, (Is, H), 0.3)
    Wr = rng.standard_normal((H, E)).astype(np.float32)
    y = om.layer_forward(x, Wr, None, Wgu, Wd, k, sgu, sd)["y"]
    np.testing.assert_allclose(y, om.dense_swiglu_ffn(x, sgu, sd), rtol=1e-13)


def test_expert_relabelling_and_token_order_equivariance():
    rng = np.random.default_rng(11)
    T, H, E, I, k = 10, 16, 7, 8, 3
    x = _bf(rng, (T, H), 1)
    Wr = rng.standard_normal((H, E)).astype(np.float32)
    Wgu, Wd = _bf(rng, (E, H, 2 * I), 0.3), _bf(rng, (E, I, H), 0.3)
    y = om.layer_forward(x, Wr, None, Wgu, Wd, k)["y"]
    p = rng.permutation(E)
    y_relabel = om.layer_forward(x, Wr[:, p], None, Wgu[p], Wd[p], k)["y"]
    np.testing.assert_allclose(y_relabel, y, rtol=1e-12, atol=1e-14)
    q = rng.permutation(T)
    y_perm = om.layer_forward(x[q], Wr, None, Wgu, Wd, k)["y"]
    np.testing.assert_allclose(y_perm, y[q], rtol=1e-12, atol=1e-14)


def test_gate_and_up_halves_are_not_interchangeable():
    """Swapping the halves of W_gate_up must change y (catches a column mix-up)."""
    rng = np.random.default_rng(12)
    T, H, E, I, k = 6, 16, 4, 8, 2
    x = _bf(rng, (T, H), 1)
    Wr = rng.standard_normal((H, E)).astype(np.float32)
    Wgu, Wd = _bf(rng, (E, H, 2 * I), 0.3), _bf(rng, (E, I, H), 0.3)
    swapped = np.concatenate([Wgu[:, :, I:], Wgu[:, :, :I]], axis=2)
    a = om.layer_forward(x, Wr, None, Wgu, Wd, k)["y"]
    b = om.layer_forward(x, Wr, None, swapped, Wd, k)["y"]
    assert np.abs(a - b).max() > 1e-3 * np.abs(a).max()


def test_token_subset_path_agrees_with_full_layer():
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(cfg)
    full = om.layer_forward(inp.x, inp.w_router, inp.bias, inp.w_gate_up, inp.w_down, cfg.k)
    toks = [0, 5, 17, 63]
    sub = om.layer_forward_tokens(inp.x, toks, full["ids"], full["w"],
                                  lambda e: inp.w_gate_up[e], lambda e: inp.w_down[e])
    np.testing.assert_allclose(sub, full["y"][toks], rtol=1e-12, atol=1e-15)
    y2 = om.down_combine(full["h"], full["offsets"], full["inv_perm"], full["w"],
                         lambda e: inp.w_down[e])
    np.testing.assert_allclose(y2, full["y"], rtol=1e-13, atol=1e-16)


def test_token_subset_path_with_shared_expert_matches_bruteforce_loops():
    """The per-token path's shared-expert branch (the checker of the full-size
    Ling-like parity test) against the pure-Python loops: the shared FFN is
    added once per token with weight 1, over its own I_s split of the
    columns.  Dropping the branch, scaling it by a routing weight or
    splitting [H, 2 I_s] at the routed I would each fail here."""
    rng = np.random.default_rng(21)
    T, H, E, I, k, Is = 6, 8, 5, 3, 2, 4
    x = _bf(rng, (T, H), 1.0)
    Wr = (rng.standard_normal((H, E)) * 0.5).astype(np.float32)
    b = synth.zipf_bias(E, 1.2)
    Wgu, Wd = _bf(rng, (E, H, 2 * I), 0.5), _bf(rng, (E, I, H), 0.5)
    sgu, sd = _bf(rng, (H, 2 * Is), 0.5), _bf(rng, (Is, H), 0.5)
    want = _bruteforce_layer(x, Wr, b, Wgu, Wd, k, sgu, sd)
    ids, w = om.topk_route(om.router_logits(x, Wr, b), k)
    toks = [0, 2, 5]
    got = om.layer_forward_tokens(x, toks, ids, w, lambda e: Wgu[e], lambda e: Wd[e], sgu, sd)
    np.testing.assert_allclose(got, want[toks], rtol=1e-11, atol=1e-12)
    without = om.layer_forward_tokens(x, toks, ids, w, lambda e: Wgu[e], lambda e: Wd[e])
    assert np.abs(got - without).max() > 1e-2 * np.abs(got).max()


def test_token_subset_path_worked_example_with_shared_expert():
    """The two-token worked example through the per-token path: the shared
    term 2*silu(1), -4*silu(1) is added to each token's closed-form output."""
    x, Wr, Wgu, Wd, y = _worked_example()
    Wsgu = np.array([[1, 1], [1, 1]], np.float32)
    Wsd = np.array([[2, -4]], np.float32)
    s = sig(1)
    ids, w = om.topk_route(om.router_logits(bits(x), Wr), 2)
    got = om.layer_forward_tokens(bits(x), [1, 0], ids, w, lambda e: bits(Wgu)[e], lambda e: bits(Wd)[e],
                                  bits(Wsgu), bits(Wsd))
    np.testing.assert_allclose(got, (y + np.array([[2 * s, -4 * s]] * 2))[[1, 0]], rtol=1e-13)


# ---------------------------------------------------------------- inputs

def test_logit_gap_enforcement():
    cfg = synth.CONFIGS["tiny"].with_(T=256)
    inp = synth.make_inputs(cfg)
    before = oracle.gap.bad_gap_rows(inp.x, inp.w_router, inp.bias, cfg.k, 1e-3)
    x0 = inp.x.copy()
    n = oracle.enforce_logit_gap(inp)
    assert n >= before.size
    assert oracle.gap.bad_gap_rows(inp.x, inp.w_router, inp.bias, cfg.k, 1e-3).size == 0
    changed = np.nonzero((inp.x != x0).any(1))[0]
    assert set(changed.tolist()) <= set(before.tolist())   # only failing rows are redrawn
    inp2 = synth.make_inputs(cfg)
    oracle.enforce_logit_gap(inp2)
    np.testing.assert_array_equal(inp2.x, inp.x)


def test_zipf_bias_makes_expert_zero_hottest():
    cfg = synth.CONFIGS["ling_skewed_t4096"].with_(T=256, H=512)
    b = synth.zipf_bias(cfg.E, 1.2)
    assert b[0] == 0.0 and b[9] == pytest.approx(-1.2 * math.log(10))
    inp = synth.make_inputs(cfg, experts=False)
    ids, _ = om.topk_route(om.router_logits(inp.x, inp.w_router, inp.bias), cfg.k)
    counts = np.bincount(ids.reshape(-1), minlength=cfg.E)
    assert counts.argmax() == 0 and counts[0] > 0.5 * cfg.T


def test_oracle_matches_frozen_tiny_regression():
    """Guards against unintended changes to the oracle's arithmetic (the
    fixture is written by tests/golden/make_golden.py from the oracle)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_regression.npz")
    want = np.load(path)
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(cfg)
    oracle.enforce_logit_gap(inp)
    import hashlib
    assert hashlib.sha256(inp.x.tobytes()).digest() == want["x_sha256"].tobytes()
    got = om.layer_forward(inp.x, inp.w_router, inp.bias, inp.w_gate_up, inp.w_down, cfg.k)
    for key in ("ids", "offsets", "sorted_token_ids"):
        np.testing.assert_array_equal(got[key], want[key])
    np.testing.assert_allclose(got["w"], want["w"], rtol=1e-13)
    np.testing.assert_allclose(got["y"][:8], want["y8"], rtol=1e-12, atol=1e-15)
