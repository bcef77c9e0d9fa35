"""CPU oracle for the routed-expert MoE FFN layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  The CUDA library never calls it, and it shares
no code with the library: it reads the same input bytes (bf16 bit patterns,
fp32 router weights) and computes everything in float64 with plain numpy.

What it computes (plain definitions, in the order the layer applies them):

1. Router logits  l[t,e] = sum_h x[t,h] * W_router[h,e]  (+ bias[e]).
   The pages name routing and top-k as the first stage of the MoE path
   (Qwen-3.5-397B-on-Ironwood page, sec. 4.2 "MoE track"; sec. 8.2 "router
   gating and top-k fusion"); the benchmark configurations fix the rule:
   softmax over the router logits, then top-k, then renormalise.
2. Top-k: a full sort of each token's logits by (logit descending, expert id
   ascending), first k kept.  Softmax is monotone, so this is the top-k of
   the softmax probabilities.
3. Weights  w_j = p_j / sum_{i in top-k} p_i  with p = softmax(l).  The full
   softmax denominator cancels, so w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
   over the k selected logits (l_0 = the largest).
4. Permutation into expert-contiguous order (the "scatter into each expert's
   input buffer" of the Ling-2.6-1T / SGLang-JAX page, "routing + FFN +
   gather" paragraph; the ragged gather of the Qwen page, sec. 4.2): a stable
   counting sort of the flattened slots s = t*k + j by expert id, so rows are
   expert-major and token-ascending within an expert.
5. Expert FFN with SwiGLU (Qwen page sec. 4.2, "grouped GEMM V2 with fused
   activation"): [g, u] = x[t] @ W_gate_up[e] (columns [0,I) gate, [I,2I) up),
   h = silu(g) * u with silu(z) = z * sigmoid(z), o = h @ W_down[e].
6. Weighted gather-combine back to token order (Qwen page sec. 7.2,
   un-permute and gather-reduce; Ling page, Fused MoE V2):
   y[t] = sum_{j=0}^{k-1} w[t,j] * o[t,j]  (+ shared-expert FFN of x[t] with
   weight 1 when the layer has one -- "top-8 routing plus a shared expert",
   Ling page, introduction).

Router scoring variants (steps 1-3 replaced; everything after is unchanged).
The systems-engineering handbook page on Qwen 3.5-397B MoE on Ironwood
("key optimisations", step 1 "expert load balancing") names hot experts and
a balancing term in the router but gives no formula, and the Ling page says
only that router logits get a per-expert bias.  Besides the rule above (bias added to the logits, so it moves both
selection and weights: scoring "softmax"), two plain forms in which a
per-expert bias b steers only which experts are picked are supported:

- "softmax_select_bias": the k experts with the largest l + b (descending,
  ties to the lower id) are selected; their weights are the softmax of the
  unbiased logits over the selected set, w_j = exp(l_j) / sum_i exp(l_i).
- "sigmoid": s = sigmoid(l) per expert; the k experts with the largest
  s + b are selected (same order rule); w_j = s_j / sum_i s_i over them.

Without a bias both select exactly what "softmax" selects (sigmoid and
exp are monotone); the weights differ for "sigmoid".

Nothing is rounded to bf16 inside the oracle; y stays float64.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_to_f64", "router_logits", "topk_route", "permute", "silu", "swiglu_ffn_rows",
    "expert_down_rows", "dense_swiglu_ffn", "layer_forward", "layer_forward_tokens",
    "h_rows", "down_combine", "SCORINGS", "selection_keys", "route_scored",
    "TEST_INFRASTRUCTURE_ONLY",
]

SCORINGS = ("softmax", "softmax_select_bias", "sigmoid")

TEST_INFRASTRUCTURE_ONLY = True


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly.

    A bf16 value is the top half of an fp32 word, so shifting the 16 bits
    into the high half of a uint32 gives the fp32 value, which widens to
    float64 without rounding.
    """
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def router_logits(x_bits: np.ndarray, w_router: np.ndarray, bias: np.ndarray | None = None
                  ) -> np.ndarray:
    """Step 1: l = x @ W_router (+ bias), float64.  x [T,H] bf16 bits, W [H,E] fp32."""
    l = bf16_to_f64(x_bits) @ np.asarray(w_router, np.float64)
    if bias is not None:
        l = l + np.asarray(bias, np.float64)[None, :]
    return l


def topk_route(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """Steps 2-3: ids [T,k] int32 (descending logit, ties to the lower id) and
    renormalised softmax weights [T,k] float64."""
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    expert = np.arange(E)
    for t in range(T):
        # lexsort: last key is primary -> sort by -logit, then by expert id
        order = np.lexsort((expert, -logits[t]))
        sel = order[:k]
        ids[t] = sel
        z = np.exp(logits[t, sel] - logits[t, sel[0]])
        w[t] = z / z.sum()
    return ids, w


def _sigmoid(z: np.ndarray) -> np.ndarray:
    """1 / (1 + exp(-z)), evaluated without overflow for either sign."""
    z = np.asarray(z, np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def selection_keys(l_raw: np.ndarray, bias, scoring: str) -> np.ndarray:
    """The per-expert value whose k largest decide the selection, from the
    unbiased logits l_raw [T,E]: l + b ("softmax", "softmax_select_bias") or
    sigmoid(l) + b ("sigmoid")."""
    if scoring not in SCORINGS:
        raise ValueError(f"unknown scoring {scoring!r}")
    l = np.asarray(l_raw, np.float64)
    base = _sigmoid(l) if scoring == "sigmoid" else l
    if bias is None:
        return base
    return base + np.asarray(bias, np.float64)[None, :]


def route_scored(l_raw: np.ndarray, bias, k: int, scoring: str = "softmax"
                 ) -> tuple[np.ndarray, np.ndarray]:
    """Steps 2-3 under a scoring rule (module docstring): ids [T,k] int32 in
    descending key order (ties to the lower id) and weights [T,k] float64 in
    the same slot order."""
    keys = selection_keys(l_raw, bias, scoring)
    if scoring == "softmax":
        return topk_route(keys, k)
    T, E = keys.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    l = np.asarray(l_raw, np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    expert = np.arange(E)
    for t in range(T):
        sel = np.lexsort((expert, -keys[t]))[:k]
        ids[t] = sel
        if scoring == "softmax_select_bias":
            z = np.exp(l[t, sel] - l[t, sel].max())
        else:
            z = _sigmoid(l[t, sel])
        w[t] = z / z.sum()
    return ids, w


def permute(ids: np.ndarray, E: int):
    """Step 4: counts [E], offsets [E+1] (exclusive prefix sum, offsets[E] = T*k),
    sorted_token_ids [T*k] (permuted row -> token), inv_perm [T,k] (slot -> row)."""
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].astype(np.int64).copy()
    sorted_token_ids = np.empty(T * k, np.int32)
    inv_perm = np.empty((T, k), np.int32)
    for s in range(T * k):          # ascending slot order -> stable
        e = flat[s]
        r = fill[e]
        fill[e] += 1
        sorted_token_ids[r] = s // k
        inv_perm[s // k, s % k] = r
    return counts, offsets, sorted_token_ids, inv_perm


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_ffn_rows(x_rows: np.ndarray, w_gate_up: np.ndarray) -> np.ndarray:
    """Step 5a: h = silu(x @ Wg) * (x @ Wu) for float64 rows; W_gate_up [H, 2I]
    given as bf16 bits or float64."""
    W = bf16_to_f64(w_gate_up) if w_gate_up.dtype == np.uint16 else w_gate_up
    I = W.shape[1] // 2
    gu = x_rows @ W
    return silu(gu[:, :I]) * gu[:, I:]


def expert_down_rows(h: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """Step 5b: o = h @ W_down; W_down [I, H] as bf16 bits or float64."""
    W = bf16_to_f64(w_down) if w_down.dtype == np.uint16 else w_down
    return h @ W


def dense_swiglu_ffn(x_bits: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """One SwiGLU FFN applied to every token (the shared expert's form)."""
    return expert_down_rows(swiglu_ffn_rows(bf16_to_f64(x_bits), w_gate_up), w_down)


def h_rows(x_bits, sorted_token_ids, offsets, expert_gate_up) -> np.ndarray:
    """h for every permuted row, float64 [T*k, I].  expert_gate_up(e) returns
    W_gate_up[e] (bf16 bits)."""
    x = bf16_to_f64(x_bits)
    E = len(offsets) - 1
    out = None
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        h = swiglu_ffn_rows(x[sorted_token_ids[a:b]], expert_gate_up(e))
        if out is None:
            out = np.zeros((int(offsets[E]), h.shape[1]), np.float64)
        out[a:b] = h
    return out


def down_combine(h, offsets, inv_perm, topk_w, expert_down, shared=None) -> np.ndarray:
    """Steps 5b + 6 from given permuted rows h [T*k, I]: o = h @ W_down[e] per
    row, y[t] = sum_j w[t,j] * o[inv_perm[t,j]] (j ascending) + shared[t]."""
    E = len(offsets) - 1
    o = None
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        oe = expert_down_rows(np.asarray(h[a:b], np.float64), expert_down(e))
        if o is None:
            o = np.zeros((int(offsets[E]), oe.shape[1]), np.float64)
        o[a:b] = oe
    T, k = inv_perm.shape
    y = np.zeros((T, o.shape[1]), np.float64)
    for j in range(k):
        y += np.asarray(topk_w, np.float64)[:, j:j + 1] * o[inv_perm[:, j]]
    if shared is not None:
        y += shared
    return y


def layer_forward(x_bits, w_router, bias, w_gate_up, w_down, k,
                  w_sh_gate_up=None, w_sh_down=None, scoring: str = "softmax") -> dict:
    """The whole layer for all tokens.  Returns y (float64 [T,H]) and every
    intermediate: logits (the selection keys), ids, w, counts, offsets,
    sorted_token_ids, inv_perm, h (float64, permuted order)."""
    E = w_router.shape[1]
    l_raw = router_logits(x_bits, w_router, None)
    logits = selection_keys(l_raw, bias, scoring)
    ids, w = route_scored(l_raw, bias, k, scoring)
    counts, offsets, sorted_ids, inv_perm = permute(ids, E)
    h = h_rows(x_bits, sorted_ids, offsets, lambda e: w_gate_up[e])
    shared = None
    if w_sh_gate_up is not None:
        shared = dense_swiglu_ffn(x_bits, w_sh_gate_up, w_sh_down)
    y = down_combine(h, offsets, inv_perm, w, lambda e: w_down[e], shared)
    return dict(y=y, logits=logits, ids=ids, w=w, counts=counts, offsets=offsets,
                sorted_token_ids=sorted_ids, inv_perm=inv_perm, h=h, shared=shared)


def layer_forward_tokens(x_bits, tokens, ids, w, expert_gate_up, expert_down,
                         w_sh_gate_up=None, w_sh_down=None) -> np.ndarray:
    """y for a subset of tokens (the per-token definition, step 5-6), given
    their routing.  expert_gate_up(e)/expert_down(e) return one expert's
    weights, so only the experts the sampled tokens use are ever widened."""
    tokens = np.asarray(tokens)
    x = bf16_to_f64(x_bits[tokens])
    by_expert: dict[int, list[tuple[int, int]]] = {}
    for n, t in enumerate(tokens):
        for j in range(ids.shape[1]):
            by_expert.setdefault(int(ids[t, j]), []).append((n, j))
    o = {}
    for e, slots in by_expert.items():
        rows = np.array([n for n, _ in slots])
        oe = expert_down_rows(swiglu_ffn_rows(x[rows], expert_gate_up(e)), expert_down(e))
        for (n, j), v in zip(slots, oe):
            o[(n, j)] = v
    H = x.shape[1]
    y = np.zeros((len(tokens), H), np.float64)
    for n, t in enumerate(tokens):
        for j in range(ids.shape[1]):
            y[n] += float(w[t, j]) * o[(n, j)]
    if w_sh_gate_up is not None:
        y += expert_down_rows(swiglu_ffn_rows(x, w_sh_gate_up), w_sh_down)
    return y
