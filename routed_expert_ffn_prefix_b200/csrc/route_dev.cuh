// route_dev.cuh -- device pieces of the router shared by the router kernels
// (route.cu) and the persistent few-token layer (layer_small.cu): the warp
// top-k and the split-H partial logits of a few tokens.
#pragma once

#include "kernels.h"

namespace moe {

// Top-k of one token by one warp: lane L holds the selection keys of
// experts L + 32 i in v (entries >= E ignored).  k rounds of a warp arg-max
// (larger key first, ties to the lower expert id; NaN keys are never
// chosen), then the weights.  Each round takes the lane's best by a pairwise
// tree over its EPL entries (log2 EPL dependent steps) and the warp's best by
// 5 shuffles.  sel, if given, receives the k ids too (shared memory of the
// caller).
//
// Weights.  SEL = false (softmax scoring, bias inside the logits): the keys
// are the logits and w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the k
// selected.  SEL = true (the bias steers only the selection): the weights
// come from the unbiased per-expert values in `src` -- logits, normalised as
// a softmax over the selected (exp_w), or sigmoid scores normalised by
// their sum (!exp_w).  Lane j % 32 keeps the source value of slot j; the
// max and the sum run over fixed shuffle trees.
constexpr int kNoExpert = 0x7fffffff;

__device__ __forceinline__ bool topk_better(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

// Non-NaN float -> unsigned integer with the same order (larger float,
// larger integer; -0 taken as +0, as the float comparison does; -inf the
// smallest value above 0), and back.  0 is left for "no candidate".
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = f == 0.f ? 0u : __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Expert held in entry i of a lane's EPL logits: scalar layout e = lane + 32 i;
// quad layout (16-byte loads, E % 4 == 0) e = 128 (i / 4) + 4 lane + i % 4.
template <bool QUAD>
__device__ __forceinline__ int entry_expert(int lane, int i) {
  return QUAD ? 128 * (i >> 2) + 4 * lane + (i & 3) : lane + 32 * i;
}

// Lane holding expert e (inverse of entry_expert).
template <bool QUAD>
__device__ __forceinline__ int entry_lane(int e) {
  return QUAD ? (e >> 2) & 31 : e & 31;
}

__device__ __forceinline__ float sigmoid_score(float z) { return 1.0f / (1.0f + expf(-z)); }

template <int EPL, bool QUAD = false, bool SEL = false>
__device__ __forceinline__ void warp_topk(const float (&vin)[EPL], const float (&src)[EPL], bool exp_w, int E, int k,
                                          int t, int32_t* idrow, float* wrow, int32_t* sel, DevStatus* st) {
  const int lane = threadIdx.x & 31;
  float v[EPL];
  int id[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = entry_expert<QUAD>(lane, i);
    const bool ok = e < E && !isnan(vin[i]);
    v[i] = ok ? vin[i] : -INFINITY;
    id[i] = ok ? e : kNoExpert;
  }
  float lead = 0.f, sum = 0.f;
  float held0 = 0.f, held1 = 0.f;  // values of slots lane and lane + 32 (SEL: sources; else numerators)
  for (int j = 0; j < k; ++j) {
    float tv[EPL];
    int ti[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) { tv[i] = v[i]; ti[i] = id[i]; }
#pragma unroll
    for (int w = 1; w < EPL; w <<= 1)
#pragma unroll
      for (int i = 0; i + w < EPL; i += 2 * w)
        if (topk_better(tv[i + w], ti[i + w], tv[i], ti[i])) { tv[i] = tv[i + w]; ti[i] = ti[i + w]; }
    // The warp's best: the largest key by one warp reduction over an
    // order-preserving unsigned encoding of the lanes' bests, then the lowest
    // expert id among the lanes holding that key by a second one.
    const uint32_t lane_key = ti[0] == kNoExpert ? 0u : ordered_key(tv[0]);
    const uint32_t best_key = __reduce_max_sync(0xffffffffu, lane_key);
    int bi = (int)__reduce_min_sync(0xffffffffu, lane_key == best_key ? (uint32_t)ti[0] : (uint32_t)kNoExpert);
    float bv = key_value(best_key);
    if (bi == kNoExpert) {  // no candidate left: the keys were NaN
      if (lane == 0) raise_error(st, MOE_ERR_DEVICE_BOUNDS, SITE_TOPK, t);
      bi = 0;
      bv = lead;
    }
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (id[i] == bi) {
        v[i] = -INFINITY;
        id[i] = kNoExpert;
        if constexpr (SEL) mine = src[i];
      }
    if constexpr (SEL) {
      const float ws = __shfl_sync(0xffffffffu, mine, entry_lane<QUAD>(bi));
      if (lane == (j & 31)) {
        if (j < 32) held0 = ws;
        else held1 = ws;
      }
      if (lane == 0) {
        idrow[j] = bi;
        if (sel) sel[j] = bi;
      }
    } else {
      if (j == 0) lead = bv;
      const float z = expf(bv - lead);
      sum += z;
      if (lane == (j & 31)) {  // slot j's numerator stays in a register of lane j % 32
        if (j < 32) held0 = z;
        else held1 = z;
      }
      if (lane == 0) {
        idrow[j] = bi;
        if (sel) sel[j] = bi;
      }
    }
  }
  if constexpr (SEL) {
    const bool h0 = lane < k, h1 = lane + 32 < k;
    float z0 = h0 ? held0 : 0.f, z1 = h1 ? held1 : 0.f;
    if (exp_w) {
      float m = h0 ? held0 : -INFINITY;
      if (h1) m = fmaxf(m, held1);
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
      z0 = h0 ? expf(held0 - m) : 0.f;
      z1 = h1 ? expf(held1 - m) : 0.f;
    }
    float tot = z0 + z1;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, d);
    if (h0) wrow[lane] = z0 / tot;  // a division: one selected expert gets exactly 1
    if (h1) wrow[lane + 32] = z1 / tot;
  } else {
    const float inv = 1.0f / sum;
    if (lane < k) wrow[lane] = held0 * inv;
    if (lane + 32 < k) wrow[lane + 32] = held1 * inv;
  }
}

// Selection keys and weight sources of one lane's entries from its unbiased
// logits v (in place: v becomes the keys), per scoring rule (MOE_SCORE_*):
// softmax: key = l + b; select-only bias: key = l + b, src = l; sigmoid:
// src = sigmoid(l), key = src + b.  Entries >= E get key -inf.
template <int EPL, bool QUAD>
__device__ __forceinline__ void score_entries(float (&v)[EPL], float (&src)[EPL], const float* __restrict__ bias,
                                              int E, int lane, int scoring) {
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = entry_expert<QUAD>(lane, i);
    const float l = v[i];
    const float sv = scoring == MOE_SCORE_SIGMOID ? sigmoid_score(l) : l;
    src[i] = e < E ? sv : 0.f;
    v[i] = e < E ? sv + (bias ? bias[e] : 0.f) : -INFINITY;
  }
}

// ---------------------------------------------------------------- few tokens
// For T <= kSmallRouterT the logits are a matrix-vector product whose cost is
// reading W_router (H x E fp32) once, so the work is spread over ~148 blocks:
// block item (cs, hy) owns W columns [8 cs, 8 cs + 8) (one 32-byte sector per
// row) and rows [hy * chunk, (hy + 1) * chunk).  Each thread streams its rows
// as float4s (all issued before any is used), multiplies them by the bf16 x
// staged in shared memory and the block reduces over its rows in a fixed
// order into partial slab hy.
constexpr int kSmallThreads = 256;
constexpr int kSmallCols = 8;
constexpr int kSmallPass = 128;  // rows per block pass: 8 warps x 16
constexpr int kSmallIters = 8;   // passes per block: chunk <= 1024 rows
constexpr int kSmallMaxSlots = kSmallRouterT * 64;

struct SmallGrid {
  int ncs, hs, chunk;
};

__host__ __device__ inline SmallGrid small_grid(int H, int E) {
  SmallGrid g;
  g.ncs = (E + kSmallCols - 1) / kSmallCols;
  int hs = 148 / g.ncs;
  const int hs_min = (H + kSmallPass * kSmallIters - 1) / (kSmallPass * kSmallIters);
  if (hs < hs_min) hs = hs_min;
  if (hs < 1) hs = 1;
  g.chunk = (((H + hs - 1) / hs) + 15) & ~15;
  g.hs = (H + g.chunk - 1) / g.chunk;
  return g;
}

// Barrier among the kSmallThreads threads running a router piece: the whole
// block (BAR = 0, a block of kSmallThreads), or named barrier BAR among
// threads [0, kSmallThreads) of a larger block (the persistent layer kernel,
// whose other warps skip the router pieces).
template <int BAR>
__device__ __forceinline__ void router_sync() {
  if constexpr (BAR == 0) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(kSmallThreads) : "memory");
  }
}

// Shared memory of one partial-logits item (TT tokens).
template <int TT>
struct RouterSmem {
  __nv_bfloat16 xs[TT][kSmallPass * kSmallIters];
  float red[kSmallThreads / 32][TT][kSmallCols];
};

// Partial logits of item (cs, hy) for T <= TT tokens into slab hy of
// partial [hs][T][E].  Called by all kSmallThreads threads of a block;
// ends with the partial written (no fence).
template <int TT, int BAR = 0>
__device__ __forceinline__ void router_partial(const __nv_bfloat16* __restrict__ x, const float* __restrict__ w,
                                               int T, int H, int E, int chunk, int cs, int hy,
                                               float* __restrict__ partial, RouterSmem<TT>& sm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h0 = hy * chunk, h1 = min(H, h0 + chunk);
  const int q = lane & 1, r = lane >> 1;
  const int c0 = cs * kSmallCols + q * 4;
  const bool cval = c0 < E;  // E % 4 == 0: a quad is all in or all out

  float4 wr[kSmallIters];
#pragma unroll
  for (int i = 0; i < kSmallIters; ++i) {
    const int h = h0 + warp * 16 + r + kSmallPass * i;
    wr[i] = (cval && h < h1) ? __ldcs(reinterpret_cast<const float4*>(w + (size_t)h * E + c0))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // x rows [h0, h1) of every token, zero beyond T and h1
  constexpr int kVec = kSmallPass * kSmallIters / 8;  // 16-byte vectors per staged row
  for (int i = tid; i < TT * kVec; i += kSmallThreads) {
    const int t = i / kVec, v = i - t * kVec, h = h0 + v * 8;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t < T && h < h1) val = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + h));
    reinterpret_cast<uint4*>(&sm.xs[t][0])[v] = val;
  }
  router_sync<BAR>();
  float acc[TT][4];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
  for (int i = 0; i < kSmallIters; ++i) {
    const int hl = warp * 16 + r + kSmallPass * i;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float xv = __bfloat162float(sm.xs[t][hl]);
      acc[t][0] = fmaf(xv, wr[i].x, acc[t][0]);
      acc[t][1] = fmaf(xv, wr[i].y, acc[t][1]);
      acc[t][2] = fmaf(xv, wr[i].z, acc[t][2]);
      acc[t][3] = fmaf(xv, wr[i].w, acc[t][3]);
    }
  }
  // rows of a warp (lane bits 1..4), then the 8 warps in order
#pragma unroll
  for (int d = 2; d < 32; d <<= 1)
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] += __shfl_xor_sync(0xffffffffu, acc[t][j], d);
  if (r == 0) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) sm.red[warp][t][q * 4 + j] = acc[t][j];
  }
  router_sync<BAR>();
  if (tid < TT * kSmallCols) {
    const int t = tid / kSmallCols, c = tid - t * kSmallCols;
    float sum = 0.f;
#pragma unroll
    for (int v = 0; v < kSmallThreads / 32; ++v) sum += sm.red[v][t][c];
    const int e = cs * kSmallCols + c;
    if (t < T && e < E) partial[((size_t)hy * T + t) * E + e] = sum;
  }
}

// Slab sum (slab order), scoring (MOE_SCORE_*), top-k of token t by the
// calling warp.
template <int EPL>
__device__ __forceinline__ void router_select(const float* partial, int hs, const float* __restrict__ bias, int T,
                                              int E, int k, int scoring, int t, int32_t* idrow, float* wrow,
                                              int32_t* sel, DevStatus* st) {
  const int lane = threadIdx.x & 31;
  float v[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) v[i] = 0.f;
  // G slabs loaded together, then added in slab order
  constexpr int G = EPL <= 8 ? 4 : (EPL <= 16 ? 2 : 1);
  int sp = 0;
  for (; sp + G <= hs; sp += G) {
    float p[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float* slab = partial + ((size_t)(sp + g) * T + t) * E;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        p[g][i] = e < E ? __ldcg(slab + e) : 0.f;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < EPL; ++i) v[i] += p[g][i];
  }
  for (; sp < hs; ++sp) {
    const float* slab = partial + ((size_t)sp * T + t) * E;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) v[i] += __ldcg(slab + e);
    }
  }
  float src[EPL];
  score_entries<EPL, false>(v, src, bias, E, lane, scoring);
  if (scoring == MOE_SCORE_SOFTMAX)
    warp_topk<EPL, false, false>(v, v, true, E, k, t, idrow, wrow, sel, st);
  else
    warp_topk<EPL, false, true>(v, src, scoring == MOE_SCORE_SOFTMAX_SELECT_BIAS, E, k, t, idrow, wrow, sel, st);
}

// The last block of the few-token router (kSmallThreads threads, barrier
// BAR): sums the partial slabs in slab order, selects each token's top-k
// under the scoring rule (one warp per token) and, if offsets != nullptr,
// writes the expert-contiguous permutation of the n = T*k slots (a stable
// counting sort: experts ascending, slot order within an expert), as the
// permutation kernels do; counts may be nullptr.  The outputs may be global
// or shared memory.  sel [T*k], cnt [E] and warp_sums [kSmallThreads/32]
// are shared memory of the caller.
template <int EPL, int BAR = 0>
__device__ __forceinline__ void router_finish(const float* partial, int hs, const float* __restrict__ bias, int T,
                                              int E, int k, int scoring, int32_t* ids, float* wout,
                                              int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                                              int32_t* inv_perm, DevStatus* st, int32_t* sel, int32_t* cnt,
                                              int32_t* warp_sums) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < T; t += kSmallThreads / 32)
    router_select<EPL>(partial, hs, bias, T, E, k, scoring, t, ids + (size_t)t * k, wout + (size_t)t * k,
                       sel + t * k, st);
  if (offsets == nullptr) return;
  // ---- permutation of the n = T*k slots, stable counting sort by expert
  const int n = T * k;
  for (int e = tid; e < E; e += kSmallThreads) cnt[e] = 0;
  router_sync<BAR>();
  for (int s = tid; s < n; s += kSmallThreads) atomicAdd(&cnt[sel[s]], 1);
  router_sync<BAR>();
  constexpr int EPT = kMaxExperts / kSmallThreads;  // experts per thread in the scan
  int loc[EPT], tot = 0;
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = tid * EPT + j;
    loc[j] = e < E ? cnt[e] : 0;
    tot += loc[j];
  }
  int incl = tot;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  router_sync<BAR>();
  int base = incl - tot;
  for (int v = 0; v < warp; ++v) base += warp_sums[v];
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = tid * EPT + j;
    if (e < E) {
      if (counts) counts[e] = loc[j];
      offsets[e] = base;
      cnt[e] = base;  // running position of expert e
    }
    base += loc[j];
  }
  if (tid == 0) offsets[E] = n;
  router_sync<BAR>();
  if (warp == 0) {
    for (int s0 = 0; s0 < n; s0 += 32) {
      const int s = s0 + lane;
      const int e = s < n ? sel[s] : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = e >= 0 ? cnt[e] + rank : -1;
      __syncwarp();
      if (e >= 0 && rank == 0) cnt[e] += __popc(peers);
      __syncwarp();
      if (e >= 0) {
        sorted_ids[pos] = s / k;
        inv_perm[s] = pos;
      }
    }
  }
}

}  // namespace moe
