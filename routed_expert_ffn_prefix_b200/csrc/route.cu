// route.cu -- router of the MoE layer: fp32 logits, scoring, top-k, weights.
//
// The pages put routing first on the MoE path and plan to fuse the gating
// projection with the top-k selection (Qwen 3.5-397B-on-Ironwood page,
// sec. 8.2 "router gating and top-k fusion"); the benchmark workloads fix
// the rule (softmax over the router logits, then top-k, then renormalise).
//
// Logits: two implementations.
//   * FMA: plain fp32 dot products on the CUDA cores (x is bf16, widened
//     exactly to fp32).  Used for small token counts.
//   * Tensor core: W_router (fp32) is split into three bf16 planes,
//     w = w0 + w1 + w2 (each plane carries the next 8 significand bits, so
//     the split is exact to ~2^-24 relative).  bf16 x times a bf16 plane is
//     exact in fp32, so x.w0 + x.w1 + x.w2 accumulated in fp32 by tcgen05 is
//     an fp32-accurate logit at tensor-core speed.  The three planes are
//     summed into one TMEM accumulator by the grouped GEMM (grouped_gemm.cu).
// Selection: one warp per token; each lane holds E/32 logits in registers;
// k rounds of a warp arg-max by shuffles (larger logit first, ties to the
// lower expert id); then w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the
// k selected logits, which equals softmax-then-renormalise because the full
// softmax denominator cancels.  Two further scoring rules (MOE_SCORE_*)
// select on l + b or sigmoid(l) + b and weight by the unbiased logits or
// sigmoid scores of the selected experts (route_dev.cuh); the softmax rule
// keeps its own kernel instantiation.
#include "route_dev.cuh"

namespace moe {

namespace {

__global__ void router_split_kernel(const float* __restrict__ w, int n, uint16_t* __restrict__ planes) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(p0);  // exact in fp32
    const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(p1);  // exact in fp32
    const __nv_bfloat16 p2 = __float2bfloat16_rn(r2);
    planes[i] = __bfloat16_as_ushort(p0);
    planes[(size_t)n + i] = __bfloat16_as_ushort(p1);
    planes[2 * (size_t)n + i] = __bfloat16_as_ushort(p2);
  }
}

constexpr int kFmaTok = 16;    // tokens per block
constexpr int kFmaHc = 256;    // h per shared-memory chunk
constexpr int kFmaThreads = 256;
constexpr int kFmaEPer = kMaxExperts / kFmaThreads;  // experts per thread (max)

// Block (tb, sy): tokens [16 tb, 16 tb + 16), the sy-th of gridDim.y slices of
// H (whole 256-row chunks), written to partial slab sy of `logits`.
__global__ void __launch_bounds__(kFmaThreads) router_logits_fma_kernel(const __nv_bfloat16* __restrict__ x,
                                                                        const float* __restrict__ w, int T,
                                                                        int H, int E,
                                                                        float* __restrict__ logits) {
  __shared__ float xs[kFmaTok][kFmaHc];
  const int t0 = blockIdx.x * kFmaTok;
  const int nch = (H + kFmaHc - 1) / kFmaHc;
  const int hb = (int)((long long)blockIdx.y * nch / gridDim.y) * kFmaHc;
  const int he = min(H, (int)((long long)(blockIdx.y + 1) * nch / gridDim.y) * kFmaHc);
  logits += (size_t)blockIdx.y * T * E;
  const int tid = threadIdx.x;
  float acc[kFmaTok][kFmaEPer];
#pragma unroll
  for (int i = 0; i < kFmaTok; ++i)
#pragma unroll
    for (int j = 0; j < kFmaEPer; ++j) acc[i][j] = 0.f;
  for (int h0 = hb; h0 < he; h0 += kFmaHc) {
    __syncthreads();
    for (int i = tid; i < kFmaTok * kFmaHc; i += kFmaThreads) {
      const int r = i / kFmaHc, c = i - r * kFmaHc;
      const int t = t0 + r;
      xs[r][c] = (t < T && h0 + c < he) ? __bfloat162float(x[(size_t)t * H + h0 + c]) : 0.f;
    }
    __syncthreads();
    const int hn = min(kFmaHc, he - h0);
    for (int hh = 0; hh < hn; ++hh) {
      const float* wrow = w + (size_t)(h0 + hh) * E;
#pragma unroll
      for (int j = 0; j < kFmaEPer; ++j) {
        const int e = tid + j * kFmaThreads;
        const float wv = e < E ? __ldg(wrow + e) : 0.f;
#pragma unroll
        for (int i = 0; i < kFmaTok; ++i) acc[i][j] = fmaf(xs[i][hh], wv, acc[i][j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kFmaTok; ++i) {
    const int t = t0 + i;
    if (t >= T) break;
#pragma unroll
    for (int j = 0; j < kFmaEPer; ++j) {
      const int e = tid + j * kFmaThreads;
      if (e < E) logits[(size_t)t * E + e] = acc[i][j];
    }
  }
}

constexpr int kTopkWarps = 8;

// The EPL logits of one token held by a lane (entry layout of entry_expert).
template <int EPL, bool QUAD>
__device__ __forceinline__ void load_logits(const float* __restrict__ row, int E, int lane, float (&v)[EPL]) {
  if constexpr (QUAD) {
#pragma unroll
    for (int q = 0; q < EPL / 4; ++q) {
      const int e0 = 128 * q + 4 * lane;
      const float4 f = e0 < E ? *reinterpret_cast<const float4*>(row + e0) : make_float4(0.f, 0.f, 0.f, 0.f);
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < E ? row[e] : 0.f;
    }
  }
}

// One warp per token; EPL = experts per lane (E <= 32 * EPL).  The K-split
// partial slabs are summed in slab order; UNR slabs are loaded before any is
// added so that UNR * EPL values per lane are in flight at once.  SEL: a
// scoring rule in which the bias steers only the selection (scoring is
// MOE_SCORE_SOFTMAX_SELECT_BIAS or MOE_SCORE_SIGMOID); otherwise softmax.
template <int EPL, int UNR, bool QUAD, bool SEL>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const float* __restrict__ logits, int nsplit,
                                                             size_t split_stride, const float* __restrict__ bias,
                                                             int T, int E, int k, int scoring,
                                                             int32_t* __restrict__ ids, float* __restrict__ wout,
                                                             DevStatus* st, ZeroSpan zero) {
  zero_span(zero);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  float v[EPL];
  load_logits<EPL, QUAD>(row, E, lane, v);
  int sp = 1;
  for (; sp + UNR <= nsplit; sp += UNR) {
    float p[UNR][EPL];
#pragma unroll
    for (int q = 0; q < UNR; ++q) load_logits<EPL, QUAD>(row + (size_t)(sp + q) * split_stride, E, lane, p[q]);
#pragma unroll
    for (int q = 0; q < UNR; ++q)
#pragma unroll
      for (int i = 0; i < EPL; ++i) v[i] += p[q][i];
  }
  for (; sp < nsplit; ++sp) {
    float p[EPL];
    load_logits<EPL, QUAD>(row + (size_t)sp * split_stride, E, lane, p);
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] += p[i];
  }
  float src[EPL];
  score_entries<EPL, QUAD>(v, src, bias, E, lane, SEL ? scoring : MOE_SCORE_SOFTMAX);
  warp_topk<EPL, QUAD, SEL>(v, src, scoring == MOE_SCORE_SOFTMAX_SELECT_BIAS, E, k, t, ids + (size_t)t * k,
                            wout + (size_t)t * k, nullptr, st);
}

template <int EPL, int UNR, bool QUAD = false>
cudaError_t launch_topk_t(const float* logits, int nsplit, size_t split_stride, const float* bias, int T, int E,
                          int k, int scoring, int32_t* ids, float* w, DevStatus* st, ZeroSpan zero, cudaStream_t s) {
  auto kern = scoring == MOE_SCORE_SOFTMAX ? topk_kernel<EPL, UNR, QUAD, false> : topk_kernel<EPL, UNR, QUAD, true>;
  return launch_kernel(kern, dim3((T + kTopkWarps - 1) / kTopkWarps), dim3(kTopkWarps * 32), 0, s, logits, nsplit,
                       split_stride, bias, T, E, k, scoring, ids, w, st, zero);
}


// ---------------------------------------------------------------- few tokens
// router_partial (route_dev.cuh) per block; the last block to arrive (a
// counter in the workspace status block) sums the slabs in slab order,
// selects the top-k per token and, when asked, builds the expert-contiguous
// permutation of the T*k slots (stable: slot order inside each expert) --
// routing and permutation in one launch.
template <int TT, int EPL>
__global__ void __launch_bounds__(kSmallThreads) router_small_kernel(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias, int T, int H,
    int E, int k, int scoring, int chunk, int hs, float* __restrict__ partial, unsigned int* arrivals,
    int32_t* __restrict__ ids,
    float* __restrict__ wout, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ inv_perm, DevStatus* st, ZeroSpan zero) {
  zero_span(zero);
  __shared__ RouterSmem<TT> rsm;
  __shared__ int32_t sel[kSmallMaxSlots];
  __shared__ int32_t cnt[kMaxExperts];
  __shared__ int32_t warp_sums[kSmallThreads / 32];
  __shared__ int is_last;
  const int tid = threadIdx.x;
  router_partial<TT>(x, w, T, H, E, chunk, blockIdx.x, blockIdx.y, partial, rsm);
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(arrivals, 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // ---- last block: slab sum, scoring, top-k and (in the layer) the permutation
  router_finish<EPL>(partial, hs, bias, T, E, k, scoring, ids, wout, counts, offsets, sorted_ids, inv_perm, st, sel,
                     cnt, warp_sums);
  if (tid == 0) *arrivals = 0u;  // every block has arrived: ready for the next launch
}

template <int TT, int EPL>
cudaError_t launch_router_small_t(const uint16_t* x, const float* w, const float* bias, int T, int H, int E, int k,
                                  int scoring, float* partial, unsigned int* arrivals, int32_t* ids, float* wout,
                                  int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                  DevStatus* st, ZeroSpan zero, cudaStream_t s) {
  const SmallGrid g = small_grid(H, E);
  return launch_kernel(router_small_kernel<TT, EPL>, dim3(g.ncs, g.hs), dim3(kSmallThreads), 0, s,
                       reinterpret_cast<const __nv_bfloat16*>(x), w, bias, T, H, E, k, scoring, g.chunk, g.hs,
                       partial, arrivals, ids, wout, counts, offsets, sorted_ids, inv_perm, st, zero);
}

// accumulators for 1, 4 or 16 tokens
template <int EPL, typename... A>
cudaError_t launch_router_small_e(int T, A... args) {
  if (T == 1) return launch_router_small_t<1, EPL>(args...);
  if (T <= 4) return launch_router_small_t<4, EPL>(args...);
  return launch_router_small_t<kSmallRouterT, EPL>(args...);
}

}  // namespace

cudaError_t launch_router_split(const float* w, int H, int E, uint16_t* planes, cudaStream_t s) {
  const int n = H * E;
  return launch_kernel(router_split_kernel, dim3(min(4096, (n + 255) / 256)), dim3(256), 0, s, w, n, planes);
}

int fma_router_splits(int T, int H) {
  const int tb = (T + kFmaTok - 1) / kFmaTok;
  int sp = 148 / tb;
  const int nch = (H + kFmaHc - 1) / kFmaHc;
  if (sp > nch) sp = nch;
  if (sp > 32) sp = 32;
  return sp < 1 ? 1 : sp;
}

cudaError_t launch_router_logits_fma(const uint16_t* x, const float* w, int T, int H, int E, float* logits,
                                     cudaStream_t s) {
  const dim3 grid((T + kFmaTok - 1) / kFmaTok, fma_router_splits(T, H));
  return launch_kernel(router_logits_fma_kernel, grid, dim3(kFmaThreads), 0, s,
                       reinterpret_cast<const __nv_bfloat16*>(x), w, T, H, E, logits);
}

cudaError_t launch_topk(const float* logits, int nsplit, size_t split_stride, const float* bias, int T, int E, int k,
                        int scoring, int32_t* ids, float* w, DevStatus* st, ZeroSpan zero, cudaStream_t s) {
  if (E <= 32) return launch_topk_t<1, 8>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
  if (E <= 64) return launch_topk_t<2, 8>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
  // E % 4 == 0 (and 16-byte aligned rows): each lane loads 4 experts per 16-byte load
  if (E % 4 == 0) {
    if (E <= 128)
      return launch_topk_t<4, 8, true>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
    if (E <= 256)
      return launch_topk_t<8, 4, true>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
    if (E <= 512)
      return launch_topk_t<16, 4, true>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
    return launch_topk_t<32, 2, true>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
  }
  if (E <= 128) return launch_topk_t<4, 8>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
  if (E <= 256) return launch_topk_t<8, 4>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
  if (E <= 512) return launch_topk_t<16, 4>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
  return launch_topk_t<32, 2>(logits, nsplit, split_stride, bias, T, E, k, scoring, ids, w, st, zero, s);
}

int small_router_slabs(int H, int E) { return small_grid(H, E).hs; }

cudaError_t launch_router_small(const uint16_t* x, const float* w, const float* bias, int T, int H, int E, int k,
                                int scoring, float* partial, unsigned int* arrivals, int32_t* ids, float* wout,
                                int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                DevStatus* st, ZeroSpan zero, cudaStream_t s) {
  if (T < 1 || T > kSmallRouterT || E % 4 != 0 || k > 64) return cudaErrorInvalidValue;
#define MOE_SMALL_ARGS T, x, w, bias, T, H, E, k, scoring, partial, arrivals, ids, wout, counts, offsets, sorted_ids, \
                       inv_perm, st, zero, s
  if (E <= 64) return launch_router_small_e<2>(MOE_SMALL_ARGS);
  if (E <= 128) return launch_router_small_e<4>(MOE_SMALL_ARGS);
  if (E <= 256) return launch_router_small_e<8>(MOE_SMALL_ARGS);
  if (E <= 512) return launch_router_small_e<16>(MOE_SMALL_ARGS);
  return launch_router_small_e<32>(MOE_SMALL_ARGS);
#undef MOE_SMALL_ARGS
}

}  // namespace moe
