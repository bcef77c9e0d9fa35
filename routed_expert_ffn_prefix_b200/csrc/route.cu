// route.cu -- router of the MoE layer: fp32 logits, softmax, top-k, renormalise.
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
// softmax denominator cancels.
#include "kernels.h"

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

__global__ void __launch_bounds__(kFmaThreads) router_logits_fma_kernel(const __nv_bfloat16* __restrict__ x,
                                                                        const float* __restrict__ w, int T,
                                                                        int H, int E,
                                                                        float* __restrict__ logits) {
  __shared__ float xs[kFmaTok][kFmaHc];
  const int t0 = blockIdx.x * kFmaTok;
  const int tid = threadIdx.x;
  float acc[kFmaTok][kFmaEPer];
#pragma unroll
  for (int i = 0; i < kFmaTok; ++i)
#pragma unroll
    for (int j = 0; j < kFmaEPer; ++j) acc[i][j] = 0.f;
  for (int h0 = 0; h0 < H; h0 += kFmaHc) {
    __syncthreads();
    for (int i = tid; i < kFmaTok * kFmaHc; i += kFmaThreads) {
      const int r = i / kFmaHc, c = i - r * kFmaHc;
      const int t = t0 + r;
      xs[r][c] = (t < T && h0 + c < H) ? __bfloat162float(x[(size_t)t * H + h0 + c]) : 0.f;
    }
    __syncthreads();
    const int hn = min(kFmaHc, H - h0);
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

// One warp per token; EPL = experts per lane (E <= 32 * EPL).  The K-split
// partial slabs are summed in slab order; UNR slabs are loaded before any is
// added so that UNR * EPL loads per lane are in flight at once.
template <int EPL, int UNR>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const float* __restrict__ logits, int nsplit,
                                                             size_t split_stride, const float* __restrict__ bias,
                                                             int T, int E, int k, int32_t* __restrict__ ids,
                                                             float* __restrict__ wout, DevStatus* st) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  const float NEG = -INFINITY;
  float v[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? row[e] : 0.f;
  }
  int sp = 1;
  for (; sp + UNR <= nsplit; sp += UNR) {
    float p[UNR][EPL];
#pragma unroll
    for (int q = 0; q < UNR; ++q)
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        p[q][i] = e < E ? row[(size_t)(sp + q) * split_stride + e] : 0.f;
      }
#pragma unroll
    for (int q = 0; q < UNR; ++q)
#pragma unroll
      for (int i = 0; i < EPL; ++i) v[i] += p[q][i];
  }
  for (; sp < nsplit; ++sp) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) v[i] += row[(size_t)sp * split_stride + e];
    }
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? v[i] + (bias ? bias[e] : 0.f) : NEG;
  }
  uint32_t taken = 0;
  float lead = 0.f, sum = 0.f;
  int32_t* idrow = ids + (size_t)t * k;
  float* wrow = wout + (size_t)t * k;
  for (int j = 0; j < k; ++j) {
    // lane-local best among untaken entries: larger value, then lower index
    float bv = NEG;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken >> i & 1u)) {
        if (v[i] > bv || (v[i] == bv && e < bi)) { bv = v[i]; bi = e; }
      }
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, d);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, d);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (bi == 0x7fffffff) {  // no finite candidate: logits were NaN
      if (lane == 0) raise_error(st, MOE_ERR_DEVICE_BOUNDS, SITE_TOPK, t);
      bi = 0;
      bv = lead;
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (j == 0) lead = bv;
    const float z = expf(bv - lead);
    sum += z;
    if (lane == 0) {
      idrow[j] = bi;
      wrow[j] = z;
    }
  }
  __syncwarp();
  const float inv = 1.0f / sum;
  for (int j = lane; j < k; j += 32) wrow[j] = wrow[j] * inv;
}

template <int EPL, int UNR>
cudaError_t launch_topk_t(const float* logits, int nsplit, size_t split_stride, const float* bias, int T, int E,
                          int k, int32_t* ids, float* w, DevStatus* st, cudaStream_t s) {
  topk_kernel<EPL, UNR><<<(T + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, s>>>(logits, nsplit, split_stride,
                                                                                      bias, T, E, k, ids, w, st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_split(const float* w, int H, int E, uint16_t* planes, cudaStream_t s) {
  const int n = H * E;
  router_split_kernel<<<min(4096, (n + 255) / 256), 256, 0, s>>>(w, n, planes);
  return cudaGetLastError();
}

cudaError_t launch_router_logits_fma(const uint16_t* x, const float* w, int T, int H, int E, float* logits,
                                     cudaStream_t s) {
  router_logits_fma_kernel<<<(T + kFmaTok - 1) / kFmaTok, kFmaThreads, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), w, T, H, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int nsplit, size_t split_stride, const float* bias, int T, int E, int k,
                        int32_t* ids, float* w, DevStatus* st, cudaStream_t s) {
  if (E <= 32) return launch_topk_t<1, 8>(logits, nsplit, split_stride, bias, T, E, k, ids, w, st, s);
  if (E <= 64) return launch_topk_t<2, 8>(logits, nsplit, split_stride, bias, T, E, k, ids, w, st, s);
  if (E <= 128) return launch_topk_t<4, 8>(logits, nsplit, split_stride, bias, T, E, k, ids, w, st, s);
  if (E <= 256) return launch_topk_t<8, 4>(logits, nsplit, split_stride, bias, T, E, k, ids, w, st, s);
  if (E <= 512) return launch_topk_t<16, 4>(logits, nsplit, split_stride, bias, T, E, k, ids, w, st, s);
  return launch_topk_t<32, 2>(logits, nsplit, split_stride, bias, T, E, k, ids, w, st, s);
}

}  // namespace moe
