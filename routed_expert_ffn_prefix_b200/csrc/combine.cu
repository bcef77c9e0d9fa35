// combine.cu -- weighted gather-combine of the expert outputs back to token order.
//
// The Qwen 3.5-397B-on-Ironwood page (sec. 7.2) un-permutes the [T*k, H]
// expert outputs and gather-reduces them per token; the Ling-2.6-1T /
// SGLang-JAX page fuses scatter, expert FFN and gather ("Fused MoE V2").
// Here each token's k expert rows (fp32; K-split partial slabs are first
// summed in slab order) are read through inv_perm and summed in
// slot order j = 0..k-1 in fp32 (w_j * o_j, one fused multiply-add per
// term), the shared-expert row (weight 1) is added last, and y is rounded
// to bf16 once.  A fixed summation order makes y bitwise reproducible
// run to run, whatever order the expert GEMM tiles finished in.
//
// Memory-bound: a block per (token, column slice), one 16-byte vector of a
// row (4 columns) per thread and slot, the slot loads of a thread issued
// eight rows (and, for K-split slabs, up to two slabs) at a time.
#include "gemm_units.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;

// V consecutive columns of an expert output row in one 16-byte load.
template <typename OT>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int V = 4;
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 q = __ldcs(reinterpret_cast<const float4*>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  // load when `live`, zeros otherwise (rows past the token's k slots)
  static __device__ __forceinline__ void load_if(bool live, const float* p, float (&v)[4]) {
    if (live) {
      load(p, v);
    } else {
      v[0] = v[1] = v[2] = v[3] = 0.f;
    }
  }
};
// SPLIT: the down GEMM's K was split (nsplit > 1 slabs).  The plain path is
// compiled for four resident blocks per SM (its loads in flight are what
// paces it); the slab path keeps its registers.
template <typename OT, bool SPLIT>
__global__ void __launch_bounds__(kThreads, SPLIT ? 1 : 4)
    combine_kernel(const OT* __restrict__ o, const float* __restrict__ w,
                                                         const int32_t* __restrict__ inv_perm,
                                                         const float* __restrict__ shared, int H, int k, int rows,
                                                         int nsplit, size_t split_stride,
                                                         __nv_bfloat16* __restrict__ y, DevStatus* st, int t0) {
  constexpr int V = Vec<OT>::V;
  const int t = t0 + blockIdx.y;
  __shared__ int32_t srow[64];
  __shared__ float sw[64];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int r = inv_perm[(size_t)t * k + j];
    if (r < 0 || r >= rows) {
      raise_error(st, MOE_ERR_DEVICE_BOUNDS, SITE_COMBINE, t);
      bad = 1;
    }
    srow[j] = r;
    sw[j] = w[(size_t)t * k + j];
  }
  __syncthreads();
  if (bad) return;
  const int HV = H / V;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < HV; c += gridDim.x * blockDim.x) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    if (!SPLIT) {
      // k independent row loads in flight together, then the slot-order sum
      int j = 0;
      for (; j + 8 <= k; j += 8) {
        float v[8][V];
#pragma unroll
        for (int q = 0; q < 8; ++q) Vec<OT>::load(o + (size_t)srow[j + q] * H + V * c, v[q]);
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int i = 0; i < V; ++i) acc[i] = fmaf(sw[j + q], v[q][i], acc[i]);
      }
      for (; j < k; ++j) {
        float v[V];
        Vec<OT>::load(o + (size_t)srow[j] * H + V * c, v);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(sw[j], v[i], acc[i]);
      }
    } else {
      // K-split partial slabs of the down GEMM: for 8 rows at a time, slab 0
      // and then the other slabs two at a time are loaded together; each
      // row's slabs are summed in slab order, then the slot-order sum
      int j = 0;
      for (; j < k; j += 8) {
        const int nq = k - j < 8 ? k - j : 8;
        float v[8][V];
#pragma unroll
        for (int q = 0; q < 8; ++q) Vec<OT>::load_if(q < nq, o + (size_t)srow[j + q % nq] * H + V * c, v[q]);
        int sp = 1;
        for (; sp + 2 <= nsplit; sp += 2) {
          float p[2][8][V];
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int q = 0; q < 8; ++q)
              Vec<OT>::load_if(q < nq, o + (sp + u) * split_stride + (size_t)srow[j + q % nq] * H + V * c, p[u][q]);
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
              for (int i = 0; i < V; ++i) v[q][i] += p[u][q][i];
        }
        if (sp < nsplit) {
          float p[8][V];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            Vec<OT>::load_if(q < nq, o + sp * split_stride + (size_t)srow[j + q % nq] * H + V * c, p[q]);
#pragma unroll
          for (int q = 0; q < 8; ++q)
#pragma unroll
            for (int i = 0; i < V; ++i) v[q][i] += p[q][i];
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < nq)
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = fmaf(sw[j + q], v[q][i], acc[i]);
      }
    }
    if (shared) {
#pragma unroll
      for (int q = 0; q < V; q += 4) {
        const float4 sv = __ldcs(reinterpret_cast<const float4*>(shared + (size_t)t * H + V * c + q));
        acc[q] += sv.x;
        acc[q + 1] += sv.y;
        acc[q + 2] += sv.z;
        acc[q + 3] += sv.w;
      }
    }
    uint32_t packed[V / 2];
#pragma unroll
    for (int i = 0; i < V / 2; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      packed[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    if constexpr (V == 8) {
      reinterpret_cast<uint4*>(y + (size_t)t * H)[c] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    } else {
      reinterpret_cast<uint2*>(y + (size_t)t * H)[c] = make_uint2(packed[0], packed[1]);
    }
  }
}

// h[r, i] = bf16(silu(g) * u) with g, u the sums (in slab order) of the K-split
// partial gate/up slabs P[s][r][0..2I) written by the grouped GEMM's store
// epilogue (gate in columns [0, I), up in [I, 2I)).
__global__ void __launch_bounds__(kThreads) swiglu_reduce_kernel(const float* __restrict__ p, int nsplit,
                                                               size_t split_stride, int rows, int I,
                                                               __nv_bfloat16* __restrict__ h) {
  const int I4 = I >> 2;
  const long long n = (long long)rows * I4;
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(q / I4), c = (int)(q - (long long)r * I4);
    const float* row = p + (size_t)r * 2 * I;
    float4 g = reinterpret_cast<const float4*>(row)[c];
    float4 u = reinterpret_cast<const float4*>(row + I)[c];
    int sp = 1;
    for (; sp + 2 <= nsplit; sp += 2) {  // two slabs' loads in flight together, added in slab order
      const float4 g2 = reinterpret_cast<const float4*>(row + sp * split_stride)[c];
      const float4 u2 = reinterpret_cast<const float4*>(row + sp * split_stride + I)[c];
      const float4 g3 = reinterpret_cast<const float4*>(row + (sp + 1) * split_stride)[c];
      const float4 u3 = reinterpret_cast<const float4*>(row + (sp + 1) * split_stride + I)[c];
      g.x += g2.x; g.y += g2.y; g.z += g2.z; g.w += g2.w;
      u.x += u2.x; u.y += u2.y; u.z += u2.z; u.w += u2.w;
      g.x += g3.x; g.y += g3.y; g.z += g3.z; g.w += g3.w;
      u.x += u3.x; u.y += u3.y; u.z += u3.z; u.w += u3.w;
    }
    if (sp < nsplit) {
      const float4 g2 = reinterpret_cast<const float4*>(row + sp * split_stride)[c];
      const float4 u2 = reinterpret_cast<const float4*>(row + sp * split_stride + I)[c];
      g.x += g2.x; g.y += g2.y; g.z += g2.z; g.w += g2.w;
      u.x += u2.x; u.y += u2.y; u.z += u2.z; u.w += u2.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(silu_f(g.x) * u.x, silu_f(g.y) * u.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(silu_f(g.z) * u.z, silu_f(g.w) * u.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(h + (size_t)r * I)[c] = packed;
  }
}

// row_token[inv_perm[s]] = s / k for every slot s (the token of each permuted
// row, for a down GEMM that combines in its epilogue), and the zeroing of the
// arrival counters that epilogue uses.
__global__ void row_tokens_kernel(const int32_t* __restrict__ inv_perm, int n, int k, int32_t* __restrict__ row_token,
                                  ZeroSpan zero, DevStatus* st) {
  zero_span(zero);
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n; s += gridDim.x * blockDim.x) {
    const int r = inv_perm[s];
    if (r < 0 || r >= n) {
      raise_error(st, MOE_ERR_DEVICE_BOUNDS, SITE_COMBINE, s);
    } else {
      row_token[r] = s / k;
    }
  }
}

}  // namespace

cudaError_t launch_row_tokens(const int32_t* inv_perm, int T, int k, int32_t* row_token, ZeroSpan zero, DevStatus* st,
                              cudaStream_t s) {
  const long long n = (long long)T * k;
  const long long work = n > zero.n16 ? n : zero.n16;
  const int blocks = (int)((work + kThreads - 1) / kThreads < 1184 ? (work + kThreads - 1) / kThreads : 1184);
  return launch_kernel(row_tokens_kernel, dim3(blocks), dim3(kThreads), 0, s, inv_perm, (int)n, k, row_token, zero, st);
}

cudaError_t launch_swiglu_reduce(const float* partials, int nsplit, size_t split_stride, int rows, int I, uint16_t* h,
                                 cudaStream_t s) {
  const long long n = (long long)rows * (I / 4);
  int threads = kThreads;  // few rows: smaller blocks so more SMs share the loads
  while (threads > 64 && (n + threads - 1) / threads < 148) threads >>= 1;
  const int blocks = (int)((n + threads - 1) / threads < 4096 ? (n + threads - 1) / threads : 4096);
  return launch_kernel(swiglu_reduce_kernel, dim3(blocks), dim3(threads), 0, s, partials, nsplit, split_stride,
                       rows, I, reinterpret_cast<__nv_bfloat16*>(h));
}

namespace {

template <typename OT>
cudaError_t launch_combine_t(const OT* o, const float* topk_w, const int32_t* inv_perm, const float* shared, int T,
                             int H, int k, int rows, int nsplit, size_t split_stride, uint16_t* y, DevStatus* st,
                             cudaStream_t s) {
  if (k > 64) return cudaErrorInvalidValue;
  // Few tokens: split each row over several blocks so every SM has work
  // (down to 64 threads per block); many tokens: one block per token, each
  // thread looping over its vectors.
  const int HV = H / Vec<OT>::V;
  int threads = kThreads;
  while (threads > 64 && (long long)T * ((HV + threads - 1) / threads) < 148) threads >>= 1;
  const int slices_max = (HV + threads - 1) / threads;
  int slices = (2 * 148 + T - 1) / T;
  slices = slices < 1 ? 1 : (slices > slices_max ? slices_max : slices);
  for (int t0 = 0; t0 < T; t0 += 65535) {  // grid.y limit
    const dim3 grid(slices, T - t0 < 65535 ? T - t0 : 65535);
    const cudaError_t err =
        nsplit > 1 ? launch_kernel(combine_kernel<OT, true>, grid, dim3(threads), 0, s, o, topk_w, inv_perm, shared,
                                   H, k, rows, nsplit, split_stride, reinterpret_cast<__nv_bfloat16*>(y), st, t0)
                   : launch_kernel(combine_kernel<OT, false>, grid, dim3(threads), 0, s, o, topk_w, inv_perm, shared,
                                   H, k, rows, nsplit, split_stride, reinterpret_cast<__nv_bfloat16*>(y), st, t0);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_combine(const float* o, const float* topk_w, const int32_t* inv_perm, const float* shared, int T,
                           int H, int k, int rows, int nsplit, size_t split_stride, uint16_t* y, DevStatus* st,
                           cudaStream_t s) {
  return launch_combine_t(o, topk_w, inv_perm, shared, T, H, k, rows, nsplit, split_stride, y, st, s);
}

}  // namespace moe
