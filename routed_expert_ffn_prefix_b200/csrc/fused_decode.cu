// fused_decode.cu -- the whole MoE layer for a few tokens (T <= 4) in one launch.
//
// At a few tokens the layer is a handful of matrix-vector products whose
// cost is streaming the activated experts' weights from HBM once; the
// separate kernels of the general path (router, GEMMs, combine) each pay a
// launch, a pipeline fill and a tail, which at this size cost as much as the
// streaming.  Here one cooperative launch (every block resident) runs the
// layer as four phases separated by grid barriers:
//
//   R  split-H router logits (router_partial, the same items as the
//      few-token router) into partial slabs;
//   -- barrier --
//   P  every block sums the slabs, selects the top-k of each token and builds
//      the expert-contiguous permutation and the work plan in its own shared
//      memory (identical in every block: the same data, the same order);
//      block 0 also writes them to the workspace;
//   G  gate/up: work units (expert group, 256 intermediate columns, K slice)
//      stream W_gate_up rows with 16-byte loads (8 columns per lane, 8 rows in
//      flight per warp) and multiply them by the group's <= 4 token rows of x
//      (CUDA cores: at <= 4 rows the work is a weight stream, not a GEMM);
//      each unit writes fp32 partial sums of gate and up for its K slice;
//   -- barrier --
//   D  down: units (group, 256 output columns, K slice of I) first form
//      h = bf16(silu(sum_s gate_s) * sum_s up_s) for their slice (slab
//      order), then stream W_down the same way into fp32 partial slabs;
//   -- barrier --
//   C  combine: y[t] = sum_j w_j * (sum_s o_s[row(t, j)]) in slot order, plus
//      the shared expert's row (weight 1), rounded to bf16 once.
//
// The rounding points and summation orders are fixed (slab order, warp
// order, slot order), so y is bitwise reproducible for a given grid size.
// The shared expert is one more group whose rows are all T tokens.
//
// Grid barriers count arrivals on a word of the workspace status block and
// are bounded (the block that waits too long records MOE_ERR_DEVICE_TIMEOUT
// and stops waiting).  Every block adds its arrivals for barriers it did not
// reach plus one exit arrival before it returns, and the block whose arrival
// completes the count resets the word to zero for the next launch.
#include "gemm_units.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kFT = kFusedMaxT;           // tokens
constexpr int kFThreads = kSmallThreads;  // 256: router_partial's block
constexpr int kFWarps = kFThreads / 32;
constexpr int kFCols = 256;               // weight columns per unit: 8 per lane
constexpr int kFUnroll = 8;               // weight rows per warp in flight
constexpr int kFMaxRows = kFT * kFusedMaxK + kFT;
constexpr int kFMaxGroups = kFT * kFusedMaxK + 1;
constexpr int kFBarriers = 3;

struct FusedArgs {
  const __nv_bfloat16* x;
  const float* w_router;
  const float* bias;
  int scoring;  // MOE_SCORE_*
  const __nv_bfloat16* w_gate_up;
  const __nv_bfloat16* w_down;
  const __nv_bfloat16* w_sh_gate_up;
  const __nv_bfloat16* w_sh_down;
  int T, H, E, I, k, I_s, Imax;
  int rchunk, rhs, rncs;  // router items (small_grid)
  float* rslabs;          // [rhs][T][E]
  float* gslabs;          // [kFusedMaxSplit][rows][2][Imax]: gate, up
  float* dslabs;          // [kFusedMaxSplit][rows][H]
  int32_t* ids;
  float* tw;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_ids;
  int32_t* inv_perm;
  __nv_bfloat16* y;
  DevStatus* st;
  uint64_t timeout_ns;
};

// Per-block plan (shared memory), identical in every block.
struct Plan {
  int32_t sel[kFT * kFusedMaxK];  // expert of slot s = t*k + j
  float w[kFT * kFusedMaxK];      // routing weight of slot s
  int32_t cnt[kMaxExperts];       // rows per expert, then running position
  int32_t row_of_slot[kFT * kFusedMaxK];
  int32_t e_of_row[kFT * kFusedMaxK];
  int32_t tok_of_row[kFMaxRows];
  int32_t g_expert[kFMaxGroups];  // -1: shared expert
  int32_t g_row0[kFMaxGroups];
  int32_t g_rows[kFMaxGroups];
  int32_t warp_sums[kFWarps];
  int32_t ngroups;
  int32_t nrows;
};

__device__ __forceinline__ uint32_t ld_acquire(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Arrive and wait until all blocks have arrived `target` times in total.
// Returns false (and records the timeout) if the wait ran out.
__device__ bool grid_barrier(unsigned int* bar, unsigned int target, const FusedArgs& a, int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(bar, 1u);
    const uint64_t t0 = globaltimer_ns();
    int ok = 1;
    while (ld_acquire(bar) < target) {
      if (globaltimer_ns() - t0 > a.timeout_ns) {
        raise_error(a.st, MOE_ERR_DEVICE_TIMEOUT, SITE_FUSED, (int)target);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

// Eight bf16 weights (one 16-byte load) widened to fp32.
__device__ __forceinline__ void widen8(const uint4& q, float (&w)[8]) {
  const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
    w[2 * i] = f.x;
    w[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 ld_stream16(const __nv_bfloat16* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

// acc[r][0..8) += sum over rows h in [k0, k1) (warp-strided) of
// xin(r, h) * W[h * ldw + col .. +8], for r < nr.  W rows are streamed with
// kFUnroll loads in flight per lane.
template <typename XF>
__device__ __forceinline__ void gemv_rows(const __nv_bfloat16* __restrict__ W, size_t ldw, int col, int k0, int k1,
                                          int nr, XF xin, float (&acc)[kFT][8]) {
  const int warp = threadIdx.x >> 5;
  for (int h = k0 + warp; h < k1; h += kFWarps * kFUnroll) {
    uint4 q[kFUnroll];
#pragma unroll
    for (int u = 0; u < kFUnroll; ++u) {
      const int hh = h + u * kFWarps;
      q[u] = hh < k1 ? ld_stream16(W + (size_t)hh * ldw + col) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kFUnroll; ++u) {
      const int hh = h + u * kFWarps;
      if (hh < k1) {
        float wv[8];
        widen8(q[u], wv);
#pragma unroll
        for (int r = 0; r < kFT; ++r) {
          if (r < nr) {
            const float xv = xin(r, hh);
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(xv, wv[c], acc[r][c]);
          }
        }
      }
    }
  }
}

// Sum acc over the block's warps (warp order) into out(r, c) for r < nr.
template <typename OUT>
__device__ __forceinline__ void reduce_warps(float (&acc)[kFT][8], int nr, float* red, OUT out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* mine = red + (size_t)(warp * 32 + lane) * (kFT * 8);
#pragma unroll
  for (int r = 0; r < kFT; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) mine[r * 8 + c] = acc[r][c];
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * nr * 8; i += kFThreads) {
    const int l = i / (nr * 8), rc = i - l * (nr * 8);
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) s += red[(size_t)(w * 32 + l) * (kFT * 8) + rc];
    out(rc >> 3, l * 8 + (rc & 7), s);
  }
  __syncthreads();
}

template <int EPL>
__global__ void __launch_bounds__(kFThreads) fused_decode_kernel(const FusedArgs a) {
  extern __shared__ __align__(16) uint8_t fsm[];
  Plan& P = *reinterpret_cast<Plan*>(fsm);
  uint8_t* dyn = fsm + ((sizeof(Plan) + 127) & ~size_t(127));
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(dyn);                        // [T][H]
  float* red = reinterpret_cast<float*>(dyn + (size_t)kFT * a.H * 2);                // [256][kFT*8]
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(red + kFThreads * kFT * 8);  // [kFT][Imax]
  __shared__ int bflag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  unsigned int* bar = &a.st->grid_bar;
  int arrived = 0;  // grid barriers this block has arrived at
  const int T = a.T, k = a.k, H = a.H;
  const int n = T * k;

  // ---------------------------------------------------------------- R: router partial slabs
  {
    RouterSmem<kFT>& rsm = *reinterpret_cast<RouterSmem<kFT>*>(red);
    for (int item = blockIdx.x; item < a.rncs * a.rhs; item += G) {
      router_partial<kFT>(a.x, a.w_router, T, H, a.E, a.rchunk, item % a.rncs, item / a.rncs, a.rslabs, rsm);
      __syncthreads();
    }
  }
  // x of every token into shared memory for the gate/up phase
  for (int i = tid; i < T * (H / 8); i += kFThreads)
    reinterpret_cast<uint4*>(xs)[i] = __ldg(reinterpret_cast<const uint4*>(a.x) + i);
  arrived = 1;
  if (!grid_barrier(bar, (unsigned)G * 1, a, &bflag)) goto done;

  // ---------------------------------------------------------------- P: top-k, permutation, plan
  for (int t = warp; t < T; t += kFWarps)
    router_select<EPL>(a.rslabs, a.rhs, a.bias, T, a.E, k, a.scoring, t, P.sel + t * k, P.w + t * k, nullptr,
                       a.st);
  for (int e = tid; e < a.E; e += kFThreads) P.cnt[e] = 0;
  __syncthreads();
  for (int s = tid; s < n; s += kFThreads) atomicAdd(&P.cnt[P.sel[s]], 1);
  __syncthreads();
  {
    // exclusive scan of the expert counts (block-wide, EPT experts per thread)
    constexpr int EPT = kMaxExperts / kFThreads;
    int loc[EPT], tot = 0;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = tid * EPT + j;
      loc[j] = e < a.E ? P.cnt[e] : 0;
      tot += loc[j];
    }
    int incl = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    if (lane == 31) P.warp_sums[warp] = incl;
    __syncthreads();
    int base = incl - tot;
    for (int v = 0; v < warp; ++v) base += P.warp_sums[v];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = tid * EPT + j;
      if (e < a.E) {
        if (blockIdx.x == 0) {
          a.counts[e] = loc[j];
          a.offsets[e] = base;
        }
        P.cnt[e] = base;  // running position of expert e
      }
      base += loc[j];
    }
    if (blockIdx.x == 0 && tid == 0) a.offsets[a.E] = n;
  }
  __syncthreads();
  if (warp == 0) {
    // stable ranks in slot order (rows of the same expert keep token order)
    for (int s0 = 0; s0 < n; s0 += 32) {
      const int s = s0 + lane;
      const int e = s < n ? P.sel[s] : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = e >= 0 ? P.cnt[e] + rank : -1;
      __syncwarp();
      if (e >= 0 && rank == 0) P.cnt[e] += __popc(peers);
      __syncwarp();
      if (e >= 0) {
        P.row_of_slot[s] = pos;
        P.tok_of_row[pos] = s / k;
        P.e_of_row[pos] = e;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    // groups: maximal runs of rows with the same expert, then the shared expert
    int ng = 0;
    for (int r = 0; r < n; ++r) {
      if (r == 0 || P.e_of_row[r] != P.e_of_row[r - 1]) {
        P.g_expert[ng] = P.e_of_row[r];
        P.g_row0[ng] = r;
        P.g_rows[ng] = 0;
        ++ng;
      }
      ++P.g_rows[ng - 1];
    }
    if (a.I_s > 0) {
      P.g_expert[ng] = -1;
      P.g_row0[ng] = n;
      P.g_rows[ng] = T;
      for (int t = 0; t < T; ++t) P.tok_of_row[n + t] = t;
      ++ng;
    }
    P.ngroups = ng;
    P.nrows = n + (a.I_s > 0 ? T : 0);
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int s = tid; s < n; s += kFThreads) {
      a.ids[s] = P.sel[s];
      a.tw[s] = P.w[s];
      a.inv_perm[s] = P.row_of_slot[s];
      a.sorted_ids[P.row_of_slot[s]] = s / k;
    }
  }

  // ---------------------------------------------------------------- G: gate/up partial slabs
  {
    const int ng = P.ngroups;
    int total_cb = 0;
    for (int g = 0; g < ng; ++g) total_cb += (P.g_expert[g] < 0 ? a.I_s : a.I) / kFCols;
    int S = G / (total_cb > 0 ? total_cb : 1);
    S = S < 1 ? 1 : (S > kFusedMaxSplit ? kFusedMaxSplit : S);
    if (S > H / kFCols) S = H / kFCols;
    const int units = total_cb * S;
    const size_t gslab = (size_t)P.nrows * 2 * a.Imax;  // floats per slab
    for (int u = blockIdx.x; u < units; u += G) {
      // decode (group, column block, K slice)
      int rem = u, g = 0, cbg = 0;
      for (; g < ng; ++g) {
        cbg = (P.g_expert[g] < 0 ? a.I_s : a.I) / kFCols;
        if (rem < cbg * S) break;
        rem -= cbg * S;
      }
      const int cb = rem / S, ks = rem - cb * S;
      const int Ig = P.g_expert[g] < 0 ? a.I_s : a.I;
      const __nv_bfloat16* W = P.g_expert[g] < 0 ? a.w_sh_gate_up
                                                  : a.w_gate_up + (size_t)P.g_expert[g] * H * 2 * a.I;
      const int r0 = P.g_row0[g], nr = P.g_rows[g];
      const int k0 = (int)((long long)ks * H / S), k1 = (int)((long long)(ks + 1) * H / S);
      const int col = cb * kFCols + lane * 8;
      auto xin = [&](int r, int h) { return __bfloat162float(xs[(size_t)P.tok_of_row[r0 + r] * H + h]); };
      float* slab = a.gslabs + (size_t)ks * gslab;
      for (int half = 0; half < 2; ++half) {  // 0: gate columns, 1: up columns
        float acc[kFT][8];
#pragma unroll
        for (int r = 0; r < kFT; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
        gemv_rows(W, (size_t)2 * Ig, col + half * Ig, k0, k1, nr, xin, acc);
        reduce_warps(acc, nr, red, [&](int r, int c, float v) {
          slab[((size_t)(r0 + r) * 2 + half) * a.Imax + cb * kFCols + c] = v;
        });
      }
    }
    arrived = 2;
    if (!grid_barrier(bar, (unsigned)G * 2, a, &bflag)) goto done;

    // ---------------------------------------------------------------- D: down partial slabs
    int SD = G / (ng * (H / kFCols) > 0 ? ng * (H / kFCols) : 1);
    SD = SD < 1 ? 1 : (SD > kFusedMaxSplit ? kFusedMaxSplit : SD);
    const int dunits = ng * (H / kFCols) * SD;
    const size_t dslab = (size_t)P.nrows * H;
    for (int u = blockIdx.x; u < dunits; u += G) {
      const int g = u / ((H / kFCols) * SD);
      const int rem = u - g * ((H / kFCols) * SD);
      const int cb = rem / SD, ks = rem - cb * SD;
      const int Ig = P.g_expert[g] < 0 ? a.I_s : a.I;
      const __nv_bfloat16* W = P.g_expert[g] < 0 ? a.w_sh_down : a.w_down + (size_t)P.g_expert[g] * Ig * H;
      const int r0 = P.g_row0[g], nr = P.g_rows[g];
      const int i0 = (int)((long long)ks * Ig / SD), i1 = (int)((long long)(ks + 1) * Ig / SD);
      // h for this slice: sum the gate/up slabs in slab order, SwiGLU, round to bf16
      for (int idx = tid; idx < nr * (i1 - i0); idx += kFThreads) {
        const int r = idx / (i1 - i0), i = i0 + (idx - r * (i1 - i0));
        float gs = 0.f, us = 0.f;
        for (int s = 0; s < S; ++s) {
          const float* sl = a.gslabs + (size_t)s * gslab + (size_t)(r0 + r) * 2 * a.Imax;
          gs += __ldcg(sl + i);
          us += __ldcg(sl + a.Imax + i);
        }
        hs[(size_t)r * a.Imax + i] = __float2bfloat16_rn(silu_f(gs) * us);
      }
      __syncthreads();
      const int col = cb * kFCols + lane * 8;
      auto hin = [&](int r, int i) { return __bfloat162float(hs[(size_t)r * a.Imax + i]); };
      float acc[kFT][8];
#pragma unroll
      for (int r = 0; r < kFT; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
      gemv_rows(W, (size_t)H, col, i0, i1, nr, hin, acc);
      float* slab = a.dslabs + (size_t)ks * dslab;
      reduce_warps(acc, nr, red, [&](int r, int c, float v) {
        slab[(size_t)(r0 + r) * H + cb * kFCols + c] = v;
      });
    }
    arrived = 3;
    if (!grid_barrier(bar, (unsigned)G * 3, a, &bflag)) goto done;

    // ---------------------------------------------------------------- C: combine
    const bool shared = a.I_s > 0;
    for (int item = blockIdx.x * kFThreads + tid; item < T * (H / 8); item += G * kFThreads) {
      const int t = item / (H / 8), c8 = item - t * (H / 8);
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
      for (int j = 0; j < k; ++j) {
        const int row = P.row_of_slot[t * k + j];
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = 0.f;
        for (int s = 0; s < SD; ++s) {
          const float4* p = reinterpret_cast<const float4*>(a.dslabs + (size_t)s * dslab + (size_t)row * H + c8 * 8);
          const float4 lo = __ldcg(p), hi = __ldcg(p + 1);
          v[0] += lo.x; v[1] += lo.y; v[2] += lo.z; v[3] += lo.w;
          v[4] += hi.x; v[5] += hi.y; v[6] += hi.z; v[7] += hi.w;
        }
        const float wj = P.w[t * k + j];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(wj, v[c], acc[c]);
      }
      if (shared) {
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = 0.f;
        for (int s = 0; s < SD; ++s) {
          const float4* p =
              reinterpret_cast<const float4*>(a.dslabs + (size_t)s * dslab + (size_t)(n + t) * H + c8 * 8);
          const float4 lo = __ldcg(p), hi = __ldcg(p + 1);
          v[0] += lo.x; v[1] += lo.y; v[2] += lo.z; v[3] += lo.w;
          v[4] += hi.x; v[5] += hi.y; v[6] += hi.z; v[7] += hi.w;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += v[c];
      }
      uint32_t packed[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        packed[i] = *reinterpret_cast<uint32_t*>(&b2);
      }
      reinterpret_cast<uint4*>(a.y + (size_t)t * H)[c8] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }

done:
  // arrivals for the barriers this block did not reach, plus the exit arrival;
  // the block completing the count returns the word to zero
  __syncthreads();
  if (tid == 0) {
    const unsigned int inc = (unsigned)(kFBarriers - arrived) + 1u;
    const unsigned int total = (unsigned)G * (kFBarriers + 1);
    const unsigned int old = atomicAdd(bar, inc);
    if (old + inc == total) atomicExch(bar, 0u);
  }
}

}  // namespace

bool fused_decode_supported(int T, int H, int E, int I, int k, int I_s) {
  if (T < 1 || T > kFusedMaxT || k > kFusedMaxK || E % 4 != 0 || E > kMaxExperts) return false;
  if (H % kFCols != 0 || I % kFCols != 0 || (I_s > 0 && I_s % kFCols != 0)) return false;
  if (H > 8192 || I > 4096 || I_s > 4096) return false;
  return true;
}

size_t fused_decode_smem(int H, int I, int I_s) {
  const int Imax = I > I_s ? I : I_s;
  return ((sizeof(Plan) + 127) & ~size_t(127)) + (size_t)kFT * H * 2 + (size_t)kFThreads * kFT * 8 * 4 +
         (size_t)kFT * Imax * 2;
}

cudaError_t launch_fused_decode(const uint16_t* x, const float* w_router, const float* bias, int scoring,
                                const uint16_t* w_gate_up, const uint16_t* w_down, const uint16_t* w_sh_gate_up,
                                const uint16_t* w_sh_down, int I_s, int T, int H, int E, int I, int k,
                                float* rslabs, float* gslabs, float* dslabs, int32_t* ids, float* tw,
                                int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                uint16_t* y, DevStatus* st, uint64_t timeout_ns, int num_sms, cudaStream_t s) {
  FusedArgs a{};
  a.x = reinterpret_cast<const __nv_bfloat16*>(x);
  a.w_router = w_router;
  a.bias = bias;
  a.scoring = scoring;
  a.w_gate_up = reinterpret_cast<const __nv_bfloat16*>(w_gate_up);
  a.w_down = reinterpret_cast<const __nv_bfloat16*>(w_down);
  a.w_sh_gate_up = reinterpret_cast<const __nv_bfloat16*>(w_sh_gate_up);
  a.w_sh_down = reinterpret_cast<const __nv_bfloat16*>(w_sh_down);
  a.T = T;
  a.H = H;
  a.E = E;
  a.I = I;
  a.k = k;
  a.I_s = I_s;
  a.Imax = I > I_s ? I : I_s;
  const SmallGrid rg = small_grid(H, E);
  a.rchunk = rg.chunk;
  a.rhs = rg.hs;
  a.rncs = rg.ncs;
  a.rslabs = rslabs;
  a.gslabs = gslabs;
  a.dslabs = dslabs;
  a.ids = ids;
  a.tw = tw;
  a.counts = counts;
  a.offsets = offsets;
  a.sorted_ids = sorted_ids;
  a.inv_perm = inv_perm;
  a.y = reinterpret_cast<__nv_bfloat16*>(y);
  a.st = st;
  a.timeout_ns = timeout_ns;
  const size_t smem = fused_decode_smem(H, I, I_s);
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms * per_sm);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
  };
  if (E <= 64) return run(fused_decode_kernel<2>);
  if (E <= 128) return run(fused_decode_kernel<4>);
  if (E <= 256) return run(fused_decode_kernel<8>);
  if (E <= 512) return run(fused_decode_kernel<16>);
  return run(fused_decode_kernel<32>);
}

}  // namespace moe
