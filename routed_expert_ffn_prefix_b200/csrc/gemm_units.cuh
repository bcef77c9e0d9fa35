// gemm_units.cuh -- work-unit scheduling shared by the grouped GEMM kernels.
//
// A work unit is (group, column block, row pass, K split).  Units are
// numbered group by group (groups = experts, in expert order); inside a group
// the column block varies slowest and the K split fastest.  Every role of a
// persistent block walks the same unit sequence u = first, first + stride, ...
// and decodes it independently from a per-group prefix of unit counts kept in
// shared memory.
#pragma once

#include "kernels.h"

namespace moe {

constexpr int kBK = 64;  // k per pipeline stage (one 128-byte swizzle row of bf16)


struct Unit {
  int group, nb, row0, rows, ks, kb, ke;  // ks: K split; [kb, ke): its k-steps (of kBK)
  int passes;                             // row passes of this group (units re-streaming the same weights)
};

// Routing metadata (offsets, row indices, slot rows and weights) is read
// with generic loads, never the read-only path: the persistent few-token
// layer computes it in the same launch and keeps it in each block's shared
// memory.

// The unit prefix of a GEMM in shared memory: ustart[g] (g < ngroups) is the
// first unit of group g; ustart[kPrefixRows + g] (g <= ngroups) the first
// permuted row of group g, so decoding a unit reads no global memory.
constexpr int kPrefixRows = kMaxExperts + 1;
constexpr int kPrefixInts = 2 * kPrefixRows;

template <int NT>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, const int* ustart, int ngroups, int u) {
  int lo = 0, hi = ngroups - 1;  // last group with ustart[g] <= u (skips empty groups)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ustart[mid] <= u) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int b = ustart[kPrefixRows + g], e = ustart[kPrefixRows + g + 1];
  const int passes = (e - b + NT - 1) / NT;
  const int S = a.k_splits;
  const int local = u - ustart[g];
  Unit r;
  r.group = g;
  r.nb = local / (passes * S);
  const int rem = local - r.nb * passes * S;
  const int pass = rem / S;
  r.ks = rem - pass * S;
  r.row0 = b + pass * NT;
  r.rows = min(NT, e - r.row0);
  r.passes = passes;
  const int nkt = a.K / kBK;
  r.kb = r.ks * nkt / S;
  r.ke = (r.ks + 1) * nkt / S;
  return r;
}

// One warp: per-group unit counts -> exclusive prefix and the groups' row
// ranges in shared memory (kPrefixInts ints at ustart), with the ranges
// checked.  The group boundaries come from `soffsets` (shared memory, when
// the caller already holds them) or else from a.offsets in global memory,
// all loaded at once (one round trip, not one per group).  Returns the total
// unit count in *total_out (0 on bad metadata).
template <int NT>
__device__ void build_unit_prefix(const GemmArgs& a, int ngroups, int* ustart, int* total_out,
                                  const int* soffsets = nullptr) {
  const int lane = lane_id();
  int* rbeg = ustart + kPrefixRows;
  constexpr int kPer = (kPrefixRows + 31) / 32;
  int v[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = lane + 32 * j;
    v[j] = 0;
    if (i <= ngroups) {
      if (soffsets != nullptr) v[j] = soffsets[i];
      else if (a.offsets != nullptr) v[j] = __ldcg(a.offsets + i);
      else v[j] = i == 0 ? 0 : a.single_rows;
    }
  }
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = lane + 32 * j;
    if (i <= ngroups) rbeg[i] = v[j];
  }
  __syncwarp();
  const int per = (ngroups + 31) / 32;
  const int g0 = min(ngroups, lane * per), g1 = min(ngroups, g0 + per);
  int sum = 0, bad = -1;
  for (int g = g0; g < g1; ++g) {
    const int b = rbeg[g], e = rbeg[g + 1];
    if (b < 0 || e < b || e > a.rows_cap) bad = g;
    ustart[g] = sum;
    sum += (e > b && bad < 0) ? ((e - b + NT - 1) / NT) * a.n_blocks * a.k_splits : 0;
  }
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int w = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += w;
  }
  const int base = incl - sum;
  for (int g = g0; g < g1; ++g) ustart[g] += base;
  const int any_bad = __reduce_max_sync(0xffffffffu, bad);
  if (lane == 31) {
    if (any_bad >= 0) {
      raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_GEMM_OFFSETS, any_bad);
      *total_out = 0;
    } else {
      *total_out = incl;
    }
  }
  __syncwarp();
}

// silu(g) = g * sigmoid(g); h is rounded to bf16 right after, so the fast
// exponential and division are accurate enough.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// ---------------------------------------------------------------- last-arriver reduction
// The K-split gate/up slabs of a row, or the k expert-output rows of a token,
// are produced by different work units on different SMs, in no fixed order.
// Instead of a separate pass over them, every epilogue warp counts its
// stores on a per-(key, column chunk) counter; the warp whose arrival
// completes a counter reduces that chunk.  The reduction itself always runs
// in the same order (K slabs ascending, then slots j = 0..k-1), so the
// result does not depend on which warp finishes: it is bitwise the same as
// a separate pass in that order.  No warp ever waits for another.
constexpr int kMaxKSplit = 8;

__device__ __forceinline__ uint32_t atom_add_relaxed_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// h[r, c] = bf16(silu(sum_s gate_s) * sum_s up_s) for this lane's column:
// cols[0] = gate column, cols[1] = up column of the fp32 slab rows (lane = column).
__device__ __forceinline__ void finish_swiglu_row(const GemmArgs& a, int r, const int (&cols)[2]) {
  if (cols[1] >= a.n_valid) return;  // never taken: the K-split gate/up units cover exactly 2I columns
  const float* p = reinterpret_cast<const float*>(a.out) + (size_t)r * a.ld_out;
  const int S = a.k_splits;
  float g[kMaxKSplit], u[kMaxKSplit];
#pragma unroll
  for (int s = 0; s < kMaxKSplit; ++s) {
    if (s < S) {
      g[s] = __ldcg(p + (size_t)s * a.split_stride + cols[0]);
      u[s] = __ldcg(p + (size_t)s * a.split_stride + cols[1]);
    }
  }
  float gs = g[0], us = u[0];
#pragma unroll
  for (int s = 1; s < kMaxKSplit; ++s) {
    if (s < S) {
      gs += g[s];
      us += u[s];
    }
  }
  if (cols[0] < a.fin_ld)
    reinterpret_cast<__nv_bfloat16*>(a.fin_out)[(size_t)r * a.fin_ld + cols[0]] = __float2bfloat16_rn(silu_f(gs) * us);
}

// y[t, c] = bf16(sum_{j<k} w[t,j] * (sum_s o_s[inv_perm[t,j], c]) + shared[t, c]) for this
// lane's columns (one per MMA tile of the unit), slots in order, fp32.
template <int MT>
__device__ __forceinline__ void finish_combine_row(const GemmArgs& a, int t, const int (&cols)[MT]) {
  const int lane = lane_id(), k = a.topk, S = a.k_splits;
  const float* o = reinterpret_cast<const float*>(a.out);
  int ra = 0, rb = 0;
  float wa = 0.f, wb = 0.f;
  if (lane < k) {
    ra = a.inv_perm[(size_t)t * k + lane];
    wa = a.topk_w[(size_t)t * k + lane];
  }
  if (lane + 32 < k) {
    rb = a.inv_perm[(size_t)t * k + lane + 32];
    wb = a.topk_w[(size_t)t * k + lane + 32];
  }
  const bool bad = (lane < k && (ra < 0 || ra >= a.rows_cap)) || (lane + 32 < k && (rb < 0 || rb >= a.rows_cap));
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_COMBINE, t);
    return;
  }
  // output columns past n_valid (the pair kernel's last block when H % 512 != 0) are never read
  bool live[MT];
#pragma unroll
  for (int i = 0; i < MT; ++i) live[i] = cols[i] < a.n_valid;
  float acc[MT];
#pragma unroll
  for (int i = 0; i < MT; ++i) acc[i] = 0.f;
  for (int j0 = 0; j0 < k; j0 += 8) {
    float v[8][MT];
    int rr[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int j = j0 + q;
      rr[q] = __shfl_sync(0xffffffffu, j < 32 ? ra : rb, j & 31);
      if (j < k) {
#pragma unroll
        for (int i = 0; i < MT; ++i) v[q][i] = live[i] ? __ldcg(o + (size_t)rr[q] * a.ld_out + cols[i]) : 0.f;
      }
    }
    for (int s = 1; s < S; ++s) {
      const float* os = o + (size_t)s * a.split_stride;
      float p[8][MT];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (j0 + q < k) {
#pragma unroll
          for (int i = 0; i < MT; ++i) p[q][i] = live[i] ? __ldcg(os + (size_t)rr[q] * a.ld_out + cols[i]) : 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (j0 + q < k) {
#pragma unroll
          for (int i = 0; i < MT; ++i) v[q][i] += p[q][i];
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int j = j0 + q;
      const float wj = __shfl_sync(0xffffffffu, j < 32 ? wa : wb, j & 31);
      if (j < k) {
#pragma unroll
        for (int i = 0; i < MT; ++i) acc[i] = fmaf(wj, v[q][i], acc[i]);
      }
    }
  }
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.fin_out) + (size_t)t * a.fin_ld;
#pragma unroll
  for (int i = 0; i < MT; ++i) {
    if (live[i]) {
      float v = acc[i];
      if (a.shared) v += __ldcg(a.shared + (size_t)t * a.ld_out + cols[i]);
      y[cols[i]] = __float2bfloat16_rn(v);
    }
  }
}

// One epilogue warp, after storing rows [r0, r0 + nr) of output chunk
// `chunk`, and after a __syncwarp() and a __threadfence() by every lane
// since those stores (the release: the stores are visible device-wide before
// any counter moves): count the arrivals with relaxed atomics and reduce
// every key this warp completed, after another fence (the acquire: every
// other warp's stores counted on that key are visible to the loads).
// Warp-uniform arguments.
template <int MT, int EPI>
__device__ __forceinline__ void arrive_rows(const GemmArgs& a, int r0, int nr, int chunk, const int (&cols)[MT]) {
  const int lane = lane_id();
  int key = -1;
  bool fin = false;
  if (lane < nr) {
    const int r = r0 + lane;
    key = r;
    if constexpr (EPI == EPI_DOWN_COMBINE) {
      key = a.row_token[r];
      if (key < 0 || key >= a.n_tokens) {
        raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_GEMM_EPILOGUE, r);
        key = -1;
      }
    }
    if (key >= 0) {
      uint32_t* c = a.arrivals + (size_t)key * a.cnt_stride + chunk;
      const uint32_t done = atom_add_relaxed_gpu(c, 1u) + 1u;
      if (done == (uint32_t)a.arrive_target) {
        fin = true;
        *c = 0u;  // every arrival has been counted: zero again for the next kernel
      } else if (done > (uint32_t)a.arrive_target) {
        raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_GEMM_EPILOGUE, r);
      }
    }
  }
  uint32_t m = __ballot_sync(0xffffffffu, fin);
  if (m == 0u) return;
  __syncwarp();
  __threadfence();  // acquire side, before any lane reads other warps' rows
  while (m) {
    const int i = __ffs(m) - 1;
    m &= m - 1u;
    const int kk = __shfl_sync(0xffffffffu, key, i);
    if constexpr (EPI == EPI_DOWN_COMBINE) {
      finish_combine_row<MT>(a, kk, cols);
    } else {
      static_assert(EPI != EPI_SWIGLU_SPLIT || MT == 2, "the split SwiGLU needs the gate and the up tile");
      finish_swiglu_row(a, kk, cols);
    }
  }
}

}  // namespace moe
