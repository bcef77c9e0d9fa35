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

__device__ __forceinline__ int group_rows_begin(const GemmArgs& a, int g) {
  return a.offsets ? __ldg(a.offsets + g) : 0;
}
__device__ __forceinline__ int group_rows_end(const GemmArgs& a, int g) {
  return a.offsets ? __ldg(a.offsets + g + 1) : a.single_rows;
}

template <int NT>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, const int* ustart, int ngroups, int u) {
  int lo = 0, hi = ngroups - 1;  // last group with ustart[g] <= u (skips empty groups)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ustart[mid] <= u) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int b = group_rows_begin(a, g), e = group_rows_end(a, g);
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

// Warp 0: per-group unit counts -> exclusive prefix in shared memory, with
// the row ranges checked.  Returns the total unit count (0 on bad metadata).
template <int NT>
__device__ void build_unit_prefix(const GemmArgs& a, int ngroups, int* ustart, int* total_out) {
  const int lane = lane_id();
  const int per = (ngroups + 31) / 32;
  const int g0 = min(ngroups, lane * per), g1 = min(ngroups, g0 + per);
  int sum = 0, bad = -1;
  for (int g = g0; g < g1; ++g) {
    const int b = group_rows_begin(a, g), e = group_rows_end(a, g);
    if (b < 0 || e < b || e > a.rows_cap) bad = g;
    ustart[g] = sum;
    sum += (e > b && bad < 0) ? ((e - b + NT - 1) / NT) * a.n_blocks * a.k_splits : 0;
  }
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
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
}

// silu(g) = g * sigmoid(g); h is rounded to bf16 right after, so the fast
// exponential and division are accurate enough.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

}  // namespace moe
