// permute.cu -- routing metadata: per-expert counts, offsets, the permutation
// of slots (t, j) into expert-contiguous order and its inverse.
//
// The pages gather each expert's token rows into a contiguous buffer from
// the routing indices and handle each expert's variable row count with
// minimal padding (Qwen 3.5-397B-on-Ironwood page, sec. 4.2); the gathered
// order must later be undone to bring results back to token order
// (same page, sec. 7.2).  Here the order is fixed: experts ascending, and
// within an expert the slots in ascending flattened index s = t*k + j
// (token ascending), so the permutation is deterministic and can be
// checked bit for bit.  Atomics would make positions run-dependent; instead:
//
//   1. hist:    block b counts the expert ids of its chunk of 1024 slots.
//   2. scan:    one block turns the [blocks, E] counts into each block's
//               starting rank within each expert (a running sum down every
//               column, one thread per expert), then scans the expert totals
//               into offsets.
//   3. scatter: each block splits its chunk into four 256-slot runs, one per
//               warp, ranks the runs against each other per expert, and each
//               warp walks its run in order, 32 slots at a time; lanes with
//               the same expert are ranked by __match_any_sync, so a slot's
//               row = offsets[e] + earlier slots of e in earlier blocks, runs
//               and lanes.
// Up to 8192 slots (decode-sized batches) the three steps run in one block
// of 32 warps instead (one launch): per-warp histograms in shared memory,
// a block scan, and the same in-order warp walk.
#include "kernels.h"

namespace moe {

namespace {

constexpr int kChunk = kPermuteChunk;  // slots per block (hist/scatter)
constexpr int kScatterWarps = 4;
constexpr int kRun = kChunk / kScatterWarps;  // slots walked in order by one warp

__global__ void hist_kernel(const int32_t* __restrict__ ids, int n, int E, int32_t* __restrict__ block_hist,
                            DevStatus* st) {
  extern __shared__ int32_t h[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int s0 = blockIdx.x * kChunk;
  for (int i = threadIdx.x; i < kChunk; i += blockDim.x) {
    const int s = s0 + i;
    if (s < n) {
      const int e = ids[s];
      if (e < 0 || e >= E) {
        raise_error(st, MOE_ERR_DEVICE_BOUNDS, SITE_PERMUTE_IDS, s);
      } else {
        atomicAdd(&h[e], 1);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[(size_t)blockIdx.x * E + e] = h[e];
}

// Single block of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ block_hist, int nblk, int E,
                                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int32_t tot[kMaxExperts];
  __shared__ int32_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // block_hist[b][e] <- rows of expert e in blocks < b.  One thread per
  // expert walks its column; consecutive threads read consecutive experts
  // (coalesced) and each batch of 8 loads is issued before any is used.
  for (int e = tid; e < E; e += blockDim.x) {
    int carry = 0;
    int b0 = 0;
    for (; b0 + 8 <= nblk; b0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = block_hist[(size_t)(b0 + j) * E + e];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        block_hist[(size_t)(b0 + j) * E + e] = carry;
        carry += v[j];
      }
    }
    for (; b0 < nblk; ++b0) {
      const int v = block_hist[(size_t)b0 * E + e];
      block_hist[(size_t)b0 * E + e] = carry;
      carry += v;
    }
    tot[e] = carry;
    counts[e] = carry;
  }
  __syncthreads();
  // exclusive scan of the expert totals (E <= 1024 = blockDim)
  const int v = tid < E ? tot[tid] : 0;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sums[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, ws, d);
      if (lane >= d) ws += o;
    }
    warp_sums[lane] = ws;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - v + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (tid < E) offsets[tid] = excl;
  if (tid == E - 1) offsets[E] = excl + v;
}

__global__ void __launch_bounds__(kScatterWarps * 32) scatter_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                                   int k, const int32_t* __restrict__ block_hist,
                                                                   const int32_t* __restrict__ offsets,
                                                                   int32_t* __restrict__ sorted_ids,
                                                                   int32_t* __restrict__ inv_perm) {
  extern __shared__ int32_t base[];  // [kScatterWarps][E]: next row of expert e for warp w
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int s0 = blockIdx.x * kChunk + w * kRun;
  for (int i = tid; i < kScatterWarps * E; i += blockDim.x) base[i] = 0;
  __syncthreads();
  for (int i = lane; i < kRun; i += 32) {
    const int s = s0 + i;
    if (s < n) {
      const int e = ids[s];
      if (e >= 0 && e < E) atomicAdd(&base[w * E + e], 1);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int run = offsets[e] + block_hist[(size_t)blockIdx.x * E + e];
    for (int j = 0; j < kScatterWarps; ++j) {
      const int c = base[j * E + e];
      base[j * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  int* mine = base + w * E;
  for (int r = 0; r < kRun; r += 32) {
    const int s = s0 + r + lane;
    int e = s < n ? ids[s] : -1;
    if (e >= E) e = -1;  // out-of-range ids were reported by hist_kernel; skip them here
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int pos = e >= 0 ? mine[e] + rank : -1;
    __syncwarp();
    if (e >= 0 && rank == 0) mine[e] += __popc(peers);
    __syncwarp();
    if (e >= 0) {
      sorted_ids[pos] = s / k;
      inv_perm[s] = pos;
    }
  }
}

constexpr int kFusedWarps = 32;
constexpr int kFusedMaxSlots = kFusedWarps * kRun;  // 8192

// Whole permutation in one block (n <= kFusedMaxSlots): warp w owns slots
// [w*kRun, (w+1)*kRun).
__global__ void __launch_bounds__(kFusedWarps * 32) permute_fused_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                                       int k, int32_t* __restrict__ counts,
                                                                       int32_t* __restrict__ offsets,
                                                                       int32_t* __restrict__ sorted_ids,
                                                                       int32_t* __restrict__ inv_perm, DevStatus* st) {
  extern __shared__ int32_t wh[];  // [kFusedWarps][E] counts, then bases
  __shared__ int32_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < kFusedWarps * E; i += blockDim.x) wh[i] = 0;
  __syncthreads();
  const int s0 = w * kRun;
  for (int i = lane; i < kRun; i += 32) {
    const int s = s0 + i;
    if (s < n) {
      const int e = ids[s];
      if (e < 0 || e >= E) raise_error(st, MOE_ERR_DEVICE_BOUNDS, SITE_PERMUTE_IDS, s);
      else atomicAdd(&wh[w * E + e], 1);
    }
  }
  __syncthreads();
  // per expert (thread e): rows of e owned by earlier warps, and the total
  int tot = 0;
  if (tid < E) {
    for (int j = 0; j < kFusedWarps; ++j) {
      const int c = wh[j * E + tid];
      wh[j * E + tid] = tot;
      tot += c;
    }
    counts[tid] = tot;
  }
  // exclusive scan of the totals over experts (E <= 1024 = blockDim)
  int incl = tot;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int ws = warp_sums[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, ws, d);
      if (lane >= d) ws += o;
    }
    warp_sums[lane] = ws;
  }
  __syncthreads();
  const int excl = incl - tot + (w > 0 ? warp_sums[w - 1] : 0);
  if (tid < E) {
    offsets[tid] = excl;
    if (tid == E - 1) offsets[E] = excl + tot;
    for (int j = 0; j < kFusedWarps; ++j) wh[j * E + tid] += excl;
  }
  __syncthreads();
  int* mine = wh + w * E;
  for (int r = 0; r < kRun; r += 32) {
    const int s = s0 + r + lane;
    int e = s < n ? ids[s] : -1;
    if (e >= E) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int pos = e >= 0 ? mine[e] + rank : -1;
    __syncwarp();
    if (e >= 0 && rank == 0) mine[e] += __popc(peers);
    __syncwarp();
    if (e >= 0) {
      sorted_ids[pos] = s / k;
      inv_perm[s] = pos;
    }
  }
}

}  // namespace

int permute_num_blocks(int T, int k) { return (T * k + kChunk - 1) / kChunk; }

cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_ids, int32_t* inv_perm, int32_t* block_hist, DevStatus* st,
                           cudaStream_t s) {
  const int n = T * k;
  if (n <= kFusedMaxSlots) {
    const size_t sh = (size_t)kFusedWarps * E * sizeof(int32_t);
    static std::atomic<int> configured[kMaxDevices];
    cudaError_t err = once_per_device(configured, [&] {
      return cudaFuncSetAttribute(permute_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)((size_t)kFusedWarps * kMaxExperts * sizeof(int32_t)));
    });
    if (err != cudaSuccess) return err;
    return launch_kernel(permute_fused_kernel, dim3(1), dim3(kFusedWarps * 32), sh, s, ids, n, E, k, counts, offsets,
                         sorted_ids, inv_perm, st);
  }
  const int nblk = permute_num_blocks(T, k);
  cudaError_t err = launch_kernel(hist_kernel, dim3(nblk), dim3(256), (size_t)E * sizeof(int32_t), s, ids, n, E,
                                  block_hist, st);
  if (err != cudaSuccess) return err;
  err = launch_kernel(scan_kernel, dim3(1), dim3(1024), 0, s, block_hist, nblk, E, counts, offsets);
  if (err != cudaSuccess) return err;
  return launch_kernel(scatter_kernel, dim3(nblk), dim3(kScatterWarps * 32),
                       (size_t)kScatterWarps * E * sizeof(int32_t), s, ids, n, E, k, block_hist, offsets, sorted_ids,
                       inv_perm);
}

}  // namespace moe
