// kernels.h -- host-side launchers of the MoE kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "common.cuh"

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxK = 64;          // largest top-k any entry point accepts
constexpr int kPermuteChunk = 1024; // slots per block of the multi-block permutation (histogram rows)
constexpr int kMxRawSteps = 2;      // k-steps of 64 per TMA box of FP8 codes (box rows of 64 * this bytes)
constexpr int kMaxDevices = 64;

// Runs `setup` once per (call site, device): kernel attributes and occupancy
// queries are per device and never change, so they stay off the per-call path.
template <typename F>
inline cudaError_t once_per_device(std::atomic<int>* done, F&& setup) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return setup();
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  err = setup();
  if (err == cudaSuccess) done[dev].store(1, std::memory_order_release);
  return err;
}

// Launches `kern` on stream s (checked arguments, one call form for all kernels).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Arguments of the grouped GEMM (see grouped_gemm.cu).  "Rows" are token
// rows (the MMA's N side); "columns" are weight columns (the MMA's M side).
struct GemmArgs {
  const int32_t* offsets;  // [groups+1] row ranges per group, or nullptr: one group of single_rows rows
  const int32_t* row_index;  // permuted row -> source row of b_src (gather), or nullptr: identity
  const uint16_t* b_src;     // [src_rows, K] bf16, K contiguous
  int src_rows;
  int groups;
  int single_rows;
  int K;            // reduction length, multiple of 64
  int krep;         // repeats of the K loop (weight planes summed into one accumulator)
  int a_dim2_rep;   // 1: weight tile's 3rd coordinate is the repeat index; 0: the group index
  int n_blocks;     // column blocks per group (each = two 128-column MMA tiles)
  int col_stride;   // first weight column of block nb = nb * col_stride
  int col1_off;     // second MMA tile's columns start col1_off after the first
  void* out;
  int ld_out;          // output row stride (elements)
  int out_col_stride;  // output column of block nb = nb * out_col_stride (+ lane)
  int out_col1_off;    // store epilogue: second tile's output columns offset
  int n_valid;         // output columns < n_valid are written
  int rows_cap;        // offsets[groups] may not exceed this (rows of out / row_index)
  int rows_evict_last; // token-row gathers keep their lines in L2 (evict-last hint) instead of normal
  int k_splits;        // K range split across this many work units (store epilogue only)
  size_t split_stride; // elements between the partial-result slabs of consecutive K splits
  DevStatus* status;
  uint64_t timeout_ns;
  // Last-arriver reduction (EPI_SWIGLU_SPLIT, EPI_DOWN_COMBINE).  After a
  // warp has stored its fp32 rows of a 32-column chunk it adds one to the
  // counter of every (key, chunk) it covered; the warp that brings a counter
  // to arrive_target reduces that key's chunk in a fixed order, writes the
  // result and sets the counter back to zero.  Counters must be zero when
  // the kernel starts.
  uint32_t* arrivals;       // [keys][cnt_stride] counters
  int cnt_stride;           // counters per key (column chunks of the output row)
  int arrive_target;        // arrivals per (key, chunk): k_splits (gate/up) or topk * k_splits (down)
  // EPI_SWIGLU_SPLIT: h [rows][fin_ld] bf16 = silu(sum of the gate slabs) * (sum of the up slabs).
  // EPI_DOWN_COMBINE: y [n_tokens][fin_ld] bf16 = sum_j topk_w[t,j] * (slab-summed o[inv_perm[t,j]]) + shared[t].
  uint16_t* fin_out;
  int fin_ld;
  const int32_t* row_token;  // permuted row -> token (down-combine key)
  const int32_t* inv_perm;   // [n_tokens][topk] slot -> permuted row
  const float* topk_w;       // [n_tokens][topk]
  const float* shared;       // [n_tokens][ld_out] f32 shared-expert rows, or nullptr
  int topk;
  int n_tokens;
};

// SWIGLU: h = bf16(silu(gate) * up); STORE_F32: fp32 rows (K splits to their
// own slabs); SWIGLU_SPLIT: fp32 gate/up slabs of a K split, the last slab
// of each row chunk to land sums them and writes h; DOWN_COMBINE: fp32
// expert-output rows (per K slab), the last of a token's k * k_splits row
// chunks to land writes that chunk of y (weighted slot-order sum + shared).
enum Epilogue { EPI_SWIGLU = 0, EPI_STORE_F32 = 1, EPI_SWIGLU_SPLIT = 2, EPI_DOWN_COMBINE = 3 };

// MMA tiles (128 weight columns each) per work unit of the given tile
// policy and epilogue; the caller sets n_blocks/col_stride/out_col_stride
// for units of 128 * that many columns.
int gemm_tiles_per_unit(int tiles, int epilogue);

// The grouped GEMM on block-scaled FP8 weights (grouped_gemm_mx.cu): code_map
// covers the E4M3 codes of W^T [E, N, K] u8 (boxes of kMxRawSteps * 64 codes
// x 128 columns, swizzled over the box row: 64-byte swizzle for one k-step,
// 128-byte for two), scale_map the E8M0 scales [E, K/32, N] u8 (boxes of 128
// columns x 2 * kMxRawSteps rows).  Units of 128-column tiles as in the
// single-SM kernel (two tiles per unit, col_stride and col1_off multiples of
// 128, krep 1); epilogue EPI_SWIGLU, EPI_SWIGLU_SPLIT or EPI_STORE_F32;
// tiles MOE_TILES_SMALL (32-row passes, decoded weights in TMEM) or anything
// else (256-row passes).
cudaError_t launch_grouped_gemm_mx(const CUtensorMap& code_map, const CUtensorMap& scale_map, const GemmArgs& a,
                                   int epilogue, int tiles, int num_sms, cudaStream_t stream);

// Large-row groups on SM pairs (grouped_gemm_pair.cu): 256 token rows per
// unit, two 128-column weight tiles per unit (the same n_blocks/col_stride/
// col1_off/out_col_stride as the single-SM kernel with two tiles per unit);
// output columns must come in whole chunks of 32 (n_valid % 32 == 0).
// rows_map != nullptr: the rows are contiguous (a.row_index == nullptr) and
// rows_map covers them (bf16 [1][src_rows][K], boxes of 64 x 128 x 1,
// 128-byte swizzle); each SM then loads its half of a unit's rows with one
// TMA box per stage, and writes its fp32 output rows through out_map (fp32
// [1][rows][ld_out], boxes of 32 x 16 x 1, no swizzle) by bulk tensor
// stores (EPI_STORE_F32, no K split).  rows_map == nullptr, out_map !=
// nullptr: EPI_SWIGLU writes h through out_map (bf16 [1][rows][ld_out],
// boxes of 32 x 16 x 1) the same way.
cudaError_t launch_grouped_gemm_pair(const CUtensorMap& wmap, const CUtensorMap* rows_map, const CUtensorMap* out_map,
                                     const GemmArgs& a, int epilogue, int num_sms, cudaStream_t stream);

// tiles: MOE_TILES_SMALL or MOE_TILES_LARGE.
cudaError_t launch_grouped_gemm(const CUtensorMap& wmap, const GemmArgs& a, int epilogue, int tiles,
                                int num_sms, cudaStream_t stream);

// A span of device memory a kernel zeroes (grid-stride, 16-byte stores)
// before its own work: the routing kernels clear the arrival counters of the
// expert GEMMs' last-arriver epilogues this way, in every layer call.
struct ZeroSpan {
  uint4* p;
  int n16;  // 16-byte words
};
__device__ __forceinline__ void zero_span(const ZeroSpan& z) {
  const int nthreads = gridDim.x * gridDim.y * blockDim.x;
  const int tid = (blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
  for (int i = tid; i < z.n16; i += nthreads) z.p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Router.
cudaError_t launch_router_split(const float* w, int H, int E, uint16_t* planes, cudaStream_t s);
// fp32 CUDA-core logits into fma_router_splits(T, H) partial slabs [T, E].
int fma_router_splits(int T, int H);
cudaError_t launch_router_logits_fma(const uint16_t* x, const float* w, int T, int H, int E, float* logits,
                                     cudaStream_t s);
// logits: nsplit partial slabs of [T, E], split_stride elements apart, summed in slab order;
// scoring: MOE_SCORE_*.
cudaError_t launch_topk(const float* logits, int nsplit, size_t split_stride, const float* bias, int T, int E, int k,
                        int scoring, int32_t* ids, float* w, DevStatus* st, ZeroSpan zero, cudaStream_t s);

// Permutation.
int permute_num_blocks(int T, int k);
cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_ids, int32_t* inv_perm, int32_t* block_hist, DevStatus* st,
                           cudaStream_t s);

// Combine.
// o: nsplit partial slabs [rows, H] (split_stride elements apart) summed in slab order.
cudaError_t launch_combine(const float* o, const float* topk_w, const int32_t* inv_perm, const float* shared,
                           int T, int H, int k, int rows, int nsplit, size_t split_stride, uint16_t* y, DevStatus* st,
                           cudaStream_t s);

// row_token[inv_perm[t, j]] = t for every slot, and the counters in `zero` cleared.
cudaError_t launch_row_tokens(const int32_t* inv_perm, int T, int k, int32_t* row_token, ZeroSpan zero, DevStatus* st,
                              cudaStream_t s);

// h = bf16(silu(sum_s gate_s) * sum_s up_s) from K-split partial slabs [rows, 2I].
cudaError_t launch_swiglu_reduce(const float* partials, int nsplit, size_t split_stride, int rows, int I, uint16_t* h,
                                 cudaStream_t s);

// Router for a few tokens (T <= kSmallRouterT, E % 4 == 0): fp32 logits with
// H split over blocks; the last block to finish sums the partial slabs
// (small_router_slabs(H, E) of them, [slab][T][E] in `partial`) in slab
// order, selects the top-k under the scoring rule (MOE_SCORE_*) and, if counts != nullptr, writes the
// permutation (counts, offsets, sorted_ids, inv_perm) as launch_permute
// would.  *arrivals must be zero on entry and is zero again on exit.
constexpr int kSmallRouterT = 16;

int small_router_slabs(int H, int E);
cudaError_t launch_router_small(const uint16_t* x, const float* w, const float* bias, int T, int H, int E, int k,
                                int scoring, float* partial, unsigned int* arrivals, int32_t* ids, float* wout,
                                int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* inv_perm,
                                DevStatus* st, ZeroSpan zero, cudaStream_t s);

// The whole layer for T <= kSmallRouterT tokens in one persistent launch on
// the tensor cores (layer_small.cu): the few-token router, then the gate/up
// and the down grouped GEMM as one sequence of work units, the combine in the
// down GEMM's epilogue.  E % 4 == 0, no shared expert.
struct LayerParams {
  const uint16_t* x;
  const float* w_router;
  const float* bias;
  int scoring;
  int T, H, E, k;
  float* partial;  // router partial slabs [small_router_slabs(H, E)][T][E]
  int32_t *ids, *counts, *offsets, *sids, *inv;
  float* tw;
  uint32_t* expert_done;  // [E][I/128]: epilogue warps done with each gate/up column block of each expert
  ZeroSpan zero;          // the arrival counters of both GEMMs and expert_done, cleared in the launch
  GemmArgs gu, dn;        // the two GEMMs (gate/up: SwiGLU, or K-split slabs + SwiGLU; down: combine)
  DevStatus* st;
  uint64_t timeout_ns;
};
bool layer_small_supported(int T, int E, int I_s);
cudaError_t launch_layer_small(const CUtensorMap& gu_map, const CUtensorMap& dn_map, const LayerParams& p,
                               int num_sms, cudaStream_t s);

cudaError_t launch_selftest_timeout(DevStatus* st, uint64_t timeout_ns, cudaStream_t s);

}  // namespace moe
