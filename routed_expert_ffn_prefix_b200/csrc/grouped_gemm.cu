// grouped_gemm.cu -- persistent grouped GEMM on tcgen05/TMEM for the MoE expert FFN.
//
// Both expert GEMMs of the layer (gate/up with the SwiGLU epilogue, and
// down) and the tensor-core router run through this kernel.  It follows
// the grouped matmul of the Qwen 3.5-397B-on-Ironwood page (sec. 4.2,
// "grouped GEMM V2 with fused activation": SwiGLU inside the matmul, ragged
// per-expert row counts with minimal padding, token rows gathered straight
// from HBM with no padded permuted copy), re-designed for sm_100a:
//
//   * Orientation: the weight columns are the MMA's M side (128 per MMA
//     tile) and the expert's token rows are the N side (16..256).  An
//     expert's weight tile is therefore streamed from HBM once and applied
//     to every row routed to it, whatever the row count -- the layer is
//     bound by streaming the activated experts' weights, and decode-sized
//     groups of 1..30 rows need no padding to 128.
//   * A work unit = (group, column block, row pass).  A column block holds
//     MT (1 or 2) 128-column MMA tiles sharing the same token rows: for
//     gate/up (MT = 2) they are the gate and the up columns of the same 128
//     intermediate units, so SwiGLU is computed in the epilogue from two TMEM
//     accumulators; for down they are 128 or 256 adjacent output columns.
//   * Weight tiles arrive by TMA (128-byte swizzle, MN-major operand), token
//     rows by cp.async 16-byte gathers written in the same swizzle (K-major
//     operand), both into a multi-stage shared-memory ring guarded by
//     mbarriers.  One thread issues tcgen05.mma into TMEM; eight epilogue
//     warps (two per TMEM lane quarter, splitting the rows) drain TMEM with
//     tcgen05.ld.  Accumulators are double-buffered in TMEM when 2*MT*NT
//     columns fit in its 512, so a unit's epilogue overlaps the next unit's
//     MMAs; the single-tile mode (MT = 1) exists to get that overlap at 256
//     rows for the down GEMM, whose short K loop makes its epilogue heavy.
//   * A unit may cover a slice of K (split-K, store epilogue only): each
//     slice writes its own partial slab, summed later in a fixed order, so
//     results stay bitwise reproducible.  The router uses this to spread
//     small token counts over every SM.
//   * Every wait is bounded (see common.cuh); routing metadata is range
//     checked before it is used as an address.
//
// Warp roles (416 threads): warps 0-7 epilogue, warps 8-11 producers,
// warp 12 TMEM allocation + MMA issue.
#include "gemm_pipeline.cuh"

namespace moe {

namespace {

template <int NT, int ST, int MT, int EPI, int BK>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const PipeSmem<NT, ST, MT, BK> sm = PipeSmem<NT, ST, MT, BK>::carve(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ngroups = a.offsets ? a.groups : 1;
  sm.init(tid, warp);
  if (warp == kEpiWarps && lane == 0) prefetch_tmap(&wmap);
  if (warp == 0) build_unit_prefix<NT>(a, ngroups, sm.ustart, sm.total_units);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;
  const OnePhase<NT> sched{&a, &wmap, sm.ustart, ngroups};
  gemm_roles<NT, ST, MT, BK, EPI, EPI>(sm, sched, tmem, blockIdx.x, gridDim.x, *sm.total_units, a.status,
                                       a.timeout_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg<NT, ST, MT, BK>::TMEM_COLS);
  }
}

template <int NT, int ST, int MT, int EPI, int BK = 64>
cudaError_t launch_cfg(const CUtensorMap& wmap, const GemmArgs& a, int num_sms, cudaStream_t stream) {
  using C = Cfg<NT, ST, MT, BK>;
  auto kern = grouped_gemm_kernel<NT, ST, MT, EPI, BK>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t err = once_per_device(configured, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3(num_sms), dim3(kGemmThreads), C::SMEM_BYTES, stream, wmap, a);
}

}  // namespace

int gemm_tiles_per_unit(int tiles, int epilogue) {
  (void)tiles;
  (void)epilogue;
  return 2;  // measured: one tile per unit doubles the token-row re-reads and loses more than it overlaps
}

template <int NT, int ST>
cudaError_t launch_epi(const CUtensorMap& wmap, const GemmArgs& a, int epilogue, int num_sms, cudaStream_t stream) {
  switch (epilogue) {
    case EPI_SWIGLU: return launch_cfg<NT, ST, 2, EPI_SWIGLU>(wmap, a, num_sms, stream);
    case EPI_SWIGLU_SPLIT: return launch_cfg<NT, ST, 2, EPI_SWIGLU_SPLIT>(wmap, a, num_sms, stream);
    case EPI_DOWN_COMBINE: return launch_cfg<NT, ST, 2, EPI_DOWN_COMBINE>(wmap, a, num_sms, stream);
    default: return launch_cfg<NT, ST, 2, EPI_STORE_F32>(wmap, a, num_sms, stream);
  }
}

cudaError_t launch_grouped_gemm(const CUtensorMap& wmap, const GemmArgs& a, int epilogue, int tiles, int num_sms,
                                cudaStream_t stream) {
  if (tiles == MOE_TILES_LARGE) return launch_epi<256, 3>(wmap, a, epilogue, num_sms, stream);
  // Small groups (decode): 128-row passes, 4 stages -- measured ~5% faster
  // than 64-row passes with 5 stages at 1-30 rows per expert.
  return launch_epi<128, 4>(wmap, a, epilogue, num_sms, stream);
}

}  // namespace moe
