// layer_small.cu -- the whole MoE layer for a few tokens in one persistent
// launch on the tensor cores.
//
// With a handful of tokens the layer is a stream of the selected experts'
// weights, and separate kernels lose the stream at every boundary: the
// router's tail, each GEMM's pipeline ramp and its last, partly idle wave.
// The Muse Spark on TPU v7 page ("changing dependencies") issues the expert
// weight DMA as soon as the selection is known and runs the layer as one
// program; here one cooperative launch of the grouped GEMM's warp roles
// (gemm_pipeline.cuh) on every SM does:
//
//   1. routing: the blocks compute the split-H partial logits of the router
//      items (route_dev.cuh) and count themselves in; once all are in, every
//      block sums the partials, selects the top-k and builds the permutation
//      and its unit schedule in its own shared memory (the same values in
//      every block; nothing to publish, no second wait); the GEMM roles read
//      the routing from there, and block 0 alone writes it out for the
//      caller.  Meanwhile every block has initialised its pipeline and
//      allocated TMEM.
//   2. one sequence of work units: first every gate/up unit (SwiGLU; for a
//      K split, the slab sum + SwiGLU by the last slab to land), then every
//      down unit.  A down unit's producers wait until the gate/up units that
//      write the columns of h its K slice reads have finished their
//      epilogues (a counter per expert and gate/up column block), so the
//      down stream of early experts runs under the gate/up stream of later
//      ones instead of after it.  No block waits for a unit that is
//      not already running: gate/up units never wait, and every block takes
//      its units in increasing order, all gate/up units before any down unit.
//   3. the weighted, slot-order combine in the down GEMM's epilogue (the last
//      of each token's k rows to land writes that chunk of y).
//
// Every wait is bounded; the block that finishes last returns the router's
// arrival word and the exit word to zero.
#include "gemm_pipeline.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kLNT = 128, kLST = 4, kLMT = 2, kLBK = 64;  // the decode tiles of the grouped GEMM
using LCfg = Cfg<kLNT, kLST, kLMT, kLBK>;
using LSmem = PipeSmem<kLNT, kLST, kLMT, kLBK>;

// The two GEMMs as one unit sequence: [0, total0) gate/up, then down.
struct LayerSched {
  static constexpr int kPhases = 2;
  const GemmArgs* gu;
  const GemmArgs* dn;
  const CUtensorMap* gu_map;
  const CUtensorMap* dn_map;
  const int* ustart;   // gate/up unit prefix
  const int* ustart1;  // down unit prefix
  int ngroups, total0;
  uint32_t* expert_done;
  DevStatus* st;
  uint64_t timeout_ns;

  __device__ PUnit decode(int u) const {
    if (u < total0) return PUnit{decode_unit<kLNT>(*gu, ustart, ngroups, u), 0};
    return PUnit{decode_unit<kLNT>(*dn, ustart1, ngroups, u - total0), 1};
  }
  __device__ const GemmArgs& args(int phase) const { return phase ? *dn : *gu; }
  __device__ const CUtensorMap* tmap(int phase) const { return phase ? dn_map : gu_map; }

  // Gate/up units of expert e, and of one of its column blocks.
  __device__ int units0(int e) const { return (e + 1 < ngroups ? ustart[e + 1] : total0) - ustart[e]; }
  __device__ int units0_per_block(int e) const { return units0(e) / gu->n_blocks; }
  static_assert(kPrefixInts > kMaxExperts, "unit starts come first in the prefix");

  // A down unit of expert e reads the columns [64 kb, 64 ke) of e's rows of
  // h, written by e's gate/up column blocks kb/2 .. (ke-1)/2 (128 columns
  // each): wait (lane 0 of each producer warp, bounded) until every
  // epilogue warp of every gate/up unit of those blocks has counted itself
  // done.
  __device__ bool before_loads(const PUnit& pu, volatile int* abort_flag) const {
    if (pu.phase == 0) return true;
    const int e = pu.un.group, nbg = gu->n_blocks;
    const uint32_t target = (uint32_t)(units0_per_block(e) * kEpiWarps);
    int ok = 1;
    if (lane_id() == 0) {
      const uint64_t t0 = globaltimer_ns();
      for (int nb = pu.un.kb / 2; nb <= (pu.un.ke - 1) / 2 && ok; ++nb) {
        while (ld_acquire_gpu(expert_done + (size_t)e * nbg + nb) < target) {
          if (*abort_flag) {
            ok = 0;
            break;
          }
          if (globaltimer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            raise_error(st, MOE_ERR_DEVICE_TIMEOUT, SITE_LAYER, 1000 + e);
            ok = 0;
            break;
          }
          __nanosleep(32);
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __threadfence();  // acquire side: this warp's row gathers come after the counters were seen
    return ok != 0;
  }

  // Every lane's h stores (and a K-split's finishing sums) are made visible
  // device-wide before the warp counts the unit done for its column block.
  __device__ void after_epilogue(const PUnit& pu) const {
    if (pu.phase != 0) return;
    __threadfence();
    __syncwarp();
    if (lane_id() == 0) atomicAdd(expert_done + (size_t)pu.un.group * gu->n_blocks + pu.un.nb, 1u);
  }
};

// Shared memory beyond the pipeline's: each block's copy of the routing
// metadata the GEMM roles read (permuted row -> token, slot -> row, slot
// weights) and of the two GEMMs' arguments pointing at it.
struct LayerMeta {
  int32_t sids[kSmallMaxSlots];
  int32_t inv[kSmallMaxSlots];
  float tw[kSmallMaxSlots];
  GemmArgs gu, dn;
};
constexpr int kLayerSmemBytes = LCfg::SMEM_BYTES + (int)((sizeof(LayerMeta) + 15) & ~size_t(15));
static_assert(kLayerSmemBytes <= 232448, "shared memory budget of the persistent layer");

template <int TT>
struct RouterOverlay {
  static constexpr size_t kRsm = (sizeof(RouterSmem<TT>) + 15) & ~size_t(15);
  static constexpr size_t kBytes = kRsm + 4 * (kSmallMaxSlots + kMaxExperts + kSmallThreads / 32 + kMaxExperts + 1);
  static_assert(kSmallRouterT * kMaxK <= kSmallMaxSlots, "slot arrays hold every slot");
};

template <int TT, int EPL, int EPI_GU>
__global__ void __launch_bounds__(kGemmThreads, 1)
    layer_small_kernel(const __grid_constant__ CUtensorMap gu_map, const __grid_constant__ CUtensorMap dn_map,
                       const __grid_constant__ LayerParams p) {
  static_assert(RouterOverlay<TT>::kBytes <= (size_t)kLST * LCfg::STAGE_BYTES, "router overlay fits in the stage ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const LSmem sm = LSmem::carve(smem);
  LayerMeta& meta = *reinterpret_cast<LayerMeta*>(smem + LCfg::SMEM_BYTES - 1024);  // past the prefixes
  __shared__ int s_total1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  sm.init(tid, warp);
  if (warp == kEpiWarps && lane == 0) {
    prefetch_tmap(&gu_map);
    prefetch_tmap(&dn_map);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;

  // ---------------------------------------------------------------- 1. routing
  // The router's shared memory overlays the stage ring, which no load has
  // touched yet.
  RouterSmem<TT>& rsm = *reinterpret_cast<RouterSmem<TT>*>(sm.ring);
  int32_t* sel = reinterpret_cast<int32_t*>(sm.ring + RouterOverlay<TT>::kRsm);
  int32_t* cnt = sel + kSmallMaxSlots;
  int32_t* wsum = cnt + kMaxExperts;
  int32_t* soff = wsum + kSmallThreads / 32;  // [E + 1] expert offsets
  const SmallGrid rg = small_grid(p.H, p.E);
  const int nitems = rg.ncs * rg.hs;
  const int rblocks = nitems < (int)gridDim.x ? nitems : (int)gridDim.x;  // blocks with router items
  const bool router_block = (int)blockIdx.x < rblocks;
  if (router_block && tid < kSmallThreads) {
    for (int i = blockIdx.x * kSmallThreads + tid; i < p.zero.n16; i += rblocks * kSmallThreads)
      p.zero.p[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int it = blockIdx.x; it < nitems; it += rblocks)
      router_partial<TT, 1>(reinterpret_cast<const __nv_bfloat16*>(p.x), p.w_router, p.T, p.H, p.E, rg.chunk,
                            it % rg.ncs, it / rg.ncs, p.partial, rsm);
  }
  __syncthreads();
  // Every block waits until all partial slabs (and the zeroed counters) are
  // in, then selects, weights and permutes the few tokens itself: the same
  // deterministic computation in every block, so each block has the routing
  // in its own shared memory at once (no block publishes it to the others),
  // and every block writes the same values to the routing outputs.
  if (tid == 0) {
    if (router_block) {
      __threadfence();
      atomicAdd(&p.st->arrivals, 1u);
    }
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(&p.st->arrivals) < (uint32_t)rblocks) {
      if (globaltimer_ns() - t0 > p.timeout_ns) {
        raise_error(p.st, MOE_ERR_DEVICE_TIMEOUT, SITE_LAYER, 0);
        *sm.abort_flag = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  const bool go = *sm.abort_flag == 0;
  const int n = p.T * p.k;
  if (go && tid < kSmallThreads)
    router_finish<EPL, 1>(p.partial, rg.hs, p.bias, p.T, p.E, p.k, p.scoring, sel, meta.tw, nullptr, soff,
                          meta.sids, meta.inv, p.st, sel, cnt, wsum);
  if (tid == 0) {
    meta.gu = p.gu;
    meta.gu.row_index = meta.sids;
    meta.dn = p.dn;
    meta.dn.row_token = meta.sids;
    meta.dn.inv_perm = meta.inv;
    meta.dn.topk_w = meta.tw;
  }
  __syncthreads();
  // ---------------------------------------------------------------- 2. the expert GEMMs
  if (go) {
    if (warp == 0) build_unit_prefix<kLNT>(p.gu, p.E, sm.ustart, sm.total_units, soff);
    if (warp == 1) build_unit_prefix<kLNT>(p.dn, p.E, sm.ustart1, &s_total1, soff);
    if (blockIdx.x == 0 && warp >= 2) {  // the routing outputs, for the caller
      for (int i = tid - 64; i < n; i += kGemmThreads - 64) {
        p.ids[i] = sel[i];
        p.tw[i] = meta.tw[i];
        p.sids[i] = meta.sids[i];
        p.inv[i] = meta.inv[i];
      }
      for (int e = tid - 64; e <= p.E; e += kGemmThreads - 64) {
        p.offsets[e] = soff[e];
        if (e < p.E) p.counts[e] = soff[e + 1] - soff[e];
      }
    }
  }
  fence_proxy_async_smem();  // the router's generic writes to the ring, before any TMA or cp.async write there
  __syncthreads();
  const int total0 = go ? *sm.total_units : 0;
  const int total = go ? total0 + s_total1 : 0;
  const LayerSched sched{&meta.gu, &meta.dn, &gu_map, &dn_map, sm.ustart, sm.ustart1, p.E, total0, p.expert_done,
                         p.st, p.timeout_ns};
  gemm_roles<kLNT, kLST, kLMT, kLBK, EPI_GU, EPI_DOWN_COMBINE>(sm, sched, tmem, blockIdx.x, gridDim.x, total, p.st,
                                                               p.timeout_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, LCfg::TMEM_COLS);
  }
  // ---------------------------------------------------------------- 3. leave the words at zero
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&p.st->exits, 1u) == gridDim.x - 1) {  // every block is past its routing wait
      p.st->exits = 0u;
      p.st->arrivals = 0u;
    }
  }
}

template <int TT, int EPL, int EPI_GU>
cudaError_t launch_t(const CUtensorMap& gu_map, const CUtensorMap& dn_map, const LayerParams& p, int num_sms,
                     cudaStream_t s) {
  auto kern = layer_small_kernel<TT, EPL, EPI_GU>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t err = once_per_device(configured, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLayerSmemBytes);
  });
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kLayerSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every block resident: the routing and expert waits need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, gu_map, dn_map, p);
}

template <int TT, int EPL>
cudaError_t launch_e(const CUtensorMap& gu_map, const CUtensorMap& dn_map, const LayerParams& p, int num_sms,
                     cudaStream_t s) {
  return p.gu.k_splits > 1 ? launch_t<TT, EPL, EPI_SWIGLU_SPLIT>(gu_map, dn_map, p, num_sms, s)
                           : launch_t<TT, EPL, EPI_SWIGLU>(gu_map, dn_map, p, num_sms, s);
}

template <int TT>
cudaError_t launch_tt(const CUtensorMap& gu_map, const CUtensorMap& dn_map, const LayerParams& p, int num_sms,
                      cudaStream_t s) {
  if (p.E <= 256) return launch_e<TT, 8>(gu_map, dn_map, p, num_sms, s);
  if (p.E <= 512) return launch_e<TT, 16>(gu_map, dn_map, p, num_sms, s);
  return launch_e<TT, 32>(gu_map, dn_map, p, num_sms, s);
}

}  // namespace

bool layer_small_supported(int T, int E, int I_s) {
  return T >= 1 && T <= kSmallRouterT && E % 4 == 0 && E <= kMaxExperts && I_s == 0;
}

cudaError_t launch_layer_small(const CUtensorMap& gu_map, const CUtensorMap& dn_map, const LayerParams& p,
                               int num_sms, cudaStream_t s) {
  if (!layer_small_supported(p.T, p.E, 0) || p.k > kMaxK) return cudaErrorInvalidValue;
  return p.T == 1 ? launch_tt<1>(gu_map, dn_map, p, num_sms, s) : launch_tt<kSmallRouterT>(gu_map, dn_map, p, num_sms, s);
}

}  // namespace moe
