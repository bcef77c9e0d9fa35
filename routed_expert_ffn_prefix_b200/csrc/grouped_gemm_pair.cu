// grouped_gemm_pair.cu -- grouped expert GEMM on SM pairs (tcgen05 cta_group::2).
//
// The variant of the grouped GEMM selected with MOE_TILES_PAIR
// (grouped_gemm.cu has the design notes shared by both).  Same orientation
// as the single-SM kernel -- weight columns are the MMA's M side, the
// expert's token rows its N side -- but one MMA spans the two SMs of a
// cluster: M = 256 weight columns (128 in each SM's TMEM lanes), N = the
// unit's rows rounded up to 16 (<= 256), of which each SM gathers half.
//
// Why: at prefill sizes (~160 rows per expert) the single-SM kernel is paced
// by the gathered token rows (32 KB per 64-deep stage at 256 rows) and only
// three stages fit in shared memory.  Here each SM stages 32 KB of weights
// (its 128 columns of the two tiles) but only 16 KB of rows, so four stages
// fit, and every SM still streams each weight byte once per 256-row pass.
//
//   * gate/up: the two tiles are the gate and the up columns of the same 256
//     intermediate units (128 per SM), so SwiGLU stays thread-local;
//   * down: the two tiles are 2 x 256 adjacent output columns.
//
// Rows by TMA (RTMA, the down GEMM): the operand rows are h, already in
// expert order, so each SM loads its half of a unit's rows with one TMA box
// per stage (128 rows; rows past the unit's are loaded but not read by the
// MMA) instead of gathering them row by row.
// Output rows by TMA (OTMA: the down GEMM's fp32 rows, the gate/up GEMM's
// bf16 h rows): each epilogue warp stages 16 rows x 32 columns at a time in
// shared memory and issues a bulk tensor store, so TMEM is released once the
// rows are staged and the stores drain while the next unit's MMAs run
// (written by plain stores, all SMs' epilogues contended for the write
// bandwidth at once and held the MMAs for ~8K cycles per down unit).
//
// Synchronisation (cluster of 2; rank 0 = leader issues every MMA):
//   full[s]  (leader): 128 cp.async arrivals of the leader's rows, the
//            leader's expect_tx for both SMs' weight bytes, and one relayed
//            arrival from the peer once its rows have landed.  Both SMs' TMA
//            weight loads complete their bytes on the leader's barrier.
//   xfull[s] (peer):   the peer's 128 cp.async arrivals; the peer's relay
//            thread waits on it, fences the writes into the async proxy and
//            arrives on the leader's full[s].
//            With RTMA both SMs' row boxes complete their bytes on the
//            leader's full[s] as the weights do: its only arrival is the
//            leader's expect_tx, and there is no relay.
//   empty[s], tfull (both): arrived by the leader's commits, multicast to
//            both SMs of the pair.
//   tempty (leader): one arrival per epilogue warp of both SMs.
// Every wait is bounded; both SMs meet at a cluster barrier before TMEM is
// released and the blocks exit.
//
// Warp roles (416 threads): warps 0-7 epilogue, warps 8-11 producers
// (cp.async rows; thread 0 also issues the weight TMA), warp 12: TMEM
// allocation, MMA issue (leader) or completion relay (peer).
#include "gemm_units.cuh"

namespace moe {

namespace {

constexpr int kPEpiWarps = 8;
constexpr int kPProdWarps = 4;
constexpr int kPCtlWarp = kPEpiWarps + kPProdWarps;
constexpr int kPThreads = (kPCtlWarp + 1) * 32;
constexpr int kPProdThreads = kPProdWarps * 32;
constexpr int kPBoxBytes = 64 * kBK * 2;  // 8 KB: one 64-column TMA box of weights
constexpr int kPATileBytes = 2 * kPBoxBytes;  // 16 KB: this SM's 128 columns of one tile

// NT: rows per pass (N <= NT, NT/2 gathered per SM); ST: pipeline stages;
// MT: MMA tiles per unit (gate + up, or 1-2 output blocks of 256 columns).
template <int NT, int ST, int MT>
struct PCfg {
  static constexpr int ROWS = NT / 2;
  static constexpr int A_BYTES = MT * kPATileBytes;
  static constexpr int B_BYTES = ROWS * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NBUF = (2 * MT * NT <= 512) ? 2 : 1;  // accumulators double-buffered if they fit
  static constexpr int TMEM_COLS = 512;
  static constexpr int OSTAGE_OFF = (ST * STAGE_BYTES + 512 + 4 * kPrefixInts + 1023) & ~1023;  // fp32 row staging
  static constexpr int OSTAGE_BYTES = kPEpiWarps * 16 * 32 * 4;                // 16 rows x 32 columns per warp
  static constexpr int SMEM_BYTES = OSTAGE_OFF + OSTAGE_BYTES + 1024;
  static_assert(NT % 32 == 0 && NT >= 32 && NT <= 256, "row pass must be 32..256, multiple of 32");
  static_assert(MT == 1 || MT == 2, "one or two MMA tiles per unit");
  static_assert(MT * NT * NBUF <= TMEM_COLS, "accumulators must fit in TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte swizzle alignment");
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Relayed "rows landed" signal.  The rows were written to this SM's own
// shared memory and are read by this SM's own tensor core (each SM computes
// its half of M from its own A tile), and they have fully landed before the
// relay observes its local barrier; a release at cluster scope here costs
// about 1,300 cycles per stage (measured) and would pace the whole pipeline,
// so the arrive is relaxed, after a proxy fence for the tensor core's reads.
__device__ __forceinline__ void remote_arrive_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bulk tensor store of a shared-memory box (fp32 rows), tracked by this
// thread's bulk-async group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk stores have finished reading their shared-memory sources
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// TMA tile load whose completion is signalled on a barrier of either SM of the pair.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the barrier at this smem offset in both SMs of the pair once the
// MMAs issued so far have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}

// Arrive on the leader's barrier (rank 0 only) once the MMAs issued so far have completed.
__device__ __forceinline__ void mma_commit_pair_leader(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)1)
      : "memory");
}

template <int NT, int ST, int MT, int EPI, bool RTMA, bool OTMA>
__global__ void __launch_bounds__(kPThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap rmap,
                             const __grid_constant__ CUtensorMap omap, const GemmArgs a) {
  using C = PCfg<NT, ST, MT>;
  static_assert(!RTMA || C::ROWS == 128, "row boxes of 128 rows");
  static_assert(!RTMA || EPI == EPI_STORE_F32, "rows by TMA: the down GEMM's store epilogue");
  static_assert(!OTMA || EPI == EPI_STORE_F32 || EPI == EPI_SWIGLU, "output rows by TMA: fp32 rows or h");
  static_assert(C::OSTAGE_OFF % 1024 == 0, "staging aligned for bulk copies");
  static_assert(EPI != EPI_SWIGLU || MT == 2, "SwiGLU needs the gate and the up tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * C::STAGE_BYTES);
  uint64_t* xfull = full + ST;
  uint64_t* empty = xfull + ST;
  uint64_t* tfull = empty + ST;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* total_units = abort_flag + 1;
  int* ustart = reinterpret_cast<int*>(smem + ST * C::STAGE_BYTES + 512);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int ngroups = a.offsets ? a.groups : 1;

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full + s, RTMA ? 1 : kPProdThreads + 2);  // (leader rows +) leader expect_tx (+ peer relay)
      mbar_init(xfull + s, kPProdThreads);     // peer rows
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 2 * kPEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kPCtlWarp) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == kPEpiWarps && lane == 0) {
    prefetch_tmap(&wmap);
    if (RTMA) prefetch_tmap(&rmap);
    if (OTMA) prefetch_tmap(&omap);
  }
  if (warp == 0) build_unit_prefix<NT>(a, ngroups, ustart, total_units);
  tc_fence_before();
  cluster_sync();  // barriers of both SMs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = *total_units;

  if (warp >= kPEpiWarps && warp < kPCtlWarp) {
    // ------------------------------------------------------------ producers
    // This SM gathers rows [rank * nh, rank * nh + nh) of the unit (nh = N/2)
    // and loads its 128 weight columns of both tiles.
    const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_PRODUCER};
    const int pt = tid - kPEpiWarps * 32;
    const int chunk = pt & 7, rsub = pt >> 3;
    constexpr int kRowsPerThread = C::ROWS / (kPProdThreads / 8);
    // Weight tiles are streamed past L2 (evict-first), as in the single-SM kernel.
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_rows = a.rows_evict_last ? policy_evict_last() : policy_evict_normal();
    const __nv_bfloat16* bsrc = reinterpret_cast<const __nv_bfloat16*>(a.b_src);
    uint64_t* rows_bar_base = leader ? full : xfull;
    const uint32_t full_leader = map_to_rank(smem_u32(full), 0);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int u = pair; u < total && ok; u += npairs) {
      const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
      const int nh = ((un.rows + 15) & ~15) >> 1;
      const int my0 = (int)rank * nh;
      int src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int c = rsub + 16 * i;
        int sr = -1;
        if (c < nh && my0 + c < un.rows) {
          const int r = un.row0 + my0 + c;
          sr = a.row_index ? __ldg(a.row_index + r) : r;
          if (sr < 0 || sr >= a.src_rows) {
            raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_GEMM_GATHER, r);
            sr = -1;
          }
        }
        src[i] = sr;
      }
      const int wcol = un.nb * a.col_stride + (int)rank * 128;  // this SM's 128 columns of tile 0
      const int nk = un.ke - un.kb, kiters = nk * a.krep;
      for (int it = 0; it < kiters; ++it) {
        const int rep = it / nk, kt = un.kb + (it - rep * nk);
        if (!mbar_wait(&empty[stage], phase ^ 1u, wc, 100 + stage)) { ok = false; break; }
        uint8_t* sA = smem + stage * C::STAGE_BYTES;
        const uint32_t sb = smem_u32(sA + C::A_BYTES);
        if (pt == 0) {  // the weight tiles first: they come from HBM, the rows mostly from L2
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (C::A_BYTES + (RTMA ? C::B_BYTES : 0)));
          const int d2 = a.a_dim2_rep ? rep : un.group;
          const uint32_t fb = full_leader + stage * 8;
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const int c = wcol + t * a.col1_off;
            tma_load_3d_pair(sA + t * kPATileBytes, &wmap, fb, c, kt * kBK, d2, pol_w);
            tma_load_3d_pair(sA + t * kPATileBytes + kPBoxBytes, &wmap, fb, c + 64, kt * kBK, d2, pol_w);
          }
          // rows map: 3D [1][src_rows][K], like the weight maps
          if constexpr (RTMA) tma_load_3d_pair(sA + C::A_BYTES, &rmap, fb, kt * kBK, un.row0 + my0, 0, pol_rows);
        }
        if constexpr (!RTMA) {
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            if (src[i] >= 0) {
              const int c = rsub + 16 * i;
              cp_async_16(sb + c * 128 + ((chunk ^ (c & 7)) << 4),
                          bsrc + (size_t)src[i] * a.K + kt * kBK + chunk * 8, pol_rows);
            }
          }
          cp_async_arrive_noinc(&rows_bar_base[stage]);
        }
        if (++stage == ST) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait_all();
    if (!ok && pt == 0) {
      // Aborted: weight tiles this SM requested may still be landing in its
      // shared memory (their completion is counted on the leader); give them
      // time to arrive before the block can exit.
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 50000ull) {
      }
    }
  } else if (warp == kPCtlWarp) {
    if (leader) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_MMA};
        int stage = 0;
        uint32_t phase = 0;
        int acc_it = 0;
        bool ok = true;
        // Descriptors of stage 0; a stage, a k slice and a tile add to the
        // start-address field (address / 16, below 2^14 in shared memory).
        // A = weights (MN-major): +16 k = two 8-row groups = 2048 B, the two
        // 64-column halves of a tile one TMA box apart; B = rows (K-major):
        // +16 k = 32 B inside the swizzled row.
        const uint64_t ad0 = smem_desc_sw128(smem_u32(smem), kPBoxBytes, 1024);
        const uint64_t bd0 = smem_desc(smem_u32(smem) + C::A_BYTES, 16, 1024, kLayoutSw128);
        for (int u = pair; u < total && ok; u += npairs) {
          const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
          const int buf = C::NBUF == 2 ? (acc_it & 1) : 0;
          const uint32_t apar = C::NBUF == 2 ? ((acc_it >> 1) & 1) : (acc_it & 1);
          if (!mbar_wait(&tempty[buf], apar ^ 1u, wc, 200 + buf)) break;
          tc_fence_after();
          const uint32_t d0 = tmem + buf * MT * NT;
          // A = weights (MN-major), M = 256 over the pair; B = rows (K-major), N = rows rounded to 16.
          const int N = (un.rows + 15) & ~15;
          const uint32_t idesc = idesc_bf16_f32(256, N, /*A MN-major*/ true, /*B K-major*/ false);
          const int kiters = (un.ke - un.kb) * a.krep;
          uint32_t acc = 0;
          for (int it = 0; it < kiters; ++it) {
            if (!mbar_wait(&full[stage], phase, wc, 300 + stage)) { ok = false; break; }
            tc_fence_after();
            fence_proxy_async_smem();
            const uint64_t soff = (uint32_t)(stage * C::STAGE_BYTES) >> 4;
            const uint64_t ads = ad0 + soff, bds = bd0 + soff;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
              for (int t = 0; t < MT; ++t)
                mma_bf16_pair(d0 + t * NT, ads + ((t * kPATileBytes + kk * 2048) >> 4), bds + 2 * kk, idesc, acc);
              acc = 1;
            }
            mma_commit_pair(&empty[stage]);
            if (++stage == ST) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          mma_commit_pair(&tfull[buf]);
          ++acc_it;
        }
        mma_commit_pair_leader(mma_done);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(mma_done, 0) && globaltimer_ns() - t0 < a.timeout_ns) {
        }
      }
    } else if (lane == 0) {
      // ---------------------------------------------------------- peer relay
      // Forward "this SM's rows of stage s have landed" to the leader.
      const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_PRODUCER};
      const uint32_t full_leader = map_to_rank(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < total && ok && !RTMA; u += npairs) {
        const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
        const int kiters = (un.ke - un.kb) * a.krep;
        for (int it = 0; it < kiters; ++it) {
          if (!mbar_wait(&xfull[stage], phase, wc, 500 + stage)) { ok = false; break; }
          fence_proxy_async_smem();
          remote_arrive_relaxed(full_leader + stage * 8);
          if (++stage == ST) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-7)
    // Warp w reads TMEM lanes 32*(w%4).. = this SM's weight columns
    // 32*(w%4).. (one column per thread) and the 32-row chunks
    // c0 = 32*(w/4) + 64*j of the unit's rows (TMEM column = row).
    const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_EPILOGUE};
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t tempty_leader = map_to_rank(smem_u32(tempty), 0);
    int acc_it = 0;
    for (int u = pair; u < total; u += npairs) {
      const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
      const int buf = C::NBUF == 2 ? (acc_it & 1) : 0;
      const uint32_t apar = C::NBUF == 2 ? ((acc_it >> 1) & 1) : (acc_it & 1);
      if (!mbar_wait(&tfull[buf], apar, wc, 400 + buf)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * MT * NT;
      const int col = un.nb * a.out_col_stride + (int)rank * 128 + quarter * 32 + lane;
      for (int c0 = half * 32; c0 < un.rows; c0 += 64) {
        const int nr = min(32, un.rows - c0);
        if (EPI == EPI_SWIGLU) {
          float g[32], v[32];
          tmem_ld_4x16(tbase + c0, tbase + c0 + 16, tbase + NT + c0, tbase + NT + c0 + 16, g, g + 16, v, v + 16);
          if constexpr (OTMA) {  // whole 32-row chunks by bulk tensor stores, as the fp32 rows below
            const int cb = col - lane;
            if (nr == 32 && cb + 32 <= a.n_valid) {
              __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem + C::OSTAGE_OFF) + warp * (16 * 32);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  stg[j * 32 + lane] = __float2bfloat16_rn(silu_f(g[hh * 16 + j]) * v[hh * 16 + j]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  tma_store_3d(&omap, stg, cb, un.row0 + c0 + hh * 16, 0);
                  bulk_commit();
                }
              }
              continue;
            }
          }
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
          if (col < a.n_valid) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nr)
                out[(size_t)(un.row0 + c0 + j) * a.ld_out + col] = __float2bfloat16_rn(silu_f(g[j]) * v[j]);
            }
          }
        } else {  // fp32 rows (EPI_STORE_F32, and the rows of the down-combine reduction)
          // both tiles' 32 rows in one batch of TMEM loads (one wait), then the stores
          float v[MT][32];
          if constexpr (MT == 2) {
            tmem_ld_4x16(tbase + c0, tbase + c0 + 16, tbase + NT + c0, tbase + NT + c0 + 16, v[0], v[0] + 16, v[1],
                         v[1] + 16);
          } else {
            tmem_ld_2x16(tbase + c0, tbase + c0 + 16, v[0], v[0] + 16);
          }
          if constexpr (OTMA) {
            // whole 32-row chunks of in-range columns by bulk tensor stores (a
            // box must not reach past the unit's rows: they are another
            // expert's); a partial chunk by plain stores below
            const int cb = col - lane;  // this warp's first column
            if (nr == 32 && cb + (MT - 1) * a.out_col1_off + 32 <= a.n_valid) {
              float* stg = reinterpret_cast<float*>(smem + C::OSTAGE_OFF) + warp * (16 * 32);
#pragma unroll
              for (int t = 0; t < MT; ++t) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  if (lane == 0) bulk_wait_read_all();  // the previous box has left the buffer
                  __syncwarp();
#pragma unroll
                  for (int j = 0; j < 16; ++j) stg[j * 32 + lane] = v[t][hh * 16 + j];
                  fence_proxy_async_smem();
                  __syncwarp();
                  if (lane == 0) {
                    tma_store_3d(&omap, stg, cb + t * a.out_col1_off, un.row0 + c0 + hh * 16, 0);
                    bulk_commit();
                  }
                }
              }
              continue;
            }
          }
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const int ct = col + t * a.out_col1_off;
            if (ct < a.n_valid) {
              float* out = reinterpret_cast<float*>(a.out) + (size_t)un.ks * a.split_stride;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nr) out[(size_t)(un.row0 + c0 + j) * a.ld_out + ct] = v[t][j];
            }
          }
        }
      }
      // TMEM is free once this warp's loads are done (tcgen05.wait::ld inside
      // the loads), whatever its stores: a release at cluster scope would
      // also wait for every global store above to drain (~1,200 cycles per
      // unit, measured) while the next unit's MMAs wait for this arrival.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive_relaxed(tempty_leader + buf * 8);
      ++acc_it;
      if constexpr (EPI == EPI_DOWN_COMBINE) {
        // TMEM is released; now count this warp's stored rows and reduce the
        // chunks they complete while the next unit's MMAs run.
        __syncwarp();
        __threadfence();
        int cols[MT];
        cols[0] = col;
        if constexpr (MT == 2) cols[1] = col + a.out_col1_off;
        const int chunk = (un.nb * 2 + (int)rank) * 4 + quarter;
        for (int c0 = half * 32; c0 < un.rows; c0 += 64)
          arrive_rows<MT, EPI>(a, un.row0 + c0, min(32, un.rows - c0), chunk, cols);
      }
    }
    if constexpr (OTMA) {  // every bulk store of this warp complete before the block leaves
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  // Both SMs finish every access to each other's shared memory and barriers
  // before TMEM is released and either block exits.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kPCtlWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

template <int NT, int ST, int MT, int EPI, bool RTMA = false, bool OTMA = false>
cudaError_t launch_pair(const CUtensorMap& wmap, const CUtensorMap* rmap, const CUtensorMap* omap, const GemmArgs& a,
                        int num_sms, cudaStream_t stream) {
  using C = PCfg<NT, ST, MT>;
  auto kern = grouped_gemm_pair_kernel<NT, ST, MT, EPI, RTMA, OTMA>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t err = once_per_device(configured, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // One pair per co-resident cluster slot (persistent); the slot count is
  // queried once per device.
  static std::atomic<int> queried[kMaxDevices];
  static int slots[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  cfg.gridDim = dim3(num_sms & ~1, 1, 1);
  if (dev >= 0 && dev < kMaxDevices) {
    once_per_device(queried, [&] {
      int clusters = 0;
      slots[dev] = (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess) ? clusters : 0;
      return cudaSuccess;
    });
    if (slots[dev] > 0 && 2 * slots[dev] < (int)cfg.gridDim.x) cfg.gridDim = dim3(2 * slots[dev], 1, 1);
  }
  return cudaLaunchKernelEx(&cfg, kern, wmap, RTMA ? *rmap : wmap, OTMA ? *omap : wmap, a);
}

}  // namespace

cudaError_t launch_grouped_gemm_pair(const CUtensorMap& wmap, const CUtensorMap* rows_map, const CUtensorMap* out_map,
                                     const GemmArgs& a, int epilogue, int num_sms, cudaStream_t stream) {
  // 256-row passes.  Measured alternatives with gathered rows (isolated
  // kernel, in one process; 8192-token prefill shape / Zipf-skewed
  // 4096-token shape):
  //   gate/up 256/4: 1.58 / 3.58 ms; 192/5: 1.62 / 3.73 ms; 128/5: 2.56 / 4.52 ms
  //   down    256/4: 1.12 / 2.07 ms; 192/5: 0.98 / 2.11 ms; 128/5: 1.45 / 2.33 ms
  // but inside the layer, where h was just written and partly sits in L2,
  // the 192/5 down GEMM measured slower (1.11 vs 1.07 ms; 2.32 vs 2.24 ms).
  // One 256-column tile per unit with a double-buffered accumulator and
  // gathered rows: down 1.03 / 2.35 ms.
  // rows_map (the down GEMM's rows, contiguous): the rows by TMA, one box per
  // stage and SM instead of 1024 row-chunk copies; in the layer, down
  // 1.07-1.10 vs 1.12-1.16 ms (prefill) and 2.19-2.24 vs 2.22-2.23 ms
  // (skewed).  With one 256-column tile per unit and double-buffered
  // accumulators on top, the skewed shape lost 10% (h read twice as often).
  if (rows_map != nullptr) {
    if (a.row_index != nullptr || epilogue != EPI_STORE_F32 || out_map == nullptr || a.k_splits != 1)
      return cudaErrorInvalidValue;
    return launch_pair<256, 4, 2, EPI_STORE_F32, true, true>(wmap, rows_map, out_map, a, num_sms, stream);
  }
  if (out_map != nullptr) {
    if (epilogue != EPI_SWIGLU || a.k_splits != 1) return cudaErrorInvalidValue;
    return launch_pair<256, 4, 2, EPI_SWIGLU, false, true>(wmap, nullptr, out_map, a, num_sms, stream);
  }
  switch (epilogue) {
    case EPI_SWIGLU: return launch_pair<256, 4, 2, EPI_SWIGLU>(wmap, nullptr, nullptr, a, num_sms, stream);
    case EPI_DOWN_COMBINE:
      return launch_pair<256, 4, 2, EPI_DOWN_COMBINE>(wmap, nullptr, nullptr, a, num_sms, stream);
    case EPI_STORE_F32: return launch_pair<256, 4, 2, EPI_STORE_F32>(wmap, nullptr, nullptr, a, num_sms, stream);
    default: return cudaErrorInvalidValue;  // the K split (and its SwiGLU reduction) runs on single SMs only
  }
}

}  // namespace moe
