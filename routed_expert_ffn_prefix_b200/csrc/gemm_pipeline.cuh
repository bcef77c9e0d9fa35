// gemm_pipeline.cuh -- the warp roles of the single-SM grouped GEMM (producers,
// MMA issuer, epilogue), written once for the kernels that run them: the
// grouped GEMM of one weight matrix (grouped_gemm.cu) and the persistent
// few-token layer, which runs the gate/up and the down GEMM as one sequence
// of work units in a single launch (layer_small.cu).
//
// A schedule object tells the roles which work units exist and what each
// one is: decode(u) resolves unit u to its GEMM ("phase": 0 or 1) and its
// (group, column block, row pass, K split); args(phase)/tmap(phase) give that
// GEMM's arguments and weight tensor map; before_loads() may hold the
// producers back until the unit's inputs exist, and after_epilogue() reports
// a finished unit.  Every role walks the same units u = first, first +
// stride, ... and decodes them independently.
//
// Design notes of the pipeline itself are in grouped_gemm.cu.
#pragma once

#include "gemm_units.cuh"

namespace moe {

constexpr int kEpiWarps = 8;
constexpr int kProdWarps = 4;
constexpr int kMmaWarp = kEpiWarps + kProdWarps;
constexpr int kGemmThreads = (kMmaWarp + 1) * 32;
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kEpiThreads = kEpiWarps * 32;

template <int NT, int ST, int MT, int BK>
struct Cfg {
  // A stage holds BK of K: MT weight tiles of 128 columns (two 64-column TMA
  // boxes each, MN-major) and NT token rows (K-major, BK*2 bytes per row).
  static constexpr int ROW_BYTES = BK * 2;
  static constexpr int BOX_BYTES = 64 * BK * 2;
  static constexpr int ATILE_BYTES = 2 * BOX_BYTES;
  static constexpr int CHUNKS = ROW_BYTES / 16;  // 16-byte chunks per token row
  static constexpr uint32_t ROW_LAYOUT = BK == 64 ? kLayoutSw128 : kLayoutSw64;
  static constexpr uint32_t ROW_SBO = 8 * ROW_BYTES;  // one swizzle atom = 8 rows
  static constexpr int SUB = kBK / BK;  // stages per 64-wide k-step of the unit schedule
  static constexpr int B_BYTES = NT * ROW_BYTES;
  static constexpr int A_BYTES = MT * ATILE_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NBUF = (2 * MT * NT <= 512) ? 2 : 1;
  static constexpr int ACC_COLS = NBUF * MT * NT;
  static constexpr int TMEM_COLS = ACC_COLS <= 32 ? 32 : ACC_COLS <= 64 ? 64 : ACC_COLS <= 128 ? 128
                                   : ACC_COLS <= 256 ? 256 : 512;
  // ring + barriers/flags (256) + the unit prefixes of two GEMMs + alignment slack
  static constexpr int SMEM_BYTES = ST * STAGE_BYTES + 256 + 2 * 4 * kPrefixInts + 1024;
  static_assert(NT % 32 == 0 && NT >= 32 && NT <= 256, "row pass must be 32..256, multiple of 32");
  static_assert(MT == 1 || MT == 2, "one or two MMA tiles per unit");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte swizzle alignment");
  static_assert(BK == 64 || BK == 32, "stage depth: one 128-byte or 64-byte swizzle row");
};

// Physical 16-byte chunk of logical chunk `chunk` in row `row` of a K-major
// tile: the swizzle XORs the chunk index with row bits (128-byte: row % 8;
// 64-byte: (row / 2) % 4), matching what the MMA descriptor expects.
template <int BK>
__device__ __forceinline__ int swizzled_chunk(int chunk, int row) {
  return BK == 64 ? (chunk ^ (row & 7)) : (chunk ^ ((row >> 1) & 3));
}

// Shared-memory state of the pipeline: the stage ring, its barriers and the
// per-block flags.  carve() lays it out at the 1024-byte aligned base.
template <int NT, int ST, int MT, int BK>
struct PipeSmem {
  using C = Cfg<NT, ST, MT, BK>;
  uint8_t* ring;
  uint64_t *full, *empty, *tfull, *tempty, *mma_done;
  uint32_t* tmem_slot;
  int* abort_flag;
  int* total_units;
  int* ustart;   // [kPrefixInts] unit prefix of GEMM 0
  int* ustart1;  // [kPrefixInts] unit prefix of GEMM 1
  __device__ static PipeSmem carve(uint8_t* smem) {
    PipeSmem p;
    p.ring = smem;
    p.full = reinterpret_cast<uint64_t*>(smem + ST * C::STAGE_BYTES);
    p.empty = p.full + ST;
    p.tfull = p.empty + ST;
    p.tempty = p.tfull + 2;
    p.mma_done = p.tempty + 2;
    p.tmem_slot = reinterpret_cast<uint32_t*>(p.mma_done + 1);
    p.abort_flag = reinterpret_cast<int*>(p.tmem_slot + 1);
    p.total_units = p.abort_flag + 1;
    p.ustart = reinterpret_cast<int*>(smem + ST * C::STAGE_BYTES + 256);
    p.ustart1 = p.ustart + kPrefixInts;
    return p;
  }
  // Barrier init (thread 0) and TMEM allocation (warp kMmaWarp); the caller
  // follows with tc_fence_before / __syncthreads / tc_fence_after.
  __device__ void init(int tid, int warp) const {
    if (tid == 0) {
      for (int s = 0; s < ST; ++s) {
        mbar_init(full + s, kProdThreads + 1);  // producer cp.async arrivals + 1 expect_tx arrival
        mbar_init(empty + s, 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(tfull + b, 1);
        mbar_init(tempty + b, kEpiThreads);
      }
      mbar_init(mma_done, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    if (warp == kMmaWarp) {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
};

// A work unit resolved to its GEMM.
struct PUnit {
  Unit un;
  int phase;
};

// The schedule of one grouped GEMM (grouped_gemm.cu).
template <int NT>
struct OnePhase {
  static constexpr int kPhases = 1;
  const GemmArgs* a;
  const CUtensorMap* map;
  const int* ustart;
  int ngroups;
  __device__ PUnit decode(int u) const { return PUnit{decode_unit<NT>(*a, ustart, ngroups, u), 0}; }
  __device__ const GemmArgs& args(int) const { return *a; }
  __device__ const CUtensorMap* tmap(int) const { return map; }
  __device__ bool before_loads(const PUnit&, volatile int*) const { return true; }
  __device__ void after_epilogue(const PUnit&) const {}
};

// Epilogue of one unit by one epilogue warp: drain its TMEM lane quarter
// (one weight column per thread) for the 32-row chunks c0 = 32*half +
// 32*HALVES*j (HALVES warps per lane quarter) and store them (SwiGLU -> bf16, or fp32 rows / K slabs); for the
// last-arriver epilogues, release TMEM first, then count the stored rows and
// reduce the chunks they complete while the next unit's MMAs run.
template <int NT, int MT, int EPI, int HALVES = 2>
__device__ __forceinline__ void epilogue_unit(const GemmArgs& a, const Unit& un, uint32_t tbase, int quarter,
                                              int half, uint64_t* tempty_buf) {
  const int lane = lane_id();
  // argument fields in registers (the arguments may live in shared memory)
  const int ld_out = a.ld_out, n_valid = a.n_valid, out_col1_off = a.out_col1_off;
  const int col = un.nb * a.out_col_stride + quarter * 32 + lane;
  __nv_bfloat16* const hout = reinterpret_cast<__nv_bfloat16*>(a.out);
  float* const fout = reinterpret_cast<float*>(a.out) + (size_t)un.ks * a.split_stride;
  for (int c0 = half * 32; c0 < un.rows; c0 += 32 * HALVES) {
    const int nr = min(32, un.rows - c0);
    if constexpr (EPI == EPI_SWIGLU) {
      float g[32], v[32];
      tmem_ld_4x16(tbase + c0, tbase + c0 + 16, tbase + NT + c0, tbase + NT + c0 + 16, g, g + 16, v, v + 16);
      if (col < n_valid) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (j < nr) hout[(size_t)(un.row0 + c0 + j) * ld_out + col] = __float2bfloat16_rn(silu_f(g[j]) * v[j]);
        }
      }
    } else {  // fp32 rows (EPI_STORE_F32, and the slabs / rows of the last-arriver reductions)
      // both tiles' 32 rows in one batch of TMEM loads (one wait), then the stores
      float v[MT][32];
      if constexpr (MT == 2) {
        tmem_ld_4x16(tbase + c0, tbase + c0 + 16, tbase + NT + c0, tbase + NT + c0 + 16, v[0], v[0] + 16, v[1],
                     v[1] + 16);
      } else {
        tmem_ld_2x16(tbase + c0, tbase + c0 + 16, v[0], v[0] + 16);
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int ct = col + t * out_col1_off;
        if (ct < n_valid) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nr) fout[(size_t)(un.row0 + c0 + j) * ld_out + ct] = v[t][j];
        }
      }
    }
  }
  tc_fence_before();
  mbar_arrive(tempty_buf);
  if constexpr (EPI == EPI_SWIGLU_SPLIT || EPI == EPI_DOWN_COMBINE) {
    __syncwarp();
    __threadfence();
    int cols[MT];
    cols[0] = col;
    if constexpr (MT == 2) cols[1] = col + out_col1_off;
    const int chunk = un.nb * 4 + quarter;
    for (int c0 = half * 32; c0 < un.rows; c0 += 32 * HALVES)
      arrive_rows<MT, EPI>(a, un.row0 + c0, min(32, un.rows - c0), chunk, cols);
  }
}

// The three roles over the schedule's units [first, total) with stride
// `stride`.  EPI0 / EPI1: epilogues of GEMM 0 / GEMM 1.  status/timeout_ns
// for the bounded waits.
template <int NT, int ST, int MT, int BK, int EPI0, int EPI1, typename Sched>
__device__ __forceinline__ void gemm_roles(const PipeSmem<NT, ST, MT, BK>& sm, const Sched& S, uint32_t tmem,
                                           int first, int stride, int total, DevStatus* status,
                                           uint64_t timeout_ns) {
  using C = Cfg<NT, ST, MT, BK>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp >= kEpiWarps && warp < kMmaWarp) {
    // ------------------------------------------------------------ producers
    const WaitCtx wc{status, sm.abort_flag, timeout_ns, SITE_GEMM_PRODUCER};
    const int pt = tid - kEpiThreads;
    const int chunk = pt % C::CHUNKS, rsub = pt / C::CHUNKS;  // 16-byte chunk of a row; first row
    constexpr int kRowStep = kProdThreads / C::CHUNKS;
    constexpr int kRowsPerThread = NT / kRowStep;
    // Weight tiles are streamed past L2 (evict-first): keeping them (even for
    // groups with several row passes) measured slower, because it displaces
    // the token rows, which every column block of the group reads again.
    const uint64_t pol_w = policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;  // per stage: loads issued / parity of the last issue
    bool ok = true;
    for (int u = first; u < total && ok; u += stride) {
      const PUnit pu = S.decode(u);
      const Unit& un = pu.un;
      const GemmArgs& a = S.args(pu.phase);
      const CUtensorMap* wmap = S.tmap(pu.phase);
      if (!S.before_loads(pu, sm.abort_flag)) {
        ok = false;
        break;
      }
      // The unit's argument fields in registers: the arguments may live in
      // shared memory, which every asm statement below could clobber.
      const uint64_t pol_rows = a.rows_evict_last ? policy_evict_last() : policy_evict_normal();
      const __nv_bfloat16* const bsrc = reinterpret_cast<const __nv_bfloat16*>(a.b_src);
      const int K = a.K, col1_off = a.col1_off, krep = a.krep, dim2_rep = a.a_dim2_rep;
      int src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int c = rsub + kRowStep * i;
        int sr = -1;
        if (c < un.rows) {
          const int r = un.row0 + c;
          sr = a.row_index ? a.row_index[r] : r;  // generic load: global, or a block's shared copy
          if (sr < 0 || sr >= a.src_rows) {
            raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_GEMM_GATHER, r);
            sr = -1;
          }
        }
        src[i] = sr;
      }
      const int col0 = un.nb * a.col_stride;
      const int nk = (un.ke - un.kb) * C::SUB, kiters = nk * krep;  // stages per repeat, total
      for (int it = 0; it < kiters; ++it) {
        const int rep = it / nk;
        const int k0 = un.kb * kBK + (it - rep * nk) * BK;
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, wc, 100 + stage)) { ok = false; break; }
        uint8_t* sA = sm.ring + stage * C::STAGE_BYTES;
        const uint32_t sB = smem_u32(sA + C::A_BYTES);
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          if (src[i] >= 0) {
            const int c = rsub + kRowStep * i;
            cp_async_16(sB + c * C::ROW_BYTES + (swizzled_chunk<BK>(chunk, c) << 4),
                        bsrc + (size_t)src[i] * K + k0 + chunk * 8, pol_rows);
          }
        }
        cp_async_arrive_noinc(&sm.full[stage]);
        if (pt == 0) {
          mbar_arrive_expect_tx(&sm.full[stage], C::A_BYTES);
          const int d2 = dim2_rep ? rep : un.group;
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const int c = col0 + t * col1_off;
            tma_load_3d(sA + t * C::ATILE_BYTES, wmap, &sm.full[stage], c, k0, d2, pol_w);
            tma_load_3d(sA + t * C::ATILE_BYTES + C::BOX_BYTES, wmap, &sm.full[stage], c + 64, k0, d2, pol_w);
          }
        }
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == ST) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait_all();
    if (!ok && pt == 0) {
      // Aborted: let every load still in flight land before the block exits.
      for (int s = 0; s < ST; ++s) {
        if (!(issued_mask >> s & 1u)) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sm.full[s], (issued_par >> s) & 1u) && globaltimer_ns() - t0 < timeout_ns) {
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const WaitCtx wc{status, sm.abort_flag, timeout_ns, SITE_GEMM_MMA};
      int stage = 0;
      uint32_t phase = 0;
      int acc_it = 0;
      bool ok = true;
      for (int u = first; u < total && ok; u += stride) {
        const PUnit pu = S.decode(u);
        const Unit& un = pu.un;
        const GemmArgs& a = S.args(pu.phase);
        const int buf = C::NBUF == 2 ? (acc_it & 1) : 0;
        const uint32_t apar = C::NBUF == 2 ? ((acc_it >> 1) & 1) : (acc_it & 1);
        if (!mbar_wait(&sm.tempty[buf], apar ^ 1u, wc, 200 + buf)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + buf * MT * NT;
        const int N = (un.rows + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(128, N, /*A MN-major*/ true, /*B K-major*/ false);
        const int kiters = (un.ke - un.kb) * C::SUB * a.krep;  // read once, before the loop's asm
        uint32_t acc = 0;
        for (int it = 0; it < kiters; ++it) {
          if (!mbar_wait(&sm.full[stage], phase, wc, 300 + stage)) { ok = false; break; }
          tc_fence_after();
          fence_proxy_async_smem();
          const uint32_t sA = smem_u32(sm.ring + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // B (rows, K-major): +16 k = 32 B inside the swizzled row.
            const uint64_t bd = smem_desc(sB + kk * 32, 16, C::ROW_SBO, C::ROW_LAYOUT);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              // A (weights, MN-major): +16 k = two 8-row groups = 2048 B; the two
              // 64-column halves of a tile sit one TMA box apart.
              const uint64_t ad = smem_desc_sw128(sA + t * C::ATILE_BYTES + kk * 2048, C::BOX_BYTES, 1024);
              mma_bf16(d0 + t * NT, ad, bd, idesc, acc);
            }
            acc = 1;
          }
          mma_commit(&sm.empty[stage]);
          if (++stage == ST) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&sm.tfull[buf]);
        ++acc_it;
      }
      // Every MMA issued by this thread has finished once mma_done flips.
      mma_commit(sm.mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(sm.mma_done, 0) && globaltimer_ns() - t0 < timeout_ns) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-7)
    // Warp w reads TMEM lanes 32*(w%4).. (one weight column per thread) and
    // handles the 32-row chunks c0 = 32*(w/4) + 64*j of the unit's rows.
    const WaitCtx wc{status, sm.abort_flag, timeout_ns, SITE_GEMM_EPILOGUE};
    const int quarter = warp & 3, half = warp >> 2;
    int acc_it = 0;
    for (int u = first; u < total; u += stride) {
      const PUnit pu = S.decode(u);
      const int buf = C::NBUF == 2 ? (acc_it & 1) : 0;
      const uint32_t apar = C::NBUF == 2 ? ((acc_it >> 1) & 1) : (acc_it & 1);
      if (!mbar_wait(&sm.tfull[buf], apar, wc, 400 + buf)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * MT * NT;
      if (Sched::kPhases == 1 || pu.phase == 0)
        epilogue_unit<NT, MT, EPI0>(S.args(0), pu.un, tbase, quarter, half, &sm.tempty[buf]);
      else if constexpr (Sched::kPhases > 1)
        epilogue_unit<NT, MT, EPI1>(S.args(1), pu.un, tbase, quarter, half, &sm.tempty[buf]);
      S.after_epilogue(pu);
      ++acc_it;
    }
  }
}

}  // namespace moe
