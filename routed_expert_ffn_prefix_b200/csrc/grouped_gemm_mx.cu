// grouped_gemm_mx.cu -- grouped expert GEMM on block-scaled FP8 weights.
//
// The expert weights are stored in 8 bits: OCP FP8 E4M3 codes, one row of K
// codes per output column (W^T [E, N, K], K contiguous), with one E8M0
// power-of-two scale per 32 consecutive weights along K ([E, K/32, N]).  The
// Qwen 3.5-397B-on-Ironwood page (sec. 6, "numerical validation") runs its
// MoE on FP8 scaling blocks; this kernel keeps the token rows and h in bf16
// and halves the bytes the layer streams, which is what bounds it.
//
// A 4-bit-significand value times a power of two is an exact bf16 value, so
// the kernel decodes every weight into bf16 on chip and runs the same
// tcgen05 kind::f16 MMA, TMEM accumulators and epilogues as the bf16 kernel:
// the products and fp32 sums are those of the bf16 layer on the dequantised
// weights.
//
//   raw ring (R stages): TMA brings the codes of kMxRawSteps k-steps (128
//     columns x 64 * kMxRawSteps codes per MMA tile, one box row per column,
//     swizzled over the row) and their scales (2 * kMxRawSteps rows of 128)
//     -- the bytes in flight from HBM, so this ring is the deep one.  Two
//     k-steps per stage make every box row a whole 128-byte line.
//   decoded stages (CS): one converter thread per weight column decodes its
//     64 codes of the k-step (its two scales in registers) into 32 bf16
//     pairs and writes them as the MMA's A operand: into tensor memory
//     (tcgen05.st; few token rows, where reading A from shared memory would
//     cost the tensor core more than the MMA itself) or into shared memory
//     in the K-major 128-byte-swizzled layout (256-row passes).  The same
//     threads gather the unit's token rows into the B tile (cp.async).
//
// Warp roles (448 threads): warps 0-3 epilogue (one TMEM lane quarter
// each), warps 4-11 converters + row gathers (warp w decodes the columns of
// TMEM lane quarter w % 4 of tile (w - 4) / 4), warp 12 TMA issue, warp 13
// TMEM allocation + MMA issue.  Every wait is bounded.
#include "gemm_pipeline.cuh"

namespace moe {

namespace {

constexpr int kXEpiWarps = 4;
constexpr int kXConvWarps = 8;
constexpr int kXTmaWarp = kXEpiWarps + kXConvWarps;
constexpr int kXMmaWarp = kXTmaWarp + 1;
constexpr int kXThreads = (kXMmaWarp + 1) * 32;
constexpr int kXConvThreads = kXConvWarps * 32;
constexpr int kXEpiThreads = kXEpiWarps * 32;
constexpr int kXMT = 2;                          // MMA tiles per unit (gate + up, or two output blocks)
constexpr int kXRK = kMxRawSteps;                // k-steps per raw stage
constexpr int kXRowBytes = kBK * kXRK;           // one column's codes per raw stage
constexpr int kXCodeBytes = 128 * kXRowBytes;    // one tile's codes per raw stage: 128 columns
constexpr int kXScaleBytes = 128 * (kBK / 32) * kXRK;  // one tile's scales per raw stage: 128 columns
constexpr int kXRawBytes = kXMT * (kXCodeBytes + kXScaleBytes);  // TMA bytes per raw stage
constexpr int kXRawStride = (kXRawBytes + 1023) & ~1023;         // stages keep the swizzle alignment
constexpr int kXATileBytes = 128 * kBK * 2;      // one decoded bf16 tile in shared memory
constexpr int kXATileCols = kBK / 2;             // one decoded tile in TMEM: 32 columns of bf16 pairs
static_assert(kXConvThreads == kXMT * 128, "one converter thread per weight column");
static_assert(kXRK == 1 || kXRK == 2, "box rows of 64 or 128 bytes");

template <int NT, int R, int CS, bool ATM>
struct XCfg {
  static constexpr int A_BYTES = ATM ? 0 : kXMT * kXATileBytes;
  static constexpr int B_BYTES = NT * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NBUF = (2 * kXMT * NT <= (ATM ? 256 : 512)) ? 2 : 1;
  static constexpr int ACC_COLS = NBUF * kXMT * NT;
  static constexpr int A_COL0 = ACC_COLS;  // decoded stages in TMEM after the accumulators
  static constexpr int TMEM_COLS = 512;
  static constexpr int RAW_OFF = CS * STAGE_BYTES;
  static constexpr int BAR_OFF = RAW_OFF + R * kXRawStride;
  static constexpr int PREFIX_OFF = BAR_OFF + 512;
  static constexpr int SMEM_BYTES = PREFIX_OFF + 4 * kPrefixInts + 1024;
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep 1024-byte swizzle alignment");
  static_assert(ACC_COLS + (ATM ? CS * kXMT * kXATileCols : 0) <= TMEM_COLS, "accumulators and A fit in TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(R <= 32 && CS <= 32, "stage masks");
  static_assert(!ATM || CS >= kXRK, "a raw stage's k-steps go to distinct TMEM stages before any is released");
};

// The decode, on the integer and bf16x2 pipes.  An E4M3 byte b becomes the
// bf16 pattern with sign -> bit 15 and its 7 exponent|mantissa bits -> bits
// 4..10, which is exactly e4m3(b) * 2^-120: a normal code lands as exponent
// field e with mantissa m/8, a subnormal one (e = 0) as the bf16 subnormal
// m * 2^-129, zero as zero.  Per pair of codes: one byte permute that
// places each code in a 16-bit half with its sign replicated above it, a
// shift by 4 and a mask (the replicated sign lands on bit 15, the bits
// between are cleared).  One bf16x2 multiply by 2^(scale code - 7) then
// gives e4m3(b) * 2^(scale code - 127), exact wherever the result is a bf16
// number (scale codes 3 and up); below that the product rounds to nearest.
// Scale codes above 134 would need a factor beyond bf16's range: a column
// whose k-step holds one takes two multiplies (2^120, then 2^(code - 127)),
// which round the same way.  Scale code 255 (NaN) gives NaN.
__device__ __forceinline__ uint32_t code_pair(uint32_t w, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(w), "r"(sel));
  return (d << 4) & 0x87F087F0u;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t factor_one(uint32_t code) {  // (2^(code - 7)) x 2, code <= 134; NaN for 255
  return code == 0xFFu ? 0x7FC07FC0u : ((code + 120u) << 7) * 0x00010001u;
}
__device__ __forceinline__ uint32_t factor_full(uint32_t code) {  // (2^(code - 127)) x 2; NaN for 255
  if (code == 0xFFu) return 0x7FC07FC0u;
  return (code ? code << 7 : 0x0040u) * 0x00010001u;
}
constexpr uint32_t kPow120x2 = 0x7B807B80u;  // (2^120) x 2

// 16 codes (four words, k ascending from the low byte) -> 8 bf16 pairs.
template <bool TWO>
__device__ __forceinline__ void decode16(const uint4& c, uint32_t f, uint32_t* out) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t p0 = code_pair(w[i], 0x9180u), p1 = code_pair(w[i], 0xB3A2u);
    if constexpr (TWO) {
      out[2 * i] = bf16x2_mul(bf16x2_mul(p0, kPow120x2), f);
      out[2 * i + 1] = bf16x2_mul(bf16x2_mul(p1, kPow120x2), f);
    } else {
      out[2 * i] = bf16x2_mul(p0, f);
      out[2 * i + 1] = bf16x2_mul(p1, f);
    }
  }
}

// 32 columns of 32-bit cells from registers into TMEM (lane quarter of the
// warp, one lane per thread); tmem_st_wait() waits until this thread's
// stores are written.
__device__ __forceinline__ void tmem_st_32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// One k-step's 64 codes of a column (four 16-byte chunks) and its two
// scales -> 32 bf16 pairs.
__device__ __forceinline__ void decode_step(const uint4* cd, uint32_t s0, uint32_t s1, uint32_t* v) {
  if (__builtin_expect((s0 > 134u && s0 != 0xFFu) || (s1 > 134u && s1 != 0xFFu), 0)) {
    const uint32_t f0 = factor_full(s0), f1 = factor_full(s1);
    decode16<true>(cd[0], f0, v);
    decode16<true>(cd[1], f0, v + 8);
    decode16<true>(cd[2], f1, v + 16);
    decode16<true>(cd[3], f1, v + 24);
  } else {
    const uint32_t f0 = factor_one(s0), f1 = factor_one(s1);
    decode16<false>(cd[0], f0, v);
    decode16<false>(cd[1], f0, v + 8);
    decode16<false>(cd[2], f1, v + 16);
    decode16<false>(cd[3], f1, v + 24);
  }
}

// D(tmem) (+)= A(tmem) x B(smem desc), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_nohint(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                                   int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

template <int NT, int R, int CS, bool ATM, int EPI>
__global__ void __launch_bounds__(kXThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap smap,
                           const GemmArgs a) {
  using C = XCfg<NT, R, CS, ATM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* raw = smem + C::RAW_OFF;
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* raw_empty = raw_full + R;
  uint64_t* ck_full = raw_empty + R;
  uint64_t* ck_empty = ck_full + CS;
  uint64_t* tfull = ck_empty + CS;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* total_units = abort_flag + 1;
  int* ustart = reinterpret_cast<int*>(smem + C::PREFIX_OFF);
  static_assert((2 * R + 2 * CS + 5) * 8 + 16 <= 512, "barrier block");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ngroups = a.offsets ? a.groups : 1;
  if (tid == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(raw_full + s, 1);              // the TMA warp's expect_tx arrival
      mbar_init(raw_empty + s, kXConvWarps);   // one arrival per converter warp
    }
    for (int s = 0; s < CS; ++s) {
      mbar_init(ck_full + s, 2 * kXConvThreads);  // per converter thread: A written, its row copies landed
      mbar_init(ck_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, kXEpiThreads);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kXMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kXTmaWarp && lane == 0) {
    prefetch_tmap(&cmap);
    prefetch_tmap(&smap);
  }
  if (warp == 0) build_unit_prefix<NT>(a, ngroups, ustart, total_units);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = *total_units;
  const int first = blockIdx.x, stride = gridDim.x;

  if (warp == kXTmaWarp) {
    // ------------------------------------------------------------ raw TMA
    if (lane == 0) {
      const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_PRODUCER};
      int r = 0;
      uint32_t ph = 0, issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int u = first; u < total && ok; u += stride) {
        const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
        const int col0 = un.nb * a.col_stride, col1_off = a.col1_off;
        // raw stages p = ks / kXRK for the unit's k-steps [kb, ke); a stage
        // that reaches past K (K % (64 * kXRK) != 0) reads zero fill there
        for (int p = un.kb / kXRK; p <= (un.ke - 1) / kXRK; ++p) {
          if (!mbar_wait(&raw_empty[r], ph ^ 1u, wc, 100 + r)) { ok = false; break; }
          uint8_t* st = raw + r * kXRawStride;
          mbar_arrive_expect_tx(&raw_full[r], kXRawBytes);
#pragma unroll
          for (int t = 0; t < kXMT; ++t) {
            const int c = col0 + t * col1_off;
            tma_load_3d_nohint(st + t * kXCodeBytes, &cmap, &raw_full[r], p * kXRowBytes, c, un.group);
            tma_load_3d_nohint(st + kXMT * kXCodeBytes + t * kXScaleBytes, &smap, &raw_full[r], c,
                               p * kXRK * (kBK / 32), un.group);
          }
          issued_mask |= 1u << r;
          issued_par = (issued_par & ~(1u << r)) | (ph << r);
          if (++r == R) { r = 0; ph ^= 1u; }
        }
      }
      if (!ok) {  // let every copy still in flight land before the block exits
        for (int s = 0; s < R; ++s) {
          if (!(issued_mask >> s & 1u)) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&raw_full[s], (issued_par >> s) & 1u) && globaltimer_ns() - t0 < a.timeout_ns) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= kXEpiWarps && warp < kXTmaWarp) {
    // ------------------------------------------------------------ converters + row gathers
    const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_PRODUCER};
    const int ct = tid - kXEpiThreads;
    const int quarter = warp & 3, t = (warp - kXEpiWarps) >> 2;
    const int n = quarter * 32 + lane;                  // this thread's weight column in tile t
    const int chunk = ct & 7, rsub = ct >> 3;           // row gathers: 16-byte chunk, first row
    constexpr int kRowStep = kXConvThreads / 8;
    constexpr int kRowsPerThread = (NT + kRowStep - 1) / kRowStep;
    // codes of column n: one box row; its 16-byte chunk j sits at j ^ ((n / 2) % 4) (64-byte swizzle)
    // or j ^ (n % 8) (128-byte swizzle)
    const int code_off = t * kXCodeBytes + n * kXRowBytes, sw = kXRK == 1 ? (n >> 1) & 3 : n & 7;
    const int scale_off = kXMT * kXCodeBytes + t * kXScaleBytes + n;
    const uint32_t a_lane = (uint32_t)(quarter * 32) << 16;
    int r = 0, c = 0;
    uint32_t rph = 0, cph = 0;
    bool ok = true;
    for (int u = first; u < total && ok; u += stride) {
      const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
      const uint64_t pol_rows = a.rows_evict_last ? policy_evict_last() : policy_evict_normal();
      const __nv_bfloat16* const bsrc = reinterpret_cast<const __nv_bfloat16*>(a.b_src);
      const int K = a.K;
      int src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int cr = rsub + kRowStep * i;
        int sr = -1;
        if (cr < un.rows) {
          const int rr = un.row0 + cr;
          sr = a.row_index ? a.row_index[rr] : rr;
          if (sr < 0 || sr >= a.src_rows) {
            raise_error(a.status, MOE_ERR_DEVICE_BOUNDS, SITE_GEMM_GATHER, rr);
            sr = -1;
          }
        }
        src[i] = sr;
      }
      // One raw stage (kXRK k-steps) per pass: its codes and scales into
      // registers, then per k-step of the unit: row gathers, decode, A
      // written.  In TMEM the stores are issued back to back and one wait
      // covers the stage's k-steps before their readiness is signalled (a
      // stage's MMAs need only the stages before it, so holding a step back
      // until its neighbour is written cannot stall the ring: CS >= kXRK).
      // In shared memory (two decoded stages) each k-step is released as
      // soon as it is written, so the MMAs of one overlap the decode of the
      // next.
      for (int p = un.kb / kXRK; p <= (un.ke - 1) / kXRK; ++p) {
        if (!mbar_wait(&raw_full[r], rph, wc, 300 + r)) { ok = false; break; }
        const uint8_t* rs = raw + r * kXRawStride;
        uint4 cd[kXRK][4];
        uint32_t s0[kXRK], s1[kXRK];
#pragma unroll
        for (int h = 0; h < kXRK; ++h) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            cd[h][j] = *reinterpret_cast<const uint4*>(rs + code_off + (((4 * h + j) ^ sw) << 4));
          s0[h] = rs[scale_off + 2 * h * 128];  // scales of the k-step's k 0-31 and 32-63
          s1[h] = rs[scale_off + (2 * h + 1) * 128];
        }
        int cs[kXRK];
#pragma unroll
        for (int h = 0; h < kXRK; ++h) {
          const int ks = p * kXRK + h;
          cs[h] = -1;
          if (ks < un.kb || ks >= un.ke) continue;
          if (!mbar_wait(&ck_empty[c], cph ^ 1u, wc, 200 + c)) { ok = false; break; }
          if constexpr (ATM) tc_fence_after();  // the MMAs that read this stage are done
          uint8_t* stg = stages + c * C::STAGE_BYTES;
          const uint32_t sB = smem_u32(stg + C::A_BYTES);
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            if (src[i] >= 0) {
              const int cr = rsub + kRowStep * i;
              cp_async_16(sB + cr * 128 + ((chunk ^ (cr & 7)) << 4),
                          bsrc + (size_t)src[i] * K + ks * kBK + chunk * 8, pol_rows);
            }
          }
          cp_async_arrive_noinc(&ck_full[c]);
          uint32_t v[32];
          decode_step(cd[h], s0[h], s1[h], v);
          if constexpr (ATM) {
            tmem_st_32(tmem + a_lane + C::A_COL0 + (c * kXMT + t) * kXATileCols, v);
          } else {
            // K-major, 128-byte swizzle: row n of 128 bytes, 16-byte chunk j at j ^ (n % 8)
            uint8_t* arow = stg + t * kXATileBytes + n * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(arow + ((j ^ (n & 7)) << 4)) =
                  make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            fence_proxy_async_smem();  // the decoded tile, before the tensor core reads it
            mbar_arrive(&ck_full[c]);
          }
          cs[h] = ATM ? c : -1;
          if (++c == CS) { c = 0; cph ^= 1u; }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[r]);  // every lane of this warp has used its codes
        if (++r == R) { r = 0; rph ^= 1u; }
        if constexpr (ATM) {
          tmem_st_wait();
          tc_fence_before();
#pragma unroll
          for (int h = 0; h < kXRK; ++h)
            if (cs[h] >= 0) mbar_arrive(&ck_full[cs[h]]);
        }
      }
    }
    if constexpr (ATM) tmem_st_wait();  // no store in flight when the block leaves (abort paths)
    cp_async_wait_all();
  } else if (warp == kXMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_MMA};
      int c = 0;
      uint32_t cph = 0;
      int acc_it = 0;
      bool ok = true;
      // Descriptors of stage 0 (K-major, 128-byte swizzle); a stage, a k
      // slice of 16 (32 bytes) and a tile add to the start-address field
      // (address / 16, below 2^14 for any shared-memory address).
      const uint64_t bd0 = smem_desc(smem_u32(stages) + C::A_BYTES, 16, 1024, kLayoutSw128);
      const uint64_t ad0 = smem_desc(smem_u32(stages), 16, 1024, kLayoutSw128);
      const uint32_t at0 = tmem + C::A_COL0;
      for (int u = first; u < total && ok; u += stride) {
        const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
        const int buf = C::NBUF == 2 ? (acc_it & 1) : 0;
        const uint32_t apar = C::NBUF == 2 ? ((acc_it >> 1) & 1) : (acc_it & 1);
        if (!mbar_wait(&tempty[buf], apar ^ 1u, wc, 400 + buf)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + buf * kXMT * NT;
        const int N = (un.rows + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(128, N, /*A K-major*/ false, /*B K-major*/ false);
        uint32_t acc = 0;
        for (int ks = un.kb; ks < un.ke; ++ks) {
          if (!mbar_wait(&ck_full[c], cph, wc, 500 + c)) { ok = false; break; }
          tc_fence_after();
          fence_proxy_async_smem();
          const uint64_t soff = (uint32_t)(c * C::STAGE_BYTES) >> 4;
          const uint64_t bds = bd0 + soff, ads = ad0 + soff;
          const uint32_t ats = at0 + c * (kXMT * kXATileCols);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
            for (int t = 0; t < kXMT; ++t) {
              if constexpr (ATM)
                mma_bf16_ta(d0 + t * NT, ats + t * kXATileCols + kk * 8, bds + 2 * kk, idesc, acc);
              else
                mma_bf16(d0 + t * NT, ads + ((t * kXATileBytes) >> 4) + 2 * kk, bds + 2 * kk, idesc, acc);
            }
            acc = 1;
          }
          mma_commit(&ck_empty[c]);
          if (++c == CS) { c = 0; cph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
        ++acc_it;
      }
      mma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(mma_done, 0) && globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    const WaitCtx wc{a.status, abort_flag, a.timeout_ns, SITE_GEMM_EPILOGUE};
    int acc_it = 0;
    for (int u = first; u < total; u += stride) {
      const Unit un = decode_unit<NT>(a, ustart, ngroups, u);
      const int buf = C::NBUF == 2 ? (acc_it & 1) : 0;
      const uint32_t apar = C::NBUF == 2 ? ((acc_it >> 1) & 1) : (acc_it & 1);
      if (!mbar_wait(&tfull[buf], apar, wc, 600 + buf)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16) + buf * kXMT * NT;
      epilogue_unit<NT, kXMT, EPI, 1>(a, un, tbase, warp, 0, &tempty[buf]);
      ++acc_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kXMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int NT, int R, int CS, bool ATM, int EPI>
cudaError_t launch_x(const CUtensorMap& cmap, const CUtensorMap& smap, const GemmArgs& a, int num_sms,
                     cudaStream_t stream) {
  using C = XCfg<NT, R, CS, ATM>;
  auto kern = grouped_gemm_mx_kernel<NT, R, CS, ATM, EPI>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t err = once_per_device(configured, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3(num_sms), dim3(kXThreads), C::SMEM_BYTES, stream, cmap, smap, a);
}

template <int NT, int R, int CS, bool ATM>
cudaError_t launch_xe(const CUtensorMap& cmap, const CUtensorMap& smap, const GemmArgs& a, int epilogue,
                      int num_sms, cudaStream_t stream) {
  switch (epilogue) {
    case EPI_SWIGLU: return launch_x<NT, R, CS, ATM, EPI_SWIGLU>(cmap, smap, a, num_sms, stream);
    case EPI_SWIGLU_SPLIT: return launch_x<NT, R, CS, ATM, EPI_SWIGLU_SPLIT>(cmap, smap, a, num_sms, stream);
    case EPI_STORE_F32: return launch_x<NT, R, CS, ATM, EPI_STORE_F32>(cmap, smap, a, num_sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_grouped_gemm_mx(const CUtensorMap& code_map, const CUtensorMap& scale_map, const GemmArgs& a,
                                   int epilogue, int tiles, int num_sms, cudaStream_t stream) {
  if (a.krep != 1 || a.col_stride % 128 != 0 || a.col1_off % 128 != 0 || a.K % kBK != 0)
    return cudaErrorInvalidValue;
  // Few rows per expert (decode): 32-row passes with the decoded weights in
  // TMEM, six k-steps of them in flight beside a raw ring of 5 x 2 k-steps.
  // Many rows: 256-row passes with the decoded weights in shared memory.
  static_assert(kXRK == 2, "ring depths below are counted for two k-steps per raw stage");
  if (tiles == MOE_TILES_SMALL) return launch_xe<32, 5, 6, true>(code_map, scale_map, a, epilogue, num_sms, stream);
  return launch_xe<256, 2, 2, false>(code_map, scale_map, a, epilogue, num_sms, stream);
}

}  // namespace moe
