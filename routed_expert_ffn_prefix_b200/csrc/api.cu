// api.cu -- the C ABI declared in include/moe.h: argument checks, workspace
// layout, TMA descriptors and the order of the layer's kernels.
#include <mutex>

#include "kernels.h"

using namespace moe;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded device wait

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Tensor-core router tiling: row tiles of 256 tokens from T >= 2048, else 64;
// the K range (H) is split so that about two work units land on each of the
// 148 SMs.  A function of the shapes only, so the workspace layout and the
// launch always agree.
// MOE_ROUTER_AUTO: a few tokens -> the one-launch split-H router; else tensor
// cores whenever the 16-byte row pitch of the split planes allows it
// (E % 8 == 0), else fp32 CUDA cores.
inline bool valid_scoring(int scoring) {
  return scoring == MOE_SCORE_SOFTMAX || scoring == MOE_SCORE_SOFTMAX_SELECT_BIAS || scoring == MOE_SCORE_SIGMOID;
}

inline int resolve_router(int impl, int T, int E) {
  if (impl != MOE_ROUTER_AUTO) return impl;
  if (T <= kSmallRouterT && E % 4 == 0) return MOE_ROUTER_SMALL;
  return E % 8 == 0 ? MOE_ROUTER_TC : MOE_ROUTER_FMA;
}

inline int router_tiles(int T) { return T >= 2048 ? MOE_TILES_LARGE : MOE_TILES_SMALL; }
inline int router_splits(int T, int H, int E) {
  const int nt = router_tiles(T) == MOE_TILES_LARGE ? 256 : 128;
  const int cols = 128 * gemm_tiles_per_unit(router_tiles(T), EPI_STORE_F32);
  const int base = ((T + nt - 1) / nt) * ((E + cols - 1) / cols);
  int s = (296 + base - 1) / base;
  const int nkt = H / 64;
  if (s > nkt) s = nkt;
  if (s > 32) s = 32;
  return s < 1 ? 1 : s;
}
// Router partial slabs the logits region must hold.
inline int router_slabs(int T, int H, int E) {
  int s = router_splits(T, H, E);
  if (fma_router_splits(T, H) > s) s = fma_router_splits(T, H);
  if (T <= kSmallRouterT) {
    const int ss = small_router_slabs(H, E);
    if (ss > s) s = ss;
  }
  return s;
}

// K splits of the two expert GEMMs (SMALL tiles only).  When even the upper
// bound on work units, min(E, T*k) + T*k/128 row passes times the column
// blocks, leaves SMs idle, each unit's K range is split so that about two
// units land on each of the 148 SMs; every slice keeps >= 4 k-steps of 64.
// A function of the shapes only, like the workspace layout.
struct SplitPlan {
  int gate_up, down;
};
inline int split_for(long long units, int nkt) {
  if (units >= 148) return 1;
  long long s = 296 / units;
  if (s > nkt / 4) s = nkt / 4;
  if (s > 8) s = 8;
  return s < 1 ? 1 : (int)s;
}
inline SplitPlan split_plan(int T, int H, int E, int I, int k, int tiles) {
  if (tiles != MOE_TILES_SMALL || H <= 0 || I <= 0) return {1, 1};
  const long long rows = (long long)T * k;
  const long long passes = (rows < E ? rows : E) + rows / 128;
  return {split_for(passes * (I / 128), H / 64), split_for(passes * (H / 256), I / 64)};
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Arrival counters of the last-arriver epilogues: one per (row, 32-column
// chunk of the gate or up tile) for a K-split gate/up GEMM, one per (token,
// column chunk) for the down GEMM with the combine.  Chunks per down row:
// 8 per 512 output columns (SM pairs), which also covers the single-SM
// kernel's 4 per 256.  A multiple of 64 words, so the region has no
// alignment padding and the routing kernels zero all of it with 16-byte
// stores.
// The persistent few-token layer runs both GEMMs at once, so it takes the
// gate/up counters, the down counters and one done-counter per expert and
// gate/up column block side by side; the multi-kernel path uses the region from its start for each GEMM.
inline int down_cnt_stride(int H) { return ((H + 511) / 512) * 8; }
inline size_t gate_up_cnt_words(int T, int I, int k, const SplitPlan& sp) {
  return sp.gate_up > 1 ? (size_t)T * k * (I / 128) * 4 : 0;
}
inline size_t down_cnt_words(int T, int H) { return (size_t)T * down_cnt_stride(H); }
inline size_t arrival_words(int T, int H, int E, int I, int k) {
  const SplitPlan sp = split_plan(T, H, E, I, k, MOE_TILES_SMALL);
  const size_t w = gate_up_cnt_words(T, I, k, sp) + down_cnt_words(T, H) + (size_t)E * (I / 128);
  return (w + 63) & ~size_t(63);
}
// K-split partial slabs (f32 elements) of the two GEMMs.
inline size_t split_gate_up_elems(int T, int I, int k, const SplitPlan& sp) {
  return sp.gate_up > 1 ? (size_t)sp.gate_up * T * k * 2 * I : 0;
}
inline size_t split_down_elems(int T, int H, int k, const SplitPlan& sp) {
  return sp.down > 1 ? (size_t)sp.down * T * k * H : 0;
}

// ---------------------------------------------------------------- workspace
moe_workspace_layout_t make_layout(int T, int H, int E, int I, int k, int I_s) {
  moe_workspace_layout_t L{};
  const size_t tk = (size_t)T * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.status = take(sizeof(DevStatus));
  L.topk_ids = take(tk * 4);
  L.topk_w = take(tk * 4);
  L.counts = take((size_t)E * 4);
  L.offsets = take((size_t)(E + 1) * 4);
  L.sorted_token_ids = take(tk * 4);
  L.inv_perm = take(tk * 4);
  L.block_hist = take((size_t)permute_num_blocks(T, k) * E * 4);
  L.logits = take((size_t)(H > 0 ? router_slabs(T, H, E) : 1) * T * E * 4);
  L.router_split = take((size_t)3 * H * E * 2);
  L.h = take(tk * I * 2);
  L.o = take(tk * H * 4);
  L.h_shared = take((size_t)T * I_s * 2);
  L.o_shared = take(I_s > 0 ? (size_t)T * H * 4 : 0);
  // Sized for SMALL tiles, the only policy that splits K.
  // gate/up slabs, then down slabs (the persistent few-token layer holds both at once)
  const SplitPlan sp = split_plan(T, H, E, I, k, MOE_TILES_SMALL);
  L.split = take((split_gate_up_elems(T, I, k, sp) + split_down_elems(T, H, k, sp)) * 4);
  L.arrivals = take(arrival_words(T, H, E, I, k) * 4);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- CUDA helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor maps of the weight matrices, [d2][d1][d0] with d0 contiguous:
//   kMapBf16:  bf16, box 64 x 64 x 1, 128-byte swizzle (the bf16 kernels);
//   kMapCodes: u8 FP8 codes [E][N][K], box 64*kMxRawSteps x 128 x 1, swizzled
//              over the box row (64 or 128 bytes);
//   kMapScales: u8 E8M0 scales, box 128 x 2*kMxRawSteps x 1, no swizzle;
//   kMapRows:  bf16 rows [rows][K] (K contiguous), box 64 x 128 x 1, 128-byte swizzle;
//   kMapOutF32: fp32 rows [rows][N] (N contiguous), box 32 x 16 x 1, no swizzle (bulk stores);
//   kMapOutBf16: bf16 rows [rows][N], box 32 x 16 x 1, no swizzle (bulk stores).
// A descriptor depends only on (kind, address, extents), so the last few
// are memoised: a steady stream of calls on the same weights skips the
// encode.
enum MapKind { kMapBf16 = 0, kMapCodes = 1, kMapScales = 2, kMapRows = 3, kMapOutF32 = 4, kMapOutBf16 = 5 };
struct MapCacheEntry {
  const void* base;
  uint64_t d0, d1, d2;
  int kind;
  CUtensorMap map;
};
constexpr int kMapCache = 16;
std::mutex g_map_mutex;
MapCacheEntry g_map_cache[kMapCache];
int g_map_next = 0;

bool encode_map(CUtensorMap* m, int kind, const void* base, uint64_t d0, uint64_t d1, uint64_t d2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const bool out = kind == kMapOutF32 || kind == kMapOutBf16;  // bulk-store boxes of 32 x 16, no swizzle
  const bool bf16 = kind == kMapBf16 || kind == kMapRows || kind == kMapOutBf16;
  const bool f32 = kind == kMapOutF32;
  const uint64_t esz = bf16 ? 2 : f32 ? 4 : 1;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * esz, d0 * d1 * esz};
  cuuint32_t box[3] = {out ? 32u : bf16 ? 64u : kind == kMapScales ? 128u : 64u * kMxRawSteps,
                       out ? 16u : kind == kMapBf16 ? 64u : kind == kMapScales ? 2u * kMxRawSteps : 128u, 1};
  const CUtensorMapSwizzle code_swizzle = kMxRawSteps == 1 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m,
             bf16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
             : f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                   : CU_TENSOR_MAP_DATA_TYPE_UINT8,
             3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             out    ? CU_TENSOR_MAP_SWIZZLE_NONE
             : bf16 ? CU_TENSOR_MAP_SWIZZLE_128B
                    : kind == kMapCodes ? code_swizzle : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, int kind, const void* base, uint64_t d0, uint64_t d1, uint64_t d2) {
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (const MapCacheEntry& e : g_map_cache) {
      if (e.base == base && e.d0 == d0 && e.d1 == d1 && e.d2 == d2 && e.kind == kind) {
        *m = e.map;
        return true;
      }
    }
  }
  if (!encode_map(m, kind, base, d0, d1, d2)) return false;
  std::lock_guard<std::mutex> lock(g_map_mutex);
  g_map_cache[g_map_next] = MapCacheEntry{base, d0, d1, d2, kind, *m};
  g_map_next = (g_map_next + 1) % kMapCache;
  return true;
}

bool make_weight_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2) {
  return make_map(m, kMapBf16, base, d0, d1, d2);
}

// Block-scaled FP8 weights of one expert matrix W [E, K, N]: codes of W^T
// [E, N, K] and their scales [E, K/32, N].
struct MxWeights {
  const uint8_t* codes;
  const uint8_t* scales;
};
bool make_mx_maps(CUtensorMap* cm, CUtensorMap* sm, const MxWeights& w, uint64_t N, uint64_t K, uint64_t E) {
  return make_map(cm, kMapCodes, w.codes, K, N, E) && make_map(sm, kMapScales, w.scales, N, K / 32, E);
}

struct DeviceInfo {
  int num_sms;
};

moe_status_t check_device(DeviceInfo* info) {
  int dev = 0, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_ARCH;
  info->num_sms = sms;
  return MOE_OK;
}

inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                     \
  do {                                    \
    const moe_status_t _s = (expr);       \
    if (_s != MOE_OK) return _s;          \
  } while (0)

// ---------------------------------------------------------------- argument checks
moe_status_t check_shapes(int T, int H, int E, int I, int k, bool need_I) {
  if (T < 1 || H < 1 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > kMaxK) return MOE_ERR_INVALID_ARG;
  if ((long long)T * k >= (1ll << 31)) return MOE_ERR_INVALID_ARG;
  if (H % 256 != 0) return MOE_ERR_ALIGNMENT;
  if (need_I) {
    if (I < 1) return MOE_ERR_INVALID_ARG;
    if (I % 128 != 0) return MOE_ERR_ALIGNMENT;
  }
  return MOE_OK;
}

moe_status_t check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || ws_bytes < need) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

template <typename... P>
bool all_nonnull(P... p) {
  return ((p != nullptr) && ...);
}
template <typename... P>
bool all_aligned(P... p) {
  return (aligned16(p) && ...);
}

inline DevStatus* status_of(void* ws) { return reinterpret_cast<DevStatus*>(ws); }
template <typename Tp>
inline Tp* at(void* ws, size_t off) {
  return reinterpret_cast<Tp*>(static_cast<char*>(ws) + off);
}

int choose_tiles(int policy, long long rows, int groups) {
  if (policy != MOE_TILES_AUTO) return policy;
  // Mean rows per group: small groups stream weights under few rows (128-row
  // passes on single SMs); large ones run on SM pairs, which stage half the
  // gathered rows per SM (measured on the 8192-token prefill shape: gate/up
  // 1.60 vs 1.77 ms, down 1.10 vs 1.16 ms against the 256-row single-SM
  // tiles; slower than single SMs at ~10 rows per expert).
  return rows > 64ll * groups ? MOE_TILES_PAIR : MOE_TILES_SMALL;
}

// ---------------------------------------------------------------- stage launchers (no checks)
// perm: permutation outputs for the one-launch router (nullptr: routing only)
struct PermOut {
  int32_t *counts, *offsets, *sorted_ids, *inv_perm;
};

moe_status_t run_route(const uint16_t* x, const float* w_router, const float* bias, int T, int H, int E, int k,
                       int scoring, int32_t* ids, float* w, int impl, void* ws, const moe_workspace_layout_t& L,
                       const DeviceInfo& dev, cudaStream_t s, const PermOut* perm = nullptr,
                       ZeroSpan zero = ZeroSpan{nullptr, 0}) {
  DevStatus* st = status_of(ws);
  float* logits = at<float>(ws, L.logits);
  impl = resolve_router(impl, T, E);
  if (impl == MOE_ROUTER_SMALL) {
    if (T > kSmallRouterT) return MOE_ERR_INVALID_ARG;
    if (E % 4 != 0) return MOE_ERR_ALIGNMENT;
    return cuda_status(launch_router_small(x, w_router, bias, T, H, E, k, scoring, logits, &st->arrivals, ids, w,
                                           perm ? perm->counts : nullptr, perm ? perm->offsets : nullptr,
                                           perm ? perm->sorted_ids : nullptr, perm ? perm->inv_perm : nullptr, st,
                                           zero, s));
  }
  int nsplit = 1;
  if (impl == MOE_ROUTER_TC) {
    if (E % 8 != 0) return MOE_ERR_ALIGNMENT;
    uint16_t* planes = at<uint16_t>(ws, L.router_split);
    MOE_TRY(cuda_status(launch_router_split(w_router, H, E, planes, s)));
    CUtensorMap map;
    if (!make_weight_map(&map, planes, (uint64_t)E, (uint64_t)H, 3)) return MOE_ERR_CUDA;
    nsplit = router_splits(T, H, E);
    const int cols = 128 * gemm_tiles_per_unit(router_tiles(T), EPI_STORE_F32);
    GemmArgs a{};
    a.offsets = nullptr;
    a.row_index = nullptr;
    a.b_src = x;
    a.src_rows = T;
    a.groups = 1;
    a.single_rows = T;
    a.K = H;
    a.krep = 3;
    a.a_dim2_rep = 1;
    a.n_blocks = (E + cols - 1) / cols;
    a.col_stride = cols;
    a.col1_off = 128;
    a.out = logits;
    a.ld_out = E;
    a.out_col_stride = cols;
    a.out_col1_off = 128;
    a.n_valid = E;
    a.rows_cap = T;
    a.k_splits = nsplit;
    a.split_stride = (size_t)T * E;
    a.status = st;
    a.timeout_ns = kDefaultTimeoutNs;
    MOE_TRY(cuda_status(launch_grouped_gemm(map, a, EPI_STORE_F32, router_tiles(T), dev.num_sms, s)));
  } else {
    MOE_TRY(cuda_status(launch_router_logits_fma(x, w_router, T, H, E, logits, s)));
    nsplit = fma_router_splits(T, H);
  }
  return cuda_status(launch_topk(logits, nsplit, (size_t)T * E, bias, T, E, k, scoring, ids, w, st, zero, s));
}

// Arguments of the gate/up GEMM on single-SM tiles: units of 128
// intermediate columns, the gate and the up tile of the same columns, SwiGLU
// into h [rows, I] bf16.  With nsplit > 1 the units cover K slices and store
// fp32 partial slabs [nsplit][rows][2I] at `partials` (gate columns [0, I),
// up [I, 2I)); arrivals != nullptr (zeroed counters, one per row and
// 32-column chunk) lets the last slab of each row chunk to land sum them and
// write h in its epilogue.
GemmArgs gate_up_args(const uint16_t* x, int src_rows, const int32_t* offsets, const int32_t* row_index, int rows,
                      int H, int E, int I, uint16_t* h, DevStatus* st, int nsplit = 1, float* partials = nullptr,
                      uint32_t* arrivals = nullptr) {
  GemmArgs a{};
  a.offsets = offsets;
  a.row_index = row_index;
  a.b_src = x;
  a.src_rows = src_rows;
  a.groups = E;
  a.single_rows = rows;
  a.K = H;
  a.krep = 1;
  a.a_dim2_rep = 0;
  a.n_blocks = I / 128;
  a.col_stride = 128;
  a.col1_off = I;
  a.out = h;
  a.ld_out = I;
  a.out_col_stride = 128;
  a.out_col1_off = 0;
  a.n_valid = I;
  a.rows_cap = rows;
  a.k_splits = 1;
  a.split_stride = 0;
  a.status = st;
  a.timeout_ns = kDefaultTimeoutNs;
  if (nsplit > 1) {
    a.out = partials;
    a.ld_out = 2 * I;
    a.out_col1_off = I;
    a.n_valid = 2 * I;
    a.k_splits = nsplit;
    a.split_stride = (size_t)rows * 2 * I;
    if (arrivals != nullptr) {
      a.arrivals = arrivals;
      a.cnt_stride = a.n_blocks * 4;
      a.arrive_target = nsplit;
      a.fin_out = h;
      a.fin_ld = I;
    }
  }
  return a;
}

moe_status_t run_swiglu(const uint16_t* x, int src_rows, const uint16_t* w_gate_up, const int32_t* offsets,
                        const int32_t* row_index, int rows, int H, int E, int I, int tiles, uint16_t* h,
                        DevStatus* st, const DeviceInfo& dev, cudaStream_t s, int nsplit = 1,
                        float* partials = nullptr, uint32_t* arrivals = nullptr, const MxWeights* mx = nullptr) {
  if (mx != nullptr) {  // block-scaled FP8 weights: single-SM tiles of the FP8 kernel
    CUtensorMap cm, sm;
    if (!make_mx_maps(&cm, &sm, *mx, 2ull * I, (uint64_t)H, (uint64_t)E)) return MOE_ERR_CUDA;
    const int xt = tiles == MOE_TILES_SMALL ? MOE_TILES_SMALL : MOE_TILES_LARGE;
    const GemmArgs a = gate_up_args(x, src_rows, offsets, row_index, rows, H, E, I, h, st, nsplit, partials, arrivals);
    if (nsplit > 1) {
      if (arrivals != nullptr) return cuda_status(launch_grouped_gemm_mx(cm, sm, a, EPI_SWIGLU_SPLIT, xt, dev.num_sms, s));
      MOE_TRY(cuda_status(launch_grouped_gemm_mx(cm, sm, a, EPI_STORE_F32, xt, dev.num_sms, s)));
      return cuda_status(launch_swiglu_reduce(partials, nsplit, a.split_stride, rows, I, h, s));
    }
    return cuda_status(launch_grouped_gemm_mx(cm, sm, a, EPI_SWIGLU, xt, dev.num_sms, s));
  }
  CUtensorMap map;
  if (!make_weight_map(&map, w_gate_up, 2ull * I, (uint64_t)H, (uint64_t)E)) return MOE_ERR_CUDA;
  if (tiles == MOE_TILES_PAIR) {  // 256 intermediate columns per unit (128 per SM of the pair)
    GemmArgs a = gate_up_args(x, src_rows, offsets, row_index, rows, H, E, I, h, st);
    a.n_blocks = (I + 255) / 256;
    a.col_stride = 256;
    a.out_col_stride = 256;
    // h [rows, I] bf16 leaves by bulk tensor stores (boxes of 16 rows)
    CUtensorMap hmap;
    const bool h_tma = rows >= 16;
    if (h_tma && !make_map(&hmap, kMapOutBf16, h, (uint64_t)I, (uint64_t)rows, 1)) return MOE_ERR_CUDA;
    return cuda_status(launch_grouped_gemm_pair(map, nullptr, h_tma ? &hmap : nullptr, a, EPI_SWIGLU, dev.num_sms, s));
  }
  const GemmArgs a = gate_up_args(x, src_rows, offsets, row_index, rows, H, E, I, h, st, nsplit, partials, arrivals);
  if (nsplit > 1) {
    if (arrivals != nullptr) return cuda_status(launch_grouped_gemm(map, a, EPI_SWIGLU_SPLIT, tiles, dev.num_sms, s));
    MOE_TRY(cuda_status(launch_grouped_gemm(map, a, EPI_STORE_F32, tiles, dev.num_sms, s)));
    return cuda_status(launch_swiglu_reduce(partials, nsplit, a.split_stride, rows, I, h, s));
  }
  return cuda_status(launch_grouped_gemm(map, a, EPI_SWIGLU, tiles, dev.num_sms, s));
}

// The weighted combine taken into the down GEMM's epilogue (see Epilogue).
struct CombineArgs {
  const int32_t* row_token;  // sorted_token_ids
  const int32_t* inv_perm;
  const float* topk_w;
  const float* shared;  // [T, H] f32 or nullptr
  uint16_t* y;
  uint32_t* arrivals;  // zeroed, down_cnt_stride(H) per token
  int T, k;
};

// Arguments of the down GEMM on single-SM tiles: units of 256 output
// columns (two 128-column tiles), fp32 rows o [rows, H]; nsplit > 1: K slices
// into partial slabs [nsplit][rows][H] at o.  comb != nullptr: the last of
// each token's k * nsplit row chunks to land also writes that chunk of y.
GemmArgs down_args(const uint16_t* h, const int32_t* offsets, int rows, int H, int E, int I, float* o, DevStatus* st,
                   int nsplit = 1, const CombineArgs* comb = nullptr) {
  GemmArgs a{};
  a.offsets = offsets;
  a.row_index = nullptr;
  a.b_src = h;
  a.src_rows = rows;
  a.groups = E;
  a.single_rows = rows;
  a.K = I;
  a.krep = 1;
  a.a_dim2_rep = 0;
  a.n_blocks = H / 256;
  a.col_stride = 256;
  a.col1_off = 128;
  a.out = o;
  a.ld_out = H;
  a.out_col_stride = 256;
  a.out_col1_off = 128;
  a.n_valid = H;
  a.rows_cap = rows;
  a.k_splits = nsplit;
  a.split_stride = nsplit > 1 ? (size_t)rows * H : 0;
  a.status = st;
  a.timeout_ns = kDefaultTimeoutNs;
  if (comb != nullptr) {
    a.arrivals = comb->arrivals;
    a.cnt_stride = down_cnt_stride(H);
    a.arrive_target = comb->k * nsplit;
    a.fin_out = comb->y;
    a.fin_ld = H;
    a.row_token = comb->row_token;
    a.inv_perm = comb->inv_perm;
    a.topk_w = comb->topk_w;
    a.shared = comb->shared;
    a.topk = comb->k;
    a.n_tokens = comb->T;
  }
  return a;
}

moe_status_t run_down(const uint16_t* h, const uint16_t* w_down, const int32_t* offsets, int rows, int H, int E,
                      int I, int tiles, float* o, DevStatus* st, const DeviceInfo& dev, cudaStream_t s,
                      int nsplit = 1, const CombineArgs* comb = nullptr, const MxWeights* mx = nullptr) {
  if (mx != nullptr) {  // block-scaled FP8 weights: fp32 rows (the combine kernel follows)
    if (comb != nullptr) return MOE_ERR_INVALID_ARG;
    CUtensorMap cm, sm;
    if (!make_mx_maps(&cm, &sm, *mx, (uint64_t)H, (uint64_t)I, (uint64_t)E)) return MOE_ERR_CUDA;
    const int xt = tiles == MOE_TILES_SMALL ? MOE_TILES_SMALL : MOE_TILES_LARGE;
    const GemmArgs a = down_args(h, offsets, rows, H, E, I, o, st, nsplit);
    return cuda_status(launch_grouped_gemm_mx(cm, sm, a, EPI_STORE_F32, xt, dev.num_sms, s));
  }
  CUtensorMap map;
  if (!make_weight_map(&map, w_down, (uint64_t)H, (uint64_t)I, (uint64_t)E)) return MOE_ERR_CUDA;
  GemmArgs a = down_args(h, offsets, rows, H, E, I, o, st, nsplit, comb);
  const int epi = comb != nullptr ? EPI_DOWN_COMBINE : EPI_STORE_F32;
  if (tiles == MOE_TILES_PAIR) {
    if (nsplit > 1) return MOE_ERR_INVALID_ARG;
    // 2 x 256 output columns per unit (128 of each per SM of the pair); the
    // h rows are contiguous, so with the fp32 store epilogue they come by TMA
    // (boxes of 128 rows, when there are that many)
    a.n_blocks = (H + 511) / 512;
    a.col_stride = 512;
    a.col1_off = 256;
    a.out_col_stride = 512;
    a.out_col1_off = 256;
    CUtensorMap rmap, omap;
    const bool rows_tma = epi == EPI_STORE_F32 && rows >= 128;
    if (rows_tma && (!make_map(&rmap, kMapRows, h, (uint64_t)I, (uint64_t)rows, 1) ||
                     !make_map(&omap, kMapOutF32, o, (uint64_t)H, (uint64_t)rows, 1)))
      return MOE_ERR_CUDA;
    return cuda_status(
        launch_grouped_gemm_pair(map, rows_tma ? &rmap : nullptr, rows_tma ? &omap : nullptr, a, epi, dev.num_sms, s));
  }
  return cuda_status(launch_grouped_gemm(map, a, epi, tiles, dev.num_sms, s));
}

// The layer (moe_forward_ex, moe_forward_mx): bf16 expert weights, or with
// mx_gu/mx_dn block-scaled FP8 ones (w_gate_up/w_down unused then).
moe_status_t forward_impl(const uint16_t* x, const float* w_router, const float* bias, const uint16_t* w_gate_up,
                          const uint16_t* w_down, const MxWeights* mx_gu, const MxWeights* mx_dn,
                          const uint16_t* w_sh_gate_up, const uint16_t* w_sh_down, int I_s, int T, int H, int E,
                          int I, int k, uint16_t* y, void* workspace, size_t workspace_bytes,
                          moe_forward_options_t* options, void* stream) {
  const bool mx = mx_gu != nullptr;
  if (!all_nonnull(x, w_router, y)) return MOE_ERR_INVALID_ARG;
  if (mx ? !(mx_dn && all_nonnull(mx_gu->codes, mx_gu->scales, mx_dn->codes, mx_dn->scales))
         : !all_nonnull(w_gate_up, w_down))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shapes(T, H, E, I, k, true));
  const bool shared = w_sh_gate_up != nullptr || w_sh_down != nullptr || I_s != 0;
  if (shared) {
    if (!all_nonnull(w_sh_gate_up, w_sh_down) || I_s < 1) return MOE_ERR_INVALID_ARG;
    if (I_s % 128 != 0) return MOE_ERR_ALIGNMENT;
    if (!all_aligned(w_sh_gate_up, w_sh_down)) return MOE_ERR_ALIGNMENT;
  }
  const int tile_policy = options ? options->tile_policy : MOE_TILES_AUTO;
  const int router_impl = options ? options->router_impl : MOE_ROUTER_AUTO;
  const int scoring = options ? options->scoring : MOE_SCORE_SOFTMAX;
  const int combine = options ? options->combine : MOE_COMBINE_AUTO;
  if (combine < MOE_COMBINE_AUTO || combine > MOE_COMBINE_SEPARATE) return MOE_ERR_INVALID_ARG;
  if (tile_policy < MOE_TILES_AUTO || tile_policy > MOE_TILES_PERSISTENT) return MOE_ERR_INVALID_ARG;
  if (router_impl < MOE_ROUTER_AUTO || router_impl > MOE_ROUTER_SMALL) return MOE_ERR_INVALID_ARG;
  if (!valid_scoring(scoring)) return MOE_ERR_INVALID_ARG;
  if (mx && (tile_policy == MOE_TILES_PERSISTENT || combine == MOE_COMBINE_FUSED))
    return MOE_ERR_INVALID_ARG;  // the FP8 kernel runs the multi-kernel layer with the combine kernel
  if (!all_aligned(x, w_router, y) || (bias && !aligned16(bias))) return MOE_ERR_ALIGNMENT;
  if (mx ? !all_aligned(mx_gu->codes, mx_gu->scales, mx_dn->codes, mx_dn->scales) : !all_aligned(w_gate_up, w_down))
    return MOE_ERR_ALIGNMENT;
  const moe_workspace_layout_t L = make_layout(T, H, E, I, k, shared ? I_s : 0);
  MOE_TRY(check_ws(workspace, workspace_bytes, L.total));
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  DevStatus* st = status_of(ws);
  int32_t* ids = at<int32_t>(ws, L.topk_ids);
  float* tw = at<float>(ws, L.topk_w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offs = at<int32_t>(ws, L.offsets);
  int32_t* sids = at<int32_t>(ws, L.sorted_token_ids);
  int32_t* inv = at<int32_t>(ws, L.inv_perm);
  uint16_t* h = at<uint16_t>(ws, L.h);
  float* o = at<float>(ws, L.o);
  const int rows = T * k;

  void* const* ev = options ? options->stage_events : nullptr;
  auto mark = [&](int i) -> moe_status_t {
    if (ev && ev[i]) return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s));
    return MOE_OK;
  };
  int launches = 0;

  // A few tokens, on request: the whole layer in one persistent launch on the tensor cores.
  if (tile_policy == MOE_TILES_PERSISTENT) {
    if (!layer_small_supported(T, E, shared ? I_s : 0)) return MOE_ERR_INVALID_ARG;
    if (router_impl != MOE_ROUTER_AUTO && router_impl != MOE_ROUTER_SMALL) return MOE_ERR_INVALID_ARG;
    const SplitPlan sp = split_plan(T, H, E, I, k, MOE_TILES_SMALL);
    CUtensorMap gmap, dmap;
    if (!make_weight_map(&gmap, w_gate_up, 2ull * I, (uint64_t)H, (uint64_t)E) ||
        !make_weight_map(&dmap, w_down, (uint64_t)H, (uint64_t)I, (uint64_t)E))
      return MOE_ERR_CUDA;
    uint32_t* arr = at<uint32_t>(ws, L.arrivals);
    const size_t gu_cnt = gate_up_cnt_words(T, I, k, sp), dn_cnt = down_cnt_words(T, H);
    float* gu_slabs = at<float>(ws, L.split);
    float* dn_slabs = gu_slabs + split_gate_up_elems(T, I, k, sp);
    LayerParams p{};
    p.x = x;
    p.w_router = w_router;
    p.bias = bias;
    p.scoring = scoring;
    p.T = T;
    p.H = H;
    p.E = E;
    p.k = k;
    p.partial = at<float>(ws, L.logits);
    p.ids = ids;
    p.counts = counts;
    p.offsets = offs;
    p.sids = sids;
    p.inv = inv;
    p.tw = tw;
    p.expert_done = arr + gu_cnt + dn_cnt;
    p.zero = ZeroSpan{reinterpret_cast<uint4*>(arr), (int)(arrival_words(T, H, E, I, k) / 4)};
    p.gu = gate_up_args(x, T, offs, sids, rows, H, E, I, h, st, sp.gate_up, gu_slabs, arr);
    const CombineArgs comb{sids, inv, tw, nullptr, y, arr + gu_cnt, T, k};
    p.dn = down_args(h, offs, rows, H, E, I, sp.down > 1 ? dn_slabs : o, st, sp.down, &comb);
    p.st = st;
    p.timeout_ns = kDefaultTimeoutNs;
    MOE_TRY(mark(0));
    MOE_TRY(cuda_status(launch_layer_small(gmap, dmap, p, dev.num_sms, s)));
    for (int i = 1; i < 7; ++i) MOE_TRY(mark(i));
    if (options) options->launches = 1;
    return MOE_OK;
  }

  const int ri = resolve_router(router_impl, T, E);
  int tiles = choose_tiles(tile_policy, rows, E);
  if (mx) {
    // The FP8 kernel runs on single SMs; its small tiles are 32-row passes,
    // which AUTO takes while the mean expert holds at most 24 rows.
    if (tile_policy == MOE_TILES_AUTO) tiles = rows <= 24ll * E ? MOE_TILES_SMALL : MOE_TILES_LARGE;
    if (tiles == MOE_TILES_PAIR) tiles = MOE_TILES_LARGE;
  }
  const SplitPlan sp = split_plan(T, H, E, I, k, tiles);
  // Last-arriver epilogues: the K-split gate/up GEMM sums its slabs in its
  // epilogue unless SEPARATE is asked for; the down GEMM combines in its
  // epilogue only on request (FUSED), because a separate combine kernel
  // measured faster at every size (see the combine options in moe.h).
  const bool fuse_swiglu = combine != MOE_COMBINE_SEPARATE && sp.gate_up > 1;
  const bool fuse_combine = combine == MOE_COMBINE_FUSED;
  uint32_t* arrivals = at<uint32_t>(ws, L.arrivals);
  // the routing kernel zeroes the arrival counters of the fused epilogues
  const bool need_zero = fuse_swiglu || fuse_combine;
  const ZeroSpan zero{need_zero ? reinterpret_cast<uint4*>(arrivals) : nullptr,
                      need_zero ? (int)(arrival_words(T, H, E, I, k) / 4) : 0};
  MOE_TRY(mark(0));
  if (ri == MOE_ROUTER_SMALL) {
    const PermOut perm{counts, offs, sids, inv};
    MOE_TRY(run_route(x, w_router, bias, T, H, E, k, scoring, ids, tw, ri, ws, L, dev, s, &perm, zero));
    launches += 1;
    MOE_TRY(mark(1));
  } else {
    MOE_TRY(run_route(x, w_router, bias, T, H, E, k, scoring, ids, tw, ri, ws, L, dev, s, nullptr, zero));
    launches += ri == MOE_ROUTER_TC ? 3 : 2;
    MOE_TRY(mark(1));
    MOE_TRY(cuda_status(
        launch_permute(ids, T, E, k, counts, offs, sids, inv, at<int32_t>(ws, L.block_hist), st, s)));
    launches += rows <= 8192 ? 1 : 3;
  }
  MOE_TRY(mark(2));
  float* split = at<float>(ws, L.split);
  float* o_sh = nullptr;
  if (shared) {
    uint16_t* h_sh = at<uint16_t>(ws, L.h_shared);
    o_sh = at<float>(ws, L.o_shared);
    const int sh_tiles = choose_tiles(tile_policy, T, 1);
    MOE_TRY(run_swiglu(x, T, w_sh_gate_up, nullptr, nullptr, T, H, 1, I_s, sh_tiles, h_sh, st, dev, s));
    MOE_TRY(run_down(h_sh, w_sh_down, nullptr, T, H, 1, I_s, sh_tiles, o_sh, st, dev, s));
    launches += 2;
  }
  MOE_TRY(mark(3));
  MOE_TRY(run_swiglu(x, T, w_gate_up, offs, sids, rows, H, E, I, tiles, h, st, dev, s, sp.gate_up, split,
                     fuse_swiglu ? arrivals : nullptr, mx_gu));
  launches += (sp.gate_up > 1 && !fuse_swiglu) ? 2 : 1;
  MOE_TRY(mark(4));
  float* od = sp.down > 1 ? split : o;
  if (fuse_combine) {
    const CombineArgs comb{sids, inv, tw, o_sh, y, arrivals, T, k};
    MOE_TRY(run_down(h, w_down, offs, rows, H, E, I, tiles, od, st, dev, s, sp.down, &comb));
    launches += 1;
    MOE_TRY(mark(5));
  } else {
    MOE_TRY(run_down(h, w_down, offs, rows, H, E, I, tiles, od, st, dev, s, sp.down, nullptr, mx_dn));
    MOE_TRY(mark(5));
    MOE_TRY(cuda_status(launch_combine(od, tw, inv, o_sh, T, H, k, rows, sp.down, (size_t)rows * H, y, st, s)));
    launches += 2;  // down GEMM, combine
  }
  MOE_TRY(mark(6));
  if (options) options->launches = launches;
  return MOE_OK;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null pointer or unsupported shape";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT: pointer or dimension not aligned as required";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
    case MOE_ERR_UNSUPPORTED_ARCH: return "MOE_ERR_UNSUPPORTED_ARCH: device is not sm_100";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS: routing metadata out of range on the device";
    default: return "unknown moe status";
  }
}

int moe_abi_version(void) { return 2; }

moe_status_t moe_workspace_layout(int T, int H, int E, int I, int k, int I_s, moe_workspace_layout_t* out) {
  if (out == nullptr || I_s < 0) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shapes(T, H, E, I, k, true));
  if (I_s > 0 && I_s % 128 != 0) return MOE_ERR_ALIGNMENT;
  *out = make_layout(T, H, E, I, k, I_s);
  return MOE_OK;
}

moe_status_t moe_workspace_size(int T, int H, int E, int I, int k, int I_s, size_t* bytes) {
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  moe_workspace_layout_t L;
  MOE_TRY(moe_workspace_layout(T, H, E, I, k, I_s, &L));
  *bytes = L.total;
  return MOE_OK;
}

moe_status_t moe_get_device_status(const void* workspace, void* stream, int32_t* out) {
  if (workspace == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DevStatus h{};
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  *out = h.code;
  return MOE_OK;
}

moe_status_t moe_clear_device_status(void* workspace, void* stream) {
  if (workspace == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, sizeof(DevStatus), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_route_scored(const uint16_t* x, const float* w_router, const float* bias, int T, int H, int E,
                              int k, int scoring, int32_t* topk_ids, float* topk_w, int router_impl, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!all_nonnull(x, w_router, topk_ids, topk_w)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shapes(T, H, E, 0, k, false));
  if (router_impl < MOE_ROUTER_AUTO || router_impl > MOE_ROUTER_SMALL) return MOE_ERR_INVALID_ARG;
  if (!valid_scoring(scoring)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned(x, w_router, topk_ids, topk_w) || (bias && !aligned16(bias))) return MOE_ERR_ALIGNMENT;
  const moe_workspace_layout_t L = make_layout(T, H, E, 0, k, 0);
  MOE_TRY(check_ws(workspace, workspace_bytes, L.h));
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  return run_route(x, w_router, bias, T, H, E, k, scoring, topk_ids, topk_w, router_impl, workspace, L, dev,
                   static_cast<cudaStream_t>(stream));
}

moe_status_t moe_route_ex(const uint16_t* x, const float* w_router, const float* bias, int T, int H, int E, int k,
                          int32_t* topk_ids, float* topk_w, int router_impl, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return moe_route_scored(x, w_router, bias, T, H, E, k, MOE_SCORE_SOFTMAX, topk_ids, topk_w, router_impl, workspace,
                          workspace_bytes, stream);
}

moe_status_t moe_route(const uint16_t* x, const float* w_router, const float* bias, int T, int H, int E, int k,
                       int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes, void* stream) {
  return moe_route_ex(x, w_router, bias, T, H, E, k, topk_ids, topk_w, MOE_ROUTER_AUTO, workspace,
                      workspace_bytes, stream);
}

moe_status_t moe_permute(const int32_t* topk_ids, int T, int E, int k, int32_t* counts, int32_t* offsets,
                         int32_t* sorted_token_ids, int32_t* inv_perm, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (!all_nonnull(topk_ids, counts, offsets, sorted_token_ids, inv_perm)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shapes(T, 256, E, 0, k, false));
  if (!all_aligned(topk_ids, counts, offsets, sorted_token_ids, inv_perm)) return MOE_ERR_ALIGNMENT;
  const moe_workspace_layout_t L = make_layout(T, 0, E, 0, k, 0);
  MOE_TRY(check_ws(workspace, workspace_bytes, L.logits));
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  return cuda_status(launch_permute(topk_ids, T, E, k, counts, offsets, sorted_token_ids, inv_perm,
                                    at<int32_t>(workspace, L.block_hist), status_of(workspace),
                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_swiglu(const uint16_t* x, const uint16_t* w_gate_up, const int32_t* offsets,
                                const int32_t* sorted_token_ids, int T, int H, int E, int I, int k,
                                int tile_policy, uint16_t* h, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (!all_nonnull(x, w_gate_up, offsets, sorted_token_ids, h)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shapes(T, H, E, I, k, true));
  if (tile_policy < MOE_TILES_AUTO || tile_policy > MOE_TILES_PAIR) return MOE_ERR_INVALID_ARG;
  if (!all_aligned(x, w_gate_up, offsets, sorted_token_ids, h)) return MOE_ERR_ALIGNMENT;
  MOE_TRY(check_ws(workspace, workspace_bytes, sizeof(DevStatus)));
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  const int rows = T * k;
  return run_swiglu(x, T, w_gate_up, offsets, sorted_token_ids, rows, H, E, I,
                    choose_tiles(tile_policy, rows, E), h, status_of(workspace), dev,
                    static_cast<cudaStream_t>(stream));
}

moe_status_t moe_grouped_down(const uint16_t* h, const uint16_t* w_down, const int32_t* offsets, int rows, int H,
                              int E, int I, int tile_policy, float* o, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (!all_nonnull(h, w_down, o)) return MOE_ERR_INVALID_ARG;
  if (rows < 1 || E < 1 || E > kMaxExperts || H < 1 || I < 1) return MOE_ERR_INVALID_ARG;
  if (offsets == nullptr && E != 1) return MOE_ERR_INVALID_ARG;
  if (H % 256 != 0 || I % 128 != 0) return MOE_ERR_ALIGNMENT;
  if (tile_policy < MOE_TILES_AUTO || tile_policy > MOE_TILES_PAIR) return MOE_ERR_INVALID_ARG;
  if (!all_aligned(h, w_down, o) || (offsets && !aligned16(offsets))) return MOE_ERR_ALIGNMENT;
  MOE_TRY(check_ws(workspace, workspace_bytes, sizeof(DevStatus)));
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  return run_down(h, w_down, offsets, rows, H, E, I, choose_tiles(tile_policy, rows, E), o, status_of(workspace),
                  dev, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_down_combine(const uint16_t* h, const uint16_t* w_down, const float* topk_w,
                              const int32_t* inv_perm, const int32_t* offsets, const float* shared_out, int T,
                              int H, int E, int I, int k, int tile_policy, uint16_t* y, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!all_nonnull(h, w_down, topk_w, inv_perm, offsets, y)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shapes(T, H, E, I, k, true));
  if (tile_policy < MOE_TILES_AUTO || tile_policy > MOE_TILES_PAIR) return MOE_ERR_INVALID_ARG;
  if (!all_aligned(h, w_down, topk_w, inv_perm, offsets, y) || (shared_out && !aligned16(shared_out)))
    return MOE_ERR_ALIGNMENT;
  const moe_workspace_layout_t L = make_layout(T, H, E, I, k, 0);
  MOE_TRY(check_ws(workspace, workspace_bytes, L.total));
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = T * k;
  float* o = at<float>(workspace, L.o);
  DevStatus* st = status_of(workspace);
  // The combine runs in the down GEMM's epilogue; its token row of each
  // permuted row is not an argument here, so it is derived from inv_perm
  // into the workspace's sorted_token_ids region, and the arrival counters
  // are zeroed, in one small kernel.
  int32_t* sids = at<int32_t>(workspace, L.sorted_token_ids);
  uint32_t* arrivals = at<uint32_t>(workspace, L.arrivals);
  MOE_TRY(cuda_status(launch_row_tokens(inv_perm, T, k, sids,
                                        ZeroSpan{reinterpret_cast<uint4*>(arrivals),
                                                 (int)(arrival_words(T, H, E, I, k) / 4)},
                                        st, s)));
  const CombineArgs comb{sids, inv_perm, topk_w, shared_out, y, arrivals, T, k};
  return run_down(h, w_down, offsets, rows, H, E, I, choose_tiles(tile_policy, rows, E), o, st, dev, s, 1, &comb);
}

moe_status_t moe_forward_ex(const uint16_t* x, const float* w_router, const float* bias, const uint16_t* w_gate_up,
                            const uint16_t* w_down, const uint16_t* w_sh_gate_up, const uint16_t* w_sh_down, int I_s,
                            int T, int H, int E, int I, int k, uint16_t* y, void* workspace,
                            size_t workspace_bytes, moe_forward_options_t* options, void* stream) {
  return forward_impl(x, w_router, bias, w_gate_up, w_down, nullptr, nullptr, w_sh_gate_up, w_sh_down, I_s, T, H, E,
                      I, k, y, workspace, workspace_bytes, options, stream);
}

moe_status_t moe_forward_mx(const uint16_t* x, const float* w_router, const float* bias,
                            const uint8_t* w_gate_up_codes, const uint8_t* w_gate_up_scales,
                            const uint8_t* w_down_codes, const uint8_t* w_down_scales,
                            const uint16_t* w_sh_gate_up, const uint16_t* w_sh_down, int I_s, int T, int H, int E,
                            int I, int k, uint16_t* y, void* workspace, size_t workspace_bytes,
                            moe_forward_options_t* options, void* stream) {
  const MxWeights gu{w_gate_up_codes, w_gate_up_scales}, dn{w_down_codes, w_down_scales};
  return forward_impl(x, w_router, bias, nullptr, nullptr, &gu, &dn, w_sh_gate_up, w_sh_down, I_s, T, H, E, I, k, y,
                      workspace, workspace_bytes, options, stream);
}

moe_status_t moe_forward(const uint16_t* x, const float* w_router, const float* bias, const uint16_t* w_gate_up,
                         const uint16_t* w_down, const uint16_t* w_sh_gate_up, const uint16_t* w_sh_down, int I_s,
                         int T, int H, int E, int I, int k, uint16_t* y, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return moe_forward_ex(x, w_router, bias, w_gate_up, w_down, w_sh_gate_up, w_sh_down, I_s, T, H, E, I, k, y,
                        workspace, workspace_bytes, nullptr, stream);
}

moe_status_t moe_selftest_timeout(void* workspace, size_t workspace_bytes, uint64_t timeout_ns, void* stream) {
  MOE_TRY(check_ws(workspace, workspace_bytes, sizeof(DevStatus)));
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  DeviceInfo dev;
  MOE_TRY(check_device(&dev));
  return cuda_status(launch_selftest_timeout(status_of(workspace), timeout_ns, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
