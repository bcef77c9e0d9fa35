/*
 * moe.h -- C ABI of the B200 (sm_100a) routed-expert MoE FFN layer.
 *
 * The layer (one GPU, all experts resident):
 *
 *   route    l = x . W_router (+ bias), fp32; p = softmax(l) over E experts;
 *            the k largest p per token (descending, ties to the lower id);
 *            w_j = p_j / sum of the k selected p.  (Two further scoring
 *            rules, in which the bias steers only the selection:
 *            MOE_SCORE_* below.)
 *   permute  slots (t, j) sorted into expert-contiguous order, experts
 *            ascending, tokens ascending within an expert.
 *   gate/up  per permuted row r (token t, expert e):
 *            [g | u] = x[t] . W_gate_up[e];  h[r] = bf16(silu(g) * u).
 *   down     o[r] = h[r] . W_down[e]  (fp32).
 *   combine  y[t] = bf16( sum_{j=0..k-1} w[t,j] * o[inv_perm[t,j]]  (j ascending,
 *            fp32)  + s[t] ),  s = shared-expert FFN of x[t] when present.
 *
 * Passages defining the steps (page title, section):
 *   - Qwen 3.5-397B MoE on Ironwood (TPU v7x), sec. 4.2 "MoE track":
 *     top_k = 10 routing, SparseCore ragged gather of token rows straight
 *     from HBM (no padded permuted tensor), grouped GEMM V2 with SwiGLU
 *     fused into the main matmul loop, minimal per-expert padding.
 *   - same page, sec. 7.2 "chunked pipeline": un-permute and
 *     gather-reduce of the [T*k, H] expert outputs back to token order.
 *   - same page, sec. 8.2: router gating projection fused with top-k.
 *   - Ling-2.6-1T on TPU v7x with SGLang-JAX, "Fused MoE V2" paragraph:
 *     scatter + expert FFN + gather as one fused unit; top-8 routing plus
 *     a shared expert.
 *   - the benchmark workload definitions: softmax over router logits,
 *     then top-k, then renormalise.
 *
 * Conventions for every call:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, row
 *     major, densely packed.  bf16 tensors are passed as uint16_t bit
 *     patterns.  The library never allocates, frees or keeps a pointer
 *     past the call; work is enqueued on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and the call returns without waiting.
 *   - Process-wide state: the library keeps two host-side caches, both pure
 *     functions of their keys and guarded by a mutex, so every call stays
 *     re-entrant: kernel attributes and cluster occupancy per device, and
 *     the last 16 TMA tensor descriptors keyed by (weight address,
 *     extents).  A cached descriptor is rebuilt whenever the key differs;
 *     it holds an address value but the library never dereferences it
 *     outside a call that passes the same pointer again.
 *   - Shapes: T >= 1 tokens, H % 256 == 0, I % 128 == 0 (I_s likewise),
 *     1 <= k <= min(E, 64), E <= 1024, T*k < 2^31.
 *   - Alignment: every pointer 16-byte aligned (workspace 256-byte).
 *   - Workspace: caller-allocated device memory of at least
 *     moe_workspace_size() bytes for the layer's shapes; every call takes
 *     the same workspace (each stage uses its own region of it).  Calls
 *     that share a workspace must be stream-ordered.  Its status block
 *     (offset 0) must be cleared once, with moe_clear_device_status(),
 *     before the workspace is first used.
 *   - Errors in the arguments are found on the host before anything is
 *     enqueued: the call returns the status and launches nothing.
 *     Errors found on the device (a bounds check on routing metadata, a
 *     bounded wait that ran out) are written to a status word in the
 *     workspace, read with moe_get_device_status(); the kernel that finds
 *     one skips the rest of its work and exits.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,      /* null pointer, bad shape, k > E, ... */
  MOE_ERR_ALIGNMENT = 2,        /* pointer or shape not aligned as required */
  MOE_ERR_WORKSPACE = 3,        /* workspace missing or too small */
  MOE_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5,   /* a bounded device-side wait ran out */
  MOE_ERR_UNSUPPORTED_ARCH = 6, /* current device is not sm_100 */
  MOE_ERR_DEVICE_BOUNDS = 7     /* device found routing metadata out of range */
} moe_status_t;

/* Tile policy of the grouped expert GEMMs (moe_forward_ex / grouped calls). */
enum {
  MOE_TILES_AUTO = 0,   /* chosen from the mean rows per expert, T*k/E: SMALL up to 64, else PAIR */
  MOE_TILES_SMALL = 1,  /* <= 128 token rows per tile pass, 4-stage ring: decode */
  MOE_TILES_LARGE = 2,  /* <= 256 token rows per tile pass, 3-stage ring: prefill */
  MOE_TILES_PAIR = 3,   /* SM pairs (2-SM tcgen05 MMA): 256 weight columns per MMA, 128 per SM; <= 256
                           token rows per pass, half gathered by each SM; 4-stage ring: prefill */
  MOE_TILES_PERSISTENT = 4 /* moe_forward_ex only, T <= 16, E % 4 == 0, no shared expert: the whole
                              layer in one persistent launch on the tensor cores -- the few-token
                              router, then the gate/up and the down grouped GEMM as one sequence of
                              work units (a down unit starts once its expert's gate/up units are
                              done), the weighted combine in the down GEMM's epilogue */
};

/* Router logits implementation. */
enum {
  MOE_ROUTER_AUTO = 0,
  MOE_ROUTER_FMA = 1,   /* fp32 CUDA-core dot products */
  MOE_ROUTER_TC = 2,    /* fp32 W split into three bf16 terms, tcgen05 MMA, fp32 accumulate */
  MOE_ROUTER_SMALL = 3  /* T <= 16, E % 4 == 0: fp32 CUDA-core dot products with H split over
                           ~148 blocks; the last block sums the partials, selects the top-k and
                           (in moe_forward) builds the permutation -- one launch */
};
/* MOE_ROUTER_AUTO picks SMALL when T <= 16 and E % 4 == 0, else TC when
 * E % 8 == 0, else FMA. */

/* Where the weighted combine runs (moe_forward_ex options).  Both give
 * bitwise the same y: the k expert rows of a token (each first summed over
 * its K slabs, slab order) are summed in slot order j = 0..k-1 in fp32, the
 * shared-expert row is added last, and y is rounded to bf16 once.
 *   FUSED:    in the down GEMM's epilogue.  Each epilogue warp counts the
 *             rows it stored on a per-(token, 64-column chunk) counter in
 *             the workspace; the warp whose store completes a token's chunk
 *             (the last of its k rows, times the K slabs) sums the chunk and
 *             writes it to y.  No warp waits for another.  A K-split
 *             gate/up GEMM likewise sums its slabs and applies SwiGLU in the
 *             epilogue of the last slab to land.  No combine launch.
 *   SEPARATE: the down GEMM writes fp32 rows; a combine kernel (and, for a
 *             K-split gate/up GEMM, a slab-sum + SwiGLU kernel) follows. */
enum {
  MOE_COMBINE_AUTO = 0,  /* the K-split gate/up's slab sum + SwiGLU in its epilogue, the combine in its own
                            kernel: the fused combine measured slower at every size (its finishing warps
                            gather a token's k rows one token at a time, while a separate kernel has
                            every SM's warps loading at once) */
  MOE_COMBINE_FUSED = 1,
  MOE_COMBINE_SEPARATE = 2
};

/* Router scoring: how the k experts of a token are selected and weighted
 * from its fp32 logits l[e] and the optional per-expert bias b[e].  The
 * systems-engineering handbook page on Qwen 3.5-397B MoE on Ironwood
 * ("key optimisations", step 1 "expert load balancing") names hot experts
 * and a balancing term in the router, and the Ling page a per-expert
 * router bias, neither with a formula; SOFTMAX is the rule of
 * the layer's workloads, the other two are the common forms in which the
 * bias steers only the selection.  In every form the k selected are listed
 * by descending key, ties to the lower expert id. */
enum {
  MOE_SCORE_SOFTMAX = 0,             /* key = l + b; w_j = softmax over the selected keys */
  MOE_SCORE_SOFTMAX_SELECT_BIAS = 1, /* key = l + b; w_j = softmax over the selected unbiased l */
  MOE_SCORE_SIGMOID = 2              /* s = sigmoid(l); key = s + b; w_j = s_j / sum of the selected s */
};

/* Human-readable name of a status code (static storage). */
const char *moe_status_string(int status);

/* ABI version of this header (incremented on incompatible changes). */
int moe_abi_version(void);

/* Byte offsets of the intermediates inside the workspace (for inspection
 * after moe_forward; all 256-byte aligned).  Regions:
 *   topk_ids [T,k] i32, topk_w [T,k] f32, counts [E] i32, offsets [E+1] i32,
 *   sorted_token_ids [T*k] i32, inv_perm [T,k] i32, h [T*k, I] bf16,
 *   o [T*k, H] f32 (expert outputs, permuted order), h_shared [T, I_s] bf16,
 *   o_shared [T, H] f32,
 *   logits [S, T, E] f32 (S router partial slabs), router_split [3, H, E]
 *   bf16, block_hist (permute), split: K-split partial slabs of the expert
 *   GEMMs when few tokens leave SMs idle (f32; 0 bytes when unused),
 *   arrivals: u32 counters of the combine in the down GEMM's epilogue (one
 *   per token and 64 output columns) and of a K-split gate/up GEMM's
 *   SwiGLU (one per row and 32 intermediate columns).  Each layer call
 *   zeroes them in its routing kernel and leaves them zero. */
typedef struct moe_workspace_layout {
  size_t status, topk_ids, topk_w, counts, offsets, sorted_token_ids, inv_perm;
  size_t h, o, h_shared, o_shared, logits, router_split, block_hist, split;
  size_t arrivals;
  size_t total;
} moe_workspace_layout_t;

moe_status_t moe_workspace_layout(int T, int H, int E, int I, int k, int I_s,
                                  moe_workspace_layout_t *out);

/* Workspace bytes needed for the layer shapes (I_s = 0: no shared expert). */
moe_status_t moe_workspace_size(int T, int H, int E, int I, int k, int I_s, size_t *bytes);

/* Reads the device status word of `workspace` (synchronises `stream`).
 * *out receives MOE_OK or the first error a kernel recorded. */
moe_status_t moe_get_device_status(const void *workspace, void *stream, int32_t *out);

/* Resets the workspace status block (stream-ordered): the status word to
 * MOE_OK and the counters the few-token router and the one-launch layer keep
 * beside it (each returns its counter to zero when it finishes; after a
 * device timeout, clear the block before the next call). */
moe_status_t moe_clear_device_status(void *workspace, void *stream);

/* Route: topk_ids [T,k] i32 and topk_w [T,k] f32 from x [T,H] bf16,
 * W_router [H,E] f32 and an optional per-expert logit bias [E] f32 (NULL
 * for none; added before softmax).  Logits are fp32; ids follow descending
 * logit with ties to the lower expert id. */
moe_status_t moe_route(const uint16_t *x, const float *w_router, const float *bias,
                       int T, int H, int E, int k,
                       int32_t *topk_ids, float *topk_w,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Same, with the logits implementation chosen explicitly (MOE_ROUTER_*). */
moe_status_t moe_route_ex(const uint16_t *x, const float *w_router, const float *bias,
                          int T, int H, int E, int k,
                          int32_t *topk_ids, float *topk_w, int router_impl,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Same, under a scoring rule (MOE_SCORE_*; moe_route_ex is MOE_SCORE_SOFTMAX).
 * bias may be NULL under every rule.  An unknown rule returns
 * MOE_ERR_INVALID_ARG. */
moe_status_t moe_route_scored(const uint16_t *x, const float *w_router, const float *bias,
                              int T, int H, int E, int k, int scoring,
                              int32_t *topk_ids, float *topk_w, int router_impl,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Permute: counts [E], offsets [E+1] (exclusive prefix sum, offsets[E] =
 * T*k), sorted_token_ids [T*k] (permuted row -> token) and inv_perm [T,k]
 * (slot -> permuted row) from topk_ids [T,k].  Deterministic: experts
 * ascending, tokens ascending within an expert.  An id outside [0,E) sets
 * MOE_ERR_DEVICE_BOUNDS in the device status word. */
moe_status_t moe_permute(const int32_t *topk_ids, int T, int E, int k,
                         int32_t *counts, int32_t *offsets,
                         int32_t *sorted_token_ids, int32_t *inv_perm,
                         void *workspace, size_t workspace_bytes, void *stream);

/* moe_permute without a workspace.  The source pages have no counterpart to
 * this call; it exists for callers that cannot allocate device memory when
 * they call -- a serving loop that reserves all memory at start-up and
 * forbids allocation afterwards, a plugin inside a framework that owns every
 * device allocation, or code that must avoid the device-wide
 * synchronisation cudaMalloc/cudaFree can cause.  The outputs are identical
 * to moe_permute's.  The kernels' scratch lives in a 512 KiB array built
 * into the library, which every GPU that loads the library holds until the
 * process exits; the call itself allocates and frees nothing.
 * Limits: T*k <= 131072 (larger batches return MOE_ERR_WORKSPACE and enqueue
 * nothing); E <= 1024 and k <= min(E, 64) as for every call (else
 * MOE_ERR_INVALID_ARG).
 * The first call from each device's context looks up the array's device
 * address (cudaGetSymbolAddress); make that first call before any stream
 * capture.  A device reset gives the device a new context, and the next
 * call looks the address up again.
 * All calls share the one array: calls that overlap on the GPU (other
 * streams, other host threads) race and must be serialised by the caller.
 * No device status word is kept: a slot whose id lies outside [0,E) is
 * skipped -- it is counted nowhere, no row is assigned to it and its
 * inv_perm entry is left unwritten (it keeps whatever the caller's buffer
 * held) -- so offsets[E] then falls short of T*k.  Check offsets[E] == T*k
 * before passing the outputs to the expert GEMMs or the combine. */
moe_status_t moe_permute_noalloc(const int32_t *topk_ids, int T, int E, int k,
                                 int32_t *counts, int32_t *offsets,
                                 int32_t *sorted_token_ids, int32_t *inv_perm, void *stream);

/* Grouped gate/up GEMM with SwiGLU: for every permuted row r in
 * [offsets[e], offsets[e+1]), h[r, :] = bf16(silu(g) * u) with
 * [g | u] = x[sorted_token_ids[r], :] . W_gate_up[e]  (W_gate_up [E, H, 2I],
 * columns [0,I) gate, [I,2I) up; fp32 accumulation).  The rows of x are
 * gathered inside the kernel; no permuted copy of x is made.  h is
 * [T*k, I] bf16.  tile_policy: MOE_TILES_*. */
moe_status_t moe_grouped_swiglu(const uint16_t *x, const uint16_t *w_gate_up,
                                const int32_t *offsets, const int32_t *sorted_token_ids,
                                int T, int H, int E, int I, int k, int tile_policy,
                                uint16_t *h, void *workspace, size_t workspace_bytes,
                                void *stream);

/* Grouped down GEMM: o[r, :] = h[r, :] . W_down[e] for every permuted row
 * (W_down [E, I, H] bf16, h [R, I] bf16, o [R, H] f32, R = offsets[E]).
 * offsets may be NULL for one group of R = rows rows (E must then be 1). */
moe_status_t moe_grouped_down(const uint16_t *h, const uint16_t *w_down, const int32_t *offsets,
                              int rows, int H, int E, int I, int tile_policy, float *o,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Down GEMM + weighted combine: y [T,H] bf16 from h [T*k, I] bf16 (permuted
 * order), W_down [E, I, H] bf16, topk_w [T,k] f32, inv_perm [T,k] i32,
 * offsets [E+1] i32 and an optional shared-expert output shared_out [T,H]
 * f32 (NULL for none), added after the k routed terms.  Expert output rows
 * stay fp32; the k terms of a token are summed in slot order j = 0..k-1 in
 * fp32, so y is bitwise reproducible. */
moe_status_t moe_down_combine(const uint16_t *h, const uint16_t *w_down,
                              const float *topk_w, const int32_t *inv_perm,
                              const int32_t *offsets, const float *shared_out,
                              int T, int H, int E, int I, int k, int tile_policy,
                              uint16_t *y, void *workspace, size_t workspace_bytes,
                              void *stream);

/* The whole layer: y [T,H] bf16.  W_sh_gate_up [H, 2 I_s] and W_sh_down
 * [I_s, H] describe the optional shared expert (both NULL and I_s = 0 for
 * none).  Intermediates stay in the workspace (moe_workspace_layout).
 * When T*k is so small that the expert GEMMs have fewer work units than
 * the GPU has SMs, their K range is split and the partial slabs are summed
 * in a fixed order (gate/up before SwiGLU, down inside the combine); y is
 * bitwise reproducible for given shapes either way. */
moe_status_t moe_forward(const uint16_t *x, const float *w_router, const float *bias,
                         const uint16_t *w_gate_up, const uint16_t *w_down,
                         const uint16_t *w_sh_gate_up, const uint16_t *w_sh_down, int I_s,
                         int T, int H, int E, int I, int k,
                         uint16_t *y, void *workspace, size_t workspace_bytes, void *stream);

/* moe_forward with explicit choices (MOE_TILES_*, MOE_ROUTER_*), optional
 * stage timing events and a launch count. */
typedef struct moe_forward_options {
  int tile_policy;
  int router_impl;
  /* Optional timing hooks: a non-NULL stage_events[i] (a cudaEvent_t owned
   * by the caller) is recorded on the stream at stage boundary i:
   * 0 before routing, 1 after routing, 2 after the permutation, 3 after the
   * shared expert, 4 after the gate/up GEMM, 5 after the down GEMM, 6 after
   * the combine.  With MOE_ROUTER_SMALL routing and permutation are one
   * kernel (events 1 and 2 are recorded together after it). */
  void *stage_events[7];
  /* Output: the number of kernels this call enqueued. */
  int launches;
  /* Router scoring rule (MOE_SCORE_*; 0, the zero-initialised default, is
   * MOE_SCORE_SOFTMAX). */
  int scoring;
  /* Where the weighted combine (and, when K is split, the slab sum + SwiGLU
   * of the gate/up GEMM) runs (MOE_COMBINE_*; 0 is MOE_COMBINE_AUTO). */
  int combine;
  int reserved[3];
} moe_forward_options_t;

moe_status_t moe_forward_ex(const uint16_t *x, const float *w_router, const float *bias,
                            const uint16_t *w_gate_up, const uint16_t *w_down,
                            const uint16_t *w_sh_gate_up, const uint16_t *w_sh_down, int I_s,
                            int T, int H, int E, int I, int k,
                            uint16_t *y, void *workspace, size_t workspace_bytes,
                            moe_forward_options_t *options, void *stream);

/* The layer on block-scaled FP8 expert weights.  Each routed expert matrix
 * W [E, K, N] (W_gate_up: K = H, N = 2I; W_down: K = I, N = H) is given as
 * OCP FP8 E4M3 codes of its transpose, [E, N, K] u8 with K contiguous (1
 * sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 =
 * subnormals; 0x7F/0xFF = NaN; largest 448), and one OCP E8M0 scale per 32
 * consecutive weights along K of each column, [E, K/32, N] u8
 * (2^(code - 127); 0xFF = NaN): the weight W[e, k, n] is
 * e4m3(code[e, n, k]) * 2^(scale[e, k/32, n] - 127).  Token rows, h and the
 * shared expert stay bf16.  Passage: Qwen 3.5-397B MoE on Ironwood (TPU
 * v7x), sec. 6 "numerical validation" (accumulation across FP8 scaling
 * blocks); the Ironwood systems handbook page runs Microscaling formats.
 * Every such weight with a scale code in 3..246 is an exact bf16 value (4
 * significant bits times a power of two, within bf16's range), so the layer
 * computes exactly what moe_forward_ex computes on the dequantised weights,
 * with the same rounding points; only the expert-weight bytes halve (plus
 * 1/32 for the scales).  Below scale code 3 a weight smaller than bf16's
 * least subnormal step is rounded to nearest bf16; above 246 a weight beyond
 * bf16's finite range decodes to +-inf.  Everything else as moe_forward_ex, except: the tile policy
 * PERSISTENT and MOE_COMBINE_FUSED are not available
 * (MOE_ERR_INVALID_ARG), and PAIR runs as LARGE (single-SM 256-row passes).
 * The two E4M3 NaN patterns are not supported as weights (they decode as
 * +-480, not NaN).  Codes and scales pointers 16-byte aligned. */
moe_status_t moe_forward_mx(const uint16_t *x, const float *w_router, const float *bias,
                            const uint8_t *w_gate_up_codes, const uint8_t *w_gate_up_scales,
                            const uint8_t *w_down_codes, const uint8_t *w_down_scales,
                            const uint16_t *w_sh_gate_up, const uint16_t *w_sh_down, int I_s,
                            int T, int H, int E, int I, int k,
                            uint16_t *y, void *workspace, size_t workspace_bytes,
                            moe_forward_options_t *options, void *stream);

/* Failure-detection self test: launches one block that waits, with the
 * library's bounded wait, on a barrier nothing will complete.  After
 * timeout_ns the wait gives up, the kernel records MOE_ERR_DEVICE_TIMEOUT
 * in the workspace status word and returns; the context stays usable.
 * Read the result with moe_get_device_status(). */
moe_status_t moe_selftest_timeout(void *workspace, size_t workspace_bytes,
                                  uint64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
