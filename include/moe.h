/*
 * moe.h - C ABI of libmoe.so: the forward pass of one Mixture-of-Experts layer
 * on one NVIDIA B200 (sm_100a).
 *
 * The pass, in the notation of "MoE 训练加速实战：DeepEP + Grouped GeMM +
 * Aux-Loss-Free" §2.2 "Router 数学" (N experts, token x in R^d, W_r in R^{d x N}):
 *
 *   g(x)   = x W_r (+ b)                               router logits, fp32
 *   s(x)   = softmax(g(x))                             fp32, max-subtracted
 *   y      = sum_{i in top-k(g)} s_i / (sum_{j in top-k} s_j) * Expert_i(x)
 *
 * with each expert a SwiGLU FFN  Expert_i(x) = (silu(x W1_i) * (x W3_i)) W2_i,
 * a per-expert capacity C = ceil(capacity_factor * T * k / N) whose overflow is
 * dropped in token order ("负载均衡策略：MoE训练稳定性保障", section "专家容量裁剪"),
 * the kept assignments permuted into expert-contiguous rows (the single-GPU
 * counterpart of the dispatch all-to-all, §3.2 of the first page), the experts
 * run as one grouped GEMM (§4.2 "数学等价性"), and the load-balance statistics of
 * L_aux = (T/N) sum_i y_i z_i ("负载均衡策略", section "辅助损失函数").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer on the current CUDA device, owned
 *    by the caller.  The library never allocates, frees or synchronises: work is
 *    enqueued on `stream` (NULL = the legacy default stream) in call order.
 *    The only exception is moe_read_flags(), which waits for the stream.
 *  - Tensors are dense, row-major, with no padding between rows.
 *  - "act" tensors (x, xp, h, out_rows, y, shared_out, expert weights) have the
 *    config's act_dtype: MOE_F32 (float) or MOE_BF16 (uint16 bf16 bit patterns).
 *    The router weight, bias, logits and routing weights are always fp32.
 *  - Each call validates its arguments on the host before it launches anything
 *    and returns a moe_status_t.  No call traps, aborts or throws.  A failed
 *    launch returns MOE_ERR_CUDA (the CUDA error string is available from
 *    moe_last_cuda_error()).  Conditions only the GPU can see (non-finite
 *    logits, an out-of-range expert index, a pipeline wait that ran out) set
 *    bits in the flags word at the start of the workspace; read them with
 *    moe_read_flags().
 *  - Buffers that kernels read or write with 16-byte vectors (x, xp, h,
 *    out_rows, y, shared_out, weights) must be 16-byte aligned
 *    (MOE_ERR_MISALIGNED).
 *  - bf16 layers need d % 64 == 0 and f % 64 == 0 (and f_shared % 64 == 0):
 *    the expert GEMMs step through K in 64-element slabs (MOE_ERR_UNSUPPORTED).
 *  - Limits: 1 <= N <= 256, 1 <= k <= min(N, 32), T * k < 2^31, T >= 0 (T = 0
 *    is a valid empty batch: outputs are left untouched, statistics are zeroed).
 *  - Results are deterministic: the same inputs give the same bytes.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* NULL where required, bad sizes, k > N, ... */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes */
  MOE_ERR_MISALIGNED = 3,    /* a vector-accessed buffer is not 16-byte aligned */
  MOE_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than the query says */
  MOE_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  MOE_ERR_NONFINITE = 6,     /* (from moe_read_flags) non-finite router logits */
  MOE_ERR_DEVICE = 7,        /* (from moe_read_flags) bad index / device wait ran out */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

/* Number format of the routed experts' GEMMs (moe_config_t.gemm_format). */
typedef enum {
  MOE_GEMM_ACT = 0,    /* the act_dtype (bf16 or fp32), the default */
  MOE_GEMM_MXFP8 = 1,  /* block-scaled FP8: E4M3 codes, one E8M0 scale per 32 values along K */
} moe_gemm_format_t;

/* Bits of the device flags word (moe_read_flags). */
#define MOE_FLAG_NONFINITE_LOGITS 0x1u  /* some router logit was NaN or +-Inf */
#define MOE_FLAG_BAD_EXPERT_INDEX 0x2u  /* topk_idx outside [0,N) or repeated in a row */
#define MOE_FLAG_WAIT_TIMEOUT     0x4u  /* a GEMM pipeline wait exceeded its bound */

typedef struct {
  int64_t T;               /* tokens in the batch */
  int32_t d;               /* model dimension */
  int32_t N;               /* routed experts */
  int32_t k;               /* experts per token (top-k) */
  int32_t f;               /* SwiGLU hidden size of a routed expert */
  int32_t f_shared;        /* hidden size of the shared expert; 0 = no shared expert */
  double capacity_factor;  /* C = ceil(capacity_factor * T * k / N), exact on this double */
  int32_t capacity;        /* >= 0: use this C instead of the formula; < 0: derive */
  moe_dtype_t act_dtype;   /* MOE_F32 or MOE_BF16 */
  int32_t seg_align;       /* expert segments start at multiples of this many rows; 0 -> 128 */
  int32_t gemm_format;     /* moe_gemm_format_t; MOE_GEMM_MXFP8 needs act_dtype MOE_BF16,
                              d % 128 == 0, f % 128 == 0 and seg_align % 128 == 0 */
} moe_config_t;

typedef struct {
  const float* w_router;     /* [d, N] fp32 */
  const float* router_bias;  /* [N] fp32, added to the logits; NULL = none */
  const void* w1;            /* [N][d][f] act: gate projection */
  const void* w3;            /* [N][d][f] act: up projection */
  const void* w2;            /* [N][f][d] act: down projection */
  const void* ws1;           /* [d][f_shared] act, shared expert gate; NULL if f_shared == 0 */
  const void* ws3;           /* [d][f_shared] act, shared expert up */
  const void* ws2;           /* [f_shared][d] act, shared expert down */
  const float* selection_bias; /* [N] fp32 Aux-Loss-Free bias, added to g for the top-k
                                  choice only (the weights use the unbiased softmax);
                                  NULL = none.  Update it with moe_bias_update(). */
  /* Block-scaled FP8 copies of the routed experts (gemm_format MOE_GEMM_MXFP8;
     written by moe_mx_quantize_weight): K-major codes and their scales. */
  const void* w1_mx;         /* [N][f][d] E4M3 codes of W1 (K = d) */
  const void* w1_sf;         /* scales of w1_mx: N * f * d / 32 bytes */
  const void* w3_mx;         /* [N][f][d] codes of W3 */
  const void* w3_sf;
  const void* w2_mx;         /* [N][d][f] codes of W2 (K = f) */
  const void* w2_sf;         /* N * d * f / 32 bytes */
  /* Optional bf16 split of w_router made by moe_router_split (bf16 layers); NULL =
     moe_layer_fwd splits w_router itself on every call. */
  const void* w_router_split;
} moe_weights_t;

/* Load-balance and capacity statistics.  Device pointers; each may be NULL. */
typedef struct {
  float* y_frac;        /* [N] y_i: share of the T*k top-k selections (before the drop) */
  float* z_mean;        /* [N] z_i: mean softmax score over the T tokens */
  float* l_aux_p3;      /* [1] (T/N) * sum_i y_i z_i  ("负载均衡策略", "辅助损失函数") */
  float* l_aux_switch;  /* [1] N * sum_i y_i z_i      (Switch form, §5.2 of the first page) */
  int32_t* counts;      /* [N] top-k selections per expert before the drop */
  int32_t* kept;        /* [N] min(counts, C) */
  int32_t* num_dropped; /* [1] sum_i (counts_i - kept_i) */
  /* Router z-loss and load-health figures ("负载均衡策略", hyper-parameter table,
     z_loss_weight; "ms-swift + Megatron：MoE模型加速10倍实测" §3.3 "监控与诊断"). */
  float* z_loss;        /* [1] mean over tokens of (log sum_i exp g_ti)^2 (unbiased g) */
  float* load_std;      /* [1] population std over experts of counts_i / (T*k) */
  float* top2_ratio;    /* [1] share of the T*k selections taken by the two busiest experts */
  float* avg_tokens_per_expert; /* [1] sum_i kept_i / N (filled by the dispatch step) */
} moe_stats_t;

/* Human-readable name of a status. Never NULL. */
const char* moe_status_string(moe_status_t status);

/* Text of the last CUDA error seen by this thread ("" if none). Never NULL. */
const char* moe_last_cuda_error(void);

/* Library version string. */
const char* moe_version(void);

/*
 * moe_capacity - host-only: the per-expert capacity C of `cfg`.
 * "负载均衡策略：MoE训练稳定性保障", section "专家容量裁剪": capacity_factor times
 * the ideal share, e.g. 1024 tokens / 8 experts * 1.25 = 160; with k experts per
 * token the ideal share is T*k/N.  If cfg->capacity >= 0 that value is returned.
 * The product is evaluated exactly (128-bit integers) on the given double.
 * Errors: MOE_ERR_INVALID_ARG for NULL, T < 0, N < 1, k < 1, capacity_factor
 * not finite or < 0, or a capacity above 2^31-1.
 */
moe_status_t moe_capacity(const moe_config_t* cfg, int32_t* capacity);

/*
 * moe_workspace_size - host-only sizes the caller must provide.
 *   layer_bytes: workspace of moe_layer_fwd (routing arrays, the permuted rows,
 *                the SwiGLU hidden rows and the expert outputs);
 *   op_bytes:    workspace of the single-step entry points (moe_route,
 *                moe_route_from_logits, moe_dispatch, moe_expert_ffn,
 *                moe_shared_expert_ffn, moe_combine);
 *   max_rows:    rows the caller must allocate for xp / h / out_rows:
 *                min(T*k, N*min(C,T)) + N*(seg_align-1).
 * Any output pointer may be NULL.  Errors as moe_capacity, plus the shape checks.
 */
moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* layer_bytes,
                                size_t* op_bytes, int64_t* max_rows);

/*
 * moe_route - router GEMM, fp32 softmax, top-k and renormalised weights.
 * "MoE 训练加速实战" §2.2 "Router 数学": g = x W_r, scores = softmax(g), the k
 * largest g selected (ties: lower expert index first; slots in descending g),
 * weight_j = s_{idx_j} / sum_{j'} s_{idx_j'}.
 *   x          [T, d] act          input tokens (read)
 *   w_router   [d, N] fp32, bias [N] fp32 or NULL
 *   selection_bias [N] fp32 or NULL: Aux-Loss-Free bias ("MoE 训练加速实战" §5.3):
 *              the experts are ranked on the fp32 sum g + selection_bias, while the
 *              weights, z_i and the z-loss use the unbiased g
 *   logits_out [T, N] fp32 or NULL: g including the bias (never the selection bias)
 *   topk_idx   [T, k] int32 (written), topk_w [T, k] fp32 (written)
 *   stats      may be NULL: fills y_frac, z_mean, l_aux_p3, l_aux_switch, counts,
 *              z_loss, load_std, top2_ratio
 *   ws         op workspace (>= op_bytes); its flags word is cleared first.
 * Non-finite logits raise MOE_FLAG_NONFINITE_LOGITS (read with moe_read_flags).
 */
moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* w_router,
                       const float* router_bias, const float* selection_bias, float* logits_out,
                       int32_t* topk_idx, float* topk_w, moe_stats_t* stats, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/*
 * moe_route_with_split - moe_route with the bf16 split of the router weight
 * made beforehand by moe_router_split (see there), as moe_layer_fwd takes it in
 * moe_weights_t.w_router_split: the same computation ("MoE 训练加速实战" §2.2,
 * g = x W_r with the router in fp32) and the same results, byte for byte,
 * without the per-call split of W_r.
 *   w_router_split  device, 16-byte aligned, the split of this w_router for
 *                   cfg's d and N (moe_router_split_bytes); owned by the caller,
 *                   read only.  NULL: moe_route exactly.  fp32 layers (no
 *                   tensor-core router) ignore it.
 * All other arguments and errors as moe_route; a misaligned split gives
 * MOE_ERR_MISALIGNED.
 */
moe_status_t moe_route_with_split(const moe_config_t* cfg, const void* x, const float* w_router,
                                  const void* w_router_split, const float* router_bias,
                                  const float* selection_bias, float* logits_out, int32_t* topk_idx,
                                  float* topk_w, moe_stats_t* stats, void* ws, size_t ws_bytes,
                                  moe_stream_t stream);

/*
 * moe_route_from_logits - the same softmax / top-k / weights / statistics as
 * moe_route, starting from caller-supplied fp32 logits [T, N] (no GEMM), with
 * an optional selection_bias [N] as in moe_route.  This is the entry point on
 * which routing is compared bit-for-bit with a reference.
 */
moe_status_t moe_route_from_logits(const moe_config_t* cfg, const float* logits,
                                   const float* selection_bias, int32_t* topk_idx,
                                   float* topk_w, moe_stats_t* stats, void* ws,
                                   size_t ws_bytes, moe_stream_t stream);

/*
 * moe_router_split / moe_router_split_bytes - the bf16 form of the fp32 router
 * weight that the tensor-core router multiplies ("MoE 训练加速实战" §2.2,
 * g = x W_r, with the router kept in fp32, §1 pain point 4): every weight w of
 * W_r [d, N] is split exactly into three bf16 values, w = hi + mid + lo (hi =
 * bf16(w), mid = bf16(w - hi), lo = w - hi - mid), stored as [3][d][NP] with
 * NP = 64, 128 or 256 (the smallest of those >= N; columns N..NP-1 zero).  x is
 * bf16, so each product x*hi, x*mid, x*lo is exact and their fp32 sum is x*w
 * up to the order of the additions.  moe_layer_fwd uses a split passed in
 * moe_weights_t.w_router_split instead of making its own; the split stays
 * valid while W_r is unchanged.  split: device, 16-byte aligned, >= the bytes
 * that moe_router_split_bytes reports; d % 64 == 0, N <= 256 (else
 * MOE_ERR_UNSUPPORTED).
 */
moe_status_t moe_router_split_bytes(int32_t d, int32_t N, size_t* bytes);
moe_status_t moe_router_split(const float* w_router, int32_t d, int32_t N, void* split, size_t bytes,
                              moe_stream_t stream);

/*
 * moe_bias_update - one Aux-Loss-Free bias step ("MoE 训练加速实战" §5.4):
 *   selection_bias[i] += gamma * sign(1/N - f_i),   f_i = counts[i] / (T*k),
 * with the sign taken exactly on integers, sign(T*k - N*counts[i]), and one fp32
 * addition.  counts [N] int32 are a routing call's top-k selections before the
 * capacity drop (moe_stats_t.counts of moe_route / moe_layer_fwd on the same
 * cfg).  selection_bias [N] fp32 is read and written in place on `stream`.
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers, a bad cfg or a non-finite gamma.
 */
moe_status_t moe_bias_update(const moe_config_t* cfg, float* selection_bias, const int32_t* counts,
                             float gamma, moe_stream_t stream);

/*
 * moe_dispatch - capacity clip and permutation into expert-contiguous rows.
 * "负载均衡策略", section "专家容量裁剪" (at most C tokens per expert, the rest
 * dropped) and "ETP专家并行加速MoE模型", section "动态路由下的高效通信" (tokens are
 * re-shuffled to their experts).  Within expert e the assignments are ranked in
 * token order; rank < C is kept.
 *   x         [T, d] act (read)
 *   topk_idx  [T, k] int32 in [0, N), distinct within a row (read)
 *   row_map   [T, k] int32 (written): seg_off[e] + rank, or -1 if dropped
 *   seg_off   [N+1] int32 (written): segment starts, multiples of seg_align;
 *             seg_off[N] = rows in use
 *   seg_count [N] int32 (written): kept rows of each expert = min(count, C)
 *   xp        [max_rows, d] act (written): xp[row_map[t][j]] = x[t] bit for bit;
 *             rows between segments are not written
 *   stats     may be NULL: fills counts, kept, num_dropped, avg_tokens_per_expert
 * An index outside [0, N) or repeated in a row raises MOE_FLAG_BAD_EXPERT_INDEX;
 * that slot is dropped.
 */
moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                          int32_t* row_map, int32_t* seg_off, int32_t* seg_count, void* xp,
                          moe_stats_t* stats, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_dispatch_static - moe_dispatch without a workspace: it allocates nothing
 * and takes no scratch buffer from the caller.  The pages have no counterpart of
 * this entry point.  It is meant for callers that cannot allocate device memory
 * at the point where they dispatch: for example code whose device memory is
 * owned by another allocator (a framework's memory pool), or a runtime that
 * allocates only at start-up and must not call cudaMalloc (which can fail, and
 * synchronises the device) while it serves batches.
 *
 * Inputs, outputs, results and errors are those of moe_dispatch, except:
 *  - the scratch (per-block token masks and rank bases, counts, a ticket) lives
 *    in one fixed array of MOE_DISPATCH_STATIC_SCRATCH_BYTES in the library's
 *    device memory; every GPU that loads the library holds it until the process
 *    exits;
 *  - a batch needs ceil(T/32) * N <= MOE_DISPATCH_STATIC_MAX_CELLS (e.g. T up to
 *    16384 with N = 256); larger batches return MOE_ERR_WORKSPACE and launch
 *    nothing;
 *  - device_flags (may be NULL) receives the MOE_FLAG_* bits by bitwise OR; the
 *    caller zeroes it beforehand.  With NULL a bad index is still dropped
 *    (row_map -1) but not reported.
 *  - all calls share the one array and it keeps the last call's contents (each
 *    call rewrites every part it reads).  Calls whose work overlaps on the GPU
 *    (different streams, or several host threads) race on it: order them.
 *  - every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress), so the address stays right after cudaDeviceReset;
 *    the first call on a device also loads the library's device code there:
 *    make that first call before any stream capture.
 */
#define MOE_DISPATCH_STATIC_MAX_CELLS 131072
#define MOE_DISPATCH_STATIC_SCRATCH_BYTES (2u * 4u * MOE_DISPATCH_STATIC_MAX_CELLS + 2048u)
moe_status_t moe_dispatch_static(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                 int32_t* row_map, int32_t* seg_off, int32_t* seg_count, void* xp,
                                 moe_stats_t* stats, uint32_t* device_flags, moe_stream_t stream);

/*
 * Block-scaled FP8 ("MoE 训练加速实战" §9.1: FP8 forward with bf16 activations;
 * the pages fix no format).  A tensor of R rows by K values (K a multiple of
 * 128) is stored as R x K E4M3 codes (row-major) plus one E8M0 scale byte per
 * 32 consecutive values of a row: the value of code c in block b is
 * e4m3(c) * 2^(scale_b - 127), where scale_b - 127 is the smallest exponent e
 * with max|v| <= 448 * 2^e over the block, and each code is v / 2^e rounded to
 * the nearest E4M3 value (ties to even).  The scale bytes use the layout the
 * tensor cores read: 512-byte atoms for 128 rows x 4 blocks, atoms in order
 * (row / 128, block / 4), and inside an atom row m, block j at byte
 * 16 * (m % 32) + 4 * (m / 32) + j % 4; a buffer for R rows holds
 * ceil(R / 128) * 128 * K / 32 bytes.
 */

/*
 * moe_mx_quantize_weight - quantize G matrices w [G][K][N] (bf16, N contiguous,
 * the layout of W1/W3 with K = d, N = f, or of W2 with K = f, N = d) along K:
 * codes [G][N][K] (K-major) and sf (G * N * K / 32 bytes, N counting rows).
 * K and N multiples of 128 (MOE_ERR_UNSUPPORTED otherwise); every buffer
 * 16-byte aligned.  Bit-exact and deterministic.
 */
moe_status_t moe_mx_quantize_weight(const void* w, int64_t G, int32_t K, int32_t N, void* codes, void* sf,
                                    moe_stream_t stream);

/*
 * moe_dispatch_mx - moe_dispatch for a MOE_GEMM_MXFP8 layer: the same row map,
 * segments and statistics, with each kept row quantized on the way: xp_codes
 * [max_rows, d] E4M3 codes and xp_sf (scales of max_rows rows, K = d).  x is
 * bf16.  Rows between segments are not written.
 */
moe_status_t moe_dispatch_mx(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                             int32_t* row_map, int32_t* seg_off, int32_t* seg_count, void* xp_codes,
                             void* xp_sf, moe_stats_t* stats, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * moe_expert_ffn_mx - the routed experts of a MOE_GEMM_MXFP8 layer as one
 * grouped GEMM pair on the tcgen05 block-scaled FP8 tensor cores
 * (kind::mxf8f6f4, scales applied inside the MMA, fp32 accumulation):
 *   h[r] = silu(xp[r] W1_e) * (xp[r] W3_e), written as FP8 codes h_codes
 *          [max_rows, f] + h_sf (blocks of 32 along f)
 *   out_rows[r] = h[r] W2_e, bf16 [max_rows, d]
 * Inputs: xp_codes / xp_sf from moe_dispatch_mx, weights->w{1,3,2}_mx/_sf.
 */
moe_status_t moe_expert_ffn_mx(const moe_config_t* cfg, const void* xp_codes, const void* xp_sf,
                               const int32_t* seg_off, const int32_t* seg_count,
                               const moe_weights_t* weights, void* h_codes, void* h_sf,
                               void* out_rows, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn - all routed experts as one grouped GEMM pair, SwiGLU fused.
 * "MoE 训练加速实战" §4.1-4.2: one kernel serves every expert, y_i = W_i x_i.
 * For every expert e and row r in [seg_off[e], seg_off[e] + seg_count[e]):
 *   h[r]        = silu(xp[r] W1_e) * (xp[r] W3_e)      (fp32 math, one rounding to act)
 *   out_rows[r] = h[r] W2_e                            (fp32 accumulation)
 *   xp, h, out_rows: [max_rows, d], [max_rows, f], [max_rows, d] act.
 * Rows outside the segments are neither read for results nor written.
 * bf16 runs on the tcgen05 tensor cores; fp32 runs on the CUDA cores.
 */
moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* xp, const int32_t* seg_off,
                            const int32_t* seg_count, const moe_weights_t* weights, void* h,
                            void* out_rows, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_shared_expert_ffn - the always-on shared expert ("MoE 训练加速实战" §2.3
 * spec table and §9.1: DeepSeek-V3 uses one) over all T tokens:
 *   shared_out[t] = (silu(x[t] Ws1) * (x[t] Ws3)) Ws2
 *   h_shared [T, f_shared] act scratch; shared_out [T, d] act.
 * MOE_ERR_INVALID_ARG if cfg->f_shared == 0.
 */
moe_status_t moe_shared_expert_ffn(const moe_config_t* cfg, const void* x,
                                   const moe_weights_t* weights, void* h_shared,
                                   void* shared_out, void* ws, size_t ws_bytes,
                                   moe_stream_t stream);

/*
 * moe_combine - weighted sum back to token order ("MoE 训练加速实战" §2.1,
 * "权重加和"):  y[t] = sum_{j=0..k-1, row_map[t][j] >= 0} topk_w[t][j] *
 * out_rows[row_map[t][j]]  (+ shared_out[t]), accumulated in fp32 in slot
 * order, rounded once to act.  Dropped slots add nothing; the kept weights are
 * not renormalised.  shared_out may be NULL.  y [T, d] act (written).
 */
moe_status_t moe_combine(const moe_config_t* cfg, const void* out_rows, const int32_t* row_map,
                         const float* topk_w, const void* shared_out, void* y, void* ws,
                         size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer_fwd - the whole layer: route, dispatch, routed experts, shared
 * expert (if cfg->f_shared > 0), combine.  With gemm_format MOE_GEMM_MXFP8 the
 * dispatch quantizes the rows and the routed experts run in block-scaled FP8
 * from weights->w*_mx (the bf16 w1/w3/w2 are not read; the shared expert stays
 * bf16).  x [T, d] act (read), y [T, d] act
 * (written), stats may be NULL (every field is filled), ws >= layer_bytes of
 * moe_workspace_size.  weights->selection_bias (may be NULL) steers the top-k
 * choice as in moe_route; the layer does not update it.  The permuted rows and
 * the expert outputs share one workspace region.
 */
moe_status_t moe_layer_fwd(const moe_config_t* cfg, const moe_weights_t* weights,
                           const void* x, void* y, moe_stats_t* stats, void* ws,
                           size_t ws_bytes, moe_stream_t stream);

/*
 * Backward pass of one layer ("MoE 训练加速实战" §5.2: the training loss is the
 * main loss plus a weighted auxiliary loss; "负载均衡策略": z_loss_weight;
 * "ms-swift + Megatron：MoE模型加速10倍实测" §2.3: only the experts a token was
 * routed to receive its gradient).  moe_layer_bwd returns the gradient of
 *   L = <dy, y> + aux_weight * L_aux + z_weight * z_loss
 * with y the output of moe_layer_fwd on the same inputs, L_aux = N sum_i f_i P_i
 * (the l_aux_switch statistic: f_i the selection share, a count without
 * gradient; P_i the mean softmax score) and z_loss the z_loss statistic.  The
 * routing decisions (top-k set, capacity drops) carry no gradient, nor does the
 * selection bias.  The call recomputes the forward pass from x (activation
 * recomputation) and needs nothing saved from it; a router split in
 * weights->w_router_split (moe_router_split) is used there as in
 * moe_layer_fwd, with the same result.  bf16 layers with
 * gemm_format MOE_GEMM_ACT and seg_align a multiple of 64 (MOE_ERR_UNSUPPORTED
 * otherwise).  Weight gradients are fp32 and overwrite their buffers; dx is
 * bf16.  Deterministic.
 */
typedef struct {
  void* dx;              /* [T, d] bf16 */
  float* dw_router;      /* [d, N] */
  float* drouter_bias;   /* [N], or NULL; written only when weights->router_bias is set */
  float* dw1;            /* [N][d][f] */
  float* dw3;            /* [N][d][f] */
  float* dw2;            /* [N][f][d] */
  float* dws1;           /* [d][f_shared] (f_shared > 0), else NULL */
  float* dws3;           /* [d][f_shared] */
  float* dws2;           /* [f_shared][d] */
} moe_grads_t;

/* Bytes of the workspace of moe_layer_bwd. */
moe_status_t moe_backward_workspace_size(const moe_config_t* cfg, size_t* bytes);

moe_status_t moe_layer_bwd(const moe_config_t* cfg, const moe_weights_t* weights, const void* x,
                           const void* dy, float aux_weight, float z_weight, moe_grads_t* grads,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_set_wait_limit_ns - failure handling (the pages define no such call):
 * the time bound of the pipeline waits of the tensor-core GEMMs (the bf16 and
 * block-scaled FP8 grouped GEMMs and the router GEMM: a stage's operands, a
 * free stage, an accumulator) for kernels launched after this call, process
 * wide.  ns = 0 restores the default of 2 s, within which every legitimate wait
 * ends; a shorter bound makes those waits run out on purpose, which is how the
 * timeout path is tested: the kernel then raises MOE_FLAG_WAIT_TIMEOUT, still
 * waits (with the default bound) for the copies and MMAs it has in flight,
 * frees its tensor memory and returns, leaving the outputs undefined.
 * Errors: MOE_ERR_INVALID_ARG for ns above 2 s.
 */
moe_status_t moe_set_wait_limit_ns(uint64_t ns);

/*
 * moe_read_flags - wait for `stream`, then copy the workspace's device flags
 * word (MOE_FLAG_* bits, cleared by moe_route / moe_route_from_logits /
 * moe_layer_fwd) to *flags.  Returns MOE_ERR_NONFINITE or MOE_ERR_DEVICE when a
 * bit is set, MOE_OK otherwise.
 */
moe_status_t moe_read_flags(const void* ws, size_t ws_bytes, uint32_t* flags,
                            moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
