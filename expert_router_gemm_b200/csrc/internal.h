// Internal declarations shared by the host entry points (moe_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- routing
// The router kernel is instantiated for a padded expert count NP (a power of
// two >= 8, >= N); experts N..NP-1 are masked.  Each block handles route_bt(NP)
// tokens with 256 threads.
constexpr int kRouteThreads = 256;

inline constexpr int route_np(int N) {
  return N <= 8 ? 8 : N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
}
inline constexpr int route_bt(int np) {
  return np == 8 ? 256 : np == 16 ? 256 : np == 32 ? 128 : np == 64 ? 128 : np == 128 ? 64 : 32;
}

struct RouteArgs {
  int64_t T;
  int d, N, k;
  int x_is_bf16;            // 1: x holds bf16 bits, 0: fp32
  const void* x;            // [T, d] (GEMM mode) or nullptr
  const float* w_router;    // [d, N]
  const float* bias;        // [N] or nullptr
  const float* sel_bias;    // [N] or nullptr: added to the logits for the top-k choice only
  const float* logits_in;   // [T, N] (logits mode) or nullptr
  int n_partials;           // logits mode: logits_in holds this many [T, N] partial sums (>= 1),
                            // added in order, then the bias (if any) is added
  float* logits_out;        // [T, N] or nullptr
  int32_t* topk_idx;        // [T, k]
  float* topk_w;            // [T, k]
  int32_t* cnt_acc;         // [N] zeroed: top-k counts (statistics)
  unsigned long long* z_acc;  // [N] zeroed: sum of softmax scores, 32 fraction bits
  uint32_t* ticket;         // [1] zeroed: blocks finished (last one finalises)
  double* zl_part;          // [blocks] per-block sums of logsumexp^2 (z-loss)
  int want_stats;           // fill `stats` (else the statistics are skipped)
  moe_stats_t stats;        // device pointers, each may be null
  uint32_t* flags;
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
// The route kernel's blocks hold at least this many tokens (sizes zl_part).
constexpr int kRouteMinBlockTokens = 16;

// b[i] += gamma * sign(T*k - N*counts[i]) for i < N (one block).
cudaError_t launch_bias_update(float* b, const int32_t* counts, int64_t Tk, int N, float gamma, cudaStream_t s);

// Router GEMM on the tensor cores (bf16 x) over the three bf16 parts of W_r
// ([3][d][router_split_width(N)] bf16, made by launch_router_split): fp32
// partial sums over up to kRouterMaxPartials K slices, slice z at
// partials + z * T * N, without the bias; *n_partials receives the number of
// slices.  `split` is a split made earlier, or (make_split) one is first
// written to split_buf.  The softmax / top-k pass (launch_route) then runs in
// logits mode on the partials.
constexpr int kRouterTcMinExperts = 1;  // every bf16 layer
constexpr int kRouterMaxPartials = 4;
int router_split_width(int N);
size_t router_split_bytes(int d, int N);
cudaError_t launch_router_split(const float* w_router, int d, int N, void* split, cudaStream_t s);
cudaError_t launch_router_tc(const RouteArgs& a, const void* split, bool make_split, void* split_buf, float* partials,
                             int* n_partials, cudaStream_t s);
// z-loss partial slots (RouteArgs.zl_part) for T tokens
size_t router_zl_slots(int64_t T);

// 2-D bf16 TMA tensor map over a row-major [outer, inner] tensor, 128-byte
// swizzle, zero fill outside the tensor.
bool make_tma_2d_bf16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer);
// 3-D fp32 tensor map [outer][mid][inner] (inner contiguous), 128-byte swizzle,
// for tiled stores of [box_mid x box_inner] blocks (box_inner * 4 == 128).
bool make_tma_3d_f32_sw128(CUtensorMap* m, void* ptr, uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_inner,
                           uint32_t box_mid);
// The same over bytes (FP8 codes).
bool make_tma_2d_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                    uint32_t box_outer);
// Bytes without swizzle (boxes copied as laid out, e.g. 512-byte scale atoms).
bool make_tma_2d_u8_plain(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                          uint32_t box_outer);

// --------------------------------------------------------------- dispatch
constexpr int kDispatchTokens = 32;   // tokens per dispatch block (one bit each)

struct DispatchArgs {
  int64_t T;
  int d, N, k, capacity, align, elem_bytes;
  const void* x;
  const int32_t* topk_idx;
  int32_t* row_map;
  int32_t* seg_off;
  int32_t* seg_count;
  void* xp;
  uint8_t* xp_sf;           // non-null: xp receives block-scaled FP8 codes and these
                            // scale bytes (tile-interleaved, d/32 per row)
  int32_t* row_token;       // non-null: no rows are copied; row_token[row_map[t][j]] = t instead
                            // (the grouped GEMM then gathers its A rows from x)
  uint32_t* mask;           // [blocks, N] scratch
  int32_t* base;            // [blocks, N] scratch
  int32_t* counts;          // [N] scratch
  uint32_t* ticket;         // [1] scratch
  moe_stats_t stats;
  uint32_t* flags;
};
cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s);

// Validates a dispatch call and fills every field of `a` except the scratch
// pointers (mask, base, counts, ticket) and flags; *blocks receives the number
// of 32-token blocks.  Host only, touches no device state.
moe_status_t dispatch_prepare(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                              int32_t* row_map, int32_t* seg_off, int32_t* seg_count, void* xp,
                              const moe_stats_t* stats, DispatchArgs* a, int64_t* blocks);
// T == 0: zero the segment table and the dispatch statistics.
moe_status_t dispatch_empty(const DispatchArgs& a, cudaStream_t s);
// MOE_OK for cudaSuccess, else MOE_ERR_CUDA with the error kept for moe_last_cuda_error().
moe_status_t cuda_error_status(cudaError_t e);

// ------------------------------------------------------------ expert FFN
// One grouped SwiGLU FFN over G groups of rows.  Group g owns rows
// [row0_g, row0_g + count_g) of `a` / `h` / `out`, where row0_g = seg_off[g]
// and count_g = seg_count[g]; with seg_off == nullptr there is one group of
// `dense_rows` rows starting at row 0.
struct FfnArgs {
  int G;
  int dense_rows;
  int max_count;            // upper bound of count_g (grid sizing of the fp32 path)
  int64_t mean_rows;        // expected rows per group (tile-shape choice of the bf16 path)
  int64_t max_rows;         // rows of a / h / out buffers
  int d, f;
  const int32_t* seg_off;
  const int32_t* seg_count;
  const void* a;            // [rows, d], or x [a_token_rows, d] when a_token is set
  const int32_t* a_token;   // bf16 path, optional: row r of a group reads row a_token[r] of `a`
                            // (GEMM1 gathers the token rows; entries past a group's count unused)
  int64_t a_token_rows;     // rows of `a` when a_token is set
  const void* w1;           // [G][d][f]
  const void* w3;           // [G][d][f]
  const void* w2;           // [G][f][d]
  void* h;                  // [rows, f]
  void* out;                // [rows, d]
  void* save_g;             // bf16 path, optional: [rows, f] gate / up pre-activations of GEMM1
  void* save_u;
  uint32_t* flags;
};
cudaError_t launch_ffn_bf16(const FfnArgs& a, cudaStream_t s);
// Bound of the bf16 grouped GEMM's pipeline waits for later launches (0: the default).
void set_pipeline_wait_ns(uint64_t ns);
// The bf16 layer pass lets GEMM1 gather token rows from x (MOE_GATHER=lsu|tma)
// instead of copying them into the permuted buffer first.
bool layer_gathers_rows();
cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t s);

// Block-scaled FP8 (E4M3 codes, one E8M0 scale byte per 32 values along K,
// scales in the tile-interleaved layout of mx_sf_offset) grouped SwiGLU FFN:
// a = FP8 codes of the permuted rows [rows, d] with a_sf; w1/w3 [G][f][d] and w2
// [G][d][f] K-major codes with their scales; h = FP8 codes [rows, f] with h_sf
// (written by GEMM1, read by GEMM2); out [rows, d] bf16.  d and f are
// multiples of 128 and segments start at multiples of 128 rows.
struct FfnMxArgs {
  int G;
  int64_t mean_rows;        // expected rows per expert (tile-shape choice)
  int64_t max_rows;
  int d, f;
  const int32_t* seg_off;
  const int32_t* seg_count;
  const uint8_t* a;
  const uint8_t* a_sf;
  const uint8_t* w1;
  const uint8_t* w1_sf;
  const uint8_t* w3;
  const uint8_t* w3_sf;
  const uint8_t* w2;
  const uint8_t* w2_sf;
  uint8_t* h;
  uint8_t* h_sf;
  void* out;
  uint32_t* flags;
};
cudaError_t launch_ffn_mx(const FfnMxArgs& a, cudaStream_t s);
// The same bound for the block-scaled FP8 grouped GEMM, and for the router GEMM.
void set_mx_pipeline_wait_ns(uint64_t ns);
void set_router_wait_ns(uint64_t ns);

// Quantize G weights [G][K][N] (bf16, N contiguous) to K-major FP8 codes
// [G][N][K] and scale bytes [G][N/128][K/128][512]; K, N multiples of 128.
cudaError_t launch_mx_quantize_weight(const uint16_t* w, int64_t G, int K, int N, uint8_t* codes, uint8_t* sf,
                                      cudaStream_t s);

// Byte offset of the scale of (row, 32-element block kb) in a tile-interleaved
// scale buffer with n_kblocks blocks per row: 512-byte atoms of 128 rows x 4
// blocks ordered (row tile, K tile); inside an atom 16 (m % 32) + 4 (m / 32) + j.
__host__ __device__ inline int64_t mx_sf_offset(int64_t row, int kb, int n_kblocks) {
  const int64_t atom = (row >> 7) * (n_kblocks >> 2) + (kb >> 2);
  const int m = static_cast<int>(row & 127);
  return atom * 512 + 16 * (m & 31) + 4 * (m >> 5) + (kb & 3);
}
// bytes of the scales of `rows` rows of K values
__host__ __device__ inline int64_t mx_sf_bytes(int64_t rows, int K) { return (rows + 127) / 128 * 128 * (K / 32); }

// --------------------------------------------------------------- backward
// Row groups of the backward GEMMs: the experts' segments (seg_off [G+1],
// seg_count [G]) or, with seg_off == nullptr, one dense group of dense_rows rows.
struct BwdGroups {
  int G;
  int dense_rows;
  int64_t max_rows;
  const int32_t* seg_off;
  const int32_t* seg_count;
  uint32_t* flags;
};
// dH = dO W2^T per group, then dG = dH * u * silu'(g), dU = dH * silu(g) (bf16;
// rows of a segment past its kept count are written as zeros).
cudaError_t launch_dgrad_swiglu(const BwdGroups& s, int d, int f, const void* dO, const void* w2, const void* g,
                                const void* u, void* dG, void* dU, cudaStream_t st);
// dXp = dG W1^T + dU W3^T per group (bf16, kept rows).
cudaError_t launch_dgrad_plain2(const BwdGroups& s, int d, int f, const void* dG, const void* dU, const void* w1,
                                const void* w3, void* dXp, cudaStream_t st);
// out[g] = A_g^T B_g over the rows of group g (its padded segment, whose extra
// rows are zero): A [rows][M], B [rows][N] bf16, out [G][M][N] fp32.
cudaError_t launch_wgrad(const BwdGroups& s, int M, int N, const void* a, const void* b, float* out, cudaStream_t st);

struct BwdSmallArgs {
  int64_t T;
  int d, N, k, f;
  float aux_weight, z_weight;
  const uint16_t* dy;        // [T, d]
  const float* logits;       // [T, N] (router logits incl. the router bias)
  const int32_t* topk_idx;   // [T, k]
  const float* topk_w;       // [T, k]
  const int32_t* row_map;    // [T, k]
  const int32_t* counts;     // [N] top-k selections per expert
  const uint16_t* out_rows;  // [rows, d] expert outputs o
  uint16_t* dO;              // [rows, d]
  float* dw;                 // [T, k] gradient of the routing weights
  float* dg;                 // [T, N] gradient of the logits
};
// dO[row] = w * dy[t] and dw[t][j] = <dy[t], o[row]> for kept slots (dw = 0 for
// dropped ones).
cudaError_t launch_combine_bwd(const BwdSmallArgs& a, cudaStream_t s);
// Router backward: renormalised weights, softmax, Switch auxiliary loss and
// z-loss gradients -> dg.
cudaError_t launch_router_bwd(const BwdSmallArgs& a, cudaStream_t s);
// Zero the rows [seg_off[e] + seg_count[e], seg_off[e+1]) of up to four bf16
// row buffers (row widths cols[i], multiples of 8).
struct PadBufs {
  void* buf[4];
  int cols[4];
  int n;
};
cudaError_t launch_zero_pad_rows(int N, const int32_t* seg_off, const int32_t* seg_count, const PadBufs& b,
                                 cudaStream_t s);
// The router's two gradient products (x bf16 [T, d], dg fp32 [T, N], W_r fp32
// [d, N]): dW_r = x^T dg (fp32 [d, N]), dbias = sum_t dg[t] (may be null) and
// dxr = dg W_r^T (fp32, router_dxr_rows(T) rows of d; rows >= T are scratch).
// Wide routers (N >= 64, T >= 64) run on the tensor cores through the weight-
// gradient GEMM: the fp32 operands split into bf16 parts (dg = hi + lo,
// W_r = hi + lo; x is bf16 already), the part products summed in fp32.  Small
// routers run on CUDA cores.  Partial sums are added in a fixed order.
size_t router_grad_scratch_bytes(int64_t T, int d, int N);
int64_t router_dxr_rows(int64_t T);
cudaError_t launch_router_grads(int64_t T, int d, int N, const uint16_t* x, const float* dg, const float* w_router,
                                float* dw_router, float* dbias, float* dxr, void* scratch, uint32_t* flags,
                                cudaStream_t s);
// dx[t] = sum over kept slots of dXp[row] + dxr[t] (+ dxs[t]), one rounding to bf16.
cudaError_t launch_dx_gather(int64_t T, int d, int k, const int32_t* row_map, const uint16_t* dXp, const float* dxr,
                             const uint16_t* dxs, uint16_t* dx, cudaStream_t s);

// ---------------------------------------------------------------- combine
struct CombineArgs {
  int64_t T;
  int d, k, is_bf16;
  const void* out_rows;
  const int32_t* row_map;
  const float* topk_w;
  const void* shared_out;   // or nullptr
  void* y;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

// flags word bits used by kernels (mirror of the public MOE_FLAG_* values)
constexpr uint32_t kFlagNonfinite = MOE_FLAG_NONFINITE_LOGITS;
constexpr uint32_t kFlagBadIndex = MOE_FLAG_BAD_EXPERT_INDEX;
constexpr uint32_t kFlagTimeout = MOE_FLAG_WAIT_TIMEOUT;

int device_sm_count();    // cached per device

// Whether forward-path kernels are launched to overlap the end of the
// previous kernel of their stream (programmatic dependent launch; MOE_PDL=0
// turns it off).
bool launch_overlap_enabled();

// Launches `kernel` so that it may start while the previous kernel of the
// stream finishes; the kernel must call grid_dep_wait() before it reads
// anything that kernel wrote (and before any early return).
template <typename... Params, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = launch_overlap_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe
