// Capacity clip and permutation into expert-contiguous rows.
//
// "负载均衡策略：MoE训练稳定性保障", section "专家容量裁剪": each expert processes at
// most C = ceil(capacity_factor * T * k / N) tokens and the overflow is dropped;
// the drop order here is token order (the earliest C assignments of an expert
// are kept).  "ETP专家并行加速MoE模型", section "动态路由下的高效通信": the tokens
// are re-shuffled to their experts; on one GPU that is a stable scatter into one
// buffer with a contiguous segment per expert.
//
// Three kernels, no atomics whose order matters and no spin waits:
//   1. mask:    per block of 32 tokens, a 32-bit token mask per expert
//               (bit t set iff token t of the block chose the expert);
//   2. scan:    per expert, exclusive prefix of popcount(mask) over the blocks
//               (-> rank base of every block) and the total count; the last block
//               to finish (ticket counter, no waiting) turns the counts into
//               kept = min(count, C) and the aligned segment offsets;
//   3. scatter: rank of (t, e) = base[block][e] + popcount of the mask bits below
//               t, kept iff rank < C; row = seg_off[e] + rank; one warp per token
//               copies x[t] with 16-byte vectors to each of its kept rows.  In the
//               layer pass the rows are not copied: an index kernel records the
//               token of every kept row and the grouped GEMM gathers from x.
#include <cuda_fp8.h>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kMaskThreads = 256;
constexpr int kScatterTokens = 8;                         // tokens per scatter block
constexpr int kScatterThreads = 32 * kScatterTokens;      // one warp per token
// 16-byte vectors each lane loads before it stores them: 8 in the copying
// scatter (0.128 against 0.132 ms per Qwen3-shaped dispatch in the layer loop,
// same box), 4 in the quantizing one
constexpr int kCopyUnroll = 8;
constexpr int kQuantUnroll = 4;

// true iff slot j of token t holds a valid expert index not used by an earlier slot
__device__ __forceinline__ bool slot_valid(const int32_t* idx_row, int j, int e, int N) {
  if (e < 0 || e >= N) return false;
  for (int j2 = 0; j2 < j; ++j2)
    if (idx_row[j2] == e) return false;
  return true;
}

__global__ void __launch_bounds__(kMaskThreads) dispatch_mask_kernel(const DispatchArgs a) {
  __shared__ uint32_t m[256];
  grid_dep_wait();
  grid_dep_launch();
  const int tid = threadIdx.x;
  const int N = a.N, k = a.k;
  for (int e = tid; e < N; e += kMaskThreads) m[e] = 0u;
  if (blockIdx.x == 0 && tid == 0) *a.ticket = 0u;
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kDispatchTokens;
  for (int s = tid; s < kDispatchTokens * k; s += kMaskThreads) {
    const int tl = s / k, j = s % k;
    const int64_t t = t0 + tl;
    if (t >= a.T) continue;
    const int32_t* row = a.topk_idx + t * k;
    const int e = row[j];
    if (!slot_valid(row, j, e, N)) {
      atomicOr(a.flags, kFlagBadIndex);
      continue;
    }
    atomicOr(&m[e], 1u << tl);
  }
  __syncthreads();
  for (int e = tid; e < N; e += kMaskThreads)
    a.mask[static_cast<int64_t>(blockIdx.x) * N + e] = m[e];
}

// grid: ceil(N / 32) blocks of 32 warps; lane = expert, warp = a run of blocks
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(const DispatchArgs a, int blocks) {
  __shared__ int part[32][33];
  __shared__ int is_last;
  __shared__ int kept_s[256];
  __shared__ int drop_s[256];
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  const int e = blockIdx.x * 32 + lane;
  const int chunk = (blocks + 31) / 32;
  const int b_lo = min(blocks, warp * chunk), b_hi = min(blocks, b_lo + chunk);

  int s = 0;
  if (e < N)
    for (int b = b_lo; b < b_hi; ++b) s += __popc(a.mask[static_cast<int64_t>(b) * N + e]);
  part[warp][lane] = s;
  __syncthreads();
  int excl = 0;
  for (int w = 0; w < warp; ++w) excl += part[w][lane];
  if (e < N) {
    int run = excl;
    for (int b = b_lo; b < b_hi; ++b) {
      a.base[static_cast<int64_t>(b) * N + e] = run;
      run += __popc(a.mask[static_cast<int64_t>(b) * N + e]);
    }
    if (warp == 31) a.counts[e] = run;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // last block: kept counts, aligned segment offsets, statistics
  for (int x = threadIdx.x; x < N; x += blockDim.x) {
    const int c = __ldcg(a.counts + x);
    const int kept = min(c, a.capacity);
    kept_s[x] = kept;
    drop_s[x] = c - kept;
    a.seg_count[x] = kept;
    if (a.stats.counts) a.stats.counts[x] = c;
    if (a.stats.kept) a.stats.kept[x] = kept;
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scan of the aligned segment sizes: 8 experts per lane, then a warp scan
    const int per = (N + 31) / 32;
    const int x_lo = min(N, lane * per), x_hi = min(N, x_lo + per);
    long long local = 0, drop = 0, kept_sum = 0;
    for (int x = x_lo; x < x_hi; ++x) {
      local += (kept_s[x] + a.align - 1) / a.align * static_cast<long long>(a.align);
      drop += drop_s[x];
      kept_sum += kept_s[x];
    }
    long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      drop += __shfl_xor_sync(0xffffffffu, drop, o);
      kept_sum += __shfl_xor_sync(0xffffffffu, kept_sum, o);
    }
    long long off = incl - local;
    for (int x = x_lo; x < x_hi; ++x) {
      a.seg_off[x] = static_cast<int32_t>(off);
      off += (kept_s[x] + a.align - 1) / a.align * static_cast<long long>(a.align);
    }
    if (lane == 31) a.seg_off[N] = static_cast<int32_t>(incl);
    if (lane == 0 && a.stats.num_dropped) a.stats.num_dropped[0] = static_cast<int32_t>(drop);
    if (lane == 0 && a.stats.avg_tokens_per_expert)
      a.stats.avg_tokens_per_expert[0] = static_cast<float>(static_cast<double>(kept_sum) / N);
  }
}

// One warp per token; a block covers 8 consecutive tokens of one 32-token mask
// block (small blocks keep several resident per SM).
__global__ void __launch_bounds__(kScatterThreads) dispatch_scatter_kernel(const DispatchArgs a) {
  __shared__ uint32_t m[256];
  __shared__ int base_s[256];
  __shared__ int off_s[256];
  __shared__ int rows_s[kScatterTokens][32];
  grid_dep_wait();
  grid_dep_launch();
  const int N = a.N, k = a.k;
  const int64_t t_first = static_cast<int64_t>(blockIdx.x) * kScatterTokens;
  const int64_t blk = t_first / kDispatchTokens;                      // mask block
  for (int e = threadIdx.x; e < N; e += kScatterThreads) {
    m[e] = a.mask[blk * N + e];
    base_s[e] = a.base[blk * N + e];
    off_s[e] = a.seg_off[e];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = t_first + warp;
  const int pos = static_cast<int>(t - blk * kDispatchTokens);        // bit of t in its mask word
  if (t >= a.T) return;

  if (lane < k) {
    const int32_t* row = a.topk_idx + t * k;
    const int e = row[lane];
    int r = -1;
    if (slot_valid(row, lane, e, N)) {
      const int rank = base_s[e] + __popc(m[e] & ((1u << pos) - 1u));
      if (rank < a.capacity) r = off_s[e] + rank;
    }
    a.row_map[t * k + lane] = r;
    rows_s[warp][lane] = r;
  }
  __syncwarp();

  // copy the row once from HBM, write it to each kept slot (16-byte vectors)
  const int64_t nvec = static_cast<int64_t>(a.d) * a.elem_bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.x) + t * nvec * 16);
  uint4* dst = static_cast<uint4*>(a.xp);
  for (int64_t c = lane; c < nvec; c += 32 * kCopyUnroll) {
    uint4 v[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u)
      if (c + 32 * u < nvec) v[u] = src[c + 32 * u];
    for (int j = 0; j < k; ++j) {
      const int r = rows_s[warp][j];
      if (r < 0) continue;
      uint4* drow = dst + static_cast<int64_t>(r) * nvec;
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u)
        if (c + 32 * u < nvec) drow[c + 32 * u] = v[u];
    }
  }
}

// The permutation as an index only: each kept slot's row gets its token number
// (row_token[row] = t) and nothing is copied; the grouped GEMM then gathers the
// token rows of x itself.  One block per 32-token mask block, one thread per
// (token, slot).
__global__ void __launch_bounds__(kMaskThreads) dispatch_index_kernel(const DispatchArgs a) {
  __shared__ uint32_t m[256];
  __shared__ int base_s[256];
  __shared__ int off_s[256];
  grid_dep_wait();
  grid_dep_launch();
  const int N = a.N, k = a.k;
  const int64_t blk = blockIdx.x;
  for (int e = threadIdx.x; e < N; e += kMaskThreads) {
    m[e] = a.mask[blk * N + e];
    base_s[e] = a.base[blk * N + e];
    off_s[e] = a.seg_off[e];
  }
  __syncthreads();
  const int64_t t0 = blk * kDispatchTokens;
  for (int s = threadIdx.x; s < kDispatchTokens * k; s += kMaskThreads) {
    const int pos = s / k, j = s % k;
    const int64_t t = t0 + pos;
    if (t >= a.T) break;
    const int32_t* row = a.topk_idx + t * k;
    const int e = row[j];
    int r = -1;
    if (slot_valid(row, j, e, N)) {
      const int rank = base_s[e] + __popc(m[e] & ((1u << pos) - 1u));
      if (rank < a.capacity) r = off_s[e] + rank;
    }
    a.row_map[t * k + j] = r;
    if (r >= 0) a.row_token[r] = static_cast<int32_t>(t);
  }
}

// The same permutation with the rows quantized on the way: block-scaled FP8
// (E4M3 codes, one E8M0 scale per 32 values of d, the smallest power of two
// that keeps the block within 448).  A warp reads its bf16 token row once;
// four lanes hold one block of 32 values (8 each), so the block maximum is two
// shuffles.  Codes go to every kept row, the scale byte to the tile-interleaved
// scale buffer of the rows.
__device__ __forceinline__ uint32_t e4m3x4_rn(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(kScatterThreads) dispatch_scatter_mx_kernel(const DispatchArgs a) {
  __shared__ uint32_t m[256];
  __shared__ int base_s[256];
  __shared__ int off_s[256];
  __shared__ int rows_s[kScatterTokens][32];
  grid_dep_wait();
  grid_dep_launch();
  const int N = a.N, k = a.k;
  const int64_t t_first = static_cast<int64_t>(blockIdx.x) * kScatterTokens;
  const int64_t blk = t_first / kDispatchTokens;
  for (int e = threadIdx.x; e < N; e += kScatterThreads) {
    m[e] = a.mask[blk * N + e];
    base_s[e] = a.base[blk * N + e];
    off_s[e] = a.seg_off[e];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = t_first + warp;
  const int pos = static_cast<int>(t - blk * kDispatchTokens);
  if (t >= a.T) return;

  if (lane < k) {
    const int32_t* row = a.topk_idx + t * k;
    const int e = row[lane];
    int r = -1;
    if (slot_valid(row, lane, e, N)) {
      const int rank = base_s[e] + __popc(m[e] & ((1u << pos) - 1u));
      if (rank < a.capacity) r = off_s[e] + rank;
    }
    a.row_map[t * k + lane] = r;
    rows_s[warp][lane] = r;
  }
  __syncwarp();

  const int d = a.d;
  const int nvec = d / 8;                          // 16-byte vectors (8 bf16) per row
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + t * d);
  uint8_t* codes = static_cast<uint8_t*>(a.xp);
  for (int c0 = 0; c0 < nvec; c0 += 32 * kQuantUnroll) {
    uint4 v[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int c = c0 + 32 * u + lane;
      v[u] = c < nvec ? src[c] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int c = c0 + 32 * u + lane;           // d % 32 == 0: a block's 4 lanes are all in or all out
      const float f[8] = {bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y), bf16_hi(v[u].y),
                          bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w), bf16_hi(v[u].w)};
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      if (c >= nvec) continue;
      const int ex = mx_exponent(amax);
      const float inv = mx_inv_scale(ex);
      const uint2 q = make_uint2(e4m3x4_rn(f[0] * inv, f[1] * inv, f[2] * inv, f[3] * inv),
                                 e4m3x4_rn(f[4] * inv, f[5] * inv, f[6] * inv, f[7] * inv));
      for (int j = 0; j < k; ++j) {
        const int r = rows_s[warp][j];
        if (r < 0) continue;
        *reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r) * d + 8 * c) = q;
        if ((lane & 3) == 0) a.xp_sf[mx_sf_offset(r, c / 4, d / 32)] = static_cast<uint8_t>(ex + 127);
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t s) {
  const int blocks = static_cast<int>((a.T + kDispatchTokens - 1) / kDispatchTokens);
  // each kernel may start while the one before it finishes (it waits for its
  // results first)
  cudaError_t e = launch_overlapped(dispatch_mask_kernel, dim3(blocks), dim3(kMaskThreads), 0, s, a);
  if (e == cudaSuccess)
    e = launch_overlapped(dispatch_scan_kernel, dim3((a.N + 31) / 32), dim3(1024), 0, s, a, blocks);
  if (e != cudaSuccess) return e;
  const unsigned sblocks = static_cast<unsigned>((a.T + kScatterTokens - 1) / kScatterTokens);
  if (a.row_token != nullptr)
    return launch_overlapped(dispatch_index_kernel, dim3(blocks), dim3(kMaskThreads), 0, s, a);
  if (a.xp_sf != nullptr)
    return launch_overlapped(dispatch_scatter_mx_kernel, dim3(sblocks), dim3(kScatterThreads), 0, s, a);
  return launch_overlapped(dispatch_scatter_kernel, dim3(sblocks), dim3(kScatterThreads), 0, s, a);
}

}  // namespace moe
