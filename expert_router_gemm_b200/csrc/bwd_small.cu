// The memory-bound and small steps of the layer backward.
//
// Gradient of L = <dy, y> + aux_weight * L_aux + z_weight * z_loss, where
// y = sum_j w_j o_j over the kept slots ("MoE 训练加速实战：DeepEP + Grouped
// GeMM + Aux-Loss-Free" §2.2 for y, §5.2 for the loss with the Switch auxiliary
// term N sum_i f_i P_i; "负载均衡策略：MoE训练稳定性保障", z_loss_weight):
//   combine_bwd:   dO[row] = w_tj dy_t,  dw_tj = <dy_t, o_row>  (0 for dropped)
//   router_bwd:    w_j = s_{e_j} / S over the k chosen experts ->
//                  ds_{e_j} = (dw_j - sum_j' dw_j' w_j') / S;
//                  ds_i += aux_weight N f_i / T  (P_i = mean_t s_ti, f_i a count);
//                  dg = s * (ds - <ds, s>) + z_weight (2 / T) lse s
//   router_wgrad:  dW_r = x^T dg, dbias = sum_t dg_t   (fp32, chunked over T,
//                  chunk partials added in a fixed order)
//   router_dgrad:  dxr = dg W_r^T (fp32)
//   dx_gather:     dx_t = sum_j dXp[row_tj] + dxr_t (+ dxs_t), one rounding
//   zero_pad_rows: the padding rows of expert segments (read by the weight-
//                  gradient GEMMs, which reduce over whole padded segments)
// All reductions run in a fixed order: results are deterministic.
#include <math.h>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRowThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x < 32) {
    s = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0.f;
    s = warp_sum(s);
  }
  return s;  // valid in thread 0
}

// one block per token
__global__ void __launch_bounds__(kRowThreads) combine_bwd_kernel(const BwdSmallArgs a) {
  __shared__ float red[32];
  const int64_t t = blockIdx.x;
  const int d = a.d, k = a.k;
  const int nvec = d / 8;
  const uint4* dyv = reinterpret_cast<const uint4*>(a.dy + t * d);
  for (int j = 0; j < k; ++j) {
    const int r = a.row_map[t * k + j];
    if (r < 0) {
      if (threadIdx.x == 0) a.dw[t * k + j] = 0.f;
      continue;
    }
    const float w = a.topk_w[t * k + j];
    const uint4* ov = reinterpret_cast<const uint4*>(a.out_rows + static_cast<int64_t>(r) * d);
    uint4* dov = reinterpret_cast<uint4*>(a.dO + static_cast<int64_t>(r) * d);
    float dot = 0.f;
    for (int c = threadIdx.x; c < nvec; c += kRowThreads) {
      const uint4 y4 = dyv[c], o4 = ov[c];
      const float yv[8] = {bf16_lo(y4.x), bf16_hi(y4.x), bf16_lo(y4.y), bf16_hi(y4.y),
                           bf16_lo(y4.z), bf16_hi(y4.z), bf16_lo(y4.w), bf16_hi(y4.w)};
      const float ovv[8] = {bf16_lo(o4.x), bf16_hi(o4.x), bf16_lo(o4.y), bf16_hi(o4.y),
                            bf16_lo(o4.z), bf16_hi(o4.z), bf16_lo(o4.w), bf16_hi(o4.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(yv[i], ovv[i], dot);
      dov[c] = make_uint4(pack_bf16x2(w * yv[0], w * yv[1]), pack_bf16x2(w * yv[2], w * yv[3]),
                          pack_bf16x2(w * yv[4], w * yv[5]), pack_bf16x2(w * yv[6], w * yv[7]));
    }
    dot = block_sum(dot, red);
    if (threadIdx.x == 0) a.dw[t * k + j] = dot;
  }
}

// one warp per token; lane j holds slot j, lane l holds experts l, l+32, ...
template <int NPL>
__global__ void __launch_bounds__(kRowThreads) router_bwd_kernel(const BwdSmallArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * (kRowThreads / 32) + warp;
  if (t >= a.T) return;
  const int N = a.N, k = a.k;
  const float* g = a.logits + t * N;
  float gv[NPL];
  float m = -INFINITY;
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    gv[c] = e < N ? g[e] : -INFINITY;
    m = fmaxf(m, gv[c]);
  }
  m = warp_max(m);
  float sum = 0.f, s[NPL];
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    s[c] = e < N ? expf(gv[c] - m) : 0.f;
    sum += s[c];
  }
  sum = warp_sum(sum);
#pragma unroll
  for (int c = 0; c < NPL; ++c) s[c] /= sum;
  const float lse = m + logf(sum);

  // slots: lane j < k
  int ej = -1;
  float wj = 0.f, dwj = 0.f, sj = 0.f;
  if (lane < k) {
    ej = a.topk_idx[t * k + lane];
    wj = a.topk_w[t * k + lane];
    dwj = a.dw[t * k + lane];
    sj = expf(g[ej] - m) / sum;
  }
  const float S = warp_sum(sj);
  const float dww = warp_sum(dwj * wj);
  const float ds_sel = lane < k ? (dwj - dww) / S : 0.f;

  const float aux_c = a.aux_weight * static_cast<float>(N) / (static_cast<float>(a.T) * static_cast<float>(a.T) * k);
  float ds[NPL];
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    ds[c] = e < N ? aux_c * static_cast<float>(a.counts[e]) : 0.f;   // aux_weight N f_e / T
  }
  for (int j = 0; j < k; ++j) {
    const int e = __shfl_sync(0xffffffffu, ej, j);
    const float v = __shfl_sync(0xffffffffu, ds_sel, j);
#pragma unroll
    for (int c = 0; c < NPL; ++c)
      if (lane + 32 * c == e) ds[c] += v;
  }
  float dot = 0.f;
#pragma unroll
  for (int c = 0; c < NPL; ++c) dot = fmaf(ds[c], s[c], dot);
  dot = warp_sum(dot);
  const float zc = a.z_weight * 2.0f / static_cast<float>(a.T) * lse;
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    if (e < N) a.dg[t * N + e] = s[c] * (ds[c] - dot) + zc * s[c];
  }
}

// grid (N experts, n_buf): zero the padding rows of each expert segment
__global__ void zero_pad_rows_kernel(const int32_t* seg_off, const int32_t* seg_count, const PadBufs bufs) {
  const int e = blockIdx.x, b = blockIdx.y;
  const int64_t r0 = seg_off[e] + seg_count[e], r1 = seg_off[e + 1];
  const int nvec = bufs.cols[b] / 8;
  uint4* base = static_cast<uint4*>(bufs.buf[b]);
  for (int64_t r = r0; r < r1; ++r)
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) base[r * nvec + c] = make_uint4(0u, 0u, 0u, 0u);
}

// ---------------------------------------------------------------- router GEMMs (CUDA cores)
constexpr int RT = 64;        // output tile
constexpr int RK = 32;        // reduction slab
constexpr int kChunkRows = 512;  // rows of T per partial of the weight gradient

// partial[z][c][i] = sum_{t in chunk z} x[t][c] dg[t][i]; row c = d of the
// partial holds sum_t dg[t][i] (the bias), computed as x = 1.
__global__ void __launch_bounds__(256) router_wgrad_kernel(int64_t T, int d, int N, const uint16_t* __restrict__ x,
                                                          const float* __restrict__ dg, float* __restrict__ part) {
  __shared__ __align__(16) float xs[RK][RT + 4];
  __shared__ __align__(16) float gs[RK][RT + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads, 4 x 4 outputs each
  const int c0 = blockIdx.x * RT, i0 = blockIdx.y * RT;
  const bool bias_tile = c0 >= d;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.z) * kChunkRows;
  const int64_t t_end = t_begin + kChunkRows < T ? t_begin + kChunkRows : T;
  float acc[4][4] = {};
  for (int64_t tb = t_begin; tb < t_end; tb += RK) {
    for (int v = threadIdx.x; v < RK * RT; v += 256) {
      const int r = v / RT, c = v % RT;
      const int64_t t = tb + r;
      float xv = 0.f, gv = 0.f;
      if (t < t_end) {
        if (bias_tile)
          xv = c == 0 ? 1.f : 0.f;
        else if (c0 + c < d)
          xv = __uint_as_float(static_cast<uint32_t>(x[t * d + c0 + c]) << 16);
        if (i0 + c < N) gv = dg[t * N + i0 + c];
      }
      xs[r][c] = xv;
      gs[r][c] = gv;
    }
    __syncthreads();
#pragma unroll 8
    for (int r = 0; r < RK; ++r) {
      const float4 x4 = *reinterpret_cast<const float4*>(&xs[r][ty * 4]);
      const float4 g4 = *reinterpret_cast<const float4*>(&gs[r][tx * 4]);
      const float xa[4] = {x4.x, x4.y, x4.z, x4.w};
      const float ga[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xa[a], ga[b], acc[a][b]);
    }
    __syncthreads();
  }
  float* pz = part + static_cast<int64_t>(blockIdx.z) * (d + 1) * N;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int c = c0 + ty * 4 + a;
    if (c > d || (bias_tile && c != d)) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = i0 + tx * 4 + b;
      if (i < N) pz[static_cast<int64_t>(c) * N + i] = acc[a][b];
    }
  }
}

__global__ void router_wgrad_reduce_kernel(int n_chunks, int d, int N, const float* __restrict__ part,
                                           float* __restrict__ dw, float* __restrict__ dbias) {
  const int64_t total = static_cast<int64_t>(d + 1) * N;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < n_chunks; ++z) s += part[z * total + v];
    if (v < static_cast<int64_t>(d) * N)
      dw[v] = s;
    else if (dbias != nullptr)
      dbias[v - static_cast<int64_t>(d) * N] = s;
  }
}

// The same two products for wide routers (N > 64) with 128 x 128 output tiles:
// 256 threads, each an 8 x 8 register tile (rows {4ty + a, 64 + 4ty + a} and
// columns {4tx + b, 64 + 4tx + b}, a, b < 4), so that every 64 FMAs read four
// 16-byte words of shared memory.  Reduction slabs of 16.
constexpr int WT = 128;
constexpr int WK = 16;
constexpr int WP = WT + 4;   // padded smem row (floats): 16-byte aligned rows

__device__ __forceinline__ void tile_fma_8x8(const float (*as)[WP], const float (*bs)[WP], int tx, int ty,
                                             float (&acc)[8][8]) {
#pragma unroll 4
  for (int r = 0; r < WK; ++r) {
    const float4 a0 = *reinterpret_cast<const float4*>(&as[r][ty * 4]);
    const float4 a1 = *reinterpret_cast<const float4*>(&as[r][64 + ty * 4]);
    const float4 b0 = *reinterpret_cast<const float4*>(&bs[r][tx * 4]);
    const float4 b1 = *reinterpret_cast<const float4*>(&bs[r][64 + tx * 4]);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
  }
}

__device__ __forceinline__ int tile_row(int ty, int a) { return a < 4 ? ty * 4 + a : 64 + ty * 4 + (a - 4); }

// partial[z][c][i] = sum_{t in chunk z} x[t][c] dg[t][i] for c <= d (row d: x = 1,
// the bias gradient)
__global__ void __launch_bounds__(256) router_wgrad_wide_kernel(int64_t T, int d, int N, const uint16_t* __restrict__ x,
                                                               const float* __restrict__ dg,
                                                               float* __restrict__ part) {
  __shared__ __align__(16) float xs[WK][WP];
  __shared__ __align__(16) float gs[WK][WP];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int c0 = blockIdx.x * WT, i0 = blockIdx.y * WT;
  const int64_t t_begin = static_cast<int64_t>(blockIdx.z) * kChunkRows;
  const int64_t t_end = t_begin + kChunkRows < T ? t_begin + kChunkRows : T;
  float acc[8][8] = {};
  for (int64_t tb = t_begin; tb < t_end; tb += WK) {
#pragma unroll
    for (int u = 0; u < WK * WT / 256; ++u) {   // one row of 128 per 128 threads: coalesced
      const int v = threadIdx.x + 256 * u;
      const int r = v / WT, c = v % WT;
      const int64_t t = tb + r;
      float xv = 0.f, gv = 0.f;
      if (t < t_end) {
        if (c0 + c < d)
          xv = __uint_as_float(static_cast<uint32_t>(x[t * d + c0 + c]) << 16);
        else if (c0 + c == d)
          xv = 1.f;
        if (i0 + c < N) gv = dg[t * N + i0 + c];
      }
      xs[r][c] = xv;
      gs[r][c] = gv;
    }
    __syncthreads();
    tile_fma_8x8(xs, gs, tx, ty, acc);
    __syncthreads();
  }
  float* pz = part + static_cast<int64_t>(blockIdx.z) * (d + 1) * N;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int c = c0 + tile_row(ty, a);
    if (c > d) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int i = i0 + tile_row(tx, b);
      if (i < N) pz[static_cast<int64_t>(c) * N + i] = acc[a][b];
    }
  }
}

// dxr[t][c] = sum_i dg[t][i] W_r[c][i]
__global__ void __launch_bounds__(256) router_dgrad_wide_kernel(int64_t T, int d, int N, const float* __restrict__ dg,
                                                               const float* __restrict__ wr,
                                                               float* __restrict__ dxr) {
  __shared__ __align__(16) float gs[WK][WP];   // [i][t]
  __shared__ __align__(16) float ws[WK][WP];   // [i][c]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * WT;
  const int c0 = blockIdx.y * WT;
  float acc[8][8] = {};
  for (int ib = 0; ib < N; ib += WK) {
#pragma unroll
    for (int u = 0; u < WK * WT / 256; ++u) {   // i fastest: 64-byte pieces of the rows of dg and W_r
      const int v = threadIdx.x + 256 * u;
      const int r = v / WK, i = v % WK;
      const int64_t t = t0 + r;
      const int c = c0 + r;
      gs[i][r] = (t < T && ib + i < N) ? dg[t * N + ib + i] : 0.f;
      ws[i][r] = (c < d && ib + i < N) ? wr[static_cast<int64_t>(c) * N + ib + i] : 0.f;
    }
    __syncthreads();
    tile_fma_8x8(gs, ws, tx, ty, acc);
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int64_t t = t0 + tile_row(ty, a);
    if (t >= T) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int c = c0 + tile_row(tx, b);
      if (c < d) dxr[t * d + c] = acc[a][b];
    }
  }
}

// dxr[t][c] = sum_i dg[t][i] W_r[c][i]
__global__ void __launch_bounds__(256) router_dgrad_kernel(int64_t T, int d, int N, const float* __restrict__ dg,
                                                          const float* __restrict__ wr, float* __restrict__ dxr) {
  __shared__ __align__(16) float gs[RK][RT + 4];   // [i][t]
  __shared__ __align__(16) float ws[RK][RT + 4];   // [i][c]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * RT;
  const int c0 = blockIdx.y * RT;
  float acc[4][4] = {};
  for (int ib = 0; ib < N; ib += RK) {
    for (int v = threadIdx.x; v < RK * RT; v += 256) {
      const int r = v / RK, i = v % RK;   // i fastest: coalesced along the rows of dg and W_r
      const int64_t t = t0 + r;
      const int c = c0 + r;
      gs[i][r] = (t < T && ib + i < N) ? dg[t * N + ib + i] : 0.f;
      ws[i][r] = (c < d && ib + i < N) ? wr[static_cast<int64_t>(c) * N + ib + i] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int i = 0; i < RK; ++i) {
      const float4 g4 = *reinterpret_cast<const float4*>(&gs[i][ty * 4]);
      const float4 w4 = *reinterpret_cast<const float4*>(&ws[i][tx * 4]);
      const float ga[4] = {g4.x, g4.y, g4.z, g4.w};
      const float wa[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(ga[a], wa[b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t t = t0 + ty * 4 + a;
    if (t >= T) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int c = c0 + tx * 4 + b;
      if (c < d) dxr[t * d + c] = acc[a][b];
    }
  }
}

// one block per token: dx = sum of the kept slots' dXp rows + dxr (+ dxs)
__global__ void __launch_bounds__(kRowThreads) dx_gather_kernel(int d, int k, const int32_t* __restrict__ row_map,
                                                                const uint16_t* __restrict__ dXp,
                                                                const float* __restrict__ dxr,
                                                                const uint16_t* __restrict__ dxs,
                                                                uint16_t* __restrict__ dx) {
  const int64_t t = blockIdx.x;
  const int nvec = d / 8;
  for (int c = threadIdx.x; c < nvec; c += kRowThreads) {
    float acc[8];
    const float4* r4 = reinterpret_cast<const float4*>(dxr + t * d + 8 * c);
    const float4 p0 = r4[0], p1 = r4[1];
    acc[0] = p0.x;
    acc[1] = p0.y;
    acc[2] = p0.z;
    acc[3] = p0.w;
    acc[4] = p1.x;
    acc[5] = p1.y;
    acc[6] = p1.z;
    acc[7] = p1.w;
    for (int j = 0; j < k; ++j) {
      const int r = row_map[t * k + j];
      if (r < 0) continue;
      const uint4 v = reinterpret_cast<const uint4*>(dXp + static_cast<int64_t>(r) * d)[c];
      acc[0] += bf16_lo(v.x);
      acc[1] += bf16_hi(v.x);
      acc[2] += bf16_lo(v.y);
      acc[3] += bf16_hi(v.y);
      acc[4] += bf16_lo(v.z);
      acc[5] += bf16_hi(v.z);
      acc[6] += bf16_lo(v.w);
      acc[7] += bf16_hi(v.w);
    }
    if (dxs != nullptr) {
      const uint4 v = reinterpret_cast<const uint4*>(dxs + t * d)[c];
      acc[0] += bf16_lo(v.x);
      acc[1] += bf16_hi(v.x);
      acc[2] += bf16_lo(v.y);
      acc[3] += bf16_hi(v.y);
      acc[4] += bf16_lo(v.z);
      acc[5] += bf16_hi(v.z);
      acc[6] += bf16_lo(v.w);
      acc[7] += bf16_hi(v.w);
    }
    reinterpret_cast<uint4*>(dx + t * d)[c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                         pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace

cudaError_t launch_combine_bwd(const BwdSmallArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  combine_bwd_kernel<<<static_cast<unsigned>(a.T), kRowThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const BwdSmallArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((a.T + 7) / 8);
  switch ((a.N + 31) / 32) {
    case 1: router_bwd_kernel<1><<<blocks, kRowThreads, 0, s>>>(a); break;
    case 2: router_bwd_kernel<2><<<blocks, kRowThreads, 0, s>>>(a); break;
    case 3:
    case 4: router_bwd_kernel<4><<<blocks, kRowThreads, 0, s>>>(a); break;
    default: router_bwd_kernel<8><<<blocks, kRowThreads, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_zero_pad_rows(int N, const int32_t* seg_off, const int32_t* seg_count, const PadBufs& b,
                                 cudaStream_t s) {
  if (b.n <= 0) return cudaSuccess;
  zero_pad_rows_kernel<<<dim3(static_cast<unsigned>(N), static_cast<unsigned>(b.n)), 256, 0, s>>>(seg_off, seg_count,
                                                                                                 b);
  return cudaGetLastError();
}

size_t router_wgrad_scratch_floats(int64_t T, int d, int N) {
  const int64_t chunks = (T + kChunkRows - 1) / kChunkRows;
  return static_cast<size_t>(chunks) * (d + 1) * N;
}

cudaError_t launch_router_wgrad(int64_t T, int d, int N, const uint16_t* x, const float* dg, float* dw_router,
                                float* dbias, float* scratch, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int chunks = static_cast<int>((T + kChunkRows - 1) / kChunkRows);
  if (N > 64) {
    router_wgrad_wide_kernel<<<dim3(static_cast<unsigned>(d / WT + 1), static_cast<unsigned>((N + WT - 1) / WT),
                                    static_cast<unsigned>(chunks)),
                               256, 0, s>>>(T, d, N, x, dg, scratch);
    router_wgrad_reduce_kernel<<<256, 256, 0, s>>>(chunks, d, N, scratch, dw_router, dbias);
    return cudaGetLastError();
  }
  router_wgrad_kernel<<<dim3(static_cast<unsigned>(d / RT + 1), static_cast<unsigned>((N + RT - 1) / RT),
                             static_cast<unsigned>(chunks)),
                        256, 0, s>>>(T, d, N, x, dg, scratch);
  router_wgrad_reduce_kernel<<<256, 256, 0, s>>>(chunks, d, N, scratch, dw_router, dbias);
  return cudaGetLastError();
}

cudaError_t launch_router_dgrad(int64_t T, int d, int N, const float* dg, const float* w_router, float* dxr,
                                cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (N > 64) {
    router_dgrad_wide_kernel<<<dim3(static_cast<unsigned>((T + WT - 1) / WT), static_cast<unsigned>((d + WT - 1) / WT)),
                               256, 0, s>>>(T, d, N, dg, w_router, dxr);
    return cudaGetLastError();
  }
  router_dgrad_kernel<<<dim3(static_cast<unsigned>((T + RT - 1) / RT), static_cast<unsigned>((d + RT - 1) / RT)), 256,
                        0, s>>>(T, d, N, dg, w_router, dxr);
  return cudaGetLastError();
}

cudaError_t launch_dx_gather(int64_t T, int d, int k, const int32_t* row_map, const uint16_t* dXp, const float* dxr,
                             const uint16_t* dxs, uint16_t* dx, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  dx_gather_kernel<<<static_cast<unsigned>(T), kRowThreads, 0, s>>>(d, k, row_map, dXp, dxr, dxs, dx);
  return cudaGetLastError();
}

}  // namespace moe
