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

#include <algorithm>

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

// ---------------------------------------------------------------- router gradients
namespace {

constexpr int kColsumRows = 32;   // rows per block of the bias column sums

// Tensor-core path: sizes of the operand and partial buffers.
struct RgPlan {
  bool tc;
  int64_t T, Tp;        // Tp = T rounded up to 8 (16-byte rows of the transposed operand)
  int d, N, Np, Nk;     // Np = N rounded up to 8, Nk = N rounded up to 64
  int chunk, G;         // weight gradient: G row chunks of `chunk` rows (the last one ragged)
  int bias_blocks;      // column sums of dg: blocks of kColsumRows rows
  size_t parts, wpart, table, at, bt, bias, end;   // scratch offsets (bytes)
  int64_t cc_chunks;    // CUDA-core path: rows chunks of kChunkRows
};

size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

RgPlan rg_plan(int64_t T, int d, int N) {
  RgPlan P{};
  P.T = T;
  P.d = d;
  P.N = N;
  P.tc = N >= 64 && T >= 64;
  P.Tp = (T + 7) / 8 * 8;
  P.Np = (N + 7) / 8 * 8;
  P.Nk = (N + 63) / 64 * 64;
  P.chunk = static_cast<int>(std::max<int64_t>(1024, (T + 255) / 256 + 63) / 64 * 64);
  P.G = static_cast<int>((T + P.chunk - 1) / P.chunk);
  P.bias_blocks = static_cast<int>((T + kColsumRows - 1) / kColsumRows);
  P.cc_chunks = (T + kChunkRows - 1) / kChunkRows;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at_ = o;
    o = up(o + bytes, 256);
    return at_;
  };
  if (P.tc) {
    P.parts = take(2ull * T * P.Np * 2);                        // dg hi / lo, bf16 [2][T][Np]
    P.wpart = take(2ull * P.G * d * P.Np * 4);                  // fp32 [2][G][d][Np]
    P.table = take(4ull * (P.G + 1));                           // chunk row offsets
    P.at = take(3ull * P.Nk * P.Tp * 2);                        // [dg_hi^T; dg_hi^T; dg_lo^T] bf16
    P.bt = take(3ull * P.Nk * d * 2);                           // [W_hi^T; W_lo^T; W_hi^T] bf16
    P.bias = take(4ull * P.bias_blocks * N);                    // column sums of dg per kColsumRows rows
  } else {
    P.wpart = take(4ull * P.cc_chunks * (d + 1) * N);
  }
  P.end = o;
  return P;
}

__device__ __forceinline__ void split2(float v, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
  hi = *reinterpret_cast<const uint16_t*>(&h);
  lo = *reinterpret_cast<const uint16_t*>(&l);
}

// parts[0][t][i] = hi(dg[t][i]), parts[1][t][i] = lo(dg[t][i]); zero for N <= i < Np
__global__ void dg_split_kernel(int64_t T, int N, int Np, const float* __restrict__ dg, uint16_t* __restrict__ parts) {
  const int64_t total = T * Np;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = v / Np;
    const int i = static_cast<int>(v - t * Np);
    uint16_t hi = 0, lo = 0;
    if (i < N) split2(dg[t * N + i], hi, lo);
    parts[v] = hi;
    parts[total + v] = lo;
  }
}

// Transposed split of a fp32 [R, N] matrix into three stacked bf16 blocks of
// [Nk][Rp] (rows i >= N and columns r >= R zero): block b holds part
// (sel >> b) & 1 of src^T (0 = hi, 1 = lo).  32 x 32 tiles through shared memory.
__global__ void split_transpose_kernel(int64_t R, int64_t Rp, int N, int Nk, const float* __restrict__ src,
                                       uint16_t* __restrict__ out, int sel) {
  __shared__ float tile[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int i0 = blockIdx.y * 32;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int64_t r = r0 + y;
    const int i = i0 + threadIdx.x;
    tile[y][threadIdx.x] = (r < R && i < N) ? src[r * N + i] : 0.f;
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int i = i0 + y;
    const int64_t r = r0 + threadIdx.x;
    if (r >= Rp) continue;
    uint16_t hi, lo;
    split2(tile[threadIdx.x][y], hi, lo);
#pragma unroll
    for (int b = 0; b < 3; ++b) out[(static_cast<int64_t>(b) * Nk + i) * Rp + r] = ((sel >> b) & 1) ? lo : hi;
  }
}

__global__ void chunk_table_kernel(int G, int chunk, int64_t T, int32_t* __restrict__ table) {
  for (int g = threadIdx.x; g <= G; g += blockDim.x)
    table[g] = static_cast<int32_t>(static_cast<int64_t>(g) * chunk < T ? static_cast<int64_t>(g) * chunk : T);
}

// part[b][i] = sum of dg[t][i] over the kColsumRows rows of block b, in row order
__global__ void __launch_bounds__(256) dg_colsum_kernel(int64_t T, int N, const float* __restrict__ dg,
                                                        float* __restrict__ part) {
  const int i = threadIdx.x;
  if (i >= N) return;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kColsumRows;
  const int64_t t1 = t0 + kColsumRows < T ? t0 + kColsumRows : T;
  float s = 0.f;
  for (int64_t t = t0; t < t1; t += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = t + u < t1 ? dg[(t + u) * N + i] : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) s += v[u];
  }
  part[static_cast<int64_t>(blockIdx.x) * N + i] = s;
}

// dw[c][i] = sum over (part, chunk) of wpart[part][chunk][c][i] (parts outer, chunks
// inner); dbias[i] = sum over blocks of colsum[b][i]
__global__ void router_grad_reduce_kernel(int G, int d, int N, int Np, int bias_blocks, const float* __restrict__ wpart,
                                          const float* __restrict__ colsum, float* __restrict__ dw,
                                          float* __restrict__ dbias) {
  const int64_t total = static_cast<int64_t>(d) * N;
  const int64_t plane = static_cast<int64_t>(d) * Np;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total + N;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (v < total) {
      const int64_t c = v / N;
      const int i = static_cast<int>(v - c * N);
      float s = 0.f;
      for (int q = 0; q < 2 * G; ++q) s += wpart[q * plane + c * Np + i];
      dw[v] = s;
    } else if (dbias != nullptr) {
      const int i = static_cast<int>(v - total);
      float s = 0.f;
      for (int b = 0; b < bias_blocks; ++b) s += colsum[static_cast<int64_t>(b) * N + i];
      dbias[i] = s;
    }
  }
}

}  // namespace

size_t router_grad_scratch_bytes(int64_t T, int d, int N) { return rg_plan(T, d, N).end; }

int64_t router_dxr_rows(int64_t T) { return (T + 7) / 8 * 8; }

cudaError_t launch_router_grads(int64_t T, int d, int N, const uint16_t* x, const float* dg, const float* w_router,
                                float* dw_router, float* dbias, float* dxr, void* scratch, uint32_t* flags,
                                cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const RgPlan P = rg_plan(T, d, N);
  uint8_t* sc = static_cast<uint8_t*>(scratch);
  if (!P.tc) {
    const int chunks = static_cast<int>(P.cc_chunks);
    float* part = reinterpret_cast<float*>(sc + P.wpart);
    router_wgrad_kernel<<<dim3(static_cast<unsigned>(d / RT + 1), static_cast<unsigned>((N + RT - 1) / RT),
                               static_cast<unsigned>(chunks)),
                          256, 0, s>>>(T, d, N, x, dg, part);
    router_wgrad_reduce_kernel<<<256, 256, 0, s>>>(chunks, d, N, part, dw_router, dbias);
    router_dgrad_kernel<<<dim3(static_cast<unsigned>((T + RT - 1) / RT), static_cast<unsigned>((d + RT - 1) / RT)),
                          256, 0, s>>>(T, d, N, dg, w_router, dxr);
    return cudaGetLastError();
  }
  uint16_t* parts = reinterpret_cast<uint16_t*>(sc + P.parts);
  float* wpart = reinterpret_cast<float*>(sc + P.wpart);
  int32_t* table = reinterpret_cast<int32_t*>(sc + P.table);
  uint16_t* at_ = reinterpret_cast<uint16_t*>(sc + P.at);
  uint16_t* bt = reinterpret_cast<uint16_t*>(sc + P.bt);
  float* colsum = reinterpret_cast<float*>(sc + P.bias);
  const int sms = device_sm_count();

  // dW_r = x^T dg_hi + x^T dg_lo, per chunk of rows (fills the GPU), then the fixed-order sum
  dg_split_kernel<<<4 * sms, 256, 0, s>>>(T, N, P.Np, dg, parts);
  chunk_table_kernel<<<1, 256, 0, s>>>(P.G, P.chunk, T, table);
  dg_colsum_kernel<<<P.bias_blocks, 256, 0, s>>>(T, N, dg, colsum);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BwdGroups chunks{};
  chunks.G = P.G;
  chunks.max_rows = T;
  chunks.seg_off = table;
  chunks.flags = flags;
  for (int q = 0; q < 2 && e == cudaSuccess; ++q)
    e = launch_wgrad(chunks, d, P.Np, x, parts + static_cast<int64_t>(q) * T * P.Np,
                     wpart + static_cast<int64_t>(q) * P.G * d * P.Np, s);
  if (e != cudaSuccess) return e;
  router_grad_reduce_kernel<<<2 * sms, 256, 0, s>>>(P.G, d, N, P.Np, P.bias_blocks, wpart, colsum, dw_router, dbias);

  // dxr = dg W_r^T = [dg_hi | dg_hi | dg_lo] [W_hi | W_lo | W_hi]^T: one GEMM over 3 Nk stacked rows
  split_transpose_kernel<<<dim3(static_cast<unsigned>((P.Tp + 31) / 32), static_cast<unsigned>(P.Nk / 32)),
                           dim3(32, 8), 0, s>>>(T, P.Tp, N, P.Nk, dg, at_, 0b100);   // hi, hi, lo
  split_transpose_kernel<<<dim3(static_cast<unsigned>((d + 31) / 32), static_cast<unsigned>(P.Nk / 32)),
                           dim3(32, 8), 0, s>>>(d, d, N, P.Nk, w_router, bt, 0b010);   // hi, lo, hi
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BwdGroups stacked{};
  stacked.G = 1;
  stacked.dense_rows = 3 * P.Nk;
  stacked.max_rows = 3 * P.Nk;
  stacked.flags = flags;
  return launch_wgrad(stacked, static_cast<int>(P.Tp), d, at_, bt, dxr, s);
}

cudaError_t launch_dx_gather(int64_t T, int d, int k, const int32_t* row_map, const uint16_t* dXp, const float* dxr,
                             const uint16_t* dxs, uint16_t* dx, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  dx_gather_kernel<<<static_cast<unsigned>(T), kRowThreads, 0, s>>>(d, k, row_map, dXp, dxr, dxs, dx);
  return cudaGetLastError();
}

}  // namespace moe
