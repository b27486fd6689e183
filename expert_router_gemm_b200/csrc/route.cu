// Router: g = x W_r (+ b) in fp32, scores = softmax(g) (max-subtracted, fp32),
// top-k of g with ties to the lower expert index, weights s_i / sum_topk s_j,
// plus per-block partials of the load-balance statistics.
//
// "MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §2.2 "Router 数学"
// (g = x W_r, scores = softmax(g), the top-k renormalised weights), §1 pain
// point 4 (router kept in fp32 against softmax 0/0), and for the statistics
// "负载均衡策略：MoE训练稳定性保障", section "辅助损失函数" (y_i, z_i).
//
// One kernel per token block.  The logits tile comes either from a CUDA-core
// FFMA GEMM over shared-memory tiles (fp32 layers) or from the tensor-core
// router's split-K partial sums (bf16 layers: added in split order, then the
// bias); a warp then takes its tokens two to four at a time through the
// softmax (shuffle-tree sum, 32-bit reduction for the max) and the top-k (two
// 32-bit warp reductions per slot).
#include <math.h>

#include "device_utils.cuh"
#include "internal.h"
#include "route_dev.cuh"

namespace moe {
namespace {

constexpr int KC = 32;  // K slab of the router GEMM

template <int NP> struct RouteShape;
template <> struct RouteShape<8> { static constexpr int TX = 1, RT = 1; };
template <> struct RouteShape<16> { static constexpr int TX = 2, RT = 2; };
template <> struct RouteShape<32> { static constexpr int TX = 4, RT = 2; };
template <> struct RouteShape<64> { static constexpr int TX = 8, RT = 4; };
template <> struct RouteShape<128> { static constexpr int TX = 16, RT = 4; };
template <> struct RouteShape<256> { static constexpr int TX = 32, RT = 4; };

template <int NP>
struct RouteSmem {
  static constexpr int TX = RouteShape<NP>::TX;
  static constexpr int RT = RouteShape<NP>::RT;
  static constexpr int TY = kRouteThreads / TX;
  static constexpr int BT = TY * RT;
  union {
    struct {
      float xs[BT][KC + 4];  // rows padded to keep float4 reads conflict-free
      float ws[KC][NP];
    } g;
    float lg[BT][NP + 1];
  } u;
  RouteStatsSmem<NP, kRouteThreads / 32> st;
  int hist[NP];
};

// Tokens per block in logits mode (no GEMM tile to fill): small blocks keep
// every SM busy even when T is small or N has few experts, and give each SM
// enough warps to hide the latency of the per-token reductions (two tokens per
// warp: 16.9 us on the Qwen3-shaped router under ncu; one per warp: 19.0 us).
constexpr int kLogitsTokens = 16;

template <int NP, bool FROM_LOGITS>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  using S = RouteSmem<NP>;
  constexpr int TX = S::TX, RT = S::RT, BT = FROM_LOGITS ? kLogitsTokens : S::BT;
  static_assert(FROM_LOGITS || BT == route_bt(NP), "route block size mismatch");
  static_assert(BT <= S::BT, "the logits tile holds at most S::BT tokens");
  static_assert(NP / TX == 8, "each thread owns 8 experts");
  static_assert(BT >= kRouteMinBlockTokens, "z-loss partials are sized for kRouteMinBlockTokens-token blocks");
  __shared__ __align__(16) S sm;
  grid_dep_wait();   // the router GEMM's partial sums are complete
  grid_dep_launch();

  const int tid = threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * BT;
  const int N = a.N, d = a.d, k = a.k;
  const int64_t T = a.T;

  for (int e = tid; e < NP; e += kRouteThreads) sm.hist[e] = 0;

  if constexpr (!FROM_LOGITS) {
    // ---------------- router GEMM on CUDA cores ----------------
    const int tx = tid % TX, ty = tid / TX;
    float acc[RT][8];
#pragma unroll
    for (int q = 0; q < RT; ++q)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q][i] = 0.f;

    for (int k0 = 0; k0 < d; k0 += KC) {
      if (a.x_is_bf16) {
        const uint16_t* xb = static_cast<const uint16_t*>(a.x);
        for (int v = tid; v < BT * (KC / 8); v += kRouteThreads) {
          const int r = v / (KC / 8), c = (v % (KC / 8)) * 8;
          const int64_t t = t0 + r;
          uint4 q = make_uint4(0u, 0u, 0u, 0u);
          if (t < T && k0 + c < d) q = *reinterpret_cast<const uint4*>(xb + t * d + k0 + c);
          float4 lo = make_float4(bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y));
          float4 hi = make_float4(bf16_lo(q.z), bf16_hi(q.z), bf16_lo(q.w), bf16_hi(q.w));
          *reinterpret_cast<float4*>(&sm.u.g.xs[r][c]) = lo;
          *reinterpret_cast<float4*>(&sm.u.g.xs[r][c + 4]) = hi;
        }
      } else {
        const float* xf = static_cast<const float*>(a.x);
        for (int v = tid; v < BT * (KC / 4); v += kRouteThreads) {
          const int r = v / (KC / 4), c = (v % (KC / 4)) * 4;
          const int64_t t = t0 + r;
          float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
          if (t < T && k0 + c < d) q = *reinterpret_cast<const float4*>(xf + t * d + k0 + c);
          *reinterpret_cast<float4*>(&sm.u.g.xs[r][c]) = q;
        }
      }
      for (int v = tid; v < KC * NP; v += kRouteThreads) {
        const int kk = v / NP, e = v % NP;
        float w = 0.f;
        if (k0 + kk < d && e < N) w = a.w_router[static_cast<int64_t>(k0 + kk) * N + e];
        sm.u.g.ws[kk][e] = w;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < KC; kk += 4) {
        float4 xv[RT];
#pragma unroll
        for (int q = 0; q < RT; ++q) xv[q] = *reinterpret_cast<const float4*>(&sm.u.g.xs[ty * RT + q][kk]);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const float4 w0 = *reinterpret_cast<const float4*>(&sm.u.g.ws[kk + s][tx * 4]);
          const float4 w1 = *reinterpret_cast<const float4*>(&sm.u.g.ws[kk + s][NP / 2 + tx * 4]);
#pragma unroll
          for (int q = 0; q < RT; ++q) {
            const float xq = s == 0 ? xv[q].x : s == 1 ? xv[q].y : s == 2 ? xv[q].z : xv[q].w;
            acc[q][0] = fmaf(xq, w0.x, acc[q][0]);
            acc[q][1] = fmaf(xq, w0.y, acc[q][1]);
            acc[q][2] = fmaf(xq, w0.z, acc[q][2]);
            acc[q][3] = fmaf(xq, w0.w, acc[q][3]);
            acc[q][4] = fmaf(xq, w1.x, acc[q][4]);
            acc[q][5] = fmaf(xq, w1.y, acc[q][5]);
            acc[q][6] = fmaf(xq, w1.z, acc[q][6]);
            acc[q][7] = fmaf(xq, w1.w, acc[q][7]);
          }
        }
      }
      __syncthreads();
    }
    // logits tile (+ bias); padding experts get -inf
#pragma unroll
    for (int q = 0; q < RT; ++q)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = i < 4 ? tx * 4 + i : NP / 2 + tx * 4 + (i - 4);
        float v = acc[q][i];
        if (e < N) {
          if (a.bias != nullptr) v += a.bias[e];
        } else {
          v = -INFINITY;
        }
        sm.u.lg[ty * RT + q][e] = v;
      }
    __syncthreads();
    if (a.logits_out != nullptr) {
      for (int v = tid; v < BT * N; v += kRouteThreads) {
        const int r = v / N, e = v % N;
        if (t0 + r < T) a.logits_out[(t0 + r) * N + e] = sm.u.lg[r][e];
      }
    }
  } else {
    // logits = partial sums added in order (one for caller-supplied logits), + bias
    const int64_t pstride = T * N;
    if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(a.logits_in) & 15) == 0 &&
        (a.logits_out == nullptr || (reinterpret_cast<uintptr_t>(a.logits_out) & 15) == 0)) {
      // 16-byte vectors, every load of a thread issued before the adds (the
      // same additions, in the same order, as the scalar path below)
      const int nq = N >> 2;
#pragma unroll 4
      for (int v = tid; v < BT * nq; v += kRouteThreads) {
        const int r = v / nq, e = (v % nq) * 4;
        float4 g = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (t0 + r < T) {
          const float4* src = reinterpret_cast<const float4*>(a.logits_in + (t0 + r) * N + e);
          float4 part[kRouterMaxPartials];
#pragma unroll
          for (int z = 0; z < kRouterMaxPartials; ++z)
            if (z < a.n_partials) part[z] = src[z * (pstride >> 2)];
          g = part[0];
#pragma unroll
          for (int z = 1; z < kRouterMaxPartials; ++z)
            if (z < a.n_partials) {
              g.x += part[z].x;
              g.y += part[z].y;
              g.z += part[z].z;
              g.w += part[z].w;
            }
          if (a.bias != nullptr) {
            g.x += a.bias[e];
            g.y += a.bias[e + 1];
            g.z += a.bias[e + 2];
            g.w += a.bias[e + 3];
          }
          if (a.logits_out != nullptr) *reinterpret_cast<float4*>(a.logits_out + (t0 + r) * N + e) = g;
        }
        sm.u.lg[r][e] = g.x;
        sm.u.lg[r][e + 1] = g.y;
        sm.u.lg[r][e + 2] = g.z;
        sm.u.lg[r][e + 3] = g.w;
      }
      for (int v = tid; v < BT * (NP - N); v += kRouteThreads) sm.u.lg[v / (NP - N)][N + v % (NP - N)] = -INFINITY;
    } else {
      for (int v = tid; v < BT * NP; v += kRouteThreads) {
        const int r = v / NP, e = v % NP;
        float g = -INFINITY;
        if (e < N && t0 + r < T) {
          const float* src = a.logits_in + (t0 + r) * N + e;
          g = src[0];
          for (int z = 1; z < a.n_partials; ++z) g += src[z * pstride];
          if (a.bias != nullptr) g += a.bias[e];
          if (a.logits_out != nullptr) a.logits_out[(t0 + r) * N + e] = g;
        }
        sm.u.lg[r][e] = g;
      }
    }
    __syncthreads();
  }

  // ---------------- softmax + top-k, TPW tokens per warp at a time ----------------
  constexpr int NW = kRouteThreads / 32;
  constexpr int TPW = BT / NW < 4 ? BT / NW : 4;
  static_assert(TPW >= 1 && BT % (NW * TPW) == 0, "whole token groups per warp");
  const int warp = tid >> 5, lane = tid & 31;
  float zacc[RouteLane<NP>::NPL];
#pragma unroll
  for (int c = 0; c < RouteLane<NP>::NPL; ++c) zacc[c] = 0.f;
  double zl = 0.0;
  route_tokens<NP, NW, TPW>(a, &sm.u.lg[0][0], NP + 1, BT, t0, warp, lane, sm.hist, zacc, zl);
  if (!a.want_stats) return;
  route_stats<NP, NW>(a, sm.st, sm.hist, zacc, zl, warp, lane, tid, blockIdx.x, gridDim.x,
                      [] { __syncthreads(); });
}

__global__ void bias_update_kernel(float* b, const int32_t* counts, int64_t Tk, int N, float gamma) {
  const int i = threadIdx.x;
  if (i >= N) return;
  const int64_t diff = Tk - static_cast<int64_t>(N) * counts[i];
  const float sgn = diff > 0 ? 1.f : diff < 0 ? -1.f : 0.f;
  b[i] = __fadd_rn(b[i], gamma * sgn);  // gamma * sgn is exact: one rounding, as written
}

template <int NP>
cudaError_t launch_np(const RouteArgs& a, cudaStream_t s) {
  const int bt = a.logits_in != nullptr ? kLogitsTokens : route_bt(NP);
  const unsigned blocks = static_cast<unsigned>((a.T + bt - 1) / bt);
  // may start while the router GEMM before it finishes (it waits for its results first)
  if (a.logits_in != nullptr)
    return launch_overlapped(route_kernel<NP, true>, dim3(blocks), dim3(kRouteThreads), 0, s, a);
  return launch_overlapped(route_kernel<NP, false>, dim3(blocks), dim3(kRouteThreads), 0, s, a);
}

}  // namespace

cudaError_t launch_bias_update(float* b, const int32_t* counts, int64_t Tk, int N, float gamma, cudaStream_t s) {
  bias_update_kernel<<<1, 256, 0, s>>>(b, counts, Tk, N, gamma);
  return cudaGetLastError();
}

size_t router_zl_slots(int64_t T) { return static_cast<size_t>((T + kRouteMinBlockTokens - 1) / kRouteMinBlockTokens); }

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  switch (route_np(a.N)) {
    case 8: return launch_np<8>(a, s);
    case 16: return launch_np<16>(a, s);
    case 32: return launch_np<32>(a, s);
    case 64: return launch_np<64>(a, s);
    case 128: return launch_np<128>(a, s);
    default: return launch_np<256>(a, s);
  }
}

}  // namespace moe
