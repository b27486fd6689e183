// Router: g = x W_r (+ b) in fp32, scores = softmax(g) (max-subtracted, fp32),
// top-k of g with ties to the lower expert index, weights s_i / sum_topk s_j,
// plus per-block partials of the load-balance statistics.
//
// "MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §2.2 "Router 数学"
// (g = x W_r, scores = softmax(g), the top-k renormalised weights), §1 pain
// point 4 (router kept in fp32 against softmax 0/0), and for the statistics
// "负载均衡策略：MoE训练稳定性保障", section "辅助损失函数" (y_i, z_i).
//
// One kernel per token block: the GEMM tile is accumulated in registers
// (CUDA-core FFMA over smem tiles), written to a shared logits tile, then one
// warp per token does the softmax and the top-k by warp-shuffle reductions.
#include <math.h>

#include "device_utils.cuh"
#include "internal.h"

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
  float zw[kRouteThreads / 32][NP];
  int hist[NP];
};

template <int NP, bool FROM_LOGITS>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  using S = RouteSmem<NP>;
  constexpr int TX = S::TX, RT = S::RT, BT = S::BT;
  static_assert(BT == route_bt(NP), "route block size mismatch");
  static_assert(NP / TX == 8, "each thread owns 8 experts");
  __shared__ __align__(16) S sm;

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
    for (int v = tid; v < BT * NP; v += kRouteThreads) {
      const int r = v / NP, e = v % NP;
      float g = -INFINITY;
      if (e < N && t0 + r < T) g = a.logits_in[(t0 + r) * N + e];
      sm.u.lg[r][e] = g;
    }
    __syncthreads();
  }

  // ---------------- softmax + top-k, one warp per token ----------------
  constexpr int NPL = NP >= 32 ? NP / 32 : 1;  // logits held per lane
  const int warp = tid >> 5, lane = tid & 31;
  float zacc[NPL];
#pragma unroll
  for (int c = 0; c < NPL; ++c) zacc[c] = 0.f;

  for (int tl = warp; tl < BT; tl += kRouteThreads / 32) {
    const int64_t t = t0 + tl;
    if (t >= T) break;
    float v[NPL];
    bool bad = false;
#pragma unroll
    for (int c = 0; c < NPL; ++c) {
      const int e = lane + 32 * c;
      v[c] = e < NP ? sm.u.lg[tl][e] : -INFINITY;
      if (e < N && !isfinite(v[c])) bad = true;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.flags, kFlagNonfinite);

    float m = -INFINITY;
#pragma unroll
    for (int c = 0; c < NPL; ++c) m = fmaxf(m, v[c]);
    m = warp_max(m);
    float ex[NPL], sum = 0.f;
#pragma unroll
    for (int c = 0; c < NPL; ++c) {
      ex[c] = (lane + 32 * c < N) ? expf(v[c] - m) : 0.f;
      sum += ex[c];
    }
    sum = warp_sum(sum);
    float s[NPL];
#pragma unroll
    for (int c = 0; c < NPL; ++c) {
      s[c] = ex[c] / sum;
      zacc[c] += s[c];
      if (isnan(v[c])) v[c] = -INFINITY;  // out of contract; keeps the selection well defined
    }

    // top-k on the logits: k rounds of a warp arg-max, (larger value, lower index) first
    uint32_t taken = 0;
    int my_idx = 0;
    float my_s = 0.f, ssum = 0.f;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        const int e = lane + 32 * c;
        if (e < N && !((taken >> c) & 1u) && (v[c] > bv || (v[c] == bv && e < bi))) {
          bv = v[c];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      const int owner = bi & 31, slot = bi >> 5;
      float sv = 0.f;
      if (lane == owner) {
        taken |= 1u << slot;
#pragma unroll
        for (int c = 0; c < NPL; ++c)
          if (c == slot) sv = s[c];
      }
      sv = __shfl_sync(0xffffffffu, sv, owner);
      ssum += sv;
      if (lane == j) {
        my_idx = bi;
        my_s = sv;
      }
    }
    if (lane < k) {
      a.topk_idx[t * k + lane] = my_idx;
      a.topk_w[t * k + lane] = my_s / ssum;
      atomicAdd(&sm.hist[my_idx], 1);
    }
  }

#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    if (e < NP) sm.zw[warp][e] = zacc[c];
  }
  __syncthreads();
  for (int e = tid; e < N; e += kRouteThreads) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < kRouteThreads / 32; ++w) z += sm.zw[w][e];
    a.zpart[static_cast<int64_t>(blockIdx.x) * N + e] = z;
    a.hist[static_cast<int64_t>(blockIdx.x) * N + e] = sm.hist[e];
  }
}

// Column sums of the per-block partials, in a fixed order, and the L_aux
// scalars.  One warp per expert; lanes stride over the blocks.
__global__ void __launch_bounds__(1024) route_stats_kernel(const RouteStatsArgs a) {
  __shared__ double prod[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  for (int e = warp; e < N; e += 32) {
    long long cnt = 0;
    double z = 0.0;
    for (int b = lane; b < a.blocks; b += 32) {
      cnt += a.hist[static_cast<int64_t>(b) * N + e];
      z += static_cast<double>(a.zpart[static_cast<int64_t>(b) * N + e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      z += __shfl_xor_sync(0xffffffffu, z, o);
    }
    if (lane == 0) {
      const double y = a.T > 0 ? static_cast<double>(cnt) / (static_cast<double>(a.T) * a.k) : 0.0;
      const double zm = a.T > 0 ? z / static_cast<double>(a.T) : 0.0;
      if (a.stats.counts) a.stats.counts[e] = static_cast<int32_t>(cnt);
      if (a.stats.y_frac) a.stats.y_frac[e] = static_cast<float>(y);
      if (a.stats.z_mean) a.stats.z_mean[e] = static_cast<float>(zm);
      prod[e] = y * zm;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double acc = 0.0;
    for (int e = 0; e < N; ++e) acc += prod[e];
    if (a.stats.l_aux_p3) a.stats.l_aux_p3[0] = static_cast<float>(static_cast<double>(a.T) / N * acc);
    if (a.stats.l_aux_switch) a.stats.l_aux_switch[0] = static_cast<float>(N * acc);
  }
}

template <int NP>
cudaError_t launch_np(const RouteArgs& a, cudaStream_t s) {
  const int bt = route_bt(NP);
  const unsigned blocks = static_cast<unsigned>((a.T + bt - 1) / bt);
  if (a.logits_in != nullptr)
    route_kernel<NP, true><<<blocks, kRouteThreads, 0, s>>>(a);
  else
    route_kernel<NP, false><<<blocks, kRouteThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

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

cudaError_t launch_route_stats(const RouteStatsArgs& a, cudaStream_t s) {
  route_stats_kernel<<<1, 1024, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
