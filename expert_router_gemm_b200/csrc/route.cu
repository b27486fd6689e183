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
  double zl[kRouteThreads / 32];
  int hist[NP];
};

// Monotone map of a float to an unsigned key (larger float -> larger key; -0.0
// maps like +0.0) and back.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Tokens per block in logits mode (no GEMM tile to fill): small blocks keep
// every SM busy even when T is small or N has few experts, and give each SM
// enough warps to hide the latency of the per-token reductions.
constexpr int kLogitsTokens = 16;

template <int NP, bool FROM_LOGITS>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  using S = RouteSmem<NP>;
  constexpr int TX = S::TX, RT = S::RT, BT = FROM_LOGITS ? kLogitsTokens : S::BT;
  static_assert(FROM_LOGITS || BT == route_bt(NP), "route block size mismatch");
  static_assert(BT <= S::BT, "the logits tile holds at most S::BT tokens");
  static_assert(NP / TX == 8, "each thread owns 8 experts");
  static_assert(BT >= kRouteMinBlockTokens, "z-loss partials are sized for 16-token blocks");
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
  // The TPW tokens of a warp are processed in lock step so that their shuffle
  // reductions overlap.
  constexpr int NPL = NP >= 32 ? NP / 32 : 1;  // logits held per lane
  constexpr int NW = kRouteThreads / 32;
  constexpr int TPW = BT / NW < 4 ? BT / NW : 4;
  static_assert(TPW >= 1 && BT % (NW * TPW) == 0, "whole token groups per warp");
  const int warp = tid >> 5, lane = tid & 31;
  float zacc[NPL];
#pragma unroll
  for (int c = 0; c < NPL; ++c) zacc[c] = 0.f;
  double zl = 0.0;  // this warp's sum of logsumexp^2 (every lane holds the same value)
  // Aux-Loss-Free selection bias of the lane's experts (0 where there is none)
  const bool biased = a.sel_bias != nullptr;
  float sb[NPL];
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    sb[c] = (biased && e < N) ? a.sel_bias[e] : 0.f;
  }

  for (int tl0 = warp * TPW; tl0 < BT; tl0 += NW * TPW) {
    float v[TPW][NPL], s[TPW][NPL];
    bool valid[TPW];
    bool bad = false;
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      valid[q] = tl0 + q < BT && t0 + tl0 + q < T;
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        const int e = lane + 32 * c;
        v[q][c] = (valid[q] && e < NP) ? sm.u.lg[tl0 + q][e] : -INFINITY;
        if (valid[q] && e < N && !isfinite(v[q][c])) bad = true;
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.flags, kFlagNonfinite);

    // max of the token's logits: one 32-bit reduction of the order-preserving
    // keys of the lanes' maxima (NaN is out of contract and counts as -inf)
    float m[TPW], sum[TPW];
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      float lm = -INFINITY;
#pragma unroll
      for (int c = 0; c < NPL; ++c) lm = fmaxf(lm, v[q][c]);
      if (isnan(lm)) lm = -INFINITY;
      m[q] = key_value(__reduce_max_sync(0xffffffffu, order_key(lm)));
    }
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      sum[q] = 0.f;
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        s[q][c] = (valid[q] && lane + 32 * c < N) ? expf(v[q][c] - m[q]) : 0.f;
        sum[q] += s[q][c];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int q = 0; q < TPW; ++q) sum[q] += __shfl_xor_sync(0xffffffffu, sum[q], o);
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      if (valid[q]) {
        const float lse = m[q] + logf(sum[q]);  // log-partition of the unbiased logits
        zl += static_cast<double>(lse) * lse;
        const float inv = 1.f / sum[q];
#pragma unroll
        for (int c = 0; c < NPL; ++c) zacc[c] += s[q][c] * inv;
      }
#pragma unroll
      for (int c = 0; c < NPL; ++c)
        if (isnan(v[q][c])) v[q][c] = -INFINITY;  // out of contract; keeps the selection defined
    }

    // top-k on the logits (plus the selection bias, in fp32, when there is
    // one): larger score first, ties to the lower expert index.  A lane holds
    // the order-preserving 32-bit keys of its experts' scores (-0.0 taken as
    // +0.0, so equal scores tie; 0 for padding experts, below every score),
    // sorted, with the slot numbers c (expert lane + 32 c) packed 3 bits each.
    // A round's winner is the warp max of the leading keys, then among the
    // lanes holding it the lowest expert index: two 32-bit reductions.  The
    // winning lane drops its head; lane j keeps the winner of round j.
    uint32_t hk[TPW][NPL], cpk[TPW];
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      int cs[NPL];
#pragma unroll
      for (int c = 0; c < NPL; ++c) {
        const int e = lane + 32 * c;
        hk[q][c] = e < N ? order_key(biased ? v[q][c] + sb[c] : v[q][c]) : 0u;
        cs[c] = c;
      }
#pragma unroll
      for (int i = 1; i < NPL; ++i)
#pragma unroll
        for (int j2 = i; j2 > 0; --j2)
          if (hk[q][j2] > hk[q][j2 - 1]) {  // strict: equal keys keep the lower c first
            const uint32_t th = hk[q][j2];
            hk[q][j2] = hk[q][j2 - 1];
            hk[q][j2 - 1] = th;
            const int tc = cs[j2];
            cs[j2] = cs[j2 - 1];
            cs[j2 - 1] = tc;
          }
      cpk[q] = 0u;
#pragma unroll
      for (int c = 0; c < NPL; ++c) cpk[q] |= static_cast<uint32_t>(cs[c]) << (3 * c);
    }
    uint32_t won_h[TPW], won_e[TPW];
#pragma unroll
    for (int q = 0; q < TPW; ++q) won_h[q] = won_e[q] = 0u;
    for (int j = 0; j < k; ++j) {
#pragma unroll
      for (int q = 0; q < TPW; ++q) {
        const uint32_t h = hk[q][0];
        const uint32_t hmax = __reduce_max_sync(0xffffffffu, h);
        const uint32_t inv_e = 0xFFFFFFFFu - static_cast<uint32_t>(lane + 32 * (cpk[q] & 7u));
        const uint32_t emax = __reduce_max_sync(0xffffffffu, h == hmax ? inv_e : 0u);
        if (h == hmax && inv_e == emax) {  // keys are unique: exactly one lane drops its head
#pragma unroll
          for (int c = 0; c + 1 < NPL; ++c) hk[q][c] = hk[q][c + 1];
          hk[q][NPL - 1] = 0u;
          cpk[q] >>= 3;
        }
        if (lane == j) {
          won_h[q] = hmax;
          won_e[q] = 0xFFFFFFFFu - emax;
        }
      }
    }
    // Lane j < k: the weight of slot j, s_e / sum of the k chosen s (summed in
    // slot order), from the unbiased logit with the softmax's own expression.
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      const int e = static_cast<int>(won_e[q]);
      float sv = 0.f;
      if (lane < k) {
        const float ve = biased ? sm.u.lg[tl0 + q][e] : key_value(won_h[q]);
        sv = expf(ve - m[q]) / sum[q];
      }
      float ssum = __shfl_sync(0xffffffffu, sv, 0);
      for (int j = 1; j < k; ++j) ssum += __shfl_sync(0xffffffffu, sv, j);
      if (valid[q] && lane < k) {
        const int64_t t = t0 + tl0 + q;
        a.topk_idx[t * k + lane] = e;
        a.topk_w[t * k + lane] = sv / ssum;
        if (a.want_stats) atomicAdd(&sm.hist[e], 1);
      }
    }
  }
  if (!a.want_stats) return;

  // ---------------- load-balance statistics ----------------
  // Block partials (fixed-order fp32 sum of the block's softmax scores, integer
  // counts) go to global accumulators with integer atomics: the z sums as fixed
  // point with 32 fraction bits, so the totals do not depend on block order.
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    if (e < NP) sm.zw[warp][e] = zacc[c];
  }
  if (lane == 0) sm.zl[warp] = zl;
  __syncthreads();
  for (int e = tid; e < N; e += kRouteThreads) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) z += sm.zw[w][e];
    atomicAdd(a.z_acc + e, static_cast<unsigned long long>(__double2ull_rn(static_cast<double>(z) * 4294967296.0)));
    if (sm.hist[e] != 0) atomicAdd(a.cnt_acc + e, sm.hist[e]);
  }
  if (tid == 0) {  // the block's z-loss partial, summed over its warps in order
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < NW; ++w) t += sm.zl[w];
    a.zl_part[blockIdx.x] = t;
  }
  __threadfence();
  __syncthreads();
  __shared__ int is_last;
  if (tid == 0) is_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double* prod = reinterpret_cast<double*>(&sm.u);   // the logits tile is no longer needed
  const double tk = static_cast<double>(T) * k;
  for (int e = tid; e < N; e += kRouteThreads) {
    const int cnt = __ldcg(a.cnt_acc + e);
    const double zsum = static_cast<double>(__ldcg(a.z_acc + e)) * (1.0 / 4294967296.0);
    const double y = static_cast<double>(cnt) / tk;
    const double zm = zsum / static_cast<double>(T);
    if (a.stats.counts) a.stats.counts[e] = cnt;
    if (a.stats.y_frac) a.stats.y_frac[e] = static_cast<float>(y);
    if (a.stats.z_mean) a.stats.z_mean[e] = static_cast<float>(zm);
    prod[e] = y * zm;
    sm.hist[e] = cnt;
  }
  __syncthreads();
  if (warp == 0) {
    // L_aux, and the load figures: std of the shares f_i, the two largest counts
    double acc = 0.0, fsum = 0.0;
    int c1 = 0, c2 = 0;  // largest and second largest count seen by this lane
    for (int e = lane; e < N; e += 32) {
      acc += prod[e];
      fsum += static_cast<double>(sm.hist[e]) / tk;
      const int c = sm.hist[e];
      if (c > c1) {
        c2 = c1;
        c1 = c;
      } else if (c > c2) {
        c2 = c;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      acc += __shfl_xor_sync(0xffffffffu, acc, o);
      fsum += __shfl_xor_sync(0xffffffffu, fsum, o);
      const int o1 = __shfl_xor_sync(0xffffffffu, c1, o), o2 = __shfl_xor_sync(0xffffffffu, c2, o);
      const int hi = max(c1, o1), lo = max(min(c1, o1), max(c2, o2));
      c1 = hi;
      c2 = lo;
    }
    const double fmean = fsum / N;
    double var = 0.0;
    for (int e = lane; e < N; e += 32) {
      const double dv = static_cast<double>(sm.hist[e]) / tk - fmean;
      var += dv * dv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) var += __shfl_xor_sync(0xffffffffu, var, o);
    if (lane == 0) {
      if (a.stats.l_aux_p3) a.stats.l_aux_p3[0] = static_cast<float>(static_cast<double>(T) / N * acc);
      if (a.stats.l_aux_switch) a.stats.l_aux_switch[0] = static_cast<float>(N * acc);
      if (a.stats.load_std) a.stats.load_std[0] = static_cast<float>(sqrt(var / N));
      if (a.stats.top2_ratio) a.stats.top2_ratio[0] = static_cast<float>(static_cast<double>(c1 + c2) / tk);
    }
  } else if (warp == 1 && a.stats.z_loss != nullptr) {
    // z-loss: the blocks' partials in block order (a fixed reduction tree)
    double t = 0.0;
    for (unsigned b0 = lane; b0 < gridDim.x; b0 += 32 * 8) {  // 8 loads in flight, then the adds in block order
      double v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = b0 + 32 * u < gridDim.x ? __ldcg(a.zl_part + b0 + 32 * u) : 0.0;
#pragma unroll
      for (int u = 0; u < 8; ++u) t += v[u];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) a.stats.z_loss[0] = static_cast<float>(t / static_cast<double>(T));
  }
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
  if (a.logits_in != nullptr)
    route_kernel<NP, true><<<blocks, kRouteThreads, 0, s>>>(a);
  else
    route_kernel<NP, false><<<blocks, kRouteThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bias_update(float* b, const int32_t* counts, int64_t Tk, int N, float gamma, cudaStream_t s) {
  bias_update_kernel<<<1, 256, 0, s>>>(b, counts, Tk, N, gamma);
  return cudaGetLastError();
}

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
