// Device-side routing of a tile of tokens whose fp32 logits sit in shared
// memory: softmax, top-k with the renormalised weights, and the load-balance
// statistics of the routing kernel (route.cu), whether its logits come from a
// CUDA-core GEMM tile, from the tensor-core router's partial sums or from the
// caller.
//
// "MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §2.2 "Router 数学"
// (scores = softmax(g), top-k of g, weights s_i / sum_topk s_j), §1 pain point 4
// (fp32 router), §5.3 (selection bias for the choice only); "负载均衡策略：MoE训练
// 稳定性保障", section "辅助损失函数" (y_i, z_i, L_aux) and the z_loss_weight row of
// its hyper-parameter table; "ms-swift + Megatron：MoE模型加速10倍实测" §3.3 (load
// figures).
#pragma once

#include <math.h>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {

// Monotone map of a float to an unsigned key (larger float -> larger key; -0.0
// maps like +0.0) and back.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int NP>
struct RouteLane {
  static constexpr int NPL = NP >= 32 ? NP / 32 : 1;  // experts held per lane: lane + 32 c
};

// Softmax and top-k of the BT tokens t0 .. t0+BT-1 whose logits (bias included,
// padding experts N..NP-1 at -inf) are the rows of `lg` (row stride LS floats).
// Warp `warp` of NW takes TPW tokens at a time, in lock step so that their warp
// reductions overlap.  Writes topk_idx / topk_w, adds the selections to `hist`
// (shared, when statistics are wanted), accumulates this lane's softmax scores
// per expert slot in zacc and the warp's sum of logsumexp^2 in zl (same value in
// every lane), and raises the non-finite flag.
template <int NP, int NW, int TPW>
__device__ __forceinline__ void route_tokens(const RouteArgs& a, const float* lg, int LS, int BT, int64_t t0,
                                             int warp, int lane, int* hist, float (&zacc)[RouteLane<NP>::NPL],
                                             double& zl) {
  constexpr int NPL = RouteLane<NP>::NPL;
  const int N = a.N, k = a.k;
  const int64_t T = a.T;
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
        v[q][c] = (valid[q] && e < NP) ? lg[(tl0 + q) * LS + e] : -INFINITY;
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
        const float ve = biased ? lg[(tl0 + q) * LS + e] : key_value(won_h[q]);
        sv = expf(ve - m[q]) / sum[q];
      }
      float ssum = __shfl_sync(0xffffffffu, sv, 0);
      for (int j = 1; j < k; ++j) ssum += __shfl_sync(0xffffffffu, sv, j);
      if (valid[q] && lane < k) {
        const int64_t t = t0 + tl0 + q;
        a.topk_idx[t * k + lane] = e;
        a.topk_w[t * k + lane] = sv / ssum;
        if (a.want_stats) atomicAdd(&hist[e], 1);
      }
    }
  }
}

// Shared memory of route_stats.
template <int NP, int NW>
struct RouteStatsSmem {
  float zw[NW][NP];
  double zl[NW];
  double prod[NP];
  int is_last;
};

// The statistics of a group of NW warps (nthreads = 32 NW threads, thread index
// tid, synchronised by `sync`) that has routed some tokens: the group's fp32
// sums of softmax scores (zacc of every lane, summed over the warps in order)
// and its counts (hist) go to the global accumulators with integer atomics
// (the z sums as fixed point with 32 fraction bits), so the totals do not
// depend on the order of the groups; the group's z-loss partial goes to slot
// `group`.  The last of n_groups groups to finish (ticket counter, no waiting)
// computes y, z, both L_aux forms, the load figures and the z-loss, adding the
// z-loss partials in slot order.
template <int NP, int NW, typename Sync>
__device__ __forceinline__ void route_stats(const RouteArgs& a, RouteStatsSmem<NP, NW>& sm, int* hist,
                                            const float (&zacc)[RouteLane<NP>::NPL], double zl, int warp, int lane,
                                            int tid, unsigned group, unsigned n_groups, Sync sync) {
  constexpr int NPL = RouteLane<NP>::NPL;
  constexpr int nthreads = 32 * NW;
  const int N = a.N, k = a.k;
  const int64_t T = a.T;
#pragma unroll
  for (int c = 0; c < NPL; ++c) {
    const int e = lane + 32 * c;
    if (e < NP) sm.zw[warp][e] = zacc[c];
  }
  if (lane == 0) sm.zl[warp] = zl;
  sync();
  for (int e = tid; e < N; e += nthreads) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) z += sm.zw[w][e];
    atomicAdd(a.z_acc + e, static_cast<unsigned long long>(__double2ull_rn(static_cast<double>(z) * 4294967296.0)));
    if (hist[e] != 0) atomicAdd(a.cnt_acc + e, hist[e]);
  }
  if (tid == 0) {  // the group's z-loss partial, summed over its warps in order
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < NW; ++w) t += sm.zl[w];
    a.zl_part[group] = t;
  }
  __threadfence();
  sync();
  if (tid == 0) sm.is_last = atomicAdd(a.ticket, 1u) == n_groups - 1;
  sync();
  if (!sm.is_last) return;
  __threadfence();
  const double tk = static_cast<double>(T) * k;
  for (int e = tid; e < N; e += nthreads) {
    const int cnt = __ldcg(a.cnt_acc + e);
    const double zsum = static_cast<double>(__ldcg(a.z_acc + e)) * (1.0 / 4294967296.0);
    const double y = static_cast<double>(cnt) / tk;
    const double zm = zsum / static_cast<double>(T);
    if (a.stats.counts) a.stats.counts[e] = cnt;
    if (a.stats.y_frac) a.stats.y_frac[e] = static_cast<float>(y);
    if (a.stats.z_mean) a.stats.z_mean[e] = static_cast<float>(zm);
    sm.prod[e] = y * zm;
    hist[e] = cnt;
  }
  sync();
  if (warp == 0) {
    // L_aux, and the load figures: std of the shares f_i, the two largest counts
    double acc = 0.0, fsum = 0.0;
    int c1 = 0, c2 = 0;  // largest and second largest count seen by this lane
    for (int e = lane; e < N; e += 32) {
      acc += sm.prod[e];
      fsum += static_cast<double>(hist[e]) / tk;
      const int c = hist[e];
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
      const double dv = static_cast<double>(hist[e]) / tk - fmean;
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
    // z-loss: the groups' partials in slot order (a fixed reduction tree)
    double t = 0.0;
    for (unsigned b0 = lane; b0 < n_groups; b0 += 32 * 8) {  // 8 loads in flight, then the adds in slot order
      double v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = b0 + 32 * u < n_groups ? __ldcg(a.zl_part + b0 + 32 * u) : 0.0;
#pragma unroll
      for (int u = 0; u < 8; ++u) t += v[u];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) a.stats.z_loss[0] = static_cast<float>(t / static_cast<double>(T));
  }
}

}  // namespace moe
