// Weighted combine back to token order:
//   y[t] = sum_{j : row_map[t][j] >= 0} w[t][j] * O[row_map[t][j]]  (+ S[t])
// "MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §2.1 (the layer graph
// ends in "权重加和", the weighted sum) and §2.2 (the top-k formula).  Dropped
// slots add nothing and the kept weights are not renormalised.  The sum is
// accumulated in fp32 in slot order, the shared-expert row is added last, and
// the result is rounded once.  One block per token; 16-byte vector loads.  For
// the common slot counts the slot loop is unrolled so that the loads of all k
// expert rows are in flight together before the (slot-ordered) accumulation.
#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kCombineThreads = 128;

__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4& v) {
  acc[0] = fmaf(w, bf16_lo(v.x), acc[0]);
  acc[1] = fmaf(w, bf16_hi(v.x), acc[1]);
  acc[2] = fmaf(w, bf16_lo(v.y), acc[2]);
  acc[3] = fmaf(w, bf16_hi(v.y), acc[3]);
  acc[4] = fmaf(w, bf16_lo(v.z), acc[4]);
  acc[5] = fmaf(w, bf16_hi(v.z), acc[5]);
  acc[6] = fmaf(w, bf16_lo(v.w), acc[6]);
  acc[7] = fmaf(w, bf16_hi(v.w), acc[7]);
}

__device__ __forceinline__ void add8(float (&acc)[8], const uint4& v) {
  acc[0] += bf16_lo(v.x);
  acc[1] += bf16_hi(v.x);
  acc[2] += bf16_lo(v.y);
  acc[3] += bf16_hi(v.y);
  acc[4] += bf16_lo(v.z);
  acc[5] += bf16_hi(v.z);
  acc[6] += bf16_lo(v.w);
  acc[7] += bf16_hi(v.w);
}

// KS > 0: k == KS, slot loop unrolled; KS == 0: any k (runtime loop)
template <int KS>
__global__ void __launch_bounds__(kCombineThreads) combine_bf16_kernel(const CombineArgs a) {
  __shared__ int rows[32];
  __shared__ float wts[32];
  grid_dep_wait();
  grid_dep_launch();
  const int64_t t = blockIdx.x;
  const int k = KS > 0 ? KS : a.k;
  if (threadIdx.x < k) {
    rows[threadIdx.x] = a.row_map[t * k + threadIdx.x];
    wts[threadIdx.x] = a.topk_w[t * k + threadIdx.x];
  }
  __syncthreads();
  const int nvec = a.d / 8;
  const uint4* O = static_cast<const uint4*>(a.out_rows);
  const uint4* S = static_cast<const uint4*>(a.shared_out);
  uint4* Y = static_cast<uint4*>(a.y);
  for (int c = threadIdx.x; c < nvec; c += kCombineThreads) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if constexpr (KS > 0) {
      uint4 v[KS];
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        const int r = rows[j];
        v[j] = r >= 0 ? O[static_cast<int64_t>(r) * nvec + c] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < KS; ++j)
        if (rows[j] >= 0) fma8(acc, wts[j], v[j]);
    } else {
      for (int j = 0; j < k; ++j) {
        const int r = rows[j];
        if (r < 0) continue;
        fma8(acc, wts[j], O[static_cast<int64_t>(r) * nvec + c]);
      }
    }
    if (S != nullptr) add8(acc, S[t * nvec + c]);
    Y[t * nvec + c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                 pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

__global__ void __launch_bounds__(kCombineThreads) combine_f32_kernel(const CombineArgs a) {
  __shared__ int rows[32];
  __shared__ float wts[32];
  grid_dep_wait();
  grid_dep_launch();
  const int64_t t = blockIdx.x;
  const int k = a.k;
  if (threadIdx.x < k) {
    rows[threadIdx.x] = a.row_map[t * k + threadIdx.x];
    wts[threadIdx.x] = a.topk_w[t * k + threadIdx.x];
  }
  __syncthreads();
  const int nvec = a.d / 4;
  const float4* O = static_cast<const float4*>(a.out_rows);
  const float4* S = static_cast<const float4*>(a.shared_out);
  float4* Y = static_cast<float4*>(a.y);
  for (int c = threadIdx.x; c < nvec; c += kCombineThreads) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int r = rows[j];
      if (r < 0) continue;
      const float4 v = O[static_cast<int64_t>(r) * nvec + c];
      const float w = wts[j];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    if (S != nullptr) {
      const float4 v = S[t * nvec + c];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    Y[t * nvec + c] = acc;
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  // may start while the expert GEMM before it finishes (it waits for its results first)
  const dim3 grid(static_cast<unsigned>(a.T)), block(kCombineThreads);
  if (!a.is_bf16) return launch_overlapped(combine_f32_kernel, grid, block, 0, s, a);
  switch (a.k) {
    case 1: return launch_overlapped(combine_bf16_kernel<1>, grid, block, 0, s, a);
    case 2: return launch_overlapped(combine_bf16_kernel<2>, grid, block, 0, s, a);
    case 4: return launch_overlapped(combine_bf16_kernel<4>, grid, block, 0, s, a);
    case 6: return launch_overlapped(combine_bf16_kernel<6>, grid, block, 0, s, a);
    case 8: return launch_overlapped(combine_bf16_kernel<8>, grid, block, 0, s, a);
    default: return launch_overlapped(combine_bf16_kernel<0>, grid, block, 0, s, a);
  }
}

}  // namespace moe
