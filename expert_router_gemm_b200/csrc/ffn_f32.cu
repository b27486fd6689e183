// fp32 grouped SwiGLU FFN on the CUDA cores (the fp32 layer: no fp32 tensor-core
// format matches its 1e-5 tolerance at full fp32 input precision).
//   h[r]   = silu(a[r] W1_g) * (a[r] W3_g)     silu(u) = u / (1 + exp(-u))
//   out[r] = h[r] W2_g
// for the rows r of group g ("MoE 训练加速实战：DeepEP + Grouped GeMM +
// Aux-Loss-Free" §4.2: the grouped GEMM computes y_i = W_i x_i for every expert
// in one launch).  grid = (row tiles, column tiles, groups); a block whose row
// tile lies beyond its group's count exits at once.  Accumulation is fp32 FMA
// in K order.
#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int TS = 32;  // tile edge

__device__ __forceinline__ float silu_f32(float u) { return u / (1.0f + expf(-u)); }

// First row and row count of group g, clamped to the buffers (a segment table
// that points outside them raises MOE_FLAG_BAD_EXPERT_INDEX and is skipped).
__device__ __forceinline__ int64_t group_rows(const FfnArgs& a, int g, int* count) {
  int64_t r0 = 0;
  int c = a.dense_rows;
  if (a.seg_off != nullptr) {
    r0 = a.seg_off[g];
    c = a.seg_count[g];
  }
  if (r0 < 0 || c < 0 || r0 + c > a.max_rows) {
    if (threadIdx.x == 0 && threadIdx.y == 0 && blockIdx.x == 0 && blockIdx.y == 0) atomicOr(a.flags, kFlagBadIndex);
    r0 = 0;
    c = 0;
  }
  *count = c;
  return r0;
}

__global__ void __launch_bounds__(256) ffn1_f32_kernel(const FfnArgs a) {
  __shared__ float As[TS][TS + 1];
  __shared__ float B1s[TS][TS + 1];
  __shared__ float B3s[TS][TS + 1];
  grid_dep_wait();   // the dispatch's rows and segment table are complete
  grid_dep_launch();
  const int g = blockIdx.z;
  int count = 0;
  const int64_t seg0 = group_rows(a, g, &count);
  const int m0 = blockIdx.x * TS;
  if (m0 >= count) return;
  const int64_t row0 = seg0 + m0;
  const int n0 = blockIdx.y * TS;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int d = a.d, f = a.f;
  const float* A = static_cast<const float*>(a.a);
  const float* W1 = static_cast<const float*>(a.w1) + static_cast<int64_t>(g) * d * f;
  const float* W3 = static_cast<const float*>(a.w3) + static_cast<int64_t>(g) * d * f;
  float ga[4] = {0.f, 0.f, 0.f, 0.f}, ua[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < d; k0 += TS) {
    for (int i = ty; i < TS; i += 8) {
      As[i][tx] = (m0 + i < count && k0 + tx < d) ? A[(row0 + i) * d + k0 + tx] : 0.f;
      const bool bk = k0 + i < d && n0 + tx < f;
      B1s[i][tx] = bk ? W1[static_cast<int64_t>(k0 + i) * f + n0 + tx] : 0.f;
      B3s[i][tx] = bk ? W3[static_cast<int64_t>(k0 + i) * f + n0 + tx] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < TS; ++kk) {
      const float b1 = B1s[kk][tx], b3 = B3s[kk][tx];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float av = As[ty + 8 * r][kk];
        ga[r] = fmaf(av, b1, ga[r]);
        ua[r] = fmaf(av, b3, ua[r]);
      }
    }
    __syncthreads();
  }
  float* H = static_cast<float*>(a.h);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = m0 + ty + 8 * r, col = n0 + tx;
    if (row < count && col < f) H[(row0 + ty + 8 * r) * f + col] = silu_f32(ga[r]) * ua[r];
  }
}

__global__ void __launch_bounds__(256) ffn2_f32_kernel(const FfnArgs a) {
  __shared__ float As[TS][TS + 1];
  __shared__ float Bs[TS][TS + 1];
  grid_dep_wait();   // h is complete
  grid_dep_launch();
  const int g = blockIdx.z;
  int count = 0;
  const int64_t seg0 = group_rows(a, g, &count);
  const int m0 = blockIdx.x * TS;
  if (m0 >= count) return;
  const int64_t row0 = seg0 + m0;
  const int n0 = blockIdx.y * TS;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int d = a.d, f = a.f;
  const float* H = static_cast<const float*>(a.h);
  const float* W2 = static_cast<const float*>(a.w2) + static_cast<int64_t>(g) * f * d;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < f; k0 += TS) {
    for (int i = ty; i < TS; i += 8) {
      As[i][tx] = (m0 + i < count && k0 + tx < f) ? H[(row0 + i) * f + k0 + tx] : 0.f;
      Bs[i][tx] = (k0 + i < f && n0 + tx < d) ? W2[static_cast<int64_t>(k0 + i) * d + n0 + tx] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < TS; ++kk) {
      const float b = Bs[kk][tx];
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = fmaf(As[ty + 8 * r][kk], b, acc[r]);
    }
    __syncthreads();
  }
  float* O = static_cast<float*>(a.out);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = m0 + ty + 8 * r, col = n0 + tx;
    if (row < count && col < d) O[(row0 + ty + 8 * r) * d + col] = acc[r];
  }
}

}  // namespace

cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t s) {
  if (a.max_count <= 0 || a.G <= 0) return cudaSuccess;
  const dim3 block(TS, 8);
  const unsigned mt = static_cast<unsigned>((a.max_count + TS - 1) / TS);
  // each may start while the kernel before it finishes (it waits for its results first)
  cudaError_t e = launch_overlapped(ffn1_f32_kernel, dim3(mt, (a.f + TS - 1) / TS, a.G), block, 0, s, a);
  if (e != cudaSuccess) return e;
  return launch_overlapped(ffn2_f32_kernel, dim3(mt, (a.d + TS - 1) / TS, a.G), block, 0, s, a);
}

}  // namespace moe
