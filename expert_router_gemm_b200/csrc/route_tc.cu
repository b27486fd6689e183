// Router GEMM on the tcgen05 tensor cores for bf16 layers (any N <= 256; the
// weight split is padded to a multiple of 64 experts with zeros):
//   logits[t, e] = sum_c x[t, c] * W_r[c, e]  (+ b[e])        fp32 result
// ("MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §2.2: g = x W_r; the
// router stays fp32, §1 pain point 4).
//
// fp32 accuracy from bf16 tensor-core inputs: every fp32 router weight w is
// split exactly into three bf16 values, w = hi + mid + lo (hi = bf16(w),
// mid = bf16(w - hi), lo = w - hi - mid, which fits in 8 significant bits).  x
// is already bf16, so every product x*hi, x*mid, x*lo is exact and the three
// MMAs of a K slab accumulate x*w in the fp32 tensor-memory accumulator.  The
// result differs from a CUDA-core fp32 dot product only in summation order.
//
// One CTA per 128-token x BN-expert tile (BN = 64 or 128), 192 threads:
// warp 0 lane 0 issues the TMA loads (x slab 128 x 64, three weight slabs
// 64 x BN per stage), warp 1 allocates TMEM and lane 0 issues the MMAs, warps
// 2-5 move the accumulator to registers, add the bias and store fp32 logits.
// The softmax / top-k pass then runs on these logits (route.cu, logits mode).
// Every mbarrier wait is bounded (MOE_FLAG_WAIT_TIMEOUT).
#include <algorithm>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int CHUNK = 64 * BK * 2;     // 8 KB: 64 expert columns x 64 K rows
constexpr int kThreads = 192;

template <int BN>
struct RtCfg {
  static constexpr int PART_BYTES = (BN / 64) * CHUNK;      // one of hi / mid / lo
  static constexpr int STAGE_BYTES = A_BYTES + 3 * PART_BYTES;
  static constexpr int STAGES = BN == 64 ? 5 : 3;
  static constexpr int TMEM_COLS = BN;                      // power of two >= 32
};

struct RtTail {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull;
  uint32_t tmem_base;
  uint32_t abort;
};

template <int BN>
constexpr size_t rt_smem_bytes() {
  return 1024 + static_cast<size_t>(RtCfg<BN>::STAGES) * RtCfg<BN>::STAGE_BYTES + sizeof(RtTail);
}

struct RtParams {
  int64_t T;
  int N, d;
  const float* bias;   // [N] or nullptr
  float* logits;       // [T, N]
  uint32_t* flags;
};

// W_r fp32 [d, N] -> three bf16 slabs [3][d][NP] (columns N..NP-1 zero)
__global__ void split_router_kernel(const float* __restrict__ w, uint16_t* __restrict__ out, int d, int N,
                                    int NP) {
  const int64_t total = static_cast<int64_t>(d) * NP;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / NP;
    const int c = static_cast<int>(i % NP);
    const float v = c < N ? w[r * N + c] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    out[i] = *reinterpret_cast<const uint16_t*>(&hi);
    out[total + i] = *reinterpret_cast<const uint16_t*>(&mid);
    out[2 * total + i] = *reinterpret_cast<const uint16_t*>(&lo);
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const RtParams p) {
  using C = RtCfg<BN>;
  constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN, 1);
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  RtTail& tl = *reinterpret_cast<RtTail*>(base + C::STAGES * C::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int KB = p.d / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_addr(&tl.full[s]), 1);
      mbar_init(smem_addr(&tl.empty[s]), 1);
    }
    mbar_init(smem_addr(&tl.tfull), 1);
    tl.abort = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&tl.tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl.tmem_base;
  volatile uint32_t* abort = &tl.abort;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0, last_par = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout)) break;
        const uint32_t fb = smem_addr(&tl.full[stage]);
        mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
        const uint32_t sa = smem_addr(base + stage * C::STAGE_BYTES);
        tma_load_2d(sa, &tmX, fb, kb * BK, m0);
#pragma unroll
        for (int part = 0; part < 3; ++part)
#pragma unroll
          for (int ch = 0; ch < BN / 64; ++ch)
            tma_load_2d(sa + A_BYTES + part * C::PART_BYTES + ch * CHUNK, &tmW, fb, n0 + 64 * ch,
                        part * p.d + kb * BK);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < C::STAGES; ++s)
        if ((issued >> s) & 1u)
          mbar_wait(smem_addr(&tl.full[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true, any = false;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_addr(base + stage * C::STAGE_BYTES);
#pragma unroll
        for (int part = 0; part < 3; ++part)
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sa + A_BYTES + part * C::PART_BYTES + kk * 2048, CHUNK, 1024);
            tc_mma_f16(tmem, adesc, bdesc, kIdesc, (kb | part | kk) != 0 ? 1u : 0u);
          }
        any = true;
        tc_commit(smem_addr(&tl.empty[stage]));
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) *abort = 1u;
      if (any) {  // hand the accumulator to the epilogue; every MMA has drained before TMEM is freed
        tc_commit(smem_addr(&tl.tfull));
        mbar_wait(smem_addr(&tl.tfull), 0u, nullptr, p.flags, kFlagTimeout);
      }
    }
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int64_t t = static_cast<int64_t>(m0) + row;
    if (KB > 0 && mbar_wait(smem_addr(&tl.tfull), 0u, abort, p.flags, kFlagTimeout)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + c, v);
        tmem_ld_wait();
        if (t < p.T) {
          float* dst = p.logits + t * p.N + n0 + c;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = n0 + c + i;
            if (e < p.N) dst[i] = __uint_as_float(v[i]) + (p.bias != nullptr ? p.bias[e] : 0.f);
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& mx, const CUtensorMap& mw, const RtParams& p, cudaStream_t s) {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(router_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(rt_smem_bytes<BN>()));
  });
  if (r != cudaSuccess) return r;
  const dim3 grid(static_cast<unsigned>((p.T + BM - 1) / BM), static_cast<unsigned>((p.N + BN - 1) / BN));
  router_tc_kernel<BN><<<grid, kThreads, rt_smem_bytes<BN>(), s>>>(mx, mw, p);
  return cudaGetLastError();
}

}  // namespace

// the split slabs are [3][d][NPS] with NPS = N rounded up to a multiple of 64
static int split_cols(int N) { return (N + 63) / 64 * 64; }
size_t router_split_bytes(int d, int N) { return 3ull * d * split_cols(N) * sizeof(uint16_t); }

cudaError_t launch_router_tc(const RouteArgs& a, void* split, float* logits, cudaStream_t s) {
  const int NP = split_cols(a.N);
  const int64_t total = static_cast<int64_t>(a.d) * NP;
  const int threads = 256;
  const int blocks = static_cast<int>(std::min<int64_t>((total + threads - 1) / threads, 4 * device_sm_count()));
  split_router_kernel<<<blocks, threads, 0, s>>>(a.w_router, static_cast<uint16_t*>(split), a.d, a.N, NP);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mw;
  if (!make_tma_2d_bf16(&mx, a.x, a.d, a.T, BK, BM) || !make_tma_2d_bf16(&mw, split, NP, 3ull * a.d, 64, BK))
    return cudaErrorInvalidValue;
  RtParams p{a.T, a.N, a.d, a.bias, logits, a.flags};
  // 64-wide expert tiles while they fit in one wave, else 128-wide
  const int64_t m_tiles = (a.T + BM - 1) / BM;
  if (m_tiles * (NP / 64) <= device_sm_count() || NP < 128) return launch_bn<64>(mx, mw, p, s);
  return launch_bn<128>(mx, mw, p, s);
}

}  // namespace moe
