// Router GEMM on the tcgen05 tensor cores for bf16 layers (any N <= 256; the
// weight split is padded with zero columns to whole expert tiles):
//   logits[t, e] = sum_c x[t, c] * W_r[c, e]                   fp32 result
// written as 1, 2 or 4 partial sums over K slices (split z covers its share of
// the K slabs, so small layers still fill the GPU); the softmax / top-k kernel
// adds the partials in split order, then the bias.  No atomics: the result does
// not depend on scheduling.
// ("MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §2.2: g = x W_r; the
// router stays fp32, §1 pain point 4).
//
// fp32 accuracy from bf16 tensor-core inputs: every fp32 router weight w is
// split exactly into three bf16 values, w = hi + mid + lo (hi = bf16(w),
// mid = bf16(w - hi), lo = w - hi - mid, which fits in 8 significant bits).  x
// is already bf16, so every product x*hi, x*mid, x*lo is exact.  Per K step
// one MMA runs over the hi and mid parts side by side (staged as adjacent
// 64-column chunks: twice the columns, one pass over A) into fp32 tensor-memory
// accumulators of x*hi and x*mid, and one over the lo part into a third; the
// epilogue adds hi + (mid + lo).  Where a logit is a single product, mid + lo
// is exact and the logit is the correctly rounded x*w; otherwise the result
// differs from a CUDA-core fp32 dot product only in summation order.  The
// split is made per call (split_router_kernel) unless the caller passes one
// made once by moe_router_split.
//
// 192 threads per CTA: warp 0 lane 0 issues the TMA loads (x slab 128 x 64 and
// the three weight slabs of this CTA's experts per stage), warp 1 allocates TMEM
// and lane 0 issues the MMAs, warps 2-5 move the accumulators through registers
// and shared memory to the fp32 partial sums (whole 128-byte row pieces).  The
// operand stream is latency-bound (each CTA streams its own tokens), so the
// work per staged byte decides the speed:
//   CG = 1: one CTA per 128 tokens x 64 experts (M=128; N=128 for hi|mid, 64
//           for lo), N <= 64;
//   CG = 2: a CTA pair per 256 tokens x 128 experts (cta_group::2, M=256;
//           N=256 for hi|mid, 128 for lo): each CTA stages its own 128 tokens
//           and 64 of the experts' weight columns, so each staged byte feeds
//           twice the MMA work.
// Every mbarrier wait is bounded (MOE_FLAG_WAIT_TIMEOUT).
#include <algorithm>
#include <atomic>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                // tokens per CTA
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int CHUNK = 64 * BK * 2;     // 8 KB: 64 expert columns x 64 K rows
constexpr int kThreads = 192;

template <int BN, int CG>
struct RtCfg {
  static constexpr int COLS = BN / CG;                        // weight columns staged per CTA
  static constexpr int CHUNKS = COLS / 64;
  static constexpr int PART_BYTES = CHUNKS * CHUNK;           // one of hi / mid / lo
  static constexpr int STAGE_BYTES = A_BYTES + 3 * PART_BYTES;
  static constexpr int STAGES = STAGE_BYTES <= 40 * 1024 ? 5 : 3;
  // accumulators: x*hi and x*mid side by side (one MMA over the adjacent hi and
  // mid chunks, 2*BN columns), then x*lo (BN columns)
  static constexpr int LO_COL = 2 * BN;
  static constexpr int TMEM_COLS = 3 * BN <= 256 ? 256 : 512;  // power of two >= 3*BN
  static constexpr uint32_t IDESC_HM = idesc_bf16_f32(BM * CG, 2 * BN, 1);
  static constexpr uint32_t IDESC_LO = idesc_bf16_f32(BM * CG, BN, 1);
  static_assert(COLS == 64, "one 64-column chunk per part per CTA: hi and mid adjacent");
  static_assert(2 * BN <= 256, "the hi|mid MMA is at most 256 columns wide");
};

struct RtTail {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull;
  uint32_t tmem_base;
  uint32_t abort;
};

template <int BN, int CG>
constexpr size_t rt_smem_bytes() {
  return 1024 + static_cast<size_t>(RtCfg<BN, CG>::STAGES) * RtCfg<BN, CG>::STAGE_BYTES + sizeof(RtTail);
}

struct RtParams {
  int64_t T;
  int N, d;
  int kb_per_split;    // K slabs per split (blockIdx.z = split)
  float* partials;     // [splits][T, N]: split z writes partials + z * T * N
  uint64_t wait_ns;    // bound of the pipeline waits (those that also watch the abort flag);
                       // the waits that drain copies and MMAs in flight keep kWaitLimitNs
  uint32_t* flags;
};

// Bound of the pipeline waits (moe_set_wait_limit_ns); 0 = kWaitLimitNs.
std::atomic<uint64_t> g_router_wait_ns{0};

// W_r fp32 [d, N] -> three bf16 slabs [3][d][NP] (columns N..NP-1 zero).
// Block (32, 8): threadIdx.y picks one of 8 rows, a thread splits 4 adjacent
// columns and stores each slab's 4 values as one 8-byte word.
__device__ __forceinline__ void split3(float v, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h);
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(m);
  const __nv_bfloat16 l = __float2bfloat16_rn(r2);
  hi = *reinterpret_cast<const uint16_t*>(&h);
  mid = *reinterpret_cast<const uint16_t*>(&m);
  lo = *reinterpret_cast<const uint16_t*>(&l);
}

__global__ void __launch_bounds__(256) split_router_kernel(const float* __restrict__ w, uint16_t* __restrict__ out,
                                                           int d, int N, int NP) {
  const int r = blockIdx.x * blockDim.y + threadIdx.y;
  if (r >= d) return;
  const int64_t plane = static_cast<int64_t>(d) * NP;
  const float* wr = w + static_cast<int64_t>(r) * N;
  for (int c = threadIdx.x * 4; c < NP; c += blockDim.x * 4) {
    uint16_t p[3][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split3(c + i < N ? wr[c + i] : 0.f, p[0][i], p[1][i], p[2][i]);
    const int64_t o = static_cast<int64_t>(r) * NP + c;
#pragma unroll
    for (int s = 0; s < 3; ++s)
      *reinterpret_cast<uint2*>(out + s * plane + o) =
          make_uint2(p[s][0] | (static_cast<uint32_t>(p[s][1]) << 16), p[s][2] | (static_cast<uint32_t>(p[s][3]) << 16));
  }
}

template <int BN, int CG>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const RtParams p) {
  using C = RtCfg<BN, CG>;
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  RtTail& tl = *reinterpret_cast<RtTail*>(base + C::STAGES * C::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;  // 0: this CTA issues the MMAs
  const int m0 = (static_cast<int>(blockIdx.x) / CG) * (BM * CG) + static_cast<int>(rank) * BM;  // my tokens
  const int n0 = blockIdx.y * BN;                           // the tile's first expert
  const int ncol = n0 + static_cast<int>(rank) * C::COLS;   // my weight columns
  const int kb0 = blockIdx.z * p.kb_per_split;              // this split's K slabs
  const int KB = max(0, min(p.d / BK - kb0, p.kb_per_split));
  float* const logits = p.partials + static_cast<int64_t>(blockIdx.z) * p.T * p.N;

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
    if (CG == 2) {
      tmem_alloc_pair(smem_addr(&tl.tmem_base), C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(&tl.tmem_base), C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (CG == 2)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl.tmem_base;
  volatile uint32_t* abort = &tl.abort;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0, last_par = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout, p.wait_ns)) break;
        const uint32_t fb_local = smem_addr(&tl.full[stage]);
        const uint32_t sa = smem_addr(base + stage * C::STAGE_BYTES);
        if (CG == 1) {
          mbar_arrive_expect_tx(fb_local, C::STAGE_BYTES);
          tma_load_2d(sa, &tmX, fb_local, (kb0 + kb) * BK, m0);
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ch = 0; ch < C::CHUNKS; ++ch)
              tma_load_2d(sa + A_BYTES + part * C::PART_BYTES + ch * CHUNK, &tmW, fb_local, ncol + 64 * ch,
                          part * p.d + (kb0 + kb) * BK);
        } else {
          // both CTAs' bytes complete on the even CTA's barrier
          const uint32_t fb = rank == 0 ? fb_local : mapa_shared(fb_local, 0);
          if (rank == 0) mbar_arrive_expect_tx(fb_local, 2 * C::STAGE_BYTES);
          tma_load_2d_pair(sa, &tmX, fb, (kb0 + kb) * BK, m0);
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ch = 0; ch < C::CHUNKS; ++ch)
              tma_load_2d_pair(sa + A_BYTES + part * C::PART_BYTES + ch * CHUNK, &tmW, fb, ncol + 64 * ch,
                               part * p.d + (kb0 + kb) * BK);
        }
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // every load issued here has landed before the CTA may exit
      for (int s = 0; s < C::STAGES; ++s)
        if ((issued >> s) & 1u) {
          if (rank == 0)
            mbar_wait(smem_addr(&tl.full[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
          else
            mbar_wait(smem_addr(&tl.empty[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true, any = false;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_addr(base + stage * C::STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(sa + kk * 32, 16, 1024);
          // the hi and mid chunks are adjacent: one MMA over both (chunk stride CHUNK)
          const uint64_t bdesc_hm = smem_desc_sw128(sa + A_BYTES + kk * 2048, CHUNK, 1024);
          const uint64_t bdesc_lo = smem_desc_sw128(sa + A_BYTES + 2 * C::PART_BYTES + kk * 2048, CHUNK, 1024);
          const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
          if (CG == 2) {
            tc_mma_f16_pair(tmem, adesc, bdesc_hm, C::IDESC_HM, acc);
            tc_mma_f16_pair(tmem + C::LO_COL, adesc, bdesc_lo, C::IDESC_LO, acc);
          } else {
            tc_mma_f16(tmem, adesc, bdesc_hm, C::IDESC_HM, acc);
            tc_mma_f16(tmem + C::LO_COL, adesc, bdesc_lo, C::IDESC_LO, acc);
          }
        }
        any = true;
        const uint32_t e = smem_addr(&tl.empty[stage]);
        if (CG == 2) {
          tc_commit_pair_both(e);
        } else {
          tc_commit(e);
        }
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) *abort = 1u;
      if (any) {  // hand the accumulator to the epilogues; every MMA has drained before TMEM is freed
        const uint32_t f = smem_addr(&tl.tfull);
        if (CG == 2) {
          tc_commit_pair_both(f);
        } else {
          tc_commit(f);
        }
        mbar_wait(f, 0u, nullptr, p.flags, kFlagTimeout);
      }
    }
  } else {
    // Epilogue: a warp owns 32 accumulator rows (tokens).  Each 32-column
    // chunk goes through shared memory (the stage buffers, idle once every MMA
    // has completed) so that the global stores are whole 128-byte row pieces.
    const int quad = warp & 3;
    float* stg = reinterpret_cast<float*>(base) + quad * 32 * 33;  // 32 x 33 words: conflict-free both ways
    if (KB > 0 && mbar_wait(smem_addr(&tl.tfull), 0u, abort, p.flags, kFlagTimeout, p.wait_ns)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        // experts c .. c+31 of the tile: CTA r of a pair staged experts 64r ..
        // 64r+63, whose x*hi and x*mid sums are columns 128r + j and
        // 128r + 64 + j of the hi|mid accumulator (j = expert mod 64); x*lo
        // sums follow at LO_COL + expert
        const uint32_t row = static_cast<uint32_t>(quad * 32) << 16;
        const int hi_col = c + 64 * (c / 64);
        uint32_t vh[32], vm[32], vl[32];
        tmem_ld32(tmem + row + hi_col, vh);
        tmem_ld32(tmem + row + hi_col + 64, vm);
        tmem_ld32(tmem + row + C::LO_COL + c, vl);
        tmem_ld_wait();
        // hi + (mid + lo): mid + lo is the exact product with the weight's low
        // 16 bits whenever a logit is a single product, so that logit is the
        // correctly rounded x * w
#pragma unroll
        for (int i = 0; i < 32; ++i)
          stg[lane * 33 + i] =
              __fadd_rn(__uint_as_float(vh[i]), __fadd_rn(__uint_as_float(vm[i]), __uint_as_float(vl[i])));
        __syncwarp();
        const int e = n0 + c + lane;
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
          const int64_t t = static_cast<int64_t>(m0) + quad * 32 + r;
          if (t < p.T && e < p.N) logits[t * p.N + e] = stg[r * 33 + lane];
        }
        __syncwarp();
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  if (CG == 2)
    cluster_sync();  // the even CTA's MMAs (which write both CTAs' TMEM) have drained
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, int CG>
cudaError_t launch_tile(const CUtensorMap& mx, const CUtensorMap& mw, const RtParams& p, int splits, cudaStream_t s) {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(router_tc_kernel<BN, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(rt_smem_bytes<BN, CG>()));
  });
  if (r != cudaSuccess) return r;
  cudaLaunchConfig_t cfg = {};
  const int64_t tiles_m = (p.T + BM * CG - 1) / (BM * CG);
  cfg.gridDim = dim3(static_cast<unsigned>(tiles_m * CG), static_cast<unsigned>((p.N + BN - 1) / BN),
                     static_cast<unsigned>(splits));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = rt_smem_bytes<BN, CG>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, router_tc_kernel<BN, CG>, mx, mw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The split slabs are [3][d][NPS]: N rounded up to the expert width of a tile
// (128 for CTA pairs, used when N > 64; else 64), padded with zeros.
int split_width(int N) { return N > 64 ? (N + 127) / 128 * 128 : (N + 63) / 64 * 64; }

}  // namespace

int router_split_width(int N) { return split_width(N); }

void set_router_wait_ns(uint64_t ns) { g_router_wait_ns.store(ns, std::memory_order_relaxed); }

size_t router_split_bytes(int d, int N) { return 3ull * d * split_width(N) * sizeof(uint16_t); }

cudaError_t launch_router_split(const float* w_router, int d, int N, void* split, cudaStream_t s) {
  split_router_kernel<<<(d + 7) / 8, dim3(32, 8), 0, s>>>(w_router, static_cast<uint16_t*>(split), d, N,
                                                         split_width(N));
  return cudaGetLastError();
}

cudaError_t launch_router_tc(const RouteArgs& a, const void* split, bool make_split, void* split_buf, float* partials,
                             int* n_partials, cudaStream_t s) {
  const bool pairs = a.N > 64;
  const int NP = split_width(a.N);
  if (make_split) {
    cudaError_t e = launch_router_split(a.w_router, a.d, a.N, split_buf, s);
    if (e != cudaSuccess) return e;
    split = split_buf;
  }
  CUtensorMap mx, mw;
  if (!make_tma_2d_bf16(&mx, a.x, a.d, a.T, BK, BM) || !make_tma_2d_bf16(&mw, split, NP, 3ull * a.d, 64, BK))
    return cudaErrorInvalidValue;
  // Split K while the grid stays within one wave and every split keeps >= 8 slabs.
  const int tile_m = pairs ? 2 * BM : BM;
  const int tile_n = pairs ? 128 : 64;
  const int64_t ctas = (a.T + tile_m - 1) / tile_m * ((a.N + tile_n - 1) / tile_n) * (pairs ? 2 : 1);
  const int kb_total = a.d / BK;
  int splits = 1;
  while (splits < kRouterMaxPartials && ctas * splits * 2 <= device_sm_count() && kb_total / (splits * 2) >= 8)
    splits *= 2;
  const int kbs = (kb_total + splits - 1) / splits;
  splits = (kb_total + kbs - 1) / kbs;  // every split has at least one slab
  *n_partials = splits;
  const uint64_t w = g_router_wait_ns.load(std::memory_order_relaxed);
  RtParams p{a.T, a.N, a.d, kbs, partials, w == 0 ? kWaitLimitNs : w, a.flags};
  if (pairs) return launch_tile<128, 2>(mx, mw, p, splits, s);
  return launch_tile<64, 1>(mx, mw, p, splits, s);
}

}  // namespace moe
