// bf16 grouped SwiGLU FFN on the 5th-generation tensor cores (sm_100a).
//
// "MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §4.1-4.2: one kernel
// serves every expert (y_i = W_i x_i), instead of one GEMM launch per expert,
// and tiles are formed per expert.  Two launches of one persistent kernel:
//   GEMM1 (SWIGLU): h[r] = silu(xp[r] W1_e) * (xp[r] W3_e)  -> bf16
//   GEMM2 (PLAIN):  out[r] = h[r] W2_e                       -> bf16
//
// Design (per CTA, one CTA per SM, 192 threads):
//   warp 0 lane 0   TMA producer: A tile 128 x 64 (K-major rows of the permuted
//                   activations) and B tile 64 x 256 (rows of the row-major weight,
//                   i.e. MN-major) per stage, 128-byte swizzle, 4-stage ring.
//   warp 1 lane 0   MMA issuer: tcgen05.mma kind::f16, M=128 N=256 K=16, fp32
//                   accumulator in tensor memory; two accumulators (512 TMEM
//                   columns) so the epilogue of tile i overlaps the main loop of
//                   tile i+1.  Warp 1 also allocates and frees the TMEM.
//   warps 2-5       epilogue: tcgen05.ld of the accumulator rows, SwiGLU in fp32
//                   (gate = columns 0-127, up = columns 128-255 of one tile, so
//                   both halves of a hidden unit sit in the same CTA), one
//                   rounding to bf16, masked stores of the valid rows.
// Tiles are ordered (expert, N tile, M tile) with M fastest, so CTAs running at
// the same time share weight slabs in L2; every CTA derives the tile list from
// the device-side segment table, so no host synchronisation is needed.
// Every mbarrier wait is bounded; on a timeout the kernel raises
// MOE_FLAG_WAIT_TIMEOUT, waits (bounded) for its own copies and MMAs in flight,
// frees its TMEM and returns.
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                    // rows per tile (MMA M)
constexpr int BK = 64;                     // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int MMA_N = 256;                 // accumulator columns per tile
constexpr int MMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_CHUNK = 64 * BK * 2;       // 8 KB: 64 output columns x 64 K rows
constexpr int B_BYTES = 4 * B_CHUNK;       // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * MMA_N;
constexpr int kMaxGroups = 256;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, MMA_N, /*b_mn_major=*/1);

enum { MODE_SWIGLU = 0, MODE_PLAIN = 1 };

struct TcParams {
  const int32_t* seg_off;    // [G+1] or nullptr (one dense group of dense_rows rows)
  const int32_t* seg_count;  // [G]
  int G;
  int dense_rows;
  int64_t max_rows;          // rows of the A and output buffers
  int K;                     // reduction length (multiple of 64)
  int n_out;                 // output columns
  uint16_t* out;             // [max_rows, n_out] bf16
  uint32_t* flags;
};

struct TcTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
  int32_t tile_start[kMaxGroups + 1];
  int32_t row0[kMaxGroups];
  int32_t count[kMaxGroups];
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + sizeof(TcTail);

struct Tile {
  int g, m0, n0;
};

__device__ __forceinline__ Tile decode_tile(const TcTail& s, int G, int bn, int t) {
  int lo = 0, hi = G;  // largest g with tile_start[g] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= t)
      lo = mid;
    else
      hi = mid;
  }
  const int local = t - s.tile_start[lo];
  const int mt = (s.count[lo] + BM - 1) / BM;
  Tile r;
  r.g = lo;
  r.n0 = (local / mt) * bn;
  r.m0 = (local % mt) * BM;
  return r;
}

__device__ __forceinline__ float silu_f32(float u) { return u / (1.0f + expf(-u)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const TcParams p) {
  constexpr int BN = MODE == MODE_SWIGLU ? MMA_N / 2 : MMA_N;  // output columns per tile
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * A_BYTES;
  TcTail& tl = *reinterpret_cast<TcTail*>(base + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.seg_off != nullptr ? p.G : 1;
  const int n_tiles = (p.n_out + BN - 1) / BN;
  const int KB = p.K / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_addr(&tl.full[s]), 1);
      mbar_init(smem_addr(&tl.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&tl.tfull[a]), 1);
      mbar_init(smem_addr(&tl.tempty[a]), 128);
    }
    mbar_init(smem_addr(&tl.drain), 1);
    tl.abort = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (MODE == MODE_SWIGLU) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&tl.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    // segment table -> per-group row range (clamped to the buffer) and tile prefix
    const int per = (G + 31) / 32;
    const int g_lo = min(G, lane * per), g_hi = min(G, g_lo + per);
    int local = 0;
    for (int g = g_lo; g < g_hi; ++g) {
      int r0 = 0, c = p.dense_rows;
      if (p.seg_off != nullptr) {
        r0 = p.seg_off[g];
        c = p.seg_count[g];
      }
      if (r0 < 0 || c < 0 || static_cast<int64_t>(r0) + c > p.max_rows) {
        atomicOr(p.flags, kFlagBadIndex);
        r0 = 0;
        c = 0;
      }
      tl.row0[g] = r0;
      tl.count[g] = c;
      local += (c + BM - 1) / BM * n_tiles;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g_lo; g < g_hi; ++g) {
      tl.tile_start[g] = run;
      run += (tl.count[g] + BM - 1) / BM * n_tiles;
    }
    if (lane == 31) tl.tile_start[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tl.tmem_base;
  const int total = tl.tile_start[G];
  volatile uint32_t* abort = &tl.abort;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t stage = 0, phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const Tile tile = decode_tile(tl, G, BN, t);
        const int a_row = tl.row0[tile.g] + tile.m0;
        const int b_row = tile.g * p.K;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_addr(&tl.full[stage]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          tma_load_2d(smem_addr(sA + stage * A_BYTES), &tmA, fb, kb * BK, a_row);
          const uint32_t bdst = smem_addr(sB + stage * B_BYTES);
          const int ky = b_row + kb * BK;
          if (MODE == MODE_SWIGLU) {
            tma_load_2d(bdst, &tmB0, fb, tile.n0, ky);
            tma_load_2d(bdst + B_CHUNK, &tmB0, fb, tile.n0 + 64, ky);
            tma_load_2d(bdst + 2 * B_CHUNK, &tmB1, fb, tile.n0, ky);
            tma_load_2d(bdst + 3 * B_CHUNK, &tmB1, fb, tile.n0 + 64, ky);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) tma_load_2d(bdst + i * B_CHUNK, &tmB0, fb, tile.n0 + 64 * i, ky);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every load issued by this thread has landed before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u)
          mbar_wait(smem_addr(&tl.full[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true, issued_any = false;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        if (!mbar_wait(smem_addr(&tl.tempty[acc]), acc_phase ^ 1u, abort, p.flags, kFlagTimeout)) break;
        tc_fence_after();
        issued_any = true;
        const uint32_t d_tmem = tmem_base + acc * MMA_N;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_addr(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            // A: K-major, advance 16 elements (32 bytes) inside the swizzle row
            const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            // B: MN-major, advance 16 K rows = two 8-row swizzle atoms (2048 bytes)
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, B_CHUNK, 1024);
            tc_mma_f16(d_tmem, adesc, bdesc, kIdesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(smem_addr(&tl.empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(smem_addr(&tl.tfull[acc]));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // all MMAs issued by this thread are complete before TMEM is released
      if (issued_any) {
        tc_commit(smem_addr(&tl.drain));
        mbar_wait(smem_addr(&tl.drain), 0u, nullptr, p.flags, kFlagTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31 belong to this warp
    const int r_in_tile = quad * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tile = decode_tile(tl, G, BN, t);
      if (!mbar_wait(smem_addr(&tl.tfull[acc]), acc_phase, abort, p.flags, kFlagTimeout)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * MMA_N;
      const int row = tile.m0 + r_in_tile;
      const bool valid = row < tl.count[tile.g];
      uint16_t* orow = p.out + (static_cast<int64_t>(tl.row0[tile.g]) + row) * p.n_out;
      if (MODE == MODE_SWIGLU) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + c, gv);
          tmem_ld32(tbase + BN + c, uv);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
              const float h1 = silu_f32(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            const int col = tile.n0 + c;
            if (col + 32 <= p.n_out) {
              uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
              for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            } else {
              for (int i = 0; i < 32 && col + i < p.n_out; ++i)
                orow[col + i] = static_cast<uint16_t>((pk[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            const int col = tile.n0 + c;
            if (col + 32 <= p.n_out) {
              uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
              for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            } else {
              for (int i = 0; i < 32 && col + i < p.n_out; ++i)
                orow[col + i] = static_cast<uint16_t>((pk[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&tl.tempty[acc]));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
template <int MODE>
cudaError_t set_smem_attr() {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(tc_ffn_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
  });
  return r;
}

template <int MODE>
cudaError_t launch_gemm(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const TcParams& p,
                        int64_t bound_tiles, cudaStream_t s) {
  cudaError_t e = set_smem_attr<MODE>();
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::min<int64_t>(device_sm_count(), std::max<int64_t>(bound_tiles, 1)));
  tc_ffn_gemm_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(A, B0, B1, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_bf16(const FfnArgs& a, cudaStream_t s) {
  if (a.max_rows <= 0 || a.G <= 0) return cudaSuccess;
  const bool dense = a.seg_off == nullptr;
  const uint64_t G = dense ? 1 : static_cast<uint64_t>(a.G);
  CUtensorMap mA1, mW1, mW3, mA2, mW2;
  if (!make_tma_2d_bf16(&mA1, a.a, a.d, a.max_rows, BK, BM) ||
      !make_tma_2d_bf16(&mW1, a.w1, a.f, G * a.d, 64, BK) || !make_tma_2d_bf16(&mW3, a.w3, a.f, G * a.d, 64, BK) ||
      !make_tma_2d_bf16(&mA2, a.h, a.f, a.max_rows, BK, BM) || !make_tma_2d_bf16(&mW2, a.w2, a.d, G * a.f, 64, BK))
    return cudaErrorInvalidValue;

  TcParams p{};
  p.seg_off = a.seg_off;
  p.seg_count = a.seg_count;
  p.G = static_cast<int>(G);
  p.dense_rows = a.dense_rows;
  p.max_rows = a.max_rows;
  p.flags = a.flags;
  const int64_t m_bound = (a.max_rows + BM - 1) / BM + (dense ? 0 : a.G);

  p.K = a.d;
  p.n_out = a.f;
  p.out = static_cast<uint16_t*>(a.h);
  cudaError_t e = launch_gemm<MODE_SWIGLU>(mA1, mW1, mW3, p, m_bound * ((a.f + 127) / 128), s);
  if (e != cudaSuccess) return e;

  p.K = a.f;
  p.n_out = a.d;
  p.out = static_cast<uint16_t*>(a.out);
  return launch_gemm<MODE_PLAIN>(mA2, mW2, mW2, p, m_bound * ((a.d + 255) / 256), s);
}

}  // namespace moe
