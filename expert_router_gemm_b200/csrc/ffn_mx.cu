// Block-scaled FP8 grouped SwiGLU FFN on the 5th-generation tensor cores.
//
// FP8 expert GEMMs with bf16 activations at the layer boundary ("MoE 训练加速实战：
// DeepEP + Grouped GeMM + Aux-Loss-Free" §9.1, precision row; §4.1-4.2 for the
// grouped GEMM, y_i = W_i x_i).  Operands are E4M3 codes with one power-of-two
// (E8M0) scale per 32 values along K, the block-scaled FP8 that sm_100a
// multiplies natively (tcgen05.mma kind::mxf8f6f4.block_scale): the scales are
// applied inside the MMA, so the fp32 accumulator holds the exact-operand sum.
//   GEMM1 (SWIGLU): h[r] = silu(xp[r] W1_e) * (xp[r] W3_e), quantized to FP8
//                   (blocks of 32 along f) in the epilogue -> codes + scales
//   GEMM2 (PLAIN):  out[r] = h[r] W2_e -> bf16
//
// Per CTA (one per SM, 192 threads), one 128 x 256 tile at a time:
//   warp 0 lane 0   producer: per K stage of 128 values (128 bytes per row),
//                   TMA loads of A (128 rows) and B (256 K-major weight rows,
//                   two boxes), plus three 512-byte scale atoms (bulk copies);
//   warp 1          allocates all 512 TMEM columns; lane 0 copies the stage's
//                   scale atoms into TMEM (tcgen05.cp) and issues four K=32 MMAs
//                   whose scale-factor id picks the 32-value block;
//   warps 2-5       epilogue (tcgen05.ld, SwiGLU + FP8 quantization or bf16).
// TMEM: accumulator 0 at columns [0, 256), accumulator 1 at [224, 480) and the
// scales at [480, 492).  The two accumulators share 32 columns so that both fit
// beside the scales; the epilogue drains buffer 0 from its last 32 columns
// down and buffer 1 from its first 32 columns up, and releases the next tile's
// MMA as soon as the shared columns are read.
// Every mbarrier wait is bounded; on a timeout the kernel raises
// MOE_FLAG_WAIT_TIMEOUT, waits (bounded) for its own copies and MMAs in flight,
// frees its TMEM and returns.
#include <cuda_fp8.h>

#include <algorithm>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                    // rows per tile
constexpr int BK = 128;                    // K per stage (bytes per row)
constexpr int MMA_N = 256;
constexpr int MMA_K = 32;
constexpr int A_BYTES = BM * BK;           // 16 KB
constexpr int B_HALF = 128 * BK;           // 16 KB: 128 weight rows
constexpr int B_BYTES = 2 * B_HALF;        // 32 KB
constexpr int SF_ATOM = 512;               // scales of 128 rows x 4 K blocks
constexpr int SF_BYTES = 3 * SF_ATOM;      // A atom + two B atoms
constexpr int STAGES = 4;
constexpr int STAGE_TX = A_BYTES + B_BYTES + SF_BYTES;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr uint32_t kAcc1Col = 224;         // accumulator 1 starts here (shares [224, 256))
constexpr uint32_t kSfaCol = 480;
constexpr uint32_t kSfbCol = 484;          // two atoms: rows 0-127 then 128-255 of B
constexpr int kMaxGroups = 256;

enum { MODE_SWIGLU = 0, MODE_PLAIN = 1 };

struct MxParams {
  const int32_t* seg_off;
  const int32_t* seg_count;
  int G;
  int64_t max_rows;
  int K;                     // reduction length (multiple of 128)
  int n_out;                 // output columns (multiple of 128)
  const uint8_t* a_sf;       // scales of A
  const uint8_t* b0_sf;      // scales of B (W1 or W2)
  const uint8_t* b1_sf;      // scales of W3 (SwiGLU)
  uint8_t* out8;             // SwiGLU: h codes [max_rows, n_out]
  uint8_t* out8_sf;          // SwiGLU: h scales (n_out / 32 per row)
  uint16_t* out16;           // plain: bf16 [max_rows, n_out]
  uint32_t* flags;
};

struct MxTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t drained;          // epilogue read the columns shared with the next tile's accumulator
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
  int32_t tile_start[kMaxGroups + 1];
  int32_t row0[kMaxGroups];
  int32_t count[kMaxGroups];
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(STAGES) * (A_BYTES + B_BYTES + SF_BYTES) + sizeof(MxTail);

struct Tile {
  int g, m0, n0;
};

__device__ __forceinline__ Tile decode_tile(const MxTail& s, int G, int bn, int t) {
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

__device__ __forceinline__ float silu_f32(float u) { return __fdividef(u, 1.0f + __expf(-u)); }

// four floats (already divided by the block scale) -> four E4M3 codes, round to
// nearest even, saturating; byte i holds value i
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmB1, const MxParams p) {
  constexpr int BN = MODE == MODE_SWIGLU ? MMA_N / 2 : MMA_N;  // output columns per tile
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * A_BYTES;
  uint8_t* sSF = sB + STAGES * B_BYTES;
  MxTail& tl = *reinterpret_cast<MxTail*>(sSF + STAGES * SF_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = static_cast<int>(blockIdx.x);
  const int n_units = static_cast<int>(gridDim.x);
  const int G = p.G;
  const int n_tiles = (p.n_out + BN - 1) / BN;
  const int KT = p.K / BK;            // K stages (= scale atoms per 128-row tile)
  const int NT = p.n_out / 128;       // 128-row tiles of one expert's weight

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_addr(&tl.full[s]), 1);
      mbar_init(smem_addr(&tl.empty[s]), 1);
    }
    mbar_init(smem_addr(&tl.tfull[0]), 1);
    mbar_init(smem_addr(&tl.tfull[1]), 1);
    mbar_init(smem_addr(&tl.drained), 128);
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
    const int per = (G + 31) / 32;
    const int g_lo = min(G, lane * per), g_hi = min(G, g_lo + per);
    int local = 0;
    for (int g = g_lo; g < g_hi; ++g) {
      int r0 = p.seg_off[g], c = p.seg_count[g];
      if (r0 < 0 || c < 0 || (r0 & (BM - 1)) != 0 || static_cast<int64_t>(r0) + c > p.max_rows) {
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
      for (int t = unit; ok && t < total; t += n_units) {
        const Tile tile = decode_tile(tl, G, BN, t);
        const int a_row = tl.row0[tile.g] + tile.m0;
        const int b_row = tile.g * p.n_out + tile.n0;
        const uint8_t* sfa = p.a_sf + static_cast<int64_t>(a_row / BM) * KT * SF_ATOM;
        const int nt0 = tile.n0 / 128;
        const int nt1 = MODE == MODE_SWIGLU ? nt0 : min(nt0 + 1, NT - 1);
        const uint8_t* sfb0 = p.b0_sf + (static_cast<int64_t>(tile.g) * NT + nt0) * KT * SF_ATOM;
        const uint8_t* sfb1 = (MODE == MODE_SWIGLU ? p.b1_sf : p.b0_sf) +
                              (static_cast<int64_t>(tile.g) * NT + nt1) * KT * SF_ATOM;
        for (int kb = 0; kb < KT; ++kb) {
          if (!mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_addr(&tl.full[stage]);
          const uint32_t a_dst = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_addr(sB + stage * B_BYTES);
          const uint32_t sf_dst = smem_addr(sSF + stage * SF_BYTES);
          mbar_arrive_expect_tx(fb, STAGE_TX);
          tma_load_2d(a_dst, &tmA, fb, kb * BK, a_row);
          if (MODE == MODE_SWIGLU) {
            tma_load_2d(b_dst, &tmB0, fb, kb * BK, b_row);           // W1 rows n0 .. n0+127
            tma_load_2d(b_dst + B_HALF, &tmB1, fb, kb * BK, b_row);  // W3 rows n0 .. n0+127
          } else {
            tma_load_2d(b_dst, &tmB0, fb, kb * BK, b_row);
            tma_load_2d(b_dst + B_HALF, &tmB0, fb, kb * BK, b_row + 128);
          }
          bulk_load(sf_dst, sfa + kb * SF_ATOM, SF_ATOM, fb);
          bulk_load(sf_dst + SF_ATOM, sfb0 + kb * SF_ATOM, SF_ATOM, fb);
          bulk_load(sf_dst + 2 * SF_ATOM, sfb1 + kb * SF_ATOM, SF_ATOM, fb);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy issued by this thread has landed before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(smem_addr(&tl.full[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, j = 0;
      bool ok = true, issued_any = false;
      for (int t = unit; ok && t < total; t += n_units, ++j) {
        // the previous tile's epilogue has read the columns this accumulator shares with it
        if (j > 0 && !mbar_wait(smem_addr(&tl.drained), (j - 1) & 1u, abort, p.flags, kFlagTimeout)) break;
        tc_fence_after();
        issued_any = true;
        const uint32_t d_tmem = tmem_base + (acc ? kAcc1Col : 0u);
        for (int kb = 0; kb < KT; ++kb) {
          if (!mbar_wait(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_addr(sB + stage * B_BYTES);
          const uint32_t sf_addr = smem_addr(sSF + stage * SF_BYTES);
          // scale atoms -> TMEM (executed in order with the MMAs issued around them)
          tc_cp_32x128b_x4(tmem_base + kSfaCol, smem_desc_plain(sf_addr, 16, 128));
          tc_cp_32x128b_x4(tmem_base + kSfbCol, smem_desc_plain(sf_addr + SF_ATOM, 16, 128));
          tc_cp_32x128b_x4(tmem_base + kSfbCol + 4, smem_desc_plain(sf_addr + 2 * SF_ATOM, 16, 128));
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            // A and B K-major: advance 32 values (32 bytes) inside the swizzle row
            const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            const uint32_t sel = static_cast<uint32_t>(kk) << 30;   // scale byte kk of each word
            tc_mma_mxf8(d_tmem, adesc, bdesc, idesc_mxf8(BM, MMA_N, static_cast<uint32_t>(kk)),
                        (tmem_base + kSfaCol) | sel, (tmem_base + kSfbCol) | sel, (kb | kk) != 0 ? 1u : 0u);
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
      (void)acc_phase;
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
    for (int t = unit; t < total; t += n_units) {
      const Tile tile = decode_tile(tl, G, BN, t);
      if (!mbar_wait(smem_addr(&tl.tfull[acc]), acc_phase, abort, p.flags, kFlagTimeout)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + (acc ? kAcc1Col : 0u);
      const int row = tile.m0 + r_in_tile;
      const bool valid = row < tl.count[tile.g];
      const int64_t grow = static_cast<int64_t>(tl.row0[tile.g]) + row;
      if (MODE == MODE_SWIGLU) {
        // pair q: gate columns [32q, 32q+32), up columns [128+32q, ...); one
        // pair = one block of 32 hidden units = one FP8 scale
#pragma unroll 1
        for (int it = 0; it < 4; ++it) {
          const int q = acc == 0 ? 3 - it : it;
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + 32 * q, gv);
          tmem_ld32(tbase + 128 + 32 * q, uv);
          tmem_ld_wait();
          if (it == 0) {
            tc_fence_before();
            mbar_arrive(smem_addr(&tl.drained));
          }
          if (valid) {
            float h[32];
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              h[i] = silu_f32(__uint_as_float(gv[i])) * __uint_as_float(uv[i]);
              amax = fmaxf(amax, fabsf(h[i]));
            }
            const int e = mx_exponent(amax);
            const float inv = mx_inv_scale(e);
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              w[i] = e4m3x4(h[4 * i] * inv, h[4 * i + 1] * inv, h[4 * i + 2] * inv, h[4 * i + 3] * inv);
            const int col = tile.n0 + 32 * q;
            uint4* dst = reinterpret_cast<uint4*>(p.out8 + grow * p.n_out + col);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            p.out8_sf[mx_sf_offset(grow, col / 32, p.n_out / 32)] = static_cast<uint8_t>(e + 127);
          }
        }
      } else {
        uint16_t* orow = p.out16 + grow * p.n_out;
#pragma unroll 1
        for (int it = 0; it < 8; ++it) {
          const int c = 32 * (acc == 0 ? 7 - it : it);
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (it == 0) {
            tc_fence_before();
            mbar_arrive(smem_addr(&tl.drained));
          }
          const int col = tile.n0 + c;
          if (valid && col < p.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) dst[s4] = make_uint4(pk[4 * s4], pk[4 * s4 + 1], pk[4 * s4 + 2], pk[4 * s4 + 3]);
          }
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- weight quantization
// grid (K/32, N/128, G), 128 threads: a [32 K] x [128 N] tile of one expert's
// weight; thread n quantizes the 32 values of column n (one block) and writes
// its 32 codes (K-major) and its scale byte.
__global__ void __launch_bounds__(128) mx_quantize_weight_kernel(const uint16_t* __restrict__ w, int K, int N,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ sf) {
  __shared__ uint16_t tile[32][128];
  const int64_t g = blockIdx.z;
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 128, n = threadIdx.x;
  const uint16_t* src = w + (g * K + k0) * static_cast<int64_t>(N) + n0;
#pragma unroll 4
  for (int k = 0; k < 32; ++k) tile[k][n] = src[static_cast<int64_t>(k) * N + n];
  __syncthreads();
  float v[32];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    v[k] = __uint_as_float(static_cast<uint32_t>(tile[k][n]) << 16);
    amax = fmaxf(amax, fabsf(v[k]));
  }
  const int e = mx_exponent(amax);
  const float inv = mx_inv_scale(e);
  uint32_t q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = e4m3x4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv, v[4 * i + 3] * inv);
  const int64_t row = g * N + n0 + n;  // K-major row of the output
  uint4* dst = reinterpret_cast<uint4*>(codes + row * K + k0);
  dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
  dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
  sf[mx_sf_offset(row, k0 / 32, K / 32)] = static_cast<uint8_t>(e + 127);
}

// ---------------------------------------------------------------- host side
template <int MODE>
cudaError_t launch_gemm(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const MxParams& p,
                        int64_t bound_units, cudaStream_t s) {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(tc_mx_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
  });
  if (r != cudaSuccess) return r;
  const int units = static_cast<int>(std::min<int64_t>(device_sm_count(), std::max<int64_t>(bound_units, 1)));
  tc_mx_gemm_kernel<MODE><<<units, kThreads, kSmemBytes, s>>>(A, B0, B1, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_mx(const FfnMxArgs& a, cudaStream_t s) {
  if (a.max_rows <= 0 || a.G <= 0) return cudaSuccess;
  const uint64_t G = static_cast<uint64_t>(a.G);
  CUtensorMap mA1, mW1, mW3, mA2, mW2;
  if (!make_tma_2d_u8(&mA1, a.a, a.d, a.max_rows, BK, BM) || !make_tma_2d_u8(&mW1, a.w1, a.d, G * a.f, BK, 128) ||
      !make_tma_2d_u8(&mW3, a.w3, a.d, G * a.f, BK, 128) || !make_tma_2d_u8(&mA2, a.h, a.f, a.max_rows, BK, BM) ||
      !make_tma_2d_u8(&mW2, a.w2, a.f, G * a.d, BK, 128))
    return cudaErrorInvalidValue;
  MxParams p{};
  p.seg_off = a.seg_off;
  p.seg_count = a.seg_count;
  p.G = a.G;
  p.max_rows = a.max_rows;
  p.flags = a.flags;
  const int64_t m_bound = (a.max_rows + BM - 1) / BM + a.G;
  // GEMM1: K = d, n_out = f, h codes and scales out
  p.K = a.d;
  p.n_out = a.f;
  p.a_sf = a.a_sf;
  p.b0_sf = a.w1_sf;
  p.b1_sf = a.w3_sf;
  p.out8 = a.h;
  p.out8_sf = a.h_sf;
  cudaError_t e = launch_gemm<MODE_SWIGLU>(mA1, mW1, mW3, p, m_bound * (a.f / 128), s);
  if (e != cudaSuccess) return e;
  // GEMM2: K = f, n_out = d, bf16 out
  p.K = a.f;
  p.n_out = a.d;
  p.a_sf = a.h_sf;
  p.b0_sf = a.w2_sf;
  p.b1_sf = a.w2_sf;
  p.out8 = nullptr;
  p.out8_sf = nullptr;
  p.out16 = static_cast<uint16_t*>(a.out);
  return launch_gemm<MODE_PLAIN>(mA2, mW2, mW2, p, m_bound * ((a.d + 255) / 256), s);
}

cudaError_t launch_mx_quantize_weight(const uint16_t* w, int64_t G, int K, int N, uint8_t* codes, uint8_t* sf,
                                      cudaStream_t s) {
  if (G <= 0) return cudaSuccess;
  mx_quantize_weight_kernel<<<dim3(K / 32, N / 128, static_cast<unsigned>(G)), 128, 0, s>>>(w, K, N, codes, sf);
  return cudaGetLastError();
}

}  // namespace moe
