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
// Persistent, 192 threads per CTA, one CTA per SM:
//   warp 0 lane 0   producer: per K stage of 128 values (128 bytes per row),
//                   TMA loads of A and of the K-major weight rows, plus the
//                   stage's 512-byte scale atoms (A, and B rows 0-127 / 128-255);
//   warp 1          allocates all 512 TMEM columns; lane 0 copies the scale
//                   atoms into TMEM (tcgen05.cp) and issues four K=32 MMAs whose
//                   scale-factor id picks the 32-value block;
//   warps 2-5       epilogue (tcgen05.ld, SwiGLU + FP8 quantization or bf16).
// CG = 1: a CTA computes a 128 x 256 tile alone (M=128 MMA), four stages of
//   16 KB A + 32 KB B + 1.5 KB scales.
// CG = 2: a cluster of two CTAs computes a 256 x 256 tile with one
//   cta_group::2 MMA issued by the even CTA; each CTA stages its own 128 rows of
//   A, its own 128 rows of B (SwiGLU: CTA 0 the W1 rows, CTA 1 the W3 rows) and
//   the scales of its A rows and of all 256 B rows (the B scales are needed by
//   both halves of the tile), six stages of 33.5 KB.  Every load is a TMA tensor
//   load counted on the even CTA's barrier; the MMA commits to both CTAs'
//   barriers; both epilogues release the accumulator on the even CTA's barrier.
// TMEM: accumulator 0 at columns [0, 256), accumulator 1 at [224, 480) and two
// scale sets at [480, 504), used by alternate stages so that the copy of a
// stage's scales need not wait for the previous stage's MMAs to read theirs.  The two accumulators share 32 columns so that both fit
// beside the scales; the epilogue drains buffer 0 from its last 32 columns
// down and buffer 1 from its first 32 columns up, and releases the next tile's
// MMA as soon as the shared columns are read.
// Every mbarrier wait is bounded; on a timeout the kernel raises
// MOE_FLAG_WAIT_TIMEOUT, waits (bounded) for its own copies and MMAs in flight,
// frees its TMEM and returns.
#include <cuda_fp8.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                    // rows per CTA
constexpr int BK = 128;                    // K per stage (bytes per row)
constexpr int MMA_N = 256;
constexpr int MMA_K = 32;
constexpr int A_BYTES = BM * BK;           // 16 KB
constexpr int B_HALF = 128 * BK;           // 16 KB: 128 weight rows
constexpr int SF_ATOM = 512;               // scales of 128 rows x 4 K blocks
constexpr int SF_BYTES = 3 * SF_ATOM;      // A atom + two B atoms
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr uint32_t kAcc1Col = 224;         // accumulator 1 starts here (shares [224, 256))
constexpr uint32_t kSfaCol = 480;          // scale set 0; set 1 is 12 columns further
constexpr uint32_t kSfbCol = 484;          // two atoms: rows 0-127 then 128-255 of B
constexpr uint32_t kSfSet = 12;            // columns of one scale set (two sets: [480, 504))
constexpr int kMaxGroups = 256;

enum { MODE_SWIGLU = 0, MODE_PLAIN = 1 };

template <int CG>
struct Cfg {
  static constexpr int B_BYTES = CG == 1 ? 2 * B_HALF : B_HALF;   // B rows staged by one CTA
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SF_BYTES;
  static constexpr int STAGES = CG == 1 ? 4 : 6;
  static constexpr int TILE_M = BM * CG;
};

struct MxParams {
  const int32_t* seg_off;
  const int32_t* seg_count;
  int G;
  int64_t max_rows;
  int K;                     // reduction length (multiple of 128)
  int n_out;                 // output columns (multiple of 128)
  const uint8_t* a_sf;       // scales of A (CG = 1: bulk copies; CG = 2: TMA maps)
  const uint8_t* b0_sf;      // scales of B (W1 or W2)
  const uint8_t* b1_sf;      // scales of W3 (SwiGLU)
  uint8_t* out8;             // SwiGLU: h codes [max_rows, n_out]
  uint8_t* out8_sf;          // SwiGLU: h scales (n_out / 32 per row)
  uint16_t* out16;           // plain: bf16 [max_rows, n_out]
  uint64_t wait_ns;          // bound of the pipeline waits (those that also watch the abort flag);
                             // the waits that drain copies and MMAs in flight keep kWaitLimitNs
  uint32_t* flags;
};

struct MxTail {
  uint64_t full[6];
  uint64_t empty[6];
  uint64_t tfull[2];
  uint64_t drained;          // epilogue read the columns shared with the next tile's accumulator
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
  int32_t tile_start[kMaxGroups + 1];
  int32_t row0[kMaxGroups];
  int32_t count[kMaxGroups];
};

template <int CG>
constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(Cfg<CG>::STAGES) * Cfg<CG>::STAGE_BYTES + sizeof(MxTail);
}

struct Tile {
  int g, m0, n0;
};

__device__ __forceinline__ Tile decode_tile(const MxTail& s, int G, int bn, int tile_m, int t) {
  int lo = 0, hi = G;  // largest g with tile_start[g] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= t)
      lo = mid;
    else
      hi = mid;
  }
  const int local = t - s.tile_start[lo];
  const int mt = (s.count[lo] + tile_m - 1) / tile_m;
  Tile r;
  r.g = lo;
  r.n0 = (local / mt) * bn;
  r.m0 = (local % mt) * tile_m;
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

// Scale atoms as TMA tensors (CG = 2): the scale buffer viewed as [atoms * 4]
// rows of 128 bytes, one atom = a 4-row box.
template <int MODE, int CG>
__global__ void __launch_bounds__(kThreads, 1)
    tc_mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmSA,
                      const __grid_constant__ CUtensorMap tmSB0, const __grid_constant__ CUtensorMap tmSB1,
                      const MxParams p) {
  using C = Cfg<CG>;
  constexpr int BN = MODE == MODE_SWIGLU ? MMA_N / 2 : MMA_N;  // output columns per tile
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + C::STAGES * A_BYTES;
  uint8_t* sSF = sB + C::STAGES * C::B_BYTES;
  MxTail& tl = *reinterpret_cast<MxTail*>(sSF + C::STAGES * SF_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;   // 0: this CTA issues the MMAs
  const int unit = CG == 2 ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int n_units = CG == 2 ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int G = p.G;
  const int n_tiles = (p.n_out + BN - 1) / BN;
  const int KT = p.K / BK;            // K stages (= scale atoms per 128-row tile)
  const int NT = p.n_out / 128;       // 128-row tiles of one expert's weight

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_addr(&tl.full[s]), 1);
      mbar_init(smem_addr(&tl.empty[s]), 1);
    }
    mbar_init(smem_addr(&tl.tfull[0]), 1);
    mbar_init(smem_addr(&tl.tfull[1]), 1);
    mbar_init(smem_addr(&tl.drained), 128 * CG);
    mbar_init(smem_addr(&tl.drain), 1);
    tl.abort = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (MODE == MODE_SWIGLU) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(smem_addr(&tl.tmem_base), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(&tl.tmem_base), kTmemCols);
      tmem_relinquish();
    }
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
      local += (c + C::TILE_M - 1) / C::TILE_M * n_tiles;
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
      run += (tl.count[g] + C::TILE_M - 1) / C::TILE_M * n_tiles;
    }
    if (lane == 31) tl.tile_start[G] = incl;
  }
  tc_fence_before();
  if (CG == 2)
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA signal
  else
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
        const Tile tile = decode_tile(tl, G, BN, C::TILE_M, t);
        const int a_row = tl.row0[tile.g] + tile.m0 + static_cast<int>(rank) * BM;
        // B rows this CTA stages: CG = 1 all 256; CG = 2 its 128
        const int b_row = tile.g * p.n_out + tile.n0 + (MODE == MODE_PLAIN ? static_cast<int>(rank) * 128 : 0);
        const int nt0 = tile.n0 / 128;
        const int nt1 = MODE == MODE_SWIGLU ? nt0 : min(nt0 + 1, NT - 1);
        const int64_t sfa_atom = static_cast<int64_t>(a_row / BM) * KT;
        const int64_t sfb0_atom = (static_cast<int64_t>(tile.g) * NT + nt0) * KT;
        const int64_t sfb1_atom = (static_cast<int64_t>(tile.g) * NT + nt1) * KT;
        for (int kb = 0; kb < KT; ++kb) {
          if (!mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_addr(&tl.full[stage]);
          const uint32_t a_dst = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_addr(sB + stage * C::B_BYTES);
          const uint32_t sf_dst = smem_addr(sSF + stage * SF_BYTES);
          if (CG == 1) {
            mbar_arrive_expect_tx(fb_local, C::STAGE_BYTES);
            tma_load_2d(a_dst, &tmA, fb_local, kb * BK, a_row);
            if (MODE == MODE_SWIGLU) {
              tma_load_2d(b_dst, &tmB0, fb_local, kb * BK, b_row);           // W1 rows n0 .. n0+127
              tma_load_2d(b_dst + B_HALF, &tmB1, fb_local, kb * BK, b_row);  // W3 rows n0 .. n0+127
            } else {
              tma_load_2d(b_dst, &tmB0, fb_local, kb * BK, b_row);
              tma_load_2d(b_dst + B_HALF, &tmB0, fb_local, kb * BK, b_row + 128);
            }
            bulk_load(sf_dst, p.a_sf + (sfa_atom + kb) * SF_ATOM, SF_ATOM, fb_local);
            bulk_load(sf_dst + SF_ATOM, p.b0_sf + (sfb0_atom + kb) * SF_ATOM, SF_ATOM, fb_local);
            bulk_load(sf_dst + 2 * SF_ATOM, (MODE == MODE_SWIGLU ? p.b1_sf : p.b0_sf) + (sfb1_atom + kb) * SF_ATOM,
                      SF_ATOM, fb_local);
          } else {
            // both CTAs' bytes complete on the even CTA's barrier
            const uint32_t fb = rank == 0 ? fb_local : mapa_shared(fb_local, 0);
            if (rank == 0) mbar_arrive_expect_tx(fb_local, 2 * C::STAGE_BYTES);
            tma_load_2d_pair(a_dst, &tmA, fb, kb * BK, a_row);
            tma_load_2d_pair(b_dst, (MODE == MODE_SWIGLU && rank == 1) ? &tmB1 : &tmB0, fb, kb * BK, b_row);
            tma_load_2d_pair(sf_dst, &tmSA, fb, 0, static_cast<int>((sfa_atom + kb) * 4));
            tma_load_2d_pair(sf_dst + SF_ATOM, &tmSB0, fb, 0, static_cast<int>((sfb0_atom + kb) * 4));
            tma_load_2d_pair(sf_dst + 2 * SF_ATOM, MODE == MODE_SWIGLU ? &tmSB1 : &tmSB0, fb, 0,
                             static_cast<int>((sfb1_atom + kb) * 4));
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every copy issued by this thread has landed before the CTA may exit: the
      // even CTA sees its barrier complete; the odd CTA sees the MMA that
      // consumed the load release the stage.
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
      // ---------------------------------------------------------------- MMA issuer
      uint32_t stage = 0, phase = 0, acc = 0, j = 0, sfset = 0;
      bool ok = true, issued_any = false;
      // Descriptors of stage 0 at K offset 0.  Their start-address field is the
      // shared address / 16 (14 bits, no carry below 256 KB), so a stage or a
      // 32-byte K step is a constant added to the descriptor: this thread's
      // instruction stream per K stage stays short next to the MMAs it feeds.
      const uint64_t adesc0 = smem_desc_sw128(smem_addr(sA), 16, 1024);
      const uint64_t bdesc0 = smem_desc_sw128(smem_addr(sB), 16, 1024);
      const uint64_t sfdesc0 = smem_desc_plain(smem_addr(sSF), 16, 128);
      for (int t = unit; ok && t < total; t += n_units, ++j) {
        // the previous tile's epilogue has read the columns this accumulator shares with it
        if (j > 0 && !mbar_wait(smem_addr(&tl.drained), (j - 1) & 1u, abort, p.flags, kFlagTimeout, p.wait_ns))
          break;
        tc_fence_after();
        issued_any = true;
        const uint32_t d_tmem = tmem_base + (acc ? kAcc1Col : 0u);
        for (int kb = 0; kb < KT; ++kb) {
          if (!mbar_wait(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc_s = adesc0 + stage * static_cast<uint32_t>(A_BYTES >> 4);
          const uint64_t bdesc_s = bdesc0 + stage * static_cast<uint32_t>(C::B_BYTES >> 4);
          const uint64_t sfdesc_s = sfdesc0 + stage * static_cast<uint32_t>(SF_BYTES >> 4);
          // scale atoms -> this stage's TMEM scale set (executed in order with
          // the MMAs issued around them)
          const uint32_t sfa_col = tmem_base + kSfaCol + sfset * kSfSet;
          const uint32_t sfb_col = tmem_base + kSfbCol + sfset * kSfSet;
          sfset ^= 1u;
          constexpr uint32_t kAtom16 = SF_ATOM >> 4;
          if (CG == 2) {
            tc_cp_32x128b_x4_pair(sfa_col, sfdesc_s);
            tc_cp_32x128b_x4_pair(sfb_col, sfdesc_s + kAtom16);
            tc_cp_32x128b_x4_pair(sfb_col + 4, sfdesc_s + 2 * kAtom16);
          } else {
            tc_cp_32x128b_x4(sfa_col, sfdesc_s);
            tc_cp_32x128b_x4(sfb_col, sfdesc_s + kAtom16);
            tc_cp_32x128b_x4(sfb_col + 4, sfdesc_s + 2 * kAtom16);
          }
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            // A and B K-major: advance 32 values (32 bytes) inside the swizzle row
            const uint64_t adesc = adesc_s + static_cast<uint64_t>(kk * 2);
            const uint64_t bdesc = bdesc_s + static_cast<uint64_t>(kk * 2);
            const uint32_t sel = static_cast<uint32_t>(kk) << 30;   // scale byte kk of each word
            const uint32_t idesc = idesc_mxf8(C::TILE_M, MMA_N, static_cast<uint32_t>(kk));
            if (CG == 2)
              tc_mma_mxf8_pair(d_tmem, adesc, bdesc, idesc, sfa_col | sel, sfb_col | sel, (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma_mxf8(d_tmem, adesc, bdesc, idesc, sfa_col | sel, sfb_col | sel, (kb | kk) != 0 ? 1u : 0u);
          }
          if (CG == 2) {
            tc_commit_pair_both(smem_addr(&tl.empty[stage]));
          } else {
            tc_commit(smem_addr(&tl.empty[stage]));
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (CG == 2) {
          tc_commit_pair_both(smem_addr(&tl.tfull[acc]));
        } else {
          tc_commit(smem_addr(&tl.tfull[acc]));
        }
        acc ^= 1u;
      }
      if (issued_any) {
        if (CG == 2)
          tc_commit_pair(smem_addr(&tl.drain));
        else
          tc_commit(smem_addr(&tl.drain));
        mbar_wait(smem_addr(&tl.drain), 0u, nullptr, p.flags, kFlagTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31 belong to this warp
    const int r_in_tile = static_cast<int>(rank) * BM + quad * 32 + lane;
    const uint32_t drained = smem_addr(&tl.drained);
    uint32_t acc = 0, acc_phase = 0;
    for (int t = unit; t < total; t += n_units) {
      const Tile tile = decode_tile(tl, G, BN, C::TILE_M, t);
      if (!mbar_wait(smem_addr(&tl.tfull[acc]), acc_phase, abort, p.flags, kFlagTimeout, p.wait_ns)) break;
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
            if (CG == 2 && rank != 0)
              mbar_arrive_cluster(mapa_shared(drained, 0));
            else
              mbar_arrive(drained);
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
            if (CG == 2 && rank != 0)
              mbar_arrive_cluster(mapa_shared(drained, 0));
            else
              mbar_arrive(drained);
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
  if (CG == 2)
    cluster_sync();  // the even CTA's MMAs (which write both CTAs' TMEM) have drained
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2)
      tmem_dealloc_pair(tmem_base, kTmemCols);
    else
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
// scale buffer of `rows` x K values as a TMA tensor: [atoms * 4 rows][128 bytes]
bool make_sf_map(CUtensorMap* m, const void* sf, int64_t rows, int K) {
  const uint64_t atoms = static_cast<uint64_t>((rows + 127) / 128) * (K / 128);
  return make_tma_2d_u8_plain(m, sf, 128, atoms * 4, 128, 4);
}

template <int MODE, int CG>
cudaError_t launch_gemm(const CUtensorMap* maps, const MxParams& p, int64_t bound_units, cudaStream_t s) {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(tc_mx_gemm_kernel<MODE, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes<CG>()));
  });
  if (r != cudaSuccess) return r;
  int units = device_sm_count() / CG;
  units = static_cast<int>(std::min<int64_t>(units, std::max<int64_t>(bound_units, 1)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units * CG), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<CG>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, tc_mx_gemm_kernel<MODE, CG>, &cfg) == cudaSuccess &&
        max_clusters > 0 && max_clusters < units)
      cfg.gridDim.x = static_cast<unsigned>(max_clusters * 2);
  }
  e = cudaLaunchKernelEx(&cfg, tc_mx_gemm_kernel<MODE, CG>, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Bound of the pipeline waits (moe_set_wait_limit_ns); 0 = kWaitLimitNs.
std::atomic<uint64_t> g_mx_wait_ns{0};

uint64_t mx_pipeline_wait_ns() {
  const uint64_t v = g_mx_wait_ns.load(std::memory_order_relaxed);
  return v == 0 ? kWaitLimitNs : v;
}

// CTA pairs halve the B operand each SM stages, but measured no faster here
// (Qwen3-shaped layer: 1.32 vs 1.23-1.32 ms; tensor pipe 52 % vs 58 % busy):
// the limit is the hand-over between tiles (the next tile's MMA waits until
// the epilogue has read the 32 accumulator columns the two buffers share), not
// the operand stream.  Single CTAs are the default; MOE_FFN_CTA_GROUP=1|2
// forces one variant (tests run both).
int choose_cta_group(const FfnMxArgs& a) {
  static int forced = [] {
    const char* v = std::getenv("MOE_FFN_CTA_GROUP");
    return v ? std::atoi(v) : 0;
  }();
  (void)a;
  if (forced == 1 || forced == 2) return forced;
  return 1;
}

template <int CG>
cudaError_t launch_pair(const FfnMxArgs& a, const CUtensorMap& mA1, const CUtensorMap& mW1, const CUtensorMap& mW3,
                        const CUtensorMap& mA2, const CUtensorMap& mW2, cudaStream_t s) {
  MxParams p{};
  p.seg_off = a.seg_off;
  p.seg_count = a.seg_count;
  p.G = a.G;
  p.max_rows = a.max_rows;
  p.flags = a.flags;
  p.wait_ns = mx_pipeline_wait_ns();
  const int64_t m_bound = (a.max_rows + Cfg<CG>::TILE_M - 1) / Cfg<CG>::TILE_M + a.G;
  CUtensorMap maps[6];
  // GEMM1: K = d, n_out = f, h codes and scales out
  p.K = a.d;
  p.n_out = a.f;
  p.a_sf = a.a_sf;
  p.b0_sf = a.w1_sf;
  p.b1_sf = a.w3_sf;
  p.out8 = a.h;
  p.out8_sf = a.h_sf;
  maps[0] = mA1;
  maps[1] = mW1;
  maps[2] = mW3;
  if (CG == 2 && (!make_sf_map(&maps[3], a.a_sf, a.max_rows, a.d) ||
                  !make_sf_map(&maps[4], a.w1_sf, static_cast<int64_t>(a.G) * a.f, a.d) ||
                  !make_sf_map(&maps[5], a.w3_sf, static_cast<int64_t>(a.G) * a.f, a.d)))
    return cudaErrorInvalidValue;
  if (CG == 1) maps[3] = maps[4] = maps[5] = mA1;   // unused
  cudaError_t e = launch_gemm<MODE_SWIGLU, CG>(maps, p, m_bound * (a.f / 128), s);
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
  maps[0] = mA2;
  maps[1] = mW2;
  maps[2] = mW2;
  if (CG == 2 && (!make_sf_map(&maps[3], a.h_sf, a.max_rows, a.f) ||
                  !make_sf_map(&maps[4], a.w2_sf, static_cast<int64_t>(a.G) * a.d, a.f)))
    return cudaErrorInvalidValue;
  if (CG == 2) maps[5] = maps[4];
  if (CG == 1) maps[3] = maps[4] = maps[5] = mA2;
  return launch_gemm<MODE_PLAIN, CG>(maps, p, m_bound * ((a.d + 255) / 256), s);
}

}  // namespace

void set_mx_pipeline_wait_ns(uint64_t ns) { g_mx_wait_ns.store(ns, std::memory_order_relaxed); }

cudaError_t launch_ffn_mx(const FfnMxArgs& a, cudaStream_t s) {
  if (a.max_rows <= 0 || a.G <= 0) return cudaSuccess;
  const uint64_t G = static_cast<uint64_t>(a.G);
  const int cg = choose_cta_group(a);
  CUtensorMap mA1, mW1, mW3, mA2, mW2;   // B boxes are 128 weight rows
  if (!make_tma_2d_u8(&mA1, a.a, a.d, a.max_rows, BK, BM) || !make_tma_2d_u8(&mW1, a.w1, a.d, G * a.f, BK, 128) ||
      !make_tma_2d_u8(&mW3, a.w3, a.d, G * a.f, BK, 128) || !make_tma_2d_u8(&mA2, a.h, a.f, a.max_rows, BK, BM) ||
      !make_tma_2d_u8(&mW2, a.w2, a.f, G * a.d, BK, 128))
    return cudaErrorInvalidValue;
  if (cg == 2) return launch_pair<2>(a, mA1, mW1, mW3, mA2, mW2, s);
  return launch_pair<1>(a, mA1, mW1, mW3, mA2, mW2, s);
}

cudaError_t launch_mx_quantize_weight(const uint16_t* w, int64_t G, int K, int N, uint8_t* codes, uint8_t* sf,
                                      cudaStream_t s) {
  if (G <= 0) return cudaSuccess;
  mx_quantize_weight_kernel<<<dim3(K / 32, N / 128, static_cast<unsigned>(G)), 128, 0, s>>>(w, K, N, codes, sf);
  return cudaGetLastError();
}

}  // namespace moe
