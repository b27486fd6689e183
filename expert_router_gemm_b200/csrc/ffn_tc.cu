// bf16 grouped SwiGLU FFN on the 5th-generation tensor cores (sm_100a).
//
// "MoE 训练加速实战：DeepEP + Grouped GeMM + Aux-Loss-Free" §4.1-4.2: one kernel
// serves every expert (y_i = W_i x_i), instead of one GEMM launch per expert,
// and tiles are formed per expert.  Two launches of one persistent kernel:
//   GEMM1 (SWIGLU): h[r] = silu(xp[r] W1_e) * (xp[r] W3_e)  -> bf16
//   GEMM2 (PLAIN):  out[r] = h[r] W2_e                       -> bf16
//
// Per CTA (one per SM, 192 threads):
//   warp 0          TMA producer: A slab 128 x 64 (K-major rows of the permuted
//                   activations) and B slab 64 x (256/CG) (rows of the row-major
//                   weight, i.e. MN-major), 128-byte swizzle, multi-stage ring.
//                   Lane 0 loads a permuted-row A slab as one tile.  Given a
//                   row -> token table instead (a layer pass whose dispatch
//                   copies no rows, MOE_GATHER=lsu|tma), the 32 lanes gather the
//                   slab's 128 token rows straight from x, as 16-byte cp.async
//                   copies or four rows per tile::gather4 load.
//   warp 1          allocates 512 TMEM columns (two accumulators, so the
//                   epilogue of tile i overlaps the main loop of tile i+1);
//                   lane 0 issues tcgen05.mma kind::f16, K=16, fp32 accumulator.
//   warps 2-5       epilogue: tcgen05.ld of the accumulator rows, SwiGLU in fp32
//                   (gate = columns 0-127, up = columns 128-255 of one tile, so
//                   both halves of a hidden unit meet in one thread), one
//                   rounding to bf16, stores of the valid rows.
// CG = 1: each CTA computes a 128 x 256 accumulator tile alone (M=128 MMA).
// CG = 2: a cluster of two CTAs on two SMs computes a 256 x 256 tile with one
//   cta_group::2 MMA (M=256) issued by the even CTA: each CTA stages its own 128
//   rows of A and its own 128 columns of B (for SwiGLU: CTA 0 the W1 columns,
//   CTA 1 the W3 columns), so per SM the operand traffic per flop is 2/3 of
//   CG = 1 and seven 32 KB stages fit instead of four 48 KB ones.  Both CTAs'
//   loads count on the even CTA's barrier, its MMA commits to both CTAs'
//   barriers, and both epilogues release the accumulator on the even CTA's
//   barrier.  A pair tile covers 256 rows of one expert; an expert with an odd
//   number of 128-row tiles leaves the second CTA's half of its last pair tile
//   partly or fully outside the segment (computed, not stored).
// Tiles are ordered (expert, N tile, M tile) with M fastest, so CTAs running at
// the same time share weight slabs in L2; every CTA derives the tile list from
// the device-side segment table, so no host synchronisation is needed.
// Every mbarrier wait is bounded; on a timeout the kernel raises
// MOE_FLAG_WAIT_TIMEOUT, waits (bounded) for its own copies and MMAs in flight,
// frees its TMEM and returns.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                    // rows per CTA (A slab rows)
constexpr int BK = 64;                     // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int MMA_N = 256;                 // accumulator columns per tile
constexpr int MMA_K = 16;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_CHUNK = 64 * BK * 2;       // 8 KB: 64 output columns x 64 K rows
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * MMA_N;
constexpr int kMaxGroups = 256;

enum { MODE_SWIGLU = 0, MODE_PLAIN = 1 };
enum { A_TILE = 0, A_GATHER_TMA = 1, A_GATHER_LSU = 2 };

template <int CG>
struct Cfg {
  static constexpr int B_CHUNKS = 4 / CG;                   // 64-column chunks of B per CTA
  static constexpr int B_BYTES = B_CHUNKS * B_CHUNK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // per CTA
  static constexpr int STAGES = CG == 1 ? 4 : 7;
  static constexpr int TILE_M = BM * CG;                    // accumulator rows of one (pair) tile
  static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, MMA_N, /*b_mn_major=*/1);
};

struct TcParams {
  const int32_t* seg_off;    // [G+1] or nullptr (one dense group of dense_rows rows)
  const int32_t* seg_count;  // [G]
  int G;
  int dense_rows;
  int64_t max_rows;          // rows of the A and output buffers
  int K;                     // reduction length (multiple of 64)
  int n_out;                 // output columns
  const int32_t* a_token;    // non-null: A row r (absolute) is row a_token[r] of a_src [a_token_rows, K]
                             // (rows past a group's count read row 0; indices outside a_src too)
  const void* a_src;         //   the gathered tensor (bf16), also under tmA (one-row boxes)
  int a_token_rows;
  int a_gather;              //   A_GATHER_TMA or A_GATHER_LSU
  uint16_t* out;             // [max_rows, n_out] bf16
  uint16_t* save_g;          // SwiGLU, optional: gate and up pre-activations [max_rows, n_out]
  uint16_t* save_u;          //   (bf16), kept for the backward pass
  int v8;                    // output rows start on 32-byte boundaries: 32-byte stores
  uint64_t wait_ns;          // bound of the pipeline waits (those that also watch the abort flag);
                             // the waits that drain copies and MMAs in flight keep kWaitLimitNs
  uint32_t* flags;
};

struct TcTail {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t afull[8];   // odd CTA of a pair: its cp.async A slab of the stage has landed
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
  int32_t tile_start[kMaxGroups + 1];
};

template <int CG>
constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(Cfg<CG>::STAGES) * Cfg<CG>::STAGE_BYTES + sizeof(TcTail);
}

struct Tile {
  int g, m0, n0;
};

// The rows [row0, row0 + count) of group g in the A / output buffers, read
// from the segment table (L2-resident, a few loads per tile); a group outside
// the buffers counts as empty (the prologue raises the bad-index flag for it).
__device__ __forceinline__ int2 group_rows(const TcParams& p, int g) {
  int r0 = 0, c = p.dense_rows;
  if (p.seg_off != nullptr) {
    r0 = __ldg(p.seg_off + g);
    c = __ldg(p.seg_count + g);
  }
  if (r0 < 0 || c < 0 || static_cast<int64_t>(r0) + c > p.max_rows) {
    r0 = 0;
    c = 0;
  }
  return make_int2(r0, c);
}

// tile t -> (group, first row of the (pair) tile, first output column)
__device__ __forceinline__ Tile decode_tile(const TcTail& s, const TcParams& p, int G, int bn, int tile_m, int t) {
  int lo = 0, hi = G;  // largest g with tile_start[g] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= t)
      lo = mid;
    else
      hi = mid;
  }
  const int local = t - s.tile_start[lo];
  const int mt = (group_rows(p, lo).y + tile_m - 1) / tile_m;
  Tile r;
  r.g = lo;
  r.n0 = (local / mt) * bn;
  r.m0 = (local % mt) * tile_m;
  return r;
}

// silu(u) = u / (1 + e^-u) with the fast exponential and division: the result is
// rounded to bf16 (8 significant bits), far above their fp32 error.  For very
// negative u, e^-u overflows to inf and the quotient is -0.
__device__ __forceinline__ float silu_f32(float u) { return __fdividef(u, 1.0f + __expf(-u)); }

__device__ __forceinline__ void store_row32(uint16_t* orow, int col, int n_out, const uint32_t (&pk)[16],
                                            bool v8) {
  if (v8 && col + 32 <= n_out) {  // two 32-byte stores: each sector is written whole, once
    uint32_t* dst = reinterpret_cast<uint32_t*>(orow + col);
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(pk[0]), "r"(pk[1]),
                 "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]), "r"(pk[7])
                 : "memory");
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 8), "r"(pk[8]), "r"(pk[9]),
                 "r"(pk[10]), "r"(pk[11]), "r"(pk[12]), "r"(pk[13]), "r"(pk[14]), "r"(pk[15])
                 : "memory");
  } else if (col + 32 <= n_out) {
    uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (col + i < n_out) orow[col + i] = static_cast<uint16_t>((pk[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu);
  }
}

// The B operand of one K slab, as this CTA loads it: 64-column chunk i comes
// from tensor map b_box_map(...) at column b_box_col(...).
//   CG = 1, SwiGLU: W1 columns n0, n0+64 then W3 columns n0, n0+64
//   CG = 1, plain:  W2 columns n0 + 64 i, i < 4
//   CG = 2, SwiGLU: CTA 0 the two W1 chunks, CTA 1 the two W3 chunks
//   CG = 2, plain:  CTA r the chunks at n0 + 128 r and n0 + 128 r + 64
template <int MODE, int CG>
__device__ __forceinline__ const CUtensorMap* b_box_map(const CUtensorMap* b0, const CUtensorMap* b1, uint32_t rank,
                                                       int i) {
  if (MODE != MODE_SWIGLU) return b0;
  if (CG == 1) return i < 2 ? b0 : b1;
  return rank == 0 ? b0 : b1;
}
template <int MODE, int CG>
__device__ __forceinline__ int b_box_col(int n0, uint32_t rank, int i) {
  if (CG == 1) return MODE == MODE_SWIGLU ? n0 + 64 * (i & 1) : n0 + 64 * i;
  return MODE == MODE_SWIGLU ? n0 + 64 * i : n0 + 128 * static_cast<int>(rank) + 64 * i;
}

template <int MODE, int CG, int AMODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const TcParams p) {
  using C = Cfg<CG>;
  constexpr int BN = MODE == MODE_SWIGLU ? MMA_N / 2 : MMA_N;  // output columns per tile
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + C::STAGES * A_BYTES;
  TcTail& tl = *reinterpret_cast<TcTail*>(base + C::STAGES * C::STAGE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;  // 0: this CTA issues the MMAs
  const int unit = CG == 2 ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int n_units = CG == 2 ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int G = p.seg_off != nullptr ? p.G : 1;
  const int n_tiles = (p.n_out + BN - 1) / BN;
  const int KB = p.K / BK;

  if (warp == 0 && lane == 0) {
    // full: the expect-tx arrival; with a cp.async slab also one arrival per
    // producer lane, and on a pair one relayed arrival for the odd CTA's slab
    // (counted on afull, 32 lanes, in the odd CTA)
    const uint32_t full_count = AMODE == A_GATHER_LSU ? (CG == 2 ? 34u : 33u) : 1u;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_addr(&tl.full[s]), full_count);
      mbar_init(smem_addr(&tl.empty[s]), 1);
      mbar_init(smem_addr(&tl.afull[s]), 32);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&tl.tfull[a]), 1);
      mbar_init(smem_addr(&tl.tempty[a]), 128 * CG);
    }
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
  // the kernel before this one (the dispatch, or GEMM1 for GEMM2) has finished
  // and its rows and segment table are visible; the next kernel may launch
  grid_dep_wait();
  grid_dep_launch();
  if (warp == 2) {
    // segment table -> per-group row range (clamped to the buffer) and tile prefix
    const int per = (G + 31) / 32;
    const int g_lo = min(G, lane * per), g_hi = min(G, g_lo + per);
    int local = 0;
    for (int g = g_lo; g < g_hi; ++g) {
      if (p.seg_off != nullptr) {
        const int r0 = p.seg_off[g], c = p.seg_count[g];
        if (r0 < 0 || c < 0 || static_cast<int64_t>(r0) + c > p.max_rows) atomicOr(p.flags, kFlagBadIndex);
      }
      local += (group_rows(p, g).y + C::TILE_M - 1) / C::TILE_M * n_tiles;
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
      run += (group_rows(p, g).y + C::TILE_M - 1) / C::TILE_M * n_tiles;
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
    // ------------------------------------------------------------------ producer
    // A arrives one of three ways: a slab of permuted rows as one TMA tile
    // (lane 0); or, with a row -> token table, the slab's 128 token rows of x
    // gathered by the whole warp, either as tile::gather4 TMA loads (lane i:
    // rows 4i..4i+3) or as 16-byte cp.async copies into the swizzled slab (lane
    // i: chunk i % 8 of rows i / 8, i / 8 + 4, ...), each lane arriving on the
    // stage's barrier when its copies have landed.  Lane 0 waits for free
    // stages, posts the expected TMA bytes and loads B.
    constexpr int amode = AMODE;
    if (amode != A_TILE || lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int t = unit; ok && t < total; t += n_units) {
        const Tile tile = decode_tile(tl, p, G, BN, C::TILE_M, t);
        const int2 gr = group_rows(p, tile.g);
        const int a_row = gr.x + tile.m0 + static_cast<int>(rank) * BM;
        const int b_row = tile.g * p.K;
        const int r_base = tile.m0 + static_cast<int>(rank) * BM;   // this CTA's first row in the group
        // token of row r of this CTA's slab (rows past the group's count read row 0)
        auto token_of = [&](int r) {
          const int v = r_base + r < gr.y ? __ldg(p.a_token + gr.x + r_base + r) : 0;
          return static_cast<unsigned>(v) < static_cast<unsigned>(p.a_token_rows) ? v : 0;
        };
        int tok4[4] = {0, 0, 0, 0};
        int tok32[amode == A_GATHER_LSU ? 32 : 1];
        if constexpr (amode == A_GATHER_TMA) {
#pragma unroll
          for (int i = 0; i < 4; ++i) tok4[i] = token_of(4 * lane + i);
        } else if constexpr (amode == A_GATHER_LSU) {
#pragma unroll
          for (int i = 0; i < 32; ++i) tok32[i] = token_of(4 * i + (lane >> 3));
        }
        for (int kb = 0; kb < KB; ++kb) {
          bool free_stage = true;
          if (lane == 0) free_stage = mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout, p.wait_ns);
          if (amode != A_TILE) free_stage = __shfl_sync(0xffffffffu, free_stage ? 1 : 0, 0) != 0;
          if (!free_stage) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_addr(&tl.full[stage]);
          const uint32_t a_dst = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_addr(sB + stage * C::B_BYTES);
          const int ky = b_row + kb * BK;
          // both CTAs' TMA bytes of a pair complete on the even CTA's barrier
          const uint32_t fb = (CG == 1 || rank == 0) ? fb_local : mapa_shared(fb_local, 0);
          const uint32_t tx = static_cast<uint32_t>((amode == A_GATHER_LSU ? 0 : A_BYTES) + C::B_BYTES);
          if (lane == 0 && (CG == 1 || rank == 0)) mbar_arrive_expect_tx(fb_local, CG * tx);
          if constexpr (amode == A_TILE) {
            if (CG == 1)
              tma_load_2d(a_dst, &tmA, fb, kb * BK, a_row);
            else
              tma_load_2d_pair(a_dst, &tmA, fb, kb * BK, a_row);
          } else if constexpr (amode == A_GATHER_TMA) {
            __syncwarp();
            if (CG == 1)
              tma_gather4(a_dst + lane * 4 * 128, &tmA, fb, kb * BK, tok4[0], tok4[1], tok4[2], tok4[3]);
            else
              tma_gather4_pair(a_dst + lane * 4 * 128, &tmA, fb, kb * BK, tok4[0], tok4[1], tok4[2], tok4[3]);
          } else {
            // chunk c of row r lands at 16 * (c ^ (r % 8)) in the row's 128 bytes:
            // the 128-byte swizzle of a 1024-byte aligned slab
            const int c = lane & 7;
            const uint16_t* xs = static_cast<const uint16_t*>(p.a_src) + kb * BK + c * 8;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int r = 4 * i + (lane >> 3);
              cp_async_16(a_dst + r * 128 + ((c ^ (r & 7)) << 4), xs + static_cast<int64_t>(tok32[i]) * p.K);
            }
            // the odd CTA of a pair counts its slab on its own barrier; its MMA
            // warp relays the completion to the even CTA
            cp_async_arrive_noinc(CG == 2 && rank != 0 ? smem_addr(&tl.afull[stage]) : fb_local);
          }
          if (lane == 0) {
#pragma unroll
            for (int i = 0; i < Cfg<CG>::B_CHUNKS; ++i) {
              if (CG == 1)
                tma_load_2d(b_dst + i * B_CHUNK, b_box_map<MODE, CG>(&tmB0, &tmB1, rank, i), fb,
                            b_box_col<MODE, CG>(tile.n0, rank, i), ky);
              else
                tma_load_2d_pair(b_dst + i * B_CHUNK, b_box_map<MODE, CG>(&tmB0, &tmB1, rank, i), fb,
                                 b_box_col<MODE, CG>(tile.n0, rank, i), ky);
            }
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy into shared memory lands before the CTA may exit
      if (amode == A_GATHER_LSU) cp_async_wait_all();
      // Every TMA load issued by this warp has landed before the CTA may exit
      // (all lanes' loads of a stage complete on the stage's one barrier): the
      // even CTA sees its barrier complete; the odd CTA sees the MMA that
      // consumed the load release the stage.
      if (lane == 0) {
        for (int s = 0; s < C::STAGES; ++s)
          if ((issued >> s) & 1u) {
            if (rank == 0)
              mbar_wait(smem_addr(&tl.full[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
            else
              mbar_wait(smem_addr(&tl.empty[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
          }
      }
    }
  } else if (warp == 1) {
    constexpr bool lsu_a = AMODE == A_GATHER_LSU;
    if (CG == 2 && lane == 0 && rank != 0 && lsu_a) {
      // ------------------------------------------------------ relay (odd CTA)
      // The odd CTA's producer lanes count each stage's cp.async slab on afull;
      // this thread forwards it, in the producer's stage order, as one arrival
      // on the even CTA's full barrier (cp.async completion can only signal a
      // barrier of the issuing CTA).
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int t = unit; ok && t < total; t += n_units) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(smem_addr(&tl.afull[stage]), phase, abort, p.flags, kFlagTimeout, p.wait_ns)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          mbar_arrive_cluster(mapa_shared(smem_addr(&tl.full[stage]), 0));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    } else if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true, issued_any = false;
      // Descriptors of stage 0 at K offset 0.  Their start-address field is the
      // shared address / 16 (14 bits, no carry below 256 KB), so a stage or a K
      // step is a constant added to the descriptor: this thread's instruction
      // stream per K stage stays short next to the MMAs it feeds.
      const uint64_t adesc0 = smem_desc_sw128(smem_addr(sA), 16, 1024);
      const uint64_t bdesc0 = smem_desc_sw128(smem_addr(sB), B_CHUNK, 1024);
      for (int t = unit; ok && t < total; t += n_units) {
        if (!mbar_wait(smem_addr(&tl.tempty[acc]), acc_phase ^ 1u, abort, p.flags, kFlagTimeout, p.wait_ns)) break;
        tc_fence_after();
        issued_any = true;
        const uint32_t d_tmem = tmem_base + acc * MMA_N;
        for (int kb = 0; kb < KB; ++kb) {
          // with a cp.async slab on a CTA pair, the odd CTA announces its half by an
          // arrival of its own: acquire at cluster scope (only then: it costs)
          if (!mbar_wait<CG == 2 && lsu_a>(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout,
                                            p.wait_ns)) {
            ok = false;
            break;
          }
          if (lsu_a) fence_proxy_async_smem();   // cp.async (generic proxy) writes -> MMA operand reads
          tc_fence_after();
          const uint64_t adesc_s = adesc0 + stage * static_cast<uint32_t>(A_BYTES >> 4);
          const uint64_t bdesc_s = bdesc0 + stage * static_cast<uint32_t>(C::B_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            // A: K-major, advance 16 elements (32 bytes) inside the swizzle row
            const uint64_t adesc = adesc_s + static_cast<uint64_t>(kk * (32 >> 4));
            // B: MN-major, advance 16 K rows = two 8-row swizzle atoms (2048 bytes)
            const uint64_t bdesc = bdesc_s + static_cast<uint64_t>(kk * (2048 >> 4));
            if (CG == 2)
              tc_mma_f16_pair(d_tmem, adesc, bdesc, C::IDESC, (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma_f16(d_tmem, adesc, bdesc, C::IDESC, (kb | kk) != 0 ? 1u : 0u);
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
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // every MMA issued by this thread completes before TMEM is released
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
    uint32_t acc = 0, acc_phase = 0;
    for (int t = unit; t < total; t += n_units) {
      const Tile tile = decode_tile(tl, p, G, BN, C::TILE_M, t);
      const int2 gr = group_rows(p, tile.g);
      if (!mbar_wait(smem_addr(&tl.tfull[acc]), acc_phase, abort, p.flags, kFlagTimeout, p.wait_ns)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * MMA_N;
      const int row = tile.m0 + r_in_tile;
      const bool valid = row < gr.y;
      uint16_t* orow = p.out + (static_cast<int64_t>(gr.x) + row) * p.n_out;
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
            store_row32(orow, tile.n0 + c, p.n_out, pk, p.v8);
            if (p.save_g != nullptr) {
              const int64_t off = (static_cast<int64_t>(gr.x) + row) * p.n_out;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(gv[2 * i]), __uint_as_float(gv[2 * i + 1]));
              store_row32(p.save_g + off, tile.n0 + c, p.n_out, pk, p.v8);
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(uv[2 * i]), __uint_as_float(uv[2 * i + 1]));
              store_row32(p.save_u + off, tile.n0 + c, p.n_out, pk, p.v8);
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
            store_row32(orow, tile.n0 + c, p.n_out, pk, p.v8);
          }
        }
      }
      tc_fence_before();
      const uint32_t te = smem_addr(&tl.tempty[acc]);
      if (CG == 2 && rank != 0)
        mbar_arrive_cluster(mapa_shared(te, 0));
      else
        mbar_arrive(te);
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

// ---------------------------------------------------------------- host side
template <int MODE, int CG, int AMODE>
cudaError_t set_smem_attr() {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(tc_ffn_gemm_kernel<MODE, CG, AMODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes<CG>()));
  });
  return r;
}

template <int MODE, int CG, int AMODE = A_TILE>
cudaError_t launch_gemm(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const TcParams& p,
                        int64_t bound_units, cudaStream_t s) {
  cudaError_t e = set_smem_attr<MODE, CG, AMODE>();
  if (e != cudaSuccess) return e;
  int units = device_sm_count() / CG;
  units = static_cast<int>(std::min<int64_t>(units, std::max<int64_t>(bound_units, 1)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units * CG), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<CG>();
  cfg.stream = s;
  // CTA pairs may start while the kernel before them finishes (the kernel waits
  // for its results first).  Single-CTA tiles are launched plainly: overlapped,
  // the DeepSeek-shaped layer ran ~10 % slower at the power cap (its clock
  // settled ~120 MHz lower), while the pair launches gained 1-3 % on the
  // Qwen3-shaped layer.
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (CG == 2 && launch_overlap_enabled()) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (CG == 2) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    // persistent: no more pairs than can be resident at once
    int max_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, tc_ffn_gemm_kernel<MODE, CG, AMODE>, &cfg) == cudaSuccess &&
        max_clusters > 0 && max_clusters < units)
      cfg.gridDim.x = static_cast<unsigned>(max_clusters * 2);
  }
  e = cudaLaunchKernelEx(&cfg, tc_ffn_gemm_kernel<MODE, CG, AMODE>, A, B0, B1, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// CTA pairs pay off when experts have many rows; with few rows per expert the
// 256-row pair tiles waste more of the MMA work on rows past the segment end.
// MOE_FFN_CTA_GROUP=1|2 forces one variant (tests run both).
// every row of a bf16 [rows, n] buffer starts on a 32-byte boundary (null: no buffer)
bool rows_32b_aligned(const uint16_t* p, int n) {
  return (reinterpret_cast<uintptr_t>(p) & 31u) == 0 && n % 16 == 0;
}

// Whether the layer pass gathers GEMM1's token rows from x instead of reading
// the permuted copy, and how: MOE_GATHER=tma (tile::gather4 TMA loads) or lsu
// (cp.async copies).  Unset or anything else: no gather.  Both gathers measured
// slower than the copy on the Qwen3-shaped layer (GEMM1 2.29 ms with cp.async,
// about 3.5 ms with gather4, against 1.26 ms reading the permuted rows as TMA
// tiles, under ncu), so the copy is the default.
int gather_mode() {
  static int mode = [] {
    const char* v = std::getenv("MOE_GATHER");
    if (v == nullptr) return static_cast<int>(A_TILE);
    if (v[0] == 't') return static_cast<int>(A_GATHER_TMA);
    if (v[0] == 'l') return static_cast<int>(A_GATHER_LSU);
    return static_cast<int>(A_TILE);
  }();
  return mode;
}

// Bound of the grouped GEMM's pipeline waits (moe_set_wait_limit_ns); 0 = kWaitLimitNs.
std::atomic<uint64_t> g_pipeline_wait_ns{0};

uint64_t pipeline_wait_ns() {
  const uint64_t v = g_pipeline_wait_ns.load(std::memory_order_relaxed);
  return v == 0 ? kWaitLimitNs : v;
}

int choose_cta_group(const FfnArgs& a) {
  static int forced = [] {
    const char* v = std::getenv("MOE_FFN_CTA_GROUP");
    return v ? std::atoi(v) : 0;
  }();
  if (forced == 1 || forced == 2) return forced;
  if (a.seg_off == nullptr) return 2;                     // dense shared expert: T rows
  return a.mean_rows >= 384 ? 2 : 1;
}

template <int CG>
cudaError_t launch_pair(const FfnArgs& a, const CUtensorMap& mA1, const CUtensorMap& mW1, const CUtensorMap& mW3,
                        const CUtensorMap& mA2, const CUtensorMap& mW2, TcParams p, cudaStream_t s) {
  const bool dense = a.seg_off == nullptr;
  const int tile_m = Cfg<CG>::TILE_M;
  const int64_t m_bound = (a.max_rows + tile_m - 1) / tile_m + (dense ? 0 : a.G);
  p.K = a.d;
  p.n_out = a.f;
  p.out = static_cast<uint16_t*>(a.h);
  p.save_g = static_cast<uint16_t*>(a.save_g);
  p.save_u = static_cast<uint16_t*>(a.save_u);
  p.v8 = rows_32b_aligned(p.out, p.n_out) && rows_32b_aligned(p.save_g, p.n_out) &&
         rows_32b_aligned(p.save_u, p.n_out);
  p.a_token = a.a_token;
  p.a_src = a.a;
  p.a_token_rows = static_cast<int>(a.a_token_rows);
  p.a_gather = gather_mode();
  const int64_t units1 = m_bound * ((a.f + 127) / 128);
  cudaError_t e = p.a_token == nullptr       ? launch_gemm<MODE_SWIGLU, CG>(mA1, mW1, mW3, p, units1, s)
                  : p.a_gather == A_GATHER_TMA ? launch_gemm<MODE_SWIGLU, CG, A_GATHER_TMA>(mA1, mW1, mW3, p, units1, s)
                                               : launch_gemm<MODE_SWIGLU, CG, A_GATHER_LSU>(mA1, mW1, mW3, p, units1, s);
  if (e != cudaSuccess) return e;
  p.a_token = nullptr;
  p.a_src = nullptr;
  p.a_token_rows = 0;
  p.save_g = p.save_u = nullptr;
  p.K = a.f;
  p.n_out = a.d;
  p.out = static_cast<uint16_t*>(a.out);
  p.v8 = rows_32b_aligned(p.out, p.n_out);
  return launch_gemm<MODE_PLAIN, CG>(mA2, mW2, mW2, p, m_bound * ((a.d + 255) / 256), s);
}

}  // namespace

void set_pipeline_wait_ns(uint64_t ns) { g_pipeline_wait_ns.store(ns, std::memory_order_relaxed); }

bool layer_gathers_rows() { return gather_mode() != A_TILE; }

cudaError_t launch_ffn_bf16(const FfnArgs& a, cudaStream_t s) {
  if (a.max_rows <= 0 || a.G <= 0) return cudaSuccess;
  const bool dense = a.seg_off == nullptr;
  const uint64_t G = dense ? 1 : static_cast<uint64_t>(a.G);
  CUtensorMap mA1, mW1, mW3, mA2, mW2;
  // GEMM1's A: the permuted rows as 128-row tiles, or x one row per box for the
  // row gather (the gather load's box is one row high)
  const bool gather = a.a_token != nullptr;
  if (gather && (a.a_token_rows <= 0 || a.a_token_rows >= (int64_t(1) << 31))) return cudaErrorInvalidValue;
  if (!make_tma_2d_bf16(&mA1, a.a, a.d, gather ? a.a_token_rows : a.max_rows, BK, gather ? 1 : BM) ||
      !make_tma_2d_bf16(&mW1, a.w1, a.f, G * a.d, 64, BK) || !make_tma_2d_bf16(&mW3, a.w3, a.f, G * a.d, 64, BK) ||
      !make_tma_2d_bf16(&mA2, a.h, a.f, a.max_rows, BK, BM) || !make_tma_2d_bf16(&mW2, a.w2, a.d, G * a.f, 64, BK))
    return cudaErrorInvalidValue;

  TcParams p{};
  p.wait_ns = pipeline_wait_ns();
  p.seg_off = a.seg_off;
  p.seg_count = a.seg_count;
  p.G = static_cast<int>(G);
  p.dense_rows = a.dense_rows;
  p.max_rows = a.max_rows;
  p.flags = a.flags;
  if (choose_cta_group(a) == 2) return launch_pair<2>(a, mA1, mW1, mW3, mA2, mW2, p, s);
  return launch_pair<1>(a, mA1, mW1, mW3, mA2, mW2, p, s);
}

}  // namespace moe
