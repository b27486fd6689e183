// Grouped GEMMs of the backward pass of the SwiGLU experts on the tcgen05
// tensor cores (bf16 operands, fp32 accumulation in TMEM).
//
// Only the experts a token was routed to receive its gradient ("ms-swift +
// Megatron：MoE模型加速10倍实测" §2.3: MoE gradients are sparse); per expert e
// with rows r of the permuted buffers (o = h W2, h = silu(g) * u, g = xp W1,
// u = xp W3):
//   DGRAD_SWIGLU:  dH = dO W2_e^T, then in the epilogue
//                  dG = dH * u * silu'(g),  dU = dH * silu(g)          (bf16)
//   DGRAD_PLAIN2:  dXp = dG W1_e^T + dU W3_e^T  (one K loop over 2f)   (bf16)
//   WGRAD:         dW = A_e^T B_e over the expert's rows (dW1 = xp^T dG,
//                  dW3 = xp^T dU, dW2 = h^T dO), fp32 out
// The dgrad kernels read the weights as stored ([G][n][k] row-major is the
// K-major B operand); the wgrad kernel reads both row buffers as stored
// ([rows][m] is the MN-major A operand, [rows][n] the MN-major B), with the
// reduction running over the expert's padded segment (its rows past the kept
// count are zero).  Same persistent warp-specialised structure as the forward
// kernel (TMA producer, single MMA thread, four epilogue warps, two TMEM
// accumulators).  Two tile shapes: single CTAs with 128 x 256 tiles and four
// 48 KB stages, or CTA pairs (cta_group::2, cluster of two) with 256 x 256
// tiles where each CTA stages its own 128 rows of A and 128 of the 256 B rows
// (six 32 KB stages): per SM the operand stream per flop is 2/3 of the single
// CTA's, which is what limits the single-CTA shape.  Every mbarrier wait is
// bounded.
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "device_utils.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int MMA_N = 256;
constexpr int MMA_K = 16;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int kMaxStages = 6;
constexpr int kThreads = 192;

template <int CG>
struct BwdCfg {
  static constexpr int TILE_M = BM * CG;                // accumulator rows of one (pair) tile
  static constexpr int B_ROWS = MMA_N / CG;             // rows of the N side this CTA stages
  static constexpr int B_BYTES = B_ROWS * BK * 2;       // 32 KB single, 16 KB pair
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = CG == 1 ? 4 : 6;
  static_assert(STAGES <= kMaxStages, "barrier arrays");
};
constexpr int kTmemCols = 2 * MMA_N;
constexpr int kMaxGroups = 256;

enum { KIND_DGRAD_SWIGLU = 0, KIND_DGRAD_PLAIN2 = 1, KIND_WGRAD = 2 };

struct BwdParams {
  const int32_t* seg_off;   // [G+1] or nullptr (one dense group of dense_rows rows)
  const int32_t* seg_count;
  int G;
  int dense_rows;
  int64_t max_rows;
  int K;                    // dgrad: reduction length of one phase (multiple of 64)
  int M;                    // wgrad: rows of the weight gradient
  int n_out;                // output columns
  const uint16_t* g;        // DGRAD_SWIGLU: saved gate pre-activation [rows, n_out]
  const uint16_t* u;        //               saved up pre-activation
  void* out0;               // dG | dXp | dW (fp32, [G][M][n_out])
  void* out1;               // dU
  uint32_t* flags;
};

struct Tail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
  int32_t tile_start[kMaxGroups + 1];
  int32_t row0[kMaxGroups];
  int32_t count[kMaxGroups];   // dgrad: kept rows; wgrad: padded rows (the reduction length)
  int32_t pad[kMaxGroups];     // dgrad: rows of the group's padded segment (rows past it belong to the next)
};

// fp32 output staging of the weight-gradient epilogue: one 32 x 32 block
// (4 KB, 128-byte swizzled as the TMA store reads it) per epilogue warp
constexpr int kStageBlock = 32 * 32 * 4;
constexpr size_t kStagingBytes = 4 * kStageBlock;
template <int CG>
constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(BwdCfg<CG>::STAGES) * BwdCfg<CG>::STAGE_BYTES + kStagingBytes + sizeof(Tail);
}
static_assert(smem_bytes<1>() <= 232448 && smem_bytes<2>() <= 232448, "shared memory per CTA");

struct Tile {
  int g, m0, n0;
};

// dgrad: per group ceil(count/TILE_M) row tiles x n_tiles, row tiles fastest;
// wgrad: per group ceil(M/TILE_M) tiles x n_tiles, M tiles fastest
template <int KIND, int TILE_M>
__device__ __forceinline__ Tile decode(const Tail& s, int G, int n_tiles, int m_tiles_w, int t) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_start[mid] <= t)
      lo = mid;
    else
      hi = mid;
  }
  const int local = t - s.tile_start[lo];
  const int mt = KIND == KIND_WGRAD ? m_tiles_w : (s.count[lo] + TILE_M - 1) / TILE_M;
  Tile r;
  r.g = lo;
  r.n0 = (local / mt) * MMA_N;
  r.m0 = (local % mt) * TILE_M;
  (void)n_tiles;
  return r;
}

__device__ __forceinline__ float sigmoid_f32(float v) { return __fdividef(1.0f, 1.0f + __expf(-v)); }

__device__ __forceinline__ void store_bf16_32(uint16_t* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                       pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void load_bf16_32(const uint16_t* src, float (&v)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = s4[q];
    v[8 * q + 0] = bf16_lo(w.x);
    v[8 * q + 1] = bf16_hi(w.x);
    v[8 * q + 2] = bf16_lo(w.y);
    v[8 * q + 3] = bf16_hi(w.y);
    v[8 * q + 4] = bf16_lo(w.z);
    v[8 * q + 5] = bf16_hi(w.z);
    v[8 * q + 6] = bf16_lo(w.w);
    v[8 * q + 7] = bf16_hi(w.w);
  }
}

template <int KIND, int CG>
__global__ void __launch_bounds__(kThreads, 1)
    tc_bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                       const BwdParams p) {
  constexpr bool A_MN = KIND == KIND_WGRAD;   // A stored [K rows][M], else [M rows][K]
  constexpr bool B_MN = KIND == KIND_WGRAD;   // B stored [K rows][N], else [N rows][K]
  constexpr int PHASES = KIND == KIND_DGRAD_PLAIN2 ? 2 : 1;
  using C = BwdCfg<CG>;
  constexpr int STAGES = C::STAGES, TILE_M = C::TILE_M, B_BYTES = C::B_BYTES, STAGE_BYTES = C::STAGE_BYTES;
  constexpr uint32_t IDESC = idesc_bf16_f32_ab(TILE_M, MMA_N, A_MN ? 1 : 0, B_MN ? 1 : 0);
  extern __shared__ uint8_t dsmem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * A_BYTES;
  uint8_t* sStage = base + STAGES * STAGE_BYTES;   // 1024-byte aligned
  Tail& tl = *reinterpret_cast<Tail*>(sStage + kStagingBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;   // 0: this CTA issues the MMAs
  const int unit = static_cast<int>(blockIdx.x) / CG, n_units = static_cast<int>(gridDim.x) / CG;
  const int G = p.seg_off != nullptr ? p.G : 1;
  const int n_tiles = (p.n_out + MMA_N - 1) / MMA_N;
  const int m_tiles_w = (p.M + TILE_M - 1) / TILE_M;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_addr(&tl.full[s]), 1);
      mbar_init(smem_addr(&tl.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&tl.tfull[a]), 1);
      mbar_init(smem_addr(&tl.tempty[a]), 128 * CG);
    }
    mbar_init(smem_addr(&tl.drain), 1);
    tl.abort = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (PHASES == 2) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
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
      int r0 = 0, c = p.dense_rows, pad = p.dense_rows;
      if (p.seg_off != nullptr) {
        r0 = p.seg_off[g];
        pad = p.seg_off[g + 1] - r0;
        c = KIND == KIND_WGRAD ? pad : p.seg_count[g];
      }
      if (r0 < 0 || c < 0 || pad < c || static_cast<int64_t>(r0) + pad > p.max_rows) {
        atomicOr(p.flags, kFlagBadIndex);
        r0 = 0;
        c = 0;
        pad = 0;
      }
      tl.row0[g] = r0;
      tl.count[g] = c;
      tl.pad[g] = pad;
      local += (KIND == KIND_WGRAD ? m_tiles_w : (c + TILE_M - 1) / TILE_M) * n_tiles;
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
      run += (KIND == KIND_WGRAD ? m_tiles_w : (tl.count[g] + TILE_M - 1) / TILE_M) * n_tiles;
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

  // K slabs of a tile
  auto slabs_of = [&](const Tile& tile) -> int {
    if (KIND == KIND_WGRAD) return (tl.count[tile.g] + BK - 1) / BK;
    return PHASES * (p.K / BK);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t stage = 0, phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int t = unit; ok && t < total; t += n_units) {
        const Tile tile = decode<KIND, TILE_M>(tl, G, n_tiles, m_tiles_w, t);
        const int KS = slabs_of(tile);
        const int row0 = tl.row0[tile.g];
        const int m_mine = tile.m0 + static_cast<int>(rank) * BM;          // this CTA's 128 rows of the tile
        const int n_mine = static_cast<int>(rank) * C::B_ROWS;             // this CTA's share of the 256 N rows
        for (int kb = 0; kb < KS; ++kb) {
          if (!mbar_wait(smem_addr(&tl.empty[stage]), phase ^ 1u, abort, p.flags, kFlagTimeout)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_addr(&tl.full[stage]);
          // both CTAs' bytes complete on the even CTA's barrier
          const uint32_t fb = (CG == 1 || rank == 0) ? fb_local : mapa_shared(fb_local, 0);
          if (CG == 1 || rank == 0) mbar_arrive_expect_tx(fb_local, CG * STAGE_BYTES);
          const uint32_t a_dst = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_addr(sB + stage * B_BYTES);
          auto load = [&](uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y) {
            if (CG == 2)
              tma_load_2d_pair(dst, map, fb, x, y);
            else
              tma_load_2d(dst, map, fb, x, y);
          };
          if (KIND == KIND_WGRAD) {
            const int y = row0 + kb * BK;     // reduction runs over the group's rows
            load(a_dst, &tmA0, m_mine, y);
            load(a_dst + A_BYTES / 2, &tmA0, m_mine + 64, y);
#pragma unroll
            for (int c = 0; c < C::B_ROWS / 64; ++c) load(b_dst + c * 8192, &tmB0, tile.n0 + n_mine + 64 * c, y);
          } else {
            const int ph = kb / (p.K / BK);
            const int x = (kb - ph * (p.K / BK)) * BK;
            const int b_row = tile.g * p.n_out + tile.n0 + n_mine;   // weight rows [G][n_out][K]
            const CUtensorMap* ma = ph == 0 ? &tmA0 : &tmA1;
            const CUtensorMap* mb = ph == 0 ? &tmB0 : &tmB1;
            load(a_dst, ma, x, row0 + m_mine);
#pragma unroll
            for (int c = 0; c < C::B_ROWS / 128; ++c) load(b_dst + c * 16384, mb, x, b_row + 128 * c);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every load issued by this thread has landed before the CTA may exit:
      // the even CTA sees its barrier complete; the odd CTA sees the MMA that
      // consumed the load release the stage.
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) {
          if (CG == 1 || rank == 0)
            mbar_wait(smem_addr(&tl.full[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
          else
            mbar_wait(smem_addr(&tl.empty[s]), (last_par >> s) & 1u, nullptr, p.flags, kFlagTimeout);
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true, issued_any = false;
      for (int t = unit; ok && t < total; t += n_units) {
        const Tile tile = decode<KIND, TILE_M>(tl, G, n_tiles, m_tiles_w, t);
        const int KS = slabs_of(tile);
        if (!mbar_wait(smem_addr(&tl.tempty[acc]), acc_phase ^ 1u, abort, p.flags, kFlagTimeout)) break;
        tc_fence_after();
        issued_any = true;
        const uint32_t d_tmem = tmem_base + acc * MMA_N;
        for (int kb = 0; kb < KS; ++kb) {
          if (!mbar_wait(smem_addr(&tl.full[stage]), phase, abort, p.flags, kFlagTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_addr(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            // K-major: advance 16 values (32 bytes) in the swizzle row; MN-major:
            // advance 16 K rows (two 8-row swizzle atoms, 2048 bytes), 64-column
            // chunks 8 KB apart
            const uint64_t adesc = A_MN ? smem_desc_sw128(a_addr + kk * 2048, A_BYTES / 2, 1024)
                                        : smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bdesc = B_MN ? smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                        : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            if (CG == 2)
              tc_mma_f16_pair(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma_f16(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          if (CG == 2)
            tc_commit_pair_both(smem_addr(&tl.empty[stage]));
          else
            tc_commit(smem_addr(&tl.empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        // with no K slab (empty group) this arrives at once
        if (CG == 2)
          tc_commit_pair_both(smem_addr(&tl.tfull[acc]));
        else
          tc_commit(smem_addr(&tl.tfull[acc]));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
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
    // this CTA's TMEM lanes hold rows rank * 128 + (0 .. 127) of the (pair) tile
    const int quad = warp & 3;
    const int r_in_tile = static_cast<int>(rank) * BM + quad * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int t = unit; t < total; t += n_units) {
      const Tile tile = decode<KIND, TILE_M>(tl, G, n_tiles, m_tiles_w, t);
      if (!mbar_wait(smem_addr(&tl.tfull[acc]), acc_phase, abort, p.flags, kFlagTimeout)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * MMA_N;
      const bool empty_k = slabs_of(tile) == 0;   // wgrad of an expert with no rows: zeros
#pragma unroll 1
      for (int c = 0; c < MMA_N; c += 32) {
        const int col = tile.n0 + c;
        uint32_t v[32];
        if (!empty_k) {
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (col >= p.n_out) continue;
        if (KIND == KIND_WGRAD) {
          // the warp's 32 rows x 32 columns go to its staging block in the
          // 128-byte swizzled layout (16-byte chunk q of row r at chunk q ^ (r % 8):
          // conflict-free), then one TMA store writes the block to dW[g]; the
          // 3-D tensor map clips rows past M and columns past n_out
          const int m_first = tile.m0 + static_cast<int>(rank) * BM + quad * 32;
          if (m_first < p.M) {
            uint8_t* stg = sStage + quad * kStageBlock;
            if (lane == 0) bulk_wait_read_all();   // this warp's previous store has read the block
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                  make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                              __uint_as_float(v[4 * q + 3]));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmA1, smem_addr(stg), col, m_first, tile.g);
              bulk_commit();
            }
          }
        } else {
          const int row = tile.m0 + r_in_tile;
          const bool valid = row < tl.count[tile.g];
          const int64_t grow = static_cast<int64_t>(tl.row0[tile.g]) + row;
          // rows past the group's padded segment belong to the next group (or
          // past a dense group's end): a tile taller than the padding stops there
          if (row >= tl.pad[tile.g] || grow >= p.max_rows) continue;
          if (KIND == KIND_DGRAD_SWIGLU) {
            // every row of the tile is written: rows past the kept count (the
            // segment's padding) get zeros, so the weight-gradient GEMMs may
            // reduce over whole padded segments
            float dg[32], du[32];
            if (valid) {
              float gv[32], uv[32];
              load_bf16_32(p.g + grow * p.n_out + col, gv);
              load_bf16_32(p.u + grow * p.n_out + col, uv);
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float dh = __uint_as_float(v[i]);
                const float sg = sigmoid_f32(gv[i]);
                const float silu = gv[i] * sg;
                dg[i] = dh * uv[i] * sg * (1.0f + gv[i] * (1.0f - sg));
                du[i] = dh * silu;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) dg[i] = du[i] = 0.f;
            }
            store_bf16_32(static_cast<uint16_t*>(p.out0) + grow * p.n_out + col, dg);
            store_bf16_32(static_cast<uint16_t*>(p.out1) + grow * p.n_out + col, du);
          } else if (valid) {
            float o[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(v[i]);
            store_bf16_32(static_cast<uint16_t*>(p.out0) + grow * p.n_out + col, o);
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
    if (KIND == KIND_WGRAD && lane == 0) bulk_wait_all();   // every store issued by this warp has landed
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

template <int KIND, int CG>
cudaError_t launch_cg(const CUtensorMap& A0, const CUtensorMap& A1, const CUtensorMap& B0, const CUtensorMap& B1,
                      const BwdParams& p, int64_t bound_units, cudaStream_t s) {
  static std::once_flag once[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaError_t r = cudaSuccess;
  std::call_once(once[dev & 63], [&] {
    r = cudaFuncSetAttribute(tc_bwd_gemm_kernel<KIND, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes<CG>()));
  });
  if (r != cudaSuccess) return r;
  const int units = static_cast<int>(std::min<int64_t>(device_sm_count() / CG, std::max<int64_t>(bound_units, 1)));
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
  }
  e = cudaLaunchKernelEx(&cfg, tc_bwd_gemm_kernel<KIND, CG>, A0, A1, B0, B1, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// CTA pairs for the dgrad GEMMs when groups average at least 384 rows (so that
// 256-row pair tiles are mostly filled); MOE_BWD_CTA_GROUP=1|2 forces a shape
// for every kind (tests).
bool use_pairs_bwd(bool pairs_pay) {
  static int forced = [] {
    const char* v = std::getenv("MOE_BWD_CTA_GROUP");
    return v ? std::atoi(v) : 0;
  }();
  if (forced == 1 || forced == 2) return forced == 2;
  return pairs_pay;
}

// m_units: row tiles (dgrad) or M tiles (wgrad) counted in 128-row units, all groups
template <int KIND>
cudaError_t launch(const CUtensorMap& A0, const CUtensorMap& A1, const CUtensorMap& B0, const CUtensorMap& B1,
                   const BwdParams& p, bool pairs_pay, int64_t m_units, int n_tiles, cudaStream_t s) {
  if (use_pairs_bwd(pairs_pay))
    return launch_cg<KIND, 2>(A0, A1, B0, B1, p, (m_units + 1) / 2 * n_tiles, s);
  return launch_cg<KIND, 1>(A0, A1, B0, B1, p, m_units * n_tiles, s);
}

// dgrad groups average at least 384 rows (the padded buffer over the groups)
bool dgrad_pairs_pay(const BwdGroups& s) {
  const int64_t G = s.seg_off != nullptr ? s.G : 1;
  return (s.seg_off != nullptr ? s.max_rows : s.dense_rows) / G >= 384;
}

BwdParams base_params(const BwdGroups& s) {
  BwdParams p{};
  p.seg_off = s.seg_off;
  p.seg_count = s.seg_count;
  p.G = s.seg_off != nullptr ? s.G : 1;
  p.dense_rows = s.dense_rows;
  p.max_rows = s.max_rows;
  p.flags = s.flags;
  return p;
}

int64_t row_tiles_bound(const BwdGroups& s) {
  return (s.max_rows + BM - 1) / BM + (s.seg_off != nullptr ? s.G : 0);
}

}  // namespace

cudaError_t launch_dgrad_swiglu(const BwdGroups& s, int d, int f, const void* dO, const void* w2, const void* g,
                                const void* u, void* dG, void* dU, cudaStream_t st) {
  if (s.max_rows <= 0) return cudaSuccess;
  const uint64_t G = s.seg_off != nullptr ? s.G : 1;
  CUtensorMap mA, mB;
  if (!make_tma_2d_bf16(&mA, dO, d, s.max_rows, BK, BM) || !make_tma_2d_bf16(&mB, w2, d, G * f, BK, 128))
    return cudaErrorInvalidValue;
  BwdParams p = base_params(s);
  p.K = d;
  p.n_out = f;
  p.g = static_cast<const uint16_t*>(g);
  p.u = static_cast<const uint16_t*>(u);
  p.out0 = dG;
  p.out1 = dU;
  return launch<KIND_DGRAD_SWIGLU>(mA, mA, mB, mB, p, dgrad_pairs_pay(s), row_tiles_bound(s), (f + MMA_N - 1) / MMA_N,
                                   st);
}

cudaError_t launch_dgrad_plain2(const BwdGroups& s, int d, int f, const void* dG, const void* dU, const void* w1,
                                const void* w3, void* dXp, cudaStream_t st) {
  if (s.max_rows <= 0) return cudaSuccess;
  const uint64_t G = s.seg_off != nullptr ? s.G : 1;
  CUtensorMap mA0, mA1, mB0, mB1;
  if (!make_tma_2d_bf16(&mA0, dG, f, s.max_rows, BK, BM) || !make_tma_2d_bf16(&mA1, dU, f, s.max_rows, BK, BM) ||
      !make_tma_2d_bf16(&mB0, w1, f, G * d, BK, 128) || !make_tma_2d_bf16(&mB1, w3, f, G * d, BK, 128))
    return cudaErrorInvalidValue;
  BwdParams p = base_params(s);
  p.K = f;
  p.n_out = d;
  p.out0 = dXp;
  return launch<KIND_DGRAD_PLAIN2>(mA0, mA1, mB0, mB1, p, dgrad_pairs_pay(s), row_tiles_bound(s),
                                   (d + MMA_N - 1) / MMA_N, st);
}

cudaError_t launch_wgrad(const BwdGroups& s, int M, int N, const void* a, const void* b, float* out,
                         cudaStream_t st) {
  if (s.max_rows <= 0) return cudaSuccess;
  const int G = s.seg_off != nullptr ? s.G : 1;
  CUtensorMap mA, mB, mOut;
  if (!make_tma_2d_bf16(&mA, a, M, s.max_rows, 64, BK) || !make_tma_2d_bf16(&mB, b, N, s.max_rows, 64, BK) ||
      !make_tma_3d_f32_sw128(&mOut, out, N, M, G, 32, 32))
    return cudaErrorInvalidValue;
  BwdParams p = base_params(s);
  p.M = M;
  p.n_out = N;
  p.out0 = out;
  // single CTAs: the weight gradient is bound by its fp32 output writes, and
  // CTA pairs measured no faster
  return launch<KIND_WGRAD>(mA, mOut, mB, mB, p, false, static_cast<int64_t>(G) * ((M + BM - 1) / BM),
                            (N + MMA_N - 1) / MMA_N, st);
}

}  // namespace moe
