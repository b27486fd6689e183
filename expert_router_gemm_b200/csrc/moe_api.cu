// Host side of libmoe.so: argument validation, the exact capacity formula, the
// workspace layout and the C-ABI entry points declared in include/moe.h.
// Everything here runs on the host; every step of the computation runs in the
// CUDA kernels of route.cu, dispatch.cu, ffn_tc.cu, ffn_f32.cu and combine.cu.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>

#include "internal.h"

namespace moe {

bool launch_overlap_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_PDL");
    return v == nullptr || v[0] != '0';
  }();
  return on;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int& c = cache[dev & 63];
  if (c == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    c = v;
  }
  return c;
}

}  // namespace moe

namespace {

using namespace moe;

thread_local char g_last_cuda_error[256] = "";

moe_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

constexpr size_t kAlign = 256;
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Validated, derived sizes of one configuration.
struct Dims {
  int64_t T;
  int d, N, k, f, fs, C, align, elem;
  bool bf16;
  bool mx;             // routed-expert GEMMs in block-scaled FP8
  int64_t max_rows;    // rows of xp / h / out buffers
  int64_t max_count;   // upper bound of one expert's kept rows: min(C, T)
};

// C = ceil(cf * T * k / N) evaluated exactly on the double cf = m * 2^e.
moe_status_t exact_capacity(double cf, int64_t T, int k, int N, int32_t* out) {
  if (!std::isfinite(cf) || cf < 0.0) return MOE_ERR_INVALID_ARG;
  using u128 = unsigned __int128;
  if (cf == 0.0 || T == 0) {
    *out = 0;
    return MOE_OK;
  }
  int ex = 0;
  const double fr = std::frexp(cf, &ex);                       // cf = fr * 2^ex, fr in [0.5, 1)
  const uint64_t m = static_cast<uint64_t>(std::ldexp(fr, 53));  // exact 53-bit integer
  const int e = ex - 53;                                       // cf = m * 2^e
  const u128 P = static_cast<u128>(m) * static_cast<u128>(T) * static_cast<u128>(k);
  u128 c;
  if (e >= 0) {
    if (e > 40) return MOE_ERR_INVALID_ARG;                    // >= 2^40 / 256: beyond int32
    const u128 num = P << e;
    c = (num + static_cast<u128>(N) - 1) / static_cast<u128>(N);
  } else if (-e > 110) {
    c = 1;                                                     // 0 < value < 1
  } else {
    const u128 den = static_cast<u128>(N) << (-e);
    c = (P + den - 1) / den;
  }
  if (c > static_cast<u128>(INT32_MAX)) return MOE_ERR_INVALID_ARG;
  *out = static_cast<int32_t>(c);
  return MOE_OK;
}

moe_status_t derive(const moe_config_t* cfg, Dims* D) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  if (cfg->T < 0 || cfg->d < 1 || cfg->N < 1 || cfg->k < 1 || cfg->f < 1 || cfg->f_shared < 0 ||
      cfg->seg_align < 0)
    return MOE_ERR_INVALID_ARG;
  if (cfg->k > cfg->N) return MOE_ERR_INVALID_ARG;
  if (cfg->act_dtype != MOE_F32 && cfg->act_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (cfg->N > 256 || cfg->k > 32 || cfg->seg_align > 4096) return MOE_ERR_UNSUPPORTED;
  if (cfg->T * static_cast<int64_t>(cfg->k) >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  D->T = cfg->T;
  D->d = cfg->d;
  D->N = cfg->N;
  D->k = cfg->k;
  D->f = cfg->f;
  D->fs = cfg->f_shared;
  D->bf16 = cfg->act_dtype == MOE_BF16;
  D->elem = D->bf16 ? 2 : 4;
  if (cfg->gemm_format != MOE_GEMM_ACT && cfg->gemm_format != MOE_GEMM_MXFP8) return MOE_ERR_INVALID_ARG;
  D->mx = cfg->gemm_format == MOE_GEMM_MXFP8;
  D->align = cfg->seg_align == 0 ? 128 : cfg->seg_align;
  if (D->bf16) {
    if (D->d % 64 || D->f % 64 || D->fs % 64) return MOE_ERR_UNSUPPORTED;
  } else {
    if (D->d % 4) return MOE_ERR_UNSUPPORTED;  // rows are moved as 16-byte vectors
  }
  if (D->mx && (!D->bf16 || D->d % 128 || D->f % 128 || D->align % 128)) return MOE_ERR_UNSUPPORTED;
  if (cfg->capacity >= 0) {
    D->C = cfg->capacity;
  } else {
    moe_status_t s = exact_capacity(cfg->capacity_factor, cfg->T, cfg->k, cfg->N, &D->C);
    if (s != MOE_OK) return s;
  }
  D->max_count = std::min<int64_t>(D->C, D->T);
  const int64_t rows = std::min<int64_t>(D->T * D->k, static_cast<int64_t>(D->N) * D->max_count);
  D->max_rows = rows + static_cast<int64_t>(D->N) * (D->align - 1);
  if (D->max_rows >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Workspace layout.  The first bytes (flags word, route ticket, route count and
// z accumulators) are zeroed by one memset at the start of every routing call.
// In an FP8 layer the xp region holds the bf16 expert outputs, h the FP8 codes
// of h, and x8 / x8sf / h8sf the FP8 rows and the two scale buffers.
struct Layout {
  size_t flags, rticket, rcnt, rz, zero_end, rzl, rsplit, rlogits, dmask, dbase, dcounts, dticket, op_end;
  size_t idx, w, row_map, seg_off, seg_count, rtok, xp, h, hs, sh, x8, x8sf, h8sf, layer_end;
};

Layout layout(const Dims& D) {
  Layout L{};
  const int64_t db = (D.T + kDispatchTokens - 1) / kDispatchTokens;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = round_up(o + bytes, kAlign);
    return at;
  };
  L.flags = 0;
  L.rticket = sizeof(uint32_t);
  take(kAlign);
  L.rcnt = take(sizeof(int32_t) * D.N);
  L.rz = take(sizeof(unsigned long long) * D.N);
  L.zero_end = o;
  L.rzl = take(sizeof(double) * router_zl_slots(D.T));
  const bool tc_router = D.bf16 && D.N >= kRouterTcMinExperts;
  L.rsplit = take(tc_router ? router_split_bytes(D.d, D.N) : 0);
  L.rlogits = take(tc_router ? sizeof(float) * kRouterMaxPartials * D.T * D.N : 0);
  L.dmask = take(sizeof(uint32_t) * db * D.N);
  L.dbase = take(sizeof(int32_t) * db * D.N);
  L.dcounts = take(sizeof(int32_t) * D.N);
  L.dticket = take(sizeof(uint32_t));
  L.op_end = o;
  L.idx = take(sizeof(int32_t) * D.T * D.k);
  L.w = take(sizeof(float) * D.T * D.k);
  L.row_map = take(sizeof(int32_t) * D.T * D.k);
  L.seg_off = take(sizeof(int32_t) * (D.N + 1));
  L.seg_count = take(sizeof(int32_t) * D.N);
  L.rtok = take(sizeof(int32_t) * D.max_rows);                   // row -> token (bf16 layer: GEMM1 gathers)
  L.xp = take(static_cast<size_t>(D.elem) * D.max_rows * D.d);  // permuted rows / expert outputs
  L.h = take(static_cast<size_t>(D.elem) * D.max_rows * D.f);
  L.hs = take(static_cast<size_t>(D.elem) * (D.fs ? D.T * D.fs : 0));
  L.sh = take(static_cast<size_t>(D.elem) * (D.fs ? D.T * D.d : 0));
  L.x8 = take(D.mx ? static_cast<size_t>(D.max_rows) * D.d : 0);
  L.x8sf = take(D.mx ? static_cast<size_t>(mx_sf_bytes(D.max_rows, D.d)) : 0);
  L.h8sf = take(D.mx ? static_cast<size_t>(mx_sf_bytes(D.max_rows, D.f)) : 0);
  L.layer_end = o;
  return L;
}

// Workspace of the backward pass: the op head (flags, routing and dispatch
// scratch) of the forward layout, then its own arrays.  Row buffers are reused
// in place: o becomes dO, g and u become dG and dU, xp becomes dXp.
struct BwdLayout {
  size_t idx, w, row_map, seg_off, seg_count, logits, counts, dw, dg, dxr, rws, xp, g, u, h, o, gs, us, hs, dxs, end;
};

BwdLayout bwd_layout(const Dims& D) {
  const Layout L = layout(D);
  BwdLayout B{};
  size_t o = L.op_end;
  auto take = [&](size_t bytes) {
    const size_t at_ = o;
    o = round_up(o + bytes, kAlign);
    return at_;
  };
  const size_t T = static_cast<size_t>(D.T), R = static_cast<size_t>(D.max_rows);
  B.idx = take(4 * T * D.k);
  B.w = take(4 * T * D.k);
  B.row_map = take(4 * T * D.k);
  B.seg_off = take(4 * (D.N + 1));
  B.seg_count = take(4 * D.N);
  B.logits = take(4 * T * D.N);
  B.counts = take(4 * D.N);
  B.dw = take(4 * T * D.k);
  B.dg = take(4 * T * D.N);
  B.dxr = take(4 * static_cast<size_t>(router_dxr_rows(D.T)) * D.d);
  B.rws = take(router_grad_scratch_bytes(D.T, D.d, D.N));
  B.xp = take(2 * R * D.d);
  B.g = take(2 * R * D.f);
  B.u = take(2 * R * D.f);
  B.h = take(2 * R * D.f);
  B.o = take(2 * R * D.d);
  B.gs = take(D.fs ? 2 * T * D.fs : 0);
  B.us = take(D.fs ? 2 * T * D.fs : 0);
  B.hs = take(D.fs ? 2 * T * D.fs : 0);
  B.dxs = take(D.fs ? 2 * T * D.d : 0);
  B.end = o;
  return B;
}

template <typename P>
P at(void* ws, size_t off) {
  return reinterpret_cast<P>(static_cast<uint8_t*>(ws) + off);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || ws_bytes < need) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

bool route_stats_requested(const moe_stats_t* s) {
  return s != nullptr && (s->y_frac || s->z_mean || s->l_aux_p3 || s->l_aux_switch || s->counts || s->z_loss ||
                          s->load_std || s->top2_ratio);
}

moe_status_t do_route(const Dims& D, const void* x, const float* w_router, const float* bias,
                      const float* sel_bias, const float* logits_in, float* logits_out, int32_t* topk_idx,
                      float* topk_w, const moe_stats_t* stats, void* ws, cudaStream_t st,
                      const void* w_split = nullptr) {
  const Layout L = layout(D);
  cudaError_t e = cudaMemsetAsync(ws, 0, L.zero_end, st);
  if (e != cudaSuccess) return cuda_status(e);
  const bool want_stats = route_stats_requested(stats);
  if (D.T == 0) {  // empty batch: statistics are zero
    if (want_stats) {
      const moe_stats_t& s = *stats;
      if (e == cudaSuccess && s.y_frac) e = cudaMemsetAsync(s.y_frac, 0, sizeof(float) * D.N, st);
      if (e == cudaSuccess && s.z_mean) e = cudaMemsetAsync(s.z_mean, 0, sizeof(float) * D.N, st);
      if (e == cudaSuccess && s.counts) e = cudaMemsetAsync(s.counts, 0, sizeof(int32_t) * D.N, st);
      if (e == cudaSuccess && s.l_aux_p3) e = cudaMemsetAsync(s.l_aux_p3, 0, sizeof(float), st);
      if (e == cudaSuccess && s.l_aux_switch) e = cudaMemsetAsync(s.l_aux_switch, 0, sizeof(float), st);
      if (e == cudaSuccess && s.z_loss) e = cudaMemsetAsync(s.z_loss, 0, sizeof(float), st);
      if (e == cudaSuccess && s.load_std) e = cudaMemsetAsync(s.load_std, 0, sizeof(float), st);
      if (e == cudaSuccess && s.top2_ratio) e = cudaMemsetAsync(s.top2_ratio, 0, sizeof(float), st);
    }
    return cuda_status(e);
  }
  RouteArgs a{};
  a.T = D.T;
  a.d = D.d;
  a.N = D.N;
  a.k = D.k;
  a.x_is_bf16 = D.bf16 ? 1 : 0;
  a.x = x;
  a.w_router = w_router;
  a.bias = bias;
  a.sel_bias = sel_bias;
  a.logits_in = logits_in;
  a.logits_out = logits_out;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.cnt_acc = at<int32_t*>(ws, L.rcnt);
  a.z_acc = at<unsigned long long*>(ws, L.rz);
  a.ticket = at<uint32_t*>(ws, L.rticket);
  a.zl_part = at<double*>(ws, L.rzl);
  a.want_stats = want_stats ? 1 : 0;
  if (want_stats) a.stats = *stats;
  a.flags = at<uint32_t*>(ws, L.flags);
  a.n_partials = 1;
  if (logits_in == nullptr && D.bf16 && D.N >= kRouterTcMinExperts) {
    // tensor-core router GEMM -> fp32 partial sums over K slices (the router
    // weight's bf16 split made here unless the caller has one); the softmax /
    // top-k pass adds them (and the bias) in a fixed order and writes logits_out
    int parts = 1;
    e = launch_router_tc(a, w_split, w_split == nullptr, at<void*>(ws, L.rsplit), at<float*>(ws, L.rlogits), &parts,
                         st);
    if (e != cudaSuccess) return cuda_status(e);
    a.logits_in = at<float*>(ws, L.rlogits);
    a.n_partials = parts;
  }
  e = launch_route(a, st);
  if (e != cudaSuccess) return cuda_status(e);
  return MOE_OK;
}

moe_status_t do_dispatch(const Dims& D, const void* x, const int32_t* topk_idx, int32_t* row_map,
                         int32_t* seg_off, int32_t* seg_count, void* xp, uint8_t* xp_sf,
                         const moe_stats_t* stats, void* ws, cudaStream_t st, int32_t* row_token = nullptr) {
  const Layout L = layout(D);
  if (D.T == 0) {
    cudaError_t e = cudaMemsetAsync(seg_off, 0, sizeof(int32_t) * (D.N + 1), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(seg_count, 0, sizeof(int32_t) * D.N, st);
    if (e == cudaSuccess && stats && stats->counts) e = cudaMemsetAsync(stats->counts, 0, 4 * D.N, st);
    if (e == cudaSuccess && stats && stats->kept) e = cudaMemsetAsync(stats->kept, 0, 4 * D.N, st);
    if (e == cudaSuccess && stats && stats->num_dropped) e = cudaMemsetAsync(stats->num_dropped, 0, 4, st);
    if (e == cudaSuccess && stats && stats->avg_tokens_per_expert)
      e = cudaMemsetAsync(stats->avg_tokens_per_expert, 0, 4, st);
    return cuda_status(e);
  }
  DispatchArgs a{};
  a.T = D.T;
  a.d = D.d;
  a.N = D.N;
  a.k = D.k;
  a.capacity = D.C;
  a.align = D.align;
  a.elem_bytes = D.elem;
  a.x = x;
  a.topk_idx = topk_idx;
  a.row_map = row_map;
  a.seg_off = seg_off;
  a.seg_count = seg_count;
  a.xp = xp;
  a.xp_sf = xp_sf;
  a.row_token = row_token;
  a.mask = at<uint32_t*>(ws, L.dmask);
  a.base = at<int32_t*>(ws, L.dbase);
  a.counts = at<int32_t*>(ws, L.dcounts);
  a.ticket = at<uint32_t*>(ws, L.dticket);
  if (stats) a.stats = *stats;
  a.flags = at<uint32_t*>(ws, L.flags);
  return cuda_status(launch_dispatch(a, st));
}

moe_status_t do_ffn(const Dims& D, const void* a_rows, const int32_t* seg_off, const int32_t* seg_count,
                    const void* w1, const void* w3, const void* w2, int f, bool dense, void* h, void* out,
                    void* ws, cudaStream_t st, void* save_g = nullptr, void* save_u = nullptr,
                    const int32_t* a_token = nullptr) {
  const Layout L = layout(D);
  FfnArgs a{};
  a.G = dense ? 1 : D.N;
  a.dense_rows = dense ? static_cast<int>(D.T) : 0;
  a.max_count = dense ? static_cast<int>(D.T) : static_cast<int>(D.max_count);
  a.mean_rows = dense ? D.T : std::min<int64_t>(D.max_count, D.T * D.k / D.N);
  a.max_rows = dense ? D.T : D.max_rows;
  a.d = D.d;
  a.f = f;
  a.seg_off = dense ? nullptr : seg_off;
  a.seg_count = dense ? nullptr : seg_count;
  a.a = a_rows;
  a.a_token = a_token;
  a.a_token_rows = a_token != nullptr ? D.T : 0;
  a.w1 = w1;
  a.w3 = w3;
  a.w2 = w2;
  a.h = h;
  a.out = out;
  a.save_g = save_g;
  a.save_u = save_u;
  a.flags = at<uint32_t*>(ws, L.flags);
  if (D.T == 0) return MOE_OK;
  return cuda_status(D.bf16 ? launch_ffn_bf16(a, st) : launch_ffn_f32(a, st));
}

moe_status_t do_ffn_mx(const Dims& D, const void* xp, const void* xp_sf, const int32_t* seg_off,
                       const int32_t* seg_count, const moe_weights_t* w, void* h, void* h_sf, void* out, void* ws,
                       cudaStream_t st) {
  const Layout L = layout(D);
  FfnMxArgs a{};
  a.G = D.N;
  a.mean_rows = std::min<int64_t>(D.max_count, D.T * D.k / D.N);
  a.max_rows = D.max_rows;
  a.d = D.d;
  a.f = D.f;
  a.seg_off = seg_off;
  a.seg_count = seg_count;
  a.a = static_cast<const uint8_t*>(xp);
  a.a_sf = static_cast<const uint8_t*>(xp_sf);
  a.w1 = static_cast<const uint8_t*>(w->w1_mx);
  a.w1_sf = static_cast<const uint8_t*>(w->w1_sf);
  a.w3 = static_cast<const uint8_t*>(w->w3_mx);
  a.w3_sf = static_cast<const uint8_t*>(w->w3_sf);
  a.w2 = static_cast<const uint8_t*>(w->w2_mx);
  a.w2_sf = static_cast<const uint8_t*>(w->w2_sf);
  a.h = static_cast<uint8_t*>(h);
  a.h_sf = static_cast<uint8_t*>(h_sf);
  a.out = out;
  a.flags = at<uint32_t*>(ws, L.flags);
  if (D.T == 0) return MOE_OK;
  return cuda_status(launch_ffn_mx(a, st));
}

bool mx_weights_ok(const moe_weights_t* w) {
  return w != nullptr && w->w1_mx && w->w1_sf && w->w3_mx && w->w3_sf && w->w2_mx && w->w2_sf &&
         aligned16(w->w1_mx) && aligned16(w->w1_sf) && aligned16(w->w3_mx) && aligned16(w->w3_sf) &&
         aligned16(w->w2_mx) && aligned16(w->w2_sf);
}

moe_status_t do_combine(const Dims& D, const void* out_rows, const int32_t* row_map, const float* topk_w,
                        const void* shared_out, void* y, cudaStream_t st) {
  CombineArgs a{};
  a.T = D.T;
  a.d = D.d;
  a.k = D.k;
  a.is_bf16 = D.bf16 ? 1 : 0;
  a.out_rows = out_rows;
  a.row_map = row_map;
  a.topk_w = topk_w;
  a.shared_out = shared_out;
  a.y = y;
  return cuda_status(launch_combine(a, st));
}

bool ffn_weights_ok(const moe_weights_t* w) {
  return w != nullptr && w->w1 && w->w3 && w->w2 && aligned16(w->w1) && aligned16(w->w3) && aligned16(w->w2);
}

}  // namespace

namespace moe {

moe_status_t dispatch_prepare(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                              int32_t* row_map, int32_t* seg_off, int32_t* seg_count, void* xp,
                              const moe_stats_t* stats, DispatchArgs* a, int64_t* blocks) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (seg_off == nullptr || seg_count == nullptr) return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (x == nullptr || topk_idx == nullptr || row_map == nullptr || xp == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_MISALIGNED;
  *a = DispatchArgs{};
  a->T = D.T;
  a->d = D.d;
  a->N = D.N;
  a->k = D.k;
  a->capacity = D.C;
  a->align = D.align;
  a->elem_bytes = D.elem;
  a->x = x;
  a->topk_idx = topk_idx;
  a->row_map = row_map;
  a->seg_off = seg_off;
  a->seg_count = seg_count;
  a->xp = xp;
  a->xp_sf = nullptr;
  if (stats) a->stats = *stats;
  *blocks = (D.T + kDispatchTokens - 1) / kDispatchTokens;
  return MOE_OK;
}

moe_status_t cuda_error_status(cudaError_t e) { return cuda_status(e); }

moe_status_t dispatch_empty(const DispatchArgs& a, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(a.seg_off, 0, sizeof(int32_t) * (a.N + 1), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(a.seg_count, 0, sizeof(int32_t) * a.N, st);
  if (e == cudaSuccess && a.stats.counts) e = cudaMemsetAsync(a.stats.counts, 0, 4 * a.N, st);
  if (e == cudaSuccess && a.stats.kept) e = cudaMemsetAsync(a.stats.kept, 0, 4 * a.N, st);
  if (e == cudaSuccess && a.stats.num_dropped) e = cudaMemsetAsync(a.stats.num_dropped, 0, 4, st);
  if (e == cudaSuccess && a.stats.avg_tokens_per_expert) e = cudaMemsetAsync(a.stats.avg_tokens_per_expert, 0, 4, st);
  return cuda_status(e);
}

}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_NONFINITE: return "MOE_ERR_NONFINITE";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_last_cuda_error(void) { return g_last_cuda_error; }

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

moe_status_t moe_capacity(const moe_config_t* cfg, int32_t* capacity) {
  if (cfg == nullptr || capacity == nullptr) return MOE_ERR_INVALID_ARG;
  if (cfg->T < 0 || cfg->N < 1 || cfg->k < 1) return MOE_ERR_INVALID_ARG;
  if (cfg->capacity >= 0) {
    *capacity = cfg->capacity;
    return MOE_OK;
  }
  return exact_capacity(cfg->capacity_factor, cfg->T, cfg->k, cfg->N, capacity);
}

moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* layer_bytes, size_t* op_bytes,
                                int64_t* max_rows) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  const Layout L = layout(D);
  if (layer_bytes) *layer_bytes = L.layer_end;
  if (op_bytes) *op_bytes = L.op_end;
  if (max_rows) *max_rows = D.max_rows;
  return MOE_OK;
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* w_router, const float* router_bias,
                       const float* selection_bias, float* logits_out, int32_t* topk_idx, float* topk_w,
                       moe_stats_t* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (D.T > 0 && (x == nullptr || w_router == nullptr || topk_idx == nullptr || topk_w == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x)) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_route(D, x, w_router, router_bias, selection_bias, nullptr, logits_out, topk_idx, topk_w, stats, ws,
                  reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_route_with_split(const moe_config_t* cfg, const void* x, const float* w_router,
                                  const void* w_router_split, const float* router_bias, const float* selection_bias,
                                  float* logits_out, int32_t* topk_idx, float* topk_w, moe_stats_t* stats, void* ws,
                                  size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (D.T > 0 && (x == nullptr || w_router == nullptr || topk_idx == nullptr || topk_w == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router_split)) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_route(D, x, w_router, router_bias, selection_bias, nullptr, logits_out, topk_idx, topk_w, stats, ws,
                  reinterpret_cast<cudaStream_t>(stream), D.bf16 ? w_router_split : nullptr);
}

moe_status_t moe_route_from_logits(const moe_config_t* cfg, const float* logits, const float* selection_bias,
                                   int32_t* topk_idx, float* topk_w, moe_stats_t* stats, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (D.T > 0 && (logits == nullptr || topk_idx == nullptr || topk_w == nullptr)) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_route(D, nullptr, nullptr, nullptr, selection_bias, logits, nullptr, topk_idx, topk_w, stats, ws,
                  reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_bias_update(const moe_config_t* cfg, float* selection_bias, const int32_t* counts, float gamma,
                             moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (selection_bias == nullptr || counts == nullptr || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_bias_update(selection_bias, counts, D.T * D.k, D.N, gamma,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, int32_t* row_map,
                          int32_t* seg_off, int32_t* seg_count, void* xp, moe_stats_t* stats, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (seg_off == nullptr || seg_count == nullptr) return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (x == nullptr || topk_idx == nullptr || row_map == nullptr || xp == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp)) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_dispatch(D, x, topk_idx, row_map, seg_off, seg_count, xp, nullptr, stats, ws,
                     reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* xp, const int32_t* seg_off,
                            const int32_t* seg_count, const moe_weights_t* weights, void* h, void* out_rows,
                            void* ws, size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (weights == nullptr || !weights->w1 || !weights->w3 || !weights->w2) return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (xp == nullptr || seg_off == nullptr || seg_count == nullptr || h == nullptr || out_rows == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!ffn_weights_ok(weights) || !aligned16(xp) || !aligned16(h) || !aligned16(out_rows))
    return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_ffn(D, xp, seg_off, seg_count, weights->w1, weights->w3, weights->w2, D.f, false, h, out_rows, ws,
                reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_shared_expert_ffn(const moe_config_t* cfg, const void* x, const moe_weights_t* weights,
                                   void* h_shared, void* shared_out, void* ws, size_t ws_bytes,
                                   moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (D.fs == 0 || weights == nullptr || !weights->ws1 || !weights->ws3 || !weights->ws2) return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (x == nullptr || h_shared == nullptr || shared_out == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(weights->ws1) || !aligned16(weights->ws3) || !aligned16(weights->ws2) ||
      !aligned16(h_shared) || !aligned16(shared_out))
    return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_ffn(D, x, nullptr, nullptr, weights->ws1, weights->ws3, weights->ws2, D.fs, true, h_shared,
                shared_out, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* out_rows, const int32_t* row_map, const float* topk_w,
                         const void* shared_out, void* y, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (D.T > 0 && (out_rows == nullptr || row_map == nullptr || topk_w == nullptr || y == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(out_rows) || !aligned16(shared_out) || !aligned16(y)) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_combine(D, out_rows, row_map, topk_w, shared_out, y, reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_layer_fwd(const moe_config_t* cfg, const moe_weights_t* weights, const void* x, void* y,
                           moe_stats_t* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (weights == nullptr || weights->w_router == nullptr || (D.T > 0 && (x == nullptr || y == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (D.mx ? !(weights->w1_mx && weights->w1_sf && weights->w3_mx && weights->w3_sf && weights->w2_mx &&
               weights->w2_sf)
           : !(weights->w1 && weights->w3 && weights->w2))
    return MOE_ERR_INVALID_ARG;
  if (D.fs > 0 && (!weights->ws1 || !weights->ws3 || !weights->ws2)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !(D.mx ? mx_weights_ok(weights) : ffn_weights_ok(weights)))
    return MOE_ERR_MISALIGNED;
  if (D.fs > 0 && (!aligned16(weights->ws1) || !aligned16(weights->ws3) || !aligned16(weights->ws2)))
    return MOE_ERR_MISALIGNED;
  if (!aligned16(weights->w_router_split)) return MOE_ERR_MISALIGNED;
  const Layout L = layout(D);
  if ((s = check_ws(ws, ws_bytes, L.layer_end)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  int32_t* idx = at<int32_t*>(ws, L.idx);
  float* w = at<float*>(ws, L.w);
  int32_t* row_map = at<int32_t*>(ws, L.row_map);
  int32_t* seg_off = at<int32_t*>(ws, L.seg_off);
  int32_t* seg_count = at<int32_t*>(ws, L.seg_count);
  void* xp = at<void*>(ws, L.xp);
  void* h = at<void*>(ws, L.h);
  void* out_rows = xp;  // expert outputs: the permuted rows are dead once GEMM1 has read them
  void* shared_out = D.fs ? at<void*>(ws, L.sh) : nullptr;

  if ((s = do_route(D, x, weights->w_router, weights->router_bias, weights->selection_bias, nullptr, nullptr, idx, w,
                    stats, ws, st, D.bf16 ? weights->w_router_split : nullptr)) != MOE_OK)
    return s;
  if (D.mx) {
    void* x8 = at<void*>(ws, L.x8);
    uint8_t* x8sf = at<uint8_t*>(ws, L.x8sf);
    if ((s = do_dispatch(D, x, idx, row_map, seg_off, seg_count, x8, x8sf, stats, ws, st)) != MOE_OK) return s;
    if ((s = do_ffn_mx(D, x8, x8sf, seg_off, seg_count, weights, h, at<void*>(ws, L.h8sf), out_rows, ws, st)) !=
        MOE_OK)
      return s;
  } else if (D.bf16 && layer_gathers_rows()) {
    // no permuted copy of x: the dispatch records each kept row's token and the
    // SwiGLU GEMM gathers those rows of x itself
    int32_t* rtok = at<int32_t*>(ws, L.rtok);
    if ((s = do_dispatch(D, x, idx, row_map, seg_off, seg_count, nullptr, nullptr, stats, ws, st, rtok)) != MOE_OK)
      return s;
    if ((s = do_ffn(D, x, seg_off, seg_count, weights->w1, weights->w3, weights->w2, D.f, false, h, out_rows, ws, st,
                    nullptr, nullptr, rtok)) != MOE_OK)
      return s;
  } else {
    if ((s = do_dispatch(D, x, idx, row_map, seg_off, seg_count, xp, nullptr, stats, ws, st)) != MOE_OK) return s;
    if ((s = do_ffn(D, xp, seg_off, seg_count, weights->w1, weights->w3, weights->w2, D.f, false, h, out_rows, ws,
                    st)) != MOE_OK)
      return s;
  }
  if (D.fs > 0 && (s = do_ffn(D, x, nullptr, nullptr, weights->ws1, weights->ws3, weights->ws2, D.fs, true,
                              at<void*>(ws, L.hs), shared_out, ws, st)) != MOE_OK)
    return s;
  return do_combine(D, out_rows, row_map, w, shared_out, y, st);
}

moe_status_t moe_mx_quantize_weight(const void* w, int64_t G, int32_t K, int32_t N, void* codes, void* sf,
                                    moe_stream_t stream) {
  if (G < 0 || K < 1 || N < 1 || G > 65535) return MOE_ERR_INVALID_ARG;
  if (K % 128 || N % 128 || N / 128 > 65535) return MOE_ERR_UNSUPPORTED;
  if (G > 0 && (w == nullptr || codes == nullptr || sf == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(sf)) return MOE_ERR_MISALIGNED;
  return cuda_status(launch_mx_quantize_weight(static_cast<const uint16_t*>(w), G, K, N, static_cast<uint8_t*>(codes),
                                               static_cast<uint8_t*>(sf), reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch_mx(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, int32_t* row_map,
                             int32_t* seg_off, int32_t* seg_count, void* xp_codes, void* xp_sf, moe_stats_t* stats,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (!D.mx) return MOE_ERR_INVALID_ARG;
  if (seg_off == nullptr || seg_count == nullptr) return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (x == nullptr || topk_idx == nullptr || row_map == nullptr || xp_codes == nullptr || xp_sf == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xp_codes) || !aligned16(xp_sf)) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_dispatch(D, x, topk_idx, row_map, seg_off, seg_count, xp_codes, static_cast<uint8_t*>(xp_sf), stats, ws,
                     reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_ffn_mx(const moe_config_t* cfg, const void* xp_codes, const void* xp_sf, const int32_t* seg_off,
                               const int32_t* seg_count, const moe_weights_t* weights, void* h_codes, void* h_sf,
                               void* out_rows, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (!D.mx || weights == nullptr) return MOE_ERR_INVALID_ARG;
  if (!(weights->w1_mx && weights->w1_sf && weights->w3_mx && weights->w3_sf && weights->w2_mx && weights->w2_sf))
    return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (xp_codes == nullptr || xp_sf == nullptr || seg_off == nullptr || seg_count == nullptr ||
                  h_codes == nullptr || h_sf == nullptr || out_rows == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!mx_weights_ok(weights) || !aligned16(xp_codes) || !aligned16(xp_sf) || !aligned16(h_codes) ||
      !aligned16(h_sf) || !aligned16(out_rows))
    return MOE_ERR_MISALIGNED;
  if ((s = check_ws(ws, ws_bytes, layout(D).op_end)) != MOE_OK) return s;
  return do_ffn_mx(D, xp_codes, xp_sf, seg_off, seg_count, weights, h_codes, h_sf, out_rows, ws,
                   reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_backward_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (!D.bf16 || D.mx || D.align % 64) return MOE_ERR_UNSUPPORTED;
  if (bytes) *bytes = bwd_layout(D).end;
  return MOE_OK;
}

moe_status_t moe_layer_bwd(const moe_config_t* cfg, const moe_weights_t* weights, const void* x, const void* dy,
                           float aux_weight, float z_weight, moe_grads_t* grads, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  Dims D;
  moe_status_t s = derive(cfg, &D);
  if (s != MOE_OK) return s;
  if (!D.bf16 || D.mx || D.align % 64) return MOE_ERR_UNSUPPORTED;
  if (weights == nullptr || grads == nullptr || weights->w_router == nullptr || !weights->w1 || !weights->w3 ||
      !weights->w2 || !grads->dw_router || !grads->dw1 || !grads->dw3 || !grads->dw2 || !std::isfinite(aux_weight) ||
      !std::isfinite(z_weight))
    return MOE_ERR_INVALID_ARG;
  if (D.T > 0 && (x == nullptr || dy == nullptr || grads->dx == nullptr)) return MOE_ERR_INVALID_ARG;
  if (D.fs > 0 && (!weights->ws1 || !weights->ws3 || !weights->ws2 || !grads->dws1 || !grads->dws3 || !grads->dws2))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(grads->dx) || !ffn_weights_ok(weights) ||
      !aligned16(grads->dw1) || !aligned16(grads->dw3) || !aligned16(grads->dw2))
    return MOE_ERR_MISALIGNED;
  if (D.fs > 0 && (!aligned16(weights->ws1) || !aligned16(weights->ws3) || !aligned16(weights->ws2) ||
                   !aligned16(grads->dws1) || !aligned16(grads->dws3) || !aligned16(grads->dws2)))
    return MOE_ERR_MISALIGNED;
  if (!aligned16(weights->w_router_split)) return MOE_ERR_MISALIGNED;
  const BwdLayout B = bwd_layout(D);
  if ((s = check_ws(ws, ws_bytes, B.end)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t T = D.T;
  const int d = D.d, N = D.N, k = D.k, f = D.f, fs = D.fs;
  float* dbias = weights->router_bias != nullptr ? grads->drouter_bias : nullptr;

  if (T == 0) {  // no tokens: every weight gradient is zero
    cudaError_t e = cudaMemsetAsync(grads->dw_router, 0, sizeof(float) * d * N, st);
    if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, sizeof(float) * N, st);
    const size_t we = static_cast<size_t>(N) * d * f * sizeof(float);
    if (e == cudaSuccess) e = cudaMemsetAsync(grads->dw1, 0, we, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(grads->dw3, 0, we, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(grads->dw2, 0, we, st);
    if (fs > 0) {
      const size_t se = static_cast<size_t>(d) * fs * sizeof(float);
      if (e == cudaSuccess) e = cudaMemsetAsync(grads->dws1, 0, se, st);
      if (e == cudaSuccess) e = cudaMemsetAsync(grads->dws3, 0, se, st);
      if (e == cudaSuccess) e = cudaMemsetAsync(grads->dws2, 0, se, st);
    }
    return cuda_status(e);
  }

  int32_t* idx = at<int32_t*>(ws, B.idx);
  float* w = at<float*>(ws, B.w);
  int32_t* row_map = at<int32_t*>(ws, B.row_map);
  int32_t* seg_off = at<int32_t*>(ws, B.seg_off);
  int32_t* seg_count = at<int32_t*>(ws, B.seg_count);
  float* logits = at<float*>(ws, B.logits);
  void* xp = at<void*>(ws, B.xp);
  void* g = at<void*>(ws, B.g);
  void* u = at<void*>(ws, B.u);
  void* h = at<void*>(ws, B.h);
  void* o = at<void*>(ws, B.o);
  uint32_t* flags = at<uint32_t*>(ws, layout(D).flags);

  // forward recompute: routing (logits and counts kept), permutation, experts
  // with the SwiGLU pre-activations saved
  moe_stats_t rs{};
  rs.counts = at<int32_t*>(ws, B.counts);
  if ((s = do_route(D, x, weights->w_router, weights->router_bias, weights->selection_bias, nullptr, logits, idx, w,
                    &rs, ws, st, weights->w_router_split)) != MOE_OK)
    return s;
  if ((s = do_dispatch(D, x, idx, row_map, seg_off, seg_count, xp, nullptr, nullptr, ws, st)) != MOE_OK) return s;
  if ((s = do_ffn(D, xp, seg_off, seg_count, weights->w1, weights->w3, weights->w2, f, false, h, o, ws, st, g, u)) !=
      MOE_OK)
    return s;

  BwdSmallArgs a{};
  a.T = T;
  a.d = d;
  a.N = N;
  a.k = k;
  a.f = f;
  a.aux_weight = aux_weight;
  a.z_weight = z_weight;
  a.dy = static_cast<const uint16_t*>(dy);
  a.logits = logits;
  a.topk_idx = idx;
  a.topk_w = w;
  a.row_map = row_map;
  a.counts = rs.counts;
  a.out_rows = static_cast<const uint16_t*>(o);
  a.dO = static_cast<uint16_t*>(o);   // in place: each row is read, then overwritten, by one block
  a.dw = at<float*>(ws, B.dw);
  a.dg = at<float*>(ws, B.dg);
  cudaError_t e = launch_combine_bwd(a, st);
  PadBufs pb{};
  pb.buf[0] = xp;
  pb.cols[0] = d;
  pb.buf[1] = h;
  pb.cols[1] = f;
  pb.buf[2] = o;
  pb.cols[2] = d;
  pb.n = 3;
  if (e == cudaSuccess) e = launch_zero_pad_rows(N, seg_off, seg_count, pb, st);
  if (e == cudaSuccess) e = launch_router_bwd(a, st);

  BwdGroups grp{};
  grp.G = N;
  grp.max_rows = D.max_rows;
  grp.seg_off = seg_off;
  grp.seg_count = seg_count;
  grp.flags = flags;
  if (e == cudaSuccess) e = launch_dgrad_swiglu(grp, d, f, o, weights->w2, g, u, g, u, st);   // dG, dU in place
  if (e == cudaSuccess) e = launch_wgrad(grp, d, f, xp, g, grads->dw1, st);
  if (e == cudaSuccess) e = launch_wgrad(grp, d, f, xp, u, grads->dw3, st);
  if (e == cudaSuccess) e = launch_wgrad(grp, f, d, h, o, grads->dw2, st);
  if (e == cudaSuccess) e = launch_dgrad_plain2(grp, d, f, g, u, weights->w1, weights->w3, xp, st);   // dXp over xp
  float* dxr = at<float*>(ws, B.dxr);
  if (e == cudaSuccess)
    e = launch_router_grads(T, d, N, static_cast<const uint16_t*>(x), a.dg, weights->w_router, grads->dw_router,
                            dbias, dxr, at<void*>(ws, B.rws), flags, st);
  if (e != cudaSuccess) return cuda_status(e);

  void* dxs = nullptr;
  if (fs > 0) {  // the shared expert: one dense group of T rows, weight 1
    void* gs = at<void*>(ws, B.gs);
    void* us = at<void*>(ws, B.us);
    void* hs = at<void*>(ws, B.hs);
    dxs = at<void*>(ws, B.dxs);
    if ((s = do_ffn(D, x, nullptr, nullptr, weights->ws1, weights->ws3, weights->ws2, fs, true, hs, dxs, ws, st, gs,
                    us)) != MOE_OK)
      return s;
    BwdGroups dense{};
    dense.G = 1;
    dense.dense_rows = static_cast<int>(T);
    dense.max_rows = T;
    dense.flags = flags;
    e = launch_dgrad_swiglu(dense, d, fs, dy, weights->ws2, gs, us, gs, us, st);
    if (e == cudaSuccess) e = launch_wgrad(dense, d, fs, x, gs, grads->dws1, st);
    if (e == cudaSuccess) e = launch_wgrad(dense, d, fs, x, us, grads->dws3, st);
    if (e == cudaSuccess) e = launch_wgrad(dense, fs, d, hs, dy, grads->dws2, st);
    if (e == cudaSuccess) e = launch_dgrad_plain2(dense, d, fs, gs, us, weights->ws1, weights->ws3, dxs, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return cuda_status(launch_dx_gather(T, d, k, row_map, static_cast<const uint16_t*>(xp), dxr,
                                      static_cast<const uint16_t*>(dxs), static_cast<uint16_t*>(grads->dx), st));
}

moe_status_t moe_router_split_bytes(int32_t d, int32_t N, size_t* bytes) {
  if (d < 1 || N < 1 || bytes == nullptr) return MOE_ERR_INVALID_ARG;
  if (N > 256) return MOE_ERR_UNSUPPORTED;
  *bytes = router_split_bytes(d, N);
  return MOE_OK;
}

moe_status_t moe_router_split(const float* w_router, int32_t d, int32_t N, void* split, size_t bytes,
                              moe_stream_t stream) {
  if (d < 1 || N < 1 || w_router == nullptr || split == nullptr) return MOE_ERR_INVALID_ARG;
  if (N > 256 || d % 64) return MOE_ERR_UNSUPPORTED;
  if (bytes < router_split_bytes(d, N)) return MOE_ERR_WORKSPACE;
  if (!aligned16(split)) return MOE_ERR_MISALIGNED;
  return cuda_status(launch_router_split(w_router, d, N, split, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_set_wait_limit_ns(uint64_t ns) {
  if (ns > 2000000000ull) return MOE_ERR_INVALID_ARG;
  set_pipeline_wait_ns(ns);
  set_mx_pipeline_wait_ns(ns);
  set_router_wait_ns(ns);
  return MOE_OK;
}

moe_status_t moe_read_flags(const void* ws, size_t ws_bytes, uint32_t* flags, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < sizeof(uint32_t) || flags == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_status(e);
  *flags = v;
  if (v & MOE_FLAG_NONFINITE_LOGITS) return MOE_ERR_NONFINITE;
  if (v & (MOE_FLAG_BAD_EXPERT_INDEX | MOE_FLAG_WAIT_TIMEOUT)) return MOE_ERR_DEVICE;
  return MOE_OK;
}

}  // extern "C"
