// moe_dispatch_static: the dispatch of dispatch.cu for callers that cannot
// allocate device memory.  Its scratch (per-block token masks and rank bases,
// per-expert counts, the scan's ticket and a flags word) lives in one
// file-scope device array of fixed size that the library holds on every GPU
// that loads it.  The host never touches the array through its name: the name
// is only a host-side stand-in, so the device address is looked up with
// cudaGetSymbolAddress, with the caller's device current, on every call and
// passed to the kernels as plain pointers.  Looking it up each time (a host-side
// table lookup once the device code is loaded) keeps the address right even
// after cudaDeviceReset or a new primary context, which load the module again
// and may place the array elsewhere.
#include "internal.h"

namespace {

constexpr size_t kCells = MOE_DISPATCH_STATIC_MAX_CELLS;  // ceil(T/32) * N
constexpr size_t kMaskOff = 0;
constexpr size_t kBaseOff = kMaskOff + 4 * kCells;
constexpr size_t kCountsOff = kBaseOff + 4 * kCells;     // 256 int32
constexpr size_t kTicketOff = kCountsOff + 4 * 256;
constexpr size_t kFlagOff = kTicketOff + 256;
constexpr size_t kScratchBytes = MOE_DISPATCH_STATIC_SCRATCH_BYTES;
static_assert(kFlagOff + 256 <= kScratchBytes, "static dispatch scratch layout");

static __device__ __align__(256) uint8_t g_dispatch_scratch[kScratchBytes];

// Device address of g_dispatch_scratch in the current device's context.  The
// first lookup on a device loads the library's device code there.
cudaError_t scratch_address(uint8_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
  if (e != cudaSuccess) return e;
  if (p == nullptr) return cudaErrorInvalidSymbol;
  *out = static_cast<uint8_t*>(p);
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_dispatch_static(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                            int32_t* row_map, int32_t* seg_off, int32_t* seg_count, void* xp,
                                            moe_stats_t* stats, uint32_t* device_flags, moe_stream_t stream) {
  moe::DispatchArgs a;
  int64_t blocks = 0;
  moe_status_t s = moe::dispatch_prepare(cfg, x, topk_idx, row_map, seg_off, seg_count, xp, stats, &a, &blocks);
  if (s != MOE_OK) return s;
  if (blocks * a.N > static_cast<int64_t>(kCells)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (a.T == 0) return moe::dispatch_empty(a, st);

  uint8_t* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return moe::cuda_error_status(e);
  a.mask = reinterpret_cast<uint32_t*>(base + kMaskOff);
  a.base = reinterpret_cast<int32_t*>(base + kBaseOff);
  a.counts = reinterpret_cast<int32_t*>(base + kCountsOff);
  a.ticket = reinterpret_cast<uint32_t*>(base + kTicketOff);  // zeroed by the first kernel
  if (device_flags != nullptr) {
    a.flags = device_flags;
  } else {
    a.flags = reinterpret_cast<uint32_t*>(base + kFlagOff);    // written, never reported
  }
  return moe::cuda_error_status(moe::launch_dispatch(a, st));
}
