// kvattn_decode_noalloc: split-KV decode for callers that cannot allocate device memory.
//
// kvattn_decode takes its per-split scratch from the caller (ws, ws_bytes).  Some callers
// cannot provide it: code hosted inside another framework whose memory pool owns all device
// memory and forbids direct cudaMalloc, or latency-critical loops that must never enter the
// allocator (cudaMalloc/cudaFree may synchronise the device).  This entry point needs no
// allocation at all: its scratch is a file-scope device array of fixed size that every GPU
// loading the library keeps until the process exits.
#include <atomic>

#include "decode.cuh"

namespace kvattn {

// Large enough for every shape kvattn_decode supports on a 148-SM B200 (at most ~3.7 MB:
// 148 splits x 24 query rows x (256 + 1) floats); larger plans are refused.
constexpr size_t kNoAllocScratchBytes = size_t{4} << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch, per device.  In host code the symbol's name stands
// for a host-side shadow, not the device memory, so the address must be looked up.  Host
// threads may make their first call on a device at the same time: each looks the address up
// (the result is the same) and publishes it atomically.
std::atomic<void*> g_noalloc_addr[64] = {};
}  // namespace

}  // namespace kvattn

extern "C" {

KVATTN_API int kvattn_decode_noalloc(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                                     const int32_t* page_list, const int32_t* page_logical,
                                     const int32_t* n_pages, int max_pages, float* out, float* lse,
                                     kvattn_stream_t stream) {
  const kvattn::CallRange range_("kvattn_decode_noalloc");
  int st = validate_desc(desc);
  if (st) return st;
  if (n_q < 1 || max_pages < 0) return KVATTN_ERR_INVALID_ARG;
  // shapes kvattn_decode does not support are refused as such, before the scratch size check
  if ((desc->n_q_heads / desc->n_kv_heads) * n_q > 24) return KVATTN_ERR_UNSUPPORTED_SHAPE;
  int dev;
  if ((st = current_device_checked(&dev))) return st;
  void* scratch = kvattn::g_noalloc_addr[dev].load(std::memory_order_relaxed);
  if (!scratch) {
    // first call on this device (the device is current): look the scratch address up once
    cudaError_t e = cudaGetSymbolAddress(&scratch, kvattn::g_noalloc_scratch);
    if (e != cudaSuccess || !scratch) return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    kvattn::g_noalloc_addr[dev].store(scratch, std::memory_order_relaxed);
  }
  if (kvattn_decode_workspace_size(desc, n_q, max_pages) > kvattn::kNoAllocScratchBytes)
    return KVATTN_ERR_WORKSPACE_TOO_SMALL;
  return kvattn_decode(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse, scratch,
                       kvattn::kNoAllocScratchBytes, stream);
}

}  // extern "C"
