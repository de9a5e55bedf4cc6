// kvattn_decode_noalloc: split-KV decode for callers that cannot allocate device memory.
//
// kvattn_decode takes its per-split scratch from the caller (ws, ws_bytes).  Some callers
// cannot provide it: code hosted inside another framework whose memory pool owns all device
// memory and forbids direct cudaMalloc, or latency-critical loops that must never enter the
// allocator (cudaMalloc/cudaFree may synchronise the device).  This entry point needs no
// allocation at all: its scratch is a file-scope device array of fixed size that every GPU
// loading the library keeps until the process exits.
#include "decode.cuh"

namespace kvattn {

// Large enough for every shape kvattn_decode supports on a 148-SM B200 (at most ~3.7 MB:
// 148 splits x 24 query rows x (256 + 1) floats); larger plans are refused.
constexpr size_t kNoAllocScratchBytes = size_t{4} << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch, per device.  In host code the symbol's name stands
// for a host-side shadow, not the device memory, so the address must be looked up.
void* g_noalloc_addr[64] = {};
}  // namespace

}  // namespace kvattn

extern "C" {

KVATTN_API int kvattn_decode_noalloc(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                                     const int32_t* page_list, const int32_t* page_logical,
                                     const int32_t* n_pages, int max_pages, float* out, float* lse,
                                     kvattn_stream_t stream) {
  int st = validate_desc(desc);
  if (st) return st;
  if (n_q < 1 || max_pages < 0) return KVATTN_ERR_INVALID_ARG;
  int dev;
  if ((st = current_device_checked(&dev))) return st;
  if (!kvattn::g_noalloc_addr[dev]) {
    // first call on this device (the device is current): look the scratch address up once
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, kvattn::g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    kvattn::g_noalloc_addr[dev] = ptr;
  }
  if (kvattn_decode_workspace_size(desc, n_q, max_pages) > kvattn::kNoAllocScratchBytes)
    return KVATTN_ERR_WORKSPACE_TOO_SMALL;
  return kvattn_decode(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse,
                       kvattn::g_noalloc_addr[dev], kvattn::kNoAllocScratchBytes, stream);
}

}  // extern "C"
