// Page movement between a pinned host pool and device page slots, driven by device-side
// page lists (Adaptive KV Streaming + RDNA 4 announcement, wqu.guru: the full KV history
// stays in host RAM and the bounded working set is streamed over PCIe alongside compute;
// method list: layer L+1's transfers overlap layer L's compute).
//
// kvattn_stream_pages issues one cudaMemcpyAsync per run of consecutive pages from host page
// lists.  These kernels are the other route: the GPU reads (or writes) the device-mapped
// pinned host pool directly over PCIe, taking the page ids from device memory, so a
// selection computed on the GPU feeds the copy without a host round trip.  A few CTAs keep
// enough 16-byte requests in flight to fill the link and leave the rest of the GPU to the
// attention kernels running concurrently on another stream.
#include "common.cuh"

namespace kvattn {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;

// to_device: dst = device slot, src = host page; otherwise the reverse.
__global__ void __launch_bounds__(kGatherThreads) page_copy_kernel(const uint8_t* __restrict__ host_pool,
                                                                   int64_t host_stride, int64_t n_host,
                                                                   uint8_t* __restrict__ dev_pool, int64_t dev_stride,
                                                                   int64_t n_slots, int64_t page_bytes,
                                                                   const int32_t* __restrict__ host_ids,
                                                                   const int32_t* __restrict__ dev_slots, int n,
                                                                   int to_device) {
  const int64_t chunks = page_bytes / 16;
  for (int e = blockIdx.x; e < n; e += gridDim.x) {
    const int hid = host_ids[e], slot = dev_slots[e];
    if (slot < 0) continue;  // entry not to be moved
    if (hid < 0 || hid >= n_host || slot >= n_slots) {
      if (threadIdx.x == 0) record_error(KVATTN_ERR_BAD_PAGE);
      continue;
    }
    const uint4* src;
    uint4* dst;
    if (to_device) {
      src = reinterpret_cast<const uint4*>(host_pool + static_cast<int64_t>(hid) * host_stride);
      dst = reinterpret_cast<uint4*>(dev_pool + static_cast<int64_t>(slot) * dev_stride);
    } else {
      src = reinterpret_cast<const uint4*>(dev_pool + static_cast<int64_t>(slot) * dev_stride);
      dst = reinterpret_cast<uint4*>(const_cast<uint8_t*>(host_pool) + static_cast<int64_t>(hid) * host_stride);
    }
    for (int64_t c0 = threadIdx.x; c0 < chunks; c0 += kGatherThreads * kGatherUnroll) {
      uint4 v[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int64_t c = c0 + u * kGatherThreads;
        if (c < chunks) v[u] = src[c];
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int64_t c = c0 + u * kGatherThreads;
        if (c < chunks) dst[c] = v[u];
      }
    }
  }
}

cudaError_t launch_page_copy(const void* host_dev_ptr, int64_t host_stride, int64_t n_host, void* dev_pool,
                             int64_t dev_stride, int64_t n_slots, int64_t page_bytes, const int32_t* host_ids,
                             const int32_t* dev_slots, int n, int n_ctas, int to_device, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int grid = n_ctas > 0 ? (n_ctas < n ? n_ctas : n) : (n < 32 ? n : 32);
  page_copy_kernel<<<grid, kGatherThreads, 0, stream>>>(static_cast<const uint8_t*>(host_dev_ptr), host_stride,
                                                        n_host, static_cast<uint8_t*>(dev_pool), dev_stride, n_slots,
                                                        page_bytes, host_ids, dev_slots, n, to_device);
  return cudaGetLastError();
}

}  // namespace kvattn
