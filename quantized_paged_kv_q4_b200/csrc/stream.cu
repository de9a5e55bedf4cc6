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

namespace kvattn {

// Resident-page reuse (KVMem reproduction, lcz.me/topic/1972, recall section: the GPU
// working set follows the retrieval query; a block already on the GPU need not cross PCIe
// again).  One CTA per unit (layer, KV head) with a pool of n_slots device slots:
//   * a selected block that is resident keeps its slot;
//   * free slots are the empty ones and those holding an unselected block;
//   * misses (selected, not resident), in selection order (ascending blocks), take the free
//     slots in ascending slot order; evicted blocks stop being resident;
//   * page_list[i] = the pool page holding selected block i; the copy list names host page
//     and pool page of every miss (dst -1 past n_copies), ready for kvattn_gather_pages.
// Blocks >= n_full are not managed: their page-list entry is extra_page[unit].
constexpr int kResThreads = 1024;

__global__ void __launch_bounds__(kResThreads) resident_update_kernel(
    const int32_t* __restrict__ sel, const int32_t* __restrict__ n_sel_arr, int cap, int n_blocks, int n_full,
    int32_t* __restrict__ slot_of_block, int32_t* __restrict__ block_of_slot, int n_slots,
    const int32_t* __restrict__ host_page, int64_t first_page, const int32_t* __restrict__ extra_page,
    int32_t* __restrict__ page_list, int32_t* __restrict__ copy_host, int32_t* __restrict__ copy_dst,
    int32_t* __restrict__ n_copies) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint32_t* chosen = reinterpret_cast<uint32_t*>(sm);                  // [n_blocks / 32] bitmap
  int* free_by_rank = reinterpret_cast<int*>(chosen + (n_blocks + 31) / 32);  // [n_slots]
  __shared__ int warp_tot[kResThreads / 32];
  __shared__ int s_misses, s_free;
  const int u = blockIdx.x;
  const int32_t* su = sel + static_cast<long long>(u) * cap;
  int32_t* sob = slot_of_block + static_cast<long long>(u) * n_blocks;
  int32_t* bos = block_of_slot + static_cast<long long>(u) * n_slots;
  const int32_t* hp = host_page + static_cast<long long>(u) * n_blocks;
  int32_t* pl = page_list + static_cast<long long>(u) * cap;
  int32_t* ch = copy_host + static_cast<long long>(u) * cap;
  int32_t* cd = copy_dst + static_cast<long long>(u) * cap;
  const int ns = min(max(n_sel_arr[u], 0), cap);
  const int64_t base = first_page + static_cast<int64_t>(u) * n_slots;

  for (int w = threadIdx.x; w < (n_blocks + 31) / 32; w += kResThreads) chosen[w] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < ns; i += kResThreads) {
    const int b = su[i];
    if (b >= 0 && b < n_full) atomicOr(&chosen[b >> 5], 1u << (b & 31));
  }
  __syncthreads();
  // misses in selection order, free slots in slot order: contiguous ranges per thread
  const int pi = (ns + kResThreads - 1) / kResThreads;
  const int i0 = min(ns, threadIdx.x * pi), i1 = min(ns, i0 + pi);
  int nm = 0;
  for (int i = i0; i < i1; ++i) {
    const int b = su[i];
    if (b >= 0 && b < n_full && sob[b] < 0) ++nm;
  }
  const int ps = (n_slots + kResThreads - 1) / kResThreads;
  const int s0 = min(n_slots, threadIdx.x * ps), s1 = min(n_slots, s0 + ps);
  int nf = 0;
  for (int s = s0; s < s1; ++s) {
    const int b = bos[s];
    if (b < 0 || b >= n_full || !(chosen[b >> 5] >> (b & 31) & 1u)) ++nf;
  }
  int miss_rank = block_exclusive_scan(nm, warp_tot, &s_misses);
  int free_rank = block_exclusive_scan(nf, warp_tot, &s_free);
  const int n_miss = s_misses;
  for (int s = s0; s < s1; ++s) {
    const int b = bos[s];
    if (b < 0 || b >= n_full || !(chosen[b >> 5] >> (b & 31) & 1u)) free_by_rank[free_rank++] = s;
  }
  __syncthreads();
  if (n_miss > s_free) {  // fewer slots than selected blocks: nothing is changed
    if (threadIdx.x == 0) {
      record_error(KVATTN_ERR_INVALID_ARG);
      n_copies[u] = 0;
    }
    for (int i = threadIdx.x; i < cap; i += kResThreads) cd[i] = -1;
    return;
  }
  // evict first (every evicted block is unselected, so no selected entry reads it), then fill
  for (int r = threadIdx.x; r < n_miss; r += kResThreads) {
    const int old = bos[free_by_rank[r]];
    if (old >= 0 && old < n_blocks) sob[old] = -1;
  }
  __syncthreads();
  for (int i = i0; i < i1; ++i) {
    const int b = su[i];
    if (b < 0 || b >= n_full) {
      pl[i] = extra_page[u];
      continue;
    }
    int s = sob[b];
    if (s < 0) {
      const int r = miss_rank++;
      s = free_by_rank[r];
      bos[s] = b;
      sob[b] = s;
      ch[r] = hp[b];
      cd[r] = static_cast<int32_t>(base + s);
    }
    pl[i] = static_cast<int32_t>(base + s);
  }
  for (int r = n_miss + threadIdx.x; r < cap; r += kResThreads) {
    ch[r] = 0;
    cd[r] = -1;
  }
  if (threadIdx.x == 0) n_copies[u] = n_miss;
}

size_t resident_smem_bytes(int n_blocks, int n_slots) {
  return static_cast<size_t>((n_blocks + 31) / 32) * 4 + static_cast<size_t>(n_slots) * 4;
}

cudaError_t launch_resident_update(const int32_t* sel, const int32_t* n_sel, int cap, int n_units, int n_blocks,
                                   int n_full, int32_t* slot_of_block, int32_t* block_of_slot, int n_slots,
                                   const int32_t* host_page, int64_t first_page, const int32_t* extra_page,
                                   int32_t* page_list, int32_t* copy_host, int32_t* copy_dst, int32_t* n_copies,
                                   cudaStream_t stream) {
  resident_update_kernel<<<n_units, kResThreads, resident_smem_bytes(n_blocks, n_slots), stream>>>(
      sel, n_sel, cap, n_blocks, n_full, slot_of_block, block_of_slot, n_slots, host_page, first_page, extra_page,
      page_list, copy_host, copy_dst, n_copies);
  return cudaGetLastError();
}

cudaError_t prepare_resident_kernels() {
  return cudaFuncSetAttribute(resident_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(resident_smem_bytes(262144, 16384)));
}

}  // namespace kvattn
