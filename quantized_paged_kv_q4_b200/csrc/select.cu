// KVMem-style block summaries and top-k block selection (KVMem reproduction on one
// 7900 XTX, lcz.me/topic/1972: 128-token blocks; a retrieval query chooses which blocks
// fill a 32,768-token GPU budget, and a 16,384-token recent reserve is always kept).
//
// Readings (the pages do not define the ranking):
//   summary[b][c] = mean over the block's 128 tokens of the dequantized key (Q8_0, Q4_0, Q5_0 or
//                   Q5_1), rounded once to fp32.  Computed exactly: each fp16 scale (and
//                   Q5_1 minimum) is split into an 11-bit integer significand and an
//                   exponent, every code x significand product is shifted onto a common
//                   2^-24 grid and summed in int64 (< 2^54, no overflow), then converted to
//                   fp32 with one rounding.
//   score[b]      = sum_c (sum_j q[j][c]) * summary[b][c] in fp64.
//   selection     = the `budget` highest scores among blocks older than the recent window
//                   (ties: lower block index), plus the recent window and partial tail
//                   blocks, written in ascending order.
#include "decode.cuh"

namespace kvattn {

// ---------------------------------------------------------------- summaries
// q * h for an fp16 bit pattern h, exactly, in units of 2^-24 (the fp16 subnormal step):
// h = +-m * 2^(eff - 25) with m the 11-bit significand.  |q| <= 127 keeps it below 2^47.
__device__ __forceinline__ long long fp16_grid_units(uint16_t h, int q) {
  const int e = (h >> 10) & 31;
  const int mant = h & 1023;
  const int m = e ? (1024 | mant) : mant;
  const int eff = e ? e : 1;
  const long long term = static_cast<long long>(q * m) * (1ll << (eff - 1));
  return (h & 0x8000) ? -term : term;
}

__global__ void __launch_bounds__(256) block_summary_kernel(const uint8_t* __restrict__ k_pool, int64_t k_stride,
                                                            int64_t n_pages, const int32_t* __restrict__ page_table,
                                                            int n_blocks, int block_begin, int n_range,
                                                            int k_fmt, float* __restrict__ summaries) {
  __shared__ __align__(16) uint8_t page[kKPageBytes];
  const int unit = blockIdx.y;
  const int b = block_begin + blockIdx.x;
  const int pg = page_table[static_cast<long long>(unit) * n_blocks + b];
  if (pg < 0 || pg >= n_pages) {
    if (threadIdx.x == 0) record_error(KVATTN_ERR_BAD_PAGE);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(k_pool + static_cast<int64_t>(pg) * k_stride);
  uint4* dst = reinterpret_cast<uint4*>(page);
  const int bytes = k_fmt == kKeyQ4    ? kK4PageBytes
                    : k_fmt == kKeyQ51 ? kK5PageBytes
                    : k_fmt == kKeyQ50 ? kK50PageBytes
                                       : kKPageBytes;
  const int scale_off = k_fmt == kKeyQ4 ? kK4ScaleOffset : k_fmt == kKeyQ8 ? kKScaleOffset : kK5ScaleOffset;
  for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) dst[i] = src[i];
  __syncthreads();
  const int c = threadIdx.x;  // channel
  const int blk = c >> 5;
  // Q8_0 key byte: token-row base + 16 * T + j; Q4_0 key word: base + T * 4 + (blk & 3), then
  // the nibble of channel i = c & 7 at bit 4 * (i / 2) + 16 * (i % 2)
  const int P = c >> 6, cc = c & 63, T = (cc & 31) >> 3, j = 8 * (cc >> 5) + (cc & 7);
  const int i8 = c & 7, nib_shift = 4 * (i8 >> 1) + 16 * (i8 & 1);
  long long acc = 0;
  for (int tok = 0; tok < kPageTokens; ++tok) {
    const int G = tok >> 4, H = (tok & 15) >> 3, R = tok & 7;
    int q;
    if (k_fmt != kKeyQ8) {
      const int row = (((G * 2 + (blk >> 2)) * 2 + H) * 8 + R) * 4 + T;
      const uint32_t w = *reinterpret_cast<const uint32_t*>(page + 4 * (row * 4 + (blk & 3)));
      q = static_cast<int>((w >> nib_shift) & 15u);
      if (k_fmt == kKeyQ4) {
        q -= 8;
      } else {
        const uint32_t fifth = *reinterpret_cast<const uint32_t*>(page + kK5HighOffset + 4 * row);
        q |= static_cast<int>((fifth >> (16 * (i8 & 1) + 4 * (blk & 3) + (i8 >> 1))) & 1u) << 4;
        if (k_fmt == kKeyQ50) q -= 16;
      }
    } else {
      q = static_cast<int>(page[((((G * 4 + P) * 2 + H) * 8 + R) * 4 + T) * 16 + j]) - 128;  // offset-binary
    }
    const int si = 2 * (((G * 8 + R) * 2 + H) * 8 + blk);
    acc += fp16_grid_units(*reinterpret_cast<const uint16_t*>(page + scale_off + si), q);
    if (k_fmt == kKeyQ51) acc += fp16_grid_units(*reinterpret_cast<const uint16_t*>(page + kK5MinOffset + si), 1);
  }
  // value = acc * 2^-24 / 128
  const float r = __ll2float_rn(acc) * 4.656612873077392578125e-10f;  // 2^-31
  summaries[(static_cast<long long>(unit) * n_blocks + b) * kHeadDim + c] = r;
}

// ---------------------------------------------------------------- scores
// One warp per block.  The CTA first sums the group's query rows per channel (fp64, over the
// rows in order) into shared memory; lane l then takes channels 4l..4l+3 and 128 + 4l..4l+3.
__global__ void __launch_bounds__(256) block_score_kernel(const float* __restrict__ summaries,
                                                          const float* __restrict__ q_group, int group, int n_blocks,
                                                          int n_cand, double* __restrict__ scores) {
  // launched with programmatic dependent launch: the top-k grid behind this one may start
  // now, and this grid reads the retrieval queries only once the kernel before it completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ double u_s[kHeadDim];
  const int unit = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* qg = q_group + static_cast<long long>(unit) * group * kHeadDim;
  {
    const int c = threadIdx.x;  // blockDim.x == kHeadDim
    double u = 0.0;
    for (int j = 0; j < group; ++j) u += qg[j * kHeadDim + c];
    u_s[c] = u;
  }
  __syncthreads();
  const int b = blockIdx.x * (blockDim.x >> 5) + warp;
  if (b >= n_cand) return;
  const float* sm = summaries + (static_cast<long long>(unit) * n_blocks + b) * kHeadDim;
  double acc = 0.0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int c0 = lane * 4 + 128 * k;
    const float4 sv = *reinterpret_cast<const float4*>(sm + c0);
    acc = fma(u_s[c0], static_cast<double>(sv.x), acc);
    acc = fma(u_s[c0 + 1], static_cast<double>(sv.y), acc);
    acc = fma(u_s[c0 + 2], static_cast<double>(sv.z), acc);
    acc = fma(u_s[c0 + 3], static_cast<double>(sv.w), acc);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) scores[static_cast<long long>(unit) * n_blocks + b] = acc;
}

// ---------------------------------------------------------------- top-k + compaction
__device__ __forceinline__ unsigned long long order_key(double x) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

constexpr int kSelThreads = 1024;
constexpr int kMaxCand = 16384;

// Exclusive prefix sum of one int per thread over the CTA (kSelThreads threads); `warp_tot`
// is shared scratch of kSelThreads / 32 ints.  Returns this thread's exclusive prefix and
// writes the CTA total to *total (shared).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive over warps
    if (lane == 31) *total = t;
  }
  __syncthreads();
  const int r = x - v + (warp > 0 ? warp_tot[warp - 1] : 0);
  __syncthreads();  // warp_tot may be reused by the caller
  return r;
}

// Exclusive prefix sums of two ints per thread over the CTA (kSelThreads threads), in one
// pass; `warp_tot` is shared scratch of kSelThreads / 32 pairs, read again by no caller.
// Returns this thread's exclusive prefixes and writes the CTA totals to *total (shared).
__device__ __forceinline__ int2 block_exclusive_scan2(int a, int b, int2* warp_tot, int2* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = a, y = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xo = __shfl_up_sync(0xffffffffu, x, o), yo = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) {
      x += xo;
      y += yo;
    }
  }
  if (lane == 31) warp_tot[warp] = make_int2(x, y);
  __syncthreads();
  if (warp == 0) {
    int2 t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int xo = __shfl_up_sync(0xffffffffu, t.x, o), yo = __shfl_up_sync(0xffffffffu, t.y, o);
      if (lane >= o) {
        t.x += xo;
        t.y += yo;
      }
    }
    warp_tot[lane] = t;  // inclusive over warps
    if (lane == 31) *total = t;
  }
  __syncthreads();
  int2 r = make_int2(x - a, y - b);
  if (warp > 0) {
    r.x += warp_tot[warp - 1].x;
    r.y += warp_tot[warp - 1].y;
  }
  return r;
}

// Top-`budget` candidates by (score desc, block index asc), plus the recent window and the
// tail, compacted into ascending logical ids.  The `take`-th largest 64-bit order key is found
// by an 8-bit radix select, most significant digit first; candidates above it are taken, and
// those equal to it are taken in index order until `take` are chosen, which is exactly the
// first `take` of a sort by (score desc, index asc).  The select stops after the first pass
// whose threshold bin holds exactly as many keys as are still to be taken: every key of that
// bin is then taken, so the remaining digits cannot change the selection.
__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(const double* __restrict__ scores, int n_blocks,
                                                                 int n_cand, int n_total, int budget,
                                                                 const int32_t* __restrict__ page_table,
                                                                 int32_t* __restrict__ sel_logical,
                                                                 int32_t* __restrict__ sel_phys,
                                                                 int32_t* __restrict__ n_sel, int cap) {
  extern __shared__ __align__(16) uint8_t sm[];
  // two digit histograms: pass p counts into hist[p % 2] while the other is cleared for the
  // next pass, so a pass needs two CTA barriers; sel[p % 2] holds pass p's result
  __shared__ int hist[2][256];
  __shared__ int sel[2][3];  // digit, keys still needed inside its bin, keys in its bin
  __shared__ int2 warp_tot2[kSelThreads / 32];
  __shared__ int2 s_tot2;  // CTA totals of (equal keys, surely taken)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the decode may set up
  for (int b = threadIdx.x; b < 2 * 256; b += kSelThreads) (&hist[0][0])[b] = 0;
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the scores are complete
  const int unit = blockIdx.x;
  unsigned long long* key = reinterpret_cast<unsigned long long*>(sm);  // [n_cand]
  const double* sc = scores + static_cast<long long>(unit) * n_blocks;
  const int take = min(budget, n_cand);
  const bool selecting = take > 0 && take < n_cand;
  // the keys, with the first pass's histogram (most significant digit) counted on the way
  for (int i = threadIdx.x; i < n_cand; i += kSelThreads) {
    const unsigned long long k = order_key(sc[i]);
    key[i] = k;
    if (selecting) atomicAdd(&hist[0][static_cast<int>(k >> 56)], 1);
  }
  unsigned long long prefix = 0ull, mask = 0ull;
  int need = take;  // how many still to take among keys matching prefix under mask
  __syncthreads();
  if (selecting) {
    for (int shift = 56, pass = 0; shift >= 0; shift -= 8, ++pass) {
      int* h = hist[pass & 1];
      if (pass > 0) {
        for (int i = threadIdx.x; i < n_cand; i += kSelThreads) {
          const unsigned long long k = key[i];
          if ((k & mask) == prefix) atomicAdd(&h[static_cast<int>((k >> shift) & 255ull)], 1);
        }
        __syncthreads();
      }
      if (threadIdx.x >= 32) {
        // the other histogram was last read by the previous pass's scan, before its barrier
        for (int b = threadIdx.x - 32; b < 256; b += kSelThreads - 32) hist[(pass + 1) & 1][b] = 0;
      } else {
        // lane l owns bins 255 - 8l - e (e = 0..7), highest first; find the digit whose bin
        // holds the need-th largest remaining key
        const int lane = threadIdx.x;
        int c[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = h[255 - 8 * lane - e];
          sum += c[e];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int before = incl - sum;  // keys in higher bins than this lane's
        if (before < need && need <= incl) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (before < need && need <= before + c[e]) {
              sel[pass & 1][0] = 255 - 8 * lane - e;
              sel[pass & 1][1] = need - before;
              sel[pass & 1][2] = c[e];
            }
            before += c[e];
          }
        }
      }
      __syncthreads();
      // sel[pass % 2] is written again two passes on, after a barrier every thread passes
      // only once it has read it here
      prefix |= static_cast<unsigned long long>(sel[pass & 1][0]) << shift;
      mask |= 255ull << shift;
      need = sel[pass & 1][1];
      if (sel[pass & 1][2] == need) break;
    }
  }
  // Selection and compaction in one pass over contiguous ranges of all n_total block
  // indices, in ascending order.  A candidate is taken when its key is above the threshold,
  // or equal to it and among the first `need` equal keys in index order; the blocks past the
  // candidates (the recent window and the tail) always are.  One CTA scan of (equal keys,
  // surely taken) per thread gives the thread both the rank of its first equal key and its
  // output position: the surely taken blocks before it plus the min(need, equal keys before
  // it) equal ones taken among them.
  const bool take_all = take >= n_cand;
  const int per = (n_total + kSelThreads - 1) / kSelThreads;
  const int i0 = min(n_total, threadIdx.x * per), i1 = min(n_total, i0 + per);
  int eq = 0, sure = 0;
  for (int i = i0; i < i1; ++i) {
    if (i >= n_cand || take_all) {
      ++sure;
    } else if (selecting) {
      const unsigned long long k = key[i] & mask;
      sure += k > prefix;
      eq += k == prefix;
    }
  }
  const int2 before = block_exclusive_scan2(eq, sure, warp_tot2, &s_tot2);
  const int32_t* pt = page_table + static_cast<long long>(unit) * n_blocks;
  int32_t* out_l = sel_logical + static_cast<long long>(unit) * cap;
  int32_t* out_p = sel_phys + static_cast<long long>(unit) * cap;
  int rank = before.x;
  int pos = before.y + max(0, min(need, before.x));
  constexpr int kChunk = 4;  // page ids loaded up front, all independent
  for (int c0 = i0; c0 < i1; c0 += kChunk) {
    int32_t pg[kChunk];
#pragma unroll
    for (int e = 0; e < kChunk; ++e) pg[e] = c0 + e < i1 ? pt[c0 + e] : 0;
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const int i = c0 + e;
      if (i >= i1) break;
      bool sel;
      if (i >= n_cand || take_all) {
        sel = true;
      } else if (!selecting) {
        sel = false;
      } else {
        const unsigned long long k = key[i] & mask;
        sel = k > prefix || (k == prefix && rank++ < need);
      }
      if (sel) {
        if (pos < cap) {
          out_l[pos] = i;
          out_p[pos] = pg[e];
        }
        ++pos;
      }
    }
  }
  if (threadIdx.x == 0) n_sel[unit] = min(s_tot2.y + max(0, min(need, s_tot2.x)), cap);
}

cudaError_t launch_block_summaries(const kvattn_kv_desc& d, const int32_t* page_table, int n_units, int n_blocks,
                                   int block_begin, int block_end, float* summaries, cudaStream_t stream) {
  const int n = block_end - block_begin;
  if (n <= 0 || n_units <= 0) return cudaSuccess;
  dim3 grid(n, n_units);
  block_summary_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint8_t*>(d.k_pool), d.k_page_stride, d.n_pages,
                                                 page_table, n_blocks, block_begin, n,
                                                 key_format_id(d.k_fmt),
                                                 summaries);
  return cudaGetLastError();
}

size_t select_smem_bytes(int n_cand) { return static_cast<size_t>(n_cand > 0 ? n_cand : 1) * 8; }

cudaError_t prepare_select_kernels() {
  return cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(select_smem_bytes(kMaxCand)));
}

cudaError_t launch_select(const float* summaries, const float* q_group, int n_units, int group, int n_blocks,
                          int n_cand, int n_total, int budget, const int32_t* page_table, int32_t* sel_logical,
                          int32_t* sel_phys, int32_t* n_sel, int cap, double* scores, cudaStream_t stream) {
  // both grids use programmatic dependent launch: each may start while the kernel before it
  // on the stream drains, and waits for it (griddepcontrol.wait) before reading its inputs
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  if (n_cand > 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((n_cand + 7) / 8, n_units);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, block_score_kernel, summaries, q_group, group, n_blocks, n_cand, scores);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_units);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = select_smem_bytes(max(n_cand, 1));
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_topk_kernel, static_cast<const double*>(scores), n_blocks, n_cand, n_total,
                            budget, page_table, sel_logical, sel_phys, n_sel, cap);
}

}  // namespace kvattn
