// Chunked prefill over block-quantized KV pages (Q8_0, Q4_0 or Q5_1 keys with Q4_0 or Q8_0
// values, Q5_0 keys with Q4_1 values) on tcgen05 tensor cores (Adaptive KV Streaming + RDNA 4
// announcement, wqu.guru, method list: "online log-sum-exp prefill": the prefill of a chunk is
// computed across streamed KV pages and the partial results are accumulated by online
// log-sum-exp; the six-step validation guide, alphalab.site, build step: the q8_0-q4_0 and
// q4_0-q4_0 flash-attention KV pairs;
// Vulkan speculative-decoding report, lcz.me/topic/1398, pitfalls: the K q5_1 / V q4_0 cache;
// 7900 XTX MTP tuning notes, lcz.me/topic/593: a q5_0 / q4_1 cache).
//
// Work unit: a cluster of two CTAs = a KV head, two M-tiles of 128 query rows of that head's
// group (row r = token t * group + j: all query heads of a group share the K/V tiles), and
// one run of KV splits, walked in 64-key tiles (half pages).  The pair issues CTA-pair MMAs
// (cta_group::2, M = 256): each CTA holds the accumulators and A operands of its own 128 rows
// in its tensor memory, and half of every B operand in its shared memory, so each CTA
// dequantizes half of every tile (K^ of 32 keys, V^T of 128 dimensions) and nothing is
// copied between the CTAs.  Roles per CTA:
//
//   producer (1 thread)   bulk async copies (TMA engine) of its raw K / V bytes of a tile
//                         into a two-stage shared-memory ring
//   dequant warps (8)     raw -> K^ and V^T, each as an f16 high part (code x scale rounded
//                         once) and an f16 low part (the remainder, exact): together the
//                         dequantized values exactly (Q5_1 keys and Q4_1 values, code x
//                         scale + minimum: to the one fp32 rounding of the sum); K-major,
//                         128-byte swizzle,
//                         three deep (two with Q8_0 values)
//   MMA issuer (1 warp,   S = Q K^T (N = 64 keys, K = 256) as Q K^_hi^T + Q K^_lo^T, and
//     even CTA only)      O += P V (N = 256 dims, K = 64 keys) as P_hi V^_hi + P_lo V^_hi +
//                         P_hi V^_lo; Q and P from tensor memory
//   softmax warps (4)     thread = query row = TMEM lane: S -> causal mask -> running max
//                         (the row of O is rescaled only when its max grows by more than
//                         2^8) -> P = exp2(S log2(e) - m) split into f16 high and low parts
//                         written over S
//
// Q (bf16) is stored as Q/16 in f16, which is exact; log2(e) is applied in fp32 to S.  Every
// operand therefore carries the dequantized values to about 22 significant bits and the
// products accumulate in fp32.  The CTA writes a normalised partial (o, lse) per row; a
// second grid merges the splits.  With EXACT false (kvattn_prefill_chunk_f16) every operand is
// rounded once to f16 instead, and QK and PV take one MMA pass each.
#include "decode.cuh"
#include "tcgen05.cuh"

namespace kvattn {

struct PrefillParams {
  const uint8_t* k_pool;
  const uint8_t* v_pool;
  int64_t k_stride, v_stride, n_pages;
  const uint16_t* q;  // bf16 bits [n_q][H_q][256]
  const int32_t* q_pos;
  const int32_t* page_list;
  const int32_t* page_logical;
  const int32_t* n_pages_arr;
  float* out;
  float* lse;
  float* part_o;    // [H_kv][n_ks][rows_pad][256]
  float* part_lse;  // [H_kv][n_ks][rows_pad]  (log2 units)
  int n_q, group, n_qh, max_pages, pages_per_split, n_ks, rows_pad;
};

namespace pf {
constexpr int kRows = 128;
constexpr int kKeys = 64;
constexpr int kHalfKeys = kKeys / 2;  // keys of a tile whose K^ this CTA holds
constexpr int kSoftmaxWarps = 4;      // warps 0-3: TMEM lane quarters 0-3
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr int kDequantWarps = 8;  // warps 6-13
constexpr int kThreads = (kSoftmaxWarps + 2 + kDequantWarps) * 32;
constexpr int kDq0 = (kSoftmaxWarps + 2) * 32;  // first dequant thread
// raw bytes a CTA copies per 64-key tile: K codes (Q5_1: low nibbles, then fifth bits),
// scales (Q5_1: then minima) of its 32 keys (each region contiguous in the page), V codes of
// its 128 head dimensions for all 64 keys (four 1 KB pieces, one per 16-key group), and all
// V scales of the tile; the stage holds them in that order
template <int KF, int VF>
struct Raw {
  static constexpr bool kK5 = KF == kKeyQ51 || KF == kKeyQ50;
  static constexpr int kKc = KF == kKeyQ8 ? 8192 : 4096;  // 32 keys x 256 or 128 bytes
  static constexpr int kKh = kK5 ? 1024 : 0;              // fifth bits: 32 keys x 32 bytes
  static constexpr int kKs = 512, kVs = 1024;
  static constexpr int kKm = KF == kKeyQ51 ? 512 : 0;     // key minima
  static constexpr int kVc = VF == kValQ8 ? 8192 : 4096;  // 128 dimensions x 64 keys, 8 or 4 bits
  static constexpr int kVm = VF == kValQ41 ? 1024 : 0;    // value minima (Q4_1), as the scales
  static constexpr int kKhOff = kKc, kKsOff = kKhOff + kKh, kKmOff = kKsOff + kKs;
  static constexpr int kVcOff = kKmOff + kKm, kVsOff = kVcOff + kVc, kVmOff = kVsOff + kVs;
  static constexpr int kBytes = kVmOff + kVm;
  // the regions' offsets in a page
  static constexpr int kPageScaleOff = KF == kKeyQ8 ? kKScaleOffset : KF == kKeyQ4 ? kK4ScaleOffset : kK5ScaleOffset;
  static constexpr int kPageVScaleOff = VF == kValQ8 ? kV8ScaleOffset : kV4ScaleOffset;
};
constexpr int kRawStages = 2;
constexpr int kPart = 16384;      // one of K^_hi, K^_lo (4 atoms x [32 keys][128 B]), V^T_hi, V^T_lo ([128][128 B])
constexpr int kSet = 2 * kPart;   // hi + lo
// a CTA walks at most this many 64-key tiles (the host plan keeps pages per CTA <= 256)
constexpr int kMaxTiles = 512;
// Shared memory map (bytes) of a format pair.  Three K^ / V^T buffer sets let the dequant run
// up to two tiles ahead of the MMAs; Q8_0 values double the raw bytes of a tile, and two sets
// then fit.
template <int KF, int VF>
struct Layout {
  static constexpr int kBufs = VF == kValQ8 ? 2 : 3;
  static constexpr int kRawStageBytes = Raw<KF, VF>::kBytes;
  static constexpr int kKOff = 0;                                  // kBufs x (K^_hi, K^_lo)
  static constexpr int kVOff = kKOff + kBufs * kSet;               // kBufs x (V^T_hi, V^T_lo)
  static constexpr int kRawOff = kVOff + kBufs * kSet;             // kRawStages stages of raw tile bytes
  static constexpr int kTileOff = kRawOff + kRawStages * kRawStageBytes;  // int2 [kMaxTiles]: page, 2*logical+half
  static constexpr int kMiscOff = kTileOff + 8 * kMaxTiles;
  static constexpr int kSmemBytes = kMiscOff + 512;
  static_assert(kRawStageBytes % 16 == 0 && kSmemBytes <= 227 * 1024, "shared memory");
};
// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol0 = 0;    // S buffers [0,64), [64,128); P_hi over the first 32, P_lo over the next 32
constexpr uint32_t kOCol0 = 128;  // O [row][256 dims]: [128, 384)
constexpr uint32_t kQCol0 = 384;  // Q / 16 [row][256 dims] as f16 pairs: [384, 512)
constexpr uint32_t kIdescQK = tc::idesc_f16(2 * kRows, kKeys, 0, 0);
constexpr uint32_t kIdescPV = tc::idesc_f16(2 * kRows, 256, 0, 0);
constexpr float kLog2e = 1.4426950408889634f;
}  // namespace pf

// ---- the CTA pair (a cluster of two): shared-memory addresses in the peer, barrier
// arrivals, cluster-scope waits ----
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of this CTA's shared-memory address `a` in CTA `rank`.
__device__ __forceinline__ uint32_t map_shared(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128u(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// Named barrier over `n` threads that also ANDs a flag over them.
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
// Arrives on the barrier at shared::cluster address `addr` (this CTA's or the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// mbar_wait for barriers that the peer CTA (or a multicast commit) also arrives on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity, 0u)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait_cluster(bar, parity, 1000000u)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      record_error(KVATTN_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// The CTA's i-th candidate tile (2 per listed page): 1 if it holds a key that some row of
// the M-tile pair may see (*page, *lh = 2 * logical block + half), 0 if not, -1 if its page
// id is out of range.
__device__ __forceinline__ int pf_candidate(const PrefillParams& p, int h, int ks, int i, int np, int max_qpos,
                                            int* page_out, int* lh_out) {
  const int idx = ks * p.pages_per_split + (i >> 1);
  if (idx >= np) return 0;
  const long long li = static_cast<long long>(h) * p.max_pages + idx;
  const int page = p.page_list[li];
  const int logical = p.page_logical ? p.page_logical[li] : idx;
  const int half = i & 1;
  if (static_cast<long long>(logical) * kPageTokens + half * pf::kKeys > max_qpos) return 0;
  if (page < 0 || page >= p.n_pages) return -1;
  *page_out = page;
  *lh_out = 2 * logical + half;
  return 1;
}

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
  return row * 128 + ((chunk ^ (row & 7)) << 4);
}

// Tensor-memory address of this warp's lane quarter.
__device__ __forceinline__ uint32_t tmem_lane(uint32_t tmem, int warp) {
  return tmem + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
}

// Softmax pieces for one 64-key tile of S: this thread's row, loaded from tensor memory as
// two 32-column halves.  Independent partial maxima and sums keep dependency chains short;
// packed f32x2 arithmetic halves the instruction count.
__device__ __forceinline__ void pf_mask32(uint32_t (&v)[32], int lim, int c0) {
#pragma unroll
  for (int c = 0; c < 32; ++c)
    if (c0 + c > lim) v[c] = 0xFF800000u;  // -inf: the key is in this row's future
}

__device__ __forceinline__ float pf_max32(const uint32_t (&v)[32]) {
  float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < 32; ++c) m[c & 3] = fmaxf(m[c & 3], __uint_as_float(v[c]));
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

__device__ __forceinline__ uint64_t f32x2_pack(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

// P = exp2(S log2(e) - mu) for 32 columns, as 16 f16 pairs of high parts (wh) and, with LO, 16
// of low parts (wl: the rounded remainder); returns the sum of the 32 fp32 values of P.
template <bool LO>
__device__ __forceinline__ float pf_p32(const uint32_t (&v)[32], float mu, uint32_t (&wh)[16], uint32_t (&wl)[16]) {
  const uint64_t l2 = f32x2_pack(__float_as_uint(pf::kLog2e), __float_as_uint(pf::kLog2e));
  const uint64_t nm = f32x2_pack(__float_as_uint(-mu), __float_as_uint(-mu));
  uint64_t acc[2] = {0ull, 0ull};  // two f32x2 partial sums (0.0f bit patterns)
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    uint64_t x = f32x2_pack(v[2 * c], v[2 * c + 1]);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(x) : "l"(x), "l"(l2), "l"(nm));
    uint32_t d0, d1;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(d0), "=r"(d1) : "l"(x));
    const float p0 = fast_exp2(__uint_as_float(d0)), p1 = fast_exp2(__uint_as_float(d1));
    const uint64_t pp = f32x2_pack(__float_as_uint(p0), __float_as_uint(p1));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(acc[c & 1]) : "l"(acc[c & 1]), "l"(pp));
    wh[c] = pack_half2(p0, p1);
    if constexpr (LO) wl[c] = pack_half2(p0 - half_lo(wh[c]), p1 - half_hi(wh[c]));
  }
  uint64_t t;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(acc[0]), "l"(acc[1]));
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(t));
  return __uint_as_float(a) + __uint_as_float(b);
}

// f16 pair of a dequantized value as an exact high + low split: hi = f16(c * d) and
// lo = c * d - hi (exact in f16: c has at most 8 significant bits, d 11).
__device__ __forceinline__ void split_product(uint32_t code, uint32_t d, uint32_t& hi, uint32_t& lo) {
  hi = hmul2(code, d);
  lo = hfma2(code, d, hi ^ 0x80008000u);
}

// The same split of an affine dequantization q * d + m (Q5_1 keys): q * d is exact in fp32
// (q has at most 5 significant bits, d 11) and the sum is rounded once to fp32; hi = f16 of
// it and lo = f16 of the exact fp32 remainder carry it to about 22 significant bits.
__device__ __forceinline__ void split_affine(uint32_t code, float d, float m, uint32_t& hi, uint32_t& lo) {
  const float v0 = fmaf(half_lo(code), d, m), v1 = fmaf(half_hi(code), d, m);
  hi = pack_half2(v0, v1);
  lo = pack_half2(v0 - half_lo(hi), v1 - half_hi(hi));
}

// split_affine for a pair of values with a scale and a minimum each (Q4_1 values: the two halves
// belong to two tokens): hi = f16(q * d + m), lo = f16 of the exact fp32 remainder.
__device__ __forceinline__ void split_affine2(uint32_t code, uint32_t d, uint32_t m, uint32_t& hi, uint32_t& lo) {
  const float v0 = fmaf(half_lo(code), half_lo(d), half_lo(m)), v1 = fmaf(half_hi(code), half_hi(d), half_hi(m));
  hi = pack_half2(v0, v1);
  lo = pack_half2(v0 - half_lo(hi), v1 - half_hi(hi));
}

// x shifted left by s bits (right by -s when s < 0); s is a compile-time constant after unrolling.
__device__ __forceinline__ uint32_t shl(uint32_t x, int s) { return s >= 0 ? x << s : x >> -s; }

// EXACT: every operand as an f16 high part plus a low part (about 22 significant bits, QK as
// two MMA passes, PV as three); otherwise each dequantized value and each P rounded once to
// f16 (one pass each; the dequant writes, and the MMAs read, the high parts only).
template <int KF, int VF, bool EXACT>
__global__ void __launch_bounds__(pf::kThreads, 1) prefill_kernel(const PrefillParams p) {
  using RawF = pf::Raw<KF, VF>;
  using L = pf::Layout<KF, VF>;
  constexpr bool kV41 = VF == kValQ41, kV8 = VF == kValQ8;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kMiscOff);
  uint64_t* rawfull = bars + 0;    // [2] producer (tx bytes) -> dequant
  uint64_t* rawempty = bars + 2;   // [2] dequant -> producer
  uint64_t* kready = bars + 4;     // [3] even CTA: K^ halves of both CTAs in place -> MMA
  uint64_t* vready = bars + 7;     // [3] even CTA: V^T halves in place -> MMA
  uint64_t* kfree = bars + 10;     // [3] QK done (pair commit) -> dequant
  uint64_t* vfree = bars + 13;     // [3] PV done (pair commit) -> dequant
  uint64_t* vdone = bars + 16;     // one phase per PV (pair commit) -> softmax (rescale of O)
  uint64_t* sready = bars + 17;    // [2] QK done (pair commit) -> softmax
  uint64_t* pready = bars + 19;    // [2] even CTA: P of both CTAs written -> MMA
  uint64_t* ofinal = bars + 21;    // every MMA done (pair commit) -> epilogue, tensor-memory release
  uint64_t* qready = bars + 22;    // even CTA: Q of both CTAs in tensor memory -> MMA
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(bars + 23);
  int* s_abort = reinterpret_cast<int*>(tmem_base_s + 1);
  int* s_ntiles = s_abort + 1;
  const int2* tiles = reinterpret_cast<const int2*>(smem + L::kTileOff);

  const int mt = blockIdx.x, ks = blockIdx.y, h = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rows = p.n_q * p.group;
  const int row0 = mt * pf::kRows;
  int np = p.max_pages;
  if (p.n_pages_arr) np = min(max(p.n_pages_arr[h], 0), p.max_pages);
  // largest query position among the rows of the M-tile pair: keys beyond it are never
  // visible (the two CTAs walk the same tiles)
  int max_qpos = INT_MIN;
  {
    const int pair_row0 = (mt & ~1) * pf::kRows;
    const int t0 = pair_row0 / p.group, t1 = min(n_rows - 1, pair_row0 + 2 * pf::kRows - 1) / p.group;
    for (int t = t0; t <= t1; ++t) max_qpos = max(max_qpos, p.q_pos[t]);
  }
  const uint32_t crank = cluster_rank();
  const bool leader = crank == 0;

  if (threadIdx.x == 0) {
    for (int b = 0; b < pf::kRawStages; ++b) {
      mbar_init(&rawfull[b], 1);
      mbar_init(&rawempty[b], pf::kDequantWarps);
    }
    for (int b = 0; b < L::kBufs; ++b) {
      mbar_init(&kready[b], 2);  // one arrival from the dequant warps of each CTA
      mbar_init(&vready[b], 2);
      mbar_init(&kfree[b], 1);
      mbar_init(&vfree[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sready[b], 1);
      mbar_init(&pready[b], 2 * pf::kSoftmaxWarps);
    }
    mbar_init(vdone, 1);
    mbar_init(ofinal, 1);
    mbar_init(qready, 2 * pf::kSoftmaxWarps);
    *s_abort = 0;
    if (smem_u32(smem) & 1023) record_error(KVATTN_ERR_INVALID_ARG);
    fence_barrier_init();
  }
  if (warp == 0) {
    // the CTA's tiles in key order, compacted once: (page, 2 * logical block + half)
    int2* list = reinterpret_cast<int2*>(smem + L::kTileOff);
    int n_cand = 2 * p.pages_per_split;
    if (n_cand > pf::kMaxTiles) {
      if (lane == 0) record_error(KVATTN_ERR_INVALID_ARG);
      n_cand = 0;
    }
    int cnt = 0;
    for (int i0 = 0; i0 < n_cand; i0 += 32) {
      int page = 0, lh = 0;
      const int c = i0 + lane < n_cand ? pf_candidate(p, h, ks, i0 + lane, np, max_qpos, &page, &lh) : 0;
      if (c < 0) record_error(KVATTN_ERR_BAD_PAGE);
      const unsigned m = __ballot_sync(0xffffffffu, c > 0);
      if (c > 0) list[cnt + __popc(m & ((1u << lane) - 1u))] = make_int2(page, lh);
      cnt += __popc(m);
    }
    if (lane == 0) *s_ntiles = cnt;
  }
  if (warp == pf::kMmaWarp) {
    tc::tmem_alloc_pair(tmem_base_s, pf::kTmemCols);
    tc::tmem_relinquish_pair();
  }
  tc::fence_before_sync();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_base_s;
  const int n_tiles = *s_ntiles;

  if (warp == pf::kLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int2 tl = tiles[j];
        const int r = j % pf::kRawStages;
        if (j >= pf::kRawStages && !mbar_wait(&rawempty[r], ((j / pf::kRawStages) - 1) & 1)) {
          *s_abort = 1;
          break;
        }
        // K: this CTA's 32 keys of the tile (quarter q of the page); V: its 128 dimensions
        const int half = tl.y & 1, q = 2 * half + static_cast<int>(crank);
        uint8_t* st = smem + L::kRawOff + r * L::kRawStageBytes;
        const uint8_t* kp = p.k_pool + static_cast<int64_t>(tl.x) * p.k_stride;
        const uint8_t* vp = p.v_pool + static_cast<int64_t>(tl.x) * p.v_stride;
        mbar_arrive_expect_tx(&rawfull[r], RawF::kBytes);
        bulk_g2s(st, kp + q * RawF::kKc, RawF::kKc, &rawfull[r]);
        if constexpr (RawF::kKh > 0)
          bulk_g2s(st + RawF::kKhOff, kp + kK5HighOffset + q * RawF::kKh, RawF::kKh, &rawfull[r]);
        bulk_g2s(st + RawF::kKsOff, kp + RawF::kPageScaleOff + q * RawF::kKs, RawF::kKs, &rawfull[r]);
        if constexpr (RawF::kKm > 0)
          bulk_g2s(st + RawF::kKmOff, kp + kK5MinOffset + q * RawF::kKm, RawF::kKm, &rawfull[r]);
        // V codes: per 16-key group g of the tile half, this CTA's half of the group's bytes (the
        // 1 KB of its two block pairs in Q4 pages, the 2 KB of its four blocks in Q8_0 pages)
        constexpr int kVPiece = RawF::kVc / 4, kVGroup = 2 * kVPiece;
        for (int g = 0; g < 4; ++g)
          bulk_g2s(st + RawF::kVcOff + g * kVPiece, vp + (4 * half + g) * kVGroup + crank * kVPiece, kVPiece,
                   &rawfull[r]);
        bulk_g2s(st + RawF::kVsOff, vp + RawF::kPageVScaleOff + half * RawF::kVs, RawF::kVs, &rawfull[r]);
        if constexpr (RawF::kVm > 0)
          bulk_g2s(st + RawF::kVmOff, vp + kV41MinOffset + half * RawF::kVm, RawF::kVm, &rawfull[r]);
      }
      // every copy issued must land before the CTA may exit
      for (int jj = j - pf::kRawStages < 0 ? 0 : j - pf::kRawStages; jj < j; ++jj)
        mbar_wait(&rawfull[jj % pf::kRawStages], (jj / pf::kRawStages) & 1);
    }
  } else if (warp == pf::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    // The whole warp runs this loop (one elected lane issues each instruction); barrier
    // checks are made warp-uniform so the lanes never diverge around elect.sync.  Each pass
    // issues whichever is ready of QK of the next tile (once both CTAs' K^ halves are in
    // place and the S buffer it overwrites was consumed by PV two tiles back) and PV of the
    // oldest tile whose P is written in both CTAs.
    if (leader) {
      const uint32_t k_base = smem_u32(smem + L::kKOff);
      const uint32_t v_base = smem_u32(smem + L::kVOff);
      auto ready_all = [&](uint64_t* bar, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_try_wait_cluster(bar, par, 0u));
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(qready, 0));
      int jq = 0, jp = 0;  // next QK, next PV
      unsigned long long t_idle = 0;
      while (ok && jp < n_tiles) {
        bool did = false;
        if (jq < n_tiles && jq <= jp + 1 && ready_all(&kready[jq % L::kBufs], (jq / L::kBufs) & 1)) {
          const int b = jq % L::kBufs, s2 = jq & 1;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk) {
            const uint32_t ka = k_base + b * pf::kSet + (kk >> 2) * 4096 + (kk & 3) * 32;
            const uint32_t dcol = tmem + pf::kSCol0 + s2 * pf::kKeys, qcol = tmem + pf::kQCol0 + kk * 8;
            tc::mma_f16_ts_pair_warp(dcol, qcol, tc::sw128_desc(ka, 1024, 16), pf::kIdescQK, kk > 0 ? 1u : 0u);
            if constexpr (EXACT)
              tc::mma_f16_ts_pair_warp(dcol, qcol, tc::sw128_desc(ka + pf::kPart, 1024, 16), pf::kIdescQK, 1u);
          }
          tc::commit_pair2_warp(&sready[s2]);
          tc::commit_pair2_warp(&kfree[b]);
          ++jq;
          did = true;
        } else if (jp < jq && ready_all(&pready[jp & 1], (jp >> 1) & 1) &&
                   ready_all(&vready[jp % L::kBufs], (jp / L::kBufs) & 1)) {
          const int b = jp % L::kBufs, s2 = jp & 1;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < pf::kKeys / 16; ++kk) {
            const uint32_t va = v_base + b * pf::kSet + kk * 32;
            const uint32_t ph = tmem + pf::kSCol0 + s2 * pf::kKeys + kk * 8, pl = ph + pf::kKeys / 2;
            const uint64_t vh = tc::sw128_desc(va, 1024, 16), vl = tc::sw128_desc(va + pf::kPart, 1024, 16);
            tc::mma_f16_ts_pair_warp(tmem + pf::kOCol0, ph, vh, pf::kIdescPV, (jp > 0 || kk > 0) ? 1u : 0u);
            if constexpr (EXACT) {
              tc::mma_f16_ts_pair_warp(tmem + pf::kOCol0, pl, vh, pf::kIdescPV, 1u);
              tc::mma_f16_ts_pair_warp(tmem + pf::kOCol0, ph, vl, pf::kIdescPV, 1u);
            }
          }
          tc::commit_pair2_warp(vdone);
          tc::commit_pair2_warp(&vfree[b]);
          ++jp;
          did = true;
        }
        if (did) {
          t_idle = 0;
        } else {
          const unsigned long long now = global_timer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > kWaitTimeoutNs) {
            if (lane == 0) record_error(KVATTN_ERR_TIMEOUT);
            ok = false;
          }
          __nanosleep(32);
        }
        ok = __all_sync(0xffffffffu, ok);
      }
      if (!ok && lane == 0) *s_abort = 1;
      tc::commit_pair2_warp(ofinal);  // arrives in both CTAs when every MMA above has completed
    }
    // no MMA may still write this CTA's tensor memory when it is freed
    __all_sync(0xffffffffu, mbar_wait_cluster(ofinal, 0));
  } else if (warp < pf::kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax (thread = row)
    const int r = threadIdx.x;  // 0..127 == TMEM lane
    const int R = row0 + r;
    const int qpos = R < n_rows ? p.q_pos[R / p.group] : INT_MAX;
    const uint32_t lane_base = tmem_lane(tmem, warp);
    const uint32_t qready_lead = map_shared(smem_u32(qready), 0);
    const uint32_t pready_lead = map_shared(smem_u32(&pready[0]), 0);
    // ---- Q row: bf16 -> f16 of q / 16 (exact) into tensor memory (A operand of S = Q K^T) ----
    {
      const uint16_t* src = nullptr;
      if (R < n_rows) {
        const int t = R / p.group, jq = R % p.group;
        src = p.q + (static_cast<long long>(t) * p.n_qh + h * p.group + jq) * kHeadDim;
      }
      for (int c0 = 0; c0 < 4; ++c0) {  // 64 channels = 32 columns at a time
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 raw = make_uint4(0u, 0u, 0u, 0u);
          if (src) raw = *reinterpret_cast<const uint4*>(src + c0 * 64 + c * 8);
          const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[c * 4 + e] =
                pack_half2(__uint_as_float(in[e] << 16) * 0.0625f, __uint_as_float(in[e] & 0xFFFF0000u) * 0.0625f);
        }
        tc::st32(lane_base + pf::kQCol0 + c0 * 32, w);
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(qready_lead);
    }
    float m_ref = -INFINITY, l_sum = 0.f;  // base-2 units
    int j = 0;
    bool ok = true;
    for (; j < n_tiles && ok; ++j) {
      const int2 tl = tiles[j];
      const int b = j & 1;
      if (!mbar_wait_cluster(&sready[b], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      // the 64 scores in one tensor-memory round trip; P overwrites them
      const int lim = qpos - tl.y * pf::kKeys;  // columns beyond lim are in this row's future
      const uint32_t scol = lane_base + pf::kSCol0 + b * pf::kKeys;
      uint32_t v0[32], v1[32];
      tc::ld32(scol, v0);
      tc::ld32(scol + 32, v1);
      tc::wait_ld();
      if (__any_sync(0xffffffffu, lim < pf::kKeys - 1)) {  // warp-uniform: only diagonal tiles
        pf_mask32(v0, lim, 0);
        pf_mask32(v1, lim, 32);
      }
      const float mx = fmaxf(pf_max32(v0), pf_max32(v1)) * pf::kLog2e;
      float alpha = 1.f;
      bool resc = false;
      if (mx > m_ref + 8.f) {
        alpha = fast_exp2(m_ref - mx);  // 0 when m_ref = -inf
        resc = j > 0 && m_ref != -INFINITY;
        l_sum *= alpha;
        m_ref = mx;
      }
      const float mu = m_ref == -INFINITY ? 0.f : m_ref;
      {
        uint32_t wh[16], wl[16];
        l_sum += pf_p32<EXACT>(v0, mu, wh, wl);
        tc::st16(scol, wh);
        if constexpr (EXACT) tc::st16(scol + 32, wl);
        l_sum += pf_p32<EXACT>(v1, mu, wh, wl);
        tc::st16(scol + 16, wh);
        if constexpr (EXACT) tc::st16(scol + 48, wl);
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O is rescaled to the new maximum before PV of this tile accumulates into it; this
        // warp's rows of O hold the previous tile's PV only once that completed
        if (!mbar_wait_cluster(vdone, (j - 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const float f = resc ? alpha : 1.f;
        for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
          uint32_t v[32];
          tc::ld32(lane_base + pf::kOCol0 + c0, v);
          tc::wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * f);
          tc::st32(lane_base + pf::kOCol0 + c0, v);
        }
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(pready_lead + 8 * b);
    }
    // ---- epilogue: normalised partial (o, lse) of this row ----
    bool have = false;
    if (ok && j > 0) {
      have = mbar_wait_cluster(ofinal, 0);
      ok = have;
    }
    if (!ok) *s_abort = 1;
    tc::fence_after_sync();
    const bool direct = p.n_ks == 1;
    float* dst = nullptr;
    if (R < n_rows) {
      if (direct) {
        const int t = R / p.group, jq = R % p.group;
        dst = p.out + (static_cast<long long>(t) * p.n_qh + h * p.group + jq) * kHeadDim;
      } else {
        dst = p.part_o + ((static_cast<long long>(h) * p.n_ks + ks) * p.rows_pad + R) * kHeadDim;
      }
    }
    const float inv = (have && l_sum > 0.f) ? 1.f / l_sum : 0.f;
    const bool warp_have = __any_sync(0xffffffffu, have);
    for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
      uint32_t v[32];
      if (warp_have) {  // the load is warp-collective
        tc::ld32(lane_base + pf::kOCol0 + c0, v);
        tc::wait_ld();
      }
      if (!have) {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      if (dst) {
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(dst + c0 + c) =
              make_float4(__uint_as_float(v[c]) * inv, __uint_as_float(v[c + 1]) * inv,
                          __uint_as_float(v[c + 2]) * inv, __uint_as_float(v[c + 3]) * inv);
      }
    }
    if (R < n_rows) {
      const float l2 = (have && l_sum > 0.f) ? m_ref + log2f(l_sum) : -INFINITY;
      if (direct) {
        const int t = R / p.group, jq = R % p.group;
        p.lse[static_cast<long long>(t) * p.n_qh + h * p.group + jq] = l2 * 0.69314718055994531f;
      } else {
        p.part_lse[(static_cast<long long>(h) * p.n_ks + ks) * p.rows_pad + R] = l2;
      }
    }
  } else if (warp >= pf::kDq0 / 32) {
    // ------------------------------------------------------------ dequant (256 threads)
    // This CTA dequantizes its half of every tile (K^: its 32 keys; V^T: its 128 dimensions)
    // into its own buffers, as exact high + low f16 parts, then one thread tells the even CTA.
    const int d = threadIdx.x - pf::kDq0;
    // K task: key kl of this CTA's 32, channel quarter kP (blocks 2kP, 2kP+1), raw chunks
    // 2cp and 2cp+1 of the four; 8 consecutive threads take 8 consecutive keys, so their
    // swizzled 16-byte stores hit 8 different bank groups.
    const int kl = d & 31, kP = (d >> 5) & 3, cp = d >> 7;
    const int kGl = kl >> 4, kH = (kl >> 3) & 1, kR = kl & 7;
    // V task: channel row vR (channels vR + 8k of block 2vC + ve, vC = 2 * rank + vCl), key
    // half vh of token group vG (16 keys)
    const int vR = d & 7, vh = (d >> 3) & 1, vCl = (d >> 4) & 1, vG = (d >> 5) & 3, ve = d >> 7;
    const int vC = 2 * static_cast<int>(crank) + vCl;
    // Q8_0 V task: channel row vR8 (channels vR8 + 8k of this CTA's block vb8), key half vh8 of
    // token group vG8: the byte pairs of tokens 2T, 2T + 1 (T = 0..3) sit in words vh8 and
    // vh8 + 2 of raw chunk T of (vG8, vb8, vR8)
    const int vR8 = d & 7, vh8 = (d >> 3) & 1, vb8 = (d >> 4) & 3, vG8 = (d >> 6) & 3;
    // 16-byte chunks are read in an order rotated by (row / 2): 8 threads at a 64-byte
    // stride then touch 8 different bank groups
    const int rotK = kR >> 1, rotV = vR >> 1;
    const uint32_t own = smem_u32(smem);
    const uint32_t kready_lead = map_shared(smem_u32(&kready[0]), 0);
    const uint32_t vready_lead = map_shared(smem_u32(&vready[0]), 0);
    int j = 0;
    bool ok = true;
    for (; j < n_tiles && ok; ++j) {
      const int b = j % L::kBufs, r = j % pf::kRawStages;
      // every wait result is combined over the 256 dequant threads at the named barriers, so
      // all of them stop at the same tile when one gives up
      bool wok = mbar_wait(&rawfull[r], (j / pf::kRawStages) & 1);
      const uint32_t stu = own + L::kRawOff + r * L::kRawStageBytes;
      // ---------------- raw K, V -> registers; the stage is then released ----------------
      uint32_t kw[2][4] = {};  // per chunk i: the 4 words (8 codes of block 2kP, 8 of 2kP + 1)
      uint32_t kh[2] = {};     // Q5_1: per chunk i, the fifth bits of blocks 2kP, 2kP + 1 at bits 0-7, 16-23
      uint32_t dkw = 0, mkw = 0;
      uint2 vraw[4] = {}, dvr[4] = {}, mvr[4] = {};
      uint32_t v8w[4][2] = {}, d8[4] = {};  // Q8_0 values: per token pair T, words vh8, vh8 + 2; scales
      if (wok) {
        if constexpr (KF != kKeyQ8) {
          // 4-bit key words (Q5_1: the low nibbles) of token kl, blocks 2kP, 2kP + 1 (c = 2kP % 4,
          // 2kP % 4 + 1) of block quad Q = kP / 2, lane column T: one 8-byte load per chunk.
          // Q5_1: the word of fifth bits of (token, Q, T) holds block c at bits 4c + (0..3) of
          // each half; shifting it right by 4 * (2kP % 4) brings blocks 2kP, 2kP + 1 to bits 0-7.
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int T = (2 * cp + i + rotK) & 3;
            const int row = (((kGl * 2 + (kP >> 1)) * 2 + kH) * 8 + kR) * 4 + T;
            const uint2 w2 = lds64(stu + 4 * (row * 4 + ((2 * kP) & 3)));
            kw[i][0] = w2.x;
            kw[i][1] = w2.y;
            if constexpr (RawF::kK5) kh[i] = lds32(stu + RawF::kKhOff + 4 * row) >> (4 * ((2 * kP) & 3));
          }
        } else {
          const uint32_t kbase = stu + ((((kGl * 4 + kP) * 2 + kH) * 8 + kR) * 4) * 16;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint4 c = lds128(kbase + (((2 * cp + i + rotK) & 3) << 4));
            kw[i][0] = c.x; kw[i][1] = c.y; kw[i][2] = c.z; kw[i][3] = c.w;
          }
        }
        // scales (Q5_1: and minima) of blocks 2kP, 2kP + 1 of token kl
        const int sidx = ((kGl * 8 + kR) * 2 + kH) * 16 + 4 * kP;
        dkw = lds32(stu + RawF::kKsOff + sidx);
        if constexpr (KF == kKeyQ51) mkw = lds32(stu + RawF::kKmOff + sidx);
        // this thread's two words (block 2vC + ve, both key halves) of each raw chunk and of
        // the scales of each token pair
        if constexpr (kV8) {
          const uint32_t v8base = stu + RawF::kVcOff + vG8 * 2048 + ((vb8 * 8 + vR8) * 4) * 16;
#pragma unroll
          for (int T = 0; T < 4; ++T) {
            v8w[T][0] = lds32(v8base + T * 16 + 4 * vh8);
            v8w[T][1] = lds32(v8base + T * 16 + 4 * (vh8 + 2));
            d8[T] = lds32(stu + RawF::kVsOff + ((vG8 * 4 + T) * 8 + 4 * static_cast<int>(crank) + vb8) * 8 + 4 * vh8);
          }
        } else {
          const uint32_t vbase = stu + RawF::kVcOff + vG * 1024 + ((vCl * 8 + vR) * 4) * 16 + 8 * ve;
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) vraw[ii] = lds64(vbase + (((ii + rotV) & 3) << 4));
#pragma unroll
          for (int T = 0; T < 4; ++T) dvr[T] = lds64(stu + RawF::kVsOff + ((vG * 4 + T) * 8 + 2 * vC) * 8 + 8 * ve);
          if constexpr (RawF::kVm > 0) {
#pragma unroll
            for (int T = 0; T < 4; ++T)
              mvr[T] = lds64(stu + RawF::kVmOff + ((vG * 4 + T) * 8 + 2 * vC) * 8 + 8 * ve);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rawempty[r]);
      // ---------------- K^ (this CTA's buffer is free once QK(j - 3) completed) ----
      if (wok && j >= L::kBufs) wok = mbar_wait_cluster(&kfree[b], ((j / L::kBufs) - 1) & 1);
      const uint32_t katom = own + L::kKOff + b * pf::kSet + kP * 4096;
      if (wok) {
        const uint32_t dlo = prmt(dkw, 0u, 0x1010u), dhi = prmt(dkw, 0u, 0x3232u);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int T = (2 * cp + i + rotK) & 3;
          uint32_t c[8];  // exact codes as f16 pairs: c[0..3] block 2kP, c[4..7] block 2kP + 1
          if constexpr (KF == kKeyQ4) {
            // channel i' of a word at bit 4(i'/2) + 16(i'%2): pairs (0,1), (2,3), (4,5), (6,7)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint32_t w = kw[i][e], ws = w >> 8;
              c[4 * e + 0] = hsub2(and_or(w, 0x000F000Fu, 0x64006400u), 0x64086408u);
              c[4 * e + 1] = hfma2(and_or(w, 0x00F000F0u, 0x64006400u), 0x2C002C00u, 0xD480D480u);
              c[4 * e + 2] = hsub2(and_or(ws, 0x000F000Fu, 0x64006400u), 0x64086408u);
              c[4 * e + 3] = hfma2(and_or(ws, 0x00F000F0u, 0x64006400u), 0x2C002C00u, 0xD480D480u);
            }
          } else if constexpr (RawF::kK5) {
            // as Q4_0, with the fifth bit (channel (e, i) at bit 4e + i / 2 + 16 (i % 2) of kh)
            // moved to the 16s place of the code: bit 4 of the halves 1024 + q, bit 8 of the
            // halves 1024 + 16q; the codes q in [0, 31] (Q5_1) or q - 16 (Q5_0) are exact in f16
            constexpr uint32_t kSubLo = KF == kKeyQ50 ? 0x64106410u : 0x64006400u;  // 1024 (+ 16)
            constexpr uint32_t kAddHi = KF == kKeyQ50 ? 0xD500D500u : 0xD400D400u;  // -64 (- 16)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint32_t w = kw[i][e], ws = w >> 8, x = kh[i];
              c[4 * e + 0] = hsub2(or_and(and_or(w, 0x000F000Fu, 0x64006400u), shl(x, 4 - 4 * e), 0x00100010u),
                                   kSubLo);
              c[4 * e + 1] = hfma2(or_and(and_or(w, 0x00F000F0u, 0x64006400u), shl(x, 7 - 4 * e), 0x01000100u),
                                   0x2C002C00u, kAddHi);
              c[4 * e + 2] = hsub2(or_and(and_or(ws, 0x000F000Fu, 0x64006400u), shl(x, 2 - 4 * e), 0x00100010u),
                                   kSubLo);
              c[4 * e + 3] = hfma2(or_and(and_or(ws, 0x00F000F0u, 0x64006400u), shl(x, 5 - 4 * e), 0x01000100u),
                                   0x2C002C00u, kAddHi);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t w = kw[i][e];  // offset-binary code bytes: 1024 + (q + 128) - 1152 = q
              c[2 * e] = hsub2(prmt(w, 0x64646464u, 0x4140u), 0x64806480u);
              c[2 * e + 1] = hsub2(prmt(w, 0x64646464u, 0x4342u), 0x64806480u);
            }
          }
          uint32_t oh[8], ol[8];
          if constexpr (KF == kKeyQ51 && EXACT) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              split_affine(c[e], e < 4 ? half_lo(dkw) : half_hi(dkw), e < 4 ? half_lo(mkw) : half_hi(mkw), oh[e],
                           ol[e]);
          } else if constexpr (KF == kKeyQ51) {
            // q * d + m rounded once to f16 (one fused multiply-add)
            const uint32_t mlo = prmt(mkw, 0u, 0x1010u), mhi = prmt(mkw, 0u, 0x3232u);
#pragma unroll
            for (int e = 0; e < 8; ++e) oh[e] = hfma2(c[e], e < 4 ? dlo : dhi, e < 4 ? mlo : mhi);
          } else if constexpr (EXACT) {
#pragma unroll
            for (int e = 0; e < 8; ++e) split_product(c[e], e < 4 ? dlo : dhi, oh[e], ol[e]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) oh[e] = hmul2(c[e], e < 4 ? dlo : dhi);
          }
          sts128u(katom + swz(kl, T), oh[0], oh[1], oh[2], oh[3]);
          sts128u(katom + swz(kl, 4 + T), oh[4], oh[5], oh[6], oh[7]);
          if constexpr (EXACT) {
            sts128u(katom + pf::kPart + swz(kl, T), ol[0], ol[1], ol[2], ol[3]);
            sts128u(katom + pf::kPart + swz(kl, 4 + T), ol[4], ol[5], ol[6], ol[7]);
          }
        }
        tc::fence_proxy_async_smem();
      }
      if (!bar_and(1, 32 * pf::kDequantWarps, wok)) {
        ok = false;
        break;
      }
      if (d == 0) mbar_arrive_cluster(kready_lead + 8 * b);
      // ---------------- V^T: this CTA's 128 dimensions ----------------
      if (j >= L::kBufs) wok = mbar_wait_cluster(&vfree[b], ((j / L::kBufs) - 1) & 1);
      const uint32_t vt = own + L::kVOff + b * pf::kSet;
      if (wok) {
        if constexpr (kV8) {
          // Q8_0 values: offset-binary code bytes 2(k % 2), 2(k % 2) + 1 of word k / 2 are channel
          // vR8 + 8k of tokens 2T, 2T + 1 (1024 + (q + 128) - 1152 = q, exact in f16)
          uint32_t oh[4][4], ol[4][4];  // [k][T]
#pragma unroll
          for (int T = 0; T < 4; ++T) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t code =
                  hsub2(prmt(v8w[T][k >> 1], 0x64646464u, (k & 1) ? 0x4342u : 0x4140u), 0x64806480u);
              if constexpr (EXACT) {
                split_product(code, d8[T], oh[k][T], ol[k][T]);
              } else {
                oh[k][T] = hmul2(code, d8[T]);
              }
            }
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int row = 32 * vb8 + 8 * k + vR8;  // dimension - 128 * rank
            sts128u(vt + swz(row, 2 * vG8 + vh8), oh[k][0], oh[k][1], oh[k][2], oh[k][3]);
            if constexpr (EXACT)
              sts128u(vt + pf::kPart + swz(row, 2 * vG8 + vh8), ol[k][0], ol[k][1], ol[k][2], ol[k][3]);
          }
        } else {
          // chunk ii holds token pair (ii + rotV) & 3: two select stages undo the rotation so
          // that wv[T] is token pair T (an array indexed by the runtime rotation would be
          // placed in local memory)
          uint32_t wv[4], t[4];
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) wv[ii] = vh ? vraw[ii].y : vraw[ii].x;
#pragma unroll
          for (int x = 0; x < 4; ++x) t[x] = (rotV & 1) ? wv[(x + 3) & 3] : wv[x];
#pragma unroll
          for (int x = 0; x < 4; ++x) wv[x] = (rotV & 2) ? t[(x + 2) & 3] : t[x];
          uint32_t oh[4][4], ol[4][4];  // [k][T]
#pragma unroll
          for (int T = 0; T < 4; ++T) {
            const uint32_t W = wv[T];
            const uint32_t Ws = W >> 8;
            const uint32_t dv = vh ? dvr[T].y : dvr[T].x;
            // Q4_0: q - 8 (1024 + q - 1032, or (1024 + 16q) / 16 - 72); Q4_1: q
            constexpr uint32_t kVSubLo = kV41 ? 0x64006400u : 0x64086408u;
            constexpr uint32_t kVAddHi = kV41 ? 0xD400D400u : 0xD480D480u;
            const uint32_t v0 = hsub2(and_or(W, 0x000F000Fu, 0x64006400u), kVSubLo);
            const uint32_t v1 = hfma2(and_or(W, 0x00F000F0u, 0x64006400u), 0x2C002C00u, kVAddHi);
            const uint32_t v2 = hsub2(and_or(Ws, 0x000F000Fu, 0x64006400u), kVSubLo);
            const uint32_t v3 = hfma2(and_or(Ws, 0x00F000F0u, 0x64006400u), 0x2C002C00u, kVAddHi);
            if constexpr (kV41 && EXACT) {
              // q * d + m per token (each half of the pair has its own scale and minimum)
              const uint32_t mv = vh ? mvr[T].y : mvr[T].x;
              split_affine2(v0, dv, mv, oh[0][T], ol[0][T]);
              split_affine2(v1, dv, mv, oh[1][T], ol[1][T]);
              split_affine2(v2, dv, mv, oh[2][T], ol[2][T]);
              split_affine2(v3, dv, mv, oh[3][T], ol[3][T]);
            } else if constexpr (kV41) {
              const uint32_t mv = vh ? mvr[T].y : mvr[T].x;
              oh[0][T] = hfma2(v0, dv, mv);
              oh[1][T] = hfma2(v1, dv, mv);
              oh[2][T] = hfma2(v2, dv, mv);
              oh[3][T] = hfma2(v3, dv, mv);
            } else if constexpr (EXACT) {
              split_product(v0, dv, oh[0][T], ol[0][T]);
              split_product(v1, dv, oh[1][T], ol[1][T]);
              split_product(v2, dv, oh[2][T], ol[2][T]);
              split_product(v3, dv, oh[3][T], ol[3][T]);
            } else {
              oh[0][T] = hmul2(v0, dv);
              oh[1][T] = hmul2(v1, dv);
              oh[2][T] = hmul2(v2, dv);
              oh[3][T] = hmul2(v3, dv);
            }
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int row = 32 * (2 * vCl + ve) + 8 * k + vR;  // dimension - 128 * rank
            sts128u(vt + swz(row, 2 * vG + vh), oh[k][0], oh[k][1], oh[k][2], oh[k][3]);
            if constexpr (EXACT)
              sts128u(vt + pf::kPart + swz(row, 2 * vG + vh), ol[k][0], ol[k][1], ol[k][2], ol[k][3]);
          }
        }
        tc::fence_proxy_async_smem();
      }
      if (!bar_and(2, 32 * pf::kDequantWarps, wok)) {
        ok = false;
        break;
      }
      if (d == 0) mbar_arrive_cluster(vready_lead + 8 * b);
    }
    if (!ok) *s_abort = 1;
  }

  tc::fence_before_sync();
  __syncthreads();
  // the peer arrives on this CTA's barriers until it gets here
  cluster_sync();
  if (*s_abort && threadIdx.x == 0) record_error(KVATTN_ERR_TIMEOUT);
  if (warp == pf::kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, pf::kTmemCols);
  }
}

// The format pairs chunked prefill takes: Q8_0, Q4_0 and Q5_1 keys with Q4_0 or Q8_0 values,
// Q5_0 keys with Q4_1 values.
#define KVATTN_PREFILL_PAIRS(X)                                                                      \
  X(kKeyQ8, kValQ4) X(kKeyQ4, kValQ4) X(kKeyQ51, kValQ4) X(kKeyQ50, kValQ41) X(kKeyQ8, kValQ8) \
  X(kKeyQ4, kValQ8) X(kKeyQ51, kValQ8)

bool prefill_pair_supported(int key_fmt, int val_fmt) {
#define PF_PAIR_OK(KF, VF) if (key_fmt == KF && val_fmt == VF) return true;
  KVATTN_PREFILL_PAIRS(PF_PAIR_OK)
#undef PF_PAIR_OK
  return false;
}

cudaError_t prepare_prefill_kernels() {
  cudaError_t e = cudaSuccess;
#define PF_SET1(KF, VF, EX)                                                                          \
  if (e == cudaSuccess)                                                                              \
    e = cudaFuncSetAttribute(prefill_kernel<KF, VF, EX>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             pf::Layout<KF, VF>::kSmemBytes);
#define PF_SET(KF, VF) PF_SET1(KF, VF, true) PF_SET1(KF, VF, false)
  KVATTN_PREFILL_PAIRS(PF_SET)
#undef PF_SET
#undef PF_SET1
  return e;
}

template <int KF, int VF>
static cudaError_t launch_prefill_grid(cudaLaunchConfig_t cfg, const PrefillParams& prm, bool exact) {
  cfg.dynamicSmemBytes = pf::Layout<KF, VF>::kSmemBytes;
  return exact ? cudaLaunchKernelEx(&cfg, prefill_kernel<KF, VF, true>, prm)
               : cudaLaunchKernelEx(&cfg, prefill_kernel<KF, VF, false>, prm);
}

struct PrefillPlan {
  int n_mt, n_ks, pps, rows_pad;
  size_t lse_off, o_off, bytes;
};

// A CTA walks `spc` consecutive KV splits, merging them online in tensor memory, as long as
// the grid keeps at least ~16 waves of CTAs and the CTA's tile list fits in shared memory:
// fewer partials to write and merge.
PrefillPlan plan_prefill(int n_kv, int group, int n_q, int max_pages, int kv_split_tokens, int sm_count) {
  PrefillPlan pl{};
  const int rows = n_q * group;
  pl.n_mt = (rows + pf::kRows - 1) / pf::kRows;
  pl.n_mt += pl.n_mt & 1;  // M-tiles come in pairs (one cluster of two CTAs per pair)
  pl.rows_pad = pl.n_mt * pf::kRows;
  const int base = kv_split_tokens / kPageTokens;
  const long long splits0 = max_pages > 0 ? (max_pages + base - 1) / base : 1;
  long long spc = static_cast<long long>(n_kv) * pl.n_mt * splits0 / (static_cast<long long>(sm_count) * 16);
  spc = spc < 1 ? 1 : (spc > splits0 ? splits0 : spc);
  // pages per CTA: spc splits, at most kMaxTiles / 2 (a large split is then divided)
  const long long pps = base * spc;
  pl.pps = static_cast<int>(pps < pf::kMaxTiles / 2 ? pps : pf::kMaxTiles / 2);
  pl.n_ks = max_pages > 0 ? (max_pages + pl.pps - 1) / pl.pps : 1;
  pl.lse_off = 0;
  pl.o_off = ((sizeof(float) * static_cast<size_t>(n_kv) * pl.n_ks * pl.rows_pad + 255) / 256) * 256;
  pl.bytes = pl.n_ks > 1 ? pl.o_off + sizeof(float) * static_cast<size_t>(n_kv) * pl.n_ks * pl.rows_pad * kHeadDim : 0;
  return pl;
}

cudaError_t launch_prefill(const PrefillParams& prm0, int n_kv, int key_fmt, int val_fmt, bool exact,
                           cudaStream_t stream) {
  PrefillParams prm = prm0;
  const int rows = prm.n_q * prm.group;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.rows_pad / pf::kRows, prm.n_ks, n_kv);
    cfg.blockDim = dim3(pf::kThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaErrorInvalidValue;
#define PF_LAUNCH(KF, VF) \
  if (key_fmt == KF && val_fmt == VF) e = launch_prefill_grid<KF, VF>(cfg, prm, exact);
    KVATTN_PREFILL_PAIRS(PF_LAUNCH)
#undef PF_LAUNCH
    if (e != cudaSuccess || prm.n_ks == 1) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, n_kv);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel<8, 2>, static_cast<const float*>(prm.part_o),
                            static_cast<const float*>(prm.part_lse), prm.n_ks, prm.rows_pad, prm.group, prm.n_qh,
                            prm.out, prm.lse);
}

}  // namespace kvattn
