// Split-KV flash decode over block-quantized KV pages, for one query token or an MTP verify
// batch of up to 4 (Adaptive KV Streaming + RDNA 4 announcement, wqu.guru, method list:
// "paged decode attention extended to verify batches").  Key formats Q8_0, Q4_0, Q5_1 and
// Q5_0, value formats Q4_0, Q8_0 and Q4_1 (Vulkan speculative-decoding report, lcz.me/topic/
// 1398, "pitfalls": the legacy block quants valid as KV types; the q4_0/q4_0 and K q5_1 /
// V q4_0 caches; MTP tuning notes on one 7900 XTX, lcz.me/topic/593: a q5_0 / q4_1 cache).
//
// Grid: (split, KV head), each split a range of 16-token tiles.  One CTA per SM: lanes of warp
// 0 stream the pages into a shared-memory ring with bulk async copies (TMA engine, one K copy
// and one V copy per page, or one per region for a page shared with the next split); all warps
// consume them: twelve warps, each holding one 8-row n-tile of the head's query rows, the
// warps of a group (one per n-tile) sharing each 16-token tile.  All query rows of the KV
// head's group (group x n_q <= 24) are packed into the N dimension of legacy tensor-core MMAs
// so every KV byte is read from HBM once per group.  The arithmetic keeps the
// dequantized operands exact:
//   QK^T: f16 MMA (m16n8k16), A = the key codes decoded in registers (integers, exact in
//         f16), 16 tokens on M; B = the query row divided by its largest magnitude, as an f16
//         high part and an f16 low part (the rounded remainder: about 22 significant bits
//         together).  Each 32-channel block is accumulated on its own and multiplied by the
//         block's fp16 scale in fp32 (plus minimum x query block sum for zero-point keys).
//   PV:   f16 MMA (m16n8k16), A = V^T codes decoded in registers (exact), B = P^T (fp32
//         probabilities split into f16 high and low parts, transposed in registers with
//         movmatrix) times the per-token V block scale, again as an exact-product high part
//         and a low part.  Zero-point values add sum_t p_t m_t per block through an all-ones
//         A operand.
// The online softmax keeps a per-row running maximum and rescales the accumulators only
// when the maximum grows by more than 2^8 (p stays <= 256, safe in f16); the exact
// cross-lane maximum is only computed when a warp vote says some score crossed that bound.
// Warps merge their partial states in shared memory; CTAs write (o, lse) partials that a
// small follow-up grid (programmatic dependent launch) merges by log-sum-exp, the arithmetic
// of kvattn_merge_lse.
#include "decode.cuh"

namespace kvattn {

template <int KF, int VF, int NT>
struct DecodeCfg {
  // Twelve consumer warps, three per scheduler, so that a thread has at most 168 registers.
  // Each warp owns one n-tile (8 query rows) of a 16-token tile and all 256 channels; the NT
  // warps of a group share each tile (one per n-tile), and the groups take the CTA's tiles
  // round robin (tile k of the CTA goes to group k mod kGroups).  The query fragments sit in
  // shared memory.  (Sharing a tile between warps by channel halves or quarters, with partial
  // scores exchanged through shared memory, and sixteen warps at 128 registers, measured
  // slower.)
  static constexpr int kConsumerWarps = 12;
  static constexpr int kThreads = kConsumerWarps * 32;  // lanes of warp 0 also issue the copies
  static_assert(kConsumerWarps % NT == 0, "n-tiles per group");
  static constexpr int kGroups = kConsumerWarps / NT;   // warp groups taking tiles
  static constexpr int kNB = 8;                          // 32-channel blocks (all, per warp)
  static constexpr bool kK5 = KF == kKeyQ51 || KF == kKeyQ50;  // 5-bit key codes
  static constexpr bool kKMin = KF == kKeyQ51;                 // keys with a zero point
  static constexpr bool kVMin = VF == kValQ41;                 // values with a zero point
  static constexpr int kKBytes =
      KF == kKeyQ4 ? kK4PageBytes : KF == kKeyQ51 ? kK5PageBytes : KF == kKeyQ50 ? kK50PageBytes : kKPageBytes;
  static constexpr int kKScaleOff = KF == kKeyQ4 ? kK4ScaleOffset : kK5 ? kK5ScaleOffset : kKScaleOffset;
  static constexpr int kVBytes = VF == kValQ8 ? kV8PageBytes : VF == kValQ41 ? kV41PageBytes : kV4PageBytes;
  static constexpr int kVScaleOff = VF == kValQ8 ? kV8ScaleOffset : kV4ScaleOffset;
  static constexpr int kStageBytes = kKBytes + kVBytes;
  // Every region of a page (codes, fifth bits, scales, minima) is ordered by 16-token tile
  // first, so tiles [g0, g1) of a page are one contiguous range of each region: (offset of
  // the region, bytes per tile).  A stage holds K regions at 0 and V regions at kKBytes.
  static constexpr int kKRegions = KF == kKeyQ51 ? 4 : KF == kKeyQ50 ? 3 : 2;
  static constexpr int kVRegions = VF == kValQ41 ? 3 : 2;
  __host__ __device__ static constexpr int k_reg_off(int r) {
    return r == 0 ? 0 : r == 1 ? (kK5 ? kK5HighOffset : kKScaleOff) : r == 2 ? kK5ScaleOffset : kK5MinOffset;
  }
  __host__ __device__ static constexpr int k_reg_tile(int r) {
    return r == 0 ? (KF == kKeyQ8 ? 4096 : 2048) : r == 1 && kK5 ? 512 : 256;
  }
  __host__ __device__ static constexpr int v_reg_off(int r) { return r == 0 ? 0 : r == 1 ? kVScaleOff : kV41MinOffset; }
  __host__ __device__ static constexpr int v_reg_tile(int r) { return r == 0 ? (VF == kValQ8 ? 4096 : 2048) : 256; }
  static_assert(8 * (k_reg_tile(0) + k_reg_tile(1) + (kKRegions > 2 ? k_reg_tile(2) : 0) +
                     (kKRegions > 3 ? k_reg_tile(3) : 0)) == kKBytes, "K regions");
  static_assert(8 * (v_reg_tile(0) + v_reg_tile(1) + (kVRegions > 2 ? v_reg_tile(2) : 0)) == kVBytes, "V regions");
  static_assert(k_reg_off(1) == 8 * k_reg_tile(0) && (kKRegions < 3 || k_reg_off(2) == k_reg_off(1) + 8 * k_reg_tile(1)) &&
                (kKRegions < 4 || k_reg_off(3) == k_reg_off(2) + 8 * k_reg_tile(2)), "K region offsets");
  static_assert(v_reg_off(1) == 8 * v_reg_tile(0) && (kVRegions < 3 || v_reg_off(2) == v_reg_off(1) + 8 * v_reg_tile(1)),
                "V region offsets");
  // the query B fragments: [block][k-step][n-tile][lane][hi0, hi1, lo0, lo1]
  static constexpr int kQBytes = 8 * 2 * NT * 32 * 16;
  static constexpr int kRowsPad = NT * 8;
  // rows of the output merge buffer are padded by 4 floats: the four lanes of an MMA quad
  // store rows 2t, 2t+1 of the same dims and then fall into different banks
  static constexpr int kOStride = kHeadDim + 4;
  static constexpr int kMergeBytes = kConsumerWarps * 8 * (kOStride + 2) * 4;  // 8 rows per warp
  // Page stages: for 8 and 16 rows as many as fit beside the query fragments and the barriers
  // (at most 6).  The 24-row shape is bound by arithmetic, not by the page stream: it takes
  // the fewest stages that hold the merge buffer (at least 2), which measured faster (a
  // smaller shared-memory footprint leaves more of the SM's memory to L1).
  static constexpr int kStagesFit = (227 * 1024 - 256 - kQBytes) / kStageBytes;
  static constexpr int kStagesMin = (kMergeBytes + kStageBytes - 1) / kStageBytes < 2
                                        ? 2 : (kMergeBytes + kStageBytes - 1) / kStageBytes;
  static constexpr int kStages = NT == 3 ? kStagesMin : (kStagesFit < 6 ? kStagesFit : 6);
  static constexpr int kRingBytes = kStages * kStageBytes;
  static_assert(kMergeBytes <= kRingBytes, "merge buffer must fit in the ring");
  static constexpr int kQOffset = kRingBytes;
  static constexpr int kBarOffset = kQOffset + kQBytes;
  static constexpr int kSmemBytes = kBarOffset + 256;
  static_assert(8 * kStages + 4 * (4 * kStages + 1) <= 256, "stage bookkeeping");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

constexpr uint32_t kHalf2Magic = 0x64006400u;  // f16 1024.0 in both halves
constexpr uint32_t kByte64x4 = 0x64646464u;    // high byte of f16 1024.0, for byte permutes
constexpr uint32_t kHalf2_1032 = 0x64086408u;  // 1024 + 8
constexpr uint32_t kHalf2_1040 = 0x64106410u;  // 1024 + 16
constexpr uint32_t kHalf2_1152 = 0x64806480u;  // 1024 + 128
constexpr uint32_t kHalf2_1_16 = 0x2C002C00u;  // 1/16
constexpr uint32_t kHalf2_m72 = 0xD480D480u;   // -(64 + 8)
constexpr uint32_t kHalf2_m64 = 0xD400D400u;   // -64
constexpr uint32_t kHalf2_m80 = 0xD500D500u;   // -(64 + 16)
constexpr uint32_t kHalf2_Sign = 0x80008000u;

// B operand (probabilities times a per-token fp16 factor f) as an unevaluated f16 sum hi + lo:
// hi = f16(ph * f); ph * f - hi is exact in f16 (an 11 x 11-bit product rounded to 11 bits
// leaves at most 11 bits), and lo adds pl * f with one rounding.  hi + lo equals (ph + pl) * f
// to about 2^-22 relative.
__device__ __forceinline__ void split_scaled(uint32_t ph, uint32_t pl, uint32_t f, uint32_t& hi, uint32_t& lo) {
  hi = hmul2(ph, f);
  lo = hfma2(pl, f, hfma2(ph, f, hi ^ kHalf2_Sign));
}

// fp32 pair -> f16 hi part (round to nearest) and f16 lo part (the rounded remainder).
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_half2(x0, x1);
  lo = pack_half2(x0 - half_lo(hi), x1 - half_hi(hi));
}

// Encodes the appended tokens that fall in tokens [pos_lo, pos_lo + 16) of a page held in a
// shared-memory stage (K bytes at `stage`, V bytes k_bytes further on) into that copy, for the
// lanes of store_mask.  Kept out of line: it runs for one tile in thousands, and inlined it
// would take registers from the tile loop.
// Arguments are scalars: a reference to the kernel's parameter block would make every thread
// copy that block to its stack.
__device__ __noinline__ void patch_stage(const float* k_new, const float* v_new, int n_new, int new_pos0, int h,
                                         int n_kv, int lane, uint8_t* stage, int k_bytes, int logical, int pos_lo,
                                         int k_fmt, int v_fmt, uint32_t mask) {
  for (int n = 0; n < n_new; ++n) {
    const int pos = new_pos0 + n;
    if (pos < pos_lo || pos >= pos_lo + 16) continue;
    const long long row = (static_cast<long long>(n) * n_kv + h) * kHeadDim;
    const float4* ks = reinterpret_cast<const float4*>(k_new + row + lane * 8);
    const float4* vs = reinterpret_cast<const float4*>(v_new + row + lane * 8);
    const float4 k0 = ks[0], k1 = ks[1], v0 = vs[0], v1 = vs[1];
    const float kx[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
    const float vx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    encode_token(kx, vx, lane, stage, stage + k_bytes, pos - logical * kPageTokens, k_fmt, v_fmt, mask);
    // the stage is later refilled by the copy engine (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
  }
}

// Encodes appended token n of KV head h into its page in global memory (one warp).
__device__ __noinline__ void append_global(const float* k_new, const float* v_new, const int32_t* table,
                                           int table_blocks, uint8_t* k_pool, uint8_t* v_pool, int64_t k_stride,
                                           int64_t v_stride, int64_t n_pages, int pos, int h, int n_kv, int lane,
                                           int n, int k_fmt, int v_fmt) {
  const long long row = (static_cast<long long>(n) * n_kv + h) * kHeadDim;
  const float4* ks = reinterpret_cast<const float4*>(k_new + row + lane * 8);
  const float4* vs = reinterpret_cast<const float4*>(v_new + row + lane * 8);
  const float4 k0 = ks[0], k1 = ks[1], v0 = vs[0], v1 = vs[1];
  const int page = table[static_cast<long long>(h) * table_blocks + pos / kPageTokens];
  if (page < 0 || page >= n_pages) {
    if (lane == 0) record_error(KVATTN_ERR_BAD_PAGE);
    return;
  }
  const float kx[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
  const float vx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  encode_token(kx, vx, lane, k_pool + static_cast<int64_t>(page) * k_stride, v_pool + static_cast<int64_t>(page) * v_stride,
               pos % kPageTokens, k_fmt, v_fmt, 0xffffffffu);
}

template <int KF, int VF, int NT>
__global__ void __launch_bounds__(DecodeCfg<KF, VF, NT>::kThreads, 1) decode_kernel(const DecodeParams p) {
  using C = DecodeCfg<KF, VF, NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  int* rel_cnt = reinterpret_cast<int*>(full + C::kStages);  // [kStages] (warp, tile) pairs done
  int* st_page = rel_cnt + C::kStages;     // [kStages] the page last issued into the stage, -1: none
  int* st_logical = st_page + C::kStages;  // [kStages]
  int* st_valid = st_logical + C::kStages;  // [kStages]
  int* s_flags = st_valid + C::kStages;  // [0] abort

  // the LSE-merge grid that follows may start launching now; it waits for this grid's data
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int h = blockIdx.y;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n_rows = p.group * p.n_q;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      rel_cnt[s] = 0;
      st_page[s] = -1;
    }
    s_flags[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Launched with programmatic dependent launch: the CTAs become resident and set up while
  // the previous kernel on the stream (typically the quantize-append of the new token)
  // drains; every read of the caller's data comes after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  int np = p.max_pages;
  if (p.n_pages_arr) np = min(max(p.n_pages_arr[h], 0), p.max_pages);
  // This split's 16-token tiles [t_first, t_last) of the head's 8 np tiles, and the pages they
  // touch, [first, first + count): the CTAs' shares differ by at most one tile.  The first and
  // the last page may be shared with the neighbouring splits; each copies only its own tiles.
  const int t_first = static_cast<int>(static_cast<long long>(split) * 8 * np / p.n_splits);
  const int t_last = static_cast<int>(static_cast<long long>(split + 1) * 8 * np / p.n_splits);
  const int first = t_first >> 3;
  const int count = t_last > t_first ? ((t_last + 7) >> 3) - first : 0;
  // tiles [tile_lo(i), tile_hi(i)) of the CTA's page i are in its range
  auto tile_lo = [&](int i) { return i == 0 ? (t_first & 7) : 0; };
  auto tile_hi = [&](int i) { return i == count - 1 && (t_last & 7) ? (t_last & 7) : 8; };

  // per-warp softmax state (consumers): rows 2t, 2t + 1 of the warp's n-tile (index c)
  float m_run[2], l_run[2];
  float oacc[2 * C::kNB][4];
  // values with a zero point: sum over tokens of p * m per (block, query row), kept apart
  // from oacc (every dimension of a block gets the same term) and added at the end; an MMA
  // accumulator with the 8 blocks as M (rows g: block g, rows g + 8 unused)
  float racc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    m_run[c] = -INFINITY;
    l_run[c] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < 2 * C::kNB; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[i][e] = 0.f;

  const int grp = warp / NT;  // the warps that share a tile, one per n-tile
  const int nt0 = warp % NT;  // this warp's n-tile: query rows 8 nt0 .. 8 nt0 + 7

  // Page copies: the first kStages pages are issued up front by lanes of warp 0; after
  // that, the warp that finishes the last of a page's tiles refills its stage at once with
  // the page kStages further on, so kStages - 1 pages stay in flight while one is being
  // consumed.  Each stage carries the number of the page last issued into it.
  const int32_t* plist = p.page_list + static_cast<long long>(h) * p.max_pages;
  const int32_t* plog = p.page_logical ? p.page_logical + static_cast<long long>(h) * p.max_pages : nullptr;
  auto issue_page = [&](int i, int page, int logical) {
    const int s = i % C::kStages;
    *reinterpret_cast<volatile int*>(&st_page[s]) = i;
    st_logical[s] = logical;
    if (page < 0 || page >= p.n_pages) {
      record_error(KVATTN_ERR_BAD_PAGE);
      st_valid[s] = 0;
      mbar_arrive(&full[s]);
      return;
    }
    st_valid[s] = 1;
    uint8_t* stage = smem + s * C::kStageBytes;
    const uint8_t* ksrc = p.k_pool + static_cast<int64_t>(page) * p.k_stride;
    const uint8_t* vsrc = p.v_pool + static_cast<int64_t>(page) * p.v_stride;
    const int g0 = tile_lo(i), g1 = tile_hi(i);
    if (g0 == 0 && g1 == 8) {
      mbar_arrive_expect_tx(&full[s], C::kStageBytes);
      bulk_g2s(stage, ksrc, C::kKBytes, &full[s]);
      bulk_g2s(stage + C::kKBytes, vsrc, C::kVBytes, &full[s]);
    } else {
      // a page shared with a neighbouring split: only tiles [g0, g1) of every region
      mbar_arrive_expect_tx(&full[s], (g1 - g0) * (C::kStageBytes / 8));
#pragma unroll
      for (int r = 0; r < C::kKRegions; ++r) {
        const int o = C::k_reg_off(r) + g0 * C::k_reg_tile(r);
        bulk_g2s(stage + o, ksrc + o, (g1 - g0) * C::k_reg_tile(r), &full[s]);
      }
#pragma unroll
      for (int r = 0; r < C::kVRegions; ++r) {
        const int o = C::v_reg_off(r) + g0 * C::v_reg_tile(r);
        bulk_g2s(stage + C::kKBytes + o, vsrc + o, (g1 - g0) * C::v_reg_tile(r), &full[s]);
      }
    }
  };
  auto issue = [&](int i) {
    const int idx = first + i;
    issue_page(i, plist[idx], plog ? plog[idx] : idx);
  };
  // The first stages: lanes of warp 0 read their page ids in parallel; lane 0 issues the first
  // page before the others issue theirs, so that of all the CTAs' first requests, which reach
  // the memory system together, each CTA's first page comes first and its warps can start.
  if (warp == 0 && lane < C::kStages && lane < count) {
    const int idx = first + lane;
    const int page = plist[idx];
    const int logical = plog ? plog[idx] : idx;
    if (lane == 0) issue_page(0, page, logical);
    __syncwarp((1u << (count < C::kStages ? count : C::kStages)) - 1u);
    if (lane > 0) issue_page(lane, page, logical);
  }
  // Appended tokens: split 0 of every head encodes them into their pages in global memory, one
  // warp per token (warps 1 ..).  A CTA that streams such a page encodes the token again into
  // its shared-memory copy before using it (below), so no CTA waits for another.
  if (p.n_new > 0 && split == 0 && warp >= 1 && warp <= p.n_new)
    append_global(p.k_new, p.v_new, p.new_table, p.new_blocks, const_cast<uint8_t*>(p.k_pool),
                  const_cast<uint8_t*>(p.v_pool), p.k_stride, p.v_stride, p.n_pages, p.new_pos0 + warp - 1, h,
                  gridDim.y, lane, warp - 1, KF, VF);

  {
    // ------------------------------------------------------------------ consumers
    // query rows of this KV head: r = qi * group + j  ->  q[qi][h * group + j][:]
    // B fragments: the query row divided by its largest magnitude, split into an f16 high
    // part and an f16 low part (the rounded remainder), per block and k-step (two regs each),
    // in shared memory for the n-tile's warps; crow[c] = amax / 16 * log2(e) turns a dot
    // product with the normalised row into a base-2 softmax score.
    float crow[2];
    // zero-point keys: the sums over each block's channels of the normalised query row g of
    // the n-tile, as the B fragment (k = block 2t, 2t + 1) of an MMA that adds
    // sum_b m[token][b] qsum[b][row] to S, split into f16 high and low parts
    uint32_t qsb_hi = 0u, qsb_lo = 0u;
    float qs0 = 0.f, qs1 = 0.f;
    // query positions of this thread's accumulator rows, loaded first: every global read of
    // the setup is issued before any of them is used
    int qpos_row[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int rr = nt0 * 8 + 2 * t + c;
      qpos_row[c] = rr < n_rows ? p.q_pos[rr / p.group] : INT_MAX;
    }
    const uint32_t q_s = smem_u32(smem + C::kQOffset);
    {
      const int r = nt0 * 8 + g;
      float x[kBlocks][8];
      if (r < n_rows) {
        const int qi = r / p.group, j = r % p.group;
        const float* qr = p.q + (static_cast<long long>(qi) * p.n_qh + h * p.group + j) * kHeadDim;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
          const float4 u = *reinterpret_cast<const float4*>(qr + 32 * b + 8 * t);
          const float4 w = *reinterpret_cast<const float4*>(qr + 32 * b + 8 * t + 4);
          x[b][0] = u.x; x[b][1] = u.y; x[b][2] = u.z; x[b][3] = u.w;
          x[b][4] = w.x; x[b][5] = w.y; x[b][6] = w.z; x[b][7] = w.w;
        }
      } else {
#pragma unroll
        for (int b = 0; b < kBlocks; ++b)
#pragma unroll
          for (int e = 0; e < 8; ++e) x[b][e] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int b = 0; b < kBlocks; ++b)
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[b][e]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const float inv = amax > 0.f ? 1.f / amax : 0.f;
#pragma unroll
      for (int bl = 0; bl < C::kNB; ++bl) {
        float xv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = x[bl][e] * inv;
        // k-step 0 of the block: channels 8t+0..3, k-step 1: 8t+4..7 (k = 2t, 2t+1 | 2t+8, 2t+9)
        uint32_t hi[2][2], lo[2][2];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          split_pair(xv[4 * ks], xv[4 * ks + 1], hi[ks][0], lo[ks][0]);
          split_pair(xv[4 * ks + 2], xv[4 * ks + 3], hi[ks][1], lo[ks][1]);
        }
        // every group holds the same values; the warps of group 0 (one per n-tile) write them
        if (warp < NT) {
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                             q_s + ((((bl * 2 + ks) * NT + nt0) * 32 + lane) * 16)),
                         "r"(hi[ks][0]), "r"(hi[ks][1]), "r"(lo[ks][0]), "r"(lo[ks][1])
                         : "memory");
        }
        if constexpr (C::kKMin) {
          float sm = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sm += xv[e];
          sm += __shfl_xor_sync(0xffffffffu, sm, 1);
          sm += __shfl_xor_sync(0xffffffffu, sm, 2);
          if (bl == 2 * t) qs0 = sm;
          if (bl == 2 * t + 1) qs1 = sm;
        }
      }
      if constexpr (C::kKMin) split_pair(qs0, qs1, qsb_hi, qsb_lo);
      const float cr = amax * (1.0f / 16.0f) * 1.4426950408889634f;
      crow[0] = __shfl_sync(0xffffffffu, cr, (2 * t) * 4);
      crow[1] = __shfl_sync(0xffffffffu, cr, (2 * t + 1) * 4);
    }
    __syncthreads();
    // the smallest query position over the warp's rows (the four t-lanes of a quad hold them)
    int qpos_min = min(qpos_row[0], qpos_row[1]);
    qpos_min = min(qpos_min, __shfl_xor_sync(0xffffffffu, qpos_min, 1));
    qpos_min = min(qpos_min, __shfl_xor_sync(0xffffffffu, qpos_min, 2));

    // the B fragments (hi0, hi1, lo0, lo1) of block bl, k-step ks
    auto qfrag = [&](int bl, int ks) -> uint4 {
      return lds128(q_s + ((((bl * 2 + ks) * NT + nt0) * 32 + lane) * 16));
    };

    // The CTA's tiles in increasing order, group grp taking k = grp, grp + kGroups, ... (the
    // head's tile j = t_first + k: the CTA's page i = j / 8 - first, tile G = j % 8).  A stage
    // is refilled once every in-range tile of its page is done.  With more groups than tiles
    // per page a group skips pages, so the parity
    // of a stage's barrier alone cannot tell page i from page i - kStages.  A group therefore
    // first waits until the stage's tag names page i (issued only after every tile of page
    // i - kStages is done, so that page's phase has completed), then for the barrier phase of
    // page i (which cannot move on before this group's tile of page i is done).
    const int new_lo = p.new_pos0, new_hi = p.new_pos0 + p.n_new;  // appended positions
    const int n_tiles = t_last - t_first;
    for (int k = grp; k < n_tiles; k += C::kGroups) {
      const int j = t_first + k;  // the head's tile
      const int i = (j >> 3) - first;
      const int G = j & 7;
      const int s = i % C::kStages;
      const uint32_t par = (i / C::kStages) & 1;
      if (!wait_tag(&st_page[s], i) || !mbar_wait(&full[s], par)) {
        s_flags[0] = 1;
        break;
      }
      if (st_valid[s]) {
        const uint32_t kb = smem_u32(smem + s * C::kStageBytes);
        const uint32_t vb = kb + C::kKBytes;
        const int logical = st_logical[s];
        const bool need_mask = static_cast<long long>(logical) * kPageTokens + (kPageTokens - 1) > qpos_min;
        {
          const int pos_lo = logical * kPageTokens + 16 * G;
          if (pos_lo < new_hi && pos_lo + 16 > new_lo) {
            // an appended token in this tile: encode it into the stage, as split 0 encodes it
            // into the page in global memory.  Each of the tile's warps writes the whole token
            // (the same bytes) before it reads the tile, so none reads a partial patch.
            patch_stage(p.k_new, p.v_new, p.n_new, p.new_pos0, h, gridDim.y, lane, smem + s * C::kStageBytes,
                        C::kKBytes, logical, pos_lo, KF, VF, 0xffffffffu);
          }
          // ---------------- S = K Q^T over the 256 channels ----------------
          // Key codes enter the MMA exactly (integers in f16).  Each 32-channel block is
          // accumulated on its own (four MMAs: two k-steps, query high and low parts) and then
          // scaled by the block's fp32 scale into S; with a zero point, two more MMAs add the
          // block minima times the query block sums.
          float sacc[4] = {0.f, 0.f, 0.f, 0.f};
          // key scales of rows g (H=0) and g+8 (H=1) for the 8 blocks, fp32; zero-point keys:
          // the minima of blocks 2t, 2t + 1 of the same rows (the A fragment of the MMA that
          // adds the minimum terms)
          float dkf[2][C::kNB];
          uint32_t mka[2] = {0u, 0u};
#pragma unroll
          for (int H = 0; H < 2; ++H) {
            const uint32_t a = kb + C::kKScaleOff + (((G * 8 + g) * 2 + H) * 8) * 2;
            uint32_t w[4];
            const uint4 v = lds128(a);
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
            if constexpr (C::kKMin) mka[H] = lds32(a + (kK5MinOffset - kK5ScaleOffset) + 4 * t);
#pragma unroll
            for (int e = 0; e < C::kNB / 2; ++e) {
              dkf[H][2 * e] = half_lo(w[e]);
              dkf[H][2 * e + 1] = half_hi(w[e]);
            }
          }
          // one block: four MMAs into xb, then S += d * xb
          auto block_qk = [&](int bl, const uint32_t (&A)[2][4]) {
            float xb[4];
            const uint4 f0 = qfrag(bl, 0), f1 = qfrag(bl, 1);
            mma_f16_z(xb, A[0][0], A[0][1], A[0][2], A[0][3], f0.x, f0.y);
            mma_f16(xb, A[0][0], A[0][1], A[0][2], A[0][3], f0.z, f0.w);
            mma_f16(xb, A[1][0], A[1][1], A[1][2], A[1][3], f1.x, f1.y);
            mma_f16(xb, A[1][0], A[1][1], A[1][2], A[1][3], f1.z, f1.w);
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[e] = fmaf(dkf[e >> 1][bl], xb[e], sacc[e]);
          };
          if constexpr (KF == kKeyQ8) {
#pragma unroll
            for (int P = 0; P < C::kNB / 2; ++P) {
              const uint4 ka = lds128(kb + ((((G * 4 + P) * 2 + 0) * 8 + g) * 4 + t) * 16);
              const uint4 kc = lds128(kb + ((((G * 4 + P) * 2 + 1) * 8 + g) * 4 + t) * 16);
              // code bytes are offset-binary (q + 128)
              const uint32_t wg[4] = {ka.x, ka.y, ka.z, ka.w};
              const uint32_t w8[4] = {kc.x, kc.y, kc.z, kc.w};
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                uint32_t A[2][4];
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                  // exact code -> f16: 1024 + (q + 128) - 1152
                  A[ks][0] = hsub2(prmt(wg[2 * e + ks], kByte64x4, 0x4140u), kHalf2_1152);
                  A[ks][2] = hsub2(prmt(wg[2 * e + ks], kByte64x4, 0x4342u), kHalf2_1152);
                  A[ks][1] = hsub2(prmt(w8[2 * e + ks], kByte64x4, 0x4140u), kHalf2_1152);
                  A[ks][3] = hsub2(prmt(w8[2 * e + ks], kByte64x4, 0x4342u), kHalf2_1152);
                }
                block_qk(2 * P + e, A);
              }
            }
          } else {
            // 4- and 5-bit keys: one 32-bit word per (token, block) and lane holds channels 8t + i,
            // channel i at bit 4 * (i / 2) + 16 * (i % 2); a shift by 8 * ks and two masks give
            // the f16 pairs (4ks, 4ks + 1) and (4ks + 2, 4ks + 3) of k-step ks (1024 + q and
            // 1024 + 16q).  5-bit keys: the fifth bits of the lane's four blocks of one token
            // sit in one word, channel (c, i) at bit 16(i%2) + 4c + i/2, and are shifted to bit 4
            // or bit 8 of each half.  The code (minus 8 for Q4_0, 16 for Q5_0) is exact in f16.
#pragma unroll
            for (int Q = 0; Q < 2; ++Q) {
              const int row0 = (((G * 2 + Q) * 2 + 0) * 8 + g) * 4 + t;
              const int row1 = (((G * 2 + Q) * 2 + 1) * 8 + g) * 4 + t;
              const uint4 ka = lds128(kb + row0 * 16);
              const uint4 kc = lds128(kb + row1 * 16);
              const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
              const uint32_t wc[4] = {kc.x, kc.y, kc.z, kc.w};
              uint32_t xa5 = 0, xc5 = 0;
              if constexpr (C::kK5) {
                xa5 = lds32(kb + kK5HighOffset + row0 * 4);
                xc5 = lds32(kb + kK5HighOffset + row1 * 4);
              }
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                uint32_t A[2][4];
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                  const uint32_t xa = wa[c] >> (8 * ks), xc = wc[c] >> (8 * ks);
                  if constexpr (KF == kKeyQ4) {
                    A[ks][0] = hsub2(and_or(xa, 0x000F000Fu, kHalf2Magic), kHalf2_1032);
                    A[ks][2] = hfma2(and_or(xa, 0x00F000F0u, kHalf2Magic), kHalf2_1_16, kHalf2_m72);
                    A[ks][1] = hsub2(and_or(xc, 0x000F000Fu, kHalf2Magic), kHalf2_1032);
                    A[ks][3] = hfma2(and_or(xc, 0x00F000F0u, kHalf2Magic), kHalf2_1_16, kHalf2_m72);
                  } else {
                    const int slo = 4 - (4 * c + 2 * ks), shi = 7 - (4 * c + 2 * ks);
                    const uint32_t ha_lo = slo >= 0 ? xa5 << slo : xa5 >> -slo;
                    const uint32_t ha_hi = shi >= 0 ? xa5 << shi : xa5 >> -shi;
                    const uint32_t hc_lo = slo >= 0 ? xc5 << slo : xc5 >> -slo;
                    const uint32_t hc_hi = shi >= 0 ? xc5 << shi : xc5 >> -shi;
                    constexpr uint32_t kSubLo = KF == kKeyQ50 ? kHalf2_1040 : kHalf2Magic;
                    constexpr uint32_t kAddHi = KF == kKeyQ50 ? kHalf2_m80 : kHalf2_m64;
                    A[ks][0] = hsub2(or_and(and_or(xa, 0x000F000Fu, kHalf2Magic), ha_lo, 0x00100010u), kSubLo);
                    A[ks][2] = hfma2(or_and(and_or(xa, 0x00F000F0u, kHalf2Magic), ha_hi, 0x01000100u), kHalf2_1_16,
                                     kAddHi);
                    A[ks][1] = hsub2(or_and(and_or(xc, 0x000F000Fu, kHalf2Magic), hc_lo, 0x00100010u), kSubLo);
                    A[ks][3] = hfma2(or_and(and_or(xc, 0x00F000F0u, kHalf2Magic), hc_hi, 0x01000100u), kHalf2_1_16,
                                     kAddHi);
                  }
                }
                block_qk(4 * Q + c, A);
              }
            }
          }
          if constexpr (C::kKMin) {
            // S += sum_b m[token][b] qsum[b][row] as one MMA per part of the block sums: A =
            // the minima (tokens g, g + 8 x blocks 2t, 2t + 1; k = 8..15 is zero, exact in f16),
            // B = the block sums of the query rows; the products accumulate in fp32
            mma_f16(sacc, mka[0], mka[1], 0u, 0u, qsb_hi, 0u);
            mma_f16(sacc, mka[0], mka[1], 0u, 0u, qsb_lo, 0u);
          }
          // ---------------- online softmax (base 2) ----------------
          // The running maximum m_run of a row is shared by the 8 lanes that hold the row.
          // It only has to bound the scores to within 2^8 (p <= 256 in f16), so the exact
          // cross-lane maximum is computed only when some lane sees a score above
          // m_run + 8: one warp vote per tile instead of three shuffles per row.
          const int key0 = logical * kPageTokens + 16 * G + g;  // rows e<2: token g, e>=2: g+8
          float sv[4], lm[2];
          bool need = false;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sv[e] = sacc[e] * crow[e & 1];
            if (need_mask && key0 + 8 * (e >> 1) > qpos_row[e & 1]) sv[e] = -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            lm[c] = fmaxf(sv[c], sv[c + 2]);
            need |= lm[c] > m_run[c] + 8.f;
          }
          if (__any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              float mx = lm[c];
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
              if (mx > m_run[c] + 8.f) {
                const float alpha = fast_exp2(m_run[c] - mx);  // 0 when m_run = -inf
                l_run[c] *= alpha;
#pragma unroll
                for (int mt = 0; mt < 2 * C::kNB; ++mt) {
                  oacc[mt][c] *= alpha;
                  oacc[mt][c + 2] *= alpha;
                }
                if constexpr (C::kVMin) racc[c] *= alpha;
                m_run[c] = mx;
              }
            }
          }
          // P as f16 high and low parts, transposed in registers into B fragments
          uint32_t pbh[2], pbl[2];
          {
            float pr[4];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float mu = m_run[c] == -INFINITY ? 0.f : m_run[c];
              pr[c] = fast_exp2(sv[c] - mu);
              pr[c + 2] = fast_exp2(sv[c + 2] - mu);
              l_run[c] += pr[c] + pr[c + 2];
            }
            uint32_t h01, l01, h23, l23;
            split_pair(pr[0], pr[1], h01, l01);
            split_pair(pr[2], pr[3], h23, l23);
            pbh[0] = movmatrix_t(h01);
            pbh[1] = movmatrix_t(h23);
            pbl[0] = movmatrix_t(l01);
            pbl[1] = movmatrix_t(l23);
          }
          // ---------------- O^T += V^T P^T ----------------
          // V codes enter the MMA exactly; the per-token block scale multiplies P (as a high
          // and a low f16 part), two MMAs per 16-dimension half.
          if constexpr (VF != kValQ8) {
#pragma unroll
            for (int Cc = 0; Cc < C::kNB / 2; ++Cc) {
              const uint4 vw = lds128(vb + ((((G * 4 + Cc) * 8 + g) * 4 + t) * 16));
              const uint32_t sidx = vb + C::kVScaleOff + (((G * 4 + t) * 8 + 2 * Cc) * 4) * 2;
              const uint4 dv = lds128(sidx);
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int bl = 2 * Cc + e;
                const uint32_t W0 = e ? vw.z : vw.x, W1 = e ? vw.w : vw.y;
                const uint32_t d0 = e ? dv.z : dv.x, d1 = e ? dv.w : dv.y;
                const uint32_t W0s = W0 >> 8, W1s = W1 >> 8;
                // Q4_0: q - 8 (1024 + q - 1032, or (1024 + 16q) / 16 - 72); Q4_1: q
                constexpr uint32_t kSubLo = C::kVMin ? kHalf2Magic : kHalf2_1032;
                constexpr uint32_t kAddHi = C::kVMin ? kHalf2_m64 : kHalf2_m72;
                const uint32_t a00 = hsub2(and_or(W0, 0x000F000Fu, kHalf2Magic), kSubLo);
                const uint32_t a01 = hfma2(and_or(W0, 0x00F000F0u, kHalf2Magic), kHalf2_1_16, kAddHi);
                const uint32_t a02 = hsub2(and_or(W1, 0x000F000Fu, kHalf2Magic), kSubLo);
                const uint32_t a03 = hfma2(and_or(W1, 0x00F000F0u, kHalf2Magic), kHalf2_1_16, kAddHi);
                const uint32_t a10 = hsub2(and_or(W0s, 0x000F000Fu, kHalf2Magic), kSubLo);
                const uint32_t a11 = hfma2(and_or(W0s, 0x00F000F0u, kHalf2Magic), kHalf2_1_16, kAddHi);
                const uint32_t a12 = hsub2(and_or(W1s, 0x000F000Fu, kHalf2Magic), kSubLo);
                const uint32_t a13 = hfma2(and_or(W1s, 0x00F000F0u, kHalf2Magic), kHalf2_1_16, kAddHi);
                uint32_t bh0, bl0, bh1, bl1;
                split_scaled(pbh[0], pbl[0], d0, bh0, bl0);
                split_scaled(pbh[1], pbl[1], d1, bh1, bl1);
                mma_f16(oacc[2 * bl], a00, a01, a02, a03, bh0, bh1);
                mma_f16(oacc[2 * bl], a00, a01, a02, a03, bl0, bl1);
                mma_f16(oacc[2 * bl + 1], a10, a11, a12, a13, bh0, bh1);
                mma_f16(oacc[2 * bl + 1], a10, a11, a12, a13, bl0, bl1);
              }
            }
            if constexpr (C::kVMin) {
              // sum over the tile's tokens of p * m for all 8 blocks at once: A = the minima
              // (block g x tokens 2t, 2t + 1 | 2t + 8, 2t + 9, exact in f16; blocks 8..15 zero),
              // B = P^T as its high and low parts
              uint32_t m01, m89;
              asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                           : "=r"(m01), "=r"(m89)
                           : "r"(vb + kV41MinOffset + (((G * 4 + t) * 8 + g) * 4) * 2));
              mma_f16(racc, m01, 0u, m89, 0u, pbh[0], pbh[1]);
              mma_f16(racc, m01, 0u, m89, 0u, pbl[0], pbl[1]);
            }
          } else {
#pragma unroll
            for (int b = 0; b < C::kNB; ++b) {
              const uint4 vw = lds128(vb + ((((G * 8 + b) * 8 + g) * 4 + t) * 16));
              uint32_t d0, d1;
              asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                           : "=r"(d0), "=r"(d1)
                           : "r"(vb + kV8ScaleOffset + (((G * 4 + t) * 8 + b) * 4) * 2));
              const uint32_t w[4] = {vw.x, vw.y, vw.z, vw.w};  // offset-binary code bytes (q + 128)
              uint32_t a[4][2];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                a[q][0] = hsub2(prmt(w[q], kByte64x4, 0x4140u), kHalf2_1152);
                a[q][1] = hsub2(prmt(w[q], kByte64x4, 0x4342u), kHalf2_1152);
              }
              uint32_t bh0, bl0, bh1, bl1;
              split_scaled(pbh[0], pbl[0], d0, bh0, bl0);
              split_scaled(pbh[1], pbl[1], d1, bh1, bl1);
              mma_f16(oacc[2 * b], a[0][0], a[0][1], a[1][0], a[1][1], bh0, bh1);
              mma_f16(oacc[2 * b], a[0][0], a[0][1], a[1][0], a[1][1], bl0, bl1);
              mma_f16(oacc[2 * b + 1], a[2][0], a[2][1], a[3][0], a[3][1], bh0, bh1);
              mma_f16(oacc[2 * b + 1], a[2][0], a[2][1], a[3][0], a[3][1], bl0, bl1);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        if (atomicAdd(&rel_cnt[s], 1) == (tile_hi(i) - tile_lo(i)) * NT - 1) {
          rel_cnt[s] = 0;
          if (i + C::kStages < count) issue(i + C::kStages);
        }
      }
    }
    // reduce the per-thread partial sums over the 8 token lanes
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float l = l_run[c];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[c] = l;
    }
  }

  __syncthreads();
  if (s_flags[0]) {
    // A bounded wait expired: wait (bounded) for the copies still in flight, then leave.
    if (threadIdx.x == 0) {
      for (int s = 0; s < C::kStages; ++s) {
        const int pg = *reinterpret_cast<volatile int*>(&st_page[s]);
        if (pg < 0) continue;
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&full[s], (pg / C::kStages) & 1)) {
          if (global_timer_ns() - t0 > kWaitTimeoutNs) break;
        }
      }
    }
    return;
  }

  // ---------------- merge the CTA's softmax streams in shared memory ----------------
  // one stream per warp, over the 8 rows of its n-tile (local row lr = row % 8):
  // ms[warp][lr], ls[warp][lr], os[warp][lr][kOStride]  (all fp32)
  float* ms = reinterpret_cast<float*>(smem);
  float* ls = ms + C::kConsumerWarps * 8;
  float* os = ls + C::kConsumerWarps * 8;
  {
    // zero-point values: the minimum terms of block b for rows 2t, 2t + 1 sit in lane 4b + t
    float rv[C::kVMin ? C::kNB : 1][2];
    if constexpr (C::kVMin) {
#pragma unroll
      for (int b = 0; b < C::kNB; ++b)
#pragma unroll
        for (int c = 0; c < 2; ++c) rv[b][c] = __shfl_sync(0xffffffffu, racc[c], 4 * b + t);
    }
    if (g == 0) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        ms[warp * 8 + 2 * t + c] = m_run[c];
        ls[warp * 8 + 2 * t + c] = l_run[c];
      }
    }
#pragma unroll
    for (int mt = 0; mt < 2 * C::kNB; ++mt) {
      const int b = mt >> 1, hb = mt & 1;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int lr = 2 * t + (e & 1);
        const int dim = 32 * b + 16 * hb + g + 8 * (e >> 1);
        float v = oacc[mt][e];
        if constexpr (C::kVMin) v += rv[mt >> 1][e & 1];
        os[(warp * 8 + lr) * C::kOStride + dim] = v;
      }
    }
  }
  __syncthreads();

  const bool direct = p.n_splits == 1;
  float* part_o = p.part_o + (static_cast<long long>(h) * p.n_splits + split) * C::kRowsPad * kHeadDim;
  float* part_l = p.part_lse + (static_cast<long long>(h) * p.n_splits + split) * C::kRowsPad;
  for (int idx = threadIdx.x; idx < n_rows * (kHeadDim / 4); idx += C::kThreads) {
    const int row = idx / (kHeadDim / 4);
    const int d4 = (idx % (kHeadDim / 4)) * 4;
    // the streams that hold this row: the warps of its n-tile (warp = n-tile + NT x group)
    const int lr = row % 8;
    float M = -INFINITY;
#pragma unroll
    for (int u = row / 8; u < C::kConsumerWarps; u += NT) M = fmaxf(M, ms[u * 8 + lr]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int u = row / 8; u < C::kConsumerWarps; u += NT) {
        const float w = fast_exp2(ms[u * 8 + lr] - M);
        L += w * ls[u * 8 + lr];
        const float4 o = *reinterpret_cast<const float4*>(os + (u * 8 + lr) * C::kOStride + d4);
        acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
      }
    }
    const float invL = L > 0.f ? 1.f / L : 0.f;
    acc.x *= invL; acc.y *= invL; acc.z *= invL; acc.w *= invL;
    const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
    if (direct) {
      const int qi = row / p.group, j = row % p.group;
      const long long orow = static_cast<long long>(qi) * p.n_qh + h * p.group + j;
      *reinterpret_cast<float4*>(p.out + orow * kHeadDim + d4) = acc;
      if (d4 == 0) p.lse[orow] = lse2 * 0.69314718055994531f;
    } else {
      *reinterpret_cast<float4*>(part_o + row * kHeadDim + d4) = acc;
      if (d4 == 0) part_l[row] = lse2;
    }
  }
}

// Log-sum-exp merge of the per-split partials of kvattn_decode (and kvattn_prefill_chunk),
// launched right behind the producing grid with programmatic dependent launch: its CTAs
// start while that grid drains and wait (griddepcontrol.wait) until all partials are
// written.  One CTA per (query row, KV head), 256 threads = four groups of 64 (four
// channels each); group g takes splits g, g + 4, ...  Each thread keeps an online (max, sum,
// weighted output) over its splits, loading a batch of up to 16 splits before using any of them, and
// the four groups are combined once through shared memory.  Arithmetic of kvattn_merge_lse
// (log2 units).
constexpr int kMergeThreads = 256;
constexpr int kMergeGroups = kMergeThreads / (kHeadDim / 4);
// kBatch splits are loaded ahead per thread: 16 for decode (a few dozen splits, one round
// trip), 8 with two CTAs per SM for prefill (tens of thousands of small CTAs).
template <int kBatch, int kMinBlocks>
__global__ void __launch_bounds__(kMergeThreads, kMinBlocks) decode_merge_kernel(const float* __restrict__ part_o,
                                                                     const float* __restrict__ part_lse, int n_splits,
                                                                     int rows_pad, int group, int n_qh,
                                                                     float* __restrict__ out, float* __restrict__ lse) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the next kernel may set up
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float red_m[kMergeGroups], red_l[kMergeGroups];
  __shared__ float4 red_o[kMergeGroups][kHeadDim / 4];
  const int row = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, grp = tid / (kHeadDim / 4), d4 = tid % (kHeadDim / 4);
  const float* pl = part_lse + static_cast<long long>(h) * n_splits * rows_pad + row;
  const float* po = part_o + (static_cast<long long>(h) * n_splits * rows_pad + row) * kHeadDim + d4 * 4;
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp0 = grp; sp0 < n_splits; sp0 += kMergeGroups * kBatch) {
    float v[kBatch];
    float4 o[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int sp = sp0 + k * kMergeGroups;
      v[k] = sp < n_splits ? pl[static_cast<long long>(sp) * rows_pad] : -INFINITY;
      o[k] = sp < n_splits ? *reinterpret_cast<const float4*>(po + static_cast<long long>(sp) * rows_pad * kHeadDim)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (v[k] == -INFINITY) continue;  // a split that saw no key
      if (v[k] > m) {
        const float a = fast_exp2(m - v[k]);  // 0 when m = -inf
        l *= a;
        acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
        m = v[k];
      }
      const float w = fast_exp2(v[k] - m);
      l += w;
      acc.x += w * o[k].x; acc.y += w * o[k].y; acc.z += w * o[k].z; acc.w += w * o[k].w;
    }
  }
  if (d4 == 0) {
    red_m[grp] = m;
    red_l[grp] = l;
  }
  red_o[grp][d4] = acc;
  __syncthreads();
  if (grp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int gq = 0; gq < kMergeGroups; ++gq) M = fmaxf(M, red_m[gq]);
    float L = 0.f;
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int gq = 0; gq < kMergeGroups; ++gq) {
        const float w = fast_exp2(red_m[gq] - M);  // 0 for a group that saw no key
        L += w * red_l[gq];
        const float4 o = red_o[gq][d4];
        r.x += w * o.x; r.y += w * o.y; r.z += w * o.z; r.w += w * o.w;
      }
      const float inv = 1.f / L;
      r.x *= inv; r.y *= inv; r.z *= inv; r.w *= inv;
    }
    const int qi = row / group, j = row % group;
    const long long orow = static_cast<long long>(qi) * n_qh + h * group + j;
    *reinterpret_cast<float4*>(out + orow * kHeadDim + d4 * 4) = r;
    if (d4 == 0) lse[orow] = M != -INFINITY ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

// ---------------------------------------------------------------------------------------
int decode_rows_pad(int rows) { return ((rows + 7) / 8) * 8; }

// The merge grid of a decode plan with more than one split (a no-op for one split, where the
// split grid wrote out and lse itself).
cudaError_t launch_decode_merge(const DecodeParams& prm, int n_kv, cudaStream_t stream) {
  if (prm.n_splits == 1) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(prm.group * prm.n_q, n_kv);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel<16, 1>, static_cast<const float*>(prm.part_o),
                            static_cast<const float*>(prm.part_lse), prm.n_splits,
                            decode_rows_pad(prm.group * prm.n_q), prm.group, prm.n_qh, prm.out, prm.lse);
}

template <int KF, int VF, int NT>
static cudaError_t launch_decode_t(const DecodeParams& prm, int n_kv, cudaStream_t stream) {
  using C = DecodeCfg<KF, VF, NT>;
  // programmatic dependent launch: the grid may start while the previous kernel on the
  // stream drains; the kernel waits for it (griddepcontrol.wait) before reading any input
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(prm.n_splits, n_kv);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<KF, VF, NT>, prm);
}

// The supported (key, value) format pairs: Q8_0 keys with Q4_0 or Q8_0 values, Q4_0 and Q5_1
// keys with Q4_0 or Q8_0 values, Q5_0 keys with Q4_1 values.
#define KVATTN_DECODE_PAIRS(X) \
  X(kKeyQ8, kValQ4) X(kKeyQ8, kValQ8) X(kKeyQ4, kValQ4) X(kKeyQ4, kValQ8) X(kKeyQ51, kValQ4) \
  X(kKeyQ51, kValQ8) X(kKeyQ50, kValQ41)

bool decode_pair_supported(int key_fmt, int val_fmt) {
#define KV_PAIR_OK(KF, VF) if (key_fmt == KF && val_fmt == VF) return true;
  KVATTN_DECODE_PAIRS(KV_PAIR_OK)
#undef KV_PAIR_OK
  return false;
}

cudaError_t prepare_decode_kernels() {
  cudaError_t e;
#define KV_SET1(KF, VF, NT)                                                                   \
  e = cudaFuncSetAttribute(decode_kernel<KF, VF, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           DecodeCfg<KF, VF, NT>::kSmemBytes);                               \
  if (e != cudaSuccess) return e;
#define KV_SET(KF, VF) KV_SET1(KF, VF, 1) KV_SET1(KF, VF, 2) KV_SET1(KF, VF, 3)
  KVATTN_DECODE_PAIRS(KV_SET)
#undef KV_SET
#undef KV_SET1
  return cudaSuccess;
}

template <int KF, int VF>
static cudaError_t launch_decode_fmt(const DecodeParams& prm, int n_kv, int nt, cudaStream_t stream) {
  if (nt == 1) return launch_decode_t<KF, VF, 1>(prm, n_kv, stream);
  if (nt == 2) return launch_decode_t<KF, VF, 2>(prm, n_kv, stream);
  return launch_decode_t<KF, VF, 3>(prm, n_kv, stream);
}

cudaError_t launch_decode(const DecodeParams& prm, int n_kv, int key_fmt, int val_fmt, cudaStream_t stream) {
  const int nt = decode_rows_pad(prm.group * prm.n_q) / 8;
#define KV_LAUNCH(KF, VF) \
  if (key_fmt == KF && val_fmt == VF) return launch_decode_fmt<KF, VF>(prm, n_kv, nt, stream);
  KVATTN_DECODE_PAIRS(KV_LAUNCH)
#undef KV_LAUNCH
  return cudaErrorInvalidValue;
}

}  // namespace kvattn
