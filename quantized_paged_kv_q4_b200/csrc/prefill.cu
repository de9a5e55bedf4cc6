// Chunked prefill over Q8_0 K / Q4_0 V pages on tcgen05 tensor cores (Adaptive KV
// Streaming + RDNA 4 announcement, wqu.guru, method list: "online log-sum-exp prefill":
// the prefill of a chunk is computed across streamed KV pages and the partial results are
// accumulated by online log-sum-exp).
//
// Work unit (one CTA): a KV head h, an M-tile of 128 query rows of that head's group
// (row r = token t * group + j: all query heads of a group share the K/V tiles, so each
// dequantized tile serves 128 rows), and one KV split of kv_split_tokens keys.  The split
// is walked in 64-key tiles (half pages):
//
//   dequant warps (8)   raw Q8_0 K / Q4_0 V from global -> f16 in shared memory, block
//                       scales folded in (one f16 rounding):  K^ [64 keys][256] and
//                       V^T [256 dims][64 keys], both K-major, 128-byte swizzle
//   MMA warp (1 thread) S = Q K^T      (M = 128 rows, N = 64 keys, K = 256)  -> TMEM
//                       O^T += V^T P^T (M = 128 dims x 2, N = 128 rows, K = 64 keys) -> TMEM
//   softmax warps (4)   thread = query row: S from TMEM, causal mask, running max (the
//                       accumulators are rescaled only when the max grows by > 2^8),
//                       P = exp2(S - m) as f16 into shared memory
//
// Q (bf16) is converted to f16 and pre-scaled by log2(e)/16 so S is a base-2 score.  The
// CTA writes a normalised partial (o, lse) per row; a second grid merges the splits.
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
constexpr int kSoftmaxWarps = 4;   // warps 0-3: TMEM lane quarters 0-3
constexpr int kMmaWarp = 4;
constexpr int kDequantWarps = 8;   // warps 5-12
constexpr int kThreads = (kSoftmaxWarps + 1 + kDequantWarps) * 32;
constexpr int kDq0 = (kSoftmaxWarps + 1) * 32;  // first dequant thread
// shared memory map (bytes)
constexpr int kQOff = 0;                        // 4 atoms x [128 rows][128 B]
constexpr int kKOff = 65536;                    // 2 buffers x 4 atoms x [64 keys][128 B]
constexpr int kVOff = kKOff + 2 * 32768;        // 2 buffers x [256 dims][128 B]
constexpr int kPOff = kVOff + 2 * 32768;        // 2 buffers x [128 rows][128 B]
constexpr int kMiscOff = kPOff + 2 * 16384;     // barriers, TMEM base, row stats
constexpr int kSmemBytes = kMiscOff + 3072;   // = 227 KB, the per-CTA maximum
// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol0 = 0;     // S buffers: [0,64), [64,128)
constexpr uint32_t kOCol0 = 128;   // O^T dims 0-127: [128,256); dims 128-255: [256,384)
constexpr uint32_t kIdescQK = tc::idesc_f16(128, kKeys, 0, 0);
constexpr uint32_t kIdescPV = tc::idesc_f16(128, kRows, 0, 0);
}  // namespace pf

struct PfTile {
  int page, logical, half;
};

// The CTA's i-th candidate tile (2 per listed page); false if the tile holds no key that
// any row of the M-tile may see, or its page id is invalid.  Every role evaluates the same
// predicate, so all agree on the tile sequence.
__device__ __forceinline__ bool pf_tile(const PrefillParams& p, int h, int ks, int i, int np, int max_qpos,
                                        PfTile* tile) {
  const int idx = ks * p.pages_per_split + (i >> 1);
  if (idx >= np) return false;
  const long long li = static_cast<long long>(h) * p.max_pages + idx;
  const int page = p.page_list[li];
  const int logical = p.page_logical ? p.page_logical[li] : idx;
  const int half = i & 1;
  if (static_cast<long long>(logical) * kPageTokens + half * pf::kKeys > max_qpos) return false;
  if (page < 0 || page >= p.n_pages) return false;
  tile->page = page;
  tile->logical = logical;
  tile->half = half;
  return true;
}

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
  return row * 128 + ((chunk ^ (row & 7)) << 4);
}

__global__ void __launch_bounds__(pf::kThreads, 1) prefill_kernel(const PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + pf::kMiscOff);
  uint64_t* kready = bars + 0;   // [2] dequant -> MMA
  uint64_t* vready = bars + 2;   // [2]
  uint64_t* kfree = bars + 4;    // [2] MMA (QK done) -> dequant
  uint64_t* vfree = bars + 6;    // [2] MMA (PV done) -> dequant, softmax
  uint64_t* sready = bars + 8;   // [2] MMA -> softmax
  uint64_t* pready = bars + 10;  // [2] softmax -> MMA
  uint64_t* ofinal = bars + 12;  // MMA -> softmax (epilogue)
  uint64_t* wgbar = bars + 13;   // softmax warpgroup rendezvous
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(bars + 16);
  int* s_abort = reinterpret_cast<int*>(tmem_base_s + 1);
  int* s_any = s_abort + 1;                              // [2][4] per tile parity and softmax warp
  float* s_alpha = reinterpret_cast<float*>(s_any + 8);  // [2][128]
  float* s_l = s_alpha + 2 * pf::kRows;                  // [128]
  float* s_m = s_l + pf::kRows;                          // [128] (ends before kMiscOff + 2232)

  const int mt = blockIdx.x, ks = blockIdx.y, h = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rows = p.n_q * p.group;
  const int row0 = mt * pf::kRows;
  int np = p.max_pages;
  if (p.n_pages_arr) np = min(max(p.n_pages_arr[h], 0), p.max_pages);
  // largest query position among this M-tile's rows: keys beyond it are never visible
  int max_qpos = INT_MIN;
  {
    const int t0 = row0 / p.group, t1 = min(n_rows - 1, row0 + pf::kRows - 1) / p.group;
    for (int t = t0; t <= t1; ++t) max_qpos = max(max_qpos, p.q_pos[t]);
  }
  const int n_cand = 2 * p.pages_per_split;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&kready[b], pf::kDequantWarps);
      mbar_init(&vready[b], pf::kDequantWarps);
      mbar_init(&kfree[b], 1);
      mbar_init(&vfree[b], 1);
      mbar_init(&sready[b], 1);
      mbar_init(&pready[b], pf::kSoftmaxWarps);
    }
    mbar_init(ofinal, 1);
    mbar_init(wgbar, pf::kSoftmaxWarps);
    *s_abort = 0;
    if (smem_u32(smem) & 1023) record_error(KVATTN_ERR_INVALID_ARG);
    fence_barrier_init();
  }
  if (warp == pf::kMmaWarp) {
    tc::tmem_alloc(tmem_base_s, pf::kTmemCols);
    tc::tmem_relinquish();
  }
  // ---- Q tile: bf16 -> f16 * log2(e)/16, swizzled K-major (dequant warps) ----
  if (threadIdx.x >= pf::kDq0) {
    const int d = threadIdx.x - pf::kDq0;  // 0..255
    const int r = d >> 1, hq = d & 1;       // row, which 128 channels
    const int R = row0 + r;
    const uint16_t* src = nullptr;
    if (R < n_rows) {
      const int t = R / p.group, j = R % p.group;
      src = p.q + (static_cast<long long>(t) * p.n_qh + h * p.group + j) * kHeadDim + hq * 128;
    }
    const float sc = 1.4426950408889634f / 16.0f;
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {  // 16 chunks of 8 channels
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (src) raw = *reinterpret_cast<const uint4*>(src + c * 8);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(w[e] << 16) * sc;
        const float hi = __uint_as_float(w[e] & 0xFFFF0000u) * sc;
        o[e] = pack_half2(lo, hi);
      }
      const int chan = hq * 128 + c * 8;
      const int atom = chan >> 6, chunk = (chan & 63) >> 3;
      uint4* dst = reinterpret_cast<uint4*>(smem + pf::kQOff + atom * 16384 + swz(r, chunk));
      *dst = make_uint4(o[0], o[1], o[2], o[3]);
    }
    tc::fence_proxy_async_smem();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_base_s;

  if (warp == pf::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + pf::kQOff);
      const uint32_t k_base = smem_u32(smem + pf::kKOff);
      const uint32_t v_base = smem_u32(smem + pf::kVOff);
      const uint32_t p_base = smem_u32(smem + pf::kPOff);
      int j = 0;  // valid tiles issued (QK)
      auto issue_pv = [&](int jj) -> bool {
        const int b = jj & 1;
        const uint32_t par = (jj >> 1) & 1;
        if (!mbar_wait(&pready[b], par) || !mbar_wait(&vready[b], par)) return false;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < pf::kKeys / 16; ++kk) {
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint64_t ad = tc::sw128_desc(v_base + b * 32768 + a * 16384 + kk * 32, 1024, 16);
            const uint64_t bd = tc::sw128_desc(p_base + b * 16384 + kk * 32, 1024, 16);
            tc::mma_f16_ss(tmem + pf::kOCol0 + a * 128, ad, bd, pf::kIdescPV, (jj > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::commit(&vfree[b]);
        return true;
      };
      bool ok = true;
      for (int i = 0; i < n_cand && ok; ++i) {
        PfTile tl;
        if (!pf_tile(p, h, ks, i, np, max_qpos, &tl)) continue;
        const int b = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&kready[b], par)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(q_base + (kk >> 2) * 16384 + (kk & 3) * 32, 1024, 16);
          const uint64_t bd = tc::sw128_desc(k_base + b * 32768 + (kk >> 2) * 8192 + (kk & 3) * 32, 1024, 16);
          tc::mma_f16_ss(tmem + pf::kSCol0 + b * pf::kKeys, ad, bd, pf::kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc::commit(&sready[b]);
        tc::commit(&kfree[b]);
        if (j >= 1) ok = issue_pv(j - 1);
        ++j;
      }
      if (ok && j >= 1) ok = issue_pv(j - 1);
      if (!ok) *s_abort = 1;
      tc::commit(ofinal);  // arrives when every MMA above has completed
      mbar_wait(ofinal, 0);  // no MMA may still run when the tensor memory is freed
    }
  } else if (warp < pf::kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax (thread = row)
    const int r = threadIdx.x;  // 0..127 == TMEM lane
    const int R = row0 + r;
    const int qpos = R < n_rows ? p.q_pos[R / p.group] : INT_MAX;
    const uint32_t lane_base = tmem + ((static_cast<uint32_t>(warp) * 32) << 16);
    float m_ref = -INFINITY, l_sum = 0.f;
    uint32_t wg_phase = 0;
    int j = 0;
    bool ok = true;
    for (int i = 0; i < n_cand && ok; ++i) {
      PfTile tl;
      if (!pf_tile(p, h, ks, i, np, max_qpos, &tl)) continue;
      const int b = j & 1;
      const uint32_t par = (j >> 1) & 1;
      if (!mbar_wait(&sready[b], par)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float s[pf::kKeys];
      {
        uint32_t v[32];
        tc::ld32(lane_base + pf::kSCol0 + b * pf::kKeys, v);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(v[c]);
        tc::ld32(lane_base + pf::kSCol0 + b * pf::kKeys + 32, v);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(v[c]);
      }
      const int key0 = tl.logical * kPageTokens + tl.half * pf::kKeys;
      if (key0 + pf::kKeys - 1 > qpos) {
#pragma unroll
        for (int c = 0; c < pf::kKeys; ++c)
          if (key0 + c > qpos) s[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < pf::kKeys; ++c) mx = fmaxf(mx, s[c]);
      float alpha = 1.f;
      bool resc = false;
      if (mx > m_ref + 8.f) {
        alpha = fast_exp2(m_ref - mx);  // 0 when m_ref = -inf
        resc = j > 0 && m_ref != -INFINITY;
        l_sum *= alpha;
        m_ref = mx;
      }
      // rescale O^T columns of the rows whose maximum jumped (rare)
      // (double-buffered by tile parity: a warp can run at most one rendezvous ahead)
      int* any_b = s_any + 4 * b;
      float* alpha_b = s_alpha + pf::kRows * b;
      const unsigned any = __ballot_sync(0xffffffffu, resc);
      if (lane == 0) any_b[warp] = any != 0;
      alpha_b[r] = resc ? alpha : 1.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(wgbar);
      if (!mbar_wait(wgbar, wg_phase)) {
        ok = false;
        break;
      }
      wg_phase ^= 1;
      if (any_b[0] | any_b[1] | any_b[2] | any_b[3]) {
        // O^T must hold the previous tile's PV before it is rescaled
        if (!mbar_wait(&vfree[(j - 1) & 1], ((j - 1) >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        for (int a = 0; a < 2; ++a) {
          for (int c0 = 0; c0 < pf::kRows; c0 += 32) {
            uint32_t v[32];
            tc::ld32(lane_base + pf::kOCol0 + a * 128 + c0, v);
            tc::wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * alpha_b[c0 + c]);
            tc::st32(lane_base + pf::kOCol0 + a * 128 + c0, v);
          }
        }
        tc::wait_st();
      }
      const float mu = m_ref == -INFINITY ? 0.f : m_ref;
      // P buffer b was last read by the PV of tile j-2
      if (j >= 2 && !mbar_wait(&vfree[b], ((j - 2) >> 1) & 1)) {
        ok = false;
        break;
      }
      uint8_t* prow = smem + pf::kPOff + b * 16384;
#pragma unroll
      for (int c8 = 0; c8 < pf::kKeys / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = fast_exp2(s[c8 * 8 + 2 * e] - mu);
          const float p1 = fast_exp2(s[c8 * 8 + 2 * e + 1] - mu);
          l_sum += p0 + p1;
          w[e] = pack_half2(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + swz(r, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[b]);
      ++j;
    }
    if (!ok) *s_abort = 1;
    // ---- epilogue: normalised partial (o, lse) of every row of the tile ----
    s_l[r] = l_sum;
    s_m[r] = m_ref;
    __syncwarp();
    if (lane == 0) mbar_arrive(wgbar);
    const bool ok2 = mbar_wait(wgbar, wg_phase);
    wg_phase ^= 1;
    bool have = false;
    if (ok && ok2 && j > 0) {
      have = mbar_wait(ofinal, 0);
      ok = have;
    }
    if (!ok || !ok2) *s_abort = 1;
    tc::fence_after_sync();
    const bool direct = p.n_ks == 1;
    for (int a = 0; a < 2; ++a) {
      const int dim = a * 128 + r;
      for (int c0 = 0; c0 < pf::kRows; c0 += 32) {
        uint32_t v[32];
        if (have) {
          tc::ld32(lane_base + pf::kOCol0 + a * 128 + c0, v);
          tc::wait_ld();
        }
#pragma unroll 4
        for (int c = 0; c < 32; ++c) {
          const int rr = c0 + c, RR = row0 + rr;
          if (RR >= n_rows) break;
          const float lr = s_l[rr];
          const float o = (have && lr > 0.f) ? __uint_as_float(v[c]) / lr : 0.f;
          if (direct) {
            const int t = RR / p.group, jj = RR % p.group;
            p.out[(static_cast<long long>(t) * p.n_qh + h * p.group + jj) * kHeadDim + dim] = o;
          } else {
            p.part_o[((static_cast<long long>(h) * p.n_ks + ks) * p.rows_pad + RR) * kHeadDim + dim] = o;
          }
        }
      }
    }
    if (R < n_rows) {
      const float l2 = (have && l_sum > 0.f) ? m_ref + log2f(l_sum) : -INFINITY;
      if (direct) {
        const int t = R / p.group, jj = R % p.group;
        p.lse[static_cast<long long>(t) * p.n_qh + h * p.group + jj] = l2 * 0.69314718055994531f;
      } else {
        p.part_lse[(static_cast<long long>(h) * p.n_ks + ks) * p.rows_pad + R] = l2;
      }
    }
  } else if (warp > pf::kMmaWarp) {
    // ------------------------------------------------------------ dequant (256 threads)
    const int d = threadIdx.x - pf::kDq0;
    // K task: key n of the tile, channel quarter P (blocks 2P, 2P+1)
    const int kn = d >> 2, kP = d & 3;
    // V task: 16-key group G', block pair C, row R (channels R + 8k of both blocks), half h8
    const int vG = d >> 6, vC = (d >> 4) & 3, vR = (d >> 1) & 7, vh = d & 1;
    int j = 0;
    bool ok = true;
    for (int i = 0; i < n_cand && ok; ++i) {
      PfTile tl;
      if (!pf_tile(p, h, ks, i, np, max_qpos, &tl)) continue;
      const int b = j & 1;
      const uint8_t* kp = p.k_pool + static_cast<int64_t>(tl.page) * p.k_stride;
      const uint8_t* vp = p.v_pool + static_cast<int64_t>(tl.page) * p.v_stride;
      // ---------------- K^ ----------------
      {
        const int tok = tl.half * pf::kKeys + kn;
        const int G = tok >> 4, H = (tok >> 3) & 1, R = tok & 7;
        const uint4* src = reinterpret_cast<const uint4*>(kp + ((((G * 4 + kP) * 2 + H) * 8 + R) * 4) * 16);
        uint4 raw[4];
#pragma unroll
        for (int T = 0; T < 4; ++T) raw[T] = src[T];
        const uint32_t dkw = *reinterpret_cast<const uint32_t*>(kp + kKScaleOffset + 2 * (((G * 8 + R) * 2 + H) * 8 + 2 * kP));
        const uint32_t dlo = prmt(dkw, 0u, 0x1010u), dhi = prmt(dkw, 0u, 0x3232u);
        if (j >= 2 && !mbar_wait(&kfree[b], ((j - 2) >> 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* katom = smem + pf::kKOff + b * 32768 + kP * 8192;
#pragma unroll
        for (int T = 0; T < 4; ++T) {
          const uint32_t w[4] = {raw[T].x ^ 0x80808080u, raw[T].y ^ 0x80808080u, raw[T].z ^ 0x80808080u,
                                 raw[T].w ^ 0x80808080u};
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t sc = e < 2 ? dlo : dhi;
            o[2 * e] = hmul2(hsub2(prmt(w[e], 0x64646464u, 0x4140u), 0x64806480u), sc);
            o[2 * e + 1] = hmul2(hsub2(prmt(w[e], 0x64646464u, 0x4342u), 0x64806480u), sc);
          }
          *reinterpret_cast<uint4*>(katom + swz(kn, T)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(katom + swz(kn, 4 + T)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&kready[b]);
      }
      // ---------------- V^T ----------------
      {
        const int G = tl.half * 4 + vG;  // 16-token group inside the page
        const uint4* src = reinterpret_cast<const uint4*>(vp + ((((G * 4 + vC) * 8 + vR) * 4) * 16));
        uint4 raw[4], dvr[4];
#pragma unroll
        for (int T = 0; T < 4; ++T) {
          raw[T] = src[T];
          dvr[T] = *reinterpret_cast<const uint4*>(vp + kV4ScaleOffset + 2 * (((G * 4 + T) * 8 + 2 * vC) * 4));
        }
        if (j >= 2 && !mbar_wait(&vfree[b], ((j - 2) >> 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* vt = smem + pf::kVOff + b * 32768;
#pragma unroll
        for (int e = 0; e < 2; ++e) {  // block 2C + e
          uint32_t o[4][4];            // [k][T]
#pragma unroll
          for (int T = 0; T < 4; ++T) {
            const uint32_t W = e ? (vh ? raw[T].w : raw[T].z) : (vh ? raw[T].y : raw[T].x);
            const uint32_t dv = e ? (vh ? dvr[T].w : dvr[T].z) : (vh ? dvr[T].y : dvr[T].x);
            const uint32_t Ws = W >> 8;
            o[0][T] = hmul2(hsub2(and_or(W, 0x000F000Fu, 0x64006400u), 0x64086408u), dv);
            o[1][T] = hmul2(hfma2(and_or(W, 0x00F000F0u, 0x64006400u), 0x2C002C00u, 0xD480D480u), dv);
            o[2][T] = hmul2(hsub2(and_or(Ws, 0x000F000Fu, 0x64006400u), 0x64086408u), dv);
            o[3][T] = hmul2(hfma2(and_or(Ws, 0x00F000F0u, 0x64006400u), 0x2C002C00u, 0xD480D480u), dv);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int dim = 32 * (2 * vC + e) + 8 * k + vR;
            *reinterpret_cast<uint4*>(vt + swz(dim, 2 * vG + vh)) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
          }
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&vready[b]);
      }
      ++j;
    }
    if (!ok) *s_abort = 1;
  }

  tc::fence_before_sync();
  __syncthreads();
  if (*s_abort) record_error(KVATTN_ERR_TIMEOUT);
  if (warp == pf::kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, pf::kTmemCols);
  }
}

cudaError_t prepare_prefill_kernels() {
  return cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pf::kSmemBytes);
}

struct PrefillPlan {
  int n_mt, n_ks, pps, rows_pad;
  size_t lse_off, o_off, bytes;
};

PrefillPlan plan_prefill(int n_kv, int group, int n_q, int max_pages, int kv_split_tokens) {
  PrefillPlan pl{};
  const int rows = n_q * group;
  pl.n_mt = (rows + pf::kRows - 1) / pf::kRows;
  pl.rows_pad = pl.n_mt * pf::kRows;
  pl.pps = kv_split_tokens / kPageTokens;
  pl.n_ks = max_pages > 0 ? (max_pages + pl.pps - 1) / pl.pps : 1;
  pl.lse_off = 0;
  pl.o_off = ((sizeof(float) * static_cast<size_t>(n_kv) * pl.n_ks * pl.rows_pad + 255) / 256) * 256;
  pl.bytes = pl.n_ks > 1 ? pl.o_off + sizeof(float) * static_cast<size_t>(n_kv) * pl.n_ks * pl.rows_pad * kHeadDim : 0;
  return pl;
}

cudaError_t launch_prefill(const PrefillParams& prm0, int n_kv, cudaStream_t stream) {
  PrefillParams prm = prm0;
  const int rows = prm.n_q * prm.group;
  dim3 grid((rows + pf::kRows - 1) / pf::kRows, prm.n_ks, n_kv);
  prefill_kernel<<<grid, pf::kThreads, pf::kSmemBytes, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || prm.n_ks == 1) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, n_kv);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel, static_cast<const float*>(prm.part_o),
                            static_cast<const float*>(prm.part_lse), prm.n_ks, prm.rows_pad, prm.group, prm.n_qh,
                            prm.out, prm.lse);
}

}  // namespace kvattn
