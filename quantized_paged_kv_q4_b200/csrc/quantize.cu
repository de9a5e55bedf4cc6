// Q8_0 / Q4_0 / Q5_1 / Q5_0 / Q4_1 encoders that append new tokens into their KV pages.
//
// Formats (Vulkan speculative-decoding report, lcz.me/topic/1398, "pitfalls" and
// "configs"): 32-element blocks with one fp16 scale; Q8_0 stores int8 codes (8.5 bits per
// element), Q4_0 stores 4-bit codes q with value (q - 8) * d (18 bytes per block); the same
// list names q4_1, q5_0 and q5_1 as KV types.
// Encoder readings (the pages do not spell them out):
//   Q8_0: d = amax / 127, q = round-half-away(x * fp32(1/d)), |q| <= 127.
//   Q4_0: m = the signed element of largest magnitude (first on ties), d = m / -8,
//         q = min(15, floor(fp32(fp32(x * fp32(1/d)) + 8.5))).
//   Q5_0: as Q4_0 with 5-bit codes: d = m / -16, q = min(31, floor(x * fp32(1/d) + 16.5)),
//         value (q - 16) * d.
//   Q5_1 (same report, pitfalls: 5-bit codes with a zero point, 6 bits per element):
//         m = the block minimum, d = fp32(fp32(max - m) / 31),
//         q = min(31, floor(fp32(fp32(fp32(x - m) * fp32(1/d)) + 0.5))), value q * d + m.
//   Q4_1: as Q5_1 with 4-bit codes: d = (max - m) / 15, q = min(15, ...).
// Every operation that decides a code is an IEEE fp32 operation with round-to-nearest
// (no FMA contraction), so the codes equal those of any correct fp32 implementation.
//
// One warp encodes one (token, KV head) row: lane l owns channels [8l, 8l+8), four lanes
// form one 32-element block.  Keys are stored as Q8_0, Q4_0, Q5_1 or Q5_0, values as Q4_0,
// Q8_0 or Q4_1.
#include "decode.cuh"

namespace kvattn {

__device__ __forceinline__ int q8_code(float x, float inv) {
  const float y = __fmul_rn(x, inv);
  float r = roundf(y);  // halves away from zero
  r = fminf(fmaxf(r, -127.f), 127.f);
  return static_cast<int>(r);
}

// Offset codes: min(2 half - 1, floor(fp32(fp32(x * inv) + half + 0.5))) (half = 8: Q4_0, 16: Q5_0).
template <int HALF>
__device__ __forceinline__ int offset_code(float x, float inv) {
  const float y = __fmul_rn(x, inv);
  const float z = __fadd_rn(y, HALF + 0.5f);
  return min(2 * HALF - 1, __float2int_rz(z));  // z > 0, so truncation is floor
}
__device__ __forceinline__ int q4_code(float x, float inv) { return offset_code<8>(x, inv); }

// Q8_0 block scale of this lane's block: returns d (fp32) and writes 1/d to *inv.
__device__ __forceinline__ float q8_scale(const float (&x)[8], float* inv) {
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  const float d = __fdiv_rn(a, 127.f);
  *inv = d != 0.f ? __frcp_rn(d) : 0.f;
  return d;
}

// Offset-format block scale of this lane's block: the signed element of largest magnitude,
// first index on ties, over the four lanes of the block; returns d = m / -half (fp32) and
// writes 1/d to *inv (half = 8: Q4_0, 16: Q5_0).
template <int HALF>
__device__ __forceinline__ float offset_scale(const float (&x)[8], int lane, float* inv) {
  float best = x[0];
  int bidx = lane * 8;
#pragma unroll
  for (int e = 1; e < 8; ++e)
    if (fabsf(x[e]) > fabsf(best)) {
      best = x[e];
      bidx = lane * 8 + e;
    }
#pragma unroll
  for (int s = 1; s <= 2; s <<= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, s);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, s);
    if (fabsf(ob) > fabsf(best) || (fabsf(ob) == fabsf(best) && oi < bidx)) {
      best = ob;
      bidx = oi;
    }
  }
  const float d = __fdiv_rn(best, -static_cast<float>(HALF));
  *inv = d != 0.f ? __frcp_rn(d) : 0.f;
  return d;
}
__device__ __forceinline__ float q4_scale(const float (&x)[8], int lane, float* inv) {
  return offset_scale<8>(x, lane, inv);
}

// Zero-point block scale of this lane's block (TOP = 31: Q5_1, 15: Q4_1): writes the block
// minimum to *mn and 1/d to *inv, returns d = fp32(fp32(max - min) / TOP).
template <int TOP>
__device__ __forceinline__ float min_scale(const float (&x)[8], float* mn_out, float* inv) {
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int e = 1; e < 8; ++e) {
    mn = fminf(mn, x[e]);
    mx = fmaxf(mx, x[e]);
  }
#pragma unroll
  for (int s = 1; s <= 2; s <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, s));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, s));
  }
  const float d = __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(TOP));
  *inv = d != 0.f ? __frcp_rn(d) : 0.f;
  *mn_out = mn;
  return d;
}

template <int TOP>
__device__ __forceinline__ int min_code(float x, float mn, float inv) {
  const float y = __fmul_rn(__fsub_rn(x, mn), inv);
  return min(TOP, __float2int_rz(__fadd_rn(y, 0.5f)));  // y >= 0, so truncation is floor
}


// Encodes one token of one KV head into slot `tok` of its K page (kpg) and V page (vpg), in
// any memory space (global pages, or a page's copy in shared memory).  The 32 lanes of the
// calling warp each hold 8 channels: kx / vx are channels 8 lane .. 8 lane + 7 of K and V.
// Every lane takes part in the shuffles; only lanes whose bit is set in store_mask write, so
// a warp may write just its own 32-channel blocks (lanes 4b .. 4b + 3 hold block b).
__device__ __forceinline__ void encode_token(const float (&kx)[8], const float (&vx)[8], int lane, uint8_t* kpg,
                                             uint8_t* vpg, int tok, int k_fmt, int v_fmt, uint32_t store_mask) {
  const bool st = (store_mask >> lane) & 1u;
  const int G = tok >> 4, tl = tok & 15, H = tl >> 3, R = tok & 7;
  const int b = lane >> 2;  // this lane's block

  // ---------------- K: Q5_1 / Q5_0 ----------------
  if (k_fmt == kKeyQ51 || k_fmt == kKeyQ50) {
    const float (&x)[8] = kx;
    float mn = 0.f, inv, d;
    if (k_fmt == kKeyQ51) {
      d = min_scale<31>(x, &mn, &inv);
    } else {
      d = offset_scale<16>(x, lane, &inv);
    }
    const int T = lane & 3, c = b & 3, Q = b >> 2;
    // low nibbles as the Q4_0 key word; fifth bits of the four blocks 4Q..4Q+3 of this T
    // (lanes T + 4c + 16Q) gathered into one word, channel (c, e) at bit 16(e%2) + 4c + e/2
    uint32_t w = 0, hb = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t q = static_cast<uint32_t>(k_fmt == kKeyQ51 ? min_code<31>(x[e], mn, inv)
                                                                : offset_code<16>(x[e], inv));
      w |= (q & 15u) << (4 * (e >> 1) + 16 * (e & 1));
      hb |= (q >> 4) << (16 * (e & 1) + 4 * c + (e >> 1));
    }
    hb |= __shfl_xor_sync(0xffffffffu, hb, 4);
    hb |= __shfl_xor_sync(0xffffffffu, hb, 8);
    uint8_t* pg = kpg;
    const int row = (((G * 2 + Q) * 2 + H) * 8 + R) * 4 + T;
    if (st) *reinterpret_cast<uint32_t*>(pg + 4 * (row * 4 + c)) = w;
    if (st && c == 0) *reinterpret_cast<uint32_t*>(pg + kK5HighOffset + 4 * row) = hb;
    if (st && (lane & 3) == 0) {
      const int si = 2 * (((G * 8 + R) * 2 + H) * 8 + b);
      *reinterpret_cast<__half*>(pg + kK5ScaleOffset + si) = __float2half_rn(d);
      if (k_fmt == kKeyQ51) *reinterpret_cast<__half*>(pg + kK5MinOffset + si) = __float2half_rn(mn);
    }
  }
  // ---------------- K: Q4_0 ----------------
  else if (k_fmt == kKeyQ4) {
    const float (&x)[8] = kx;
    float inv;
    const float d = q4_scale(x, lane, &inv);
    // one 32-bit word per lane: channel 8T + e at bit 4 * (e / 2) + 16 * (e % 2)
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) w |= static_cast<uint32_t>(q4_code(x[e], inv)) << (4 * (e >> 1) + 16 * (e & 1));
    uint8_t* pg = kpg;
    const int T = lane & 3;
    const int word = ((((G * 2 + (b >> 2)) * 2 + H) * 8 + R) * 4 + T) * 4 + (b & 3);
    if (st) *reinterpret_cast<uint32_t*>(pg + 4 * word) = w;
    if (st && (lane & 3) == 0) {
      const int so = kK4ScaleOffset + 2 * (((G * 8 + R) * 2 + H) * 8 + b);
      *reinterpret_cast<__half*>(pg + so) = __float2half_rn(d);
    }
  }
  // ---------------- K: Q8_0 ----------------
  else {
    const float (&x)[8] = kx;
    float inv;
    const float d = q8_scale(x, &inv);
    // codes are stored offset-binary: the byte q + 128
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) w0 |= static_cast<uint32_t>(q8_code(x[e], inv) + 128) << (8 * e);
#pragma unroll
    for (int e = 0; e < 4; ++e) w1 |= static_cast<uint32_t>(q8_code(x[4 + e], inv) + 128) << (8 * e);
    uint8_t* pg = kpg;
    const int P = lane >> 3, T = lane & 3, jhi = (lane & 7) >> 2;
    const int off = ((((G * 4 + P) * 2 + H) * 8 + R) * 4 + T) * 16 + 8 * jhi;
    if (st) *reinterpret_cast<uint2*>(pg + off) = make_uint2(w0, w1);
    if (st && (lane & 3) == 0) {
      const int so = kKScaleOffset + 2 * (((G * 8 + R) * 2 + H) * 8 + b);
      *reinterpret_cast<__half*>(pg + so) = __float2half_rn(d);
    }
  }

  // ---------------- V: Q4_0, Q4_1 or Q8_0 ----------------
  {
    const float (&x)[8] = vx;
    uint8_t* pg = vpg;
    const int T = (tl & 7) >> 1, wlo = tl >> 3, ylo = tl & 1;
    const int k_slot = ylo + 2 * wlo;
    const int cl = lane & 3;  // which 8-channel group of the block
    float d;
    int codes[8];
    if (v_fmt != kValQ8) {
      float inv, mn = 0.f;
      if (v_fmt == kValQ41) {
        d = min_scale<15>(x, &mn, &inv);
#pragma unroll
        for (int e = 0; e < 8; ++e) codes[e] = min_code<15>(x[e], mn, inv);
      } else {
        d = q4_scale(x, lane, &inv);
#pragma unroll
        for (int e = 0; e < 8; ++e) codes[e] = q4_code(x[e], inv);
      }
      // lanes cl = 0,1 share bytes (lo, hi nibble) with y%2 = 0; lanes 2,3 with y%2 = 1
      int other[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) other[e] = __shfl_xor_sync(0xffffffffu, codes[e], 1);
      if (st && (cl & 1) == 0) {
        const int C = b >> 1, w = 2 * (b & 1) + wlo, y = 2 * ylo + (cl >> 1);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int off = ((((G * 4 + C) * 8 + e) * 4 + T) * 16) + 4 * w + y;
          pg[off] = static_cast<uint8_t>(codes[e] | (other[e] << 4));
        }
      }
      if (st && cl == 0) {
        const int so = kV4ScaleOffset + 2 * (((G * 4 + T) * 8 + b) * 4 + k_slot);
        *reinterpret_cast<__half*>(pg + so) = __float2half_rn(d);
        if (v_fmt == kValQ41)
          *reinterpret_cast<__half*>(pg + so + (kV41MinOffset - kV4ScaleOffset)) = __float2half_rn(mn);
      }
    } else {
      float inv;
      d = q8_scale(x, &inv);
#pragma unroll
      for (int e = 0; e < 8; ++e) codes[e] = q8_code(x[e], inv);
      const int w = 2 * (cl >> 1) + wlo, y = 2 * (cl & 1) + ylo;
      if (st) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int off = ((((G * 8 + b) * 8 + e) * 4 + T) * 16) + 4 * w + y;
          pg[off] = static_cast<uint8_t>(codes[e] + 128);  // offset-binary, as the K codes
        }
      }
      if (st && cl == 0) {
        const int so = kV8ScaleOffset + 2 * (((G * 4 + T) * 8 + b) * 4 + k_slot);
        *reinterpret_cast<__half*>(pg + so) = __float2half_rn(d);
      }
    }
  }
}

__global__ void __launch_bounds__(256) quantize_append_kernel(const float* __restrict__ k,
                                                              const float* __restrict__ v, int n_tok,
                                                              int n_kv, int32_t pos0,
                                                              const int32_t* __restrict__ page_table,
                                                              int n_blocks, uint8_t* k_pool, int64_t k_stride,
                                                              uint8_t* v_pool, int64_t v_stride, int64_t n_pages,
                                                              int k_fmt, int v_fmt) {
  // a kernel launched behind this one with programmatic dependent launch (decode) may start
  // its setup now; it waits for this grid to complete before reading the pages
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // this grid is itself launched that way: wait for the previous kernel before any read
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(n_tok) * n_kv) return;
  const int i = static_cast<int>(row / n_kv);
  const int h = static_cast<int>(row % n_kv);
  const int32_t pos = pos0 + i;
  const int blk = pos / kPageTokens;
  const int tok = pos % kPageTokens;
  // all global reads are issued before any of them is used
  const float4* ksrc = reinterpret_cast<const float4*>(k + row * kHeadDim + lane * 8);
  const float4* vsrc = reinterpret_cast<const float4*>(v + row * kHeadDim + lane * 8);
  const float4 kx0 = ksrc[0], kx1 = ksrc[1], vx0 = vsrc[0], vx1 = vsrc[1];
  const int page = page_table[static_cast<long long>(h) * n_blocks + blk];
  if (page < 0 || page >= n_pages) {
    if (lane == 0) record_error(KVATTN_ERR_BAD_PAGE);
    return;
  }
  const float kx[8] = {kx0.x, kx0.y, kx0.z, kx0.w, kx1.x, kx1.y, kx1.z, kx1.w};
  const float vx[8] = {vx0.x, vx0.y, vx0.z, vx0.w, vx1.x, vx1.y, vx1.z, vx1.w};
  encode_token(kx, vx, lane, k_pool + static_cast<int64_t>(page) * k_stride, v_pool + static_cast<int64_t>(page) * v_stride,
               tok, k_fmt, v_fmt, 0xffffffffu);
}

cudaError_t launch_quantize_append(const kvattn_kv_desc& desc, const float* k, const float* v, int n_tok,
                                   int32_t pos0, const int32_t* page_table, int n_blocks, cudaStream_t stream) {
  const long long rows = static_cast<long long>(n_tok) * desc.n_kv_heads;
  const int warps_per_block = 8;
  const long long grid = (rows + warps_per_block - 1) / warps_per_block;
  // programmatic dependent launch: the grid may start while the previous kernel finishes;
  // it waits for it (griddepcontrol.wait) before reading anything
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(32 * warps_per_block);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_append_kernel, k, v, n_tok, desc.n_kv_heads, pos0, page_table, n_blocks,
                            static_cast<uint8_t*>(desc.k_pool), desc.k_page_stride,
                            static_cast<uint8_t*>(desc.v_pool), desc.v_page_stride, desc.n_pages,
                            key_format_id(desc.k_fmt), value_format_id(desc.v_fmt));
}

}  // namespace kvattn
