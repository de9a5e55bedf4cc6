// Log-sum-exp merge of partial attention results computed over disjoint key sets
// (Adaptive KV Streaming + RDNA 4 announcement, wqu.guru, method list: chunked prefill
// across streamed pages accumulated by online log-sum-exp):
//   lse = ln sum_p exp(lse_p),   out = sum_p exp(lse_p - lse) * o_p,
// parts with lse_p = -inf (no visible key) contribute nothing; if every part is empty the
// row is out = 0, lse = -inf.
//
// One warp per row: lanes stride over the row in float4 chunks, so every load of o_p is a
// coalesced 512-byte access; the per-row weights are computed once per warp.
#include "common.cuh"

namespace kvattn {

__global__ void __launch_bounds__(256) merge_lse_kernel(const float* __restrict__ o_parts,
                                                        const float* __restrict__ lse_parts, int n_parts,
                                                        int rows, int dim, float* __restrict__ out,
                                                        float* __restrict__ lse, int lse_log2) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const float kLn2 = 0.69314718055994531f;
  const float kLog2e = 1.4426950408889634f;
  // maximum and normaliser in base 2
  float M = -INFINITY;
  for (int p = lane; p < n_parts; p += 32) {
    float v = lse_parts[static_cast<long long>(p) * rows + row];
    if (!lse_log2) v *= kLog2e;
    M = fmaxf(M, v);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
  float L = 0.f;
  if (M != -INFINITY) {
    for (int p = lane; p < n_parts; p += 32) {
      float v = lse_parts[static_cast<long long>(p) * rows + row];
      if (!lse_log2) v *= kLog2e;
      L += exp2f(v - M);
    }
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) L += __shfl_xor_sync(0xffffffffu, L, s);
  const float invL = (M != -INFINITY && L > 0.f) ? 1.f / L : 0.f;
  for (int d = lane * 4; d < dim; d += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int p = 0; p < n_parts; ++p) {
        float v = lse_parts[static_cast<long long>(p) * rows + row];
        if (!lse_log2) v *= kLog2e;
        const float w = exp2f(v - M) * invL;
        if (w == 0.f) continue;
        const float4 o = *reinterpret_cast<const float4*>(o_parts + (static_cast<long long>(p) * rows + row) * dim + d);
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
    }
    *reinterpret_cast<float4*>(out + row * dim + d) = acc;
  }
  if (lane == 0) {
    const float l2 = (M != -INFINITY && L > 0.f) ? M + log2f(L) : -INFINITY;
    lse[row] = lse_log2 ? l2 : l2 * kLn2;
  }
}

cudaError_t launch_merge_lse(const float* o_parts, const float* lse_parts, int n_parts, int rows, int dim,
                             float* out, float* lse, int lse_log2, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int warps = 8;
  const int grid = (rows + warps - 1) / warps;
  merge_lse_kernel<<<grid, warps * 32, 0, stream>>>(o_parts, lse_parts, n_parts, rows, dim, out, lse, lse_log2);
  return cudaGetLastError();
}

}  // namespace kvattn

namespace kvattn {

// x R for rows of 256 fp32 values, R = H_256 / 16 with H the Sylvester-Hadamard matrix
// (symmetric, orthonormal, its own inverse): the attention rotation of the Vulkan
// speculative-decoding report (pitfalls section, attention-rotation item), which spreads outlier channels
// before quantization.  One warp per row; lane l holds elements 8l .. 8l + 7: the three low
// index bits are butterflied in registers, the five high ones across lanes by shuffles.
// `in` may equal `out` (each warp reads its whole row before writing it), so neither pointer
// is declared restrict.
__global__ void __launch_bounds__(256) hadamard_kernel(const float* in, float* out, long long rows) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float4* src = reinterpret_cast<const float4*>(in + row * kHeadDim + lane * 8);
  const float4 a = src[0], b = src[1];
  float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int m = 1; m < 8; m <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!(e & m)) {
        const float u = x[e], w = x[e | m];
        x[e] = u + w;
        x[e | m] = u - w;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = lane & m;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float y = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? y - x[e] : x[e] + y;
    }
  }
  float4* dst = reinterpret_cast<float4*>(out + row * kHeadDim + lane * 8);
  dst[0] = make_float4(x[0] * 0.0625f, x[1] * 0.0625f, x[2] * 0.0625f, x[3] * 0.0625f);
  dst[1] = make_float4(x[4] * 0.0625f, x[5] * 0.0625f, x[6] * 0.0625f, x[7] * 0.0625f);
}

cudaError_t launch_hadamard(const float* in, float* out, long long rows, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  hadamard_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(in, out, rows);
  return cudaGetLastError();
}

}  // namespace kvattn
