// Parameters of the split-KV decode kernel (shared by the launcher and the C ABI layer).
#pragma once

#include "common.cuh"

namespace kvattn {

struct DecodeParams {
  const uint8_t* k_pool;
  const uint8_t* v_pool;
  int64_t k_stride, v_stride, n_pages;
  const float* q;  // [n_q][H_q][256]
  const int32_t* q_pos;
  const int32_t* page_list;
  const int32_t* page_logical;
  const int32_t* n_pages_arr;
  float* out;  // [n_q][H_q][256]
  float* lse;  // [n_q][H_q]
  float* part_o;    // [H_kv][n_splits][rows_pad][256]
  float* part_lse;  // [H_kv][n_splits][rows_pad]   (log2 units)
  int n_q, group, n_qh, max_pages, n_splits;
};

cudaError_t launch_decode(const DecodeParams& prm, int n_kv, int key_fmt, bool vq8, cudaStream_t stream);
cudaError_t prepare_decode_kernels();

}  // namespace kvattn
