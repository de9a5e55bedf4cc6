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
  // tokens to append before attending (0 for a plain decode): fp32 [n_new][H_kv][256] K and V
  // at positions new_pos0 + i, pages from new_table [H_kv][new_blocks]
  const float* k_new;
  const float* v_new;
  const int32_t* new_table;
  int n_new, new_pos0, new_blocks;
};

// Most tokens kvattn_append_decode appends in one call.
constexpr int kMaxAppend = 8;

// The split grid of a decode (partials into the workspace, or out / lse for one split) ...
cudaError_t launch_decode(const DecodeParams& prm, int n_kv, int key_fmt, int val_fmt, cudaStream_t stream);
// ... and the grid that merges the partials (nothing for one split).
cudaError_t launch_decode_merge(const DecodeParams& prm, int n_kv, cudaStream_t stream);
int decode_rows_pad(int rows);
bool decode_pair_supported(int key_fmt, int val_fmt);
// kvattn_kv_desc format codes -> kernel format ids (-1 if not a key / value format)
int key_format_id(int k_fmt);
int value_format_id(int v_fmt);
cudaError_t prepare_decode_kernels();

}  // namespace kvattn
