// C ABI of libkvattn: argument validation, split planning and kernel launches.
// No entry point allocates memory; every GPU action is stream-ordered on the caller's stream
// except kvattn_init and kvattn_device_error, which synchronise.
#include <nvtx3/nvToolsExt.h>

#include <chrono>
#include <thread>

#include "decode.cuh"

namespace kvattn {

cudaError_t launch_quantize_append(const kvattn_kv_desc&, const float*, const float*, int, int32_t, const int32_t*,
                                   int, cudaStream_t);
cudaError_t prepare_select_kernels();
cudaError_t prepare_resident_kernels();
cudaError_t launch_hadamard(const float*, float*, long long, cudaStream_t);
cudaError_t launch_resident_update(const int32_t*, const int32_t*, int, int, int, int, int32_t*, int32_t*, int,
                                   const int32_t*, int64_t, const int32_t*, int32_t*, int32_t*, int32_t*, int32_t*,
                                   cudaStream_t);
cudaError_t prepare_prefill_kernels();
bool prefill_pair_supported(int key_fmt, int val_fmt);
struct PrefillParams;
cudaError_t launch_merge_lse(const float*, const float*, int, int, int, float*, float*, int, cudaStream_t);
cudaError_t launch_block_summaries(const kvattn_kv_desc&, const int32_t*, int, int, int, int, float*, cudaStream_t);
cudaError_t launch_select(const float*, const float*, int, int, int, int, int, int, const int32_t*, int32_t*,
                          int32_t*, int32_t*, int, double*, cudaStream_t);
cudaError_t launch_page_copy(const void*, int64_t, int64_t, void*, int64_t, int64_t, int64_t, const int32_t*,
                             const int32_t*, int, int, int, cudaStream_t);

}  // namespace kvattn

namespace kvattn {

// An NVTX range named after the entry point around each call that launches GPU work, so a
// profiler timeline shows which library call every kernel belongs to (header-only NVTX 3: the
// push / pop cost a pointer check when no tool is attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

int key_format_id(int k_fmt) {
  switch (k_fmt) {
    case KVATTN_FMT_Q8_0: return kKeyQ8;
    case KVATTN_FMT_Q4_0: return kKeyQ4;
    case KVATTN_FMT_Q5_1: return kKeyQ51;
    case KVATTN_FMT_Q5_0: return kKeyQ50;
    default: return -1;
  }
}

int value_format_id(int v_fmt) {
  switch (v_fmt) {
    case KVATTN_FMT_Q4_0: return kValQ4;
    case KVATTN_FMT_Q8_0: return kValQ8;
    case KVATTN_FMT_Q4_1: return kValQ41;
    default: return -1;
  }
}

}  // namespace kvattn

using namespace kvattn;

namespace {

constexpr int kMaxDevices = 64;
bool g_inited[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return KVATTN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device_checked(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (*dev < 0 || *dev >= kMaxDevices || !g_inited[*dev]) return KVATTN_ERR_NOT_INITIALIZED;
  return KVATTN_OK;
}

int sm_count_for_planning() {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
    if (g_inited[dev]) return g_sm_count[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) return n;
  }
  cudaGetLastError();  // no device here: plan for a B200
  return 148;
}

// The SMs a grid planned for this cache may take: every SM, or the descriptor's budget.
int sm_budget_of(const kvattn_kv_desc* d) {
  const int sms = sm_count_for_planning();
  return d->sm_budget > 0 && d->sm_budget < sms ? d->sm_budget : sms;
}

int64_t page_bytes_of(int role, int fmt) {
  if (role == KVATTN_ROLE_K && fmt == KVATTN_FMT_Q8_0) return kKPageBytes;
  if (role == KVATTN_ROLE_K && fmt == KVATTN_FMT_Q4_0) return kK4PageBytes;
  if (role == KVATTN_ROLE_K && fmt == KVATTN_FMT_Q5_1) return kK5PageBytes;
  if (role == KVATTN_ROLE_K && fmt == KVATTN_FMT_Q5_0) return kK50PageBytes;
  if (role == KVATTN_ROLE_V && fmt == KVATTN_FMT_Q4_0) return kV4PageBytes;
  if (role == KVATTN_ROLE_V && fmt == KVATTN_FMT_Q8_0) return kV8PageBytes;
  if (role == KVATTN_ROLE_V && fmt == KVATTN_FMT_Q4_1) return kV41PageBytes;
  return 0;
}

int validate_desc(const kvattn_kv_desc* d) {
  if (!d) return KVATTN_ERR_INVALID_ARG;
  if (d->n_kv_heads < 1 || d->n_kv_heads > 64 || d->n_q_heads < 1 || d->n_q_heads % d->n_kv_heads)
    return KVATTN_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim || d->page_tokens != kPageTokens) return KVATTN_ERR_UNSUPPORTED_FORMAT;
  const int64_t kb = page_bytes_of(KVATTN_ROLE_K, d->k_fmt), vb = page_bytes_of(KVATTN_ROLE_V, d->v_fmt);
  if (!kb || !vb) return KVATTN_ERR_UNSUPPORTED_FORMAT;
  if (!decode_pair_supported(key_format_id(d->k_fmt), value_format_id(d->v_fmt))) return KVATTN_ERR_UNSUPPORTED_FORMAT;
  if (!d->k_pool || !d->v_pool || !aligned16(d->k_pool) || !aligned16(d->v_pool)) return KVATTN_ERR_INVALID_ARG;
  if (d->k_page_stride < kb || d->v_page_stride < vb || (d->k_page_stride & 15) || (d->v_page_stride & 15))
    return KVATTN_ERR_INVALID_ARG;
  if (d->n_pages < 1 || d->n_pages > (int64_t{1} << 31) - 1) return KVATTN_ERR_INVALID_ARG;
  if (d->sm_budget < 0 || d->reserved != 0) return KVATTN_ERR_INVALID_ARG;
  return KVATTN_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DecodePlan {
  int n_splits, rows_pad;
  size_t lse_off, o_off, bytes;
};

DecodePlan plan_decode(const kvattn_kv_desc* d, int n_q, int max_pages) {
  DecodePlan p{};
  const int group = d->n_q_heads / d->n_kv_heads;
  p.rows_pad = ((group * n_q + 7) / 8) * 8;
  const int sms = sm_budget_of(d);
  int s = sms / d->n_kv_heads;
  if (s < 1) s = 1;
  if (s > max_pages) s = max_pages < 1 ? 1 : max_pages;
  p.n_splits = s;
  p.lse_off = 0;
  p.o_off = round_up(p.lse_off + sizeof(float) * d->n_kv_heads * s * p.rows_pad, 256);
  p.bytes = s > 1 ? p.o_off + sizeof(float) * static_cast<size_t>(d->n_kv_heads) * s * p.rows_pad * kHeadDim : 0;
  return p;
}

}  // namespace

extern "C" {

KVATTN_API int kvattn_init(int device) {
  if (device < 0 || device >= kMaxDevices) return KVATTN_ERR_INVALID_ARG;
  cudaError_t e = cudaSetDevice(device);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return cuda_fail(e);
  if (prop.major != 10 || prop.minor != 0) return KVATTN_ERR_UNSUPPORTED_ARCH;
  if ((e = prepare_decode_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_select_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_prefill_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_resident_kernels()) != cudaSuccess) return cuda_fail(e);
  g_sm_count[device] = prop.multiProcessorCount;
  g_inited[device] = true;
  return KVATTN_OK;
}

KVATTN_API const char* kvattn_status_string(int s) {
  switch (s) {
    case KVATTN_OK: return "ok";
    case KVATTN_ERR_INVALID_ARG: return "invalid argument";
    case KVATTN_ERR_UNSUPPORTED_ARCH: return "unsupported architecture (needs sm_100)";
    case KVATTN_ERR_UNSUPPORTED_FORMAT: return "unsupported format";
    case KVATTN_ERR_BAD_PAGE: return "page id out of range";
    case KVATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case KVATTN_ERR_CUDA: return "CUDA error";
    case KVATTN_ERR_TIMEOUT: return "timeout";
    case KVATTN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case KVATTN_ERR_NOT_INITIALIZED: return "kvattn_init not called for this device";
    default: return "unknown status";
  }
}

KVATTN_API int kvattn_last_cuda_error(void) { return g_last_cuda_error; }

KVATTN_API int64_t kvattn_page_bytes(int role, int fmt) { return page_bytes_of(role, fmt); }

KVATTN_API int kvattn_device_error(kvattn_stream_t stream) {
  int dev;
  int st = current_device_checked(&dev);
  if (st) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  if ((e = cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int))) != cudaSuccess) return cuda_fail(e);
  const int zero = 0;
  if ((e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int))) != cudaSuccess) return cuda_fail(e);
  return v;
}

KVATTN_API int kvattn_quantize_append(const kvattn_kv_desc* desc, const float* k, const float* v, int n_tok,
                                      int32_t pos0, const int32_t* page_table, int n_blocks,
                                      kvattn_stream_t stream) {
  const CallRange range_("kvattn_quantize_append");
  int st = validate_desc(desc);
  if (st) return st;
  if (n_tok < 0 || pos0 < 0 || n_blocks < 0) return KVATTN_ERR_INVALID_ARG;
  if (n_tok == 0) return KVATTN_OK;
  if (!k || !v || !page_table || !aligned16(k) || !aligned16(v)) return KVATTN_ERR_INVALID_ARG;
  if ((static_cast<int64_t>(pos0) + n_tok - 1) / kPageTokens >= n_blocks) return KVATTN_ERR_INVALID_ARG;
  int dev;
  if ((st = current_device_checked(&dev))) return st;
  cudaError_t e = launch_quantize_append(*desc, k, v, n_tok, pos0, page_table, n_blocks,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API size_t kvattn_decode_workspace_size(const kvattn_kv_desc* desc, int n_q, int max_pages) {
  if (validate_desc(desc) || n_q < 1 || max_pages < 0) return 0;
  return plan_decode(desc, n_q, max_pages).bytes;
}

}  // extern "C"

namespace {

// Validates the arguments of a decode and fills its parameters (the split plan included).
int decode_setup(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos, const int32_t* page_list,
                 const int32_t* page_logical, const int32_t* n_pages, int max_pages, float* out, float* lse, void* ws,
                 size_t ws_bytes, DecodeParams* prm) {
  int st = validate_desc(desc);
  if (st) return st;
  if (n_q < 1 || max_pages < 0 || !q || !q_pos || !out || !lse || (max_pages > 0 && !page_list))
    return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return KVATTN_ERR_INVALID_ARG;
  const int group = desc->n_q_heads / desc->n_kv_heads;
  if (group * n_q > 24) return KVATTN_ERR_UNSUPPORTED_SHAPE;
  const DecodePlan plan = plan_decode(desc, n_q, max_pages);
  if (plan.bytes) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return KVATTN_ERR_INVALID_ARG;
    if (ws_bytes < plan.bytes) return KVATTN_ERR_WORKSPACE_TOO_SMALL;
  }
  int dev;
  if ((st = current_device_checked(&dev))) return st;
  *prm = DecodeParams{};
  prm->k_pool = static_cast<const uint8_t*>(desc->k_pool);
  prm->v_pool = static_cast<const uint8_t*>(desc->v_pool);
  prm->k_stride = desc->k_page_stride;
  prm->v_stride = desc->v_page_stride;
  prm->n_pages = desc->n_pages;
  prm->q = q;
  prm->q_pos = q_pos;
  prm->page_list = page_list;
  prm->page_logical = page_logical;
  prm->n_pages_arr = n_pages;
  prm->out = out;
  prm->lse = lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  prm->part_lse = plan.bytes ? reinterpret_cast<float*>(w + plan.lse_off) : nullptr;
  prm->part_o = plan.bytes ? reinterpret_cast<float*>(w + plan.o_off) : nullptr;
  prm->n_q = n_q;
  prm->group = group;
  prm->n_qh = desc->n_q_heads;
  prm->max_pages = max_pages;
  prm->n_splits = plan.n_splits;
  return KVATTN_OK;
}

}  // namespace

extern "C" {

KVATTN_API int kvattn_decode(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                             const int32_t* page_list, const int32_t* page_logical, const int32_t* n_pages,
                             int max_pages, float* out, float* lse, void* ws, size_t ws_bytes,
                             kvattn_stream_t stream) {
  const CallRange range_("kvattn_decode");
  DecodeParams prm;
  const int st =
      decode_setup(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse, ws, ws_bytes, &prm);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_decode(prm, desc->n_kv_heads, key_format_id(desc->k_fmt), value_format_id(desc->v_fmt), s);
  if (e == cudaSuccess) e = launch_decode_merge(prm, desc->n_kv_heads, s);
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_append_decode(const kvattn_kv_desc* desc, const float* k_new, const float* v_new, int n_new,
                                    int32_t pos0, const int32_t* page_table, int n_blocks, const float* q, int n_q,
                                    const int32_t* q_pos, const int32_t* page_list, const int32_t* page_logical,
                                    const int32_t* n_pages, int max_pages, float* out, float* lse, void* ws,
                                    size_t ws_bytes, kvattn_stream_t stream) {
  const CallRange range_("kvattn_append_decode");
  if (n_new < 1 || n_new > kMaxAppend || pos0 < 0 || n_blocks < 0) return KVATTN_ERR_INVALID_ARG;
  if (!k_new || !v_new || !page_table || !aligned16(k_new) || !aligned16(v_new)) return KVATTN_ERR_INVALID_ARG;
  if ((static_cast<int64_t>(pos0) + n_new - 1) / kPageTokens >= n_blocks) return KVATTN_ERR_INVALID_ARG;
  DecodeParams prm;
  const int st =
      decode_setup(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse, ws, ws_bytes, &prm);
  if (st) return st;
  prm.k_new = k_new;
  prm.v_new = v_new;
  prm.n_new = n_new;
  prm.new_pos0 = pos0;
  prm.new_table = page_table;
  prm.new_blocks = n_blocks;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_decode(prm, desc->n_kv_heads, key_format_id(desc->k_fmt), value_format_id(desc->v_fmt), s);
  if (e == cudaSuccess) e = launch_decode_merge(prm, desc->n_kv_heads, s);
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_decode_splits(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                                    const int32_t* page_list, const int32_t* page_logical, const int32_t* n_pages,
                                    int max_pages, float* out, float* lse, void* ws, size_t ws_bytes,
                                    kvattn_stream_t stream) {
  const CallRange range_("kvattn_decode_splits");
  DecodeParams prm;
  const int st =
      decode_setup(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, out, lse, ws, ws_bytes, &prm);
  if (st) return st;
  cudaError_t e = launch_decode(prm, desc->n_kv_heads, key_format_id(desc->k_fmt), value_format_id(desc->v_fmt),
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_decode_merge_splits(const kvattn_kv_desc* desc, int n_q, int max_pages, float* out, float* lse,
                                          void* ws, size_t ws_bytes, kvattn_stream_t stream) {
  const CallRange range_("kvattn_decode_merge_splits");
  // the same validation as the split grid's call; q, q_pos and the page list are not read
  static const float kDummy[4] __attribute__((aligned(16))) = {0.f, 0.f, 0.f, 0.f};
  static const int32_t kDummyI[1] = {0};
  DecodeParams prm;
  const int st = decode_setup(desc, kDummy, n_q, kDummyI, kDummyI, nullptr, nullptr, max_pages, out, lse, ws,
                              ws_bytes, &prm);
  if (st) return st;
  cudaError_t e = launch_decode_merge(prm, desc->n_kv_heads, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_merge_lse(const float* o_parts, const float* lse_parts, int n_parts, int rows, int dim,
                                float* out, float* lse, kvattn_stream_t stream) {
  const CallRange range_("kvattn_merge_lse");
  if (n_parts < 0 || rows < 0 || dim < 4 || (dim & 3)) return KVATTN_ERR_INVALID_ARG;
  if (rows == 0) return KVATTN_OK;
  if (!out || !lse || (n_parts > 0 && (!o_parts || !lse_parts))) return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(out) || (o_parts && !aligned16(o_parts))) return KVATTN_ERR_INVALID_ARG;
  int dev, st;
  if ((st = current_device_checked(&dev))) return st;
  cudaError_t e = launch_merge_lse(o_parts, lse_parts, n_parts, rows, dim, out, lse, 0,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_block_summaries(const kvattn_kv_desc* desc, const int32_t* page_table, int n_units,
                                      int n_blocks, int block_begin, int block_end, float* summaries,
                                      kvattn_stream_t stream) {
  const CallRange range_("kvattn_block_summaries");
  int st = validate_desc(desc);
  if (st) return st;
  if (n_units < 0 || n_blocks < 0 || block_begin < 0 || block_end < block_begin || block_end > n_blocks)
    return KVATTN_ERR_INVALID_ARG;
  if (n_units == 0 || block_end == block_begin) return KVATTN_OK;
  if (!page_table || !summaries || !aligned16(summaries) || n_units > 65535) return KVATTN_ERR_INVALID_ARG;
  int dev;
  if ((st = current_device_checked(&dev))) return st;
  cudaError_t e = launch_block_summaries(*desc, page_table, n_units, n_blocks, block_begin, block_end, summaries,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API size_t kvattn_select_workspace_size(int n_units, int n_blocks) {
  if (n_units < 0 || n_blocks < 0) return 0;
  return round_up(sizeof(double) * static_cast<size_t>(n_units) * n_blocks, 256);
}

KVATTN_API int kvattn_select_blocks(const float* summaries, const float* q_group, int n_units, int group,
                                    int n_blocks, int n_full, int n_total, int budget, int recent,
                                    const int32_t* page_table, int32_t* sel_logical, int32_t* sel_phys,
                                    int32_t* n_sel, int cap, void* ws, size_t ws_bytes, kvattn_stream_t stream) {
  const CallRange range_("kvattn_select_blocks");
  if (n_units < 0 || group < 1 || n_blocks < 0 || n_full < 0 || n_total < n_full || n_total > n_blocks ||
      budget < 0 || recent < 0 || cap < 0)
    return KVATTN_ERR_INVALID_ARG;
  if (n_units == 0) return KVATTN_OK;
  const int rec = recent < n_full ? recent : n_full;
  const int n_cand = n_full - rec;
  if (n_cand > 16384 || n_total > 65536 || n_units > 65535) return KVATTN_ERR_UNSUPPORTED_SHAPE;
  const int take = budget < n_cand ? budget : n_cand;
  if (cap < take + (n_total - n_cand)) return KVATTN_ERR_INVALID_ARG;
  if (!page_table || !sel_logical || !sel_phys || !n_sel) return KVATTN_ERR_INVALID_ARG;
  if (n_cand > 0 && (!summaries || !q_group || !aligned16(summaries) || !aligned16(q_group)))
    return KVATTN_ERR_INVALID_ARG;
  const size_t need = kvattn_select_workspace_size(n_units, n_blocks);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return KVATTN_ERR_INVALID_ARG;
  if (ws_bytes < need) return KVATTN_ERR_WORKSPACE_TOO_SMALL;
  int dev, st;
  if ((st = current_device_checked(&dev))) return st;
  cudaError_t e = launch_select(summaries, q_group, n_units, group, n_blocks, n_cand, n_total, budget, page_table,
                                sel_logical, sel_phys, n_sel, cap, static_cast<double*>(ws),
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_stream_plan(const int32_t* host_ids, const int32_t* dev_slots, int n, int32_t* run_first,
                                  int32_t* run_len, int max_runs) {
  if (n < 0 || max_runs < 0 || (n > 0 && (!host_ids || !dev_slots))) return KVATTN_ERR_INVALID_ARG;
  int runs = 0, i = 0;
  while (i < n) {
    int j = i + 1;
    while (j < n && host_ids[j] == host_ids[j - 1] + 1 && dev_slots[j] == dev_slots[j - 1] + 1) ++j;
    if (run_first && run_len && runs < max_runs) {
      run_first[runs] = i;
      run_len[runs] = j - i;
    }
    ++runs;
    i = j;
  }
  return runs;
}

KVATTN_API int kvattn_stream_pages(const void* host_pool, int64_t host_stride, void* dev_pool, int64_t dev_stride,
                                   int64_t page_bytes, const int32_t* host_ids, const int32_t* dev_slots, int n,
                                   kvattn_stream_t copy_stream, kvattn_event_t done, int* n_copies) {
  const CallRange range_("kvattn_stream_pages");
  if (n < 0 || page_bytes <= 0 || host_stride < page_bytes || dev_stride < page_bytes) return KVATTN_ERR_INVALID_ARG;
  if (n > 0 && (!host_pool || !dev_pool || !host_ids || !dev_slots)) return KVATTN_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (host_ids[i] < 0 || dev_slots[i] < 0) return KVATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(copy_stream);
  int copies = 0;
  const uint8_t* hp = static_cast<const uint8_t*>(host_pool);
  uint8_t* dp = static_cast<uint8_t*>(dev_pool);
  int i = 0;
  while (i < n) {
    int j = i + 1;
    while (j < n && host_ids[j] == host_ids[j - 1] + 1 && dev_slots[j] == dev_slots[j - 1] + 1) ++j;
    const int run = j - i;
    const uint8_t* src = hp + static_cast<int64_t>(host_ids[i]) * host_stride;
    uint8_t* dst = dp + static_cast<int64_t>(dev_slots[i]) * dev_stride;
    cudaError_t e;
    if (host_stride == page_bytes && dev_stride == page_bytes)
      e = cudaMemcpyAsync(dst, src, static_cast<size_t>(run) * page_bytes, cudaMemcpyHostToDevice, s);
    else
      e = cudaMemcpy2DAsync(dst, dev_stride, src, host_stride, page_bytes, run, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
    ++copies;
    i = j;
  }
  if (done) {
    cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(done), s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (n_copies) *n_copies = copies;
  return KVATTN_OK;
}

}  // extern "C"

namespace {

// Device address of a pinned, device-mapped host range; INVALID_ARG for anything else
// (pageable memory would fault the copy kernel, so it is refused here on the host).
int mapped_host_range(const void* host, int64_t bytes, void** dev) {
  if (!host || bytes <= 0 || !aligned16(host)) return KVATTN_ERR_INVALID_ARG;
  cudaPointerAttributes a{}, b{};
  if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
    cudaGetLastError();
    return KVATTN_ERR_INVALID_ARG;
  }
  const void* last = static_cast<const uint8_t*>(host) + (bytes - 1);
  if (cudaPointerGetAttributes(&b, last) != cudaSuccess) {
    cudaGetLastError();
    return KVATTN_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeHost || b.type != cudaMemoryTypeHost || !a.devicePointer || !b.devicePointer)
    return KVATTN_ERR_INVALID_ARG;
  if (static_cast<const uint8_t*>(b.devicePointer) - static_cast<const uint8_t*>(a.devicePointer) != bytes - 1)
    return KVATTN_ERR_INVALID_ARG;
  *dev = a.devicePointer;
  return KVATTN_OK;
}

int page_copy_common(const void* host_pool, int64_t host_stride, int64_t n_host_pages, void* dev_pool,
                     int64_t dev_stride, int64_t n_slots, int64_t page_bytes, const int32_t* host_ids,
                     const int32_t* dev_slots, int n, int n_ctas, int to_device, kvattn_stream_t stream) {
  if (n < 0 || n_ctas < 0 || page_bytes <= 0 || (page_bytes & 15) || host_stride < page_bytes ||
      dev_stride < page_bytes || (host_stride & 15) || (dev_stride & 15) || n_host_pages < 1 || n_slots < 1)
    return KVATTN_ERR_INVALID_ARG;
  if (n == 0) return KVATTN_OK;
  if (!dev_pool || !aligned16(dev_pool) || !host_ids || !dev_slots) return KVATTN_ERR_INVALID_ARG;
  int dev, st;
  if ((st = current_device_checked(&dev))) return st;
  void* hdev = nullptr;
  if ((st = mapped_host_range(host_pool, (n_host_pages - 1) * host_stride + page_bytes, &hdev))) return st;
  cudaError_t e = launch_page_copy(hdev, host_stride, n_host_pages, dev_pool, dev_stride, n_slots, page_bytes,
                                   host_ids, dev_slots, n, n_ctas, to_device, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

KVATTN_API int kvattn_gather_pages(const void* host_pool, int64_t host_stride, int64_t n_host_pages, void* dev_pool,
                                   int64_t dev_stride, int64_t n_slots, int64_t page_bytes, const int32_t* host_ids,
                                   const int32_t* dev_slots, int n, int n_ctas, kvattn_stream_t stream) {
  const CallRange range_("kvattn_gather_pages");
  return page_copy_common(host_pool, host_stride, n_host_pages, dev_pool, dev_stride, n_slots, page_bytes, host_ids,
                          dev_slots, n, n_ctas, 1, stream);
}

KVATTN_API int kvattn_scatter_pages(void* host_pool, int64_t host_stride, int64_t n_host_pages, const void* dev_pool,
                                    int64_t dev_stride, int64_t n_slots, int64_t page_bytes, const int32_t* host_ids,
                                    const int32_t* dev_slots, int n, int n_ctas, kvattn_stream_t stream) {
  const CallRange range_("kvattn_scatter_pages");
  return page_copy_common(host_pool, host_stride, n_host_pages, const_cast<void*>(dev_pool), dev_stride, n_slots,
                          page_bytes, host_ids, dev_slots, n, n_ctas, 0, stream);
}

KVATTN_API int kvattn_hadamard(const float* in, float* out, int64_t rows, kvattn_stream_t stream) {
  const CallRange range_("kvattn_hadamard");
  if (rows < 0 || (rows > 0 && (!in || !out)) || rows > (1ll << 40)) return KVATTN_ERR_INVALID_ARG;
  if (rows > 0 && (!aligned16(in) || !aligned16(out))) return KVATTN_ERR_INVALID_ARG;
  int dev;
  int st = current_device_checked(&dev);
  if (st) return st;
  cudaError_t e = launch_hadamard(in, out, rows, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_resident_update(const int32_t* sel_logical, const int32_t* n_sel, int cap, int n_units,
                                      int n_blocks, int n_full, int32_t* slot_of_block, int32_t* block_of_slot,
                                      int n_slots, const int32_t* host_page_of_block, int64_t first_page,
                                      const int32_t* extra_page, int32_t* page_list, int32_t* copy_host,
                                      int32_t* copy_dst, int32_t* n_copies, kvattn_stream_t stream) {
  const CallRange range_("kvattn_resident_update");
  if (!sel_logical || !n_sel || !slot_of_block || !block_of_slot || !host_page_of_block || !extra_page ||
      !page_list || !copy_host || !copy_dst || !n_copies)
    return KVATTN_ERR_INVALID_ARG;
  if (cap < 1 || n_units < 1 || n_units > 65535 || n_blocks < 1 || n_blocks > 262144 || n_full < 0 ||
      n_full > n_blocks || n_slots < 1 || n_slots > 16384 || first_page < 0 ||
      first_page + static_cast<int64_t>(n_units) * n_slots > INT32_MAX)
    return KVATTN_ERR_INVALID_ARG;
  int dev;
  int st = current_device_checked(&dev);
  if (st) return st;
  cudaError_t e = launch_resident_update(sel_logical, n_sel, cap, n_units, n_blocks, n_full, slot_of_block,
                                         block_of_slot, n_slots, host_page_of_block, first_page, extra_page,
                                         page_list, copy_host, copy_dst, n_copies, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

KVATTN_API int kvattn_stream_wait(kvattn_event_t event, int timeout_ms) {
  if (!event || timeout_ms < 0) return KVATTN_ERR_INVALID_ARG;
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    cudaError_t e = cudaEventQuery(static_cast<cudaEvent_t>(event));
    if (e == cudaSuccess) return KVATTN_OK;
    if (e != cudaErrorNotReady) return cuda_fail(e);
    const auto ms =
        std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
    if (ms >= timeout_ms) return KVATTN_ERR_TIMEOUT;
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

}  // extern "C"

extern "C" {

KVATTN_API size_t kvattn_prefill_workspace_size(const kvattn_kv_desc* desc, int n_q, int max_pages,
                                                int kv_split_tokens) {
  if (validate_desc(desc) || n_q < 1 || max_pages < 0 || kv_split_tokens < kPageTokens ||
      kv_split_tokens % kPageTokens || kv_split_tokens > 65536)
    return 0;
  return plan_prefill(desc->n_kv_heads, desc->n_q_heads / desc->n_kv_heads, n_q, max_pages, kv_split_tokens,
                      sm_budget_of(desc))
      .bytes;
}

}  // extern "C"

namespace {

// Validates a prefill call and launches it (exact: the ~22-bit operand splits; else one f16
// rounding per operand).
int prefill_chunk(const kvattn_kv_desc* desc, const uint16_t* q, int n_q, const int32_t* q_pos,
                  const int32_t* page_list, const int32_t* page_logical, const int32_t* n_pages, int max_pages,
                  int kv_split_tokens, float* out, float* lse, void* ws, size_t ws_bytes, kvattn_stream_t stream,
                  bool exact) {
  int st = validate_desc(desc);
  if (st) return st;
  if (!prefill_pair_supported(key_format_id(desc->k_fmt), value_format_id(desc->v_fmt)))
    return KVATTN_ERR_UNSUPPORTED_FORMAT;
  if (n_q < 1 || max_pages < 0 || !q || !q_pos || !out || !lse || (max_pages > 0 && !page_list))
    return KVATTN_ERR_INVALID_ARG;
  if (kv_split_tokens < kPageTokens || kv_split_tokens % kPageTokens || kv_split_tokens > 65536)
    return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q)) return KVATTN_ERR_INVALID_ARG;
  const int group = desc->n_q_heads / desc->n_kv_heads;
  const long long rows = static_cast<long long>(n_q) * group;
  if (rows > (1ll << 24)) return KVATTN_ERR_UNSUPPORTED_SHAPE;
  const PrefillPlan plan =
      plan_prefill(desc->n_kv_heads, group, n_q, max_pages, kv_split_tokens, sm_budget_of(desc));
  if (plan.n_ks > 65535 || plan.n_mt > (1 << 30)) return KVATTN_ERR_UNSUPPORTED_SHAPE;
  if (plan.bytes) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return KVATTN_ERR_INVALID_ARG;
    if (ws_bytes < plan.bytes) return KVATTN_ERR_WORKSPACE_TOO_SMALL;
  }
  int dev;
  if ((st = current_device_checked(&dev))) return st;
  PrefillParams prm{};
  prm.k_pool = static_cast<const uint8_t*>(desc->k_pool);
  prm.v_pool = static_cast<const uint8_t*>(desc->v_pool);
  prm.k_stride = desc->k_page_stride;
  prm.v_stride = desc->v_page_stride;
  prm.n_pages = desc->n_pages;
  prm.q = q;
  prm.q_pos = q_pos;
  prm.page_list = page_list;
  prm.page_logical = page_logical;
  prm.n_pages_arr = n_pages;
  prm.out = out;
  prm.lse = lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  prm.part_lse = plan.bytes ? reinterpret_cast<float*>(w + plan.lse_off) : nullptr;
  prm.part_o = plan.bytes ? reinterpret_cast<float*>(w + plan.o_off) : nullptr;
  prm.n_q = n_q;
  prm.group = group;
  prm.n_qh = desc->n_q_heads;
  prm.max_pages = max_pages;
  prm.pages_per_split = plan.pps;
  prm.n_ks = plan.n_ks;
  prm.rows_pad = plan.rows_pad;
  cudaError_t e =
      launch_prefill(prm, desc->n_kv_heads, key_format_id(desc->k_fmt), value_format_id(desc->v_fmt), exact,
                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVATTN_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

KVATTN_API int kvattn_prefill_chunk(const kvattn_kv_desc* desc, const uint16_t* q, int n_q, const int32_t* q_pos,
                                    const int32_t* page_list, const int32_t* page_logical, const int32_t* n_pages,
                                    int max_pages, int kv_split_tokens, float* out, float* lse, void* ws,
                                    size_t ws_bytes, kvattn_stream_t stream) {
  const CallRange range_("kvattn_prefill_chunk");
  return prefill_chunk(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, kv_split_tokens, out, lse,
                       ws, ws_bytes, stream, true);
}

KVATTN_API int kvattn_prefill_chunk_f16(const kvattn_kv_desc* desc, const uint16_t* q, int n_q, const int32_t* q_pos,
                                        const int32_t* page_list, const int32_t* page_logical, const int32_t* n_pages,
                                        int max_pages, int kv_split_tokens, float* out, float* lse, void* ws,
                                        size_t ws_bytes, kvattn_stream_t stream) {
  const CallRange range_("kvattn_prefill_chunk_f16");
  return prefill_chunk(desc, q, n_q, q_pos, page_list, page_logical, n_pages, max_pages, kv_split_tokens, out, lse,
                       ws, ws_bytes, stream, false);
}

}  // extern "C"
