/*
 * kvattn -- attention over a block-quantized, paged KV cache on NVIDIA B200 (sm_100a).
 *
 * C ABI of libkvattn.so.  Plain pointers and sizes only.  Every entry point returns an
 * int status (0 = KVATTN_OK, negative = error, see kvattn_status); none throws, none
 * allocates device memory.  All GPU work is asynchronous on the caller's stream; buffers
 * must stay valid until that work completes.  The caller owns every buffer.
 *
 * Sources (page title, section):
 *  [KVMEM]  KVMem reproduction on one 7900 XTX (lcz.me/topic/1972): test command (128-token
 *           blocks, 32,768-token budget, 16,384-token generation reserve), recall section
 *           (blocks kept on the GPU are chosen by a retrieval query).
 *  [STREAM] Adaptive KV Streaming + RDNA 4 announcement (wqu.guru): full KV history in
 *           host RAM, bounded working sets streamed over PCIe alongside compute; method list
 *           (paged decode attention extended to verify batches; chunked prefill across
 *           streamed pages merged by online log-sum-exp; layer L+1 transfers overlapped
 *           with layer L compute).
 *  [GUIDE]  Adaptive KV Streaming six-step validation guide (alphalab.site): streaming needs
 *           flash attention with Q8_0 K / Q4_0 V; its build step compiles the q4_0-q4_0 and
 *           q8_0-q4_0 flash-attention KV pairs among others.
 *  [VULKAN] Vulkan speculative-decoding report, 7900 XTX (lcz.me/topic/1398): model structure
 *           (16 layers x 4 KV heads x 256 = 16,384 elements per token), pitfalls (q4_0 =
 *           18 bytes per 32 elements; only legacy block quants are valid KV formats) and
 *           configs (q8_0 = 8.5 bits per element); summary (a q4_0/q4_0 cache holds the most
 *           tokens).
 *  [MTP]    7900 XTX llama.cpp MTP tuning notes (lcz.me/topic/593): a server command with a
 *           q5_0 K / q4_1 V cache at 131,072 context.
 *
 * Data formats (fixed by this library; the pages fix only the bits per element):
 *  - head_dim = 256, page = 128 tokens of one (layer, KV head).
 *  - Q8_0: blocks of 32 codes q in [-127,127] + one fp16 scale d; value = q * d.  A code is
 *    stored offset-binary, as the byte q + 128 (a zero byte, in a slot never written, is the
 *    code -128 with the scale 0).
 *    Q4_0: blocks of 32 4-bit codes q in [0,15] + fp16 d; value = (q - 8) * d.
 *    Q5_1: blocks of 32 5-bit codes q in [0,31] + fp16 d + fp16 minimum m; value = q * d + m
 *    ([VULKAN] pitfalls: 6 bits per element, a zero point; paired with Q4_0 values).
 *    Q5_0: 5-bit codes q in [0,31] + fp16 d; value = (q - 16) * d.  Q4_1: 4-bit codes q in
 *    [0,15] + fp16 d + fp16 minimum m; value = q * d + m ([VULKAN] pitfalls lists both among
 *    the KV types; [MTP] runs a Q5_0 K / Q4_1 V cache).
 *  - Format pairs: Q8_0, Q4_0 or Q5_1 K with Q4_0 or Q8_0 V, and Q5_0 K with Q4_1 V.  K pages
 *    are Q8_0 (34,816 B), Q4_0 (18,432 B), Q5_1 (24,576 B) or Q5_0 (22,528 B); V pages are Q4_0
 *    (18,432 B), Q8_0 (34,816 B) or Q4_1 (20,480 B).  Inside a
 *    page, codes come first and fp16 scales after them, both in tensor-core fragment order
 *    (tok = slot in page, c = channel, b = c/32, G = tok/16):
 *      K Q8_0 byte  q + 128 (tok = 16G+8H+R, c = 64P+32(j/8)+8T+j%8) at
 *                   ((((G*4+P)*2+H)*8+R)*4+T)*16+j
 *      K Q4_0 word  (tok = 16G+8H+R, b = 4Q+c, channels 32b+8T+i, i < 8) is the little-endian
 *                   uint32 at 4*(((((G*2+Q)*2+H)*8+R)*4+T)*4+c); channel i's 4-bit code sits
 *                   at bit 4*(i/2) + 16*(i%2)
 *      K Q5_1/Q5_0  low 4 bits of each code as the K Q4_0 word; bit 4 of the codes of token
 *                   16G+8H+R, channels 32(4Q+c)+8T+i in the uint32 at
 *                   16384 + 4*((((G*2+Q)*2+H)*8+R)*4+T), channel (c, i) at bit 16(i%2)+4c+i/2;
 *                   Q5_1 minimum m[16G+8H+R][b] at 22528 + 2*(((G*8+R)*2+H)*8+b)
 *      K scale      d[16G+8H+R][b] at S + 2*(((G*8+R)*2+H)*8+b), S = 32768 (Q8_0), 16384
 *                   (Q4_0) or 20480 (Q5_1, Q5_0)
 *      V Q4_0 byte  ((((G*4+C)*8+R)*4+T)*16 + 4w + y: block b = 2C+w/2, token
 *                   16G+2T+8(w%2)+y/2; low nibble c = 32b+16(y%2)+R, high nibble c+8
 *      V Q8_0 byte  q + 128 (tok = 16G+2T+8(w%2)+y%2, c = 32b+16(w/2)+8(y/2)+R) at
 *                   ((((G*8+b)*8+R)*4+T)*16 + 4w + y
 *      V Q4_1 byte  as the V Q4_0 byte (the code is q, not q - 8)
 *      V scale      d[16G+2T+k%2+8(k/2)][b] at S + 2*(((G*4+T)*8+b)*4+k), S = 16384 (Q4_0,
 *                   Q4_1) or 32768 (Q8_0); Q4_1 minima in the same arrangement at 18432
 *    kvattn_quantize_append is the supported writer.
 *  - Pages live in caller-owned pools: page p's K bytes start at k_pool + p * k_page_stride
 *    and its V bytes at v_pool + p * v_page_stride.  Pool bases and strides are multiples
 *    of 16 bytes.  K and V of one page may be interleaved in one allocation by choosing
 *    v_pool = k_pool + (K page bytes) and equal strides.
 *  - A page list names, per KV head, the physical pages to attend over and (optionally)
 *    their logical block indices; key positions are logical * 128 + slot.
 *
 * Device-side checks: every page id read on the device is checked against [0, n_pages);
 * a bad id skips the page and records KVATTN_ERR_BAD_PAGE in a per-device error word that
 * kvattn_device_error() returns and clears.  Bounded waits inside kernels record
 * KVATTN_ERR_TIMEOUT there instead of spinning forever.
 */
#ifndef KVATTN_H
#define KVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KVATTN_API __attribute__((visibility("default")))
#else
#define KVATTN_API
#endif

/* cudaStream_t / cudaEvent_t, passed opaquely (0 = the legacy default stream). */
typedef void* kvattn_stream_t;
typedef void* kvattn_event_t;

enum kvattn_status {
  KVATTN_OK = 0,
  KVATTN_ERR_INVALID_ARG = -1,        /* null pointer, bad size or alignment, bad range     */
  KVATTN_ERR_UNSUPPORTED_ARCH = -2,   /* device is not compute capability 10.0 (sm_100)     */
  KVATTN_ERR_UNSUPPORTED_FORMAT = -3, /* format / head_dim / page size not supported        */
  KVATTN_ERR_BAD_PAGE = -4,           /* a page id outside [0, n_pages) (device-side check) */
  KVATTN_ERR_WORKSPACE_TOO_SMALL = -5,
  KVATTN_ERR_CUDA = -6,               /* a CUDA runtime call failed; see kvattn_last_cuda_error */
  KVATTN_ERR_TIMEOUT = -7,            /* a bounded wait expired                             */
  KVATTN_ERR_UNSUPPORTED_SHAPE = -8,  /* e.g. more query rows per KV head than supported    */
  KVATTN_ERR_NOT_INITIALIZED = -9     /* kvattn_init was not called for the current device  */
};

enum kvattn_format {
  KVATTN_FMT_Q4_0 = 4,
  KVATTN_FMT_Q8_0 = 8,
  KVATTN_FMT_Q5_1 = 51,
  KVATTN_FMT_Q5_0 = 50, /* keys only  */
  KVATTN_FMT_Q4_1 = 41  /* values only */
};
enum kvattn_role { KVATTN_ROLE_K = 0, KVATTN_ROLE_V = 1 };

typedef struct kvattn_kv_desc {
  int32_t n_kv_heads;     /* H_kv >= 1                                                  */
  int32_t n_q_heads;      /* H_q, a multiple of H_kv; the GQA group is H_q / H_kv       */
  int32_t head_dim;       /* must be 256                                                */
  int32_t page_tokens;    /* must be 128                                                */
  int32_t k_fmt;          /* KVATTN_FMT_Q8_0, Q4_0, Q5_1 (values Q4_0 or Q8_0) or Q5_0  */
  int32_t v_fmt;          /* KVATTN_FMT_Q4_0 or Q8_0, or Q4_1 (with Q5_0 keys only)     */
  void* k_pool;           /* device memory, 16-byte aligned                              */
  void* v_pool;           /* device memory, 16-byte aligned                              */
  int64_t k_page_stride;  /* bytes between consecutive K pages (>= K page bytes, %16==0) */
  int64_t v_page_stride;  /* bytes between consecutive V pages (>= V page bytes, %16==0) */
  int64_t n_pages;        /* physical pages addressable in both pools                   */
  int32_t sm_budget;      /* 0: decode and prefill grids are sized to every SM; n > 0:   */
                          /* at most n SMs' worth of CTAs (fewer KV splits), leaving the */
                          /* other SMs to kernels that run at the same time on another   */
                          /* stream, e.g. the page copy of the streamed working set.     */
                          /* Workspace sizes follow the same plan.  Must be >= 0.        */
  int32_t reserved;       /* must be 0                                                  */
} kvattn_kv_desc;

/* ---- setup and status ------------------------------------------------------------- */

/* Checks that `device` is an sm_100 part and prepares the kernels for it (sets it current).
 * Returns KVATTN_ERR_UNSUPPORTED_ARCH on any other device.  Call once per device before any
 * other GPU entry point on it.  Not stream-ordered; do not call during stream capture. */
KVATTN_API int kvattn_init(int device);

/* Static, human-readable name of a status code. */
KVATTN_API const char* kvattn_status_string(int status);

/* The last cudaError_t seen by the library on this thread (0 if none). */
KVATTN_API int kvattn_last_cuda_error(void);

/* Synchronises `stream`, then returns and clears the current device's error word
 * (KVATTN_OK, KVATTN_ERR_BAD_PAGE or KVATTN_ERR_TIMEOUT). */
KVATTN_API int kvattn_device_error(kvattn_stream_t stream);

/* Bytes of one page of the given role and format (0 if the pair is unsupported). */
KVATTN_API int64_t kvattn_page_bytes(int role, int fmt);

/* ---- cache write path ----------------------------------------------------------------
 * Quantizes n_tok new tokens and writes them into their pages (the Q8_0 / Q4_0 / Q5_1
 * encoders of [VULKAN] pitfalls).  Q8_0: d = amax/127, q = round-half-away(x * fp32(1/d)),
 * clamped to +-127.  Q4_0: m = the element of largest magnitude, d = m/-8, q = min(15,
 * floor(x * fp32(1/d) + 8.5)).  Q5_1: m = the block minimum, d = (max - m)/31, q = min(31,
 * floor((x - m) * fp32(1/d) + 0.5)).  Every step that decides a code is rounded to fp32;
 * scales and minima are stored as fp16.  A block whose fp32 scale is nonzero but has no
 * finite fp32 reciprocal (all elements, or for Q5_1 the spread, below about 1e-36) is outside
 * the supported range: its codes are unspecified and it decodes to 0.
 *   k, v        device fp32 [n_tok][H_kv][256]
 *   pos0        position of the first token; token i goes to logical block (pos0+i)/128,
 *               slot (pos0+i)%128
 *   page_table  device int32 [H_kv][n_blocks]: logical block -> physical page
 * Other slots of the touched pages are left unchanged.  Returns INVALID_ARG if a touched
 * block is >= n_blocks. */
KVATTN_API int kvattn_quantize_append(const kvattn_kv_desc* desc, const float* k, const float* v,
                                      int n_tok, int32_t pos0, const int32_t* page_table,
                                      int n_blocks, kvattn_stream_t stream);

/* ---- split-KV flash decode / MTP verify ---------------------------------------------
 * Attention of n_q query tokens (1 = decode, up to 4 = MTP verify batch; [STREAM] method
 * list) of every query head over the pages listed for its KV head.  Query token i sits at
 * position q_pos[i]; it sees keys with position <= q_pos[i] (causal among the new tokens).
 *   q            device fp32 [n_q][H_q][256]
 *   q_pos        device int32 [n_q]
 *   page_list    device int32 [H_kv][max_pages]: physical page ids, any order
 *   page_logical device int32 [H_kv][max_pages] logical block of each listed page, or NULL
 *                (then page_list[h][i] holds logical block i)
 *   n_pages      device int32 [H_kv] pages used per head (<= max_pages), or NULL (= max_pages)
 *   out          device fp32 [n_q][H_q][256]: softmax(q.k/16) v
 *   lse          device fp32 [n_q][H_q]: natural-log log-sum-exp of the scaled scores
 *                (-inf and out = 0 for a row that sees no key)
 * Key and value codes enter the tensor-core MMAs exactly; block scales are applied in fp32
 * (keys) or folded into P as an exact f16 product plus a remainder (values), and the query
 * and P are split into f16 high and low parts, so the result matches exact attention over
 * the dequantized cache to about 2^-20 relative.
 *   ws, ws_bytes device workspace of at least kvattn_decode_workspace_size() bytes (256-byte
 *                aligned; may be NULL when that size is 0).  The keys of each KV head are
 *                split across CTAs; per-split (o, lse) partials go to the workspace and a
 *                second grid, launched behind the first, merges them.  Calls that share a
 *                workspace must not overlap on the GPU.
 * Both grids use programmatic dependent launch: each may start while the kernel before it on
 * the stream finishes, and waits for that kernel before reading any argument.
 * Supports group * n_q <= 24 query rows per KV head.  The split count depends only on the
 * arguments and the device, so results are deterministic. */
KVATTN_API size_t kvattn_decode_workspace_size(const kvattn_kv_desc* desc, int n_q, int max_pages);
KVATTN_API int kvattn_decode(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                             const int32_t* page_list, const int32_t* page_logical,
                             const int32_t* n_pages, int max_pages, float* out, float* lse,
                             void* ws, size_t ws_bytes, kvattn_stream_t stream);

/* kvattn_quantize_append of n_new tokens followed by kvattn_decode, in one grid: the same
 * bytes land in the pages and the same outputs result, without the append kernel and its
 * dependency on the stream.  The first CTA of every KV head encodes the new tokens into their
 * pages in global memory; a CTA that streams such a page encodes the token again into its
 * shared-memory copy before reading it, so no CTA waits for another.  Arguments are those of
 * the two calls (k_new, v_new device fp32 [n_new][H_kv][256] at positions pos0 .. pos0 +
 * n_new - 1, pages from page_table [H_kv][n_blocks]), with 1 <= n_new <= 8.  Errors as for
 * both calls. */
KVATTN_API int kvattn_append_decode(const kvattn_kv_desc* desc, const float* k_new, const float* v_new, int n_new,
                                    int32_t pos0, const int32_t* page_table, int n_blocks, const float* q,
                                    int n_q, const int32_t* q_pos, const int32_t* page_list,
                                    const int32_t* page_logical, const int32_t* n_pages, int max_pages,
                                    float* out, float* lse, void* ws, size_t ws_bytes, kvattn_stream_t stream);

/* The two grids of kvattn_decode, as separate calls (same arguments; kvattn_decode is
 * kvattn_decode_splits followed by kvattn_decode_merge_splits on the same stream and
 * workspace).  kvattn_decode_splits runs the split grid: per-split (o, lse) partials into ws,
 * or out / lse directly when the plan has one split.  kvattn_decode_merge_splits merges them
 * into out / lse (nothing to do for one split); it reads only the workspace, so other work may
 * run on the stream in between, as long as the workspace is not reused. */
KVATTN_API int kvattn_decode_splits(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                                    const int32_t* page_list, const int32_t* page_logical,
                                    const int32_t* n_pages, int max_pages, float* out, float* lse,
                                    void* ws, size_t ws_bytes, kvattn_stream_t stream);
KVATTN_API int kvattn_decode_merge_splits(const kvattn_kv_desc* desc, int n_q, int max_pages, float* out,
                                          float* lse, void* ws, size_t ws_bytes, kvattn_stream_t stream);

/* Same computation and arguments as kvattn_decode, for callers that cannot allocate device
 * memory (for example code hosted by a framework whose memory pool owns the device memory
 * and forbids cudaMalloc, or loops that must never enter the allocator).  It has no
 * counterpart on the source pages.  The per-split scratch is a 4 MiB file-scope device array
 * (every GPU that loads the library holds it until exit); plans larger than that return
 * KVATTN_ERR_WORKSPACE_TOO_SMALL.  The first call on a device looks up the array's device
 * address (with that device current) and should come before any stream capture.  All calls
 * on a device share that device's array, which keeps the last call's contents: calls on one
 * device whose GPU work overlaps (for example on two streams) race, so order them on one
 * stream.  Calls no allocating routine.  Shapes kvattn_decode refuses return the same status
 * here (UNSUPPORTED_SHAPE for group * n_q > 24).  The looked-up address does not survive a
 * device reset (cudaDeviceReset): the library is then unusable on that device in this
 * process, as for every other entry point. */
KVATTN_API int kvattn_decode_noalloc(const kvattn_kv_desc* desc, const float* q, int n_q, const int32_t* q_pos,
                                     const int32_t* page_list, const int32_t* page_logical,
                                     const int32_t* n_pages, int max_pages, float* out, float* lse,
                                     kvattn_stream_t stream);

/* ---- log-sum-exp merge ([STREAM] method list: online LSE accumulation) -------------
 * out = sum_p exp(lse_p - lse) * o_p with lse = ln sum_p exp(lse_p), skipping -inf parts.
 *   o_parts   device fp32 [n_parts][rows][dim];  lse_parts device fp32 [n_parts][rows]
 *   out       device fp32 [rows][dim];           lse       device fp32 [rows]
 * dim must be a multiple of 4. */
KVATTN_API int kvattn_merge_lse(const float* o_parts, const float* lse_parts, int n_parts, int rows,
                                int dim, float* out, float* lse, kvattn_stream_t stream);

/* ---- KVMem block summaries and selection ([KVMEM]) ---------------------------------
 * Summary of a full 128-token block = mean dequantized key per channel, rounded once to
 * fp32 (the per-block sum is exact in fp64 for scales within 2^28 of each other).  Keys may
 * be Q8_0, Q4_0, Q5_1 or Q5_0.
 *   page_table  device int32 [n_units][n_blocks] (a unit is one (layer, KV head))
 *   summaries   device fp32 [n_units][n_blocks][256]; blocks [block_begin, block_end) of
 *               every unit are written, others untouched. */
KVATTN_API int kvattn_block_summaries(const kvattn_kv_desc* desc, const int32_t* page_table,
                                      int n_units, int n_blocks, int block_begin, int block_end,
                                      float* summaries, kvattn_stream_t stream);

/* Per unit: score[b] = sum_{j<group, c<256} q_group[j][c] * summary[b][c] in fp64 for the
 * candidate blocks b < n_full - recent; keep the `budget` best (ties: lower b first), add the
 * recent window [n_full - recent, n_full) and the partial tail [n_full, n_total); write them
 * in ascending order.
 *   summaries   device fp32 [n_units][n_blocks][256]   (n_blocks >= n_total)
 *   q_group     device fp32 [n_units][group][256]       (the retrieval query rows)
 *   page_table  device int32 [n_units][n_blocks]
 *   sel_logical device int32 [n_units][cap], sel_phys device int32 [n_units][cap],
 *   n_sel       device int32 [n_units]; cap >= min(budget, candidates) + recent + tail.
 *   ws          device workspace of kvattn_select_workspace_size(n_units, n_blocks) bytes.
 * Candidates per unit <= 16384.
 * Scores are fp64 sums of the 256 x group products, accumulated by fused multiply-adds in a
 * fixed order; a correctly rounded sum can differ from them by at most about
 * 256 x group x 2^-53 x sum|products|.  The ids therefore equal those of an exact ranking
 * wherever the gap between the budget-th and the next candidate's score is larger than that
 * (the tests take 1e-9 of the largest score as the margin and check it per seed); blocks
 * closer than that may be ordered either way. */
KVATTN_API size_t kvattn_select_workspace_size(int n_units, int n_blocks);
KVATTN_API int kvattn_select_blocks(const float* summaries, const float* q_group, int n_units,
                                    int group, int n_blocks, int n_full, int n_total, int budget,
                                    int recent, const int32_t* page_table, int32_t* sel_logical,
                                    int32_t* sel_phys, int32_t* n_sel, int cap, void* ws,
                                    size_t ws_bytes, kvattn_stream_t stream);

/* ---- chunked prefill on tcgen05 ([STREAM] method list) -----------------------------
 * Attention of n_q bf16 query tokens (positions q_pos[i], device int32 [n_q]) over the
 * listed pages, causal.  K/V tiles are dequantized in shared memory into an f16 high part
 * (code x scale rounded once; Q5_1 keys and Q4_1 values: code x scale + minimum, summed once
 * in fp32) and an f16 low part (the remainder, exact but for that fp32 sum); Q enters as Q/16 in
 * f16 (exact) and P as an f16 high part plus the rounded remainder.  QK^T (two MMAs per
 * k-step) and PV (three) run on tcgen05 tensor cores as CTA-pair MMAs with fp32
 * accumulation in tensor memory, so every operand carries about 22 significant bits.  The
 * keys are taken in splits of kv_split_tokens (a multiple of 128, at most 65,536; a CTA may
 * walk several consecutive splits); partial results are merged by log-sum-exp.  A page id
 * outside [0, n_pages) skips its page and records KVATTN_ERR_BAD_PAGE.  Takes every format
 * pair of the descriptor: Q8_0, Q4_0 or Q5_1 K with Q4_0 or Q8_0 V, and Q5_0 K with Q4_1 V
 * ([GUIDE] build step: the q8_0-q4_0 and q4_0-q4_0 pairs; [VULKAN] pitfalls: Q5_1 K with Q4_0
 * V; [MTP]: the Q5_0 K / Q4_1 V cache).
 *   q      device bf16 bits [n_q][H_q][256];  out device fp32 [n_q][H_q][256];
 *   lse    device fp32 [n_q][H_q];  page arguments as for kvattn_decode.
 *   ws     device workspace of kvattn_prefill_workspace_size() bytes. */
KVATTN_API size_t kvattn_prefill_workspace_size(const kvattn_kv_desc* desc, int n_q, int max_pages,
                                                int kv_split_tokens);
KVATTN_API int kvattn_prefill_chunk(const kvattn_kv_desc* desc, const uint16_t* q, int n_q,
                                    const int32_t* q_pos, const int32_t* page_list,
                                    const int32_t* page_logical, const int32_t* n_pages,
                                    int max_pages, int kv_split_tokens, float* out, float* lse,
                                    void* ws, size_t ws_bytes, kvattn_stream_t stream);

/* The same chunked prefill (arguments, formats, workspace and errors as kvattn_prefill_chunk)
 * with each dequantized K/V value and each P rounded once to f16 ([STREAM] method list; the
 * tiles are dequantized to 16-bit operands in shared memory): QK^T and PV take one MMA pass
 * each instead of two and three.  Every operand then carries 11 significant bits, so an
 * output row errs by up to about 2^-11 of the largest |value| it averages when few keys
 * dominate, and far less when many keys share the weight; kvattn_prefill_chunk keeps about 22
 * bits. */
KVATTN_API int kvattn_prefill_chunk_f16(const kvattn_kv_desc* desc, const uint16_t* q, int n_q,
                                        const int32_t* q_pos, const int32_t* page_list,
                                        const int32_t* page_logical, const int32_t* n_pages,
                                        int max_pages, int kv_split_tokens, float* out,
                                        float* lse, void* ws, size_t ws_bytes,
                                        kvattn_stream_t stream);

/* ---- host page streaming ([STREAM]: full history in pinned host RAM, working set over
 * PCIe; layer L+1 prefetched while layer L computes) ----------------------------------
 * Copies n pages from a pinned host pool to device slots with cudaMemcpyAsync on
 * copy_stream, merging runs where both the host page id and the device slot increase by
 * one.  Page i: host_pool + host_ids[i]*host_stride -> dev_pool + dev_slots[i]*dev_stride,
 * page_bytes bytes.  host_ids and dev_slots are HOST arrays.  If `done` is non-null it is
 * recorded on copy_stream after the last copy.  Returns the number of copies issued through
 * *n_copies when non-null. */
KVATTN_API int kvattn_stream_pages(const void* host_pool, int64_t host_stride, void* dev_pool,
                                   int64_t dev_stride, int64_t page_bytes, const int32_t* host_ids,
                                   const int32_t* dev_slots, int n, kvattn_stream_t copy_stream,
                                   kvattn_event_t done, int* n_copies);

/* The copy plan of kvattn_stream_pages, computed on the host without touching the GPU:
 * splits the n (host id, device slot) pairs into maximal runs in which both increase by one.
 * Writes up to max_runs (first index, length) pairs into run_first / run_len (HOST arrays,
 * may be NULL when max_runs is 0) and returns the number of runs (or a negative status). */
KVATTN_API int kvattn_stream_plan(const int32_t* host_ids, const int32_t* dev_slots, int n, int32_t* run_first,
                                  int32_t* run_len, int max_runs);

/* Moves pages between a pinned host pool and device slots with a copy kernel that reads (or
 * writes) the device-mapped host memory directly over PCIe.  The page lists live in device
 * memory, so a selection computed on the GPU (kvattn_select_blocks) drives the copy with no
 * host round trip; with n_ctas small the copy shares the GPU with attention running on
 * another stream.
 *   host_pool   pinned host memory (cudaHostAlloc or registered; mapped into the device
 *               address space), n_host_pages pages of host_stride bytes.  Checked on the host:
 *               anything else (e.g. pageable memory) returns KVATTN_ERR_INVALID_ARG.
 *   dev_pool    device memory, n_slots slots of dev_stride bytes
 *   host_ids    device int32 [n]: host page of entry i;  dev_slots device int32 [n]: its slot;
 *               entries with a negative slot are skipped; ids out of range are skipped and
 *               set KVATTN_ERR_BAD_PAGE in the device error word
 *   page_bytes  bytes per page, a multiple of 16 (strides and pointers 16-byte aligned)
 *   n_ctas      CTAs of the copy kernel (0 = 32)
 * kvattn_gather_pages copies host -> device, kvattn_scatter_pages device -> host. */
KVATTN_API int kvattn_gather_pages(const void* host_pool, int64_t host_stride, int64_t n_host_pages, void* dev_pool,
                                   int64_t dev_stride, int64_t n_slots, int64_t page_bytes, const int32_t* host_ids,
                                   const int32_t* dev_slots, int n, int n_ctas, kvattn_stream_t stream);
KVATTN_API int kvattn_scatter_pages(void* host_pool, int64_t host_stride, int64_t n_host_pages, const void* dev_pool,
                                    int64_t dev_stride, int64_t n_slots, int64_t page_bytes, const int32_t* host_ids,
                                    const int32_t* dev_slots, int n, int n_ctas, kvattn_stream_t stream);

/* ---- attention rotation ([VULKAN] pitfalls, the attention-rotation item: the rotation
 * improves the precision of quantized KV) ------------------------------------------------
 * out[r] = in[r] R for `rows` rows of 256 fp32 values, R = H_256 / 16 with H the
 * Sylvester-Hadamard matrix (H[i][j] = (-1)^popcount(i & j)).  R is symmetric, orthonormal
 * and its own inverse.  The rotated pipeline: rotate K and V before kvattn_quantize_append,
 * rotate Q before kvattn_decode / kvattn_prefill_chunk (scores are unchanged in exact
 * arithmetic), rotate the output back with the same call; outlier channels are spread across
 * the block before quantization.  in == out is allowed; both 16-byte aligned.  fp32
 * butterflies: each output is within ~8 ulp-scale roundings of the exact product. */
KVATTN_API int kvattn_hadamard(const float* in, float* out, int64_t rows, kvattn_stream_t stream);

/* ---- resident-page reuse ([KVMEM] recall section: the GPU working set follows the
 * retrieval query; a block already on the GPU is not copied again) ---------------------
 * Per unit (layer, KV head) a pool of n_slots device pages, pool page first_page + unit *
 * n_slots + s for slot s.  For the selection of each unit (sel_logical, ascending and unique,
 * as kvattn_select_blocks writes it):
 *   - a selected block that is resident keeps its slot;
 *   - free slots are the empty ones and those holding a block that is not selected;
 *   - misses (selected, not resident), in ascending block order, take the free slots in
 *     ascending slot order; blocks evicted this way are no longer resident.
 * Blocks >= n_full (the tail page) are not managed; their page-list entry is
 * extra_page[unit].
 *   sel_logical   device int32 [n_units][cap];  n_sel device int32 [n_units]
 *   slot_of_block device int32 [n_units][n_blocks], -1 = not resident (state; the caller
 *                 fills it with -1 once and then only passes it back)
 *   block_of_slot device int32 [n_units][n_slots], -1 = empty (state, likewise)
 *   host_page_of_block device int32 [n_units][n_blocks]: host page id of each block
 *   page_list     device int32 [n_units][cap] out: pool page holding each selected block
 *                 (a kvattn_decode page list, with sel_logical as its page_logical)
 *   copy_host, copy_dst device int32 [n_units][cap] out: host page and pool page of every
 *                 miss, copy_dst = -1 past n_copies[unit] (ready for kvattn_gather_pages
 *                 with n = n_units * cap)
 *   n_copies      device int32 [n_units] out
 * n_slots must be >= the number of managed selected blocks; otherwise the unit is left
 * unchanged, n_copies = 0 and KVATTN_ERR_INVALID_ARG is set in the device error word.
 * Limits: n_blocks <= 262,144, n_slots <= 16,384.  Asynchronous on `stream`. */
KVATTN_API int kvattn_resident_update(const int32_t* sel_logical, const int32_t* n_sel, int cap, int n_units,
                                      int n_blocks, int n_full, int32_t* slot_of_block, int32_t* block_of_slot,
                                      int n_slots, const int32_t* host_page_of_block, int64_t first_page,
                                      const int32_t* extra_page, int32_t* page_list, int32_t* copy_host,
                                      int32_t* copy_dst, int32_t* n_copies, kvattn_stream_t stream);

/* Polls `event` until it completes or timeout_ms elapses (KVATTN_ERR_TIMEOUT). */
KVATTN_API int kvattn_stream_wait(kvattn_event_t event, int timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* KVATTN_H */
