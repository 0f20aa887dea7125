/*
 * csa.h -- C ABI of libcsa.so: C4 compressed sparse attention (DeepSeek-V4
 * style) for NVIDIA B200 (sm_100a).
 *
 * The pages this library follows, cited by title and section:
 *   [T] "Token 的一生：DSV4 架构与 DSpark" (SGLang DSV4 internals article):
 *       §1 从 DSA 到 DSV4, §2.1 什么是 C4, §2.2 C4 KV Cache 的尺寸,
 *       §3.1 FP4 量化支持, §3.2 Top-512 变换, §4 Hadamard 旋转
 *   [H] "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）：將百萬標記長上下文變為可用資源":
 *       section "Compressed Sparse Attention（CSA）" and section
 *       "低精度與儲存策略的配合"
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is DEVICE memory owned by the caller, unless its
 *    comment says otherwise.  The library never allocates device memory;
 *    scratch space comes from a caller-provided workspace whose size the
 *    matching *_workspace_size() call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream.
 *  - Return value: CSA_OK once the work is enqueued.  Arguments that are
 *    wrong on their face (null required pointer, unsupported size, format or
 *    page size) return CSA_ERR_INVALID / CSA_ERR_UNSUPPORTED before anything is
 *    launched; a failed launch returns CSA_ERR_CUDA.
 *  - `status` (nullable, one int32 in device memory): problems only the
 *    device can see -- a page id or slot out of range, a NaN logit, a length
 *    above the stated maximum -- are recorded there as a csa_status_t (the
 *    first one wins) and the offending element is skipped.  No kernel traps.
 *    The caller zeroes *status and reads it after synchronising.
 *  - Paging ([T] §2.2): a page holds PAGE_SIZE = 256 raw tokens; physical
 *    page p of the compressed cache holds the 64 compressed rows of raw page
 *    p, so one page table [bs, page_table_stride] (int32 physical page ids)
 *    serves both caches.  Raw position r of request b lives in raw slot
 *      page_table[b*stride + r/256]*256 + r%256,
 *    compressed index s in compressed slot
 *      page_table[b*stride + s/64]*64 + s%64.
 *  - A request with L raw tokens (its query tokens included) has
 *    c4_seq_lens[b] = floor(L/4) compressed rows ([T] §2.2).  A query at raw
 *    position p sees the compressed rows s < floor((p+1)/4) (blocks whose four
 *    tokens are all at or before p) and the raw window [max(0,p-W+1), p].
 *  - Query tokens are packed request-major: request b owns query rows
 *    cu_q[b] .. cu_q[b+1]-1 (cu_q has bs+1 entries, cu_q[0] = 0).  q_pos
 *    [num_q] gives each query row's raw position.  Where a call accepts
 *    q_pos = NULL, every request has exactly one query row, the decode token
 *    at position L-1, so that it sees all floor(L/4) compressed rows.
 *
 * Storage formats
 * ---------------
 *  KV row ([H] "低精度與儲存策略的配合": FP8 for most entries, BF16 for RoPE),
 *  576 channels = 512 latent + 64 RoPE; values are the 512 latent channels:
 *    CSA_FMT_FP8 : 656 bytes = 512 E4M3 codes | 4 fp32 scales (one per 128
 *                  latent channels, scale = amax/448, 1 for an all-zero block)
 *                  | 64 bf16 RoPE values
 *    CSA_FMT_BF16: 1152 bytes = 576 bf16 values
 *  Index rows (queries and keys after the Hadamard rotation, [T] §3.1, §4),
 *  dim Di in {64, 128}; each array is indexed by row (query row or slot):
 *    CSA_FMT_BF16: codes = Di bf16;            no scales
 *    CSA_FMT_FP8 : codes = Di E4M3 bytes;       scales[row] fp32 = amax/448
 *    CSA_FMT_FP4 : codes = Di/2 bytes, two E2M1 codes per byte (element 2i in
 *                  the low nibble); block_scales = Di/16 unsigned-E4M3 bytes,
 *                  sb = RN(amax_blk/(6*s)); scales[row] fp32 s = amax/2688
 *    CSA_FMT_FP4_PAGE (index keys only): the FP4 values, codes and scales of
 *                  the 64 keys of one compressed page (slots 64p .. 64p+63)
 *                  kept together in one record of R = 36*Di + 256 bytes at
 *                  byte p*R of the `k_codes` array (2560 bytes for Di = 64,
 *                  4864 for Di = 128; k_block_scales and k_scales unused).
 *                  The record is 8 groups of 8 keys, group g (keys 8g..8g+7)
 *                  at byte g*Gb with Gb = 4.5*Di + 32; for key r (= slot%64,
 *                  i = r%8) in group g = r/8:
 *                    code byte b at    g*Gb + (b/16)*128 + i*16 + b%16
 *                                      (8-key x 16-byte blocks, the tensor
 *                                      cores' unswizzled operand order)
 *                    block scale j at  g*Gb + 4*Di + i*Di/16 + j
 *                    fp32 row scale at g*Gb + 4.5*Di + 4*i
 *                  so that one copy moves a page and two pages side by side
 *                  keep one stride between groups.  Queries stay CSA_FMT_FP4.
 *  Every quantised value is rounded to nearest, ties to even, saturating.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID = 1,      /* bad argument found on the host; nothing launched   */
    CSA_ERR_UNSUPPORTED = 2,  /* well-formed but unsupported size/format            */
    CSA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed        */
    CSA_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up                 */
    CSA_ERR_BOUNDS = 5,       /* device saw an index/slot/length out of range       */
    CSA_ERR_NAN = 6,          /* device saw a NaN logit (ordered as -inf)           */
    CSA_ERR_WORKSPACE = 7     /* workspace pointer null or smaller than required    */
} csa_status_t;

typedef enum {
    CSA_FMT_BF16 = 0,
    CSA_FMT_FP8 = 1,          /* E4M3 */
    CSA_FMT_FP4 = 2,          /* E2M1 with block-16 unsigned-E4M3 scales */
    CSA_FMT_F32 = 3,          /* input-only: float32 */
    CSA_FMT_FP4_PAGE = 4      /* index keys: FP4 in one record per 64-key page */
} csa_fmt_t;

/* What csa_c4_compress writes. */
typedef enum {
    CSA_OUT_KV_BF16 = 0,      /* dim 576, KV row in CSA_FMT_BF16 into the compressed KV cache */
    CSA_OUT_KV_FP8 = 1,       /* dim 576, KV row in CSA_FMT_FP8                               */
    CSA_OUT_INDEX_BF16 = 2,   /* dim 64/128, rotated index key, bf16 codes                    */
    CSA_OUT_INDEX_FP8 = 3,    /* dim 64/128, rotated index key, FP8 codes + row scale          */
    CSA_OUT_INDEX_FP4 = 4,    /* dim 64/128, rotated index key, FP4 codes + block/row scales   */
    CSA_OUT_INDEX_FP4_PAGE = 5 /* dim 64/128, rotated index key into CSA_FMT_FP4_PAGE records  */
} csa_out_kind_t;

enum { CSA_TOPK = 512, CSA_PAGE_SIZE = 256, CSA_C4_PAGE_SIZE = 64, CSA_C4_RATIO = 4,
       CSA_KV_DIM = 576, CSA_KV_LATENT = 512, CSA_KV_ROPE = 64 };

/* Human-readable name of a status code (static storage). */
const char *csa_status_string(csa_status_t s);

/* ABI version of this header (bumped on any signature change). */
int32_t csa_abi_version(void);

/* Bytes of one KV row in `kv_fmt` (656 or 1152), 0 for an unknown format. */
int32_t csa_kv_row_bytes(int32_t kv_fmt);

/*
 * csa_kv_store -- write raw or compressed KV rows into a paged KV cache.
 * ([H] "低精度與儲存策略的配合": FP8 latent with BF16 RoPE.)
 *   rows      [n, 576] float32, row-major
 *   slots     [n] int32 destination row of each input row; negative = skip
 *   kv_fmt    CSA_FMT_FP8 or CSA_FMT_BF16
 *   cache     [num_slots, csa_kv_row_bytes(kv_fmt)] bytes
 * A slot >= num_slots records CSA_ERR_BOUNDS and is skipped.
 */
csa_status_t csa_kv_store(const float *rows, int64_t n, const int32_t *slots, int32_t kv_fmt,
                          void *cache, int64_t num_slots, int32_t *status, void *stream);

/*
 * csa_c4_compress -- step 1, the C4 compressor ([T] §2.1; [H] "Compressed
 * Sparse Attention（CSA）": softmax-gated pooling with a learned positional
 * bias).  Block j of a request pools raw rows 4j..4j+3:
 *   alpha_i[c] = softmax_i(gate[4j+i][c] + bias[i][c]),  y[j][c] = sum_i alpha_i[c] x[4j+i][c]
 * computed in float32 and rounded once into the output format.  Only
 * complete blocks are written (a block is compressed when its fourth token
 * arrives); trailing rows of an incomplete block are ignored.
 *   x, gate   [cu_x[bs], dim] float32: the new raw rows of every request,
 *             request b owning rows cu_x[b] .. cu_x[b+1]-1 (host copy of the
 *             total: total_rows)
 *   bias      [4, dim] float32, indexed by position inside the block
 *   start_pos [bs] raw position of each request's first new row; must be a
 *             multiple of 4 (else CSA_ERR_BOUNDS for that request)
 *   max_rows_per_req  host upper bound on cu_x[b+1]-cu_x[b]; rows beyond it
 *             record CSA_ERR_BOUNDS and are not compressed
 *   out_kind  see csa_out_kind_t.  KV kinds need dim = 576 and write `out`
 *             as KV rows of a compressed KV cache.  INDEX kinds need dim 64 or
 *             128 and apply the Hadamard rotation (1/sqrt(dim)) H x ([T] §4)
 *             before quantising into the index-key arrays out (codes),
 *             out_block_scales (FP4 only) and out_scales (FP8/FP4).
 *   Compressed index j of request b is written to compressed slot
 *   page_table[b*stride + j/64]*64 + j%64 (< num_slots).
 */
csa_status_t csa_c4_compress(const float *x, const float *gate, const float *bias, int32_t dim,
                             int32_t bs, const int32_t *cu_x, int64_t total_rows,
                             const int32_t *start_pos, int32_t max_rows_per_req,
                             const int32_t *page_table, int32_t page_table_stride,
                             int32_t out_kind, void *out, uint8_t *out_block_scales,
                             float *out_scales, int64_t num_slots, int32_t *status, void *stream);

/*
 * csa_hadamard_quant -- the rotation and quantisation of index queries or
 * keys ([T] §3.1 fused_q_indexer_rope_hadamard[_fp4]_quant, §4; the RoPE step
 * is upstream of this call): x' = (1/sqrt(dim)) H_dim x per row, then
 * quantised to `fmt` as described above.
 *   x         [rows, dim] in x_dtype (CSA_FMT_BF16 or CSA_FMT_F32)
 *   dim       64 or 128
 *   row_map   nullable [rows] int32: output row of input row r (for writing
 *             keys straight into a paged index cache); NULL = identity.
 *             Negative = skip; >= num_out_rows records CSA_ERR_BOUNDS.
 *   codes, block_scales, scales: output arrays indexed by output row
 *   w_in/w_out nullable [rows] float32, indexed by INPUT row: the head-gate
 *             fusion of [T] §3.1: w_out[r] = w_in[r] * scales[r] (the row
 *             scale is positive, so it commutes with the indexer's ReLU);
 *             for bf16 w_out = w_in.
 */
csa_status_t csa_hadamard_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                                int32_t fmt, const int32_t *row_map, int64_t num_out_rows,
                                void *codes, uint8_t *block_scales, float *scales,
                                const float *w_in, float *w_out, int32_t *status, void *stream);

/*
 * csa_indexer_logits -- step 2, the C4 indexer scores ([T] §1, §3.1;
 * [H] "Compressed Sparse Attention（CSA）": a light indexer in low precision):
 *   logits[t][s] = k_scale[s] * sum_h w'[t][h] * ReLU(qhat[t][h] . khat[s])
 * where qhat/khat are the stored codes' values (FP4: times their block
 * scales) and w' = w * q_scale already folds the query's row scale in
 * (csa_hadamard_quant's w_out).  Accumulation in float32.
 *   q_codes        [num_q, idx_heads, code bytes of one row]
 *   q_block_scales [num_q, idx_heads, dim/16] (FP4 only, else NULL)
 *   q_weights      [num_q, idx_heads] float32 (w')
 *   k_codes, k_block_scales, k_scales: the index-key arrays, indexed by
 *                  compressed slot (< num_slots)
 *   q_pos          nullable [num_q]: query raw positions (causal visibility
 *                  n_vis = min(c4_seq_lens[b], floor((p+1)/4))); NULL means
 *                  n_vis = c4_seq_lens[b]
 *   max_c4_len     host upper bound on c4_seq_lens[] (grid sizing); longer
 *                  rows record CSA_ERR_BOUNDS and are truncated
 *   logits         [num_q, logits_stride] float32; entries s >= n_vis of a
 *                  row are not written
 */
csa_status_t csa_indexer_logits(const void *q_codes, const uint8_t *q_block_scales,
                                const float *q_weights, int32_t num_q, int32_t idx_heads,
                                int32_t idx_dim, int32_t fmt, const void *k_codes,
                                const uint8_t *k_block_scales, const float *k_scales,
                                int64_t num_slots, const int32_t *page_table,
                                int32_t page_table_stride, const int32_t *c4_seq_lens,
                                int32_t bs, const int32_t *cu_q, const int32_t *q_pos,
                                int32_t max_c4_len, float *logits, int64_t logits_stride,
                                int32_t *status, void *stream);

/*
 * csa_topk512_page_transform -- step 3, topk_transform_512 ([T] §3.2, with
 * the page arithmetic of §2.2).  For each query row t of request b: among
 * the first n_vis logits (n_vis as in csa_indexer_logits) select the
 * min(512, n_vis) largest, ties broken toward the lower index (-0 == +0;
 * a NaN records CSA_ERR_NAN and ranks below -inf), and write them in
 * ascending logical order followed by -1 padding:
 *   c4_sparse_page_indices[t][i] = page_table[b*stride + s/64]*64 + s%64
 *   raw_indices[t][i]            = s            (nullable output)
 *   c4_page_size   must be 64 (= 256/4)
 *   workspace      >= csa_topk512_workspace_size(num_q, max_c4_len) bytes
 *                  (always checked; written only when max_c4_len > 49152, the
 *                  rows shorter than that being selected in one launch)
 * Up to 74 rows of 8193..32768 keys are selected by a thread-block cluster
 * of 4 CTAs per row (2 CTAs above 37 rows) that share the row's keys: their
 * group maxima give each CTA a bound, the keys above the lowest bound are
 * gathered into the first CTA through distributed shared memory, and it
 * selects among them.  Other rows of at most 49152 keys take one CTA per row.
 * Rows longer than 49152 keys are selected in several launches: with at most
 * 64 rows, a bound-first selection spread over every SM (the maxima of about
 * 1024-2048 groups of consecutive keys give a lower bound of the 512th key,
 * only the keys above it are kept, then one CTA per row selects among them);
 * with more rows, a per-chunk top-512 and a per-row merge.  The kernels of
 * this step read cu_q, q_pos and c4_seq_lens before waiting for the kernels
 * enqueued before them: the ordering rule of csa_sparse_mqa_decode applies to
 * those three inputs.
 */
size_t csa_topk512_workspace_size(int32_t num_q, int32_t max_c4_len);
csa_status_t csa_topk512_page_transform(const float *logits, int64_t logits_stride,
                                        int32_t num_q, const int32_t *c4_seq_lens, int32_t bs,
                                        const int32_t *cu_q, const int32_t *q_pos,
                                        const int32_t *page_table, int32_t page_table_stride,
                                        int64_t num_slots, int32_t c4_page_size,
                                        int32_t max_c4_len, int32_t *c4_sparse_page_indices,
                                        int32_t *raw_indices, void *workspace,
                                        size_t workspace_bytes, int32_t *status, void *stream);

/*
 * csa_topk512_page_transform_noalloc -- the same selection and page transform
 * as csa_topk512_page_transform, for callers that cannot hand the library a
 * workspace or call the device allocator when they make the call: plugin and
 * operator interfaces that pass only input and output buffers, or hot paths
 * that must never reach cudaMalloc.  The pages have no counterpart of this
 * entry point; it exists for those callers only.
 *
 * Scratch lives in one file-scope device array of CSA_TOPK_NOALLOC_MAX_BYTES
 * bytes inside libcsa.so: every GPU that loads the library holds that memory
 * until the process exits.  The first call on a device (with that device
 * current) looks up the array's device address once and caches it for the
 * process; make that first call before any stream capture.  The cached
 * address belongs to the device's context of that time: after cudaDeviceReset
 * on a device, do not call this entry point again in the same process (load
 * the library in a fresh process).  Rows of at most 49152 compressed keys are
 * selected in one launch that needs no scratch, so any number of them is
 * accepted; longer rows use the bound-first selection when its buffers fit
 * the array, else the per-chunk selection and merge, and calls return
 * CSA_ERR_WORKSPACE without launching when that one does not fit either.
 * Every call shares the one array (its contents persist between calls and
 * nothing in it needs to start at zero), so calls that overlap on the GPU --
 * on different streams, or from several threads -- race and must be ordered
 * by the caller.  Never calls cudaMalloc, cudaFree or any allocating routine.
 * Arguments are those of csa_topk512_page_transform without the workspace.
 */
enum { CSA_TOPK_NOALLOC_MAX_BYTES = 16 << 20 };
csa_status_t csa_topk512_page_transform_noalloc(const float *logits, int64_t logits_stride,
                                                int32_t num_q, const int32_t *c4_seq_lens,
                                                int32_t bs, const int32_t *cu_q,
                                                const int32_t *q_pos, const int32_t *page_table,
                                                int32_t page_table_stride, int64_t num_slots,
                                                int32_t c4_page_size, int32_t max_c4_len,
                                                int32_t *c4_sparse_page_indices,
                                                int32_t *raw_indices, int32_t *status,
                                                void *stream);

/*
 * csa_indexer_topk512 -- steps 2 and 3 in one call: the indexer logits of
 * csa_indexer_logits followed by the selection and page transform of
 * csa_topk512_page_transform, with the same arguments and the same results
 * (logits, c4_sparse_page_indices and raw_indices are those the two calls
 * would write, bit for bit).  Where the tensor-core indexer applies (index dim
 * 64 or 128, 16-byte aligned key codes, num_slots a positive multiple of 64),
 * each indexer CTA selects the top-512 of its own chunk of keys right after
 * computing them (the logits come back from L2 into the CTA's drained
 * shared-memory stages), and one row-level merge follows: the separate
 * chunk-selection launch and its re-read of the logits disappear.  Where rows
 * are cut into pieces longer than 64 key tiles (many query rows per request,
 * as in chunked prefill) the call runs the two separate steps instead.  This
 * fusion is the design's own step beyond the pages, which keep the indexer and
 * topk_transform_512 as separate operations ("Token 的一生" §3.2).
 *   logits       [num_q, logits_stride] fp32, written (logits_stride >= max_c4_len)
 *   workspace    >= csa_indexer_topk512_workspace_size(num_q, bs, idx_heads,
 *                   idx_dim, fmt, max_c4_len) bytes (the size depends on the
 *                   current device's SM count; query it on the device that runs)
 * Errors as for the two separate calls.
 */
size_t csa_indexer_topk512_workspace_size(int32_t num_q, int32_t bs, int32_t idx_heads,
                                          int32_t idx_dim, int32_t fmt, int32_t max_c4_len);
csa_status_t csa_indexer_topk512(const void *q_codes, const uint8_t *q_block_scales,
                                 const float *q_weights, int32_t num_q, int32_t idx_heads,
                                 int32_t idx_dim, int32_t fmt, const void *k_codes,
                                 const uint8_t *k_block_scales, const float *k_scales,
                                 int64_t num_slots, const int32_t *page_table,
                                 int32_t page_table_stride, const int32_t *c4_seq_lens, int32_t bs,
                                 const int32_t *cu_q, const int32_t *q_pos, int32_t max_c4_len,
                                 int32_t c4_page_size, float *logits, int64_t logits_stride,
                                 int32_t *c4_sparse_page_indices, int32_t *raw_indices,
                                 void *workspace, size_t workspace_bytes, int32_t *status,
                                 void *stream);

/*
 * csa_indexer_select + csa_topk512_merge -- the two launches of
 * csa_indexer_topk512 as separate calls (same arguments, same results), for
 * callers that schedule or time them apart.  csa_indexer_select writes the
 * logits and, in `workspace`, each chunk's top-512 candidates; it returns
 * CSA_ERR_UNSUPPORTED (launching nothing) where csa_indexer_topk512 would not
 * fuse -- use csa_indexer_logits + csa_topk512_page_transform there.
 * csa_topk512_merge reads that workspace: it must get the same shape arguments
 * (num_q, idx_heads, idx_dim, fmt, bs, max_c4_len), the same device and the
 * workspace untouched in between.
 */
csa_status_t csa_indexer_select(const void *q_codes, const uint8_t *q_block_scales,
                                const float *q_weights, int32_t num_q, int32_t idx_heads,
                                int32_t idx_dim, int32_t fmt, const void *k_codes,
                                const uint8_t *k_block_scales, const float *k_scales,
                                int64_t num_slots, const int32_t *page_table,
                                int32_t page_table_stride, const int32_t *c4_seq_lens, int32_t bs,
                                const int32_t *cu_q, const int32_t *q_pos, int32_t max_c4_len,
                                float *logits, int64_t logits_stride, void *workspace,
                                size_t workspace_bytes, int32_t *status, void *stream);
csa_status_t csa_topk512_merge(int32_t num_q, int32_t idx_heads, int32_t idx_dim, int32_t fmt,
                               const int32_t *c4_seq_lens, int32_t bs, const int32_t *cu_q,
                               const int32_t *q_pos, const int32_t *page_table,
                               int32_t page_table_stride, int64_t num_slots,
                               int32_t c4_page_size, int32_t max_c4_len,
                               int32_t *c4_sparse_page_indices, int32_t *raw_indices,
                               const void *workspace, size_t workspace_bytes, int32_t *status,
                               void *stream);

/*
 * csa_sparse_mqa_decode / csa_sparse_mqa_prefill -- step 4, sparse attention
 * over the selected compressed rows joined with the sliding window of raw
 * rows under ONE softmax ([T] §1; [H] "Compressed Sparse Attention（CSA）").
 * For query t of request b at raw position p and head h, with key rows
 *   S = { compressed slot c4_sparse_page_indices[t][i] >= 0 }
 *     U { raw slot of r : max(0, p-window+1) <= r <= p }:
 *   z_r = sm_scale * q[t][h] . key_r (576 dims),
 *   out[t][h] = sum_r softmax(z)_r * key_r[0:512],  lse[t][h] = ln sum_r exp(z_r).
 * A raw token may appear both in the window and inside a selected
 * compressed row; both count.
 *   q         [num_q, heads, 576] bf16;  heads in {16, 32, 64, 128}
 *   c4_cache  [num_c4_slots, row bytes]; raw_cache [num_raw_slots, row bytes]
 *   seq_lens  [bs] raw lengths L (q_pos NULL => one query per request at L-1)
 *   window    0..1024
 *   out       [num_q, heads, 512] bf16;  lse nullable [num_q, heads] float32
 *   workspace >= csa_sparse_mqa_workspace_size(num_q, heads, window, decode)
 * The two entry points compute the same function; _decode splits each
 * query's rows across CTAs (few queries, many rows each), _prefill gives each
 * query its own CTA (many queries).  FP8 rows with heads a multiple of 64 run
 * on the tensor-core kernel, whose splits (a thread-block cluster of at most 8
 * CTAs per query) merge inside the kernel and use no workspace (the partial
 * outputs cross the cluster as fp16 under a shared power of two, rounded to
 * at most 2^-11 relative, and are summed in fp32); the other
 * cases write split partials to the workspace and merge them in a second
 * launch.
 * Ordering: like every kernel of the library this one is launched with
 * programmatic dependent launch; with FP8 rows it reads q, cu_q, q_pos and
 * seq_lens before waiting for the kernels enqueued before it.  A chain of
 * launches that each let their successor start early can have several of
 * them running at once, so these inputs must not be written by any such
 * early-triggering kernel enqueued on the stream since the last ordinary
 * launch, copy or event wait (the library's own kernels never write them;
 * data written by a copy, or by work ordered before that point, is safe).
 */
size_t csa_sparse_mqa_workspace_size(int32_t num_q, int32_t heads, int32_t window,
                                     int32_t decode);
csa_status_t csa_sparse_mqa_decode(const void *q, int32_t num_q, int32_t heads,
                                   const void *c4_cache, const void *raw_cache, int32_t kv_fmt,
                                   int64_t num_c4_slots, int64_t num_raw_slots,
                                   const int32_t *c4_sparse_page_indices,
                                   const int32_t *page_table, int32_t page_table_stride,
                                   const int32_t *seq_lens, int32_t bs, const int32_t *cu_q,
                                   const int32_t *q_pos, int32_t window, float sm_scale,
                                   void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, int32_t *status, void *stream);
csa_status_t csa_sparse_mqa_prefill(const void *q, int32_t num_q, int32_t heads,
                                    const void *c4_cache, const void *raw_cache, int32_t kv_fmt,
                                    int64_t num_c4_slots, int64_t num_raw_slots,
                                    const int32_t *c4_sparse_page_indices,
                                    const int32_t *page_table, int32_t page_table_stride,
                                    const int32_t *seq_lens, int32_t bs, const int32_t *cu_q,
                                    const int32_t *q_pos, int32_t window, float sm_scale,
                                    void *out, float *lse, void *workspace,
                                    size_t workspace_bytes, int32_t *status, void *stream);

/*
 * HCA branch ("DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section "Heavily
 * Compressed Attention（HCA）": about 128x compression, then dense attention over
 * the compressed blocks).  The design's next row beyond the CSA path.
 *
 * csa_hca_compress -- csa_c4_compress with blocks of CSA_HCA_RATIO = 128 raw
 * rows: per channel, alpha_i = softmax_i(gate[128j+i] + bias[i]) over the
 * block, row j = sum_i alpha_i x[128j+i], produced only for complete blocks.
 *   bias         [128, 576] fp32
 *   start_pos    per request, a multiple of 128
 *   out          HCA KV cache, packed rows (out_kind CSA_OUT_KV_BF16 or _FP8, the
 *                layouts of csa_kv_store); row j of request b at slot
 *                page_table[b*stride + j/2]*2 + j%2 (CSA_HCA_PAGE_SIZE = 256/128
 *                compressed rows per 256-token page; the same page table as
 *                the raw cache)
 *   num_slots    rows of `out`
 * Other arguments and errors as csa_c4_compress.
 *
 * csa_hca_attention -- dense attention of each query over all its visible HCA
 * rows s < floor((p+1)/128) (and s < floor(seq_len/128)) joined with the raw
 * window [p-W+1, p] under one softmax (the window is this design's reading:
 * the pages describe it for CSA; window 0 gives the compressed rows alone).
 * Arguments as csa_sparse_mqa_decode without the index list, plus
 *   max_hca_len  an upper bound of any query's visible HCA rows;
 *                max_hca_len + window <= CSA_HCA_MAX_ROWS
 *   decode       1: few query rows per request (rows split over CTAs), 0: prefill
 *   workspace    >= csa_hca_attention_workspace_size(num_q, heads, window,
 *                   decode, max_hca_len) bytes
 */
enum { CSA_HCA_RATIO = 128, CSA_HCA_PAGE_SIZE = 2, CSA_HCA_MAX_ROWS = 16 * 48 * 32 };
csa_status_t csa_hca_compress(const float *x, const float *gate, const float *bias,
                              int32_t dim, int32_t bs, const int32_t *cu_x, int64_t total_rows,
                              const int32_t *start_pos, int32_t max_rows_per_req,
                              const int32_t *page_table, int32_t page_table_stride,
                              int32_t out_kind, void *out, int64_t num_slots, int32_t *status,
                              void *stream);
size_t csa_hca_attention_workspace_size(int32_t num_q, int32_t heads, int32_t window,
                                        int32_t decode, int32_t max_hca_len);
csa_status_t csa_hca_attention(const void *q, int32_t num_q, int32_t heads, const void *hca_cache,
                               const void *raw_cache, int32_t kv_fmt, int64_t num_hca_slots,
                               int64_t num_raw_slots, const int32_t *page_table,
                               int32_t page_table_stride, const int32_t *seq_lens, int32_t bs,
                               const int32_t *cu_q, const int32_t *q_pos, int32_t max_hca_len,
                               int32_t window, float sm_scale, int32_t decode, void *out,
                               float *lse, void *workspace, size_t workspace_bytes,
                               int32_t *status, void *stream);

/*
 * Fused rotary embedding ahead of the rotation + quantisation ([T] §3.1
 * fused_q_indexer_rope_hadamard[_fp4]_quant and §4: Q goes rope -> Hadamard ->
 * quant; K goes rope -> Hadamard -> quant -> index K cache).
 *
 * Rotary embedding: the leading rope_dim values of a row, taken as rope_dim/2
 * complex numbers x[2i] + i*x[2i+1], are multiplied by freqs_cis[pos][i]:
 *   x'[2i]   = x[2i]*cos - x[2i+1]*sin,   x'[2i+1] = x[2i]*sin + x[2i+1]*cos
 * (float32, each product and sum rounded separately); the remaining
 * dim - rope_dim values pass unchanged.
 *   freqs_cis   [max_pos, rope_dim/2, 2] float32 (cos, sin), 8-byte aligned,
 *               caller-owned; the library never builds the table
 *   rope_dim    even, 2 <= rope_dim <= dim
 *
 * csa_rope_hadamard_quant -- csa_hadamard_quant with the rotary embedding
 * first.  Row r of x sits at raw position positions[r / rows_per_pos]
 * (rows_per_pos = idx_heads for index queries laid out [num_q, idx_heads,
 * dim], 1 for keys).  A position outside [0, max_pos) records CSA_ERR_BOUNDS
 * and leaves that row unwritten (and its w_out).  Other arguments as
 * csa_hadamard_quant.
 */
csa_status_t csa_rope_hadamard_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                                     const float *freqs_cis, int32_t rope_dim, int32_t max_pos,
                                     const int32_t *positions, int32_t rows_per_pos, int32_t fmt,
                                     const int32_t *row_map, int64_t num_out_rows, void *codes,
                                     uint8_t *block_scales, float *scales, const float *w_in,
                                     float *w_out, int32_t *status, void *stream);

/*
 * csa_c4_compress_index_rope -- csa_c4_compress in an index-key mode
 * (out_kind CSA_OUT_INDEX_*) with the rotary embedding applied to each pooled
 * key between the pooling and the rotation, in the same pass: pool ->
 * rope -> Hadamard -> quant -> index K cache.  The compressed key of block j
 * (raw rows 4j..4j+3) takes the raw position 4j of the block's first row; a
 * position >= max_pos records CSA_ERR_BOUNDS and leaves the key unwritten.
 * Other arguments and errors as csa_c4_compress.
 */
csa_status_t csa_c4_compress_index_rope(const float *x, const float *gate, const float *bias,
                                        int32_t dim, int32_t bs, const int32_t *cu_x,
                                        int64_t total_rows, const int32_t *start_pos,
                                        int32_t max_rows_per_req, const int32_t *page_table,
                                        int32_t page_table_stride, int32_t out_kind,
                                        const float *freqs_cis, int32_t rope_dim,
                                        int32_t max_pos, void *out, uint8_t *out_block_scales,
                                        float *out_scales, int64_t num_slots, int32_t *status,
                                        void *stream);

/*
 * DSA comparison path ([T] §1 从 DSA 到 DSV4: the DSA indexer picks the top-k
 * raw tokens, no compression; its index K cache is FP8 (§3.1) and is not
 * Hadamard-rotated (§4); its pages hold 64 raw tokens).  The same kernels as
 * the C4 path with one key per raw token: a query at raw position p sees the
 * keys s <= p (s < min(seq_lens[b], p+1)), and key s of request b sits at
 * slot page_table[b*stride + s/64]*64 + s%64 of a cache paged by 64 tokens.
 * The attention over the selected raw rows is csa_sparse_mqa_decode/_prefill
 * with c4_cache = that 64-token-paged KV cache and window = 0.
 *
 * csa_index_quant -- csa_hadamard_quant without the rotation (the row is
 * quantised as given).
 *
 * csa_dsa_indexer_logits -- csa_indexer_logits over raw tokens: seq_lens are
 * raw lengths, n_vis = min(seq_lens[b], p+1), max_seq_len bounds seq_lens[].
 *
 * csa_dsa_topk512_page_transform -- csa_topk512_page_transform over raw
 * tokens (the same n_vis); page_size must be CSA_DSA_PAGE_SIZE (64); the
 * workspace is csa_topk512_workspace_size(num_q, max_seq_len) bytes.
 */
enum { CSA_DSA_PAGE_SIZE = 64 };

csa_status_t csa_index_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                             int32_t fmt, const int32_t *row_map, int64_t num_out_rows,
                             void *codes, uint8_t *block_scales, float *scales,
                             const float *w_in, float *w_out, int32_t *status, void *stream);
csa_status_t csa_dsa_indexer_logits(const void *q_codes, const uint8_t *q_block_scales,
                                    const float *q_weights, int32_t num_q, int32_t idx_heads,
                                    int32_t idx_dim, int32_t fmt, const void *k_codes,
                                    const uint8_t *k_block_scales, const float *k_scales,
                                    int64_t num_slots, const int32_t *page_table,
                                    int32_t page_table_stride, const int32_t *seq_lens,
                                    int32_t bs, const int32_t *cu_q, const int32_t *q_pos,
                                    int32_t max_seq_len, float *logits, int64_t logits_stride,
                                    int32_t *status, void *stream);
csa_status_t csa_dsa_topk512_page_transform(const float *logits, int64_t logits_stride,
                                            int32_t num_q, const int32_t *seq_lens, int32_t bs,
                                            const int32_t *cu_q, const int32_t *q_pos,
                                            const int32_t *page_table, int32_t page_table_stride,
                                            int64_t num_slots, int32_t page_size,
                                            int32_t max_seq_len, int32_t *sparse_page_indices,
                                            int32_t *raw_indices, void *workspace,
                                            size_t workspace_bytes, int32_t *status,
                                            void *stream);

/*
 * csa_workspace_size -- the workspace bytes of one operation, by operation
 * code (the per-operation *_workspace_size calls, behind one entry point):
 *   CSA_OP_TOPK512          csa_topk512_page_transform / csa_dsa_...: uses
 *                           max_rows (= num_q) and max_len
 *   CSA_OP_INDEXER_TOPK512  csa_indexer_topk512 / csa_indexer_select: uses
 *                           max_rows, bs, heads (= idx_heads), idx_dim, fmt, max_len
 *   CSA_OP_SPARSE_MQA       csa_sparse_mqa_decode/_prefill: uses max_rows,
 *                           heads, window, decode
 *   CSA_OP_HCA_ATTENTION    csa_hca_attention: uses max_rows, heads, window,
 *                           decode, max_len (= max_hca_len)
 * Unused arguments are ignored; an unknown op returns 0.
 */
enum { CSA_OP_TOPK512 = 1, CSA_OP_INDEXER_TOPK512 = 2, CSA_OP_SPARSE_MQA = 3,
       CSA_OP_HCA_ATTENTION = 4 };
size_t csa_workspace_size(int32_t op, int32_t bs, int32_t max_rows, int32_t max_len,
                          int32_t heads, int32_t window, int32_t decode, int32_t idx_dim,
                          int32_t fmt);

/*
 * csa_selftest_wait_timeout -- checks the library's bounded device waits: one
 * CTA waits on an mbarrier phase that nothing completes; the wait gives up
 * after the library's limit (1 s) and CSA_ERR_TIMEOUT is recorded in *status
 * (device int32, caller-owned; an earlier non-zero code is kept).  waited_ns
 * (nullable device int32) receives the time the wait took.  Asynchronous on
 * `stream`; the CUDA context stays usable.
 */
csa_status_t csa_selftest_wait_timeout(int32_t *status, int32_t *waited_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
