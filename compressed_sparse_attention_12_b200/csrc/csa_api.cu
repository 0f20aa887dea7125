// csa_api.cu -- the extern "C" entry points of libcsa.so (declared in
// include/csa.h): host-side argument validation, then the launchers.
#include <cuda_runtime.h>

#include "../../include/csa.h"
#include "launch.h"

namespace {

csa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

bool index_fmt_ok(int32_t fmt) {
    return fmt == CSA_FMT_BF16 || fmt == CSA_FMT_FP8 || fmt == CSA_FMT_FP4 ||
           fmt == CSA_FMT_FP4_PAGE;
}

// Paged FP4 keys are read by bulk copies of whole 64-key page records.
bool paged_keys_ok(int32_t fmt, const void *k_codes, int64_t num_slots) {
    return fmt != CSA_FMT_FP4_PAGE ||
           ((reinterpret_cast<uintptr_t>(k_codes) % 16) == 0 && num_slots % CSA_C4_PAGE_SIZE == 0);
}

// Formats whose queries carry FP4 block scales.
bool fp4_query(int32_t fmt) { return fmt == CSA_FMT_FP4 || fmt == CSA_FMT_FP4_PAGE; }

bool kv_fmt_ok(int32_t fmt) { return fmt == CSA_FMT_BF16 || fmt == CSA_FMT_FP8; }

// Scales that each index format needs next to its codes.
bool index_arrays_ok(int32_t fmt, const void *codes, const void *block_scales,
                     const void *scales) {
    if (!codes) return false;
    if (fmt == CSA_FMT_FP8 && !scales) return false;
    if (fmt == CSA_FMT_FP4 && (!scales || !block_scales)) return false;
    return true;       // CSA_FMT_FP4_PAGE: codes, block and row scales in one record array
}

}  // namespace

extern "C" {

const char *csa_status_string(csa_status_t s) {
    switch (s) {
        case CSA_OK: return "ok";
        case CSA_ERR_INVALID: return "invalid argument";
        case CSA_ERR_UNSUPPORTED: return "unsupported size or format";
        case CSA_ERR_CUDA: return "CUDA error";
        case CSA_ERR_TIMEOUT: return "device wait timed out";
        case CSA_ERR_BOUNDS: return "index, slot or length out of range";
        case CSA_ERR_NAN: return "NaN logit";
        case CSA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

int32_t csa_abi_version(void) { return 1; }

int32_t csa_kv_row_bytes(int32_t kv_fmt) {
    return kv_fmt == CSA_FMT_FP8 ? 656 : kv_fmt == CSA_FMT_BF16 ? 1152 : 0;
}

csa_status_t csa_kv_store(const float *rows, int64_t n, const int32_t *slots, int32_t kv_fmt,
                          void *cache, int64_t num_slots, int32_t *status, void *stream) {
    if (n < 0 || num_slots < 0) return CSA_ERR_INVALID;
    if (!kv_fmt_ok(kv_fmt)) return CSA_ERR_UNSUPPORTED;
    if (n == 0) return CSA_OK;
    if (!rows || !slots || !cache) return CSA_ERR_INVALID;
    return cuda_status(csa::launch_kv_store(rows, n, slots, kv_fmt, cache, num_slots, status,
                                            as_stream(stream)));
}

static bool rope_ok(const float *freqs_cis, int32_t rope_dim, int32_t max_pos, int32_t dim) {
    return freqs_cis && rope_dim > 0 && rope_dim <= dim && (rope_dim % 2) == 0 && max_pos > 0 &&
           (reinterpret_cast<uintptr_t>(freqs_cis) & 7) == 0;
}

static csa_status_t c4_compress(const float *x, const float *gate, const float *bias, int32_t dim,
                             int32_t bs, const int32_t *cu_x, int64_t total_rows,
                             const int32_t *start_pos, int32_t max_rows_per_req,
                             const int32_t *page_table, int32_t page_table_stride,
                             int32_t out_kind, void *out, uint8_t *out_block_scales,
                             float *out_scales, int64_t num_slots, int32_t *status,
                             void *stream, const csa::RopeArgs &rope) {
    if (bs < 0 || total_rows < 0 || max_rows_per_req < 0 || page_table_stride < 0)
        return CSA_ERR_INVALID;
    const bool kv = out_kind == CSA_OUT_KV_BF16 || out_kind == CSA_OUT_KV_FP8;
    const bool idx = out_kind == CSA_OUT_INDEX_BF16 || out_kind == CSA_OUT_INDEX_FP8 ||
                     out_kind == CSA_OUT_INDEX_FP4 || out_kind == CSA_OUT_INDEX_FP4_PAGE;
    if (!kv && !idx) return CSA_ERR_UNSUPPORTED;
    if (kv && dim != CSA_KV_DIM) return CSA_ERR_UNSUPPORTED;
    if (idx && dim != 64 && dim != 128) return CSA_ERR_UNSUPPORTED;
    if (bs == 0 || total_rows == 0 || max_rows_per_req < 4) return CSA_OK;
    if (!x || !gate || !bias || !cu_x || !start_pos || !page_table || !out) return CSA_ERR_INVALID;
    if (out_kind == CSA_OUT_INDEX_FP8 && !out_scales) return CSA_ERR_INVALID;
    if (out_kind == CSA_OUT_INDEX_FP4 && (!out_scales || !out_block_scales)) return CSA_ERR_INVALID;
    if (bs > 65535) return CSA_ERR_UNSUPPORTED;
    return cuda_status(csa::launch_c4_compress(x, gate, bias, dim, bs, cu_x, start_pos,
                                               max_rows_per_req, page_table, page_table_stride,
                                               out_kind, out, out_block_scales, out_scales,
                                               num_slots, status, as_stream(stream), rope));
}

csa_status_t csa_c4_compress(const float *x, const float *gate, const float *bias, int32_t dim,
                             int32_t bs, const int32_t *cu_x, int64_t total_rows,
                             const int32_t *start_pos, int32_t max_rows_per_req,
                             const int32_t *page_table, int32_t page_table_stride,
                             int32_t out_kind, void *out, uint8_t *out_block_scales,
                             float *out_scales, int64_t num_slots, int32_t *status,
                             void *stream) {
    return c4_compress(x, gate, bias, dim, bs, cu_x, total_rows, start_pos, max_rows_per_req,
                       page_table, page_table_stride, out_kind, out, out_block_scales, out_scales,
                       num_slots, status, stream, csa::RopeArgs());
}

csa_status_t csa_c4_compress_index_rope(const float *x, const float *gate, const float *bias,
                                        int32_t dim, int32_t bs, const int32_t *cu_x,
                                        int64_t total_rows, const int32_t *start_pos,
                                        int32_t max_rows_per_req, const int32_t *page_table,
                                        int32_t page_table_stride, int32_t out_kind,
                                        const float *freqs_cis, int32_t rope_dim,
                                        int32_t max_pos, void *out, uint8_t *out_block_scales,
                                        float *out_scales, int64_t num_slots, int32_t *status,
                                        void *stream) {
    if (out_kind != CSA_OUT_INDEX_BF16 && out_kind != CSA_OUT_INDEX_FP8 &&
        out_kind != CSA_OUT_INDEX_FP4 && out_kind != CSA_OUT_INDEX_FP4_PAGE)
        return CSA_ERR_UNSUPPORTED;
    if (!rope_ok(freqs_cis, rope_dim, max_pos, dim)) return CSA_ERR_INVALID;
    csa::RopeArgs rope;
    rope.freqs = reinterpret_cast<const float2 *>(freqs_cis);
    rope.rope_dim = rope_dim;
    rope.max_pos = max_pos;
    return c4_compress(x, gate, bias, dim, bs, cu_x, total_rows, start_pos, max_rows_per_req,
                       page_table, page_table_stride, out_kind, out, out_block_scales, out_scales,
                       num_slots, status, stream, rope);
}

csa_status_t csa_hca_compress(const float *x, const float *gate, const float *bias,
                              int32_t dim, int32_t bs, const int32_t *cu_x, int64_t total_rows,
                              const int32_t *start_pos, int32_t max_rows_per_req,
                              const int32_t *page_table, int32_t page_table_stride,
                              int32_t out_kind, void *out, int64_t num_slots, int32_t *status,
                              void *stream) {
    if (bs < 0 || total_rows < 0 || max_rows_per_req < 0 || page_table_stride < 0)
        return CSA_ERR_INVALID;
    if (out_kind != CSA_OUT_KV_BF16 && out_kind != CSA_OUT_KV_FP8) return CSA_ERR_UNSUPPORTED;
    if (dim != CSA_KV_DIM) return CSA_ERR_UNSUPPORTED;
    if (bs == 0 || total_rows == 0 || max_rows_per_req < CSA_HCA_RATIO) return CSA_OK;
    if (!x || !gate || !bias || !cu_x || !start_pos || !page_table || !out) return CSA_ERR_INVALID;
    if (bs > 65535 || max_rows_per_req / CSA_HCA_RATIO > 2147483647) return CSA_ERR_UNSUPPORTED;
    return cuda_status(csa::launch_hca_compress(x, gate, bias, bs, cu_x, start_pos,
                                                max_rows_per_req, page_table, page_table_stride,
                                                out_kind, out, num_slots, status,
                                                as_stream(stream)));
}

static csa_status_t index_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                                int32_t fmt, const int32_t *row_map, int64_t num_out_rows,
                                void *codes, uint8_t *block_scales, float *scales,
                                const float *w_in, float *w_out, int32_t *status, void *stream,
                                bool rotate, const csa::RopeArgs &rope) {
    if (rows < 0) return CSA_ERR_INVALID;
    if (x_dtype != CSA_FMT_BF16 && x_dtype != CSA_FMT_F32) return CSA_ERR_UNSUPPORTED;
    if (dim != 64 && dim != 128) return CSA_ERR_UNSUPPORTED;
    if (!index_fmt_ok(fmt)) return CSA_ERR_UNSUPPORTED;
    if (rows == 0) return CSA_OK;
    if (!x || !index_arrays_ok(fmt, codes, block_scales, scales)) return CSA_ERR_INVALID;
    if ((w_in == nullptr) != (w_out == nullptr)) return CSA_ERR_INVALID;
    if (row_map && num_out_rows < 0) return CSA_ERR_INVALID;
    return cuda_status(csa::launch_hadamard_quant(x, x_dtype, rows, dim, fmt, row_map,
                                                  num_out_rows, codes, block_scales, scales,
                                                  w_in, w_out, status, as_stream(stream), rotate,
                                                  rope));
}

csa_status_t csa_hadamard_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                                int32_t fmt, const int32_t *row_map, int64_t num_out_rows,
                                void *codes, uint8_t *block_scales, float *scales,
                                const float *w_in, float *w_out, int32_t *status, void *stream) {
    return index_quant(x, x_dtype, rows, dim, fmt, row_map, num_out_rows, codes, block_scales,
                       scales, w_in, w_out, status, stream, true, csa::RopeArgs());
}

csa_status_t csa_index_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                             int32_t fmt, const int32_t *row_map, int64_t num_out_rows,
                             void *codes, uint8_t *block_scales, float *scales,
                             const float *w_in, float *w_out, int32_t *status, void *stream) {
    return index_quant(x, x_dtype, rows, dim, fmt, row_map, num_out_rows, codes, block_scales,
                       scales, w_in, w_out, status, stream, false, csa::RopeArgs());
}

csa_status_t csa_rope_hadamard_quant(const void *x, int32_t x_dtype, int64_t rows, int32_t dim,
                                     const float *freqs_cis, int32_t rope_dim, int32_t max_pos,
                                     const int32_t *positions, int32_t rows_per_pos, int32_t fmt,
                                     const int32_t *row_map, int64_t num_out_rows, void *codes,
                                     uint8_t *block_scales, float *scales, const float *w_in,
                                     float *w_out, int32_t *status, void *stream) {
    if (rows < 0 || rows_per_pos < 1) return CSA_ERR_INVALID;
    if (rows == 0) return CSA_OK;
    if (!positions || !rope_ok(freqs_cis, rope_dim, max_pos, dim)) return CSA_ERR_INVALID;
    csa::RopeArgs rope;
    rope.freqs = reinterpret_cast<const float2 *>(freqs_cis);
    rope.pos = positions;
    rope.rope_dim = rope_dim;
    rope.max_pos = max_pos;
    rope.rows_per_pos = rows_per_pos;
    return index_quant(x, x_dtype, rows, dim, fmt, row_map, num_out_rows, codes, block_scales,
                       scales, w_in, w_out, status, stream, true, rope);
}

static csa_status_t indexer_logits(const void *q_codes, const uint8_t *q_block_scales,
                                const float *q_weights, int32_t num_q, int32_t idx_heads,
                                int32_t idx_dim, int32_t fmt, const void *k_codes,
                                const uint8_t *k_block_scales, const float *k_scales,
                                int64_t num_slots, const int32_t *page_table,
                                int32_t page_table_stride, const int32_t *c4_seq_lens,
                                int32_t bs, const int32_t *cu_q, const int32_t *q_pos,
                                int32_t max_c4_len, float *logits, int64_t logits_stride,
                                int32_t *status, void *stream, int ratio) {
    if (num_q < 0 || bs < 0 || max_c4_len < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (!index_fmt_ok(fmt)) return CSA_ERR_UNSUPPORTED;
    if (idx_dim != 64 && idx_dim != 128) return CSA_ERR_UNSUPPORTED;
    if (idx_heads < 1 || idx_heads > 128) return CSA_ERR_UNSUPPORTED;
    if (num_q == 0 || max_c4_len == 0) return CSA_OK;
    if (bs < 1 || !q_codes || !q_weights || !page_table || !c4_seq_lens || !cu_q || !logits)
        return CSA_ERR_INVALID;
    if (fp4_query(fmt) && !q_block_scales) return CSA_ERR_INVALID;
    if (!index_arrays_ok(fmt, k_codes, k_block_scales, k_scales)) return CSA_ERR_INVALID;
    if (!paged_keys_ok(fmt, k_codes, num_slots)) return CSA_ERR_UNSUPPORTED;
    if (logits_stride < max_c4_len) return CSA_ERR_INVALID;
    if (num_q > 65535) return CSA_ERR_UNSUPPORTED;
    csa::IndexerArgs a{q_codes, q_block_scales, q_weights, num_q, idx_heads, idx_dim, fmt,
                       k_codes, k_block_scales, k_scales, num_slots, page_table,
                       page_table_stride, c4_seq_lens, bs, cu_q, q_pos, max_c4_len, logits,
                       logits_stride, status};
    a.ratio = ratio;
    return cuda_status(csa::launch_indexer(a, as_stream(stream)));
}

csa_status_t csa_indexer_logits(const void *q_codes, const uint8_t *q_block_scales,
                                const float *q_weights, int32_t num_q, int32_t idx_heads,
                                int32_t idx_dim, int32_t fmt, const void *k_codes,
                                const uint8_t *k_block_scales, const float *k_scales,
                                int64_t num_slots, const int32_t *page_table,
                                int32_t page_table_stride, const int32_t *c4_seq_lens,
                                int32_t bs, const int32_t *cu_q, const int32_t *q_pos,
                                int32_t max_c4_len, float *logits, int64_t logits_stride,
                                int32_t *status, void *stream) {
    return indexer_logits(q_codes, q_block_scales, q_weights, num_q, idx_heads, idx_dim, fmt,
                          k_codes, k_block_scales, k_scales, num_slots, page_table,
                          page_table_stride, c4_seq_lens, bs, cu_q, q_pos, max_c4_len, logits,
                          logits_stride, status, stream, CSA_C4_RATIO);
}

csa_status_t csa_dsa_indexer_logits(const void *q_codes, const uint8_t *q_block_scales,
                                    const float *q_weights, int32_t num_q, int32_t idx_heads,
                                    int32_t idx_dim, int32_t fmt, const void *k_codes,
                                    const uint8_t *k_block_scales, const float *k_scales,
                                    int64_t num_slots, const int32_t *page_table,
                                    int32_t page_table_stride, const int32_t *seq_lens,
                                    int32_t bs, const int32_t *cu_q, const int32_t *q_pos,
                                    int32_t max_seq_len, float *logits, int64_t logits_stride,
                                    int32_t *status, void *stream) {
    return indexer_logits(q_codes, q_block_scales, q_weights, num_q, idx_heads, idx_dim, fmt,
                          k_codes, k_block_scales, k_scales, num_slots, page_table,
                          page_table_stride, seq_lens, bs, cu_q, q_pos, max_seq_len, logits,
                          logits_stride, status, stream, 1);
}

size_t csa_topk512_workspace_size(int32_t num_q, int32_t max_c4_len) {
    if (num_q <= 0) return 0;
    return csa::topk_workspace_bytes(num_q, max_c4_len);
}

static csa_status_t topk512(const float *logits, int64_t logits_stride,
                                        int32_t num_q, const int32_t *c4_seq_lens, int32_t bs,
                                        const int32_t *cu_q, const int32_t *q_pos,
                                        const int32_t *page_table, int32_t page_table_stride,
                                        int64_t num_slots, int32_t c4_page_size,
                                        int32_t max_c4_len, int32_t *c4_sparse_page_indices,
                                        int32_t *raw_indices, void *workspace,
                                        size_t workspace_bytes, int32_t *status, void *stream, int ratio) {
    if (num_q < 0 || bs < 0 || max_c4_len < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (c4_page_size != CSA_C4_PAGE_SIZE) return CSA_ERR_INVALID;
    if (num_q == 0) return CSA_OK;
    if (bs < 1 || !c4_seq_lens || !cu_q || !page_table || !c4_sparse_page_indices)
        return CSA_ERR_INVALID;
    if (max_c4_len > 0 && (!logits || logits_stride < max_c4_len)) return CSA_ERR_INVALID;
    if (!workspace || workspace_bytes < csa_topk512_workspace_size(num_q, max_c4_len))
        return CSA_ERR_WORKSPACE;
    if (num_q > 65535) return CSA_ERR_UNSUPPORTED;
    csa::TopkArgs a{logits, logits_stride, num_q, c4_seq_lens, bs, cu_q, q_pos, page_table,
                    page_table_stride, num_slots, max_c4_len, c4_sparse_page_indices,
                    raw_indices, workspace, status};
    a.ratio = ratio;
    return cuda_status(csa::launch_topk512(a, as_stream(stream)));
}

csa_status_t csa_topk512_page_transform(const float *logits, int64_t logits_stride,
                                        int32_t num_q, const int32_t *c4_seq_lens, int32_t bs,
                                        const int32_t *cu_q, const int32_t *q_pos,
                                        const int32_t *page_table, int32_t page_table_stride,
                                        int64_t num_slots, int32_t c4_page_size,
                                        int32_t max_c4_len, int32_t *c4_sparse_page_indices,
                                        int32_t *raw_indices, void *workspace,
                                        size_t workspace_bytes, int32_t *status, void *stream) {
    return topk512(logits, logits_stride, num_q, c4_seq_lens, bs, cu_q, q_pos, page_table,
                   page_table_stride, num_slots, c4_page_size, max_c4_len,
                   c4_sparse_page_indices, raw_indices, workspace, workspace_bytes, status,
                   stream, CSA_C4_RATIO);
}

csa_status_t csa_dsa_topk512_page_transform(const float *logits, int64_t logits_stride,
                                            int32_t num_q, const int32_t *seq_lens, int32_t bs,
                                            const int32_t *cu_q, const int32_t *q_pos,
                                            const int32_t *page_table, int32_t page_table_stride,
                                            int64_t num_slots, int32_t page_size,
                                            int32_t max_seq_len, int32_t *sparse_page_indices,
                                            int32_t *raw_indices, void *workspace,
                                            size_t workspace_bytes, int32_t *status,
                                            void *stream) {
    return topk512(logits, logits_stride, num_q, seq_lens, bs, cu_q, q_pos, page_table,
                   page_table_stride, num_slots, page_size, max_seq_len, sparse_page_indices,
                   raw_indices, workspace, workspace_bytes, status, stream, 1);
}

size_t csa_indexer_topk512_workspace_size(int32_t num_q, int32_t bs, int32_t idx_heads,
                                          int32_t idx_dim, int32_t fmt, int32_t max_c4_len) {
    if (num_q <= 0 || bs <= 0 || max_c4_len <= 0) return 0;
    size_t need = csa::topk_workspace_bytes(num_q, max_c4_len);
    if ((idx_dim == 64 || idx_dim == 128) && index_fmt_ok(fmt) && idx_heads >= 1 &&
        idx_heads <= 128) {
        csa::IndexerArgs a{};
        a.num_q = num_q;
        a.heads = idx_heads;
        a.dim = idx_dim;
        a.fmt = fmt;
        a.bs = bs;
        a.max_c4_len = max_c4_len;
        a.num_slots = 64;
        const size_t f = csa::indexer_topk_fused_bytes(a);
        if (f > need) need = f;
    }
    return need;
}

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
                                 void *stream) {
    if (num_q < 0 || bs < 0 || max_c4_len < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (c4_page_size != CSA_C4_PAGE_SIZE) return CSA_ERR_INVALID;
    if (!index_fmt_ok(fmt)) return CSA_ERR_UNSUPPORTED;
    if (idx_dim != 64 && idx_dim != 128) return CSA_ERR_UNSUPPORTED;
    if (idx_heads < 1 || idx_heads > 128) return CSA_ERR_UNSUPPORTED;
    if (num_q == 0) return CSA_OK;
    if (bs < 1 || !c4_seq_lens || !cu_q || !page_table || !c4_sparse_page_indices)
        return CSA_ERR_INVALID;
    if (num_q > 65535) return CSA_ERR_UNSUPPORTED;
    csa::TopkArgs t{logits, logits_stride, num_q, c4_seq_lens, bs, cu_q, q_pos, page_table,
                    page_table_stride, num_slots, max_c4_len, c4_sparse_page_indices,
                    raw_indices, workspace, status};
    cudaStream_t s = as_stream(stream);
    if (max_c4_len == 0) return cuda_status(csa::launch_topk512(t, s));   // -1 padding only
    if (!q_codes || !q_weights || !logits || logits_stride < max_c4_len) return CSA_ERR_INVALID;
    if (fp4_query(fmt) && !q_block_scales) return CSA_ERR_INVALID;
    if (!index_arrays_ok(fmt, k_codes, k_block_scales, k_scales)) return CSA_ERR_INVALID;
    if (!paged_keys_ok(fmt, k_codes, num_slots)) return CSA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < csa_indexer_topk512_workspace_size(
                                            num_q, bs, idx_heads, idx_dim, fmt, max_c4_len))
        return CSA_ERR_WORKSPACE;
    csa::IndexerArgs a{q_codes, q_block_scales, q_weights, num_q, idx_heads, idx_dim, fmt,
                       k_codes, k_block_scales, k_scales, num_slots, page_table,
                       page_table_stride, c4_seq_lens, bs, cu_q, q_pos, max_c4_len, logits,
                       logits_stride, status};
    if (csa::indexer_topk_fuses(a)) return cuda_status(csa::launch_indexer_topk_fused(a, t, s));
    cudaError_t e = csa::launch_indexer(a, s);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(csa::launch_topk512(t, s));
}

csa_status_t csa_indexer_select(const void *q_codes, const uint8_t *q_block_scales,
                                const float *q_weights, int32_t num_q, int32_t idx_heads,
                                int32_t idx_dim, int32_t fmt, const void *k_codes,
                                const uint8_t *k_block_scales, const float *k_scales,
                                int64_t num_slots, const int32_t *page_table,
                                int32_t page_table_stride, const int32_t *c4_seq_lens, int32_t bs,
                                const int32_t *cu_q, const int32_t *q_pos, int32_t max_c4_len,
                                float *logits, int64_t logits_stride, void *workspace,
                                size_t workspace_bytes, int32_t *status, void *stream) {
    if (num_q < 0 || bs < 0 || max_c4_len < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (!index_fmt_ok(fmt)) return CSA_ERR_UNSUPPORTED;
    if (idx_dim != 64 && idx_dim != 128) return CSA_ERR_UNSUPPORTED;
    if (idx_heads < 1 || idx_heads > 128) return CSA_ERR_UNSUPPORTED;
    if (num_q == 0 || max_c4_len == 0) return CSA_OK;
    if (bs < 1 || !q_codes || !q_weights || !page_table || !c4_seq_lens || !cu_q || !logits ||
        logits_stride < max_c4_len)
        return CSA_ERR_INVALID;
    if (fp4_query(fmt) && !q_block_scales) return CSA_ERR_INVALID;
    if (!index_arrays_ok(fmt, k_codes, k_block_scales, k_scales)) return CSA_ERR_INVALID;
    if (!paged_keys_ok(fmt, k_codes, num_slots)) return CSA_ERR_UNSUPPORTED;
    if (num_q > 65535) return CSA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < csa_indexer_topk512_workspace_size(
                                            num_q, bs, idx_heads, idx_dim, fmt, max_c4_len))
        return CSA_ERR_WORKSPACE;
    csa::IndexerArgs a{q_codes, q_block_scales, q_weights, num_q, idx_heads, idx_dim, fmt,
                       k_codes, k_block_scales, k_scales, num_slots, page_table,
                       page_table_stride, c4_seq_lens, bs, cu_q, q_pos, max_c4_len, logits,
                       logits_stride, status};
    if (!csa::indexer_topk_fuses(a)) return CSA_ERR_UNSUPPORTED;
    return cuda_status(csa::launch_indexer_select(a, workspace, as_stream(stream)));
}

csa_status_t csa_topk512_merge(int32_t num_q, int32_t idx_heads, int32_t idx_dim, int32_t fmt,
                               const int32_t *c4_seq_lens, int32_t bs, const int32_t *cu_q,
                               const int32_t *q_pos, const int32_t *page_table,
                               int32_t page_table_stride, int64_t num_slots,
                               int32_t c4_page_size, int32_t max_c4_len,
                               int32_t *c4_sparse_page_indices, int32_t *raw_indices,
                               const void *workspace, size_t workspace_bytes, int32_t *status,
                               void *stream) {
    if (num_q < 0 || bs < 0 || max_c4_len < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (c4_page_size != CSA_C4_PAGE_SIZE) return CSA_ERR_INVALID;
    if (!index_fmt_ok(fmt)) return CSA_ERR_UNSUPPORTED;
    if (idx_dim != 64 && idx_dim != 128) return CSA_ERR_UNSUPPORTED;
    if (idx_heads < 1 || idx_heads > 128) return CSA_ERR_UNSUPPORTED;
    if (num_q == 0) return CSA_OK;
    if (bs < 1 || !c4_seq_lens || !cu_q || !page_table || !c4_sparse_page_indices)
        return CSA_ERR_INVALID;
    if (num_q > 65535) return CSA_ERR_UNSUPPORTED;
    if (max_c4_len > 0 && (!workspace || workspace_bytes < csa_indexer_topk512_workspace_size(
                                             num_q, bs, idx_heads, idx_dim, fmt, max_c4_len)))
        return CSA_ERR_WORKSPACE;
    csa::IndexerArgs shape{};
    shape.num_q = num_q;
    shape.heads = idx_heads;
    shape.dim = idx_dim;
    shape.fmt = fmt;
    shape.bs = bs;
    shape.max_c4_len = max_c4_len;
    shape.num_slots = num_slots;
    csa::TopkArgs t{nullptr, 0, num_q, c4_seq_lens, bs, cu_q, q_pos, page_table,
                    page_table_stride, num_slots, max_c4_len, c4_sparse_page_indices,
                    raw_indices, const_cast<void *>(workspace), status};
    return cuda_status(csa::launch_topk_merge(shape, t, as_stream(stream)));
}

csa_status_t csa_topk512_page_transform_noalloc(const float *logits, int64_t logits_stride,
                                                int32_t num_q, const int32_t *c4_seq_lens,
                                                int32_t bs, const int32_t *cu_q,
                                                const int32_t *q_pos, const int32_t *page_table,
                                                int32_t page_table_stride, int64_t num_slots,
                                                int32_t c4_page_size, int32_t max_c4_len,
                                                int32_t *c4_sparse_page_indices,
                                                int32_t *raw_indices, int32_t *status,
                                                void *stream) {
    if (num_q < 0 || bs < 0 || max_c4_len < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (c4_page_size != CSA_C4_PAGE_SIZE) return CSA_ERR_INVALID;
    if (num_q == 0) return CSA_OK;
    if (bs < 1 || !c4_seq_lens || !cu_q || !page_table || !c4_sparse_page_indices)
        return CSA_ERR_INVALID;
    if (max_c4_len > 0 && (!logits || logits_stride < max_c4_len)) return CSA_ERR_INVALID;
    if (csa::topk_scratch_bytes(num_q, max_c4_len) > (size_t)CSA_TOPK_NOALLOC_MAX_BYTES)
        return CSA_ERR_WORKSPACE;
    if (num_q > 65535) return CSA_ERR_UNSUPPORTED;
    csa::TopkArgs a{logits, logits_stride, num_q, c4_seq_lens, bs, cu_q, q_pos, page_table,
                    page_table_stride, num_slots, max_c4_len, c4_sparse_page_indices,
                    raw_indices, nullptr, status};
    return cuda_status(csa::launch_topk512_noalloc(a, as_stream(stream)));
}

size_t csa_sparse_mqa_workspace_size(int32_t num_q, int32_t heads, int32_t window,
                                     int32_t decode) {
    if (num_q <= 0 || heads <= 0) return 0;
    return csa::attn_workspace_bytes(num_q, heads, window, decode != 0);
}

static csa_status_t sparse_mqa(const void *q, int32_t num_q, int32_t heads,
                               const void *c4_cache, const void *raw_cache, int32_t kv_fmt,
                               int64_t num_c4_slots, int64_t num_raw_slots, const int32_t *idx,
                               const int32_t *page_table, int32_t page_table_stride,
                               const int32_t *seq_lens, int32_t bs, const int32_t *cu_q,
                               const int32_t *q_pos, int32_t window, float sm_scale, void *out,
                               float *lse, void *workspace, size_t workspace_bytes,
                               int32_t *status, void *stream, bool decode, int dense_ratio = 0,
                               int max_sel = 512) {
    if (num_q < 0 || bs < 0 || page_table_stride < 0) return CSA_ERR_INVALID;
    if (!kv_fmt_ok(kv_fmt)) return CSA_ERR_UNSUPPORTED;
    if (heads != 16 && heads != 32 && heads != 64 && heads != 128) return CSA_ERR_UNSUPPORTED;
    if (window < 0 || window > 1024) return CSA_ERR_UNSUPPORTED;
    if (num_q == 0) return CSA_OK;
    if (bs < 1 || !q || (!idx && dense_ratio == 0) || !page_table || !cu_q || !out || !seq_lens)
        return CSA_ERR_INVALID;
    if (!c4_cache && num_c4_slots > 0) return CSA_ERR_INVALID;
    if (window > 0 && !raw_cache) return CSA_ERR_INVALID;
    if (!q_pos && num_q != bs) return CSA_ERR_INVALID;
    const size_t need = csa::attn_workspace_bytes(num_q, heads, window, decode, max_sel);
    if (need > 0 && (!workspace || workspace_bytes < need)) return CSA_ERR_WORKSPACE;
    if (num_q > 2147483647 / 2) return CSA_ERR_UNSUPPORTED;
    csa::AttnArgs a{q, num_q, heads, c4_cache, raw_cache, kv_fmt, num_c4_slots, num_raw_slots,
                    idx, page_table, page_table_stride, seq_lens, bs, cu_q, q_pos, window,
                    sm_scale, out, lse, workspace, status, dense_ratio, max_sel};
    return cuda_status(csa::launch_sparse_mqa(a, decode, as_stream(stream)));
}

csa_status_t csa_sparse_mqa_decode(const void *q, int32_t num_q, int32_t heads,
                                   const void *c4_cache, const void *raw_cache, int32_t kv_fmt,
                                   int64_t num_c4_slots, int64_t num_raw_slots,
                                   const int32_t *c4_sparse_page_indices,
                                   const int32_t *page_table, int32_t page_table_stride,
                                   const int32_t *seq_lens, int32_t bs, const int32_t *cu_q,
                                   const int32_t *q_pos, int32_t window, float sm_scale,
                                   void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, int32_t *status, void *stream) {
    return sparse_mqa(q, num_q, heads, c4_cache, raw_cache, kv_fmt, num_c4_slots, num_raw_slots,
                      c4_sparse_page_indices, page_table, page_table_stride, seq_lens, bs, cu_q,
                      q_pos, window, sm_scale, out, lse, workspace, workspace_bytes, status,
                      stream, true);
}

csa_status_t csa_sparse_mqa_prefill(const void *q, int32_t num_q, int32_t heads,
                                    const void *c4_cache, const void *raw_cache, int32_t kv_fmt,
                                    int64_t num_c4_slots, int64_t num_raw_slots,
                                    const int32_t *c4_sparse_page_indices,
                                    const int32_t *page_table, int32_t page_table_stride,
                                    const int32_t *seq_lens, int32_t bs, const int32_t *cu_q,
                                    const int32_t *q_pos, int32_t window, float sm_scale,
                                    void *out, float *lse, void *workspace,
                                    size_t workspace_bytes, int32_t *status, void *stream) {
    return sparse_mqa(q, num_q, heads, c4_cache, raw_cache, kv_fmt, num_c4_slots, num_raw_slots,
                      c4_sparse_page_indices, page_table, page_table_stride, seq_lens, bs, cu_q,
                      q_pos, window, sm_scale, out, lse, workspace, workspace_bytes, status,
                      stream, false);
}

}  // extern "C"

size_t csa_hca_attention_workspace_size(int32_t num_q, int32_t heads, int32_t window,
                                        int32_t decode, int32_t max_hca_len) {
    if (num_q <= 0 || heads <= 0 || max_hca_len < 0) return 0;
    return csa::attn_workspace_bytes(num_q, heads, window, decode != 0, max_hca_len);
}

csa_status_t csa_hca_attention(const void *q, int32_t num_q, int32_t heads, const void *hca_cache,
                               const void *raw_cache, int32_t kv_fmt, int64_t num_hca_slots,
                               int64_t num_raw_slots, const int32_t *page_table,
                               int32_t page_table_stride, const int32_t *seq_lens, int32_t bs,
                               const int32_t *cu_q, const int32_t *q_pos, int32_t max_hca_len,
                               int32_t window, float sm_scale, int32_t decode, void *out,
                               float *lse, void *workspace, size_t workspace_bytes,
                               int32_t *status, void *stream) {
    if (max_hca_len < 0) return CSA_ERR_INVALID;
    // at most 16 splits of 48 tiles of 32 rows per query
    if (max_hca_len + window > CSA_HCA_MAX_ROWS) return CSA_ERR_UNSUPPORTED;
    return sparse_mqa(q, num_q, heads, hca_cache, raw_cache, kv_fmt, num_hca_slots, num_raw_slots,
                      nullptr, page_table, page_table_stride, seq_lens, bs, cu_q, q_pos, window,
                      sm_scale, out, lse, workspace, workspace_bytes, status, stream, decode != 0,
                      CSA_HCA_RATIO, max_hca_len);
}

size_t csa_workspace_size(int32_t op, int32_t bs, int32_t max_rows, int32_t max_len,
                          int32_t heads, int32_t window, int32_t decode, int32_t idx_dim,
                          int32_t fmt) {
    switch (op) {
    case CSA_OP_TOPK512:
        return csa_topk512_workspace_size(max_rows, max_len);
    case CSA_OP_INDEXER_TOPK512:
        return csa_indexer_topk512_workspace_size(max_rows, bs, heads, idx_dim, fmt, max_len);
    case CSA_OP_SPARSE_MQA:
        return csa_sparse_mqa_workspace_size(max_rows, heads, window, decode);
    case CSA_OP_HCA_ATTENTION:
        return csa_hca_attention_workspace_size(max_rows, heads, window, decode, max_len);
    default:
        return 0;
    }
}
