// launch.h -- internal launchers behind the C ABI (host side, namespace csa).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace csa {

// Launches `kernel` on stream s with programmatic stream serialization, so it
// may be scheduled while the previous kernel on the stream is finishing; the
// kernel itself waits for its predecessors (pdl_begin) before reading global
// memory.  Captured into CUDA graphs as a programmatic edge.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// Raises a kernel's dynamic shared-memory limit once per device (the call is
// not a stream operation, so it is kept out of CUDA-graph captures after the
// first eager launch).  `done` is a per-kernel table indexed by device.
inline cudaError_t ensure_max_smem(const void *fn, int bytes, int *done) {
    int d = 0;
    cudaError_t e = cudaGetDevice(&d);
    if (e != cudaSuccess) return e;
    if (d < 0 || d >= 64) return cudaErrorInvalidDevice;
    if (done[d] >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[d] = bytes;
    return e;
}

cudaError_t launch_kv_store(const float *rows, int64_t n, const int32_t *slots, int fmt,
                            void *cache, int64_t num_slots, int32_t *status, cudaStream_t s);

// Rotary embedding ahead of the rotation + quantisation: freqs [max_pos][rope_dim/2]
// (cos, sin) pairs; row r of the input sits at position pos[r / rows_per_pos].
// freqs == nullptr: no rotary embedding.
struct RopeArgs {
    const float2 *freqs = nullptr;
    const int32_t *pos = nullptr;
    int rope_dim = 0, max_pos = 0, rows_per_pos = 1;
};

cudaError_t launch_hadamard_quant(const void *x, int x_dtype, int64_t rows, int dim, int fmt,
                                  const int32_t *row_map, int64_t num_out_rows, void *codes,
                                  uint8_t *block_scales, float *scales, const float *w_in,
                                  float *w_out, int32_t *status, cudaStream_t s,
                                  bool rotate = true, const RopeArgs &rope = RopeArgs());

cudaError_t launch_hca_compress(const float *x, const float *gate, const float *bias, int bs,
                                const int32_t *cu_x, const int32_t *start_pos, int max_rows,
                                const int32_t *page_table, int pt_stride, int out_kind, void *out,
                                int64_t num_slots, int32_t *status, cudaStream_t s);

cudaError_t launch_c4_compress(const float *x, const float *gate, const float *bias, int dim,
                               int bs, const int32_t *cu_x, const int32_t *start_pos,
                               int max_rows, const int32_t *page_table, int pt_stride,
                               int out_kind, void *out, uint8_t *out_block_scales,
                               float *out_scales, int64_t num_slots, int32_t *status,
                               cudaStream_t s, const RopeArgs &rope = RopeArgs());

// Shape of one indexer launch (validated by the caller).
struct IndexerArgs {
    const void *q_codes;
    const uint8_t *q_block_scales;
    const float *q_weights;
    int num_q, heads, dim, fmt;
    const void *k_codes;
    const uint8_t *k_block_scales;
    const float *k_scales;
    int64_t num_slots;
    const int32_t *page_table;
    int pt_stride;
    const int32_t *c4_seq_lens;
    int bs;
    const int32_t *cu_q;
    const int32_t *q_pos;
    int max_c4_len;
    float *logits;
    int64_t logits_stride;
    int32_t *status;
    int ratio = 4;      // raw tokens per key: visible keys s < floor((p+1)/ratio)
};
cudaError_t launch_indexer(const IndexerArgs &a, cudaStream_t s);

// Top-512: candidates per (query row, chunk) live in the workspace.
size_t topk_workspace_bytes(int num_q, int max_c4_len);
struct TopkArgs {
    const float *logits;
    int64_t logits_stride;
    int num_q;
    const int32_t *c4_seq_lens;
    int bs;
    const int32_t *cu_q;
    const int32_t *q_pos;
    const int32_t *page_table;
    int pt_stride;
    int64_t num_slots;
    int max_c4_len;
    int32_t *out_phys;
    int32_t *out_raw;
    void *workspace;
    int32_t *status;
    int ratio = 4;      // raw tokens per key, as in IndexerArgs
};
cudaError_t launch_topk512(const TopkArgs &a, cudaStream_t s);
// Same, with the scratch in the library's own device array (no workspace).
cudaError_t launch_topk512_noalloc(const TopkArgs &a, cudaStream_t s);
// Bytes of scratch the selection uses for these sizes (0 when it runs in one
// launch, rows of at most 49152 logits).
size_t topk_scratch_bytes(int num_q, int max_c4_len);
// Row-level merge of per-chunk candidates (chunk_len keys per chunk, the last
// one shorter; every chunk but a single one must hold >= 512 keys).
cudaError_t launch_topk_stage2(const TopkArgs &a, int max_chunks, int chunk_len,
                               const uint32_t *cand_key, const int32_t *cand_idx,
                               const uint2 *chunk_info, cudaStream_t s);

// Indexer whose CTAs also select their own chunk's top-512, then the row merge
// (tensor-core indexer only: indexer_tc_supported).  The size query reads only
// the shape fields of `a`.
bool indexer_tc_supported(const IndexerArgs &a);
bool indexer_topk_fuses(const IndexerArgs &a);
size_t indexer_topk_fused_bytes(const IndexerArgs &a);
cudaError_t launch_indexer_topk_fused(const IndexerArgs &a, const TopkArgs &t, cudaStream_t s);
// The two halves of the fused launch: the selecting indexer (candidates into
// `workspace`) and the row merge (reads the shape fields of `shape` only).
cudaError_t launch_indexer_select(const IndexerArgs &a, void *workspace, cudaStream_t s);
cudaError_t launch_topk_merge(const IndexerArgs &shape, const TopkArgs &t, cudaStream_t s);

struct AttnArgs {
    const void *q;
    int num_q, heads;
    const void *c4_cache, *raw_cache;
    int kv_fmt;
    int64_t num_c4_slots, num_raw_slots;
    const int32_t *idx;
    const int32_t *page_table;
    int pt_stride;
    const int32_t *seq_lens;
    int bs;
    const int32_t *cu_q;
    const int32_t *q_pos;
    int window;
    float sm_scale;
    void *out;
    float *lse;
    void *workspace;
    int32_t *status;
    // 0: the first rows of a query are its selected list idx[t][0..512).
    // HCA (128): they are all its visible compressed rows s < (p+1)/128, read
    // from c4_cache at page_table[b][s/2]*2 + s%2; max_sel bounds their count.
    int dense_ratio;
    int max_sel;
};
size_t attn_workspace_bytes(int num_q, int heads, int window, bool decode, int max_sel = 512);
cudaError_t launch_sparse_mqa(const AttnArgs &a, bool decode, cudaStream_t s);
// The tcgen05 form for FP8 rows and 64 heads per CTA (no workspace: splits of
// a query merge inside their thread-block cluster).
bool sparse_mqa_tc_supported(const AttnArgs &a);
cudaError_t launch_sparse_mqa_tc(const AttnArgs &a, bool decode, cudaStream_t s);

}  // namespace csa
