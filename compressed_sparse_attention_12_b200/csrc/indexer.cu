// indexer.cu -- step 2, the C4 indexer scores
// ("Token 的一生：DSV4 架构与 DSpark" §1 and §3: the indexer scores every
// compressed token for each query, FP8/FP4 index cache; "DeepSeek-V4 的交錯壓縮
// 注意力（CSA/HCA）", section "Compressed Sparse Attention（CSA）": a light
// indexer computed in low precision):
//   logits[t][s] = k_scale[s] * sum_h w'[t][h] * ReLU(qhat[t][h] . khat[s])
// with qhat, khat the stored codes' values (FP4 codes times their block-16
// scales) and w' the head weights with the query row scale folded in.
//
// This file holds the CUDA-core form: one thread per key, the query's heads
// dequantised once into shared memory, float32 accumulation.
#include "common.cuh"
#include "launch.h"

namespace csa {

constexpr int kIdxThreads = 128;

// Dequantise `n` consecutive index elements starting at element e0 of a row
// (values without the row scale; FP4 values include the block scale).
template <int FMT>
__device__ __forceinline__ float idx_elem(const uint8_t *codes_row, const uint8_t *bsc_row,
                                          int e) {
    if (FMT == CSA_FMT_BF16) return bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(codes_row)[e]);
    if (FMT == CSA_FMT_FP8) return e4m3_to_f32(codes_row[e]);
    const uint8_t byte = codes_row[e >> 1];
    uint32_t w = (e & 1) ? (byte >> 4) : (byte & 0xF);
    float v[8];
    e2m1x8_to_f32x8(w, v);
    return v[0] * e4m3_to_f32(bsc_row[e >> 4]);
}

template <int FMT, int DIM>
__device__ __forceinline__ void load_key(const uint8_t *codes_row, const uint8_t *bsc_row,
                                         float (&k)[DIM]) {
    if constexpr (FMT == CSA_FMT_BF16) {
        const uint4 *p = reinterpret_cast<const uint4 *>(codes_row);
#pragma unroll
        for (int i = 0; i < DIM / 8; i++) {
            uint4 u = p[i];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                k[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                k[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
    } else if constexpr (FMT == CSA_FMT_FP8) {
        const uint4 *p = reinterpret_cast<const uint4 *>(codes_row);
#pragma unroll
        for (int i = 0; i < DIM / 16; i++) {
            uint4 u = p[i];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                float2 a = e4m3x2_to_f32x2((uint16_t)(w[j] & 0xFFFF));
                float2 b = e4m3x2_to_f32x2((uint16_t)(w[j] >> 16));
                k[16 * i + 4 * j] = a.x;
                k[16 * i + 4 * j + 1] = a.y;
                k[16 * i + 4 * j + 2] = b.x;
                k[16 * i + 4 * j + 3] = b.y;
            }
        }
    } else {
        const uint32_t *p = reinterpret_cast<const uint32_t *>(codes_row);
#pragma unroll
        for (int i = 0; i < DIM / 8; i++) {
            float v[8];
            e2m1x8_to_f32x8(p[i], v);
            const float sb = e4m3_to_f32(bsc_row[i / 2]);
#pragma unroll
            for (int j = 0; j < 8; j++) k[8 * i + j] = v[j] * sb;
        }
    }
}

template <int FMT, int DIM>
__global__ void __launch_bounds__(kIdxThreads)
indexer_simple_kernel(const IndexerArgs a) {
    pdl_begin();
    extern __shared__ float q_smem[];  // [heads][DIM] then w'[heads]
    constexpr int CB = FMT == CSA_FMT_BF16 ? 2 * DIM : FMT == CSA_FMT_FP8 ? DIM : DIM / 2;
    const int t = blockIdx.y;
    int lo = 0, hi = a.bs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cu_q[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    int n = a.c4_seq_lens[b];
    if (a.q_pos) n = min(n, (a.q_pos[t] + 1) / a.ratio);
    const int cap = min(a.max_c4_len, a.pt_stride * kC4Page);
    if (n > cap) {
        if (blockIdx.x == 0 && threadIdx.x == 0) report(a.status, CSA_ERR_BOUNDS);
        n = cap;
    }
    if ((int)(blockIdx.x * kIdxThreads) >= n) return;
    const int H = a.heads;
    float *ws = q_smem + H * DIM;
    const uint8_t *qc = reinterpret_cast<const uint8_t *>(a.q_codes) + (int64_t)t * H * CB;
    const uint8_t *qb = a.q_block_scales ? a.q_block_scales + (int64_t)t * H * (DIM / 16) : nullptr;
    for (int i = threadIdx.x; i < H * DIM; i += kIdxThreads) {
        const int h = i / DIM, e = i % DIM;
        q_smem[i] = idx_elem<FMT>(qc + h * CB, qb ? qb + h * (DIM / 16) : nullptr, e);
    }
    for (int h = threadIdx.x; h < H; h += kIdxThreads) ws[h] = a.q_weights[(int64_t)t * H + h];
    __syncthreads();
    const int s = blockIdx.x * kIdxThreads + threadIdx.x;
    if (s >= n) return;
    const int32_t page = a.page_table[(int64_t)b * a.pt_stride + s / kC4Page];
    const int64_t slot = (int64_t)page * kC4Page + s % kC4Page;
    if (page < 0 || slot >= a.num_slots) {
        report(a.status, CSA_ERR_BOUNDS);
        return;
    }
    float k[DIM];
    load_key<FMT, DIM>(reinterpret_cast<const uint8_t *>(a.k_codes) + slot * CB,
                       FMT == CSA_FMT_FP4 ? a.k_block_scales + slot * (DIM / 16) : nullptr, k);
    float acc = 0.0f;
    for (int h = 0; h < H; h++) {
        const float *qh = q_smem + h * DIM;
        float dot = 0.0f;
#pragma unroll
        for (int d = 0; d < DIM; d++) dot = fmaf(qh[d], k[d], dot);
        acc = fmaf(ws[h], fmaxf(dot, 0.0f), acc);
    }
    if (FMT != CSA_FMT_BF16) acc *= a.k_scales[slot];
    a.logits[(int64_t)t * a.logits_stride + s] = acc;
}

bool indexer_tc_supported(const IndexerArgs &a);
cudaError_t launch_indexer_tc(const IndexerArgs &a, cudaStream_t s);

cudaError_t launch_indexer(const IndexerArgs &a, cudaStream_t s) {
    if (a.num_q == 0 || a.max_c4_len == 0) return cudaSuccess;
    if (indexer_tc_supported(a)) return launch_indexer_tc(a, s);
    if (a.fmt == CSA_FMT_FP4_PAGE) return cudaErrorNotSupported;     // records: tensor-core path only
    dim3 grid((a.max_c4_len + kIdxThreads - 1) / kIdxThreads, a.num_q);
    const size_t smem = (size_t)a.heads * (a.dim + 1) * sizeof(float);
#define CSA_IDX(F, D)                                                                    \
    do {                                                                                 \
        static int done[64] = {0};                                                       \
        cudaError_t e = ensure_max_smem((const void *)indexer_simple_kernel<F, D>,       \
                                        128 * (D + 1) * 4, done);                        \
        if (e != cudaSuccess) return e;                                                  \
        launch_k(indexer_simple_kernel<F, D>, grid, kIdxThreads, smem, s, a);                  \
    } while (0)
    if (a.fmt == CSA_FMT_BF16 && a.dim == 64) CSA_IDX(CSA_FMT_BF16, 64);
    else if (a.fmt == CSA_FMT_BF16) CSA_IDX(CSA_FMT_BF16, 128);
    else if (a.fmt == CSA_FMT_FP8 && a.dim == 64) CSA_IDX(CSA_FMT_FP8, 64);
    else if (a.fmt == CSA_FMT_FP8) CSA_IDX(CSA_FMT_FP8, 128);
    else if (a.dim == 64) CSA_IDX(CSA_FMT_FP4, 64);
    else CSA_IDX(CSA_FMT_FP4, 128);
#undef CSA_IDX
    return cudaGetLastError();
}

}  // namespace csa
