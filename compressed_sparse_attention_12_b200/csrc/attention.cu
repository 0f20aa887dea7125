// attention.cu -- step 4, sparse MQA over the selected compressed rows joined
// with the sliding window of raw rows under one softmax
// ("Token 的一生：DSV4 架构与 DSpark" §1: attention reads only the 512 selected
// compressed rows; "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section
// "Compressed Sparse Attention（CSA）": a sliding-window branch keeps recent
// uncompressed tokens, and section "低精度與儲存策略的配合": FP8 latent, BF16
// RoPE dims).
//
// For query t, head h and key rows r (selected compressed rows, then the
// window's raw rows):  z = sm_scale * q.k_r over 576 dims; out = softmax(z) V
// with V = the rows' 512 latent dims; lse = ln sum exp z.
//
// One CTA (4 warps) owns one query, 16 heads and a contiguous range of the
// query's row list (a "split").  Rows are gathered 64 at a time into shared
// memory as bf16: BF16 rows as stored, FP8 rows as their E4M3 codes (exact in
// bf16) with the four per-128-channel scales kept aside in float32.
// S = Q K^T runs on bf16 mma.sync tensor-core instructions per 128-channel
// block, each block's partial sum scaled by its row scale in float32; the
// online softmax is float32 (base-2 exponent); O += P V splits P (times the
// value block's row scale) into a bf16 high part and a bf16 remainder so the
// probabilities keep ~16 significant bits.  Splits write unnormalised
// partials that a second kernel merges; a single split finalises in place.
#include "common.cuh"
#include "launch.h"

namespace csa {

constexpr int kAtThreads = 128;
constexpr int kAtRows = 64;                 // rows per tile
constexpr int kAtHeads = 16;                // heads per CTA
constexpr int kAtStride = kKvDim + 8;       // bf16 elements per smem row (bank-conflict pad)
constexpr int kAtPStride = kAtRows + 8;   // floats per P row
constexpr float kLog2e = 1.4426950408889634f;

struct AtSmem {
    __nv_bfloat16 q[kAtHeads * kAtStride];
    __nv_bfloat16 kv[kAtRows * kAtStride];
    float p[kAtHeads * kAtPStride];         // probabilities of the tile, float32
    float rscale[kAtRows][4];               // per-row scales of the 4 latent blocks
    float red_max[4][kAtHeads];
    float red_sum[4][kAtHeads];
    int32_t slot[kAtRows];                  // >= 0: row slot; -1: masked
    int32_t is_raw[kAtRows];
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src));
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}

struct AtQuery {
    int b, p, nw;        // request, raw position, window rows
};

__device__ __forceinline__ AtQuery at_query(const AttnArgs &a, int t) {
    int lo = 0, hi = a.bs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cu_q[mid] <= t) lo = mid; else hi = mid - 1;
    }
    AtQuery q;
    q.b = lo;
    q.p = a.q_pos ? a.q_pos[t] : a.seq_lens[lo] - 1;
    q.nw = max(0, min(a.window, q.p + 1));
    return q;
}

// Gather rows [r0, r0+64) of the query's row list into smem as bf16.
__device__ void load_tile(const AttnArgs &a, const AtQuery &qq, int t, int r0, AtSmem &sm) {
    const int tid = threadIdx.x;
    const int row_bytes = a.kv_fmt == CSA_FMT_FP8 ? kFp8RowBytes : kBf16RowBytes;
    if (tid < kAtRows) {
        const int r = r0 + tid;
        int32_t slot = -1, raw = 0;
        if (r < kTopK) {
            slot = a.idx[(int64_t)t * kTopK + r];
            if (slot >= a.num_c4_slots) {
                report(a.status, CSA_ERR_BOUNDS);
                slot = -1;
            }
        } else if (r - kTopK < qq.nw) {
            const int pos = qq.p - qq.nw + 1 + (r - kTopK);
            const int32_t page = pos / kPage < a.pt_stride
                                     ? a.page_table[(int64_t)qq.b * a.pt_stride + pos / kPage]
                                     : -1;
            const int64_t s = (int64_t)page * kPage + pos % kPage;
            if (page < 0 || s >= a.num_raw_slots) {
                report(a.status, CSA_ERR_BOUNDS);
            } else {
                slot = (int32_t)s;
                raw = 1;
            }
        }
        sm.slot[tid] = slot;
        sm.is_raw[tid] = raw;
    }
    __syncthreads();
    const uint8_t *c4 = reinterpret_cast<const uint8_t *>(a.c4_cache);
    const uint8_t *rc = reinterpret_cast<const uint8_t *>(a.raw_cache);
    if (a.kv_fmt == CSA_FMT_BF16) {
        if (tid < kAtRows) {
            const float one = sm.slot[tid] >= 0 ? 1.0f : 0.0f;
            sm.rscale[tid][0] = sm.rscale[tid][1] = sm.rscale[tid][2] = sm.rscale[tid][3] = one;
        }
        // 72 chunks of 16 B per row
        for (int u = tid; u < kAtRows * 72; u += kAtThreads) {
            const int r = u / 72, c = u % 72;
            __nv_bfloat16 *dst = sm.kv + r * kAtStride + c * 8;
            const int32_t slot = sm.slot[r];
            if (slot < 0) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
            } else {
                const uint8_t *src = (sm.is_raw[r] ? rc : c4) + (int64_t)slot * row_bytes + c * 16;
                cp_async16(dst, src);
            }
        }
        cp_async_wait_all();
    } else {
        if (tid < kAtRows) {
            const int32_t slot = sm.slot[tid];
            float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (slot >= 0)
                sc = *reinterpret_cast<const float4 *>((sm.is_raw[tid] ? rc : c4) +
                                                       (int64_t)slot * row_bytes + 512);
            sm.rscale[tid][0] = sc.x;
            sm.rscale[tid][1] = sc.y;
            sm.rscale[tid][2] = sc.z;
            sm.rscale[tid][3] = sc.w;
        }
        // 32 code chunks (16 E4M3 codes -> 16 exact bf16) + 8 RoPE chunks per row
        for (int u = tid; u < kAtRows * 40; u += kAtThreads) {
            const int r = u / 40, c = u % 40;
            const int32_t slot = sm.slot[r];
            __nv_bfloat16 *dst = sm.kv + r * kAtStride + (c < 32 ? c * 16 : 512 + (c - 32) * 8);
            if (slot < 0) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
                if (c < 32) *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(0, 0, 0, 0);
                continue;
            }
            const uint8_t *row = (sm.is_raw[r] ? rc : c4) + (int64_t)slot * row_bytes;
            if (c < 32) {
                const uint4 u4 = *reinterpret_cast<const uint4 *>(row + c * 16);
                const uint32_t w[4] = {u4.x, u4.y, u4.z, u4.w};
                uint32_t o[8];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const float2 lo = e4m3x2_to_f32x2((uint16_t)(w[j] & 0xFFFF));
                    const float2 hi = e4m3x2_to_f32x2((uint16_t)(w[j] >> 16));
                    o[2 * j] = pack_bf16(lo.x, lo.y);
                    o[2 * j + 1] = pack_bf16(hi.x, hi.y);
                }
                *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(o[4], o[5], o[6], o[7]);
            } else {
                *reinterpret_cast<uint4 *>(dst) =
                    *reinterpret_cast<const uint4 *>(row + 528 + (c - 32) * 16);
            }
        }
    }
    __syncthreads();
}

// One CTA: query t, head group g (16 heads), split sp over the row list.
__global__ void __launch_bounds__(kAtThreads, 2)
sparse_mqa_kernel(const AttnArgs a, int splits, int tiles_per_split, float *part_o,
                  float *part_ml) {
    extern __shared__ __align__(16) uint8_t at_smem_raw[];
    AtSmem &sm = *reinterpret_cast<AtSmem *>(at_smem_raw);
    const int t = blockIdx.x, g = blockIdx.y, sp = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const AtQuery qq = at_query(a, t);
    const int n_rows = kTopK + qq.nw;
    const int tile0 = sp * tiles_per_split;
    const int tile1 = min((n_rows + kAtRows - 1) / kAtRows, tile0 + tiles_per_split);

    // Q: heads 16g..16g+15 of query t
    {
        const __nv_bfloat16 *qsrc = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                    ((int64_t)t * a.heads + g * kAtHeads) * kKvDim;
        for (int u = tid; u < kAtHeads * 72; u += kAtThreads) {
            const int h = u / 72, c = u % 72;
            cp_async16(sm.q + h * kAtStride + c * 8, qsrc + h * kKvDim + c * 8);
        }
        cp_async_wait_all();
    }

    const float scale2 = a.sm_scale * kLog2e;
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};

    for (int tile = tile0; tile < tile1; tile++) {
        const int r0 = tile * kAtRows;
        // skip tiles whose compressed entries are all padding
        if (r0 + kAtRows <= kTopK) {
            const int32_t v = a.idx[(int64_t)t * kTopK + r0 + (tid & 63)];
            if (__syncthreads_or(v >= 0) == 0) continue;
        }
        load_tile(a, qq, t, r0, sm);

        // S = Q K^T: warp w covers rows 16w..16w+15 (two n-tiles of 8).  Each
        // 128-channel latent block accumulates separately and is folded in
        // with its row scale; the RoPE block has scale 1.
        float s[2][4];
#pragma unroll
        for (int i = 0; i < 2; i++) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.0f;
        const uint32_t q_base = smem_u32(sm.q) +
                                (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kAtStride +
                                           (lane >> 4) * 8) * 2;
        const uint32_t k_base = smem_u32(sm.kv) +
                                (uint32_t)((warp * 16 + (lane & 7) + (lane >> 4) * 8) * kAtStride +
                                           ((lane >> 3) & 1) * 8) * 2;
#pragma unroll 1
        for (int blk = 0; blk < 5; blk++) {
            float acc[2][4];
#pragma unroll
            for (int i = 0; i < 2; i++) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
            const int k0 = blk * 8, nk = blk < 4 ? 8 : 4;
#pragma unroll 4
            for (int kk = k0; kk < k0 + nk; kk++) {
                uint32_t af[4], bf[4];
                ldsm_x4(af, q_base + kk * 32);
                ldsm_x4(bf, k_base + kk * 32);
                mma16816(acc[0], af, bf[0], bf[1]);
                mma16816(acc[1], af, bf[2], bf[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int row = warp * 16 + nt * 8 + 2 * tq + (j & 1);
                    const float sc = blk < 4 ? sm.rscale[row][blk] : 1.0f;
                    s[nt][j] = fmaf(acc[nt][j], sc, s[nt][j]);
                }
            }
        }
        // scale, mask, per-head tile max
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; nt++) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int row = warp * 16 + nt * 8 + 2 * tq + (j & 1);
                const float v = sm.slot[row] >= 0 ? s[nt][j] * scale2 : -INFINITY;
                s[nt][j] = v;
                tmax[j >> 1] = fmaxf(tmax[j >> 1], v);
            }
        }
#pragma unroll
        for (int h = 0; h < 2; h++) {
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
        }
        if (tq == 0) {
            sm.red_max[warp][gq] = tmax[0];
            sm.red_max[warp][gq + 8] = tmax[1];
        }
        __syncthreads();
        float m_new[2], alpha[2];
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            float mx = fmaxf(fmaxf(sm.red_max[0][hh], sm.red_max[1][hh]),
                             fmaxf(sm.red_max[2][hh], sm.red_max[3][hh]));
            m_new[h] = fmaxf(m_run[h], mx);
            alpha[h] = m_new[h] == -INFINITY ? 1.0f : exp2f(m_run[h] - m_new[h]);
        }
        float psum[2] = {0.0f, 0.0f};
#pragma unroll
        for (int nt = 0; nt < 2; nt++) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int h = j >> 1;
                const float pv = m_new[h] == -INFINITY ? 0.0f : exp2f(s[nt][j] - m_new[h]);
                s[nt][j] = pv;
                psum[h] += pv;
            }
            const int col = warp * 16 + nt * 8 + 2 * tq;
            *reinterpret_cast<float2 *>(sm.p + gq * kAtPStride + col) = make_float2(s[nt][0], s[nt][1]);
            *reinterpret_cast<float2 *>(sm.p + (gq + 8) * kAtPStride + col) =
                make_float2(s[nt][2], s[nt][3]);
        }
#pragma unroll
        for (int h = 0; h < 2; h++) {
            psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 1);
            psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 2);
        }
        if (tq == 0) {
            sm.red_sum[warp][gq] = psum[0];
            sm.red_sum[warp][gq + 8] = psum[1];
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            const float ts = sm.red_sum[0][hh] + sm.red_sum[1][hh] + sm.red_sum[2][hh] +
                             sm.red_sum[3][hh];
            l_run[h] = l_run[h] * alpha[h] + ts;
            m_run[h] = m_new[h];
        }
#pragma unroll
        for (int i = 0; i < 16; i++) {
            o[i][0] *= alpha[0];
            o[i][1] *= alpha[0];
            o[i][2] *= alpha[1];
            o[i][3] *= alpha[1];
        }
        // O[:, 128w:128w+128] += (P * rowscale_w) V, P split into bf16 hi + lo
        // (this warp's output columns are exactly latent block w).
        __syncthreads();
        const uint32_t v_base = smem_u32(sm.kv) +
                                (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kAtStride +
                                           warp * 128 + (lane >> 4) * 8) * 2;
#pragma unroll
        for (int ks = 0; ks < kAtRows / 16; ks++) {
            const int r0k = ks * 16 + 2 * tq;
            float pv[8];
            const float2 p00 = *reinterpret_cast<const float2 *>(sm.p + gq * kAtPStride + r0k);
            const float2 p10 = *reinterpret_cast<const float2 *>(sm.p + (gq + 8) * kAtPStride + r0k);
            const float2 p01 = *reinterpret_cast<const float2 *>(sm.p + gq * kAtPStride + r0k + 8);
            const float2 p11 = *reinterpret_cast<const float2 *>(sm.p + (gq + 8) * kAtPStride + r0k + 8);
            const float c0 = sm.rscale[r0k][warp], c1 = sm.rscale[r0k + 1][warp];
            const float c8 = sm.rscale[r0k + 8][warp], c9 = sm.rscale[r0k + 9][warp];
            pv[0] = p00.x * c0; pv[1] = p00.y * c1;     // a0: head g,   rows r, r+1
            pv[2] = p10.x * c0; pv[3] = p10.y * c1;     // a1: head g+8, rows r, r+1
            pv[4] = p01.x * c8; pv[5] = p01.y * c9;     // a2: head g,   rows r+8, r+9
            pv[6] = p11.x * c8; pv[7] = p11.y * c9;     // a3: head g+8, rows r+8, r+9
            uint32_t ah[4], al[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const uint16_t h0 = f32_to_bf16_bits(pv[2 * i]), h1 = f32_to_bf16_bits(pv[2 * i + 1]);
                ah[i] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                al[i] = pack_bf16(pv[2 * i] - bf16_bits_to_f32(h0),
                                  pv[2 * i + 1] - bf16_bits_to_f32(h1));
            }
#pragma unroll
            for (int np = 0; np < 8; np++) {
                uint32_t bf[4];
                ldsm_x4_t(bf, v_base + (uint32_t)(ks * 16 * kAtStride + np * 16) * 2);
                mma16816(o[2 * np], ah, bf[0], bf[1]);
                mma16816(o[2 * np], al, bf[0], bf[1]);
                mma16816(o[2 * np + 1], ah, bf[2], bf[3]);
                mma16816(o[2 * np + 1], al, bf[2], bf[3]);
            }
        }
        __syncthreads();   // smem tile reused by the next load
    }

    const int h0 = g * kAtHeads;
    if (splits == 1) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            const float inv = l_run[h] > 0.0f ? 1.0f / l_run[h] : 0.0f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                  ((int64_t)t * a.heads + h0 + hh) * kLatent;
#pragma unroll
            for (int nt = 0; nt < 16; nt++) {
                const int col = warp * 128 + nt * 8 + 2 * tq;
                *reinterpret_cast<uint32_t *>(orow + col) =
                    pack_bf16(o[nt][2 * h] * inv, o[nt][2 * h + 1] * inv);
            }
            if (a.lse && warp == 0 && tq == 0)
                a.lse[(int64_t)t * a.heads + h0 + hh] =
                    l_run[h] > 0.0f ? (m_run[h] + log2f(l_run[h])) * 0.6931471805599453f
                                    : -INFINITY;
        }
    } else {
        const int64_t pbase = (((int64_t)t * gridDim.y + g) * splits + sp) * kAtHeads;
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            float *prow = part_o + (pbase + hh) * kLatent;
#pragma unroll
            for (int nt = 0; nt < 16; nt++) {
                const int col = warp * 128 + nt * 8 + 2 * tq;
                *reinterpret_cast<float2 *>(prow + col) = make_float2(o[nt][2 * h], o[nt][2 * h + 1]);
            }
            if (warp == 0 && tq == 0) {
                part_ml[(pbase + hh) * 2] = m_run[h];
                part_ml[(pbase + hh) * 2 + 1] = l_run[h];
            }
        }
    }
}

// Merge the splits of one (query, head group): grid (num_q, groups), 256 threads.
__global__ void __launch_bounds__(256)
sparse_mqa_combine_kernel(const AttnArgs a, int splits, const float *part_o,
                          const float *part_ml) {
    const int t = blockIdx.x, g = blockIdx.y;
    const int64_t base = ((int64_t)t * gridDim.y + g) * splits;
    for (int u = threadIdx.x; u < kAtHeads * (kLatent / 2); u += blockDim.x) {
        const int hh = u / (kLatent / 2), c = (u % (kLatent / 2)) * 2;
        float M = -INFINITY;
        for (int sp = 0; sp < splits; sp++) {
            const int64_t r = (base + sp) * kAtHeads + hh;
            if (part_ml[r * 2 + 1] > 0.0f) M = fmaxf(M, part_ml[r * 2]);
        }
        float L = 0.0f, o0 = 0.0f, o1 = 0.0f;
        if (M != -INFINITY) {
            for (int sp = 0; sp < splits; sp++) {
                const int64_t r = (base + sp) * kAtHeads + hh;
                const float l = part_ml[r * 2 + 1];
                if (!(l > 0.0f)) continue;
                const float w = exp2f(part_ml[r * 2] - M);
                L += l * w;
                const float2 v = *reinterpret_cast<const float2 *>(part_o + r * kLatent + c);
                o0 += v.x * w;
                o1 += v.y * w;
            }
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                              ((int64_t)t * a.heads + g * kAtHeads + hh) * kLatent;
        *reinterpret_cast<uint32_t *>(orow + c) = pack_bf16(o0 * inv, o1 * inv);
        if (a.lse && c == 0)
            a.lse[(int64_t)t * a.heads + g * kAtHeads + hh] =
                L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
}

static int at_tiles(int window) { return (kTopK + window + kAtRows - 1) / kAtRows; }

static int at_splits(int num_q, int heads, int window, bool decode) {
    if (!decode) return 1;
    const int ctas = num_q * (heads / kAtHeads);
    int sp = (2 * 148 * 2 + ctas - 1) / ctas;
    sp = sp < 1 ? 1 : sp;
    const int nt = at_tiles(window);
    sp = sp > 4 ? 4 : sp;
    return sp > nt ? nt : sp;
}

size_t attn_workspace_bytes(int num_q, int heads, int window, bool decode) {
    const int sp = at_splits(num_q, heads, window, decode);
    if (sp == 1) return 0;
    return (size_t)num_q * heads * sp * (kLatent + 2) * sizeof(float);
}

cudaError_t launch_sparse_mqa(const AttnArgs &a, bool decode, cudaStream_t s) {
    if (a.num_q == 0) return cudaSuccess;
    const int sp = at_splits(a.num_q, a.heads, a.window, decode);
    const int nt = at_tiles(a.window);
    const int tps = (nt + sp - 1) / sp;
    const int groups = a.heads / kAtHeads;
    float *po = nullptr, *pml = nullptr;
    if (sp > 1) {
        po = (float *)a.workspace;
        pml = po + (size_t)a.num_q * a.heads * sp * kLatent;
    }
    const size_t smem = sizeof(AtSmem);
    static int done[64] = {0};
    cudaError_t e = ensure_max_smem((const void *)sparse_mqa_kernel, (int)smem, done);
    if (e != cudaSuccess) return e;
    dim3 grid(a.num_q, groups, sp);
    sparse_mqa_kernel<<<grid, kAtThreads, smem, s>>>(a, sp, tps, po, pml);
    e = cudaGetLastError();
    if (e != cudaSuccess || sp == 1) return e;
    sparse_mqa_combine_kernel<<<dim3(a.num_q, groups), 256, 0, s>>>(a, sp, po, pml);
    return cudaGetLastError();
}

}  // namespace csa
