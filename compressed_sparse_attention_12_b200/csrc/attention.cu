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
// query's row list (a "split").  Rows are gathered 32 at a time by cp.async
// into a two-stage ring (the next tile's rows land while the current one is
// computed); FP8 rows are then expanded into a bf16 tile as their E4M3 codes
// (exact in bf16) with the four per-128-channel scales kept aside in float32,
// BF16 rows are gathered straight into their tile.
// S = Q K^T runs on bf16 mma.sync tensor-core instructions per 128-channel
// block, each block's partial sum scaled by its row scale in float32; the
// online softmax is float32 (base-2 exponent); O += P V splits P (times the
// value block's row scale) into a bf16 high part and a bf16 remainder so the
// probabilities keep ~16 significant bits.  Splits write unnormalised
// partials that a second kernel merges; a single split finalises in place.
// These warp-level kernels serve BF16 rows and head counts that are not a
// multiple of 64; FP8 rows with 64-head groups run on the tcgen05 kernel of
// attention_tc.cu.
#include "attention.cuh"

namespace csa {

constexpr int kAtThreads = 128;
constexpr int kAtRows = 32;                 // rows per tile
constexpr int kAtHeads = 16;                // heads per CTA
constexpr int kAtStride = kKvDim + 8;       // bf16 elements per smem row (bank-conflict pad)
constexpr int kAtPStride = kAtRows + 8;     // floats per P row
constexpr int kAtMaxTiles = (kTopK + 1024 + kAtRows - 1) / kAtRows;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTileBytes = kAtRows * kAtStride * 2;             // one bf16 tile
constexpr int kStageBytes = kAtRows * kFp8RowBytes;             // one FP8 staging buffer
constexpr int kRegionBytes = 2 * kStageBytes + kTileBytes;      // FP8: 2 stagings + fp16 tile

struct AtSmem {                              // BF16 KV kernel
    __nv_bfloat16 q[kAtHeads * kAtStride];
    alignas(16) uint8_t region[2 * kTileBytes];   // [tile 0 | tile 1]
    float p[kAtHeads * kAtPStride];         // probabilities of the tile, float32
    float rscale[2][kAtRows][4];            // 1 for live rows, 0 for masked ones
    float red_max[4][kAtHeads];
    float red_sum[4][kAtHeads];
    int32_t slot[kAtMaxTiles * kAtRows];    // row slots of the split's tiles (-1: masked)
    int8_t is_raw[kAtMaxTiles * kAtRows];
    int16_t tiles[kAtMaxTiles];             // non-empty tiles of this split (local index)
    int32_t n_tiles;
};

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
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ __nv_bfloat16 *tile_ptr(int st, AtSmem &sm) {
    return reinterpret_cast<__nv_bfloat16 *>(sm.region + st * kTileBytes);
}

// Issues the cp.async gathers of the bf16 rows of local tile `lt` into tile `st`.
__device__ __forceinline__ void issue_loads(const AttnArgs &a, int lt, int st, AtSmem &sm) {
    const uint8_t *c4 = reinterpret_cast<const uint8_t *>(a.c4_cache);
    const uint8_t *rc = reinterpret_cast<const uint8_t *>(a.raw_cache);
    const int32_t *slots = sm.slot + lt * kAtRows;
    const int8_t *raws = sm.is_raw + lt * kAtRows;
    __nv_bfloat16 *tile = tile_ptr(st, sm);
    for (int u = threadIdx.x; u < kAtRows * 72; u += kAtThreads) {
        const int r = u / 72, c = u % 72;
        __nv_bfloat16 *dst = tile + r * kAtStride + c * 8;
        const int32_t slot = slots[r];
        if (slot < 0)
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
        else
            cp_async16(dst, (raws[r] ? rc : c4) + (int64_t)slot * kBf16RowBytes + c * 16);
    }
    cp_async_commit();
}

__device__ __forceinline__ void mma16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ FP8 KV
// The FP8 kernel keeps G groups of 16 heads in one CTA (4 warps per group):
// every gathered tile is loaded and expanded once for all of them.

template <int G>
struct AtSmem8 {
    __nv_bfloat16 q[G * kAtHeads * kAtStride];   // bf16 as loaded, then fp16 in place
    alignas(16) uint8_t region[kRegionBytes];     // [staging 0 | staging 1 | fp16 tile]
    float p[G][kAtHeads * kAtPStride];            // probabilities of the tile, per group
    float rscale[2][kAtRows][4];                  // per-row scales of the 4 latent blocks
    float rope_mul[2][kAtRows];                   // power-of-two scale of each row's RoPE part
    float qmul[G * kAtHeads];                     // power-of-two scale of each query head
    float red_max[G][4][kAtHeads];
    float red_sum[G][4][kAtHeads];
    // per warp of a group, its block's partial scores [head][row] (rows padded)
    alignas(16) float red_s[G][4][kAtHeads][kAtPStride];
    int32_t slot[kAtMaxTiles * kAtRows];          // row slots of the split's tiles (-1: masked)
    int8_t is_raw[kAtMaxTiles * kAtRows];
    int16_t tiles[kAtMaxTiles];                   // non-empty tiles of this split (local index)
    int32_t n_tiles;
};

// Issues the cp.async gathers of the packed FP8 rows of local tile `lt` into
// staging buffer `st`.
template <int G>
__device__ __forceinline__ void issue_loads8(const AttnArgs &a, int lt, int st, AtSmem8<G> &sm) {
    constexpr int kThr = kAtThreads * G;
    const uint8_t *c4 = reinterpret_cast<const uint8_t *>(a.c4_cache);
    const uint8_t *rc = reinterpret_cast<const uint8_t *>(a.raw_cache);
    const int32_t *slots = sm.slot + lt * kAtRows;
    const int8_t *raws = sm.is_raw + lt * kAtRows;
    uint8_t *stage = sm.region + st * kStageBytes;
    for (int u = threadIdx.x; u < kAtRows * 41; u += kThr) {
        const int r = u / 41, c = u % 41;
        const int32_t slot = slots[r];
        if (slot >= 0)
            cp_async16(stage + r * kFp8RowBytes + c * 16,
                       (raws[r] ? rc : c4) + (int64_t)slot * kFp8RowBytes + c * 16);
    }
    cp_async_commit();
}

// FP8 -> fp16 expansion of staging `st` (local tile `lt`): E4M3 codes exactly,
// as value x 2^-8 (a bit move, the 2^8 goes into the row scales); RoPE values
// times a per-row power of two
// that brings the row's largest magnitude into [2^13, 2^14), which converts
// exactly every bf16 value above 2^-30 of that maximum; block scales kept aside.
template <int G>
__device__ __forceinline__ void expand8(int lt, int st, AtSmem8<G> &sm) {
    constexpr int kThr = kAtThreads * G;
    const uint8_t *stage = sm.region + st * kStageBytes;
    __half *tile = reinterpret_cast<__half *>(sm.region + 2 * kStageBytes);
    const int32_t *slots = sm.slot + lt * kAtRows;
    // RoPE: 8 threads per row, 8 values (16 bytes) each; whole warps take part
    for (int u = threadIdx.x; u < kAtRows * 8; u += kThr) {
        const int r = u >> 3, c = u & 7;
        const bool valid = slots[r] >= 0;
        const uint8_t *row = stage + r * kFp8RowBytes;
        const uint4 w4 = valid ? *reinterpret_cast<const uint4 *>(row + 528 + c * 16)
                               : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
        float v[8];
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            amax = fmaxf(amax, fmaxf(fabsf(v[2 * j]), fabsf(v[2 * j + 1])));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const float m = fit_pow2(amax, 14);
        uint4 o;
        o.x = pack_f16(v[0] * m, v[1] * m);
        o.y = pack_f16(v[2] * m, v[3] * m);
        o.z = pack_f16(v[4] * m, v[5] * m);
        o.w = pack_f16(v[6] * m, v[7] * m);
        *reinterpret_cast<uint4 *>(tile + r * kAtStride + 512 + c * 8) = o;
        if (c == 0) {
            const float4 sc = valid ? *reinterpret_cast<const float4 *>(row + 512)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            // the tile holds code values x 2^-8 (see below): the scales take the 2^8
            sm.rscale[st][r][0] = sc.x * 256.0f;
            sm.rscale[st][r][1] = sc.y * 256.0f;
            sm.rscale[st][r][2] = sc.z * 256.0f;
            sm.rscale[st][r][3] = sc.w * 256.0f;
            sm.rope_mul[st][r] = valid ? 1.0f / m : 0.0f;
        }
    }
    for (int u = threadIdx.x; u < kAtRows * 32; u += kThr) {
        const int r = u / 32, c = u % 32;
        __half *dst = tile + r * kAtStride + c * 16;
        uint32_t o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (slots[r] >= 0) {
            const uint4 u4 = *reinterpret_cast<const uint4 *>(stage + r * kFp8RowBytes + c * 16);
            const uint32_t w[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                // E4M3 -> fp16 by moving the sign and the 7 exponent/mantissa bits:
                // exact, value x 2^-8 (normal and subnormal codes alike), on the
                // integer pipes (byte permute, shift, masked merge)
                const uint32_t tl = __byte_perm(w[j], 0u, 0x1404);
                const uint32_t th = __byte_perm(w[j], 0u, 0x3424);
                o[2 * j] = (tl & 0x80008000u) | ((tl >> 1) & 0x3F803F80u);
                o[2 * j + 1] = (th & 0x80008000u) | ((th >> 1) & 0x3F803F80u);
            }
        }
        *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

__device__ __forceinline__ void group_sync(int grp) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(kAtThreads) : "memory");
}

// FP8 KV on fp16 tensor cores.  One CTA: query t, head groups
// blockIdx.y*G .. +G-1 (16 heads each), split sp of the row list.  Warp w
// works for head group w/4: rows 8(w%4).. of each tile in Q K^T, latent
// columns 128(w%4).. in P V.  Scores: fp16 query (scaled per head by a power
// of two) times exact E4M3 codes, per-block partial sums scaled by the row
// scales in float32.  P V: the probabilities times the value block's row
// scale, normalised per tile by a power of two, in fp16 (11 significant bits).
template <int G>
__global__ void __launch_bounds__(kAtThreads * G, G == 1 ? 2 : 1)
sparse_mqa_fp8_kernel(const AttnArgs a, int splits, int tiles_per_split, float *part_o,
                      float *part_ml) {
    // Only inputs of the step (q, cu_q, q_pos, seq_lens) are read before the
    // wait on the preceding kernel: the query rows are loaded and converted
    // while it finishes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int kThr = kAtThreads * G;
    extern __shared__ __align__(16) uint8_t at_smem_raw[];
    AtSmem8<G> &sm = *reinterpret_cast<AtSmem8<G> *>(at_smem_raw);
    const int t = blockIdx.x, sp = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = warp >> 2, wq = warp & 3;
    const int gq = lane >> 2, tq = lane & 3;
    const int hg = blockIdx.y * G + grp;          // global 16-head group of this warp
    const AtQuery qq = at_query(a, t);
    const int n_rows = qq.nsel + qq.nw;
    const int tile0 = sp * tiles_per_split;
    const int tile1 = min((n_rows + kAtRows - 1) / kAtRows, tile0 + tiles_per_split);
    const int n_local = max(0, tile1 - tile0);
    {
        const __nv_bfloat16 *qsrc = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                    ((int64_t)t * a.heads + blockIdx.y * G * kAtHeads) * kKvDim;
        for (int u = tid; u < G * kAtHeads * 72; u += kThr) {
            const int h = u / 72, c = u % 72;
            cp_async16(sm.q + h * kAtStride + c * 8, qsrc + h * kKvDim + c * 8);
        }
        cp_async_commit();
    }
    // Q to fp16 in place: warp w converts heads 4w..4w+3, each times a power
    // of two that brings its largest magnitude into [2^13, 2^14), so every
    // bf16 value above 2^-30 of that maximum converts exactly
    cp_async_wait<0>();
    __syncthreads();
    {
        uint16_t *qh = reinterpret_cast<uint16_t *>(sm.q);
        for (int h = warp * 4; h < warp * 4 + 4; h++) {
            float v[18];
            float amax = 0.0f;
#pragma unroll
            for (int k = 0; k < 18; k++) {
                v[k] = bf16_bits_to_f32(qh[h * kAtStride + lane + 32 * k]);
                amax = fmaxf(amax, fabsf(v[k]));
            }
            amax = warp_max(amax);
            const float m = fit_pow2(amax, 14);
#pragma unroll
            for (int k = 0; k < 18; k++) {
                const __half hv = __float2half_rn(v[k] * m);
                qh[h * kAtStride + lane + 32 * k] = *reinterpret_cast<const uint16_t *>(&hv);
            }
            if (lane == 0) sm.qmul[h] = 1.0f / m;
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int u = tid; u < n_local * kAtRows; u += kThr) {
        int32_t raw;
        const int32_t slot = row_slot(a, qq, t, tile0 * kAtRows + u, &raw);
        sm.slot[u] = slot;
        sm.is_raw[u] = (int8_t)raw;
    }
    __syncthreads();
    for (int lt = warp; lt < n_local; lt += 4 * G) {
        const bool any = __any_sync(0xffffffffu, sm.slot[lt * kAtRows + lane] >= 0);
        if (lane == 0) sm.tiles[lt] = any ? 1 : 0;
    }
    __syncthreads();
    if (tid == 0) {
        int n = 0;
        for (int lt = 0; lt < n_local; lt++)
            if (sm.tiles[lt]) sm.tiles[n++] = (int16_t)lt;
        sm.n_tiles = n;
    }
    __syncthreads();
    const int nt = sm.n_tiles;
    for (int j = 0; j < 2; j++) {
        if (j < nt) issue_loads8(a, sm.tiles[j], j, sm);
        else cp_async_commit();
    }

    float qscale[2];
#pragma unroll
    for (int h = 0; h < 2; h++)
        qscale[h] = a.sm_scale * kLog2e * sm.qmul[grp * kAtHeads + gq + 8 * h];
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
    float pw = 1.0f;     // O holds (true partial output) * pw
    float *p_s = sm.p[grp];
    const uint32_t q_base =
        smem_u32(sm.q) + (uint32_t)((grp * kAtHeads + (lane & 7) + ((lane >> 3) & 1) * 8) *
                                        kAtStride + (lane >> 4) * 8) * 2;
    const __half *tile = reinterpret_cast<const __half *>(sm.region + 2 * kStageBytes);
    const uint32_t k_base =
        smem_u32(tile) + (uint32_t)((wq * 8 + (lane & 7)) * kAtStride + (lane >> 3) * 8) * 2;
    const uint32_t kb_base =
        smem_u32(tile) + (uint32_t)((lane & 7) * kAtStride + (lane >> 3) * 8) * 2;
    const uint32_t v_base =
        smem_u32(tile) + (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kAtStride + wq * 128 +
                                    (lane >> 4) * 8) * 2;

    for (int j = 0; j < nt; j++) {
        const int st = j & 1;
        if (j + 1 < nt) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncthreads();
        const int lt = sm.tiles[j];
        const int32_t *slots = sm.slot + lt * kAtRows;
        expand8(lt, st, sm);
        __syncthreads();

        // S = Q K^T split by channel block: warp wq takes latent block wq
        // (8 k-steps) for all 32 rows and the RoPE block (4 k-steps) for rows
        // 8wq..8wq+7; each partial is scaled by its rows' block scale, and the
        // four warps' partials are summed through shared memory.
        float sl[4][4], sr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int nb = 0; nb < 4; nb++) sl[nb][0] = sl[nb][1] = sl[nb][2] = sl[nb][3] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int kk = 8 * wq + 2 * i;
            uint32_t a0[4], a1[4];
            ldsm_x4(a0, q_base + kk * 32);
            ldsm_x4(a1, q_base + (kk + 1) * 32);
#pragma unroll
            for (int nb = 0; nb < 4; nb++) {
                uint32_t bf[4];
                ldsm_x4(bf, kb_base + (uint32_t)(nb * 8 * kAtStride * 2 + kk * 32));
                mma16816_f16(sl[nb], a0, bf[0], bf[1]);
                mma16816_f16(sl[nb], a1, bf[2], bf[3]);
            }
        }
#pragma unroll
        for (int i = 0; i < 2; i++) {
            const int kk = 32 + 2 * i;
            uint32_t a0[4], a1[4], bf[4];
            ldsm_x4(a0, q_base + kk * 32);
            ldsm_x4(a1, q_base + (kk + 1) * 32);
            ldsm_x4(bf, k_base + kk * 32);
            mma16816_f16(sr, a0, bf[0], bf[1]);
            mma16816_f16(sr, a1, bf[2], bf[3]);
        }
        {
            float (*rs)[kAtPStride] = sm.red_s[grp][wq];
#pragma unroll
            for (int nb = 0; nb < 4; nb++) {
                const int r0 = nb * 8 + 2 * tq;
                const float c0 = sm.rscale[st][r0][wq], c1 = sm.rscale[st][r0 + 1][wq];
                float v0 = sl[nb][0] * c0, v1 = sl[nb][1] * c1;
                float v2 = sl[nb][2] * c0, v3 = sl[nb][3] * c1;
                if (nb == wq) {
                    const float e0 = sm.rope_mul[st][r0], e1 = sm.rope_mul[st][r0 + 1];
                    v0 = fmaf(sr[0], e0, v0);
                    v1 = fmaf(sr[1], e1, v1);
                    v2 = fmaf(sr[2], e0, v2);
                    v3 = fmaf(sr[3], e1, v3);
                }
                *reinterpret_cast<float2 *>(&rs[gq][r0]) = make_float2(v0, v1);
                *reinterpret_cast<float2 *>(&rs[gq + 8][r0]) = make_float2(v2, v3);
            }
        }
        group_sync(grp);
        float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < 4; w++) {
            const float2 x = *reinterpret_cast<const float2 *>(&sm.red_s[grp][w][gq][wq * 8 + 2 * tq]);
            const float2 y =
                *reinterpret_cast<const float2 *>(&sm.red_s[grp][w][gq + 8][wq * 8 + 2 * tq]);
            s[0] += x.x;
            s[1] += x.y;
            s[2] += y.x;
            s[3] += y.y;
        }
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
            const int row = wq * 8 + 2 * tq + (jj & 1);
            const float v = slots[row] >= 0 ? s[jj] * qscale[jj >> 1] : -INFINITY;
            s[jj] = v;
            tmax[jj >> 1] = fmaxf(tmax[jj >> 1], v);
        }
#pragma unroll
        for (int h = 0; h < 2; h++) {
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
        }
        if (tq == 0) {
            sm.red_max[grp][wq][gq] = tmax[0];
            sm.red_max[grp][wq][gq + 8] = tmax[1];
        }
        group_sync(grp);
        float m_new[2], alpha[2];
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            const float mx = fmaxf(fmaxf(sm.red_max[grp][0][hh], sm.red_max[grp][1][hh]),
                                   fmaxf(sm.red_max[grp][2][hh], sm.red_max[grp][3][hh]));
            m_new[h] = fmaxf(m_run[h], mx);
            alpha[h] = m_new[h] == -INFINITY ? 1.0f : exp2f(m_run[h] - m_new[h]);
        }
        float psum[2] = {0.0f, 0.0f};
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
            const int h = jj >> 1;
            const float pv = m_new[h] == -INFINITY ? 0.0f : exp2f(s[jj] - m_new[h]);
            s[jj] = pv;
            psum[h] += pv;
        }
        {
            const int col = wq * 8 + 2 * tq;
            *reinterpret_cast<float2 *>(p_s + gq * kAtPStride + col) = make_float2(s[0], s[1]);
            *reinterpret_cast<float2 *>(p_s + (gq + 8) * kAtPStride + col) = make_float2(s[2], s[3]);
        }
#pragma unroll
        for (int h = 0; h < 2; h++) {
            psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 1);
            psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 2);
        }
        if (tq == 0) {
            sm.red_sum[grp][wq][gq] = psum[0];
            sm.red_sum[grp][wq][gq + 8] = psum[1];
        }
        group_sync(grp);
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            const float ts = sm.red_sum[grp][0][hh] + sm.red_sum[grp][1][hh] +
                             sm.red_sum[grp][2][hh] + sm.red_sum[grp][3][hh];
            l_run[h] = l_run[h] * alpha[h] + ts;
            m_run[h] = m_new[h];
        }
        // power-of-two normalisation of this tile's block-wq row scales
        const float smax = warp_max(sm.rscale[st][lane][wq]);
        const float pw_new = smax > 0.0f ? fit_pow2(smax, 0) : pw;
        const float rs = pw_new / pw;
        pw = pw_new;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            o[i][0] *= alpha[0] * rs;
            o[i][1] *= alpha[0] * rs;
            o[i][2] *= alpha[1] * rs;
            o[i][3] *= alpha[1] * rs;
        }
#pragma unroll
        for (int ks = 0; ks < kAtRows / 16; ks++) {
            const int r0k = ks * 16 + 2 * tq;
            const float2 p00 = *reinterpret_cast<const float2 *>(p_s + gq * kAtPStride + r0k);
            const float2 p10 = *reinterpret_cast<const float2 *>(p_s + (gq + 8) * kAtPStride + r0k);
            const float2 p01 = *reinterpret_cast<const float2 *>(p_s + gq * kAtPStride + r0k + 8);
            const float2 p11 =
                *reinterpret_cast<const float2 *>(p_s + (gq + 8) * kAtPStride + r0k + 8);
            const float c0 = sm.rscale[st][r0k][wq] * pw, c1 = sm.rscale[st][r0k + 1][wq] * pw;
            const float c8 = sm.rscale[st][r0k + 8][wq] * pw, c9 = sm.rscale[st][r0k + 9][wq] * pw;
            uint32_t af[4];
            af[0] = pack_f16(p00.x * c0, p00.y * c1);
            af[1] = pack_f16(p10.x * c0, p10.y * c1);
            af[2] = pack_f16(p01.x * c8, p01.y * c9);
            af[3] = pack_f16(p11.x * c8, p11.y * c9);
#pragma unroll
            for (int np = 0; np < 8; np++) {
                uint32_t bf[4];
                ldsm_x4_t(bf, v_base + (uint32_t)(ks * 16 * kAtStride + np * 16) * 2);
                mma16816_f16(o[2 * np], af, bf[0], bf[1]);
                mma16816_f16(o[2 * np + 1], af, bf[2], bf[3]);
            }
        }
        __syncthreads();   // stage `st` and the tile are free again
        if (j + 2 < nt) issue_loads8(a, sm.tiles[j + 2], st, sm);
        else cp_async_commit();
    }

    const float unpw = 1.0f / pw;
    const int h0 = hg * kAtHeads;
    if (splits == 1) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            const float inv = l_run[h] > 0.0f ? unpw / l_run[h] : 0.0f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                  ((int64_t)t * a.heads + h0 + hh) * kLatent;
#pragma unroll
            for (int n8 = 0; n8 < 16; n8++) {
                const int col = wq * 128 + n8 * 8 + 2 * tq;
                *reinterpret_cast<uint32_t *>(orow + col) =
                    pack_bf16(o[n8][2 * h] * inv, o[n8][2 * h + 1] * inv);
            }
            if (a.lse && wq == 0 && tq == 0)
                a.lse[(int64_t)t * a.heads + h0 + hh] =
                    l_run[h] > 0.0f ? (m_run[h] + log2f(l_run[h])) * 0.6931471805599453f
                                    : -INFINITY;
        }
    } else {
        const int64_t pbase =
            (((int64_t)t * (a.heads / kAtHeads) + hg) * splits + sp) * kAtHeads;
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int hh = gq + 8 * h;
            float *prow = part_o + (pbase + hh) * kLatent;
#pragma unroll
            for (int n8 = 0; n8 < 16; n8++) {
                const int col = wq * 128 + n8 * 8 + 2 * tq;
                *reinterpret_cast<float2 *>(prow + col) =
                    make_float2(o[n8][2 * h] * unpw, o[n8][2 * h + 1] * unpw);
            }
            if (wq == 0 && tq == 0) {
                part_ml[(pbase + hh) * 2] = m_run[h];
                part_ml[(pbase + hh) * 2 + 1] = l_run[h];
            }
        }
    }
}

// One CTA: query t, head group g (16 heads), split sp over the row list.
__global__ void __launch_bounds__(kAtThreads, 2)
sparse_mqa_kernel(const AttnArgs a, int splits, int tiles_per_split, float *part_o,
                  float *part_ml) {
    pdl_begin();
    extern __shared__ __align__(16) uint8_t at_smem_raw[];
    AtSmem &sm = *reinterpret_cast<AtSmem *>(at_smem_raw);
    const int t = blockIdx.x, g = blockIdx.y, sp = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const AtQuery qq = at_query(a, t);
    const int n_rows = qq.nsel + qq.nw;
    const int tile0 = sp * tiles_per_split;
    const int tile1 = min((n_rows + kAtRows - 1) / kAtRows, tile0 + tiles_per_split);

    // row slots of every tile of this split, resolved once; tiles whose rows are
    // all masked (padding of short requests) are skipped
    const int n_local = max(0, tile1 - tile0);
    for (int u = tid; u < n_local * kAtRows; u += kAtThreads) {
        int32_t raw;
        const int32_t slot = row_slot(a, qq, t, tile0 * kAtRows + u, &raw);
        sm.slot[u] = slot;
        sm.is_raw[u] = (int8_t)raw;
    }
    {
        const __nv_bfloat16 *qsrc = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                    ((int64_t)t * a.heads + g * kAtHeads) * kKvDim;
        for (int u = tid; u < kAtHeads * 72; u += kAtThreads) {
            const int h = u / 72, c = u % 72;
            cp_async16(sm.q + h * kAtStride + c * 8, qsrc + h * kKvDim + c * 8);
        }
    }
    __syncthreads();
    for (int lt = warp; lt < n_local; lt += 4) {
        const bool any = __any_sync(0xffffffffu, sm.slot[lt * kAtRows + lane] >= 0);
        if (lane == 0) sm.tiles[lt] = any ? 1 : 0;
    }
    __syncthreads();
    if (tid == 0) {
        int n = 0;
        for (int lt = 0; lt < n_local; lt++)
            if (sm.tiles[lt]) sm.tiles[n++] = (int16_t)lt;
        sm.n_tiles = n;
    }
    __syncthreads();
    const int nt = sm.n_tiles;
    for (int j = 0; j < 2; j++) {
        if (j < nt) issue_loads(a, sm.tiles[j], j, sm);
        else cp_async_commit();
    }

    const float scale2 = a.sm_scale * kLog2e;
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
    const uint32_t q_base = smem_u32(sm.q) +
                            (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kAtStride +
                                       (lane >> 4) * 8) * 2;

    for (int j = 0; j < nt; j++) {
        const int st = j & 1;
        if (j + 1 < nt) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncthreads();
        const int lt = sm.tiles[j];
        const int32_t *slots = sm.slot + lt * kAtRows;
        if (tid < kAtRows) {
            const float one = slots[tid] >= 0 ? 1.0f : 0.0f;
            sm.rscale[st][tid][0] = sm.rscale[st][tid][1] = one;
            sm.rscale[st][tid][2] = sm.rscale[st][tid][3] = one;
        }
        __syncthreads();
        const __nv_bfloat16 *tile = tile_ptr(st, sm);

        // S = Q K^T: warp w covers rows 8w..8w+7.  Each 128-channel latent block
        // accumulates separately and is folded in with its row scale.
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t k_base = smem_u32(tile) +
                                (uint32_t)((warp * 8 + (lane & 7)) * kAtStride + (lane >> 3) * 8) * 2;
#pragma unroll 1
        for (int blk = 0; blk < 5; blk++) {
            float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
            const int k0 = blk * 8, nk = blk < 4 ? 8 : 4;
#pragma unroll 4
            for (int kk = k0; kk < k0 + nk; kk += 2) {
                uint32_t a0[4], a1[4], bf[4];
                ldsm_x4(a0, q_base + kk * 32);
                ldsm_x4(a1, q_base + (kk + 1) * 32);
                ldsm_x4(bf, k_base + kk * 32);
                mma16816(acc0, a0, bf[0], bf[1]);
                mma16816(acc1, a1, bf[2], bf[3]);
            }
#pragma unroll
            for (int jj = 0; jj < 4; jj++) {
                const int row = warp * 8 + 2 * tq + (jj & 1);
                const float sc = blk < 4 ? sm.rscale[st][row][blk] : 1.0f;
                s[jj] = fmaf(acc0[jj] + acc1[jj], sc, s[jj]);
            }
        }
        // scale, mask, per-head tile max
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
            const int row = warp * 8 + 2 * tq + (jj & 1);
            const float v = slots[row] >= 0 ? s[jj] * scale2 : -INFINITY;
            s[jj] = v;
            tmax[jj >> 1] = fmaxf(tmax[jj >> 1], v);
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
            const float mx = fmaxf(fmaxf(sm.red_max[0][hh], sm.red_max[1][hh]),
                                   fmaxf(sm.red_max[2][hh], sm.red_max[3][hh]));
            m_new[h] = fmaxf(m_run[h], mx);
            alpha[h] = m_new[h] == -INFINITY ? 1.0f : exp2f(m_run[h] - m_new[h]);
        }
        float psum[2] = {0.0f, 0.0f};
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
            const int h = jj >> 1;
            const float pv = m_new[h] == -INFINITY ? 0.0f : exp2f(s[jj] - m_new[h]);
            s[jj] = pv;
            psum[h] += pv;
        }
        {
            const int col = warp * 8 + 2 * tq;
            *reinterpret_cast<float2 *>(sm.p + gq * kAtPStride + col) = make_float2(s[0], s[1]);
            *reinterpret_cast<float2 *>(sm.p + (gq + 8) * kAtPStride + col) = make_float2(s[2], s[3]);
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
        const uint32_t v_base = smem_u32(tile) +
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
            const float c0 = sm.rscale[st][r0k][warp], c1 = sm.rscale[st][r0k + 1][warp];
            const float c8 = sm.rscale[st][r0k + 8][warp], c9 = sm.rscale[st][r0k + 9][warp];
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
        __syncthreads();   // stage `st` and the tile are free again
        if (j + 2 < nt) issue_loads(a, sm.tiles[j + 2], st, sm);
        else cp_async_commit();
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
            for (int n8 = 0; n8 < 16; n8++) {
                const int col = warp * 128 + n8 * 8 + 2 * tq;
                *reinterpret_cast<uint32_t *>(orow + col) =
                    pack_bf16(o[n8][2 * h] * inv, o[n8][2 * h + 1] * inv);
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
            for (int n8 = 0; n8 < 16; n8++) {
                const int col = warp * 128 + n8 * 8 + 2 * tq;
                *reinterpret_cast<float2 *>(prow + col) = make_float2(o[n8][2 * h], o[n8][2 * h + 1]);
            }
            if (warp == 0 && tq == 0) {
                part_ml[(pbase + hh) * 2] = m_run[h];
                part_ml[(pbase + hh) * 2 + 1] = l_run[h];
            }
        }
    }
}

// Merge the splits of one (query, head): grid num_q * heads, 128 threads,
// four output columns per thread.
// Merges the split partials of one (query, head): every split's (max, sum)
// and 4-column slice are loaded before any is used (one memory round trip).
constexpr int kAtMaxSplits = 16;

template <int MAXSP>
__global__ void __launch_bounds__(128)
sparse_mqa_combine_kernel(const AttnArgs a, int splits, const float *part_o,
                          const float *part_ml) {
    pdl_begin();
    const int t = blockIdx.x / a.heads, head = blockIdx.x % a.heads;
    const int g = head / kAtHeads, hh = head % kAtHeads;
    const int groups = a.heads / kAtHeads;
    const int64_t base = ((int64_t)t * groups + g) * splits;
    const int c = threadIdx.x * 4;
    float m[MAXSP], l[MAXSP];
    float4 v[MAXSP];
#pragma unroll
    for (int sp = 0; sp < MAXSP; sp++) {
        if (sp < splits) {
            const int64_t r = (base + sp) * kAtHeads + hh;
            const float2 ml = *reinterpret_cast<const float2 *>(part_ml + r * 2);
            m[sp] = ml.x;
            l[sp] = ml.y;
            v[sp] = *reinterpret_cast<const float4 *>(part_o + r * kLatent + c);
        } else {
            m[sp] = -INFINITY;
            l[sp] = 0.0f;
            v[sp] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < MAXSP; sp++)
        if (l[sp] > 0.0f) M = fmaxf(M, m[sp]);
    float L = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
        for (int sp = 0; sp < MAXSP; sp++) {
            if (!(l[sp] > 0.0f)) continue;
            const float w = exp2f(m[sp] - M);
            L += l[sp] * w;
            acc.x += v[sp].x * w;
            acc.y += v[sp].y * w;
            acc.z += v[sp].z * w;
            acc.w += v[sp].w * w;
        }
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                          ((int64_t)t * a.heads + head) * kLatent;
    *reinterpret_cast<uint2 *>(orow + c) =
        make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
    if (a.lse && threadIdx.x == 0)
        a.lse[(int64_t)t * a.heads + head] =
            L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

static int at_tiles(int window, int max_sel = kTopK) {
    return (max_sel + window + kAtRows - 1) / kAtRows;
}

// Head groups (of 16) per CTA: the FP8 kernel takes 64 heads at a time when
// the head count allows, the BF16 kernel one group.
static int at_groups(int heads, int kv_fmt) {
    return kv_fmt == CSA_FMT_FP8 && heads % (4 * kAtHeads) == 0 ? 4 : 1;
}

static int at_splits(int num_q, int heads, int window, bool decode, int groups,
                     int max_sel = kTopK) {
    const int nt = at_tiles(window, max_sel);
    // a split holds at most kAtMaxTiles tiles (its row slots live in shared memory)
    const int need = (nt + kAtMaxTiles - 1) / kAtMaxTiles;
    if (!decode) return need;
    // split each query's rows so that the grid fills one wave of the 148 SMs
    // (two CTAs per SM with one head group, one CTA with four)
    const int per_sm = groups == 1 ? 2 : 1;
    const int ctas = num_q * (heads / (kAtHeads * groups));
    int sp = (per_sm * 148) / ctas;
    sp = sp < 1 ? 1 : sp;
    sp = sp > kAtMaxSplits ? kAtMaxSplits : sp;
    sp = sp > nt ? nt : sp;
    return sp < need ? need : sp;
}

size_t attn_workspace_bytes(int num_q, int heads, int window, bool decode, int max_sel) {
    // the larger of the two formats' needs
    int sp = at_splits(num_q, heads, window, decode, at_groups(heads, CSA_FMT_BF16), max_sel);
    const int sp8 = at_splits(num_q, heads, window, decode, at_groups(heads, CSA_FMT_FP8), max_sel);
    sp = sp8 > sp ? sp8 : sp;
    if (sp == 1) return 0;
    return (size_t)num_q * heads * sp * (kLatent + 2) * sizeof(float);
}

template <int G>
static cudaError_t launch_fp8(const AttnArgs &a, dim3 grid, int sp, int tps, float *po,
                              float *pml, cudaStream_t s) {
    static int done[64] = {0};
    const size_t smem = sizeof(AtSmem8<G>);
    cudaError_t e = ensure_max_smem((const void *)sparse_mqa_fp8_kernel<G>, (int)smem, done);
    if (e != cudaSuccess) return e;
    launch_k(sparse_mqa_fp8_kernel<G>, grid, kAtThreads * G, smem, s, a, sp, tps, po, pml);
    return cudaGetLastError();
}

cudaError_t launch_sparse_mqa(const AttnArgs &a, bool decode, cudaStream_t s) {
    if (a.num_q == 0) return cudaSuccess;
    // FP8 rows and a multiple of 64 heads: the tensor-core kernel (attention_tc.cu)
    if (sparse_mqa_tc_supported(a)) return launch_sparse_mqa_tc(a, decode, s);
    const int groups = at_groups(a.heads, a.kv_fmt);
    const int max_sel = a.dense_ratio > 0 ? a.max_sel : kTopK;
    const int sp = at_splits(a.num_q, a.heads, a.window, decode, groups, max_sel);
    const int nt = at_tiles(a.window, max_sel);
    const int tps = (nt + sp - 1) / sp;
    float *po = nullptr, *pml = nullptr;
    if (sp > 1) {
        po = (float *)a.workspace;
        pml = po + (size_t)a.num_q * a.heads * sp * kLatent;
    }
    dim3 grid(a.num_q, a.heads / (kAtHeads * groups), sp);
    cudaError_t e;
    if (a.kv_fmt == CSA_FMT_FP8) {
        e = groups == 4 ? launch_fp8<4>(a, grid, sp, tps, po, pml, s)
                        : launch_fp8<1>(a, grid, sp, tps, po, pml, s);
    } else {
        static int done[64] = {0};
        const size_t smem = sizeof(AtSmem);
        e = ensure_max_smem((const void *)sparse_mqa_kernel, (int)smem, done);
        if (e != cudaSuccess) return e;
        launch_k(sparse_mqa_kernel, grid, kAtThreads, smem, s, a, sp, tps, po, pml);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess || sp == 1) return e;
    if (sp <= 4) launch_k(sparse_mqa_combine_kernel<4>, a.num_q * a.heads, 128, 0, s, a, sp, po, pml);
    else if (sp <= 8) launch_k(sparse_mqa_combine_kernel<8>, a.num_q * a.heads, 128, 0, s, a, sp, po, pml);
    else launch_k(sparse_mqa_combine_kernel<16>, a.num_q * a.heads, 128, 0, s, a, sp, po, pml);
    return cudaGetLastError();
}

}  // namespace csa
