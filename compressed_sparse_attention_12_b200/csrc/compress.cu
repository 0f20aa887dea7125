// compress.cu -- step 1 (C4 compressor), the KV row writer, and the index
// rotation + quantisation (step 2's front half).
//
// Pages: "Token 的一生：DSV4 架构与 DSpark" §2.1 (four raw tokens pooled into one
// compressed token when the block's fourth token arrives), §3.1 (FP8/FP4
// index cache, head-gate weight fusion), §4 (Hadamard rotation before
// quantisation); "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section "Compressed
// Sparse Attention（CSA）" (softmax-gated pooling with a learned positional
// bias) and section "低精度與儲存策略的配合" (FP8 KV entries, BF16 RoPE dims).
//
// All three kernels are HBM streaming kernels: float4 loads of the inputs,
// float32 math, one rounding into the stored format.
#include "common.cuh"
#include "launch.h"

namespace csa {

// ------------------------------------------------------------------ KV rows
//
// A KV row is written by 5 warps: warps 0-3 own the four 128-channel latent
// blocks (lane l: channels 4l..4l+3 of the block), warp 4 lanes 0-15 own the
// 64 RoPE channels.  For FP8 each latent warp reduces its block's amax for the
// block scale (amax/448, 1 for an all-zero block).
constexpr int kKvRowThreads = 160;

__device__ __forceinline__ void write_kv_row(float4 v, int warp, int lane, int fmt,
                                             uint8_t *row) {
    if (fmt == CSA_FMT_FP8) {
        if (warp < 4) {
            float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
            a = warp_max(a);
            const float s = a > 0.0f ? __fdiv_rn(a, 448.0f) : 1.0f;
            uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(v.x, s), __fdiv_rn(v.y, s));
            uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(v.z, s), __fdiv_rn(v.w, s));
            *reinterpret_cast<uint32_t *>(row + warp * 128 + lane * 4) =
                (uint32_t)lo | ((uint32_t)hi << 16);
            if (lane == 0) *reinterpret_cast<float *>(row + 512 + 4 * warp) = s;
        } else if (lane < 16) {
            uint2 o;
            o.x = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
            o.y = (uint32_t)f32_to_bf16_bits(v.z) | ((uint32_t)f32_to_bf16_bits(v.w) << 16);
            *reinterpret_cast<uint2 *>(row + 528 + lane * 8) = o;
        }
    } else {
        const int c = warp * 128 + lane * 4;
        if (warp < 4 || lane < 16) {
            uint2 o;
            o.x = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
            o.y = (uint32_t)f32_to_bf16_bits(v.z) | ((uint32_t)f32_to_bf16_bits(v.w) << 16);
            *reinterpret_cast<uint2 *>(row + 2 * c) = o;
        }
    }
}

__device__ __forceinline__ int kv_channel(int warp, int lane) { return warp * 128 + lane * 4; }

__device__ __forceinline__ bool kv_active(int warp, int lane) { return warp < 4 || lane < 16; }

__global__ void __launch_bounds__(kKvRowThreads)
kv_store_kernel(const float *__restrict__ rows, int64_t n, const int32_t *__restrict__ slots,
                int fmt, uint8_t *__restrict__ cache, int64_t num_slots, int32_t *status) {
    pdl_begin();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_bytes = fmt == CSA_FMT_FP8 ? kFp8RowBytes : kBf16RowBytes;
    for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
        const int32_t slot = slots[r];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (threadIdx.x == 0) report(status, CSA_ERR_BOUNDS);
            continue;
        }
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kv_active(warp, lane))
            v = *reinterpret_cast<const float4 *>(rows + r * kKvDim + kv_channel(warp, lane));
        write_kv_row(v, warp, lane, fmt, cache + (int64_t)slot * row_bytes);
    }
}

// ------------------------------------------------------------------ index rows
//
// One warp per row of D = 32*E values, lane l owning elements [lE, lE+E).
// Rotation: x' = (1/sqrt(D)) H_D x, then the row is quantised.

template <int E>
__device__ __forceinline__ void rotate(float (&v)[E], int lane) {
    warp_fwht<E>(v, lane);
    const float inv = E == 2 ? 0.125f : 0.08838834764831845f;  // 1/sqrt(64), 1/sqrt(128)
#pragma unroll
    for (int i = 0; i < E; i++) v[i] *= inv;
}

// Quantise one rotated row and store it at output row `orow`.
// Returns the row scale (1 for bf16) so callers can fold it into weights.
template <int E>
__device__ __forceinline__ float quant_index_row(const float (&v)[E], int lane, int fmt,
                                                 int64_t orow, uint8_t *codes,
                                                 uint8_t *block_scales, float *scales) {
    constexpr int D = 32 * E;
    if (fmt == CSA_FMT_BF16) {
        uint16_t *o = reinterpret_cast<uint16_t *>(codes) + orow * D + lane * E;
#pragma unroll
        for (int i = 0; i < E; i++) o[i] = f32_to_bf16_bits(v[i]);
        return 1.0f;
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < E; i++) a = fmaxf(a, fabsf(v[i]));
    const float amax = warp_max(a);
    if (fmt == CSA_FMT_FP8) {
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint8_t *o = codes + orow * D + lane * E;
#pragma unroll
        for (int i = 0; i < E; i += 2) {
            uint16_t c = f32x2_to_e4m3x2(__fdiv_rn(v[i], s), __fdiv_rn(v[i + 1], s));
            *reinterpret_cast<uint16_t *>(o + i) = c;
        }
        if (lane == 0) scales[orow] = s;
        return s;
    }
    // FP4: row scale s_t = amax/2688, block-16 scale sb = RN(amax_blk/(6 s_t))
    // as unsigned E4M3, code = RNE(x/(sb s_t)).  A block spans 16/E lanes.
    const float st = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    float ab = a;
#pragma unroll
    for (int m = 1; m < 16 / E; m <<= 1) ab = fmaxf(ab, __shfl_xor_sync(0xffffffffu, ab, m));
    const float sbv = __fdiv_rn(ab, __fmul_rn(6.0f, st));
    const uint8_t sb = f32_to_e4m3(sbv);
    const float dq = __fmul_rn(e4m3_to_f32(sb), st);
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; i++) q[i] = 0.0f;
#pragma unroll
    for (int i = 0; i < E; i++)
        q[i] = dq > 0.0f ? __fdiv_rn(v[i], dq) : (signbit(v[i]) ? -0.0f : 0.0f);
    const uint32_t packed = f32x8_to_e2m1x8(q);
    if (fmt == CSA_FMT_FP4_PAGE) {
        // the slot's 8-key group inside its page's record: codes in 8-key x
        // 16-byte blocks, then the group's block scales, then its row scales
        constexpr int Gb = 4 * D + D / 2 + 32;
        const int r = (int)(orow & 63), i = r & 7;
        uint8_t *grp = codes + (orow >> 6) * (8 * Gb) + (r >> 3) * Gb;
        const int b = lane * (E / 2);          // this lane's first code byte (E/2 bytes, one block)
        uint8_t *o = grp + (b >> 4) * 128 + i * 16 + (b & 15);
        if (E == 4)
            *reinterpret_cast<uint16_t *>(o) = (uint16_t)(packed & 0xFFFF);
        else
            *o = (uint8_t)(packed & 0xFF);
        if ((lane % (16 / E)) == 0) grp[4 * D + i * (D / 16) + lane / (16 / E)] = sb;
        if (lane == 0) *reinterpret_cast<float *>(grp + 4 * D + D / 2 + 4 * i) = st;
        return st;
    }
    uint8_t *o = codes + orow * (D / 2) + lane * (E / 2);
    if (E == 4)
        *reinterpret_cast<uint16_t *>(o) = (uint16_t)(packed & 0xFFFF);
    else
        *o = (uint8_t)(packed & 0xFF);
    if ((lane % (16 / E)) == 0) block_scales[orow * (D / 16) + lane / (16 / E)] = sb;
    if (lane == 0) scales[orow] = st;
    return st;
}

// Rotary position embedding of the leading rope_dim values of a row held E per
// lane: consecutive pairs (x[2i], x[2i+1]) taken as the complex number
// x[2i] + i x[2i+1] and multiplied by freqs[pos][i] = (cos, sin); each product
// and sum rounded to float separately (no contraction).
template <int E>
__device__ __forceinline__ void apply_rope(float (&v)[E], int lane, const float2 *freqs,
                                           int rope_dim, int64_t pos) {
#pragma unroll
    for (int i = 0; i < E; i += 2) {
        const int d = lane * E + i;
        if (d < rope_dim) {
            const float2 cs = freqs[pos * (rope_dim / 2) + d / 2];
            const float a = v[i], b = v[i + 1];
            v[i] = __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y));
            v[i + 1] = __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x));
        }
    }
}

// ROT: apply the Hadamard rotation (the index rows of the C4 indexer) or not
// (plain per-row quantisation, the DSA indexer).  With rope.freqs set, the
// rotary embedding runs first at position rope.pos[r / rope.rows_per_pos].
template <int E, typename T, bool ROT>
__global__ void __launch_bounds__(256)
hadamard_quant_kernel(const T *__restrict__ x, int64_t rows, int fmt,
                      const int32_t *__restrict__ row_map, int64_t num_out_rows,
                      uint8_t *codes, uint8_t *block_scales, float *scales,
                      const float *__restrict__ w_in, float *w_out, int32_t *status,
                      const RopeArgs rope) {
    pdl_begin();
    constexpr int D = 32 * E;
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    int64_t orow = r;
    if (row_map) {
        orow = row_map[r];
        if (orow < 0) return;
        if (orow >= num_out_rows) {
            if (lane == 0) report(status, CSA_ERR_BOUNDS);
            return;
        }
    }
    float v[E];
#pragma unroll
    for (int i = 0; i < E; i++) {
        if constexpr (sizeof(T) == 2)
            v[i] = bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(x)[r * D + lane * E + i]);
        else
            v[i] = x[r * D + lane * E + i];
    }
    if (rope.freqs) {
        const int32_t p = rope.pos[r / rope.rows_per_pos];
        if (p < 0 || p >= rope.max_pos) {
            if (lane == 0) report(status, CSA_ERR_BOUNDS);
            return;
        }
        apply_rope<E>(v, lane, rope.freqs, rope.rope_dim, p);
    }
    if constexpr (ROT) rotate<E>(v, lane);
    const float s = quant_index_row<E>(v, lane, fmt, orow, codes, block_scales, scales);
    if (w_in && w_out && lane == 0) w_out[r] = w_in[r] * s;
}

// ------------------------------------------------------------------ compressor
//
// alpha_i[c] = softmax_i(g[4j+i][c] + b[i][c]),  y[j][c] = sum_i alpha_i[c] x[4j+i][c]
// (float32 math: y = (sum_i e_i x_i) / sum_i e_i with e_i = exp(z_i - max z)).

__device__ __forceinline__ float pool4(const float (&x)[4], const float (&z)[4]) {
    const float m = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
    float num = 0.0f, den = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float e = expf(z[i] - m);
        num = fmaf(e, x[i], num);
        den += e;
    }
    return __fdiv_rn(num, den);
}

// First input row of block `blk` of request b (or -1 when there is no such
// complete block, or the request is malformed); `j` gets the block's
// compressed index.
__device__ __forceinline__ int64_t compress_row(int b, int blk, const int32_t *cu_x,
                                                const int32_t *start_pos, int max_rows,
                                                int32_t *status, bool leader, int32_t *j,
                                                int ratio = 4) {
    const int32_t x0 = cu_x[b], n = cu_x[b + 1] - x0;
    const int32_t sp = start_pos[b];
    if (n < ratio) {                  // no complete block: nothing to compress
        if (n < 0 && leader && blk == 0) report(status, CSA_ERR_BOUNDS);
        return -1;
    }
    if (sp < 0 || (sp % ratio) != 0) {
        if (leader && blk == 0) report(status, CSA_ERR_BOUNDS);
        return -1;
    }
    if (n > max_rows && leader && blk == 0) report(status, CSA_ERR_BOUNDS);
    const int nblk = min(n, max_rows) / ratio;
    if (blk >= nblk) return -1;
    *j = sp / ratio + blk;
    return (int64_t)x0 + (int64_t)ratio * blk;
}

// Compressed slot of compressed index j of request b (rows_per_page compressed
// rows per 256-token page), or -1 (reported).
__device__ __forceinline__ int64_t compress_slot(int b, int32_t j, const int32_t *page_table,
                                                 int pt_stride, int64_t num_slots,
                                                 int32_t *status, bool leader,
                                                 int rows_per_page = kC4Page) {
    if (j / rows_per_page >= pt_stride) {
        if (leader) report(status, CSA_ERR_BOUNDS);
        return -1;
    }
    const int32_t page = page_table[(int64_t)b * pt_stride + j / rows_per_page];
    const int64_t slot = (int64_t)page * rows_per_page + j % rows_per_page;
    if (page < 0 || slot >= num_slots) {
        if (leader) report(status, CSA_ERR_BOUNDS);
        return -1;
    }
    return slot;
}

// KV mode: one compressed row per CTA of 160 threads; grid (blocks, bs).
__global__ void __launch_bounds__(kKvRowThreads)
compress_kv_kernel(const float *__restrict__ x, const float *__restrict__ gate,
                   const float *__restrict__ bias, const int32_t *cu_x,
                   const int32_t *start_pos, int max_rows, const int32_t *page_table,
                   int pt_stride, int fmt, uint8_t *out, int64_t num_slots, int32_t *status) {
    pdl_begin();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t j = 0;
    const int64_t row0 = compress_row(blockIdx.y, blockIdx.x, cu_x, start_pos, max_rows, status,
                                      threadIdx.x == 0, &j);
    if (row0 < 0) return;
    // the input rows are fetched before the page-table lookup resolves
    float4 xv[4], gv[4], bv[4];
    if (kv_active(warp, lane)) {
        const int c = kv_channel(warp, lane);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            xv[i] = *reinterpret_cast<const float4 *>(x + (row0 + i) * kKvDim + c);
            gv[i] = *reinterpret_cast<const float4 *>(gate + (row0 + i) * kKvDim + c);
            bv[i] = *reinterpret_cast<const float4 *>(bias + i * kKvDim + c);
        }
    }
    const int64_t slot = compress_slot(blockIdx.y, j, page_table, pt_stride, num_slots, status,
                                       threadIdx.x == 0);
    if (slot < 0) return;
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kv_active(warp, lane)) {
        float xs[4], zs[4];
#define CSA_POOL_LANE(F)                                                              \
        for (int i = 0; i < 4; i++) { xs[i] = xv[i].F; zs[i] = gv[i].F + bv[i].F; } \
        y.F = pool4(xs, zs);
        CSA_POOL_LANE(x)
        CSA_POOL_LANE(y)
        CSA_POOL_LANE(z)
        CSA_POOL_LANE(w)
#undef CSA_POOL_LANE
    }
    const int row_bytes = fmt == CSA_FMT_FP8 ? kFp8RowBytes : kBf16RowBytes;
    write_kv_row(y, warp, lane, fmt, out + slot * row_bytes);
}

// HCA: one compressed row of 128 raw rows per CTA of 160 threads (4 channels
// per active thread); the softmax over the block runs online (running maximum,
// rescaled sum and weighted sum), four rows in flight at a time.
__global__ void __launch_bounds__(kKvRowThreads)
compress_hca_kernel(const float *__restrict__ x, const float *__restrict__ gate,
                    const float *__restrict__ bias, const int32_t *cu_x,
                    const int32_t *start_pos, int max_rows, const int32_t *page_table,
                    int pt_stride, int fmt, uint8_t *out, int64_t num_slots, int32_t *status) {
    pdl_begin();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t j = 0;
    const int64_t row0 = compress_row(blockIdx.y, blockIdx.x, cu_x, start_pos, max_rows, status,
                                      threadIdx.x == 0, &j, kHcaRatio);
    if (row0 < 0) return;
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kv_active(warp, lane)) {
        const int c = kv_channel(warp, lane);
        float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float Z[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int i0 = 0; i0 < kHcaRatio; i0 += 4) {
            float4 xv[4], zv[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                xv[i] = *reinterpret_cast<const float4 *>(x + (row0 + i0 + i) * kKvDim + c);
                const float4 g = *reinterpret_cast<const float4 *>(gate + (row0 + i0 + i) * kKvDim + c);
                const float4 bb = *reinterpret_cast<const float4 *>(bias + (i0 + i) * kKvDim + c);
                zv[i] = make_float4(g.x + bb.x, g.y + bb.y, g.z + bb.z, g.w + bb.w);
            }
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float zz[4] = {zv[i].x, zv[i].y, zv[i].z, zv[i].w};
                const float xx[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    if (zz[k] > m[k]) {
                        const float sc = expf(m[k] - zz[k]);     // 0 on the first row
                        Z[k] = Z[k] * sc + 1.0f;
                        acc[k] = acc[k] * sc + xx[k];
                        m[k] = zz[k];
                    } else {
                        const float e = expf(zz[k] - m[k]);
                        Z[k] += e;
                        acc[k] = fmaf(e, xx[k], acc[k]);
                    }
                }
            }
        }
        y = make_float4(acc[0] / Z[0], acc[1] / Z[1], acc[2] / Z[2], acc[3] / Z[3]);
    }
    const int64_t slot = compress_slot(blockIdx.y, j, page_table, pt_stride, num_slots, status,
                                       threadIdx.x == 0, kHcaPage);
    if (slot < 0) return;
    const int row_bytes = fmt == CSA_FMT_FP8 ? kFp8RowBytes : kBf16RowBytes;
    write_kv_row(y, warp, lane, fmt, out + slot * row_bytes);
}

// Index-key mode: one compressed row per warp, 8 rows per CTA; grid
// (ceil(blocks/8), bs).  Pool, rotate, quantise into the index-key arrays.
template <int E>
__global__ void __launch_bounds__(256)
compress_index_kernel(const float *__restrict__ x, const float *__restrict__ gate,
                      const float *__restrict__ bias, const int32_t *cu_x,
                      const int32_t *start_pos, int max_rows, const int32_t *page_table,
                      int pt_stride, int fmt, uint8_t *codes, uint8_t *block_scales,
                      float *scales, int64_t num_slots, int32_t *status, const RopeArgs rope) {
    pdl_begin();
    constexpr int D = 32 * E;
    const int lane = threadIdx.x & 31;
    const int blk = blockIdx.x * 8 + (threadIdx.x >> 5);
    int32_t j = 0;
    const int64_t row0 = compress_row(blockIdx.y, blk, cu_x, start_pos, max_rows, status,
                                      lane == 0, &j);
    if (row0 < 0) return;
    float xs[E][4], zs[E][4];
#pragma unroll
    for (int e = 0; e < E; e++) {
        const int c = lane * E + e;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            xs[e][i] = x[(row0 + i) * D + c];
            zs[e][i] = gate[(row0 + i) * D + c] + bias[i * D + c];
        }
    }
    const int64_t slot = compress_slot(blockIdx.y, j, page_table, pt_stride, num_slots, status,
                                       lane == 0);
    if (slot < 0) return;
    float v[E];
#pragma unroll
    for (int e = 0; e < E; e++) v[e] = pool4(xs[e], zs[e]);
    if (rope.freqs) {
        // the compressed key of block j stands at the raw position of its first row
        const int64_t p = 4 * (int64_t)j;
        if (p >= rope.max_pos) {
            if (lane == 0) report(status, CSA_ERR_BOUNDS);
            return;
        }
        apply_rope<E>(v, lane, rope.freqs, rope.rope_dim, p);
    }
    rotate<E>(v, lane);
    quant_index_row<E>(v, lane, fmt, slot, codes, block_scales, scales);
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_kv_store(const float *rows, int64_t n, const int32_t *slots, int fmt,
                            void *cache, int64_t num_slots, int32_t *status, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int grid = (int)(n < 65535 * 8 ? n : 65535 * 8);
    launch_k(kv_store_kernel, grid, kKvRowThreads, 0, s, rows, n, slots, fmt, (uint8_t *)cache,
                                                   num_slots, status);
    return cudaGetLastError();
}

cudaError_t launch_hadamard_quant(const void *x, int x_dtype, int64_t rows, int dim, int fmt,
                                  const int32_t *row_map, int64_t num_out_rows, void *codes,
                                  uint8_t *block_scales, float *scales, const float *w_in,
                                  float *w_out, int32_t *status, cudaStream_t s, bool rotate,
                                  const RopeArgs &rope) {
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    uint8_t *c = (uint8_t *)codes;
#define CSA_HQ(E, T, R)                                                                     \
    launch_k(hadamard_quant_kernel<E, T, R>, grid, 256, 0, s, (const T *)x, rows, fmt, row_map, \
             num_out_rows, c, block_scales, scales, w_in, w_out, status, rope)
#define CSA_HQ2(E, T) do { if (rotate) CSA_HQ(E, T, true); else CSA_HQ(E, T, false); } while (0)
    if (dim == 64 && x_dtype == CSA_FMT_BF16) CSA_HQ2(2, uint16_t);
    else if (dim == 64) CSA_HQ2(2, float);
    else if (x_dtype == CSA_FMT_BF16) CSA_HQ2(4, uint16_t);
    else CSA_HQ2(4, float);
#undef CSA_HQ2
#undef CSA_HQ
    return cudaGetLastError();
}

cudaError_t launch_hca_compress(const float *x, const float *gate, const float *bias, int bs,
                                const int32_t *cu_x, const int32_t *start_pos, int max_rows,
                                const int32_t *page_table, int pt_stride, int out_kind, void *out,
                                int64_t num_slots, int32_t *status, cudaStream_t s) {
    const int max_blocks = max_rows / kHcaRatio;
    if (bs == 0 || max_blocks == 0) return cudaSuccess;
    const int fmt = out_kind == CSA_OUT_KV_FP8 ? CSA_FMT_FP8 : CSA_FMT_BF16;
    launch_k(compress_hca_kernel, dim3(max_blocks, bs), kKvRowThreads, 0, s, x, gate, bias, cu_x,
             start_pos, max_rows, page_table, pt_stride, fmt, (uint8_t *)out, num_slots, status);
    return cudaGetLastError();
}

cudaError_t launch_c4_compress(const float *x, const float *gate, const float *bias, int dim,
                               int bs, const int32_t *cu_x, const int32_t *start_pos,
                               int max_rows, const int32_t *page_table, int pt_stride,
                               int out_kind, void *out, uint8_t *out_block_scales,
                               float *out_scales, int64_t num_slots, int32_t *status,
                               cudaStream_t s, const RopeArgs &rope) {
    const int max_blocks = max_rows / 4;
    if (bs == 0 || max_blocks == 0) return cudaSuccess;
    if (out_kind == CSA_OUT_KV_BF16 || out_kind == CSA_OUT_KV_FP8) {
        const int fmt = out_kind == CSA_OUT_KV_FP8 ? CSA_FMT_FP8 : CSA_FMT_BF16;
        dim3 grid(max_blocks, bs);
        launch_k(compress_kv_kernel, grid, kKvRowThreads, 0, s, x, gate, bias, cu_x, start_pos,
                                                          max_rows, page_table, pt_stride, fmt,
                                                          (uint8_t *)out, num_slots, status);
    } else {
        const int fmt = out_kind == CSA_OUT_INDEX_FP8        ? CSA_FMT_FP8
                        : out_kind == CSA_OUT_INDEX_FP4      ? CSA_FMT_FP4
                        : out_kind == CSA_OUT_INDEX_FP4_PAGE ? CSA_FMT_FP4_PAGE
                                                             : CSA_FMT_BF16;
        dim3 grid((max_blocks + 7) / 8, bs);
        if (dim == 64)
            launch_k(compress_index_kernel<2>, grid, 256, 0, s, 
                x, gate, bias, cu_x, start_pos, max_rows, page_table, pt_stride, fmt,
                (uint8_t *)out, out_block_scales, out_scales, num_slots, status, rope);
        else
            launch_k(compress_index_kernel<4>, grid, 256, 0, s, 
                x, gate, bias, cu_x, start_pos, max_rows, page_table, pt_stride, fmt,
                (uint8_t *)out, out_block_scales, out_scales, num_slots, status, rope);
    }
    return cudaGetLastError();
}

}  // namespace csa
