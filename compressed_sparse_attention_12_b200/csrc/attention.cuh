// attention.cuh -- per-query bookkeeping shared by the sparse-attention
// kernels: the query's request, position and window, the slot of each entry
// of its row list (selected compressed rows, or every visible HCA row, then
// the raw window), and small conversion helpers.
#pragma once

#include "common.cuh"
#include "launch.h"

namespace csa {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}

struct AtQuery {
    int b, p, nw;        // request, raw position, window rows
    int nsel;            // rows before the window (512 selected, or the HCA rows)
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
    q.nsel = kTopK;
    if (a.dense_ratio > 0) {
        const int len = a.seq_lens[lo] / a.dense_ratio;
        q.nsel = max(0, min(len, (q.p + 1) / a.dense_ratio));
        if (q.nsel > a.max_sel) {
            report(a.status, CSA_ERR_BOUNDS);
            q.nsel = a.max_sel;
        }
    }
    return q;
}

// Slot of entry r of the query's row list (-1: masked).  Entries 0..511 are
// the selected compressed rows, then the window's raw positions in order.
__device__ __forceinline__ int32_t row_slot(const AttnArgs &a, const AtQuery &qq, int t, int r,
                                            int32_t *raw) {
    *raw = 0;
    if (r < qq.nsel) {
        if (a.dense_ratio > 0) {
            // HCA: every visible compressed row, kPage / ratio of them per page
            const int rpp = kPage / a.dense_ratio;
            const int32_t page = r / rpp < a.pt_stride
                                     ? a.page_table[(int64_t)qq.b * a.pt_stride + r / rpp]
                                     : -1;
            const int64_t slot = (int64_t)page * rpp + r % rpp;
            if (page < 0 || slot >= a.num_c4_slots) {
                report(a.status, CSA_ERR_BOUNDS);
                return -1;
            }
            return (int32_t)slot;
        }
        int32_t slot = a.idx[(int64_t)t * kTopK + r];
        if (slot >= a.num_c4_slots) {
            report(a.status, CSA_ERR_BOUNDS);
            slot = -1;
        }
        return slot < 0 ? -1 : slot;
    }
    if (r - qq.nsel >= qq.nw) return -1;
    const int pos = qq.p - qq.nw + 1 + (r - qq.nsel);
    const int32_t page = pos / kPage < a.pt_stride
                             ? a.page_table[(int64_t)qq.b * a.pt_stride + pos / kPage]
                             : -1;
    const int64_t s = (int64_t)page * kPage + pos % kPage;
    if (page < 0 || s >= a.num_raw_slots) {
        report(a.status, CSA_ERR_BOUNDS);
        return -1;
    }
    *raw = 1;
    return (int32_t)s;
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Power of two 2^(top - e) for amax = f * 2^e with f in [0.5, 1), so that
// amax times it lies in [2^(top-1), 2^top); 1 for amax == 0.  Exponents are
// clamped to the normal float range.
__device__ __forceinline__ float fit_pow2(float amax, int top) {
    if (!(amax > 0.0f)) return 1.0f;
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 126;
    const int k = max(-126, min(126, top - e));
    return __uint_as_float((uint32_t)(k + 127) << 23);
}

}  // namespace csa
