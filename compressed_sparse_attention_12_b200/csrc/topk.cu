// topk.cu -- step 3, the fixed-k top-512 with the paged index transform
// ("Token 的一生：DSV4 架构与 DSpark" §3.2 topk_transform_512, page arithmetic
// of §2.2).
//
// Selection is exact on order-preserving 32-bit keys of the float logits
// (-0 folded onto +0, NaN recorded and ordered below -inf).  The order is
// (logit descending, logical index ascending); outputs are listed in
// ascending logical index and padded with -1.
//
// Forms, chosen on the host by the batch's row count and longest row
// (launch_topk512):
//   * a thread-block cluster of 4 or 2 CTAs per row (up to one wave of them,
//     rows of 8193..32768 logits): topk_cluster_kernel;
//   * one CTA per row holding the row in registers (rows of at most 32768
//     logits) or in shared memory (at most 49152): topk_reg_kernel,
//     topk_row_kernel;
//   * for at most 64 longer rows, a bound from group maxima applied by every
//     chunk's CTA, then one CTA per row: the three topk_tb_* kernels;
//   * otherwise two launches:
//     stage 1: each CTA takes a chunk of logits of one query row into shared
//              memory and writes the chunk's top-512 (key, index) pairs in
//              index order plus (512th key, largest key) to the workspace
//              (select_chunk in topk.cuh; the indexer kernel can run the same
//              step on its own chunk instead);
//     stage 2: one CTA per query row selects among the row's concatenated
//              candidates (every element of the global top-512 is in its
//              chunk's top-512 under the same total order).
// Every form writes physical slots page_table[s/64]*64 + s%64 and raw indices.
#include "common.cuh"
#include "launch.h"
#include <atomic>
#include <cstdint>

#include "topk.cuh"

namespace csa {

constexpr int kTkThreads = 512;
constexpr int kTkChunk = 8192;
constexpr int kTk2Smem = 16384;      // stage-2 candidates staged in shared memory
using TkShared = TkSharedT<kTkThreads>;
// the key buffers that follow TkShared in dynamic shared memory start on a
// 16-byte boundary (they are read and written with 16-byte vectors)
constexpr size_t kTkKeysOffset = (sizeof(TkShared) + 15) & ~(size_t)15;

struct RowInfo {
    int b, n_vis;
};

// Request and visible length of query row t, found by warp 0 with coalesced
// reads of cu_q and c4_lens (one round trip for up to 32 requests) and
// published to the block through shared memory.
template <int NT>
__device__ RowInfo row_info(int t, const int32_t *cu_q, int bs, const int32_t *q_pos,
                            const int32_t *c4_lens, int max_c4_len, int pt_stride,
                            int32_t *status, bool leader, TkSharedT<NT> &sh, int ratio) {
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int pos = q_pos ? q_pos[t] : 0;
        int cnt = 0, len = 0;
        for (int base = 0; base < bs; base += 32) {
            const int i = base + lane;
            const bool le = i < bs && cu_q[i] <= t;
            const int li = i < bs ? c4_lens[i] : 0;
            const uint32_t m = __ballot_sync(0xffffffffu, le);
            const int c = __popc(m);
            // the last request whose start is <= t is entry cnt+c-1
            const int src = c > 0 ? c - 1 : 0;
            const int lsel = __shfl_sync(0xffffffffu, li, src);
            if (c > 0) len = lsel;
            cnt += c;
            if (m != 0xffffffffu) break;
        }
        if (lane == 0) {
            int n = len;
            if (q_pos) n = min(n, (pos + 1) / ratio);
            const int cap = min(max_c4_len, pt_stride * kC4Page);
            if (n > cap) {
                if (leader) report(status, CSA_ERR_BOUNDS);
                n = cap;
            }
            sh.row_b = max(cnt - 1, 0);
            sh.row_nvis = max(n, 0);
        }
    }
    __syncthreads();
    RowInfo r;
    r.b = sh.row_b;
    r.n_vis = sh.row_nvis;
    return r;
}

// Stage 1: one CTA per (query row, 8192-logit chunk).  Writes the chunk's
// top-512 (or all of it when shorter) in index order, plus the chunk's
// 512th-largest key (0 when it holds fewer) and its largest key.
__global__ void __launch_bounds__(kTkThreads)
topk_stage1_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens,
                   int bs, const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                   int pt_stride, int max_chunks, uint32_t *cand_key, int32_t *cand_idx,
                   uint2 *chunk_info, int32_t *status, int ratio) {
    pdl_begin();
    extern __shared__ __align__(16) uint8_t tk_smem[];
    TkShared &sh = *reinterpret_cast<TkShared *>(tk_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tk_smem + kTkKeysOffset);
    const int t = blockIdx.y, c = blockIdx.x;
    const RowInfo ri = row_info<kTkThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride,
                                            status, c == 0, sh, ratio);
    const int lo = c * kTkChunk;
    if (lo >= ri.n_vis) return;
    const int len = min(kTkChunk, ri.n_vis - lo);
    stage_row_keys<kTkThreads>(skeys, logits + (int64_t)t * stride + lo, len);
    __syncthreads();
    select_chunk<kTkThreads>(skeys, len, lo, cand_key + ((int64_t)t * max_chunks + c) * kTopK,
                             cand_idx + ((int64_t)t * max_chunks + c) * kTopK,
                             chunk_info + (int64_t)t * max_chunks + c, sh, status);
}

// Stage 2: one CTA per query row.  The row's top-512 are all >= L, the largest
// of the chunks' 512th keys (that chunk alone holds 512 keys >= L), so the
// candidates below L are dropped first (in index order, into shared memory),
// the threshold is found among the survivors, and the selection is written in
// ascending index order, mapped through the page table, then padded with -1.
__global__ void __launch_bounds__(kTkThreads)
topk_stage2_kernel(const int32_t *c4_lens, int bs, const int32_t *cu_q, const int32_t *q_pos,
                   int max_c4_len, const int32_t *page_table, int pt_stride, int64_t num_slots,
                   int max_chunks, int chunk_len, const uint32_t *cand_key,
                   const int32_t *cand_idx, const uint2 *chunk_info, int32_t *out_phys,
                   int32_t *out_raw, int32_t *status, int ratio) {
    pdl_begin();
    extern __shared__ __align__(16) uint8_t tk2_smem[];
    TkShared &sh = *reinterpret_cast<TkShared *>(tk2_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tk2_smem + kTkKeysOffset);
    int32_t *sidx = reinterpret_cast<int32_t *>(skeys + kTk2Smem);
    const int t = blockIdx.x;
    const RowInfo ri = row_info<kTkThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride,
                                            status, false, sh, ratio);
    const int n = ri.n_vis;
    int total = 0, nch = 0;
    if (n > 0) {
        nch = (n + chunk_len - 1) / chunk_len;
        total = (nch - 1) * kTopK + min(kTopK, n - (nch - 1) * chunk_len);
    }
    const int K = min(kTopK, total);
    const uint32_t *keys = cand_key + (int64_t)t * max_chunks * kTopK;
    const int32_t *idx = cand_idx + (int64_t)t * max_chunks * kTopK;
    uint32_t T = 0;
    int need_eq = total;
    int m = total;
    if (total > kTopK) {
        uint32_t L = 0, kmax = 0;
        for (int c = threadIdx.x; c < nch; c += kTkThreads) {
            const uint2 ci = chunk_info[(int64_t)t * max_chunks + c];
            L = max(L, ci.x);
            kmax = max(kmax, ci.y);
        }
        // A tighter bound: the F full chunks (512 candidates each: all but the
        // last) each hold m = ceil(512/F) keys >= their own m-th largest, so the
        // row's 512th key is >= the smallest of those.  Warp w finds the m-th
        // largest of chunks w, w+16, ... by a bitwise search over the key (16
        // keys per lane, one warp sum per bit).
        const int F = (n - (nch - 1) * chunk_len) >= kTopK ? nch : nch - 1;
        uint32_t Lm = 0xffffffffu;
        if (F >= 1) {
            const int mth = (kTopK + F - 1) / F;
            const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
            for (int c = warp; c < F; c += kTkThreads / 32) {
                uint32_t kk[16];
                const uint4 *src = reinterpret_cast<const uint4 *>(keys + (int64_t)c * kTopK) + lane * 4;
#pragma unroll
                for (int v = 0; v < 4; v++) {
                    const uint4 x = src[v];
                    kk[4 * v] = x.x; kk[4 * v + 1] = x.y; kk[4 * v + 2] = x.z; kk[4 * v + 3] = x.w;
                }
                uint32_t Tc = 0;
#pragma unroll 1
                for (int bit = 31; bit >= 0; bit--) {
                    const uint32_t cand = Tc | (1u << bit);
                    int cnt = 0;
#pragma unroll
                    for (int j = 0; j < 16; j++) cnt += kk[j] >= cand ? 1 : 0;
                    if (__reduce_add_sync(0xffffffffu, (unsigned)cnt) >= (unsigned)mth) Tc = cand;
                }
                Lm = min(Lm, Tc);
            }
        } else {
            Lm = 0;
        }
        uint32_t lneg = ~L;
        block_minmax<kTkThreads>(lneg, kmax, sh);     // min of ~L is ~(max of L)
        L = ~lneg;
        uint32_t dummy = 0;
        block_minmax<kTkThreads>(Lm, dummy, sh);
        L = max(L, Lm);
        // Batches of 512 x 32 candidates: thread i of a batch holds candidates
        // [32i, 32i+32) (all loads in flight at once); the survivors (keys >= L)
        // are appended in order to shared memory with one block scan per batch.
        // Rows whose survivors overflow the buffer select straight from the
        // workspace.
        constexpr int kPer = 32;
        constexpr int kBatch = kTkThreads * kPer;
        uint32_t n_surv = 0;
        bool fits = true;
#pragma unroll 1
        for (int b0 = 0; b0 < total; b0 += kBatch) {
            const int i0 = b0 + threadIdx.x * kPer;
            uint32_t kk[kPer];
            int32_t ii[kPer];
#pragma unroll
            for (int j = 0; j < kPer; j += 4) {
                const int i = i0 + j;
                if (i + 4 <= total) {
                    const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + i);
                    const int4 x4 = *reinterpret_cast<const int4 *>(idx + i);
                    kk[j] = k4.x; kk[j + 1] = k4.y; kk[j + 2] = k4.z; kk[j + 3] = k4.w;
                    ii[j] = x4.x; ii[j + 1] = x4.y; ii[j + 2] = x4.z; ii[j + 3] = x4.w;
                } else {
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        kk[j + q] = i + q < total ? keys[i + q] : 0u;
                        ii[j + q] = i + q < total ? idx[i + q] : 0;
                    }
                }
            }
            uint32_t mine = 0;
#pragma unroll
            for (int j = 0; j < kPer; j++) mine += (i0 + j < total && kk[j] >= L) ? 1u : 0u;
            uint32_t surv;
            uint32_t pos = n_surv + block_excl_scan<kTkThreads>(mine, &surv, sh);
            if (n_surv + surv > (uint32_t)kTk2Smem) {      // uniform over the block
                fits = false;
                break;
            }
#pragma unroll
            for (int j = 0; j < kPer; j++) {
                if (i0 + j < total && kk[j] >= L) {
                    skeys[pos] = kk[j];
                    sidx[pos] = ii[j];
                    pos++;
                }
            }
            n_surv += surv;
        }
        __syncthreads();
        if (fits) {
            keys = skeys;
            idx = sidx;
            m = (int)n_surv;
        }
        radix_threshold<kTkThreads>(keys, m, K, L, kmax, sh, &T, &need_eq);
    }
    const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    ordered_compact<kTkThreads>(keys, m, T, need_eq, sh, [&](int pos, int i, uint32_t) {
        const int32_t s = idx[i];
        const int32_t page = pt_row[s / kC4Page];
        const int64_t slot = (int64_t)page * kC4Page + s % kC4Page;
        int32_t phys = (int32_t)slot;
        if (page < 0 || slot >= num_slots) {
            report(status, CSA_ERR_BOUNDS);
            phys = -1;
        }
        op[pos] = phys;
        if (orw) orw[pos] = s;
    });
    for (int p = K + threadIdx.x; p < kTopK; p += kTkThreads) {
        op[p] = -1;
        if (orw) orw[p] = -1;
    }
}

// Rows of at most kTkRowMax logits in one launch: one CTA of 1024 threads per
// query row stages the whole row in shared memory as keys, selects its
// top-512 and writes the physical slots, raw indices and -1 padding.
constexpr int kTkRowThreads = 1024;
constexpr int kTkRowMax = 49152;
using TkRowShared = TkSharedT<kTkRowThreads>;
constexpr size_t kTkRowKeysOffset = (sizeof(TkRowShared) + 15) & ~(size_t)15;

__global__ void __launch_bounds__(kTkRowThreads, 1)
topk_row_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens, int bs,
                const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                const int32_t *page_table, int pt_stride, int64_t num_slots, int32_t *out_phys,
                int32_t *out_raw, int32_t *status, int ratio) {
    pdl_begin();
    extern __shared__ __align__(16) uint8_t tkr_smem[];
    TkRowShared &sh = *reinterpret_cast<TkRowShared *>(tkr_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tkr_smem + kTkRowKeysOffset);
    const int t = blockIdx.x;
    const RowInfo ri = row_info<kTkRowThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len,
                                               pt_stride, status, true, sh, ratio);
    const int len = min(ri.n_vis, kTkRowMax);     // the host keeps max_c4_len <= kTkRowMax
    stage_row_keys<kTkRowThreads>(skeys, logits + (int64_t)t * stride, len);
    __syncthreads();
    const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    uint32_t T, kmax;
    const int K = select_top512<kTkRowThreads>(skeys, len, sh, status, &T, &kmax,
                                               [&](int pos, int s, uint32_t) {
        const int32_t page = pt_row[s / kC4Page];
        const int64_t slot = (int64_t)page * kC4Page + s % kC4Page;
        int32_t phys = (int32_t)slot;
        if (page < 0 || slot >= num_slots) {
            report(status, CSA_ERR_BOUNDS);
            phys = -1;
        }
        op[pos] = phys;
        if (orw) orw[pos] = s;
    });
    for (int p = K + threadIdx.x; p < kTopK; p += kTkRowThreads) {
        op[p] = -1;
        if (orw) orw[p] = -1;
    }
}

// Rows of at most kTkRegMax logits: one CTA of 1024 threads per query row
// holds the row in registers (32 keys per thread, loaded in coalesced 16-byte
// slices), so every sweep over the row is register-only; shared memory holds
// the radix histogram and the staged candidates.
constexpr int kTkRegKpt = 32;
constexpr int kTkRegMax = kTkRowThreads * kTkRegKpt;
constexpr int kTkRegCap = 3072;      // staged candidates (keys >= the group bound)

__global__ void __launch_bounds__(kTkRowThreads, 1)
topk_reg_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens, int bs,
                const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                const int32_t *page_table, int pt_stride, int64_t num_slots, int32_t *out_phys,
                int32_t *out_raw, int32_t *status, int ratio) {
    pdl_begin();
    __shared__ TkRowShared sh;
    __shared__ uint32_t cand_key[kTkRegCap];
    __shared__ int32_t cand_idx[kTkRegCap];
    const int t = blockIdx.x;
    const RowInfo ri = row_info<kTkRowThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len,
                                               pt_stride, status, true, sh, ratio);
    const int len = min(ri.n_vis, kTkRegMax);     // the host keeps max_c4_len <= kTkRegMax
    const float *row = logits + (int64_t)t * stride;
    // coalesced: slice j of lane l in warp w is keys 1024w + 128j + 4l .. +3
    const int w0 = (int)(threadIdx.x >> 5) * 1024 + 4 * (int)(threadIdx.x & 31);
    const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
    uint32_t keys[kTkRegKpt];
#pragma unroll
    for (int j = 0; j < kTkRegKpt / 4; j++) {
        const int i0 = w0 + 128 * j;
        if (vec && i0 + 4 <= len) {
            const uint4 x = *reinterpret_cast<const uint4 *>(row + i0);
            keys[4 * j] = x.x;
            keys[4 * j + 1] = x.y;
            keys[4 * j + 2] = x.z;
            keys[4 * j + 3] = x.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; e++)
                keys[4 * j + e] = i0 + e < len ? __float_as_uint(row[i0 + e]) : 0u;
        }
    }
    const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    const int K = select_top512_regs<kTkRowThreads, kTkRegKpt>(keys, len, sh, cand_key, cand_idx,
                                                               kTkRegCap, status,
                                                               [&](int pos, int s) {
        const int32_t page = pt_row[s / kC4Page];
        const int64_t slot = (int64_t)page * kC4Page + s % kC4Page;
        int32_t phys = (int32_t)slot;
        if (page < 0 || slot >= num_slots) {
            report(status, CSA_ERR_BOUNDS);
            phys = -1;
        }
        op[pos] = phys;
        if (orw) orw[pos] = s;
    });
    for (int p = K + threadIdx.x; p < kTopK; p += kTkRowThreads) {
        op[p] = -1;
        if (orw) orw[p] = -1;
    }
}

// ------------------------------------------------------------------ cluster rows
//
// A few rows of at most kTkRegMax logits (decode batches): a cluster of C CTAs
// per row, so that the sweeps over the row's keys run on C SMs instead of one.
// CTA c of the cluster holds keys [c*chunk, (c+1)*chunk), chunk = kTkRegMax/C,
// in registers, in the layout of ordered_starts (16-byte slices of 4
// consecutive keys; warps, slices and lanes in index order).
//   1. The groups are the slices.  How many non-empty groups each CTA has
//      follows from the row length alone, so every CTA knows every CTA's quota
//      K_c = floor(512 * groups_c / groups_total) (CTA 0 also takes the
//      remainder, so the quotas sum to 512), and CTA c finds L_c, the lower
//      edge of the radix bin holding its K_c-th largest group maximum (one
//      pass).  With L the smallest L_c over the CTAs with a quota, at least
//      512 groups hold a key >= L, so every key of the top 512 is >= L (L = 0
//      when the row has fewer than 512 groups).  A CTA holding only a few
//      groups gets no quota, so its keys do not lower L.
//   2. Through distributed shared memory the CTAs exchange (L_c, largest
//      key), then their counts of keys >= L, and write those keys and their
//      indices, in index order, into CTA 0's candidate buffer.
//   3. CTA 0 selects the top 512 among the candidates as the one-CTA kernels
//      do, with the page transform and -1 padding.  If the candidates overflow
//      its buffer (heavy ties), CTA 0 stages the whole row there instead and
//      selects from it.
// Every CTA takes the same cluster barriers (branches depend on cluster-wide
// values only); every remote write lands before a barrier that its target
// passes, and no CTA is written to after it has passed its last barrier.
constexpr int kClThreads = 512;
constexpr int kClMaxC = 4;
constexpr int kClCap = 16384;                    // candidates in CTA 0 (key + index)
constexpr size_t kClSmem = (size_t)kClCap * 8;   // also holds a whole row of floats
constexpr int kClMinLen = 8192;                  // shorter rows: one CTA per row
constexpr int kClSms = 148;                      // CTAs of one wave (SMs of a B200)
static_assert(kClSmem >= (size_t)kTkRegMax * 4, "the fallback stages a whole row");
using TkClShared = TkSharedT<kClThreads>;

struct ClMail {
    uint32_t lc[kClMaxC];       // per CTA: its bound L_c (all ones: no bound)
    uint32_t kmax[kClMaxC];     // per CTA: its largest key
    uint32_t cnt[kClMaxC];      // per CTA: its keys >= L
};

// Address of `p` (this CTA's shared memory) in the shared memory of CTA
// `rank` of the cluster.
__device__ __forceinline__ uint32_t cl_map(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(r)
                 : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void cl_st(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Every thread of every CTA of the cluster arrives; writes before it are
// visible to reads after it anywhere in the cluster.
__device__ __forceinline__ void cl_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int C>
__global__ void __launch_bounds__(kClThreads, 1)
topk_cluster_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens,
                    int bs, const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                    const int32_t *page_table, int pt_stride, int64_t num_slots,
                    int32_t *out_phys, int32_t *out_raw, int32_t *status, int ratio) {
    constexpr int NT = kClThreads, KPT = kTkRegMax / (C * NT), NS = KPT / 4;
    constexpr int kChunk = NT * KPT;
    static_assert(C >= 2 && C <= kClMaxC && KPT % 4 == 0 && NS <= 32, "cluster layout");
    __shared__ TkClShared sh;
    __shared__ ClMail mail;
    extern __shared__ __align__(16) uint8_t cl_smem[];
    uint32_t *cand_key = reinterpret_cast<uint32_t *>(cl_smem);
    int32_t *cand_idx = reinterpret_cast<int32_t *>(cl_smem + (size_t)kClCap * 4);
    // this CTA has started (the wait before the first remote write pairs with it)
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    pdl_trigger();
    const int crank = blockIdx.x, t = blockIdx.y;
    const RowInfo ri = row_info<NT>(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride, status,
                                    crank == 0, sh, ratio);
    pdl_wait();
    const int len = min(ri.n_vis, kTkRegMax);     // the host keeps max_c4_len <= kTkRegMax
    const float *row = logits + (int64_t)t * stride;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // slice j of lane l in warp w: keys lo + 32*KPT*w + 128j + 4l .. +3
    const int w0 = crank * kChunk + warp * (32 * KPT) + 4 * lane;
    auto index_of = [&](int kk) { return w0 + 128 * (kk >> 2) + (kk & 3); };
    const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
    uint32_t keys[KPT];
#pragma unroll
    for (int j = 0; j < NS; j++) {
        const int i0 = w0 + 128 * j;
        if (vec && i0 + 4 <= len) {
            const uint4 x = *reinterpret_cast<const uint4 *>(row + i0);
            keys[4 * j] = x.x;
            keys[4 * j + 1] = x.y;
            keys[4 * j + 2] = x.z;
            keys[4 * j + 3] = x.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; e++)
                keys[4 * j + e] = i0 + e < len ? __float_as_uint(row[i0 + e]) : 0u;
        }
    }
    // keys, slice maxima, the CTA's smallest slice maximum and largest key
    uint32_t gm[NS];
    uint32_t gpres = 0;          // bit j: slice j holds a key
    uint32_t gmin = 0xffffffffu, kmx = 0u;
#pragma unroll
    for (int j = 0; j < NS; j++) {
        gm[j] = 0u;
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int kk = 4 * j + e;
            const bool p = index_of(kk) < len;
            const uint32_t k = p ? order_key(__uint_as_float(keys[kk]), status) : 0u;
            keys[kk] = k;
            if (p) gm[j] = max(gm[j], k);
        }
        if (index_of(4 * j) < len) {
            gpres |= 1u << j;
            gmin = min(gmin, gm[j]);
            kmx = max(kmx, gm[j]);
        }
    }
    block_minmax<NT>(gmin, kmx, sh);
    // this CTA's bound L_c
    auto groups_of = [&](int c) {
        const int m = min(len, (c + 1) * kChunk) - c * kChunk;
        return m > 0 ? (m + 3) >> 2 : 0;
    };
    int g_total = 0;
#pragma unroll
    for (int c = 0; c < C; c++) g_total += groups_of(c);
    const int K = min(kTopK, len);
    uint32_t Lc = 0u;
    if (len > kTopK && g_total >= kTopK) {
        Lc = 0xffffffffu;
        // quotas floor(512 g_c / total), the remainder to CTA 0 (which has the
        // most groups: chunks fill in order); they sum to 512 and K_c <= g_c
        int Kc = (int)((int64_t)kTopK * groups_of(crank) / g_total);
        if (crank == 0) {
            int floors = 0;
#pragma unroll
            for (int c = 0; c < C; c++) floors += (int)((int64_t)kTopK * groups_of(c) / g_total);
            Kc += kTopK - floors;
        }
        if (Kc > 0) {
            int unused;
            radix_threshold_regs<NT, NS>(gm, [&](int j) { return ((gpres >> j) & 1u) != 0u; },
                                         Kc, gmin, kmx, sh, &Lc, &unused, true);
        }
    }
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");    // every CTA has started
    if ((int)threadIdx.x < C) {
        cl_st(cl_map(&mail.lc[crank], threadIdx.x), Lc);
        cl_st(cl_map(&mail.kmax[crank], threadIdx.x), kmx);
    }
    cl_sync();
    uint32_t L = 0xffffffffu, kmax_all = 0u;
#pragma unroll
    for (int c = 0; c < C; c++) {
        L = min(L, mail.lc[c]);
        kmax_all = max(kmax_all, mail.kmax[c]);
    }
    // this CTA's candidates (keys >= L): counts per slice, then index-order offsets
    uint32_t at[NS];
#pragma unroll
    for (int j = 0; j < NS; j++) {
        at[j] = 0;
#pragma unroll
        for (int e = 0; e < 4; e++)
            at[j] += (index_of(4 * j + e) < len && keys[4 * j + e] >= L) ? 1u : 0u;
    }
    const uint32_t n_c = ordered_starts<NT, NS>(at, sh);
    if ((int)threadIdx.x < C) cl_st(cl_map(&mail.cnt[crank], threadIdx.x), n_c);
    cl_sync();
    uint32_t n_cand = 0, off = 0;
#pragma unroll
    for (int c = 0; c < C; c++) {
        off += c < crank ? mail.cnt[c] : 0u;
        n_cand += mail.cnt[c];
    }
    const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    auto emit = [&](int pos, int s) {
        const int32_t page = pt_row[s / kC4Page];
        const int64_t slot = (int64_t)page * kC4Page + s % kC4Page;
        int32_t phys = (int32_t)slot;
        if (page < 0 || slot >= num_slots) {
            report(status, CSA_ERR_BOUNDS);
            phys = -1;
        }
        op[pos] = phys;
        if (orw) orw[pos] = s;
    };
    if (n_cand <= (uint32_t)kClCap) {            // uniform over the cluster
#pragma unroll
        for (int j = 0; j < NS; j++) {
            uint32_t a = off + at[j];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int kk = 4 * j + e;
                if (index_of(kk) < len && keys[kk] >= L) {
                    cl_st(cl_map(&cand_key[a], 0), keys[kk]);
                    cl_st(cl_map(&cand_idx[a], 0), (uint32_t)index_of(kk));
                    a++;
                }
            }
        }
        cl_sync();
        if (crank != 0) return;
        uint32_t T = 0;
        int need_eq = (int)n_cand;
        if (len > kTopK) radix_threshold<NT>(cand_key, (int)n_cand, K, L, kmax_all, sh, &T, &need_eq);
        ordered_compact<NT>(cand_key, (int)n_cand, T, need_eq, sh,
                            [&](int pos, int i, uint32_t) { emit(pos, cand_idx[i]); });
    } else {
        // heavy ties: CTA 0 selects from the whole row, staged in its buffer
        if (crank != 0) return;
        uint32_t *skeys = reinterpret_cast<uint32_t *>(cl_smem);
        stage_row_keys<NT>(skeys, row, len);
        __syncthreads();
        uint32_t T, km;
        select_top512<NT>(skeys, len, sh, status, &T, &km,
                          [&](int pos, int i, uint32_t) { emit(pos, i); });
    }
    for (int p = K + threadIdx.x; p < kTopK; p += NT) {
        op[p] = -1;
        if (orw) orw[p] = -1;
    }
}

// ------------------------------------------------------------------ bound-first selection
//
// For a few long rows (decode batches): three launches spread over every SM
// instead of one CTA per row.
//   A (grid chunks x rows): the row's keys fall into G groups of g = 2^s
//     consecutive keys (g the largest power of two with n/g >= 1024, so
//     1024 <= G <= 2048 once n >= 1024; g = 1 below); each CTA writes the
//     maxima of its chunk's groups.
//   B (same grid): every CTA takes L, the lower edge of the radix bin that
//     holds the K-th largest of the row's G group maxima (K = min(512, n);
//     L = 0 when n <= K).  K groups hold a key >= L, so L is at most the
//     row's K-th largest key: every key of the top K is >= L.  The CTA writes
//     its chunk's keys >= L, in index order, to the chunk's own region of the
//     row's candidate buffer and records how many there are.
//   C (one CTA per row): gathers the chunk segments in chunk order (so in
//     index order) into shared memory -- or, when they do not fit, into a
//     second buffer in the workspace -- and selects the top K among them as
//     the one-launch kernels do, with the page transform and -1 padding.
// Each kernel looks up its row (caller inputs only) before it waits on the
// preceding kernel.
constexpr int kTbThreads = 512;
constexpr int kTbChunk = 4096;         // keys per CTA in launches A and B
constexpr int kTbMaxGroups = 2048;
constexpr int kTbCap = 16384;          // candidates selected from shared memory in launch C
constexpr int kTbMaxRows = 64;         // with more rows the per-row launches fill the GPU
constexpr int kTbMinLen = 49152;       // shorter rows: one CTA per row (registers or shared memory)

// log2 of the group size for a row of n keys
__device__ __forceinline__ int tb_group_shift(int n) {
    return n < 2048 ? 0 : 31 - __clz(n / 1024);
}

__global__ void __launch_bounds__(kTbThreads)
topk_tb_groupmax_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens,
                        int bs, const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                        int pt_stride, uint32_t *gmax, int32_t *status, int ratio) {
    pdl_trigger();
    __shared__ TkShared sh;
    __shared__ uint32_t sgm[kTbChunk];
    const int t = blockIdx.y, c = blockIdx.x;
    const RowInfo ri = row_info<kTbThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride,
                                            status, c == 0, sh, ratio);
    const int n = ri.n_vis, lo = c * kTbChunk;
    if (lo >= n) {
        pdl_wait();
        return;
    }
    const int len = min(kTbChunk, n - lo);
    const int sh_g = tb_group_shift(n);
    const int ngr = (len + (1 << sh_g) - 1) >> sh_g;      // kTbChunk is a multiple of the group size
    for (int j = threadIdx.x; j < ngr; j += kTbThreads) sgm[j] = 0u;
    __syncthreads();
    pdl_wait();
    const float *row = logits + (int64_t)t * stride + lo;
    const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
    for (int base = 0; base < len; base += 4 * kTbThreads) {   // same trip count in every lane
        const int i = base + 4 * (int)threadIdx.x;
        uint32_t k[4];
        if (vec && i + 4 <= len) {
            const float4 x = *reinterpret_cast<const float4 *>(row + i);
            k[0] = order_key(x.x, status);
            k[1] = order_key(x.y, status);
            k[2] = order_key(x.z, status);
            k[3] = order_key(x.w, status);
        } else {
#pragma unroll
            for (int e = 0; e < 4; e++) k[e] = i + e < len ? order_key(row[i + e], status) : 0u;
        }
        if (sh_g >= 2) {
            // the four keys share a group (absent ones, 0, are the smallest
            // key); the g/4 lanes of one group combine first, aligned runs of
            // lanes holding consecutive keys, and one of them updates the slot
            uint32_t m = max(max(k[0], k[1]), max(k[2], k[3]));
            const int lanes = min(1 << (sh_g - 2), 32);
            for (int o = 1; o < lanes; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((threadIdx.x & (lanes - 1)) == 0 && i < len) atomicMax(&sgm[i >> sh_g], m);
        } else {
#pragma unroll
            for (int e = 0; e < 4; e++)
                if (i + e < len) atomicMax(&sgm[(i + e) >> sh_g], k[e]);
        }
    }
    __syncthreads();
    uint32_t *g = gmax + (int64_t)t * kTbMaxGroups + (lo >> sh_g);
    for (int j = threadIdx.x; j < ngr; j += kTbThreads) g[j] = sgm[j];
}

__global__ void __launch_bounds__(kTbThreads)
topk_tb_gather_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens,
                      int bs, const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                      int pt_stride, const uint32_t *gmax, uint32_t *counts, int mc,
                      uint32_t *cand_key, int32_t *cand_idx, int64_t cs, int32_t *status,
                      int ratio) {
    pdl_trigger();
    __shared__ TkShared sh;
    __shared__ __align__(16) uint32_t skeys[kTbChunk];
    __shared__ uint32_t sg[kTbMaxGroups];
    const int t = blockIdx.y, c = blockIdx.x;
    const RowInfo ri = row_info<kTbThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride,
                                            status, false, sh, ratio);
    pdl_wait();
    const int n = ri.n_vis, lo = c * kTbChunk;
    if (lo >= n) return;
    const int len = min(kTbChunk, n - lo);
    const int K = min(kTopK, n);
    uint32_t L = 0;
    if (n > K) {
        const int sh_g = tb_group_shift(n);
        const int G = (n + (1 << sh_g) - 1) >> sh_g;      // >= K (G = n below 2048 keys)
        uint32_t kmin = 0xffffffffu, kmax = 0u;
        for (int j = threadIdx.x; j < G; j += kTbThreads) {
            const uint32_t v = gmax[(int64_t)t * kTbMaxGroups + j];
            sg[j] = v;
            kmin = min(kmin, v);
            kmax = max(kmax, v);
        }
        block_minmax<kTbThreads>(kmin, kmax, sh);          // its barrier also publishes sg
        // one radix pass: the lower edge of the bin holding the K-th largest
        // maximum is below it, so still a bound of the row's K-th key
        int need_eq;
        radix_threshold<kTbThreads>(sg, G, K, kmin, kmax, sh, &L, &need_eq, true);
    }
    stage_row_keys<kTbThreads>(skeys, logits + (int64_t)t * stride + lo, len);
    __syncthreads();
    for (int i = threadIdx.x; i < len; i += kTbThreads)
        skeys[i] = order_key(__uint_as_float(skeys[i]), status);
    __syncthreads();
    uint32_t *ok = cand_key + (int64_t)t * cs + lo;
    int32_t *oi = cand_idx + (int64_t)t * cs + lo;
    const int kept = ordered_compact<kTbThreads>(skeys, len, L, len, sh, [&](int pos, int i, uint32_t k) {
        ok[pos] = k;
        oi[pos] = lo + i;
    });
    if (threadIdx.x == 0) counts[(int64_t)t * mc + c] = (uint32_t)kept;
}

__global__ void __launch_bounds__(kTkRowThreads, 1)
topk_tb_final_kernel(const int32_t *c4_lens, int bs, const int32_t *cu_q, const int32_t *q_pos,
                     int max_c4_len, const int32_t *page_table, int pt_stride, int64_t num_slots,
                     const uint32_t *counts, int mc, const uint32_t *cand_key,
                     const int32_t *cand_idx, uint32_t *ord_key, int32_t *ord_idx, int64_t cs,
                     int32_t *out_phys, int32_t *out_raw, int32_t *status, int ratio) {
    pdl_trigger();
    extern __shared__ __align__(16) uint8_t tbc_smem[];
    TkRowShared &sh = *reinterpret_cast<TkRowShared *>(tbc_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tbc_smem + kTkRowKeysOffset);
    int32_t *sidx = reinterpret_cast<int32_t *>(skeys + kTbCap);
    __shared__ uint32_t c_pre[kTkRowThreads];
    const int t = blockIdx.x;
    const RowInfo ri = row_info<kTkRowThreads>(t, cu_q, bs, q_pos, c4_lens, max_c4_len,
                                               pt_stride, status, false, sh, ratio);
    pdl_wait();
    const int n = ri.n_vis;
    const int K = min(kTopK, n);
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    if (n > 0) {
        const int nch = (n + kTbChunk - 1) / kTbChunk;     // <= kTkRowThreads (host check)
        const uint32_t cc = (int)threadIdx.x < nch ? counts[(int64_t)t * mc + threadIdx.x] : 0u;
        uint32_t m;
        const uint32_t pre = block_excl_scan<kTkRowThreads>(cc, &m, sh);
        if ((int)threadIdx.x < nch) c_pre[threadIdx.x] = pre;
        __syncthreads();
        const bool in_smem = m <= (uint32_t)kTbCap;
        uint32_t *dk = in_smem ? skeys : ord_key + (int64_t)t * cs;
        int32_t *di = in_smem ? sidx : ord_idx + (int64_t)t * cs;
        const uint32_t *sk = cand_key + (int64_t)t * cs;
        const int32_t *si = cand_idx + (int64_t)t * cs;
        // position p of the gathered list lies in the last chunk c with
        // c_pre[c] <= p (a binary search over the chunk table), so all loads
        // of a thread are independent
        for (uint32_t p = threadIdx.x; p < m; p += kTkRowThreads) {
            int lo_c = 0, hi_c = nch - 1;
            while (lo_c < hi_c) {
                const int mid = (lo_c + hi_c + 1) >> 1;
                if (c_pre[mid] <= p) lo_c = mid; else hi_c = mid - 1;
            }
            const uint32_t src = (uint32_t)lo_c * kTbChunk + (p - c_pre[lo_c]);
            dk[p] = sk[src];
            di[p] = si[src];
        }
        __syncthreads();
        uint32_t kmin = 0xffffffffu, kmax = 0u;
        for (uint32_t i = threadIdx.x; i < m; i += kTkRowThreads) {
            kmin = min(kmin, dk[i]);
            kmax = max(kmax, dk[i]);
        }
        block_minmax<kTkRowThreads>(kmin, kmax, sh);
        uint32_t T = 0;
        int need_eq = (int)m;
        if ((int)m > K) radix_threshold<kTkRowThreads>(dk, (int)m, K, kmin, kmax, sh, &T, &need_eq);
        const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
        ordered_compact<kTkRowThreads>(dk, (int)m, T, need_eq, sh, [&](int pos, int i, uint32_t) {
            const int32_t s = di[i];
            const int32_t page = pt_row[s / kC4Page];
            const int64_t slot = (int64_t)page * kC4Page + s % kC4Page;
            int32_t phys = (int32_t)slot;
            if (page < 0 || slot >= num_slots) {
                report(status, CSA_ERR_BOUNDS);
                phys = -1;
            }
            op[pos] = phys;
            if (orw) orw[pos] = s;
        });
    }
    for (int p = max(K, 0) + threadIdx.x; p < kTopK; p += kTkRowThreads) {
        op[p] = -1;
        if (orw) orw[p] = -1;
    }
}

// Workspace of the bound-first selection, per row: group maxima, one
// candidate count per chunk, the candidates by chunk region (keys, indices)
// and the gathered overflow copy.
struct TbLayout {
    int64_t cs;          // candidates per row (max_c4_len rounded up to 4)
    int mc;              // chunks per row
    size_t gmax, counts, ck, ci, ok2, oi2, bytes;
};

static size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

static TbLayout tb_layout(int num_q, int max_c4_len) {
    TbLayout l;
    l.cs = ((int64_t)max_c4_len + 3) & ~(int64_t)3;
    l.mc = (max_c4_len + kTbChunk - 1) / kTbChunk;
    const size_t q = (size_t)num_q;
    l.gmax = 0;
    l.counts = align16(l.gmax + q * kTbMaxGroups * 4);
    l.ck = align16(l.counts + q * l.mc * 4);
    l.ci = align16(l.ck + q * l.cs * 4);
    l.ok2 = align16(l.ci + q * l.cs * 4);
    l.oi2 = align16(l.ok2 + q * l.cs * 4);
    l.bytes = align16(l.oi2 + q * l.cs * 4);
    return l;
}

static size_t tb_bytes(int num_q, int max_c4_len) { return tb_layout(num_q, max_c4_len).bytes; }

static bool tb_applies(int num_q, int max_c4_len) {
    return num_q <= kTbMaxRows && max_c4_len > kTbMinLen &&
           max_c4_len <= kTkRowThreads * kTbChunk;
}

static cudaError_t launch_topk_bound_first(const TopkArgs &a, cudaStream_t s) {
    const TbLayout l = tb_layout(a.num_q, a.max_c4_len);
    uint8_t *w = (uint8_t *)a.workspace;
    uint32_t *gmax = (uint32_t *)(w + l.gmax);
    uint32_t *counts = (uint32_t *)(w + l.counts);
    uint32_t *ck = (uint32_t *)(w + l.ck);
    int32_t *ci = (int32_t *)(w + l.ci);
    uint32_t *ok2 = (uint32_t *)(w + l.ok2);
    int32_t *oi2 = (int32_t *)(w + l.oi2);
    dim3 g(l.mc, a.num_q);
    launch_k(topk_tb_groupmax_kernel, g, kTbThreads, 0, s, a.logits, a.logits_stride,
             a.c4_seq_lens, a.bs, a.cu_q, a.q_pos, a.max_c4_len, a.pt_stride, gmax, a.status,
             a.ratio);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    launch_k(topk_tb_gather_kernel, g, kTbThreads, 0, s, a.logits, a.logits_stride,
             a.c4_seq_lens, a.bs, a.cu_q, a.q_pos, a.max_c4_len, a.pt_stride,
             (const uint32_t *)gmax, counts, l.mc, ck, ci, l.cs, a.status, a.ratio);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = kTkRowKeysOffset + (size_t)kTbCap * 8;
    static int done[64] = {0};
    e = ensure_max_smem((const void *)topk_tb_final_kernel, (int)smem, done);
    if (e != cudaSuccess) return e;
    launch_k(topk_tb_final_kernel, a.num_q, kTkRowThreads, smem, s, a.c4_seq_lens, a.bs, a.cu_q,
             a.q_pos, a.max_c4_len, a.page_table, a.pt_stride, a.num_slots,
             (const uint32_t *)counts, l.mc, (const uint32_t *)ck, (const int32_t *)ci, ok2, oi2,
             l.cs, a.out_phys, a.out_raw, a.status, a.ratio);
    return cudaGetLastError();
}

// One cluster of C CTAs per query row (rows of at most kTkRegMax logits).
template <int C>
static cudaError_t launch_topk_cluster(const TopkArgs &a, cudaStream_t s) {
    static int done[64] = {0};
    cudaError_t e = ensure_max_smem((const void *)topk_cluster_kernel<C>, (int)kClSmem, done);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, a.num_q);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = kClSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<C>, a.logits, a.logits_stride, a.c4_seq_lens,
                           a.bs, a.cu_q, a.q_pos, a.max_c4_len, a.page_table, a.pt_stride,
                           a.num_slots, a.out_phys, a.out_raw, a.status, a.ratio);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

static int topk_max_chunks(int max_c4_len) {
    return max_c4_len <= 0 ? 1 : (max_c4_len + kTkChunk - 1) / kTkChunk;
}

// Workspace of the two-stage selection: candidate keys, candidate indices
// (num_q x chunks x 512 each), then one (512th key, largest key) pair per chunk.
static size_t two_stage_bytes(int num_q, int max_c4_len) {
    const size_t chunks = (size_t)num_q * topk_max_chunks(max_c4_len);
    return chunks * kTopK * 8 + chunks * sizeof(uint2);
}

// Which selection runs for these sizes: the bound-first launches for a few
// long rows (when their workspace fits `limit`); a cluster of 4 or 2 CTAs per
// row for up to one wave of such CTAs with rows of kClMinLen .. kTkRegMax
// keys; else one CTA per row for rows of at most kTkRowMax keys; else the
// two-stage merge.
enum TopkKind { kTopkCluster4, kTopkCluster2, kTopkReg, kTopkRow, kTopkBound, kTopkTwoStage };

static TopkKind topk_kind(int num_q, int max_c4_len, size_t limit) {
    if (tb_applies(num_q, max_c4_len) && tb_bytes(num_q, max_c4_len) <= limit) return kTopkBound;
    if (max_c4_len > kClMinLen && max_c4_len <= kTkRegMax) {
        if ((int64_t)num_q * 4 <= kClSms) return kTopkCluster4;
        if ((int64_t)num_q * 2 <= kClSms) return kTopkCluster2;
    }
    if (max_c4_len <= kTkRegMax) return kTopkReg;
    if (max_c4_len <= kTkRowMax) return kTopkRow;
    return kTopkTwoStage;
}

// Workspace that covers every path launch_topk512 may take for these sizes.
size_t topk_workspace_bytes(int num_q, int max_c4_len) {
    size_t b = two_stage_bytes(num_q, max_c4_len);
    if (topk_kind(num_q, max_c4_len, SIZE_MAX) == kTopkBound) {
        const size_t tb = tb_bytes(num_q, max_c4_len);
        if (tb > b) b = tb;
    }
    return b;
}

// Scratch the selection uses when it must fit CSA_TOPK_NOALLOC_MAX_BYTES:
// the bound-first buffers where they fit, none for rows of at most kTkRowMax
// logits otherwise (one launch), the two-stage candidate buffer for longer rows.
size_t topk_scratch_bytes(int num_q, int max_c4_len) {
    switch (topk_kind(num_q, max_c4_len, (size_t)CSA_TOPK_NOALLOC_MAX_BYTES)) {
    case kTopkBound: return tb_bytes(num_q, max_c4_len);
    case kTopkTwoStage: return two_stage_bytes(num_q, max_c4_len);
    default: return 0;
    }
}

static cudaError_t launch_topk512_limited(const TopkArgs &a, cudaStream_t s, size_t limit);

cudaError_t launch_topk512(const TopkArgs &a, cudaStream_t s) {
    return launch_topk512_limited(a, s, SIZE_MAX);
}

static cudaError_t launch_topk512_limited(const TopkArgs &a, cudaStream_t s, size_t limit) {
    if (a.num_q == 0) return cudaSuccess;
    const TopkKind kind = topk_kind(a.num_q, a.max_c4_len, limit);
    if (kind == kTopkBound) return launch_topk_bound_first(a, s);
    if (kind == kTopkCluster4) return launch_topk_cluster<4>(a, s);
    if (kind == kTopkCluster2) return launch_topk_cluster<2>(a, s);
    if (kind == kTopkReg) {
        launch_k(topk_reg_kernel, a.num_q, kTkRowThreads, 0, s, a.logits, a.logits_stride,
                 a.c4_seq_lens, a.bs, a.cu_q, a.q_pos, a.max_c4_len, a.page_table, a.pt_stride,
                 a.num_slots, a.out_phys, a.out_raw, a.status, a.ratio);
        return cudaGetLastError();
    }
    if (kind == kTopkRow) {
        const size_t smem = kTkRowKeysOffset + (size_t)((a.max_c4_len + 3) & ~3) * 4;
        static int done_row[64] = {0};
        cudaError_t e = ensure_max_smem((const void *)topk_row_kernel,
                                        (int)(kTkRowKeysOffset + (size_t)kTkRowMax * 4), done_row);
        if (e != cudaSuccess) return e;
        launch_k(topk_row_kernel, a.num_q, kTkRowThreads, smem, s, a.logits, a.logits_stride,
                 a.c4_seq_lens, a.bs, a.cu_q, a.q_pos, a.max_c4_len, a.page_table, a.pt_stride,
                 a.num_slots, a.out_phys, a.out_raw, a.status, a.ratio);
        return cudaGetLastError();
    }
    const int mc = topk_max_chunks(a.max_c4_len);
    uint32_t *ck = (uint32_t *)a.workspace;
    int32_t *ci = (int32_t *)((uint8_t *)a.workspace + (size_t)a.num_q * mc * kTopK * 4);
    uint2 *info = (uint2 *)((uint8_t *)a.workspace + (size_t)a.num_q * mc * kTopK * 8);
    const size_t smem1 = kTkKeysOffset + kTkChunk * sizeof(uint32_t);
    static int done[64] = {0};
    cudaError_t e0 = ensure_max_smem((const void *)topk_stage1_kernel, (int)smem1, done);
    if (e0 != cudaSuccess) return e0;
    dim3 g1(mc, a.num_q);
    launch_k(topk_stage1_kernel, g1, kTkThreads, smem1, s, a.logits, a.logits_stride, a.c4_seq_lens, a.bs,
                                                 a.cu_q, a.q_pos, a.max_c4_len, a.pt_stride, mc,
                                                 ck, ci, info, a.status, a.ratio);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_topk_stage2(a, mc, kTkChunk, ck, ci, info, s);
}

cudaError_t launch_topk_stage2(const TopkArgs &a, int max_chunks, int chunk_len,
                               const uint32_t *cand_key, const int32_t *cand_idx,
                               const uint2 *chunk_info, cudaStream_t s) {
    const size_t smem2 = kTkKeysOffset + kTk2Smem * (sizeof(uint32_t) + sizeof(int32_t));
    static int done2[64] = {0};
    cudaError_t e = ensure_max_smem((const void *)topk_stage2_kernel, (int)smem2, done2);
    if (e != cudaSuccess) return e;
    launch_k(topk_stage2_kernel, a.num_q, kTkThreads, smem2, s, a.c4_seq_lens, a.bs, a.cu_q,
             a.q_pos, a.max_c4_len, a.page_table, a.pt_stride, a.num_slots, max_chunks, chunk_len,
             cand_key, cand_idx, chunk_info, a.out_phys, a.out_raw, a.status, a.ratio);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ no-allocation variant
//
// For callers that cannot provide a workspace: the candidates live in this
// file-scope device array (held by every GPU that loads the library until the
// process exits).  Host code may not use the array's name as a device
// address, so its address is looked up once per device with that device
// current and cached (an atomic per device: host threads may make the first
// call concurrently; they store the same value).  The cached address belongs
// to the device's context at that time and is not refreshed after a device
// reset.  Nothing in the array needs to start at zero: stage 1 writes every
// entry stage 2 reads.  Concurrent calls share it and race.
static __device__ __align__(256) uint8_t g_topk_scratch[CSA_TOPK_NOALLOC_MAX_BYTES];

cudaError_t launch_topk512_noalloc(const TopkArgs &a, cudaStream_t s) {
    static std::atomic<void *> scratch_addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    void *ptr = scratch_addr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        e = cudaGetSymbolAddress(&ptr, g_topk_scratch);
        if (e != cudaSuccess) return e;
        scratch_addr[dev].store(ptr, std::memory_order_release);
    }
    TopkArgs b = a;
    b.workspace = ptr;
    return launch_topk512_limited(b, s, (size_t)CSA_TOPK_NOALLOC_MAX_BYTES);
}

}  // namespace csa
