// topk.cu -- step 3, the fixed-k top-512 with the paged index transform
// ("Token 的一生：DSV4 架构与 DSpark" §3.2 topk_transform_512, page arithmetic
// of §2.2).
//
// Selection is exact on order-preserving 32-bit keys of the float logits
// (-0 folded onto +0, NaN recorded and ordered below -inf).  The order is
// (logit descending, logical index ascending); outputs are listed in
// ascending logical index and padded with -1.
//
// Two launches, no inter-CTA waits:
//   stage 1: each CTA takes a chunk of 8192 logits of one query row into
//            shared memory, finds the chunk's 512th key by a 3-pass radix
//            select (12/12/8-bit digits, shared-memory histograms, block
//            suffix scan), and writes the chunk's top-512 (key, index) pairs
//            in index order to the workspace.
//   stage 2: one CTA per query row repeats the select over the row's
//            concatenated candidates (every element of the global top-512 is
//            in its chunk's top-512 under the same total order) and writes
//            physical slots page_table[s/64]*64 + s%64 and raw indices.
#include "common.cuh"
#include "launch.h"

namespace csa {

constexpr int kTkThreads = 512;
constexpr int kTkChunk = 8192;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kHistBins = 4096;
constexpr int kTk2Smem = 16384;      // stage-2 candidates staged in shared memory

__device__ __forceinline__ uint32_t order_key(float f, int32_t *status) {
    uint32_t u = __float_as_uint(f);
    if (f != f) {  // NaN
        report(status, CSA_ERR_NAN);
        return 0u;
    }
    if (f == 0.0f) u = 0u;                        // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TkShared {
    uint32_t hist[kHistBins];
    uint32_t warp_a[kTkWarps];
    uint32_t warp_b[kTkWarps];
    uint32_t digit, above;
    int32_t row_b, row_nvis;
};
// the key buffers that follow TkShared in dynamic shared memory start on a
// 16-byte boundary (they are read and written with 16-byte vectors)
constexpr size_t kTkKeysOffset = (sizeof(TkShared) + 15) & ~(size_t)15;

// Exclusive scan of one value per thread over the block; returns the prefix
// and writes the block total to *total.  Uses sh.warp_a.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *total, TkShared &sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) sh.warp_a[warp] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kTkWarps; w++) {
        const uint32_t x = sh.warp_a[w];
        before += (w < warp) ? x : 0u;
        tot += x;
    }
    __syncthreads();
    *total = tot;
    return before + incl - v;
}

// Finds the K-th largest key T among keys[0..n) (K <= n) and how many keys
// equal to T belong to the top K (need_eq >= 1).  keys may point to shared
// or global memory.
__device__ void radix_threshold(const uint32_t *keys, int n, int K, TkShared &sh,
                                uint32_t *T_out, int *need_eq_out) {
    const int shifts[3] = {20, 8, 0};
    const int widths[3] = {12, 12, 8};
    uint32_t prefix = 0;
    int remaining = K;
#pragma unroll 1
    for (int p = 0; p < 3; p++) {
        const int shift = shifts[p], bits = widths[p];
        const uint32_t nb = 1u << bits;
        const uint64_t hi_mask64 = ~((1ull << (shift + bits)) - 1ull);
        const uint32_t hi_mask = (uint32_t)hi_mask64;
        for (uint32_t i = threadIdx.x; i < nb; i += kTkThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kTkThreads) {
            const uint32_t k = keys[i];
            if ((k & hi_mask) == (prefix & hi_mask))
                atomicAdd(&sh.hist[(k >> shift) & (nb - 1)], 1u);
        }
        __syncthreads();
        // Suffix scan from the top bin: thread i owns bins nb-1-8i .. nb-8-8i.
        const int per = (int)nb / kTkThreads;  // 8 (4096 bins) or 0 (256 bins)
        uint32_t mine = 0;
        uint32_t c[8];
        if (per == 8) {
#pragma unroll
            for (int j = 0; j < 8; j++) {
                c[j] = sh.hist[nb - 1 - (threadIdx.x * 8 + j)];
                mine += c[j];
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; j++) c[j] = 0;
            if (threadIdx.x < nb) c[0] = sh.hist[nb - 1 - threadIdx.x];
            mine = c[0];
        }
        uint32_t total;
        const uint32_t excl = block_excl_scan(mine, &total, sh);
        if (excl < (uint32_t)remaining && (uint32_t)remaining <= excl + mine) {
            uint32_t acc = excl;
            const int cnt = per == 8 ? 8 : 1;
            for (int j = 0; j < cnt; j++) {
                if (acc + c[j] >= (uint32_t)remaining) {
                    sh.digit = per == 8 ? nb - 1 - (threadIdx.x * 8 + j) : nb - 1 - threadIdx.x;
                    sh.above = acc;
                    break;
                }
                acc += c[j];
            }
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        remaining -= (int)sh.above;
        __syncthreads();
    }
    *T_out = prefix;
    *need_eq_out = remaining;
}

// Walks keys[0..n) in index order and calls emit(pos, i, key) for the
// selected ones: key > T, or key == T among the first need_eq such keys.
// Each warp owns one contiguous segment: it counts its segment with ballots,
// one block barrier publishes the per-warp counts, then every warp writes its
// selected elements at their global ranks.
template <typename Emit>
__device__ void ordered_compact(const uint32_t *keys, int n, uint32_t T, int need_eq, int K,
                                TkShared &sh, Emit emit) {
    (void)K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int seg = ((n + kTkWarps - 1) / kTkWarps + 31) & ~31;
    const int beg = min(n, warp * seg), end = min(n, beg + seg);
    uint32_t gt_w = 0, eq_w = 0;
    for (int i = beg + lane; i < end + lane; i += 32) {   // uniform trip count per warp
        const uint32_t k = i < end ? keys[i] : 0u;
        gt_w += __popc(__ballot_sync(0xffffffffu, i < end && k > T));
        eq_w += __popc(__ballot_sync(0xffffffffu, i < end && k == T));
    }
    if (lane == 0) {
        sh.warp_a[warp] = eq_w;
        sh.warp_b[warp] = gt_w;
    }
    __syncthreads();
    uint32_t eq_before = 0, gt_before = 0;
    for (int w = 0; w < warp; w++) {
        eq_before += sh.warp_a[w];
        gt_before += sh.warp_b[w];
    }
    __syncthreads();    // the counts may be reused by the caller's next phase
    uint32_t eq_seen = eq_before;
    uint32_t out = gt_before + min(eq_before, (uint32_t)need_eq);
    for (int i = beg + lane; i < end + lane; i += 32) {
        const uint32_t k = i < end ? keys[i] : 0u;
        const bool gt = i < end && k > T;
        const bool eq = i < end && k == T;
        const uint32_t beq = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(beq & lt) < (uint32_t)need_eq);
        const uint32_t btk = __ballot_sync(0xffffffffu, take);
        if (take) emit((int)(out + __popc(btk & lt)), i, k);
        eq_seen += __popc(beq);
        out += __popc(btk);
    }
}

struct RowInfo {
    int b, n_vis;
};

// Request and visible length of query row t, found by warp 0 with coalesced
// reads of cu_q and c4_lens (one round trip for up to 32 requests) and
// published to the block through shared memory.
__device__ RowInfo row_info(int t, const int32_t *cu_q, int bs, const int32_t *q_pos,
                            const int32_t *c4_lens, int max_c4_len, int pt_stride,
                            int32_t *status, bool leader, TkShared &sh) {
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
            if (q_pos) n = min(n, (pos + 1) / 4);
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

__global__ void __launch_bounds__(kTkThreads)
topk_stage1_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens,
                   int bs, const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                   int pt_stride, int max_chunks, uint32_t *cand_key, int32_t *cand_idx,
                   int32_t *status) {
    extern __shared__ __align__(16) uint8_t tk_smem[];
    TkShared &sh = *reinterpret_cast<TkShared *>(tk_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tk_smem + kTkKeysOffset);
    const int t = blockIdx.y, c = blockIdx.x;
    const RowInfo ri = row_info(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride, status,
                                c == 0, sh);
    const int lo = c * kTkChunk;
    if (lo >= ri.n_vis) return;
    const int len = min(kTkChunk, ri.n_vis - lo);
    const float *row = logits + (int64_t)t * stride + lo;
    if ((reinterpret_cast<uintptr_t>(row) & 15) == 0) {
        const int n4 = len / 4;
        for (int i = threadIdx.x; i < n4; i += kTkThreads) {
            const float4 v = reinterpret_cast<const float4 *>(row)[i];
            skeys[4 * i] = order_key(v.x, status);
            skeys[4 * i + 1] = order_key(v.y, status);
            skeys[4 * i + 2] = order_key(v.z, status);
            skeys[4 * i + 3] = order_key(v.w, status);
        }
        for (int i = 4 * n4 + threadIdx.x; i < len; i += kTkThreads) skeys[i] = order_key(row[i], status);
    } else {
        for (int i = threadIdx.x; i < len; i += kTkThreads) skeys[i] = order_key(row[i], status);
    }
    __syncthreads();
    const int K = min(kTopK, len);
    uint32_t T = 0;
    int need_eq = len;
    if (len > kTopK) radix_threshold(skeys, len, K, sh, &T, &need_eq);
    uint32_t *ok = cand_key + ((int64_t)t * max_chunks + c) * kTopK;
    int32_t *oi = cand_idx + ((int64_t)t * max_chunks + c) * kTopK;
    ordered_compact(skeys, len, T, need_eq, K, sh, [&](int pos, int i, uint32_t k) {
        ok[pos] = k;
        oi[pos] = lo + i;
    });
}

__global__ void __launch_bounds__(kTkThreads)
topk_stage2_kernel(const int32_t *c4_lens, int bs, const int32_t *cu_q, const int32_t *q_pos,
                   int max_c4_len, const int32_t *page_table, int pt_stride, int64_t num_slots,
                   int max_chunks, const uint32_t *cand_key, const int32_t *cand_idx,
                   int32_t *out_phys, int32_t *out_raw, int32_t *status) {
    extern __shared__ __align__(16) uint8_t tk2_smem[];
    TkShared &sh = *reinterpret_cast<TkShared *>(tk2_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tk2_smem + kTkKeysOffset);
    const int t = blockIdx.x;
    const RowInfo ri = row_info(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride, status,
                                false, sh);
    const int n = ri.n_vis;
    int total = 0;
    if (n > 0) {
        const int nch = (n + kTkChunk - 1) / kTkChunk;
        total = (nch - 1) * kTopK + min(kTopK, n - (nch - 1) * kTkChunk);
    }
    const int K = min(kTopK, total);
    const uint32_t *gkeys = cand_key + (int64_t)t * max_chunks * kTopK;
    const int32_t *idx = cand_idx + (int64_t)t * max_chunks * kTopK;
    // candidates (keys and indices) up to kTk2Smem keys are staged in shared memory; longer rows
    // are selected straight from the workspace (L2)
    const uint32_t *keys = gkeys;
    int32_t *sidx = reinterpret_cast<int32_t *>(skeys + kTk2Smem);
    if (total <= kTk2Smem) {
        for (int i = threadIdx.x * 4; i < total; i += kTkThreads * 4) {
            if (i + 4 <= total) {
                *reinterpret_cast<uint4 *>(skeys + i) = *reinterpret_cast<const uint4 *>(gkeys + i);
                *reinterpret_cast<int4 *>(sidx + i) = *reinterpret_cast<const int4 *>(idx + i);
            } else {
                for (int j = i; j < total; j++) {
                    skeys[j] = gkeys[j];
                    sidx[j] = idx[j];
                }
            }
        }
        __syncthreads();
        keys = skeys;
        idx = sidx;
    }
    const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
    uint32_t T = 0;
    int need_eq = total;
    if (total > kTopK) radix_threshold(keys, total, K, sh, &T, &need_eq);
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    ordered_compact(keys, total, T, need_eq, K, sh, [&](int pos, int i, uint32_t) {
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

static int topk_max_chunks(int max_c4_len) {
    return max_c4_len <= 0 ? 1 : (max_c4_len + kTkChunk - 1) / kTkChunk;
}

size_t topk_workspace_bytes(int num_q, int max_c4_len) {
    return (size_t)num_q * topk_max_chunks(max_c4_len) * kTopK * 8;
}

cudaError_t launch_topk512(const TopkArgs &a, cudaStream_t s) {
    if (a.num_q == 0) return cudaSuccess;
    const int mc = topk_max_chunks(a.max_c4_len);
    uint32_t *ck = (uint32_t *)a.workspace;
    int32_t *ci = (int32_t *)((uint8_t *)a.workspace + (size_t)a.num_q * mc * kTopK * 4);
    const size_t smem1 = kTkKeysOffset + kTkChunk * sizeof(uint32_t);
    static int done[64] = {0};
    cudaError_t e0 = ensure_max_smem((const void *)topk_stage1_kernel, (int)smem1, done);
    if (e0 != cudaSuccess) return e0;
    dim3 g1(mc, a.num_q);
    topk_stage1_kernel<<<g1, kTkThreads, smem1, s>>>(a.logits, a.logits_stride, a.c4_seq_lens, a.bs,
                                                 a.cu_q, a.q_pos, a.max_c4_len, a.pt_stride, mc,
                                                 ck, ci, a.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem2 = kTkKeysOffset + kTk2Smem * (sizeof(uint32_t) + sizeof(int32_t));
    static int done2[64] = {0};
    e = ensure_max_smem((const void *)topk_stage2_kernel, (int)smem2, done2);
    if (e != cudaSuccess) return e;
    topk_stage2_kernel<<<a.num_q, kTkThreads, smem2, s>>>(a.c4_seq_lens, a.bs, a.cu_q, a.q_pos,
                                                      a.max_c4_len, a.page_table, a.pt_stride,
                                                      a.num_slots, mc, ck, ci, a.out_phys,
                                                      a.out_raw, a.status);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ no-allocation variant
//
// For callers that cannot provide a workspace: the candidates live in this
// file-scope device array (held by every GPU that loads the library until the
// process exits).  Host code may not use the array's name as a device
// address, so its address is looked up once per device with that device
// current and cached.  Nothing in the array needs to start at zero: stage 1
// writes every entry stage 2 reads.  Concurrent calls share it and race.
static __device__ __align__(256) uint8_t g_topk_scratch[CSA_TOPK_NOALLOC_MAX_BYTES];

cudaError_t launch_topk512_noalloc(const TopkArgs &a, cudaStream_t s) {
    static void *scratch_addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_topk_scratch);
        if (e != cudaSuccess) return e;
        scratch_addr[dev] = ptr;
    }
    TopkArgs b = a;
    b.workspace = scratch_addr[dev];
    return launch_topk512(b, s);
}

}  // namespace csa
