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

// Block-wide min and max of one value pair per thread (uses sh.warp_a/b).
__device__ __forceinline__ void block_minmax(uint32_t &lo, uint32_t &hi, TkShared &sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
        sh.warp_a[warp] = lo;
        sh.warp_b[warp] = hi;
    }
    __syncthreads();
    lo = 0xffffffffu;
    hi = 0u;
#pragma unroll
    for (int w = 0; w < kTkWarps; w++) {
        lo = min(lo, sh.warp_a[w]);
        hi = max(hi, sh.warp_b[w]);
    }
    __syncthreads();
}

// Finds the K-th largest key T among the keys[0..n) that are >= kmin (K <= their
// count; kmax is their maximum) and how many keys equal to T belong to the top K
// (need_eq >= 1).  The radix digits are taken from d = key - kmin, 12 bits at a
// time from the highest set bit of kmax - kmin down, so that keys sharing sign
// and exponent (the usual case for one row of logits) already spread over the
// bins of the first pass; two passes resolve a range of up to 24 bits.  keys may
// point to shared or global memory.
__device__ void radix_threshold(const uint32_t *keys, int n, int K, uint32_t kmin, uint32_t kmax,
                                TkShared &sh, uint32_t *T_out, int *need_eq_out) {
    const uint32_t range = kmax - kmin;
    const int B = range == 0 ? 0 : 32 - __clz(range);
    uint32_t prefix = 0;            // resolved high bits of d
    int remaining = K;
#pragma unroll 1
    for (int done = 0; done < B;) {
        const int width = min(12, B - done);
        const int shift = B - done - width;
        const int hi = shift + width;            // bits at and above hi are resolved
        const uint32_t nb = 1u << width;
        for (uint32_t i = threadIdx.x; i < nb; i += kTkThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kTkThreads) {
            const uint32_t k = keys[i];
            const uint32_t d = k - kmin;
            const bool match = k >= kmin && (hi >= 32 || ((d ^ prefix) >> hi) == 0);
            if (match) atomicAdd(&sh.hist[(d >> shift) & (nb - 1)], 1u);
        }
        __syncthreads();
        // Suffix scan from the top bin: thread i owns bins nb-1-per*i .. nb-per*(i+1).
        const int per = nb > (uint32_t)kTkThreads ? (int)nb / kTkThreads : 1;   // 1..8
        uint32_t c[8];
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int bin = (int)nb - 1 - ((int)threadIdx.x * per + j);
            c[j] = (j < per && bin >= 0) ? sh.hist[bin] : 0u;
            mine += c[j];
        }
        uint32_t total;
        const uint32_t excl = block_excl_scan(mine, &total, sh);
        if (excl < (uint32_t)remaining && (uint32_t)remaining <= excl + mine) {
            uint32_t acc = excl;
            bool found = false;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                if (!found && j < per && acc + c[j] >= (uint32_t)remaining) {
                    found = true;
                    sh.digit = nb - 1 - (threadIdx.x * per + j);
                    sh.above = acc;
                }
                acc += c[j];
            }
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        remaining -= (int)sh.above;
        done += width;
        __syncthreads();
    }
    *T_out = kmin + prefix;
    *need_eq_out = remaining;
}

// Walks keys[0..n) in index order and calls emit(pos, i, key) for the
// selected ones: key > T, or key == T among the first need_eq such keys.
// Returns how many were selected.
// Each warp owns one contiguous segment: it counts its segment with ballots,
// one block barrier publishes the per-warp counts, then every warp writes its
// selected elements at their global ranks.
template <typename Emit>
__device__ int ordered_compact(const uint32_t *keys, int n, uint32_t T, int need_eq,
                               TkShared &sh, Emit emit) {
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
    uint32_t eq_before = 0, gt_before = 0, eq_all = 0, gt_all = 0;
    for (int w = 0; w < kTkWarps; w++) {
        eq_before += w < warp ? sh.warp_a[w] : 0u;
        gt_before += w < warp ? sh.warp_b[w] : 0u;
        eq_all += sh.warp_a[w];
        gt_all += sh.warp_b[w];
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
    return (int)(gt_all + min(eq_all, (uint32_t)need_eq));
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

// Stage 1: one CTA per (query row, 8192-logit chunk).  Writes the chunk's
// top-512 (or all of it when shorter) in index order, plus the chunk's
// 512th-largest key (0 when it holds fewer) and its largest key.
__global__ void __launch_bounds__(kTkThreads)
topk_stage1_kernel(const float *__restrict__ logits, int64_t stride, const int32_t *c4_lens,
                   int bs, const int32_t *cu_q, const int32_t *q_pos, int max_c4_len,
                   int pt_stride, int max_chunks, uint32_t *cand_key, int32_t *cand_idx,
                   uint2 *chunk_info, int32_t *status) {
    pdl_begin();
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
    uint32_t kmax = 0u;
    bool has = false;
    auto put = [&](int i, float f) {
        const uint32_t k = order_key(f, status);
        skeys[i] = k;
        kmax = max(kmax, k);
        has = true;
    };
    if ((reinterpret_cast<uintptr_t>(row) & 15) == 0) {
        const int n4 = len / 4;
        for (int i = threadIdx.x; i < n4; i += kTkThreads) {
            const float4 v = reinterpret_cast<const float4 *>(row)[i];
            put(4 * i, v.x);
            put(4 * i + 1, v.y);
            put(4 * i + 2, v.z);
            put(4 * i + 3, v.w);
        }
        for (int i = 4 * n4 + threadIdx.x; i < len; i += kTkThreads) put(i, row[i]);
    } else {
        for (int i = threadIdx.x; i < len; i += kTkThreads) put(i, row[i]);
    }
    // The keys each thread loaded form one group.  When all 512 groups are
    // non-empty the smallest group maximum is a lower bound of the 512th-largest
    // key (the 512 group maxima are distinct keys >= it); otherwise the bound
    // is 0.
    uint32_t lbound = has ? kmax : 0u;
    block_minmax(lbound, kmax, sh);     // its barrier also publishes skeys
    const int K = min(kTopK, len);
    uint32_t T = 0;
    int need_eq = len;
    if (len > kTopK) radix_threshold(skeys, len, K, lbound, kmax, sh, &T, &need_eq);
    if (threadIdx.x == 0)
        chunk_info[(int64_t)t * max_chunks + c] = make_uint2(len > kTopK ? T : 0u, kmax);
    uint32_t *ok = cand_key + ((int64_t)t * max_chunks + c) * kTopK;
    int32_t *oi = cand_idx + ((int64_t)t * max_chunks + c) * kTopK;
    ordered_compact(skeys, len, T, need_eq, sh, [&](int pos, int i, uint32_t k) {
        ok[pos] = k;
        oi[pos] = lo + i;
    });
}

// Stage 2: one CTA per query row.  The row's top-512 are all >= L, the largest
// of the chunks' 512th keys (that chunk alone holds 512 keys >= L), so the
// candidates below L are dropped first (in index order, into shared memory),
// the threshold is found among the survivors, and the selection is written in
// ascending index order, mapped through the page table, then padded with -1.
// Rows with more than 16384 candidates select straight from the workspace.
__global__ void __launch_bounds__(kTkThreads)
topk_stage2_kernel(const int32_t *c4_lens, int bs, const int32_t *cu_q, const int32_t *q_pos,
                   int max_c4_len, const int32_t *page_table, int pt_stride, int64_t num_slots,
                   int max_chunks, const uint32_t *cand_key, const int32_t *cand_idx,
                   const uint2 *chunk_info, int32_t *out_phys, int32_t *out_raw,
                   int32_t *status) {
    pdl_begin();
    extern __shared__ __align__(16) uint8_t tk2_smem[];
    TkShared &sh = *reinterpret_cast<TkShared *>(tk2_smem);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(tk2_smem + kTkKeysOffset);
    int32_t *sidx = reinterpret_cast<int32_t *>(skeys + kTk2Smem);
    const int t = blockIdx.x;
    const RowInfo ri = row_info(t, cu_q, bs, q_pos, c4_lens, max_c4_len, pt_stride, status,
                                false, sh);
    const int n = ri.n_vis;
    int total = 0, nch = 0;
    if (n > 0) {
        nch = (n + kTkChunk - 1) / kTkChunk;
        total = (nch - 1) * kTopK + min(kTopK, n - (nch - 1) * kTkChunk);
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
        uint32_t lneg = ~L;
        block_minmax(lneg, kmax, sh);     // min of ~L is ~(max of L)
        L = ~lneg;
        if (total <= kTk2Smem) {
            // Thread i holds candidates [32i, 32i+32): all loads in flight at
            // once, then the survivors (keys >= L) are compacted in order into
            // shared memory with one block scan.
            constexpr int kPer = kTk2Smem / kTkThreads;    // 32
            static_assert(kPer % 4 == 0, "16-byte loads");
            const int i0 = threadIdx.x * kPer;
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
            uint32_t pos = block_excl_scan(mine, &surv, sh);
#pragma unroll
            for (int j = 0; j < kPer; j++) {
                if (i0 + j < total && kk[j] >= L) {
                    skeys[pos] = kk[j];
                    sidx[pos] = ii[j];
                    pos++;
                }
            }
            __syncthreads();
            keys = skeys;
            idx = sidx;
            m = (int)surv;
        }
        radix_threshold(keys, m, K, L, kmax, sh, &T, &need_eq);
    }
    const int32_t *pt_row = page_table + (int64_t)ri.b * pt_stride;
    int32_t *op = out_phys + (int64_t)t * kTopK;
    int32_t *orw = out_raw ? out_raw + (int64_t)t * kTopK : nullptr;
    ordered_compact(keys, m, T, need_eq, sh, [&](int pos, int i, uint32_t) {
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

// Workspace: candidate keys, candidate indices (num_q x chunks x 512 each),
// then one (512th key, largest key) pair per chunk.
size_t topk_workspace_bytes(int num_q, int max_c4_len) {
    const size_t chunks = (size_t)num_q * topk_max_chunks(max_c4_len);
    return chunks * kTopK * 8 + chunks * sizeof(uint2);
}

cudaError_t launch_topk512(const TopkArgs &a, cudaStream_t s) {
    if (a.num_q == 0) return cudaSuccess;
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
                                                 ck, ci, info, a.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem2 = kTkKeysOffset + kTk2Smem * (sizeof(uint32_t) + sizeof(int32_t));
    static int done2[64] = {0};
    e = ensure_max_smem((const void *)topk_stage2_kernel, (int)smem2, done2);
    if (e != cudaSuccess) return e;
    launch_k(topk_stage2_kernel, a.num_q, kTkThreads, smem2, s, a.c4_seq_lens, a.bs, a.cu_q, a.q_pos,
                                                      a.max_c4_len, a.page_table, a.pt_stride,
                                                      a.num_slots, mc, ck, ci, info,
                                                      a.out_phys, a.out_raw, a.status);
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
