// topk.cuh -- block-level pieces of the fixed-k top-512 selection ("Token 的一生：
// DSV4 架构与 DSpark" §3.2 topk_transform_512), shared by the two-launch top-k
// (topk.cu) and the indexer kernel that selects its own chunk (indexer_tc.cu).
//
// Keys are order-preserving 32-bit images of the float logits (-0 folded onto
// +0, NaN recorded and ordered below -inf); the order is (key descending,
// index ascending).  NT is the block's thread count (a multiple of 32).
#pragma once

#include "common.cuh"

namespace csa {

constexpr int kHistBins = 4096;

__device__ __forceinline__ uint32_t order_key(float f, int32_t *status) {
    uint32_t u = __float_as_uint(f);
    if (f != f) {  // NaN
        report(status, CSA_ERR_NAN);
        return 0u;
    }
    if (f == 0.0f) u = 0u;                        // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
struct TkSharedT {
    uint32_t hist[kHistBins];
    uint32_t warp_a[NT / 32];
    uint32_t warp_b[NT / 32];
    uint32_t digit, above;
    int32_t row_b, row_nvis;
};

// Exclusive scan of one value per thread over the block; returns the prefix
// and writes the block total to *total.  Uses sh.warp_a.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *total,
                                                    TkSharedT<NT> &sh) {
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
    for (int w = 0; w < NT / 32; w++) {
        const uint32_t x = sh.warp_a[w];
        before += (w < warp) ? x : 0u;
        tot += x;
    }
    __syncthreads();
    *total = tot;
    return before + incl - v;
}

// Block-wide min and max of one value pair per thread (uses sh.warp_a/b).
template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t &lo, uint32_t &hi, TkSharedT<NT> &sh) {
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
    for (int w = 0; w < NT / 32; w++) {
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
template <int NT>
__device__ void radix_threshold(const uint32_t *keys, int n, int K, uint32_t kmin, uint32_t kmax,
                                TkSharedT<NT> &sh, uint32_t *T_out, int *need_eq_out) {
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
        for (uint32_t i = threadIdx.x; i < nb; i += NT) sh.hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += NT) {
            const uint32_t k = keys[i];
            const uint32_t d = k - kmin;
            const bool match = k >= kmin && (hi >= 32 || ((d ^ prefix) >> hi) == 0);
            if (match) atomicAdd(&sh.hist[(d >> shift) & (nb - 1)], 1u);
        }
        __syncthreads();
        // Suffix scan from the top bin: thread i owns bins nb-1-per*i .. nb-per*(i+1).
        const int per = (int)((nb + NT - 1) / NT);     // 1..13 for NT >= 320
        constexpr int kMaxPer = (kHistBins + NT - 1) / NT;
        uint32_t c[kMaxPer];
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < kMaxPer; j++) {
            const int bin = (int)nb - 1 - ((int)threadIdx.x * per + j);
            c[j] = (j < per && bin >= 0) ? sh.hist[bin] : 0u;
            mine += c[j];
        }
        uint32_t total;
        const uint32_t excl = block_excl_scan<NT>(mine, &total, sh);
        if (excl < (uint32_t)remaining && (uint32_t)remaining <= excl + mine) {
            uint32_t acc = excl;
            bool found = false;
#pragma unroll
            for (int j = 0; j < kMaxPer; j++) {
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
// Each warp owns one contiguous segment: it counts its segment with ballots,
// one block barrier publishes the per-warp counts, then every warp writes its
// selected elements at their global ranks.  Returns how many were selected.
template <int NT, typename Emit>
__device__ int ordered_compact(const uint32_t *keys, int n, uint32_t T, int need_eq,
                               TkSharedT<NT> &sh, Emit emit) {
    constexpr int kWarps = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int seg = ((n + kWarps - 1) / kWarps + 31) & ~31;
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
    for (int w = 0; w < kWarps; w++) {
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

// One chunk of a row: skeys[0..len) hold the float bits of the chunk's logits
// (index base + i).  Converts them to keys in place, then writes the chunk's
// top-512 (or all of it when shorter) in index order to ok/oi and the chunk's
// (512th-largest key or 0 when it holds fewer, largest key) to *info.
//
// Lower bound: thread t's keys i = t + j*NT fall into G = ceil(512/NT) groups by
// j % G.  When all NT*G groups are non-empty the smallest group maximum is at
// most the 512th-largest key (the NT*G >= 512 group maxima are distinct keys
// not below it), so the radix digits start from that bound; otherwise the
// bound is 0.
template <int NT>
__device__ void select_chunk(uint32_t *skeys, int len, int base, uint32_t *ok, int32_t *oi,
                             uint2 *info, TkSharedT<NT> &sh, int32_t *status) {
    constexpr int G = (kTopK + NT - 1) / NT;
    uint32_t gmax[G];
#pragma unroll
    for (int g = 0; g < G; g++) gmax[g] = 0u;
    bool has[G];
#pragma unroll
    for (int g = 0; g < G; g++) has[g] = false;
    uint32_t kmax = 0u;
    for (int i = threadIdx.x, j = 0; i < len; i += NT, j++) {
        const uint32_t k = order_key(__uint_as_float(skeys[i]), status);
        skeys[i] = k;
        kmax = max(kmax, k);
#pragma unroll
        for (int g = 0; g < G; g++)
            if (j % G == g) {
                gmax[g] = max(gmax[g], k);
                has[g] = true;
            }
    }
    uint32_t lbound = 0xffffffffu;
#pragma unroll
    for (int g = 0; g < G; g++) lbound = min(lbound, has[g] ? gmax[g] : 0u);
    block_minmax<NT>(lbound, kmax, sh);     // its barrier also publishes skeys
    const int K = min(kTopK, len);
    uint32_t T = 0;
    int need_eq = len;
    if (len > kTopK) radix_threshold<NT>(skeys, len, K, lbound, kmax, sh, &T, &need_eq);
    if (threadIdx.x == 0) *info = make_uint2(len > kTopK ? T : 0u, kmax);
    ordered_compact<NT>(skeys, len, T, need_eq, sh, [&](int pos, int i, uint32_t k) {
        ok[pos] = k;
        oi[pos] = base + i;
    });
}

}  // namespace csa
