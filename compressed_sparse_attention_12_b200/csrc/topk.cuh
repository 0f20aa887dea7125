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
// and writes the block total to *total.  Warp totals go through sh.warp_a and
// are scanned by every warp with shuffles (NT <= 1024).
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *total,
                                                    TkSharedT<NT> &sh) {
    constexpr int W = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) sh.warp_a[warp] = incl;
    __syncthreads();
    uint32_t x = lane < W ? sh.warp_a[lane] : 0u;
#pragma unroll
    for (int o = 1; o < W; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += n;
    }
    const uint32_t upto = __shfl_sync(0xffffffffu, x, warp > 0 ? warp - 1 : 0);
    *total = __shfl_sync(0xffffffffu, x, W - 1);
    __syncthreads();
    return (warp > 0 ? upto : 0u) + incl - v;
}

// Block-wide min and max of one value pair per thread (uses sh.warp_a/b).
template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t &lo, uint32_t &hi, TkSharedT<NT> &sh) {
    constexpr int W = NT / 32;
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
    lo = lane < W ? sh.warp_a[lane] : 0xffffffffu;
    hi = lane < W ? sh.warp_b[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
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
// With one_pass the result is only the lower edge of the top digit's bin: a
// lower bound of the K-th largest key.
template <int NT>
__device__ void radix_threshold(const uint32_t *keys, int n, int K, uint32_t kmin, uint32_t kmax,
                                TkSharedT<NT> &sh, uint32_t *T_out, int *need_eq_out,
                                bool one_pass = false) {
    const uint32_t range = kmax - kmin;
    const int B = range == 0 ? 0 : 32 - __clz(range);
    uint32_t prefix = 0;            // resolved high bits of d
    int remaining = K;
#pragma unroll 1
    for (int done = 0; done < B && !(one_pass && done > 0);) {
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

// Copies row[0..len) (float logits, as bits) into skeys[0..len).  Every
// thread keeps up to 8 loads of 16 bytes in flight before storing them, so the
// copy costs a few memory round trips rather than one per vector.
template <int NT>
__device__ __forceinline__ void stage_row_keys(uint32_t *skeys, const float *__restrict__ row,
                                               int len) {
    if ((reinterpret_cast<uintptr_t>(row) & 15) == 0) {
        const int n4 = len / 4;
        const uint4 *src = reinterpret_cast<const uint4 *>(row);
        uint4 *dst = reinterpret_cast<uint4 *>(skeys);
        for (int base = 0; base < n4; base += 8 * NT) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int i = base + u * NT + (int)threadIdx.x;
                if (i < n4) v[u] = src[i];
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int i = base + u * NT + (int)threadIdx.x;
                if (i < n4) dst[i] = v[u];
            }
        }
        for (int i = 4 * n4 + threadIdx.x; i < len; i += NT) skeys[i] = __float_as_uint(row[i]);
    } else {
        for (int base = 0; base < len; base += 8 * NT) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int i = base + u * NT + (int)threadIdx.x;
                if (i < len) v[u] = row[i];
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int i = base + u * NT + (int)threadIdx.x;
                if (i < len) skeys[i] = __float_as_uint(v[u]);
            }
        }
    }
}

// The top-512 of skeys[0..len), which hold the float bits of the logits
// (index i): converts them to keys in place, finds the threshold and calls
// emit(pos, i, key) for the selected ones in index order (pos = rank in that
// order).  Returns min(512, len); *T_out gets the 512th-largest key (0 when
// len <= 512) and *kmax_out the largest.
//
// Lower bound: thread t's keys i = t + j*NT fall into G = ceil(512/NT) groups by
// j % G.  When all NT*G groups are non-empty the smallest group maximum is at
// most the 512th-largest key (the NT*G >= 512 group maxima are distinct keys
// not below it), so the radix digits start from that bound; otherwise the
// bound is 0.
template <int NT, typename Emit>
__device__ __forceinline__ int select_top512(uint32_t *skeys, int len, TkSharedT<NT> &sh, int32_t *status,
                             uint32_t *T_out, uint32_t *kmax_out, Emit emit) {
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
    *T_out = len > kTopK ? T : 0u;
    *kmax_out = kmax;
    ordered_compact<NT>(skeys, len, T, need_eq, sh, emit);
    return K;
}

// One chunk of a row: skeys[0..len) hold the float bits of the chunk's logits
// (index base + i).  Writes the chunk's top-512 (or all of it when shorter) in
// index order to ok/oi and the chunk's (512th-largest key or 0 when it holds
// fewer, largest key) to *info.
template <int NT>
__device__ void select_chunk(uint32_t *skeys, int len, int base, uint32_t *ok, int32_t *oi,
                             uint2 *info, TkSharedT<NT> &sh, int32_t *status) {
    uint32_t T, kmax;
    select_top512<NT>(skeys, len, sh, status, &T, &kmax, [&](int pos, int i, uint32_t k) {
        ok[pos] = k;
        oi[pos] = base + i;
    });
    if (threadIdx.x == 0) *info = make_uint2(T, kmax);
}


// ---------------------------------------------------------------- register rows
// A row of at most NT*KPT keys held in registers: thread t owns the contiguous
// keys [KPT*t, KPT*t + KPT) of the row (those at or past len are absent).

// The K-th largest key T among the present keys >= kmin (as radix_threshold,
// reading the keys from registers) and how many keys equal to T are taken.
// present(j) tells which of the thread's keys take part.  With one_pass the
// result is only the top digit's lower edge: a lower bound of T.
template <int NT, int KPT, typename Present>
__device__ __forceinline__ void radix_threshold_regs(const uint32_t (&keys)[KPT], Present present,
                                                     int K, uint32_t kmin, uint32_t kmax,
                                                     TkSharedT<NT> &sh, uint32_t *T_out,
                                                     int *need_eq_out, bool one_pass = false) {
    const uint32_t range = kmax - kmin;
    const int B = range == 0 ? 0 : 32 - __clz(range);
    uint32_t prefix = 0;
    int remaining = K;
#pragma unroll 1
    for (int done = 0; done < B && !(one_pass && done > 0);) {
        const int width = min(12, B - done);
        const int shift = B - done - width;
        const int hi = shift + width;
        const uint32_t nb = 1u << width;
        for (uint32_t i = threadIdx.x; i < nb; i += NT) sh.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < KPT; j++) {
            const uint32_t k = keys[j];
            const uint32_t d = k - kmin;
            const bool match = present(j) && k >= kmin && (hi >= 32 || ((d ^ prefix) >> hi) == 0);
            if (match) atomicAdd(&sh.hist[(d >> shift) & (nb - 1)], 1u);
        }
        __syncthreads();
        const int per = (int)((nb + NT - 1) / NT);
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

// Index-order ranks for a register row: thread (warp w, lane l) holds the
// 16-byte slices j = 0..KPT/4-1 at keys 1024w + 128j + 4l .. +3 (NT = 1024,
// KPT = 32: warp w owns keys [1024w, 1024w + 1024), slices in index order,
// lanes in index order within a slice).  v[j] are per-thread counts for
// slice j (two 16-bit fields may be packed: every total stays below 2^16);
// each becomes the number of counted keys before slice j of this thread in
// index order over the whole row, in place of v[j]; returns the row total.
template <int NT, int NS>
__device__ __forceinline__ uint32_t ordered_starts(uint32_t (&v)[NS], TkSharedT<NT> &sh) {
    const int lane = threadIdx.x & 31;
    uint32_t run = 0;
#pragma unroll
    for (int j = 0; j < NS; j++) {
        uint32_t incl = v[j];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        v[j] = run + incl - v[j];
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    uint32_t tot;
    const uint32_t woff = block_excl_scan<NT>(lane == 31 ? run : 0u, &tot, sh);
#pragma unroll
    for (int j = 0; j < NS; j++) v[j] += woff;
    return tot;
}

// Top-512 of a register row of len <= NT*KPT keys in the layout of
// ordered_starts (`keys` hold the float bits on entry; key slot 4j+e is row
// index 1024w + 128j + 4l + e).  Calls emit(pos, index) for the selected keys
// with pos their rank in index order; returns min(512, len).
//
// Lower bound: the keys fall into groups of 8 (two slices of a thread); when
// there are at least 512 non-empty groups, any value at most their
// 512th-largest maximum is at most the row's 512th-largest key (512 groups
// hold a key >= it).  One radix pass over the group maxima gives such a value
// L (the lower edge of the bin holding that maximum).  The keys >= L (usually
// a little over 512) are staged in index order in cand_key/cand_idx (cap
// entries) and the selection runs over them; rows with more (heavy ties)
// select from the registers directly.
template <int NT, int KPT, typename Emit>
__device__ __forceinline__ int select_top512_regs(uint32_t (&keys)[KPT], int len,
                                                  TkSharedT<NT> &sh, uint32_t *cand_key,
                                                  int32_t *cand_idx, int cap, int32_t *status,
                                                  Emit emit) {
    static_assert(NT == 1024 && KPT == 32, "layout of ordered_starts");
    constexpr int NS = KPT / 4, NG = KPT / 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto index_of = [&](int kk) { return 1024 * warp + 128 * (kk >> 2) + 4 * lane + (kk & 3); };
    auto present = [&](int kk) { return index_of(kk) < len; };
    uint32_t gmax[NG];
    uint32_t gany = 0;        // bit g: group g holds a key
#pragma unroll
    for (int g = 0; g < NG; g++) gmax[g] = 0u;
#pragma unroll
    for (int kk = 0; kk < KPT; kk++) {
        const bool p = present(kk);
        const uint32_t k = p ? order_key(__uint_as_float(keys[kk]), status) : 0u;
        keys[kk] = k;
        if (p) {
            gmax[kk / 8] = max(gmax[kk / 8], k);
            gany |= 1u << (kk / 8);
        }
    }
    uint32_t gmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int g = 0; g < NG; g++)
        if (gany & (1u << g)) {
            gmin = min(gmin, gmax[g]);
            kmax = max(kmax, gmax[g]);
        }
    block_minmax<NT>(gmin, kmax, sh);
    uint32_t ng_total;
    block_excl_scan<NT>((uint32_t)__popc(gany), &ng_total, sh);
    const int K = min(kTopK, len);
    uint32_t L = 0u;
    if (len > kTopK && ng_total >= (uint32_t)kTopK) {
        int unused;
        radix_threshold_regs<NT, NG>(gmax, [&](int g) { return (gany >> g) & 1u; }, kTopK, gmin,
                                     kmax, sh, &L, &unused, true);
    }
    uint32_t T = 0;
    int need_eq = len;
    // candidates: the keys >= L, in index order
    uint32_t at[NS];
#pragma unroll
    for (int j = 0; j < NS; j++) {
        at[j] = 0;
#pragma unroll
        for (int e = 0; e < 4; e++) at[j] += (present(4 * j + e) && keys[4 * j + e] >= L) ? 1u : 0u;
    }
    const uint32_t n_cand = ordered_starts<NT, NS>(at, sh);
    if (n_cand <= (uint32_t)cap) {                 // uniform over the block
#pragma unroll
        for (int j = 0; j < NS; j++) {
            uint32_t a = at[j];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int kk = 4 * j + e;
                if (present(kk) && keys[kk] >= L) {
                    cand_key[a] = keys[kk];
                    cand_idx[a] = index_of(kk);
                    a++;
                }
            }
        }
        __syncthreads();
        if (len > kTopK)
            radix_threshold<NT>(cand_key, (int)n_cand, K, L, kmax, sh, &T, &need_eq);
        ordered_compact<NT>(cand_key, (int)n_cand, T, need_eq, sh,
                            [&](int pos, int i, uint32_t) { emit(pos, cand_idx[i]); });
        return K;
    }
    if (len > kTopK) radix_threshold_regs<NT, KPT>(keys, present, K, L, kmax, sh, &T, &need_eq);
    // ordered output from the registers: counts of keys above T and equal to
    // T per slice, packed 16/16 bits (totals <= 32768)
    uint32_t st[NS];
#pragma unroll
    for (int j = 0; j < NS; j++) {
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int kk = 4 * j + e;
            gt += (present(kk) && keys[kk] > T) ? 1u : 0u;
            eq += (present(kk) && keys[kk] == T) ? 1u : 0u;
        }
        st[j] = gt | (eq << 16);
    }
    ordered_starts<NT, NS>(st, sh);
#pragma unroll
    for (int j = 0; j < NS; j++) {
        uint32_t gt_before = st[j] & 0xFFFFu, eq_seen = st[j] >> 16;
        uint32_t pos = gt_before + min(eq_seen, (uint32_t)need_eq);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int kk = 4 * j + e;
            if (present(kk)) {
                const uint32_t k = keys[kk];
                bool take = k > T;
                if (k == T) {
                    take = eq_seen < (uint32_t)need_eq;
                    eq_seen++;
                }
                if (take) emit((int)pos++, index_of(kk));
            }
        }
    }
    return K;
}
}  // namespace csa
