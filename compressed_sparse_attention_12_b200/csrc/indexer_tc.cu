// indexer_tc.cu -- step 2 on the 5th-generation tensor cores (tcgen05).
//
// The indexer of "Token 的一生：DSV4 架构与 DSpark" §1/§3 (scores every
// compressed token for each query; FP8 index cache, §3.1) with the light
// low-precision indexer of "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section
// "Compressed Sparse Attention（CSA）":
//   logits[t][s] = k_scale[s] * sum_h w'[t][h] * ReLU(qhat[t][h] . khat[s]).
//
// Shape on the tensor core (keys on M so that every 128-key tile is one MMA
// tile): D[128 keys x N] = K_tile[128 x Di] * Q^T, N = (query rows of a
// group) x (heads padded to 16).  One CTA streams a contiguous run of key
// tiles of one request for one query group:
//   warp 0  TMA producer: two 64-row pages per tile straight from the paged
//           index cache (page ids from the page table) into a ring of stages,
//   warp 1  MMA issuer: Di/32-byte K-steps of tcgen05.mma into one of two
//           TMEM accumulators, commits free the stage and hand the
//           accumulator to the epilogue,
//   warps 2-9 epilogue, two groups of four warps (each group covers the four
//           TMEM lane quadrants; group 0 takes the even tiles / accumulator 0,
//           group 1 the odd tiles / accumulator 1): tcgen05.ld of the key's
//           row, ReLU, head-weighted sum per query, times the key's scale,
//           one coalesced float store.
// Formats: FP8 E4M3 (kind::f8f6f4), bf16 (kind::f16), and FP4 E2M1 with
// unsigned-E4M3 block-16 scales (kind::mxf4nvf4 block-scaled): warp 0's other
// lanes gather each tile's key block scales into the 128-row scale-factor
// layout in shared memory, the MMA thread moves them into TMEM with
// tcgen05.cp, and the query's block scales are placed in TMEM once.  All
// waits are bounded; a timeout records CSA_ERR_TIMEOUT and the CTA unwinds.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "topk.cuh"

namespace csa {

// Warps: producer, MMA, then EG epilogue groups of four (EG = 2: 320 threads,
// two CTAs per SM; EG = 4 for the 256-column accumulators of prefill-shaped
// launches: 576 threads, one CTA per SM)
template <int EG>
__host__ __device__ constexpr int tc_threads() { return 64 + 128 * EG; }
constexpr int kTcThreads = tc_threads<2>();
constexpr int kTcTile = 128;      // keys per tile (two 64-row pages)

template <int RB>
struct TcGeom {
    static constexpr int kSpan = RB >= 128 ? 128 : RB;     // swizzle span (bytes)
    static constexpr int kChunks = RB >= 128 ? RB / 128 : 1;
    static constexpr int kKSteps = RB / 32;                // 32-byte K-steps
    static constexpr int kStageBytes = kTcTile * RB;
};

struct TcParams {
    int qg;            // query rows per group
    int hi_pad;        // heads padded to a multiple of 16
    int n;             // MMA N = qg * hi_pad
    int tmem_cols;     // power of two >= 2n
    int tiles_per_cta;
    int stages;
    int num_pages;
    int nacc;          // TMEM accumulators in flight (power of two, >= 2)
};

// Where a fused launch leaves each CTA's chunk selection (all null: logits only).
// Row t, chunk c (= blockIdx.x, tiles_per_cta*128 keys) owns 512 slots at
// (t*max_chunks + c)*512 and one (512th key, largest key) pair.
struct TcSelect {
    uint32_t *cand_key;
    int32_t *cand_idx;
    uint2 *chunk_info;
    int max_chunks;
};

constexpr int kKsRing = 8;     // key-scale tiles in flight per epilogue group
// FP4 block scales of Di = 64 keys (4 bytes a key): copied as 16-byte chunks
// into a staging ring and moved into the tensor-core scale layout kSfLag
// tiles later (kSfLag < stages); Di = 128 keys gather theirs 4 bytes at a
// time straight into the layout (measured faster there)
constexpr int kSfLag = 4;
constexpr int kSfSlots = kSfLag + 1;

// Query group g of a launch.  Request b's query rows form ceil(rows_b / qg)
// groups of qg consecutive rows (the last one shorter), numbered after the
// groups of requests 0..b-1.  Sets *b_out and the group's first row *t0_out
// (-1 when g is past the last group).  Every lane of the calling warp must be
// active: the requests are scanned 32 at a time with a warp prefix sum.
__device__ __forceinline__ void query_group(const int *cu_q, int bs, int qg, int g, int *b_out,
                                            int *t0_out) {
    *b_out = 0;
    *t0_out = -1;
    if (qg == 1) {                        // one group per row
        if (g >= cu_q[bs]) return;
        int lo = 0, hi = bs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cu_q[mid] <= g) lo = mid; else hi = mid - 1;
        }
        *b_out = lo;
        *t0_out = g;
        return;
    }
    const int lane = threadIdx.x & 31;
    int before = 0;                       // groups of the requests already scanned
    for (int b0 = 0; b0 < bs; b0 += 32) {
        const int bb = b0 + lane;
        int first = 0, ng = 0;
        if (bb < bs) {
            first = cu_q[bb];
            ng = (cu_q[bb + 1] - first + qg - 1) / qg;
        }
        int incl = ng;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        const uint32_t hit = __ballot_sync(0xffffffffu, g < before + incl);
        if (hit) {
            const int src = __ffs(hit) - 1;
            const int excl = before + __shfl_sync(0xffffffffu, incl - ng, src);
            *b_out = b0 + src;
            *t0_out = __shfl_sync(0xffffffffu, first, src) + (g - excl) * qg;
            return;
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// Upper bound of the number of query groups: sum over requests of
// ceil(rows_b / qg) <= (num_q + bs * (qg - 1)) / qg, and at most num_q.
static int query_groups_bound(int num_q, int bs, int qg) {
    if (qg <= 1) return num_q;
    const long long g = ((long long)num_q + (long long)bs * (qg - 1)) / qg;
    return (int)(g < num_q ? g : num_q);
}

// Packed fp32 pair multiply-add: acc += a * b elementwise (one instruction
// for two lanes of work on sm_100).
__device__ __forceinline__ void ffma2(float2 &acc, float2 a, float2 b) {
    uint64_t d;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%1, %2};\n\tmov.b64 rb, {%3, %4};\n\tmov.b64 rc, {%5, %6};\n\t"
        "fma.rn.f32x2 %0, ra, rb, rc;\n\t}"
        : "=l"(d)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(acc.x), "f"(acc.y));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(acc.x), "=f"(acc.y) : "l"(d));
}

// acc += w[j] * ReLU(v[j]) over 16 accumulator columns (part of one query's
// run of heads) as two pair accumulators, weights read 16 bytes at a time.
__device__ __forceinline__ void relu_dot16(const uint32_t *v, const float *w, float2 (&acc)[2]) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float4 wv = *reinterpret_cast<const float4 *>(w + j);
        ffma2(acc[0], make_float2(wv.x, wv.y),
              make_float2(fmaxf(__uint_as_float(v[j]), 0.f), fmaxf(__uint_as_float(v[j + 1]), 0.f)));
        ffma2(acc[1], make_float2(wv.z, wv.w),
              make_float2(fmaxf(__uint_as_float(v[j + 2]), 0.f),
                          fmaxf(__uint_as_float(v[j + 3]), 0.f)));
    }
}

template <int FMT, int RB, int EG>
__global__ void __launch_bounds__(tc_threads<EG>(), EG == 2 ? 2 : 1)
indexer_tc_kernel(const IndexerArgs a, const __grid_constant__ CUtensorMap kmap,
                  const TcParams p, const TcSelect sel) {
    pdl_begin();
    using G = TcGeom<RB>;
    constexpr int kThreads = tc_threads<EG>();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: stages | q tile | w' | nv | barriers
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    // paged FP4 keys: one record per 64-key page, 8 groups of 8 keys, each
    // group's codes (8-key x 16-byte blocks), block scales and row scales
    // side by side; a tile is two records copied whole
    constexpr bool kPaged = FMT == CSA_FMT_FP4_PAGE;
    constexpr bool kFp4 = FMT == CSA_FMT_FP4 || kPaged;
    constexpr bool kSfStaged = kFp4 && RB == 32 && !kPaged;
    constexpr int kGb = 9 * RB + 32;                     // bytes of an 8-key group (4.5 Di + 32)
    constexpr int kRec = 8 * kGb;                        // bytes of a page record (36 Di + 256)
    constexpr int kStage = kPaged ? 2 * kRec : G::kStageBytes;
    uint8_t *stage_buf = base;
    uint8_t *q_buf = stage_buf + p.stages * kStage;
    uint8_t *sfa_buf = q_buf + ((p.n * RB + 1023) & ~1023);            // [stages][ksteps][512]
    uint8_t *sfb_buf = sfa_buf + (kFp4 ? p.stages * G::kKSteps * 512 : 0);  // [ksteps][512]
    uint8_t *sf_stage = sfb_buf + (kFp4 ? G::kKSteps * 512 : 0);    // [kSfSlots][16 * RB]
    float *w_s = reinterpret_cast<float *>(sf_stage + (kSfStaged ? kSfSlots * 16 * RB : 0));
    int *nv_s = reinterpret_cast<int *>(w_s + 256);
    uint64_t *bars = reinterpret_cast<uint64_t *>(nv_s + 16);
    uint64_t *full = bars, *empty = bars + p.stages, *tfull = bars + 2 * p.stages;
    uint64_t *tempty = tfull + p.nacc, *drain = tempty + p.nacc;
    uint64_t *sfull = drain + 1;                         // paged: the record copies per stage
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfull + p.stages);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *pg_s = const_cast<int *>(abort_flag) + 4;     // page ids of this CTA's tiles (-1: none)
    // per epilogue group, kKsRing tiles of key scales in flight (cp.async ring)
    float *ks_ring = reinterpret_cast<float *>(
        (reinterpret_cast<uintptr_t>(pg_s + 2 * p.tiles_per_cta) + 15) & ~(uintptr_t)15);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- which query group and key tiles (uniform over the CTA)
    int b, t0;
    query_group(a.cu_q, a.bs, p.qg, (int)blockIdx.y, &b, &t0);
    if (t0 < 0) return;                                     // past the last group
    const int last = a.cu_q[b + 1];
    const int nq = min(p.qg, last - t0);
    const int cap = min(a.max_c4_len, a.pt_stride * kC4Page);
    int nv_max = 0;
    int nv_q[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        int n = 0;
        if (i < nq) {
            n = a.c4_seq_lens[b];
            if (a.q_pos) n = min(n, (a.q_pos[t0 + i] + 1) / a.ratio);
            if (n > cap) {
                if (threadIdx.x == 0 && blockIdx.x == 0) report(a.status, CSA_ERR_BOUNDS);
                n = cap;
            }
            n = max(n, 0);
        }
        nv_q[i] = n;
        nv_max = max(nv_max, n);
    }
    const int ntiles = (nv_max + kTcTile - 1) / kTcTile;
    const int tile_begin = blockIdx.x * p.tiles_per_cta;
    const int tile_end = min(ntiles, tile_begin + p.tiles_per_cta);
    if (tile_begin >= tile_end) return;
    const int my_tiles = tile_end - tile_begin;
    const int32_t *pt_row = a.page_table + (int64_t)b * a.pt_stride;

    // ---- set-up
    if (warp == 0) tc::tmem_alloc(tc::saddr(tmem_slot), (uint32_t)p.tmem_cols);
    if (threadIdx.x == 32) {
        for (int s = 0; s < p.stages; s++) {
            // the producer's expect_tx arrival, and with staged block scales a
            // second one once they are in place (gathered ones add and
            // complete their own pending arrivals)
            tc::mbar_init(tc::saddr(&full[s]), kSfStaged ? 2 : 1);
            // paged: the stage (which holds the row scales) is released by the
            // epilogue warps that read them, not by the MMA
            tc::mbar_init(tc::saddr(&empty[s]), kPaged ? 4 * (EG / 2) : 1);
            if constexpr (kPaged) tc::mbar_init(tc::saddr(&sfull[s]), 1);
        }
        for (int i = 0; i < p.nacc; i++) {
            tc::mbar_init(tc::saddr(&tfull[i]), 1);
            tc::mbar_init(tc::saddr(&tempty[i]), 4 * (EG / 2));   // the warps reading it
        }
        tc::mbar_init(tc::saddr(drain), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (threadIdx.x < 4) nv_s[threadIdx.x] = nv_q[threadIdx.x];
    for (int u = threadIdx.x; u < 2 * my_tiles; u += kThreads) {
        const int pidx = tile_begin * 2 + u;
        int page = -1;
        if (pidx * kC4Page < nv_max && pidx < a.pt_stride) page = pt_row[pidx];
        pg_s[u] = page;
    }
    // query tile: row n = qi*hi_pad + h (K-major, swizzled like the key tiles)
    {
        const uint8_t *qc = reinterpret_cast<const uint8_t *>(a.q_codes);
        const int chunks16 = RB / 16;
        for (int u = threadIdx.x; u < p.n * chunks16; u += kThreads) {
            const int n = u / chunks16, c = u % chunks16;
            const int qi = n / p.hi_pad, h = n % p.hi_pad;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (qi < nq && h < a.heads)
                v = *reinterpret_cast<const uint4 *>(qc + ((int64_t)(t0 + qi) * a.heads + h) * RB +
                                                     c * 16);
            const int chunk = (c * 16) / G::kSpan, byte = (c * 16) % G::kSpan;
            *reinterpret_cast<uint4 *>(q_buf + chunk * p.n * G::kSpan +
                                       tc::swz(n, byte, G::kSpan)) = v;
        }
        for (int n = threadIdx.x; n < p.n; n += kThreads) {
            const int qi = n / p.hi_pad, h = n % p.hi_pad;
            w_s[n] = (qi < nq && h < a.heads) ? a.q_weights[(int64_t)(t0 + qi) * a.heads + h] : 0.f;
        }
        if constexpr (kFp4) {
            // scale-factor layout of 128 rows: row n = m0 + 32*m1 keeps its four
            // block scales of K-step ks at byte ks*512 + m0*16 + m1*4
            constexpr int nsf = RB / 8;      // block scales per row (Di/16; a row is Di/2 bytes)
            for (int u = threadIdx.x; u < 128 * G::kKSteps; u += kThreads) {
                const int n = u % 128, ks = u / 128;
                const int qi = n / p.hi_pad, h = n % p.hi_pad;
                uint32_t wv = 0;
                if (n < p.n && qi < nq && h < a.heads)
                    wv = *reinterpret_cast<const uint32_t *>(
                        a.q_block_scales + ((int64_t)(t0 + qi) * a.heads + h) * nsf + ks * 4);
                *reinterpret_cast<uint32_t *>(sfb_buf + ks * 512 + (n & 31) * 16 + (n >> 5) * 4) = wv;
            }
        }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (lane 0) and FP4 block-scale gather (all lanes)
        int issued = 0;
        // FP4: moves tile j's staged block scales into the scale layout of 128
        // rows (row m = m0 + 32*m1 keeps its four scales of K-step ks at byte
        // ks*512 + m0*16 + m1*4) of stage j % stages, then releases the
        // stage's second arrival.  Each lane moves the chunks it copied.
        auto sf_place = [&](int j) {
            if constexpr (kSfStaged) {
                constexpr int nsf = RB / 8;
                constexpr int kChunksPerPage = 4 * nsf;
                constexpr int KS = G::kKSteps;            // = nsf / 4
                const uint8_t *stg = sf_stage + (j % kSfSlots) * 16 * RB;
                uint8_t *dst = sfa_buf + (j % p.stages) * KS * 512;
#pragma unroll
                for (int q = lane; q < 2 * kChunksPerPage; q += 32) {
                    const int half = q / kChunksPerPage, c = q % kChunksPerPage;
                    const int32_t page = pg_s[j * 2 + half];
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (page >= 0 && page < p.num_pages)
                        v = *reinterpret_cast<const uint4 *>(stg + q * 16);
                    const int m0 = half * 64 + c * (16 / nsf);
#pragma unroll
                    for (int w = 0; w < 4; w++) {
                        const int m = m0 + w / KS, ks = w % KS;
                        const uint32_t x = w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
                        *reinterpret_cast<uint32_t *>(dst + ks * 512 + (m & 31) * 16 + (m >> 5) * 4) = x;
                    }
                }
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(tc::saddr(&full[j % p.stages]));
            }
            if constexpr (kPaged) {
                // tile j's records have landed (every lane observes the copy);
                // move their block scales into the scale layout of stage j
                const int s = j % p.stages;
                const bool got = tc::mbar_wait(tc::saddr(&sfull[s]),
                                               (uint32_t)((j / p.stages) & 1), abort_flag);
                if (!__all_sync(0xffffffffu, got)) {              // uniform over the warp
                    if (lane == 0) {
                        if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    return;
                }
                constexpr int nsf = RB / 8;                   // block scales per key
                constexpr int kCpg = RB / 16;                 // 16-byte scale chunks per group
                constexpr int KS = G::kKSteps;
                const uint8_t *stg = stage_buf + s * kStage;
                uint8_t *dst = sfa_buf + s * KS * 512;
#pragma unroll
                for (int q = lane; q < 16 * kCpg; q += 32) {
                    const int half = q / (8 * kCpg), c = q % (8 * kCpg);
                    const int g = c / kCpg, cg = c % kCpg;
                    const int32_t page = pg_s[j * 2 + half];
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (page >= 0 && page < p.num_pages)
                        v = *reinterpret_cast<const uint4 *>(stg + half * kRec + g * kGb + 8 * RB +
                                                             cg * 16);
                    const int m0 = half * 64 + g * 8 + cg * (16 / nsf);
#pragma unroll
                    for (int w = 0; w < 4; w++) {
                        const int m = m0 + w / KS, ks = w % KS;
                        const uint32_t x = w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
                        *reinterpret_cast<uint32_t *>(dst + ks * 512 + (m & 31) * 16 + (m >> 5) * 4) = x;
                    }
                }
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(tc::saddr(&full[s]));
            }
        };
        for (int i = 0; i < my_tiles; i++) {
            const int s = i % p.stages;
            const uint32_t ph = (uint32_t)((i / p.stages) & 1);
            int ok = 1;
            if (lane == 0) {
                ok = tc::mbar_wait(tc::saddr(&empty[s]), ph ^ 1u, abort_flag) ? 1 : 0;
                if (!ok) {
                    if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                    *abort_flag = 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if constexpr (kFp4 && !kSfStaged && !kPaged) {
                // key m = lane + 32*m1 of the tile: its block scales of K-step ks go
                // to byte (s*ksteps + ks)*512 + lane*16 + m1*4 by 4-byte cp.async;
                // each lane's copies hold the stage's phase open until they land
                // (the non-noinc arrive adds one pending arrival first)
                constexpr int nsf = RB / 8;      // Di/16 block scales per key
#pragma unroll
                for (int m1 = 0; m1 < 4; m1++) {
                    const int m = lane + 32 * m1;
                    const int sk = (tile_begin + i) * kTcTile + m;
                    int64_t slot = -1;
                    if (sk < nv_max) {
                        const int32_t page = pg_s[i * 2 + (m >> 6)];
                        if (page >= 0 && page < p.num_pages) slot = (int64_t)page * kC4Page + (m & 63);
                    }
#pragma unroll
                    for (int ks = 0; ks < G::kKSteps; ks++) {
                        uint8_t *dst = sfa_buf + (s * G::kKSteps + ks) * 512 + lane * 16 + m1 * 4;
                        if (slot >= 0)
                            tc::cp_async4(tc::saddr(dst), a.k_block_scales + slot * nsf + ks * 4);
                        else
                            *reinterpret_cast<uint32_t *>(dst) = 0u;
                    }
                }
                tc::cp_async_mbar_arrive(tc::saddr(&full[s]));
                __syncwarp();
            }
            if constexpr (kSfStaged && !kPaged) {
                // the tile's block scales: 16-byte chunks of each page's
                // contiguous 64 x Di/16 bytes into staging slot i % kSfSlots
                constexpr int nsf = RB / 8;               // Di/16 block scales per key
                constexpr int kChunksPerPage = 4 * nsf;   // 16-byte chunks per page
                uint8_t *stg = sf_stage + (i % kSfSlots) * 16 * RB;
#pragma unroll
                for (int q = lane; q < 2 * kChunksPerPage; q += 32) {
                    const int32_t page = pg_s[i * 2 + q / kChunksPerPage];
                    if (page >= 0 && page < p.num_pages)
                        tc::cp_async16(tc::saddr(stg + q * 16),
                                       a.k_block_scales + (int64_t)page * kC4Page * nsf +
                                           (q % kChunksPerPage) * 16);
                }
                tc::cp_async_commit();
            }
            if (!kPaged && G::kChunks == 1) {
                // one box per page: lanes 0 and 1 issue the tile's two pages
                // in one instruction
                if (lane == 0) tc::mbar_expect_tx(tc::saddr(&full[s]), G::kStageBytes);
                __syncwarp();
                if (lane < 2) {
                    int page = pg_s[i * 2 + lane];
                    if (page < 0 || page >= p.num_pages) page = 0;   // epilogue reports visible keys
                    tc::tma_load_2d(tc::saddr(stage_buf + s * kStage + lane * 64 * G::kSpan),
                                    &kmap, 0, page * kC4Page, tc::saddr(&full[s]));
                }
            } else if (lane == 0) {
                if constexpr (kPaged) tc::mbar_expect_tx(tc::saddr(&sfull[s]), kStage);
                else tc::mbar_expect_tx(tc::saddr(&full[s]), G::kStageBytes);
#pragma unroll
                for (int half = 0; half < 2; half++) {
                    int page = pg_s[i * 2 + half];
                    if (page < 0 || page >= p.num_pages) page = 0;   // epilogue reports visible keys
                    if constexpr (kPaged) {
                        // one copy per page: the whole record, one TMA box of
                        // kRec/256 rows of 256 bytes (no swizzle)
                        tc::tma_load_2d(tc::saddr(stage_buf + s * kStage + half * kRec), &kmap, 0,
                                        page * (kRec / 256), tc::saddr(&sfull[s]));
                    } else {
#pragma unroll
                        for (int c = 0; c < G::kChunks; c++)
                            tc::tma_load_2d(tc::saddr(stage_buf + s * kStage +
                                                      c * kTcTile * G::kSpan + half * 64 * G::kSpan),
                                            &kmap, c * G::kSpan, page * kC4Page,
                                            tc::saddr(&full[s]));
                    }
                }
            }
            issued++;
            if constexpr (kSfStaged || kPaged) {
                if (i >= kSfLag) {
                    if constexpr (kSfStaged) tc::cp_async_wait<kSfLag>();
                    sf_place(i - kSfLag);
                }
            }
        }
        if constexpr (kSfStaged || kPaged) {
            if constexpr (kSfStaged) tc::cp_async_wait<0>();
            for (int j = max(0, issued - kSfLag); j < issued; j++) sf_place(j);
        }
        // before leaving, every load issued must have landed
        if (lane == 0)
            for (int i = max(0, issued - p.stages); i < issued; i++)
                tc::mbar_wait(tc::saddr(&full[i % p.stages]), (uint32_t)((i / p.stages) & 1), nullptr);
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = FMT == CSA_FMT_FP8  ? tc::idesc_m128(0, 0, p.n)
                                   : FMT == CSA_FMT_BF16 ? tc::idesc_m128(1, 1, p.n)
                                                         : tc::idesc_mxf4_m128(p.n);
            // TMEM columns: [0, nacc*n) accumulators, then one set of key block
            // scales per accumulator (4 columns per K-step), then the query
            // block scales
            const uint32_t sfa_col = (uint32_t)(p.nacc * p.n);
            const uint32_t sfb_col = sfa_col + (uint32_t)(p.nacc * 4 * G::kKSteps);
            if constexpr (kFp4) {
#pragma unroll
                for (int ks = 0; ks < G::kKSteps; ks++)
                    tc::tmem_cp_32x128b_x4(tmem_base + sfb_col + 4 * ks,
                                           tc::rows16_desc(tc::saddr(sfb_buf + ks * 512)));
            }
            for (int i = 0; i < my_tiles; i++) {
                const int s = i % p.stages;
                const int acc = i & (p.nacc - 1);
                if (!tc::mbar_wait(tc::saddr(&full[s]), (uint32_t)((i / p.stages) & 1), abort_flag) ||
                    !tc::mbar_wait(tc::saddr(&tempty[acc]), (uint32_t)(((i / p.nacc) & 1) ^ 1),
                                   abort_flag)) {
                    if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                tc::fence_after_sync();
                if constexpr (kFp4) tc::fence_proxy_async();   // cp.async-written scales -> tcgen05.cp
                const uint32_t d = tmem_base + (uint32_t)(acc * p.n);
                const uint32_t sa = tc::saddr(stage_buf + s * kStage);
                const uint32_t sb = tc::saddr(q_buf);
                const uint32_t sfa = tmem_base + sfa_col + (uint32_t)(acc * 4 * G::kKSteps);
                if constexpr (kFp4) {
#pragma unroll
                    for (int ks = 0; ks < G::kKSteps; ks++)
                        tc::tmem_cp_32x128b_x4(
                            sfa + 4 * ks,
                            tc::rows16_desc(tc::saddr(sfa_buf + (s * G::kKSteps + ks) * 512)));
                }
#pragma unroll
                for (int k = 0; k < G::kKSteps; k++) {
                    const int c = (k * 32) / G::kSpan, off = (k * 32) % G::kSpan;
                    // paged keys: unswizzled, two 16-byte core matrices per K-step
                    const uint64_t ad = kPaged ? tc::kmajor_plain_desc(sa + k * 256, 128, kGb)
                                               : tc::kmajor_desc(sa + c * kTcTile * G::kSpan + off,
                                                                 G::kSpan);
                    const uint64_t bd = tc::kmajor_desc(sb + c * p.n * G::kSpan + off, G::kSpan);
                    if constexpr (FMT == CSA_FMT_FP8) tc::mma_f8f6f4(d, ad, bd, idesc, k > 0);
                    else if constexpr (FMT == CSA_FMT_BF16) tc::mma_f16(d, ad, bd, idesc, k > 0);
                    else tc::mma_mxf4nvf4(d, ad, bd, idesc, sfa + 4 * k, tmem_base + sfb_col + 4 * k,
                                          k > 0);
                }
                if constexpr (!kPaged) tc::mma_commit(tc::saddr(&empty[s]));
                tc::mma_commit(tc::saddr(&tfull[acc]));
            }
            // drain: every MMA issued has completed before TMEM is released
            tc::mma_commit(tc::saddr(drain));
            tc::mbar_wait(tc::saddr(drain), 0, nullptr);
        }
    } else {
        // ---------------- epilogue: group eg = (warp-2)/4 takes the tiles of
        // parity eg & 1; with four groups, eg >> 1 picks which half of the
        // group's query rows (and so of the accumulator columns) it reduces
        const int eg = (warp - 2) >> 2;
        const int par = eg & 1;
        const int qh = EG == 4 ? p.qg / 2 : p.qg;          // query rows per group
        const int x_lo = EG == 4 ? (eg >> 1) * qh : 0;
        const int c_lo = x_lo * p.hi_pad, c_hi = min(p.n, c_lo + qh * p.hi_pad);
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *lg = a.logits;
        // Key scale of this thread's row for the group's j-th tile (i = par + 2j):
        // a per-thread ring of kKsRing cp.async copies keeps the loads of the
        // next tiles in flight while this one is reduced.
        auto key_slot = [&](int i, bool &valid) -> int64_t {
            const int sk = (tile_begin + i) * kTcTile + row;
            valid = false;
            if (i >= my_tiles || sk >= nv_max) return -1;
            const int32_t page = pg_s[i * 2 + (row >> 6)];
            const int64_t slot = (int64_t)page * kC4Page + (row & 63);
            valid = page >= 0 && page < p.num_pages && slot < a.num_slots;
            return valid ? slot : -1;
        };
        float *my_ring = ks_ring + eg * kKsRing * kTcTile + row;
        auto ring_issue = [&](int j) {
            if constexpr (FMT != CSA_FMT_BF16 && !kPaged) {   // paged: the scales come with the tile
                bool v;
                const int64_t slot = key_slot(par + 2 * j, v);
                if (slot >= 0) tc::cp_async4(tc::saddr(my_ring + (j % kKsRing) * kTcTile),
                                             a.k_scales + slot);
                tc::cp_async_commit();
            }
        };
        // tiles j .. j+kKsRing-2 are in flight when tile j is consumed; the copy for
        // tile j+kKsRing-1 then goes to the slot read one tile earlier
#pragma unroll 1
        for (int j = 0; j < kKsRing - 1; j++) ring_issue(j);
        for (int i = par; i < my_tiles; i += 2) {
            const int acc = i & (p.nacc - 1);     // same parity as i: this group's
            const int j = (i - par) >> 1;
            const int sk = (tile_begin + i) * kTcTile + row;
            bool valid;
            const int64_t slot_i = key_slot(i, valid);
            (void)slot_i;
            if (!valid && sk < nv_max) report(a.status, CSA_ERR_BOUNDS);
            float kscale = 1.0f;
            if constexpr (FMT != CSA_FMT_BF16 && !kPaged) {
                tc::cp_async_wait<kKsRing - 2>();
                kscale = valid ? my_ring[(j % kKsRing) * kTcTile] : 0.0f;
                ring_issue(j + kKsRing - 1);
            }
            // the other group's tile is being reduced meanwhile: sleep in the wait
            if (!tc::mbar_wait_sleep(tc::saddr(&tfull[acc]), (uint32_t)((i / p.nacc) & 1),
                                     abort_flag)) {
                if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc::fence_after_sync();
            if constexpr (kPaged) {
                // the key's row scale from the tile's records (their copy has
                // completed: observed again here), then the stage is free
                const int s = i % p.stages;
                tc::mbar_wait(tc::saddr(&sfull[s]), (uint32_t)((i / p.stages) & 1), abort_flag);
                const int r = row & 63;
                kscale = valid ? *reinterpret_cast<const float *>(
                                     stage_buf + s * kStage + (row >> 6) * kRec + (r >> 3) * kGb +
                                     9 * RB + (r & 7) * 4)
                               : 0.0f;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(tc::saddr(&empty[s]));
            }
            // per query row x_lo + x of the group: sum_j w'[c+j] * ReLU(acc[c+j])
            // over its hi_pad columns (a multiple of 16)
            float out[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t ta = tmem_base + lane_addr + (uint32_t)(acc * p.n);
            if (p.hi_pad % 32 == 0) {
                // 16-column TMEM loads, double-buffered: the load of the next
                // 16 columns is in flight while these are reduced
                uint32_t va[16], vb[16];
                tc::tmem_ld16_nowait(ta + (uint32_t)c_lo, va);
                tc::tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 4; x++) {
                    if (x >= qh) break;
                    const int ce = c_lo + (x + 1) * p.hi_pad;
                    float2 sx[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    for (int c = ce - p.hi_pad; c < ce; c += 32) {
                        tc::tmem_ld16_nowait(ta + (uint32_t)(c + 16), vb);
                        relu_dot16(va, w_s + c, sx);
                        tc::tmem_wait_ld();
                        if (c + 32 < c_hi) tc::tmem_ld16_nowait(ta + (uint32_t)(c + 32), va);
                        relu_dot16(vb, w_s + c + 16, sx);
                        tc::tmem_wait_ld();
                    }
                    out[x] = (sx[0].x + sx[1].x) + (sx[0].y + sx[1].y);
                }
            } else {
#pragma unroll
                for (int x = 0; x < 4; x++) {
                    if (x >= qh) break;
                    const int cb = c_lo + x * p.hi_pad, ce = cb + p.hi_pad;
                    float2 sx[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    for (int c = cb; c < ce; c += 16) {
                        uint32_t v[16];
                        tc::tmem_ld16_nowait(ta + (uint32_t)c, v);
                        tc::tmem_wait_ld();
                        relu_dot16(v, w_s + c, sx);
                    }
                    out[x] = (sx[0].x + sx[1].x) + (sx[0].y + sx[1].y);
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::saddr(&tempty[acc]));
            if (valid) {
#pragma unroll
                for (int x = 0; x < 4; x++)
                    if (x < qh && x_lo + x < nq && sk < nv_s[x_lo + x])
                        lg[(int64_t)(t0 + x_lo + x) * a.logits_stride + sk] = out[x] * kscale;
            }
        }
        tc::cp_async_wait<0>();     // no copy into the ring outlives the loop
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) {
        __syncwarp();
        tc::tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
    }
    if constexpr (EG == 2) {    // the fused plans use two epilogue groups
    if (sel.cand_key == nullptr || *abort_flag) return;
    // ---- fused top-512 of this CTA's chunk, per query row of the group: the
    // logits just written (visible to the block after the barrier above, and
    // still in L2) come back into the drained stage buffers; the chunk's
    // candidates go to the workspace for the row-level merge
    uint32_t *skeys = reinterpret_cast<uint32_t *>(stage_buf);
    TkSharedT<kTcThreads> &tsh = *reinterpret_cast<TkSharedT<kTcThreads> *>(
        stage_buf + (size_t)p.tiles_per_cta * kTcTile * 4);
    const int k0 = tile_begin * kTcTile;
    for (int x = 0; x < nq; x++) {
        const int len = min(tile_end * kTcTile, nv_s[x]) - k0;
        if (len <= 0) continue;                    // uniform over the CTA
        stage_row_keys<kTcThreads>(skeys, a.logits + (int64_t)(t0 + x) * a.logits_stride + k0,
                                   len);
        __syncthreads();
        const int64_t c = (int64_t)(t0 + x) * sel.max_chunks + blockIdx.x;
        select_chunk<kTcThreads>(skeys, len, k0, sel.cand_key + c * kTopK, sel.cand_idx + c * kTopK,
                                 sel.chunk_info + c, tsh, a.status);
        __syncthreads();
    }
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// Tensor map over paged FP4 records as rows of 256 bytes (a record of
// rec_bytes = 256 * r is one box of r rows, unswizzled).
static bool make_record_map(CUtensorMap *m, const void *codes, int64_t num_pages, int rec_bytes) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {256, (cuuint64_t)(num_pages * (rec_bytes / 256))};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {256, (cuuint32_t)(rec_bytes / 256)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over the index-key codes as a [num_slots, row_bytes] byte matrix,
// 64-row boxes of one swizzle span.
static bool make_key_map(CUtensorMap *m, const void *codes, int64_t num_slots, int row_bytes) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const int span = row_bytes >= 128 ? 128 : row_bytes;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)num_slots};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)span, 64};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = span == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : span == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_32B;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t tc_smem_bytes(int rb, bool fp4, bool paged, const TcParams &p, int eg) {
    const size_t ks = rb / 32;
    const size_t stage = paged ? 2 * 8 * (9 * (size_t)rb + 32) : (size_t)kTcTile * rb;
    return 1024 + (size_t)p.stages * stage + (((size_t)p.n * rb + 1023) & ~(size_t)1023) +
           (fp4 ? (p.stages + 1) * ks * 512 +
                      (rb == 32 && !paged ? (size_t)kSfSlots * 16 * rb : 0) : 0) +
           256 * 4 + 16 * 4 +
           (3 * p.stages + 2 * p.nacc + 1) * 8 + 32 +
           (size_t)2 * p.tiles_per_cta * 4 + 16 + (size_t)eg * kKsRing * kTcTile * 4;
}

bool indexer_tc_supported(const IndexerArgs &a) {
    const bool fmt_ok = (a.dim == 64 || a.dim == 128) &&
                        (a.fmt == CSA_FMT_FP8 || a.fmt == CSA_FMT_BF16 || a.fmt == CSA_FMT_FP4 ||
                         a.fmt == CSA_FMT_FP4_PAGE);
    // FP4 key block scales are copied in 16-byte chunks (paged: inside the
    // 16-byte aligned records), query ones four at a time
    const bool sf_ok = (a.fmt != CSA_FMT_FP4 ||
                        (reinterpret_cast<uintptr_t>(a.k_block_scales) % 16) == 0) &&
                       ((a.fmt != CSA_FMT_FP4 && a.fmt != CSA_FMT_FP4_PAGE) ||
                        (reinterpret_cast<uintptr_t>(a.q_block_scales) % 4) == 0);
    return fmt_ok && sf_ok && a.heads <= 128 && (a.num_slots % kC4Page) == 0 &&
           a.num_slots >= kC4Page && (reinterpret_cast<uintptr_t>(a.k_codes) % 16) == 0 &&
           encode_fn() != nullptr;
}

// Launch shape of the tensor-core indexer.  `fuse`: each CTA also selects its
// chunk's top-512, so a chunk (tiles_per_cta tiles) must hold 512..8192 keys
// (fewer only when the whole row is one chunk) and its logits must fit the
// drained stage buffers next to the selection's shared state.
struct TcPlan {
    TcParams p;
    int rb, chunks;
    int eg;            // epilogue groups: 4 where 256-column accumulators split by query rows
    size_t smem;
};

static TcPlan plan_tc(const IndexerArgs &a, bool fuse) {
    TcPlan pl;
    TcParams &p = pl.p;
    const bool paged = a.fmt == CSA_FMT_FP4_PAGE;
    const bool fp4 = a.fmt == CSA_FMT_FP4 || paged;
    const int rb = a.fmt == CSA_FMT_FP8 ? a.dim : fp4 ? a.dim / 2 : 2 * a.dim;
    pl.rb = rb;
    p.hi_pad = (a.heads + 15) / 16 * 16;
    // queries of one request share the key tiles: group up to 4 of them
    // (N <= 128) when requests carry several query rows, N <= 256 when they
    // carry many (a prefill chunk: each key tile read from L2 then feeds
    // twice the MMA work; the two accumulators fill TMEM, one CTA per SM)
    const int n_max = (!fuse && !fp4 && a.num_q >= 8 * a.bs) ? 256 : 128;
    p.qg = a.num_q <= a.bs ? 1 : n_max / p.hi_pad;
    if (p.qg < 1) p.qg = 1;
    if (p.qg > 4) p.qg = 4;
    // (FP4 query groups stay within N = 128: the block-scaled MMA's query
    // scale factors are laid out for 128 columns)
    if (fp4 && p.qg * p.hi_pad > 128) p.qg = p.hi_pad >= 128 ? 1 : 128 / p.hi_pad;
    p.n = p.qg * p.hi_pad;
    // four epilogue groups (two per accumulator, each reducing half of the
    // query rows) for the wide accumulators
    pl.eg = (p.n > 128 && p.qg % 2 == 0) ? 4 : 2;
    // as many accumulators in flight (up to 8) as keep the CTA within 256 TMEM
    // columns (two CTAs per SM): the MMA of tile i waits for the epilogue of
    // tile i - nacc, so a deeper ring hides the hand-off latency of small tiles
    auto tmem_need = [&](int nacc) { return nacc * p.n + (fp4 ? (nacc * 4 + 4) * (rb / 32) : 0); };
    p.nacc = 2;
    while (p.nacc < 8 && tmem_need(2 * p.nacc) <= 256) p.nacc *= 2;
    int cols = 32;
    const int need = tmem_need(p.nacc);
    while (cols < need) cols <<= 1;
    p.tmem_cols = cols;
    p.num_pages = (int)(a.num_slots / kC4Page);
    // 64-80 KB of key tiles in flight per CTA, two CTAs per SM
    p.stages = rb == 256 ? 3 : rb == 128 ? 5 : rb == 64 ? 8 : 16;
    if (p.tmem_cols > 256) p.stages = p.n * rb > 16384 ? 2 * p.stages - 1 : 2 * p.stages;  // one CTA per SM
    const int tiles_max = (a.max_c4_len + kTcTile - 1) / kTcTile;
    const int groups = query_groups_bound(a.num_q, a.bs, p.qg);
    // one wave: at most (SMs x resident CTAs per SM) CTAs, split evenly over
    // the query groups (a second, nearly empty wave would double the time)
    int sms = 148;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    p.tiles_per_cta = fuse ? 64 : tiles_max;          // upper bound for the estimate
    // 228 KB of shared memory per SM, 1 KB of it reserved per resident CTA
    const size_t smem_est = tc_smem_bytes(rb, fp4, paged, p, pl.eg) + 1024;
    int by_smem = (int)((228 * 1024) / smem_est);
    int ctas_per_sm = 512 / cols;
    if (by_smem < ctas_per_sm) ctas_per_sm = by_smem;
    if (ctas_per_sm > 2) ctas_per_sm = 2;             // register budget: 320 threads x 102
    if (ctas_per_sm < 1) ctas_per_sm = 1;
    const int target = sms * ctas_per_sm;
    int chunks = target / groups;
    if (chunks > tiles_max) chunks = tiles_max;
    if (chunks < 1) chunks = 1;
    p.tiles_per_cta = (tiles_max + chunks - 1) / chunks;
    // when the query groups alone do not fill the wave, rows are split; keep
    // the pieces at most 64 tiles so that rows of very different lengths
    // (a ragged batch sized by its longest row) still spread over the SMs
    if (groups < target && p.tiles_per_cta > 64) p.tiles_per_cta = 64;
    if (fuse) {
        // 512..8192 keys per chunk (the logits of a chunk, 32 KB at most, and
        // the selection state fit in the >= 64 KB of stage buffers)
        if (p.tiles_per_cta > 64) p.tiles_per_cta = 64;
        if (p.tiles_per_cta < 4) p.tiles_per_cta = tiles_max < 4 ? tiles_max : 4;
        if (p.tiles_per_cta < 1) p.tiles_per_cta = 1;
    }
    pl.chunks = (tiles_max + p.tiles_per_cta - 1) / p.tiles_per_cta;
    if (pl.chunks < 1) pl.chunks = 1;
    pl.smem = tc_smem_bytes(rb, fp4, paged, p, pl.eg);
    return pl;
}

// The fused launch is used where the plain launch's pieces are at most 64
// tiles (the fused plan then only merges pieces below 4 tiles); elsewhere
// (long rows per query group, e.g. chunked prefill) the plain indexer and the
// two-stage top-k run.
bool indexer_topk_fuses(const IndexerArgs &a) {
    if (!indexer_tc_supported(a)) return false;
    return plan_tc(a, false).p.tiles_per_cta <= 64;
}

static cudaError_t launch_tc_plan(const IndexerArgs &a, const TcPlan &pl, const TcSelect &sel,
                                  cudaStream_t s) {
    CUtensorMap map{};
    if (a.fmt == CSA_FMT_FP4_PAGE) {
        if (!make_record_map(&map, a.k_codes, a.num_slots / kC4Page, 72 * pl.rb + 256))
            return cudaErrorInvalidValue;
    } else if (!make_key_map(&map, a.k_codes, a.num_slots, pl.rb)) {
        return cudaErrorInvalidValue;
    }
    const TcParams p = pl.p;
    const size_t smem = pl.smem;
    dim3 grid(pl.chunks, query_groups_bound(a.num_q, a.bs, p.qg));
    const bool fp4 = a.fmt == CSA_FMT_FP4;
    const bool paged = a.fmt == CSA_FMT_FP4_PAGE;
    const int rb = pl.rb;
#define CSA_TC_EG(F, R, E)                                                                  \
    do {                                                                                    \
        static int done[64] = {0};                                                          \
        cudaError_t e = ensure_max_smem((const void *)indexer_tc_kernel<F, R, E>, 227 * 1024, done); \
        if (e != cudaSuccess) return e;                                                     \
        launch_k(indexer_tc_kernel<F, R, E>, grid, tc_threads<E>(), smem, s, a, map, p, sel); \
    } while (0)
#define CSA_TC(F, R)                                                                        \
    do {                                                                                    \
        if (pl.eg == 4) CSA_TC_EG(F, R, 4);                                                 \
        else CSA_TC_EG(F, R, 2);                                                            \
    } while (0)
    if (a.fmt == CSA_FMT_FP8 && rb == 128) CSA_TC(CSA_FMT_FP8, 128);
    else if (a.fmt == CSA_FMT_FP8) CSA_TC(CSA_FMT_FP8, 64);
    else if (paged && rb == 64) CSA_TC_EG(CSA_FMT_FP4_PAGE, 64, 2);
    else if (paged) CSA_TC_EG(CSA_FMT_FP4_PAGE, 32, 2);
    else if (fp4 && rb == 64) CSA_TC_EG(CSA_FMT_FP4, 64, 2);
    else if (fp4) CSA_TC_EG(CSA_FMT_FP4, 32, 2);
    else if (rb == 128) CSA_TC(CSA_FMT_BF16, 128);
    else CSA_TC(CSA_FMT_BF16, 256);
#undef CSA_TC
#undef CSA_TC_EG
    return cudaGetLastError();
}

cudaError_t launch_indexer_tc(const IndexerArgs &a, cudaStream_t s) {
    const TcSelect none = {nullptr, nullptr, nullptr, 0};
    return launch_tc_plan(a, plan_tc(a, false), none, s);
}

// Candidates + chunk pairs of the fused launch for this shape (the plan reads
// only the shape fields of `a`: format, dim, heads, num_q, bs, max_c4_len).
size_t indexer_topk_fused_bytes(const IndexerArgs &a) {
    const TcPlan pl = plan_tc(a, true);
    return (size_t)a.num_q * pl.chunks * (kTopK * 8 + sizeof(uint2));
}

static TcSelect select_layout(const TcPlan &pl, int num_q, void *workspace) {
    const size_t nc = (size_t)num_q * pl.chunks;
    TcSelect sel;
    sel.cand_key = (uint32_t *)workspace;
    sel.cand_idx = (int32_t *)((uint8_t *)workspace + nc * kTopK * 4);
    sel.chunk_info = (uint2 *)((uint8_t *)workspace + nc * kTopK * 8);
    sel.max_chunks = pl.chunks;
    return sel;
}

cudaError_t launch_indexer_select(const IndexerArgs &a, void *workspace, cudaStream_t s) {
    const TcPlan pl = plan_tc(a, true);
    return launch_tc_plan(a, pl, select_layout(pl, a.num_q, workspace), s);
}

cudaError_t launch_topk_merge(const IndexerArgs &shape, const TopkArgs &t, cudaStream_t s) {
    const TcPlan pl = plan_tc(shape, true);
    const TcSelect sel = select_layout(pl, t.num_q, t.workspace);
    return launch_topk_stage2(t, pl.chunks, pl.p.tiles_per_cta * kTcTile, sel.cand_key,
                              sel.cand_idx, sel.chunk_info, s);
}

cudaError_t launch_indexer_topk_fused(const IndexerArgs &a, const TopkArgs &t, cudaStream_t s) {
    cudaError_t e = launch_indexer_select(a, t.workspace, s);
    if (e != cudaSuccess) return e;
    return launch_topk_merge(a, t, s);
}

}  // namespace csa
