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
//   warps 2-5 epilogue: tcgen05.ld of the key's row, ReLU, head-weighted sum
//           per query, times the key's scale, one coalesced float store.
// Formats: FP8 E4M3 (kind::f8f6f4) and bf16 (kind::f16).  All waits are
// bounded; a timeout records CSA_ERR_TIMEOUT and the CTA unwinds.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace csa {

constexpr int kTcThreads = 192;   // 6 warps
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
};

template <int FMT, int RB>
__global__ void __launch_bounds__(kTcThreads)
indexer_tc_kernel(const IndexerArgs a, const __grid_constant__ CUtensorMap kmap,
                  const TcParams p) {
    using G = TcGeom<RB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: stages | q tile | w' | nv | barriers
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *stage_buf = base;
    uint8_t *q_buf = stage_buf + p.stages * G::kStageBytes;
    float *w_s = reinterpret_cast<float *>(q_buf + ((p.n * RB + 1023) & ~1023));
    int *nv_s = reinterpret_cast<int *>(w_s + 256);
    uint64_t *bars = reinterpret_cast<uint64_t *>(nv_s + 16);
    uint64_t *full = bars, *empty = bars + p.stages, *tfull = bars + 2 * p.stages;
    uint64_t *tempty = tfull + 2, *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- which query group and key tiles (uniform over the CTA)
    const int t0 = blockIdx.y;
    int lo = 0, hi = a.bs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cu_q[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int first = a.cu_q[b], last = a.cu_q[b + 1];
    if (((t0 - first) % p.qg) != 0) return;                 // not a group leader
    const int nq = min(p.qg, last - t0);
    const int cap = min(a.max_c4_len, a.pt_stride * kC4Page);
    int nv_max = 0;
    int nv_q[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        int n = 0;
        if (i < nq) {
            n = a.c4_seq_lens[b];
            if (a.q_pos) n = min(n, (a.q_pos[t0 + i] + 1) / 4);
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
            tc::mbar_init(tc::saddr(&full[s]), 1);
            tc::mbar_init(tc::saddr(&empty[s]), 1);
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(tc::saddr(&tfull[i]), 1);
            tc::mbar_init(tc::saddr(&tempty[i]), 4);
        }
        tc::mbar_init(tc::saddr(drain), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (threadIdx.x < 4) nv_s[threadIdx.x] = nv_q[threadIdx.x];
    // query tile: row n = qi*hi_pad + h (K-major, swizzled like the key tiles)
    {
        const uint8_t *qc = reinterpret_cast<const uint8_t *>(a.q_codes);
        const int chunks16 = RB / 16;
        for (int u = threadIdx.x; u < p.n * chunks16; u += kTcThreads) {
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
        for (int n = threadIdx.x; n < p.n; n += kTcThreads) {
            const int qi = n / p.hi_pad, h = n % p.hi_pad;
            w_s[n] = (qi < nq && h < a.heads) ? a.q_weights[(int64_t)(t0 + qi) * a.heads + h] : 0.f;
        }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < my_tiles; i++) {
                const int s = i % p.stages;
                const uint32_t ph = (uint32_t)((i / p.stages) & 1);
                if (!tc::mbar_wait(tc::saddr(&empty[s]), ph ^ 1u, abort_flag)) {
                    if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                tc::mbar_expect_tx(tc::saddr(&full[s]), G::kStageBytes);
                const int tile = tile_begin + i;
#pragma unroll
                for (int half = 0; half < 2; half++) {
                    const int pidx = tile * 2 + half;
                    int page = 0;
                    if (pidx * kC4Page < nv_max && pidx < a.pt_stride) page = pt_row[pidx];
                    if (page < 0 || page >= p.num_pages) page = 0;   // epilogue reports visible keys
#pragma unroll
                    for (int c = 0; c < G::kChunks; c++)
                        tc::tma_load_2d(tc::saddr(stage_buf + s * G::kStageBytes +
                                                  c * kTcTile * G::kSpan + half * 64 * G::kSpan),
                                        &kmap, c * G::kSpan, page * kC4Page,
                                        tc::saddr(&full[s]));
                }
                issued++;
            }
            // before leaving, every load issued must have landed
            for (int i = max(0, issued - p.stages); i < issued; i++)
                tc::mbar_wait(tc::saddr(&full[i % p.stages]), (uint32_t)((i / p.stages) & 1), nullptr);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = FMT == CSA_FMT_FP8 ? tc::idesc_m128(0, 0, p.n)
                                                      : tc::idesc_m128(1, 1, p.n);
            for (int i = 0; i < my_tiles; i++) {
                const int s = i % p.stages;
                const int acc = i & 1;
                if (!tc::mbar_wait(tc::saddr(&full[s]), (uint32_t)((i / p.stages) & 1), abort_flag) ||
                    !tc::mbar_wait(tc::saddr(&tempty[acc]), (uint32_t)(((i >> 1) & 1) ^ 1),
                                   abort_flag)) {
                    if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d = tmem_base + (uint32_t)(acc * p.n);
                const uint32_t sa = tc::saddr(stage_buf + s * G::kStageBytes);
                const uint32_t sb = tc::saddr(q_buf);
#pragma unroll
                for (int k = 0; k < G::kKSteps; k++) {
                    const int c = (k * 32) / G::kSpan, off = (k * 32) % G::kSpan;
                    const uint64_t ad = tc::kmajor_desc(sa + c * kTcTile * G::kSpan + off, G::kSpan);
                    const uint64_t bd = tc::kmajor_desc(sb + c * p.n * G::kSpan + off, G::kSpan);
                    if (FMT == CSA_FMT_FP8) tc::mma_f8f6f4(d, ad, bd, idesc, k > 0);
                    else tc::mma_f16(d, ad, bd, idesc, k > 0);
                }
                tc::mma_commit(tc::saddr(&empty[s]));
                tc::mma_commit(tc::saddr(&tfull[acc]));
            }
            // drain: every MMA issued has completed before TMEM is released
            tc::mma_commit(tc::saddr(drain));
            tc::mbar_wait(tc::saddr(drain), 0, nullptr);
        }
    } else {
        // ---------------- epilogue (warps 2-5 cover the four TMEM lane quadrants)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *lg = a.logits;
        for (int i = 0; i < my_tiles; i++) {
            const int acc = i & 1;
            const int tile = tile_begin + i;
            const int sk = tile * kTcTile + row;
            float kscale = 0.0f;
            bool valid = false;
            if (sk < nv_max) {
                const int32_t page = pt_row[sk / kC4Page];
                const int64_t slot = (int64_t)page * kC4Page + sk % kC4Page;
                valid = page >= 0 && slot < a.num_slots && page < p.num_pages;
                if (!valid) report(a.status, CSA_ERR_BOUNDS);
                else kscale = FMT == CSA_FMT_BF16 ? 1.0f : a.k_scales[slot];
            }
            if (!tc::mbar_wait(tc::saddr(&tfull[acc]), (uint32_t)((i >> 1) & 1), abort_flag)) {
                if (!*abort_flag) report(a.status, CSA_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc::fence_after_sync();
            float out[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t ta = tmem_base + lane_addr + (uint32_t)(acc * p.n);
            for (int c0 = 0; c0 < p.n; c0 += 16) {
                float v[16];
                tc::tmem_ld16(ta + (uint32_t)c0, v);
                float sacc = 0.0f;
#pragma unroll
                for (int j = 0; j < 16; j++) sacc = fmaf(w_s[c0 + j], fmaxf(v[j], 0.0f), sacc);
                const int qi = c0 / p.hi_pad;
#pragma unroll
                for (int x = 0; x < 4; x++)
                    if (x == qi) out[x] += sacc;
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::saddr(&tempty[acc]));
            if (valid) {
#pragma unroll
                for (int x = 0; x < 4; x++)
                    if (x < nq && sk < nv_s[x])
                        lg[(int64_t)(t0 + x) * a.logits_stride + sk] = out[x] * kscale;
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) {
        __syncwarp();
        tc::tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
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

static size_t tc_smem_bytes(int rb, const TcParams &p) {
    return 1024 + (size_t)p.stages * kTcTile * rb + (((size_t)p.n * rb + 1023) & ~(size_t)1023) +
           256 * 4 + 16 * 4 + (2 * p.stages + 5) * 8 + 16;
}

bool indexer_tc_supported(const IndexerArgs &a) {
    const bool fmt_ok = (a.fmt == CSA_FMT_FP8 && (a.dim == 64 || a.dim == 128)) ||
                        (a.fmt == CSA_FMT_BF16 && (a.dim == 64 || a.dim == 128));
    return fmt_ok && a.heads <= 128 && (a.num_slots % kC4Page) == 0 && a.num_slots >= kC4Page &&
           (reinterpret_cast<uintptr_t>(a.k_codes) % 16) == 0 && encode_fn() != nullptr;
}

cudaError_t launch_indexer_tc(const IndexerArgs &a, cudaStream_t s) {
    const int rb = a.fmt == CSA_FMT_FP8 ? a.dim : 2 * a.dim;
    TcParams p;
    p.hi_pad = (a.heads + 15) / 16 * 16;
    // queries of one request share the key tiles: group up to 4 of them
    // (N <= 128) when requests carry several query rows
    p.qg = a.num_q <= a.bs ? 1 : 128 / p.hi_pad;
    if (p.qg < 1) p.qg = 1;
    if (p.qg > 4) p.qg = 4;
    p.n = p.qg * p.hi_pad;
    int cols = 32;
    while (cols < 2 * p.n) cols <<= 1;
    p.tmem_cols = cols;
    p.num_pages = (int)(a.num_slots / kC4Page);
    p.stages = rb >= 128 ? 4 : 6;
    const int tiles_max = (a.max_c4_len + kTcTile - 1) / kTcTile;
    const int groups = (a.num_q + p.qg - 1) / p.qg;
    const int ctas_per_sm = 512 / cols < 3 ? 512 / cols : 3;
    const int target = 148 * ctas_per_sm;
    int chunks = (target + groups - 1) / groups;
    if (chunks > tiles_max) chunks = tiles_max;
    if (chunks < 1) chunks = 1;
    p.tiles_per_cta = (tiles_max + chunks - 1) / chunks;
    chunks = (tiles_max + p.tiles_per_cta - 1) / p.tiles_per_cta;

    CUtensorMap map;
    if (!make_key_map(&map, a.k_codes, a.num_slots, rb)) return cudaErrorInvalidValue;
    const size_t smem = tc_smem_bytes(rb, p);
    dim3 grid(chunks, a.num_q);
#define CSA_TC(F, R)                                                                        \
    do {                                                                                    \
        static int done[64] = {0};                                                          \
        cudaError_t e = ensure_max_smem((const void *)indexer_tc_kernel<F, R>, 200 * 1024, done); \
        if (e != cudaSuccess) return e;                                                     \
        indexer_tc_kernel<F, R><<<grid, kTcThreads, smem, s>>>(a, map, p);                  \
    } while (0)
    if (a.fmt == CSA_FMT_FP8 && rb == 128) CSA_TC(CSA_FMT_FP8, 128);
    else if (a.fmt == CSA_FMT_FP8) CSA_TC(CSA_FMT_FP8, 64);
    else if (rb == 128) CSA_TC(CSA_FMT_BF16, 128);
    else CSA_TC(CSA_FMT_BF16, 256);
#undef CSA_TC
    return cudaGetLastError();
}

}  // namespace csa
