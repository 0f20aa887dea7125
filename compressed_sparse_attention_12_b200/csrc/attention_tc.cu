// attention_tc.cu -- step 4 on the fifth-generation tensor cores: sparse MQA
// over FP8 KV rows for 64 query heads per CTA
// ("Token 的一生：DSV4 架构与 DSpark" §1: attention reads only the 512 selected
// compressed rows; "DeepSeek-V4 的交錯壓縮注意力（CSA/HCA）", section
// "Compressed Sparse Attention（CSA）": the sliding window of raw rows shares
// one softmax with them; section "低精度與儲存策略的配合": FP8 latent with
// BF16 RoPE dims; section "Heavily Compressed Attention（HCA）": the same
// kernel in dense mode reads every visible HCA row).
//
// For query t, head h and the query's row list r (selected compressed rows,
// or every visible HCA row, then the window's raw rows):
//   z = sm_scale * q_h . k_r over 576 dims,  out_h = softmax(z) V,  V = 512 latent dims.
//
// One CTA owns one query, 64 heads (M = 64 of every MMA) and one split of the
// row list, in tiles of 32 rows.  Warp roles:
//   warp 17    producer: one bulk copy (TMA engine) per packed FP8 row (656
//              bytes) of a tile into a two-stage staging ring; the query's 64
//              bf16 rows arrive the same way before the wait on the preceding
//              kernel;
//   warps 8-15 converters: turn a staged tile into fp16 in the
//              128-byte-swizzled K-major layout -- E4M3 codes exactly
//              (hardware conversion), RoPE times a power of two per row --
//              keeping each row's four block scales in fp32;
//   warp 16    one thread issues tcgen05.mma: S_b = Q K_b^T for the four
//              latent blocks b and the RoPE part, each into its own TMEM
//              accumulator so every row's block scale multiplies its own
//              partial sum in fp32; then O_b += P_b V_b with V read from the
//              same tile as an MN-major operand;
//   warps 0-7  softmax, two warpgroups: thread = (head, 8 of the tile's rows);
//              combine the five partial scores with the row scales (the
//              tile maximum of a head is exchanged between the warpgroups
//              through shared memory), online softmax in
//              base 2 (the running maximum is raised only when a tile exceeds
//              it by 2^8, and only then is O rescaled in TMEM), and write
//              P_b = p x block scale x (power-of-two normaliser) as fp16 for
//              each latent block.
// S is double-buffered in TMEM (the two M = 64 accumulators of a lane
// quarter), the staged rows, the fp16 tile and P double-buffered in shared
// memory, so the softmax of tile j overlaps the score MMAs of tile j+1, the
// conversion of tile j+2 and the copies of tile j+3.
// The splits of one query form a thread-block cluster and merge their
// partial outputs inside the kernel, through distributed shared memory (no
// second kernel).
#include "attention.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kTcRows = 32;                                     // key rows per tile
constexpr int kTcHeads = 64;                                    // query heads per CTA
constexpr int kTcBufs = 2;                                      // fp16 tile buffers
constexpr int kTcStages = 2;                                    // staged-row buffers
constexpr int kTcSoft = 256;                                    // softmax threads (warps 0-7)
constexpr int kTcConv = 256;                                    // converter threads (warps 8-15)
constexpr int kTcMmaWarp = 16;
constexpr int kTcProdWarp = 17;
constexpr int kTcThreads = 32 * (kTcProdWarp + 1);              // 576
constexpr int kTcMaxSplits = 8;                                 // portable cluster size
constexpr int kTcQAtom = kTcHeads * 128;                        // 64 dims of Q: 8 KB
constexpr int kTcQBytes = 9 * kTcQAtom;
constexpr int kTcAtom = kTcRows * 128;                          // 64 dims of a tile: 4 KB
constexpr int kTcTileBytes = 9 * kTcAtom;
constexpr int kTcPBlock = kTcHeads * kTcRows * 2;               // one latent block of P: 4 KB
constexpr int kTcPBytes = 4 * kTcPBlock;
constexpr int kTcTileOff = kTcQBytes;
constexpr int kTcPOff = kTcTileOff + kTcBufs * kTcTileBytes;
constexpr int kTcStageBytes = kTcRows * kFp8RowBytes;           // 32 packed rows: 20992 B
constexpr int kTcStageOff = kTcPOff + 2 * kTcPBytes;
constexpr int kTcMiscOff = kTcStageOff + kTcStages * kTcStageBytes;
constexpr uint32_t kTcOCol = 160;              // O: TMEM columns 160..415, both lane halves
constexpr float kTcRaise = 8.0f;               // log2 headroom of p before the maximum is raised
constexpr float kTcLog2e = 1.4426950408889634f;

// the split merge's fp16 slices (64 heads x 512/splits dims each): the
// splits-1 receive slots at the end of the buffers and at least one outgoing
// slice below them
static_assert(kTcHeads * kLatent * 2 <= kTcMiscOff,
              "the split merge's slices fit in the CTA's buffers");
static_assert(kTcBufs * kTcTileBytes == kTcHeads * kKvDim * 2,
              "the query's bf16 rows are staged in the tile buffers");

struct TcMisc {
    float4 sc[kTcBufs][kTcRows];     // per row: the 4 block scales (0: masked)
    float ropef[kTcBufs][kTcRows];   // per row: the RoPE factor (0: masked)
    float smax[kTcBufs];             // largest block scale of the tile
    uint32_t vmask[kTcBufs];         // bit r: row r of the tile is live
    float qmul[kTcHeads];            // power of two applied to each head's query row
    float ml[kTcMaxSplits][kTcHeads][2];   // (running max, sum) per split and head (merge)
    float fct[kTcHeads];             // per head, this split's factor in the merged output
    float vmax[kTcMaxSplits];        // per split: the largest block scale of its rows (merge)
    float vrun;                      // largest block scale of the tiles converted so far
    union {
        float qpart[kTcHeads][6];    // set-up: per head, the largest |q| of each sixth of the row
        float mx[2][2][kTcHeads];    // main loop: tile maximum per (tile parity, warpgroup, head)
    };
    float lx[2][kTcHeads];           // row sums per (warpgroup, head) at the end
    uint64_t tile_full[kTcBufs], tile_free[kTcBufs];
    uint64_t s_full[2], s_free[2], p_full[2];
    uint64_t o_done, o_last, drain;
    uint32_t tmem_slot;
    uint32_t live[kTcStages];        // bit r: row r of the staged tile was copied
    uint64_t q_full, stage_full[kTcStages], stage_free[kTcStages], recv_full;
    int32_t abort;
};
constexpr size_t kTcSmem = 1024 + kTcMiscOff + sizeof(TcMisc);
static_assert(kTcSmem <= 232448, "shared memory per CTA");

constexpr int32_t kRawFlag = 1 << 30;

__host__ __device__ constexpr uint32_t tc_idesc_f16(int m, int n, bool b_mn) {
    return (1u << 4) | (b_mn ? (1u << 16) : 0u) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

// Descriptor of a 128-byte-swizzled MN-major operand: 64-element atoms along
// N `lbo` bytes apart, 8-row groups along K `sbo` bytes apart.
__device__ __forceinline__ uint64_t tc_mn_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((addr & 0x3FFFF) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// A descriptor moved `bytes` further along shared memory (the start address
// field holds address / 16 in its low 14 bits; no carry for addresses within
// the 228 KB of shared memory).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
    return d + (uint64_t)(bytes >> 4);
}

// 16 lanes x 8 columns, twice: threads 0-15 read columns [c, c+8) and
// threads 16-31 columns [c+16, c+24) of the same 16 lanes; no wait.
__device__ __forceinline__ void tmem_ld_16x32bx2_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Bulk copy (TMA engine) of `bytes` from this CTA's shared memory to the
// shared memory of CTA `dst` of the cluster (`dst_addr`, `bar` mapped into
// it), completing as transaction bytes on that CTA's mbarrier.
__device__ __forceinline__ void bulk_s2s_cluster(uint32_t dst_addr, uint32_t src, uint32_t bytes,
                                                 uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst_addr), "r"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Waits until every bulk copy this thread issued has read its source.
__device__ __forceinline__ void bulk_commit_wait_read() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_16x32bx2_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], 16;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr));
}

// 2^x by the hardware approximation (x = -inf gives +0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Named barrier of the softmax warpgroups (warps 0-7).
__device__ __forceinline__ void softmax_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kTcSoft) : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Four E4M3 codes -> two fp16 pairs (exact: every E4M3 value is an fp16
// value); byte i of w becomes element i.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float a) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(a) : "memory");
}

__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float a, float b) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b)
                 : "memory");
}

// Every thread of every CTA of the cluster arrives; writes before it are
// visible to reads after it anywhere in the cluster.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Bounded wait on one phase (the waiting thread sleeps between tries); on
// failure the first thread to give up records CSA_ERR_TIMEOUT and raises the
// CTA's abort flag.
__device__ __forceinline__ bool tc_wait(TcMisc &ms, uint64_t &bar, uint32_t parity,
                                        const AttnArgs &a) {
    if (tc::mbar_wait_sleep(tc::saddr(&bar), parity, &ms.abort)) return true;
    if (atomicExch(&ms.abort, 1) == 0) report(a.status, CSA_ERR_TIMEOUT);
    return false;
}

// The same for a whole warp (lane 0 waits; the outcome is the warp's).
__device__ __forceinline__ bool tc_warp_wait(TcMisc &ms, uint64_t &bar, uint32_t parity,
                                             const AttnArgs &a) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = tc_wait(ms, bar, parity, a) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__device__ __forceinline__ bool tc_aborted(TcMisc &ms) {
    return *reinterpret_cast<volatile int32_t *>(&ms.abort) != 0;
}

// Entry `r` of the query's row list is resolved in two halves so that the
// converters can read the one integer it depends on a tile ahead:
// tc_row_fetch reads it (the selected slot, or the page id of a window or HCA
// row; -1 when there is none), tc_row_code turns it into the row code:
// slot | kRawFlag for raw rows, -1 for masked entries and entries past the
// list.  Out-of-range slots and pages record CSA_ERR_BOUNDS and are masked.
__device__ __forceinline__ int32_t tc_row_fetch(const AttnArgs &a, const AtQuery &qq, int t,
                                                int r) {
    if (r < qq.nsel) {
        if (a.dense_ratio == 0) return a.idx[(int64_t)t * kTopK + r];
        const int rpp = kPage / a.dense_ratio;
        return r / rpp < a.pt_stride ? a.page_table[(int64_t)qq.b * a.pt_stride + r / rpp] : -1;
    }
    if (r - qq.nsel >= qq.nw) return -1;
    const int pos = qq.p - qq.nw + 1 + (r - qq.nsel);
    return pos / kPage < a.pt_stride ? a.page_table[(int64_t)qq.b * a.pt_stride + pos / kPage]
                                     : -1;
}

__device__ __forceinline__ int32_t tc_row_code(const AttnArgs &a, const AtQuery &qq, int r,
                                               int32_t v) {
    if (r < qq.nsel) {
        if (a.dense_ratio == 0) {
            if (v >= a.num_c4_slots) {
                report(a.status, CSA_ERR_BOUNDS);
                return -1;
            }
            return v < 0 ? -1 : v;
        }
        const int rpp = kPage / a.dense_ratio;
        const int64_t slot = (int64_t)v * rpp + r % rpp;
        if (v < 0 || slot >= a.num_c4_slots) {
            report(a.status, CSA_ERR_BOUNDS);
            return -1;
        }
        return (int32_t)slot;
    }
    if (r - qq.nsel >= qq.nw) return -1;
    const int pos = qq.p - qq.nw + 1 + (r - qq.nsel);
    const int64_t slot = (int64_t)v * kPage + pos % kPage;
    if (v < 0 || slot >= a.num_raw_slots) {
        report(a.status, CSA_ERR_BOUNDS);
        return -1;
    }
    return (int32_t)slot | kRawFlag;
}

__device__ __forceinline__ const uint8_t *tc_row_ptr(const AttnArgs &a, int32_t code) {
    const uint8_t *base = reinterpret_cast<const uint8_t *>((code & kRawFlag) ? a.raw_cache
                                                                              : a.c4_cache);
    return base + (int64_t)(code & (kRawFlag - 1)) * kFp8RowBytes;
}

// One tile's rows as read by one converter thread (c = 0..255, warp cw =
// c / 32): latent chunk `lane` (16 codes) of rows cw + 8k, the RoPE chunk (8
// values) of row c / 8, chunk c % 8, and for c < 32 the block scales of row c.
struct TcLoad {
    uint4 lat[4];
    uint4 rope;
    uint4 scale;
    uint32_t live;      // bits 0-3 latent rows, 4 RoPE row, 5 scale row
};

// Reads one staged tile (rows at stage + r * 656; bit r of `live` set when
// row r was copied, masked rows read as zeros).
__device__ __forceinline__ void tc_load(const uint8_t *stage, uint32_t live, int c, TcLoad &L) {
    const int lane = c & 31, cw = c >> 5;
    const uint4 z = make_uint4(0, 0, 0, 0);
    L.live = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const int r = cw + 8 * k;
        const uint4 w = *reinterpret_cast<const uint4 *>(stage + r * kFp8RowBytes + lane * 16);
        const bool on = (live >> r) & 1;
        L.lat[k] = on ? w : z;
        L.live |= (on ? 1u : 0u) << k;
    }
    {
        const int r = c >> 3;
        const uint4 w =
            *reinterpret_cast<const uint4 *>(stage + r * kFp8RowBytes + 528 + (c & 7) * 16);
        const bool on = (live >> r) & 1;
        L.rope = on ? w : z;
        L.live |= (on ? 1u : 0u) << 4;
    }
    L.scale = z;
    if (cw == 0) {
        const uint4 w = *reinterpret_cast<const uint4 *>(stage + lane * kFp8RowBytes + 512);
        const bool on = (live >> lane) & 1;
        L.scale = on ? w : z;
        L.live |= (on ? 1u : 0u) << 5;
    }
}

// Converts one loaded tile into tile buffer `buf` and its per-row factors.
__device__ __forceinline__ void tc_store(const TcLoad &L, int c, uint8_t *tile, TcMisc &ms,
                                         int buf) {
    const int lane = c & 31, cw = c >> 5;
    // latent: row cw + 8k, dims 16*lane .. +15 -> atom lane/4, bytes 32*(lane%4) .. +31;
    // lanes of odd atoms write their second half first (spreads the banks)
    const int atom = lane >> 2;
    const bool odd = (atom & 1) != 0;
    const int byte = (lane & 3) * 32;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const int r = cw + 8 * k;
        uint4 lo, hi;
        e4m3x4_to_f16x4(L.lat[k].x, lo.x, lo.y);
        e4m3x4_to_f16x4(L.lat[k].y, lo.z, lo.w);
        e4m3x4_to_f16x4(L.lat[k].z, hi.x, hi.y);
        e4m3x4_to_f16x4(L.lat[k].w, hi.z, hi.w);
        uint8_t *ab = tile + atom * kTcAtom;
        *reinterpret_cast<uint4 *>(ab + tc::swz(r, byte + (odd ? 16 : 0), 128)) = odd ? hi : lo;
        *reinterpret_cast<uint4 *>(ab + tc::swz(r, byte + (odd ? 0 : 16), 128)) = odd ? lo : hi;
    }
    // RoPE: 8 lanes per row; the row's values times the power of two that
    // brings its largest magnitude into [2^13, 2^14) convert to fp16 exactly
    {
        const int r = c >> 3, ch = c & 7;
        const uint32_t w[4] = {L.rope.x, L.rope.y, L.rope.z, L.rope.w};
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
        *reinterpret_cast<uint4 *>(tile + 8 * kTcAtom + tc::swz(r, ch * 16, 128)) = o;
        if (ch == 0) ms.ropef[buf][r] = (L.live >> 4) & 1 ? 1.0f / m : 0.0f;
    }
    // block scales, live rows, the tile's largest scale
    if (cw == 0) {
        const float4 s = make_float4(__uint_as_float(L.scale.x), __uint_as_float(L.scale.y),
                                     __uint_as_float(L.scale.z), __uint_as_float(L.scale.w));
        ms.sc[buf][lane] = s;
        const float mx = warp_max(fmaxf(fmaxf(s.x, s.y), fmaxf(s.z, s.w)));
        const uint32_t live = __ballot_sync(0xffffffffu, (L.live >> 5) & 1);
        if (lane == 0) {
            ms.smax[buf] = mx;
            ms.vmask[buf] = live;
            ms.vrun = fmaxf(ms.vrun, mx);      // always the same thread
        }
    }
}

__device__ __forceinline__ uint8_t *tiles_stage(uint8_t *base, int st) {
    return base + kTcStageOff + st * kTcStageBytes;
}

__global__ void __launch_bounds__(kTcThreads, 1)
sparse_mqa_tc_kernel(const AttnArgs a, int splits, int tiles_per_split) {
    // Only step inputs (q, cu_q, q_pos, seq_lens) are read before the wait on
    // the preceding kernel: the query rows are converted while it finishes.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *qs = base;
    uint8_t *tiles = base + kTcTileOff;
    uint8_t *ps = base + kTcPOff;
    TcMisc &ms = *reinterpret_cast<TcMisc *>(base + kTcMiscOff);
    const int t = blockIdx.x, hg = blockIdx.y, sp = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == kTcMmaWarp) {
        tc::tmem_alloc(tc::saddr(&ms.tmem_slot), 512);
        if (lane == 0) {
            tc::mbar_init(tc::saddr(&ms.q_full), 1);
            for (int i = 0; i < kTcStages; i++) {
                tc::mbar_init(tc::saddr(&ms.stage_full[i]), 1);
                tc::mbar_init(tc::saddr(&ms.stage_free[i]), kTcConv);
            }
            for (int i = 0; i < kTcBufs; i++) {
                tc::mbar_init(tc::saddr(&ms.tile_full[i]), kTcConv);
                tc::mbar_init(tc::saddr(&ms.tile_free[i]), 1);
            }
            for (int i = 0; i < 2; i++) {
                tc::mbar_init(tc::saddr(&ms.s_full[i]), 1);
                tc::mbar_init(tc::saddr(&ms.s_free[i]), kTcSoft);
                tc::mbar_init(tc::saddr(&ms.p_full[i]), kTcSoft);
            }
            tc::mbar_init(tc::saddr(&ms.o_done), 1);
            tc::mbar_init(tc::saddr(&ms.o_last), 1);
            tc::mbar_init(tc::saddr(&ms.drain), 1);
            tc::mbar_init(tc::saddr(&ms.recv_full), 1);
            ms.abort = 0;
            ms.vrun = 0.0f;
            tc::fence_mbar_init();
        }
    }
    __syncthreads();
    // the query's 64 bf16 rows (73728 contiguous bytes) into the tile buffers
    constexpr uint32_t kQRowBytes = kTcHeads * kKvDim * 2;
    const uint8_t *qsrc = reinterpret_cast<const uint8_t *>(a.q) +
                          ((int64_t)t * a.heads + hg * kTcHeads) * kKvDim * 2;
    if (warp == kTcProdWarp && lane == 0) {
        tc::mbar_expect_tx(tc::saddr(&ms.q_full), kQRowBytes);
        for (uint32_t off = 0; off < kQRowBytes; off += 16384)
            tc::bulk_g2s(tc::saddr(tiles + off), qsrc + off, min(16384u, kQRowBytes - off),
                         tc::saddr(&ms.q_full));
    }
    // the query's request, position and window (step inputs)
    const AtQuery qq = at_query(a, t);
    // Q to fp16, 128-byte-swizzled K-major [9 atoms][64 heads][128 B]: six
    // threads per head (warps 0-11), 96 dims each; each head times the power
    // of two that brings its largest |q| into [2^13, 2^14) (exact for every
    // bf16 value above 2^-30 of that maximum)
    const int qh = tid / 6, qpart = tid % 6;
    uint4 qv[12];
    if (tid < 6 * kTcHeads) {
        tc_warp_wait(ms, ms.q_full, 0, a);
        const uint4 *src = reinterpret_cast<const uint4 *>(tiles + qh * kKvDim * 2 + 192 * qpart);
#pragma unroll
        for (int i = 0; i < 12; i++) qv[i] = src[i];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 12; i++) {
            const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
            for (int j = 0; j < 4; j++)
                amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)),
                                         fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
        }
        ms.qpart[qh][qpart] = amax;
    }
    __syncthreads();
    if (tid < 6 * kTcHeads) {
        float amax = ms.qpart[qh][0];
#pragma unroll
        for (int i = 1; i < 6; i++) amax = fmaxf(amax, ms.qpart[qh][i]);
        const float m = fit_pow2(amax, 14);
#pragma unroll
        for (int i = 0; i < 12; i++) {
            const int g = 12 * qpart + i;              // 8-dim chunk of the row
            const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
            uint4 o;
            o.x = pack_f16(__uint_as_float(w[0] << 16) * m, __uint_as_float(w[0] & 0xFFFF0000u) * m);
            o.y = pack_f16(__uint_as_float(w[1] << 16) * m, __uint_as_float(w[1] & 0xFFFF0000u) * m);
            o.z = pack_f16(__uint_as_float(w[2] << 16) * m, __uint_as_float(w[2] & 0xFFFF0000u) * m);
            o.w = pack_f16(__uint_as_float(w[3] << 16) * m, __uint_as_float(w[3] & 0xFFFF0000u) * m);
            *reinterpret_cast<uint4 *>(qs + (g >> 3) * kTcQAtom + tc::swz(qh, (g & 7) * 16, 128)) = o;
        }
        if (qpart == 0) ms.qmul[qh] = m;
    }
    tc::fence_proxy_async();          // Q (generic writes) -> tensor core reads
    tc::fence_before_sync();
    __syncthreads();                  // Q converted; the tile buffers are free
    tc::fence_after_sync();
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int n_rows = qq.nsel + qq.nw;
    const int tile0 = sp * tiles_per_split;
    const int tile1 = min((n_rows + kTcRows - 1) / kTcRows, tile0 + tiles_per_split);
    const int nt = max(0, tile1 - tile0);
    const uint32_t tmem = ms.tmem_slot;

    // softmax state, kept for the epilogue: warp w of warpgroup wg = w / 4
    // reads TMEM lane quarter w % 4; thread (head h, half rh) owns tile rows
    // 16 rh + 8 wg .. +7
    const int wg = (warp >> 2) & 1;
    const int h = 16 * (warp & 3) + (lane & 15), rh = lane >> 4;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    float m_ref = -INFINITY, l_sum = 0.0f, pw = 0.0f;

    if (warp == kTcProdWarp) {
        // ---------------------------------------------------------------- producer
        // lane r resolves row r of each tile (its one integer read a tile
        // ahead) and copies the row into the staging buffer
        auto row = [&](int j) { return (tile0 + j) * kTcRows + lane; };
        int32_t pf = nt > 0 ? tc_row_fetch(a, qq, t, row(0)) : -1;
        int issued = 0;
        for (int j = 0; j < nt; j++) {
            const int st = j % kTcStages;
            const int32_t code = tc_row_code(a, qq, row(j), pf);
            pf = j + 1 < nt ? tc_row_fetch(a, qq, t, row(j + 1)) : -1;
            if (j >= kTcStages &&
                !tc_warp_wait(ms, ms.stage_free[st], ((j / kTcStages) - 1) & 1, a))
                break;
            const uint32_t live = __ballot_sync(0xffffffffu, code >= 0);
            if (lane == 0) {
                ms.live[st] = live;
                tc::mbar_expect_tx(tc::saddr(&ms.stage_full[st]),
                                   (uint32_t)__popc(live) * kFp8RowBytes);
            }
            __syncwarp();
            if (code >= 0)
                tc::bulk_g2s(tc::saddr(tiles_stage(base, st) + lane * kFp8RowBytes),
                             tc_row_ptr(a, code), kFp8RowBytes,
                             tc::saddr(&ms.stage_full[st]));
            issued = j + 1;
        }
        // copies still in flight land before the CTA can end
        if (lane == 0) {
            for (int j = max(0, issued - kTcStages); j < issued; j++)
                tc::mbar_wait_sleep(tc::saddr(&ms.stage_full[j % kTcStages]),
                                    (j / kTcStages) & 1, nullptr);
            tc::mbar_wait_sleep(tc::saddr(&ms.q_full), 0, nullptr);
        }
        __syncwarp();
    } else if (warp >= 8 && warp < 16) {
        // ---------------------------------------------------------------- converters
        const int c = tid - kTcSoft;
        for (int j = 0; j < nt; j++) {
            const int st = j % kTcStages, b = j % kTcBufs;
            if (!tc_wait(ms, ms.stage_full[st], (j / kTcStages) & 1, a)) break;
            if (j >= kTcBufs && !tc_wait(ms, ms.tile_free[b], ((j / kTcBufs) - 1) & 1, a))
                break;
            TcLoad L;
            tc_load(tiles_stage(base, st), ms.live[st], c, L);
            tc_store(L, c, tiles + b * kTcTileBytes, ms, b);
            tc::fence_proxy_async();
            tc::mbar_arrive(tc::saddr(&ms.tile_full[b]));
            tc::mbar_arrive(tc::saddr(&ms.stage_free[st]));
        }
    } else if (warp == kTcMmaWarp) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_s = tc_idesc_f16(64, 32, false);
            const uint32_t id_o = tc_idesc_f16(64, 128, true);
            const uint64_t qd = tc::kmajor_desc(tc::saddr(qs), 128);
            // S_j and PV_j are issued in whichever order their inputs become
            // ready (S_j: tile j converted and its S buffer read by softmax
            // j-2; PV_j: P_j written; PV first when both are), so PV_j never
            // waits behind the conversion of tile j+1.  Reuse stays safe in any order: tile j+2
            // is converted into buffer j%2 only after PV_j completed.
            int js = 0, jp = 0;
            uint64_t t_wait = tc::globaltimer();      // start of the current wait
            uint32_t idle = 0;
            while (jp < nt) {
                bool did = false;
                if (jp < js && tc::mbar_try_wait(tc::saddr(&ms.p_full[jp & 1]), (jp >> 1) & 1)) {
                    tc::fence_after_sync();
                    const int bp = jp % kTcBufs;
                    const uint64_t pd = tc::kmajor_desc(tc::saddr(ps + (jp & 1) * kTcPBytes), 64);
                    const uint64_t vd =
                        tc_mn_desc(tc::saddr(tiles + bp * kTcTileBytes), kTcAtom, 1024);
                    const uint32_t acc0 = jp > 0 ? 1u : 0u;
#pragma unroll
                    for (int blk = 0; blk < 4; blk++) {
                        const uint32_t d = tmem + ((blk >> 1) ? (16u << 16) : 0u) + kTcOCol +
                                           128u * (uint32_t)(blk & 1);
#pragma unroll
                        for (int ks = 0; ks < 2; ks++)
                            tc::mma_f16(d, desc_add(pd, blk * kTcPBlock + ks * 32),
                                        desc_add(vd, 2 * blk * kTcAtom + ks * 2048), id_o,
                                        ks > 0 ? 1u : acc0);
                    }
                    tc::mma_commit(tc::saddr(&ms.tile_free[bp]));
                    tc::mma_commit(tc::saddr(&ms.o_done));
                    jp++;
                    if (jp == nt) tc::mma_commit(tc::saddr(&ms.o_last));
                    did = true;
                }
                if (js < nt) {
                    const int b = js % kTcBufs, s = js & 1;
                    if (tc::mbar_try_wait(tc::saddr(&ms.tile_full[b]), (js / kTcBufs) & 1) &&
                        (js < 2 ||
                         tc::mbar_try_wait(tc::saddr(&ms.s_free[s]), ((js - 2) >> 1) & 1))) {
                        tc::fence_after_sync();
                        const uint64_t kd =
                            tc::kmajor_desc(tc::saddr(tiles + b * kTcTileBytes), 128);
                        const uint32_t d0 = tmem + ((uint32_t)(16 * s) << 16);
#pragma unroll
                        for (int k = 0; k < 36; k++) {
                            const int blk = k < 32 ? (k >> 3) : 4;
                            const uint32_t off = (uint32_t)((k & 3) * 32);
                            tc::mma_f16(d0 + 32 * blk, desc_add(qd, (k >> 2) * kTcQAtom + off),
                                        desc_add(kd, (k >> 2) * kTcAtom + off), id_s,
                                        (k & 7) != 0 ? 1u : 0u);
                        }
                        tc::mma_commit(tc::saddr(&ms.s_full[s]));
                        js++;
                        did = true;
                    }
                }
                if (did) {
                    idle = 0;
                } else {
                    if (tc_aborted(ms)) break;
                    if ((++idle & 63) == 0 && tc::globaltimer() - t_wait > tc::kWaitLimitNs) {
                        if (atomicExch(&ms.abort, 1) == 0) report(a.status, CSA_ERR_TIMEOUT);
                        break;
                    }
                    if (idle == 1) t_wait = tc::globaltimer();
                    __nanosleep(64);
                }
            }
            // every MMA issued has completed before TMEM or shared memory is released
            tc::mma_commit(tc::saddr(&ms.drain));
            if (!tc::mbar_wait_sleep(tc::saddr(&ms.drain), 0, nullptr)) {
                if (atomicExch(&ms.abort, 1) == 0) report(a.status, CSA_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax
        const float qsc = a.sm_scale * kTcLog2e / ms.qmul[h];
        const int r0 = 16 * rh + 8 * wg;
        for (int j = 0; j < nt; j++) {
            const int b = j % kTcBufs, s = j & 1;
            if (!tc_warp_wait(ms, ms.tile_full[b], (j / kTcBufs) & 1, a)) break;
            if (!tc_warp_wait(ms, ms.s_full[s], (j >> 1) & 1, a)) break;
            tc::fence_after_sync();
            float z[8];
            {
                uint32_t v[5][8];
                const uint32_t sa = tmem + lane_base + ((uint32_t)(16 * s) << 16) + 8 * wg;
#pragma unroll
                for (int blk = 0; blk < 5; blk++) tmem_ld_16x32bx2_x8(sa + 32 * blk, v[blk]);
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                tc::mbar_arrive(tc::saddr(&ms.s_free[s]));
                const uint32_t vm = ms.vmask[b] >> r0;
#pragma unroll
                for (int k = 0; k < 8; k++) {
                    const float4 f = ms.sc[b][r0 + k];
                    float acc = __uint_as_float(v[4][k]) * ms.ropef[b][r0 + k];
                    acc = fmaf(__uint_as_float(v[0][k]), f.x, acc);
                    acc = fmaf(__uint_as_float(v[1][k]), f.y, acc);
                    acc = fmaf(__uint_as_float(v[2][k]), f.z, acc);
                    acc = fmaf(__uint_as_float(v[3][k]), f.w, acc);
                    z[k] = (vm >> k) & 1 ? acc * qsc : -INFINITY;
                }
            }
            float mt = -INFINITY;
#pragma unroll
            for (int k = 0; k < 8; k++) mt = fmaxf(mt, z[k]);
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
            if (rh == 0) ms.mx[s][wg][h] = mt;
            softmax_sync();
            mt = fmaxf(mt, ms.mx[s][wg ^ 1][h]);
            // power-of-two normaliser of the block scales (the same for every
            // thread): set by the first tile with a non-zero scale so that
            // its largest scale maps into [8, 16), and lowered (with O
            // rescaled) only when a tile's largest scale would take P past
            // fp16 range (P <= 2^8 x 2^7)
            const float smax = ms.smax[b];
            float ratio = 1.0f;
            if (smax > 0.0f && (pw == 0.0f || smax * pw >= 128.0f)) {
                const float pw_new = fit_pow2(smax, 4);
                if (pw > 0.0f) ratio = pw_new / pw;
                pw = pw_new;
            }
            float alpha = 1.0f;
            if (mt > m_ref + kTcRaise) {
                if (m_ref != -INFINITY) alpha = exp2f(m_ref - mt);
                m_ref = mt;
            }
            const float factor = alpha * ratio;
            if (__any_sync(0xffffffffu, j > 0 && factor != 1.0f)) {
                // O of tile j-1 must have landed before it is rescaled; each
                // warpgroup rescales 128 of its lane half's 256 columns
                if (!tc_warp_wait(ms, ms.o_done, (j - 1) & 1, a)) break;
                tc::fence_after_sync();
#pragma unroll 1
                for (int c0 = 128 * wg; c0 < 128 * wg + 128; c0 += 32) {
                    uint32_t ov[32];
                    const uint32_t ta = tmem + lane_base + kTcOCol + (uint32_t)c0;
                    tc::tmem_ld32_nowait(ta, ov);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i++)
                        ov[i] = __float_as_uint(__uint_as_float(ov[i]) * factor);
                    tmem_st_32x32b_x32(ta, ov);
                }
                tmem_wait_st();
            }
            float psum = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; k++) {
                z[k] = m_ref == -INFINITY ? 0.0f : ex2_approx(z[k] - m_ref);
                psum += z[k];
                z[k] *= pw;
            }
            l_sum = l_sum * alpha + psum;
            // P_b[head][row] = p x pw x scale_b (fp16), rows r0 .. r0+7
            uint8_t *pb = ps + s * kTcPBytes;
            const uint32_t po = tc::swz(h, 32 * rh + 16 * wg, 64);
            uint32_t w[4][4];
#pragma unroll
            for (int k2 = 0; k2 < 4; k2++) {
                const float4 f0 = ms.sc[b][r0 + 2 * k2], f1 = ms.sc[b][r0 + 2 * k2 + 1];
                w[0][k2] = pack_f16(z[2 * k2] * f0.x, z[2 * k2 + 1] * f1.x);
                w[1][k2] = pack_f16(z[2 * k2] * f0.y, z[2 * k2 + 1] * f1.y);
                w[2][k2] = pack_f16(z[2 * k2] * f0.z, z[2 * k2 + 1] * f1.z);
                w[3][k2] = pack_f16(z[2 * k2] * f0.w, z[2 * k2 + 1] * f1.w);
            }
#pragma unroll
            for (int blk = 0; blk < 4; blk++)
                *reinterpret_cast<uint4 *>(pb + blk * kTcPBlock + po) =
                    make_uint4(w[blk][0], w[blk][1], w[blk][2], w[blk][3]);
            tc::fence_proxy_async();
            tc::fence_before_sync();
            tc::mbar_arrive(tc::saddr(&ms.p_full[s]));
        }
        // row sums of the head: this thread's rows, its partner's, the other warpgroup's
        l_sum += __shfl_xor_sync(0xffffffffu, l_sum, 16);
        if (rh == 0) ms.lx[wg][h] = l_sum;
        softmax_sync();
        l_sum += ms.lx[wg ^ 1][h];
        if (nt > 0) tc_warp_wait(ms, ms.o_last, 0, a);
        tc::fence_after_sync();
    }

    // ---------------------------------------------------------------- epilogue
    // the softmax warps decide together whether O is there to read (TMEM loads
    // are warp-wide)
    const bool have_o = __shfl_sync(0xffffffffu, nt > 0 && !tc_aborted(ms), 0);
    const int64_t orow0 = (int64_t)t * a.heads + hg * kTcHeads;
    if (splits == 1) {
        if (warp < 8 && (have_o || nt == 0)) {
            const float inv = (l_sum > 0.0f && pw > 0.0f) ? 1.0f / (l_sum * pw) : 0.0f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                  (orow0 + h) * kLatent + 256 * rh;
#pragma unroll 1
            for (int c0 = 128 * wg; c0 < 128 * wg + 128; c0 += 32) {
                uint32_t ov[32];
                if (have_o) {
                    tc::tmem_ld32_nowait(tmem + lane_base + kTcOCol + (uint32_t)c0, ov);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++) ov[i] = 0u;
                }
#pragma unroll
                for (int v = 0; v < 4; v++) {
                    uint4 o;
                    o.x = pack_bf16(__uint_as_float(ov[8 * v]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
                    o.y = pack_bf16(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
                    o.z = pack_bf16(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
                    o.w = pack_bf16(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
                    *reinterpret_cast<uint4 *>(orow + c0 + 8 * v) = o;
                }
            }
            if (a.lse && rh == 0 && wg == 0)
                a.lse[orow0 + h] = l_sum > 0.0f ? (m_ref + log2f(l_sum)) * 0.6931471805599453f
                                                : -INFINITY;
        }
    } else {
        // Split merge through distributed shared memory.  The (max, sum) of
        // every head and each split's largest block scale are exchanged
        // first; then each split, for every other split in turn, stages that
        // split's 512/splits output dims of its O (rescaled to the merged
        // softmax, fp16, 16-byte chunks XOR-swizzled by head) in its own
        // shared memory and pushes them with one bulk copy into the owner's
        // receive buffer; the owner adds its own slice from TMEM (fp32) and
        // writes the bf16 outputs.
        // fp16 range: a split's share of a merged output is a weighted mean of
        // value dims with weights summing to at most 1, so its magnitude is at
        // most the largest |code x block scale| of the query's rows, at most
        // 448 x the largest block scale.  Slices are sent times the power of two
        // that maps that bound into [2^14, 2^15) (exact scaling; fp16 keeps
        // 11 significant bits of every value down to 2^-28 of the bound).
        const int dpo = kLatent / splits;                       // dims per owner
        const uint32_t slice = (uint32_t)(kTcHeads * dpo * 2);  // bytes of one slice
        const int cpr = dpo / 8;                                // 16-byte chunks per row
        // receive buffer at the end of the CTA's buffers: one slot per other
        // split (slot of split r: r, or r-1 for splits after this one);
        // outgoing slices staged from the start, as many as fit below it
        uint8_t *recv = base + kTcMiscOff - (splits - 1) * slice;
        uint8_t *stg = base;
        auto recv_slot = [&](int src, int dst) { return src < dst ? src : src - 1; };
        if (warp < 4 && rh == 0) {
            // this split's (max, sum) of head h into every split's table
            const uint32_t src = tc::saddr(&ms.ml[sp][h][0]);
            for (int r = 0; r < splits; r++) st_cluster_f32x2(cluster_map(src, r), m_ref, l_sum);
        }
        if (tid < splits) st_cluster_f32(cluster_map(tc::saddr(&ms.vmax[sp]), tid), ms.vrun);
        if (tid == 0) tc::mbar_expect_tx(tc::saddr(&ms.recv_full), (uint32_t)(splits - 1) * slice);
        cluster_sync();          // every split's MMAs are done and its (max, sum) delivered
        if (warp < 4 && rh == 0) {
            float M = -INFINITY;
            for (int r = 0; r < splits; r++)
                if (ms.ml[r][h][1] > 0.0f) M = fmaxf(M, ms.ml[r][h][0]);
            float L = 0.0f;
            for (int r = 0; r < splits; r++)
                if (ms.ml[r][h][1] > 0.0f) L += ms.ml[r][h][1] * exp2f(ms.ml[r][h][0] - M);
            ms.fct[h] = (have_o && l_sum > 0.0f && pw > 0.0f && L > 0.0f)
                            ? exp2f(m_ref - M) / (L * pw)
                            : 0.0f;
            if (sp == 0 && a.lse)
                a.lse[orow0 + h] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
        }
        __syncthreads();
        float vb = 0.0f;
        for (int r = 0; r < splits; r++) vb = fmaxf(vb, ms.vmax[r]);
        const float f16s = fit_pow2(448.0f * vb, 15);          // slices are sent times f16s
        const float f16r = 1.0f / f16s;                         // exact (a power of two)
        // warps 0-15: four per TMEM lane quarter; each 16x32bx2 load gives a
        // thread 16 columns of head hq (threads 16-31 the next 16)
        const int q4 = warp & 3, wq = warp >> 2;                // wq = 0..3 for warps 0-15
        const int hq = 16 * q4 + (lane & 15), chalf = lane >> 4;
        const float fq = warp < 16 ? ms.fct[hq] : 0.0f;
        // reads 16 fp32 O values of head hq, dims d .. d+15 (d in [0, 512)), scaled by f
        auto read_o = [&](int d, float f, float (&o)[16]) {
            uint32_t v[16];
            if (have_o) {
                const uint32_t ta = tmem + ((uint32_t)(32 * q4 + 16 * (d >> 8)) << 16) + kTcOCol +
                                    (uint32_t)((d & 255) - 16 * chalf);
                tmem_ld_16x32bx2_x16(ta, v);
                tc::tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] = 0u;
            }
#pragma unroll
            for (int i = 0; i < 16; i++) o[i] = __uint_as_float(v[i]) * f;
        };
        // byte offset of 16-byte chunk j (8 fp16 dims) of head row hh in a
        // slice (cpr >= 8: at most 8 splits)
        auto slot = [&](int hh, int j) {
            return (uint32_t)((hh * cpr + (j ^ (hh & 7))) * 16);
        };
        // the outgoing slices of a round are pushed back to back (one round
        // for up to 4 splits)
        const int per_round = (int)((uint32_t)(recv - stg) / slice);
        for (int k0 = 1; k0 < splits; k0 += per_round) {
            const int k1 = min(splits, k0 + per_round);
            if (warp < 16) {
                for (int k = k0; k < k1; k++) {
                    const int owner = (sp + k) % splits;
                    uint8_t *out_slice = stg + (k - k0) * slice;
                    for (int c32 = 32 * wq; c32 < dpo; c32 += 128) {
                        const int dl = c32 + 16 * chalf;         // this thread's 16 dims
                        float o[16];
                        read_o(owner * dpo + dl, fq * f16s, o);
#pragma unroll
                        for (int v8 = 0; v8 < 2; v8++)
                            *reinterpret_cast<uint4 *>(out_slice + slot(hq, dl / 8 + v8)) =
                                make_uint4(pack_f16(o[8 * v8], o[8 * v8 + 1]),
                                           pack_f16(o[8 * v8 + 2], o[8 * v8 + 3]),
                                           pack_f16(o[8 * v8 + 4], o[8 * v8 + 5]),
                                           pack_f16(o[8 * v8 + 6], o[8 * v8 + 7]));
                    }
                }
            }
            tc::fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                for (int k = k0; k < k1; k++) {
                    const int owner = (sp + k) % splits;
                    bulk_s2s_cluster(cluster_map(tc::saddr(recv + recv_slot(sp, owner) * slice),
                                                 owner),
                                     tc::saddr(stg + (k - k0) * slice), slice,
                                     cluster_map(tc::saddr(&ms.recv_full), owner));
                }
                bulk_commit_wait_read();
            }
            __syncthreads();
        }
        // this split's own dims: its slice from TMEM plus every received slice
        const bool got = tc_warp_wait(ms, ms.recv_full, 0, a);
        if (warp < 16 && got) {
            for (int c32 = 32 * wq; c32 < dpo; c32 += 128) {
                const int dl = c32 + 16 * chalf;
                float o[16];
                read_o(sp * dpo + dl, fq, o);
                for (int r = 0; r < splits - 1; r++) {
#pragma unroll
                    for (int v8 = 0; v8 < 2; v8++) {
                        const uint4 x = *reinterpret_cast<const uint4 *>(
                            recv + r * slice + slot(hq, dl / 8 + v8));
                        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            const float2 f = __half22float2(
                                *reinterpret_cast<const __half2 *>(&w[k]));
                            o[8 * v8 + 2 * k] = fmaf(f.x, f16r, o[8 * v8 + 2 * k]);
                            o[8 * v8 + 2 * k + 1] = fmaf(f.y, f16r, o[8 * v8 + 2 * k + 1]);
                        }
                    }
                }
                __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                      (orow0 + hq) * kLatent + sp * dpo + dl;
                *reinterpret_cast<uint4 *>(orow) =
                    make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                               pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
                *reinterpret_cast<uint4 *>(orow + 8) =
                    make_uint4(pack_bf16(o[8], o[9]), pack_bf16(o[10], o[11]),
                               pack_bf16(o[12], o[13]), pack_bf16(o[14], o[15]));
            }
        }
        cluster_sync();          // no split leaves while a peer may still read its (max, sum)
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// Splits per query: decode fills the 148 SMs with up to 8 splits (a power of
// two dividing the 512 output dims); prefill uses one.
static int tc_splits(const AttnArgs &a, bool decode, int n_tiles) {
    if (!decode) return 1;
    const int ctas = a.num_q * (a.heads / kTcHeads);
    int sp = 1;
    while (sp < kTcMaxSplits && ctas * sp * 2 <= 148 && sp * 2 <= n_tiles) sp *= 2;
    return sp;
}

bool sparse_mqa_tc_supported(const AttnArgs &a) {
    return a.kv_fmt == CSA_FMT_FP8 && a.heads % kTcHeads == 0;
}

cudaError_t launch_sparse_mqa_tc(const AttnArgs &a, bool decode, cudaStream_t s) {
    static int done[64] = {0};
    cudaError_t e = ensure_max_smem((const void *)sparse_mqa_tc_kernel, (int)kTcSmem, done);
    if (e != cudaSuccess) return e;
    const int max_sel = a.dense_ratio > 0 ? a.max_sel : kTopK;
    const int n_tiles = (max_sel + a.window + kTcRows - 1) / kTcRows;
    const int sp = tc_splits(a, decode, n_tiles);
    const int tps = (n_tiles + sp - 1) / sp;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_q, a.heads / kTcHeads, sp);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = kTcSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = sp;
    cfg.attrs = attr;
    cfg.numAttrs = sp > 1 ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, sparse_mqa_tc_kernel, a, sp, tps);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
