// common.cuh -- device helpers shared by the libcsa kernels (sm_100a).
//
// Number-format conversions use the hardware's round-to-nearest-even,
// saturating PTX conversions; the fast Walsh-Hadamard transform is the
// butterfly form of the Sylvester matrix H_2n = [[H, H], [H, -H]] used by the
// index rotation of "Token 的一生：DSV4 架构与 DSpark" §4.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

constexpr int kTopK = 512;
constexpr int kPage = 256;       // raw tokens per page
constexpr int kC4Page = 64;      // compressed rows per page
constexpr int kHcaRatio = 128;   // HCA: raw rows per compressed row
constexpr int kHcaPage = 2;      // HCA compressed rows per 256-token page
constexpr int kKvDim = 576;
constexpr int kLatent = 512;
constexpr int kRope = 64;
constexpr int kFp8RowBytes = 656;
constexpr int kBf16RowBytes = 1152;

// First recorded device-side problem wins; later ones are dropped.
// Programmatic dependent launch.  Every kernel starts with this: it lets the
// next kernel on the stream be scheduled at once (its blocks become resident
// as resources free up and wait here in turn), then waits until the kernels
// this one depends on have completed and their writes are visible.  Nothing
// global is read before the wait.  Both instructions are no-ops when the
// kernel was launched without the programmatic-serialization attribute.
// The two halves of pdl_begin, for kernels that read caller inputs (request
// offsets, lengths, positions) before waiting on the preceding kernel.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void report(int32_t *status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- FP8 E4M3

// Two floats -> two E4M3 bytes (lo in bits 0-7, hi in bits 8-15), RNE, saturating.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint8_t f32_to_e4m3(float v) {
    return (uint8_t)(f32x2_to_e4m3x2(v, 0.0f) & 0xFF);
}

// Two E4M3 bytes -> half2 (exact), then float.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t v) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t v) {
    return e4m3x2_to_f32x2((uint16_t)v).x;
}

// ---------------------------------------------------------------- FP4 E2M1

// Eight floats -> four bytes of E2M1 codes; element 2i in the low nibble of
// byte i.  RNE, saturating at +-6.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return r;
}

// Four bytes of E2M1 codes -> eight floats (exact), element order as above.
__device__ __forceinline__ void e2m1x8_to_f32x8(uint32_t w, float (&v)[8]) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float2 f = __half22float2(*reinterpret_cast<__half2 *>(&h[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// ---------------------------------------------------------------- bf16

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t v) {
    return __uint_as_float(((uint32_t)v) << 16);
}

// ---------------------------------------------------------------- paging

__device__ __forceinline__ int64_t c4_slot(const int32_t *pt_row, int32_t s) {
    return (int64_t)pt_row[s / kC4Page] * kC4Page + (s % kC4Page);
}

__device__ __forceinline__ int64_t raw_slot(const int32_t *pt_row, int32_t r) {
    return (int64_t)pt_row[r / kPage] * kPage + (r % kPage);
}

// ---------------------------------------------------------------- warp helpers

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Unnormalised fast Walsh-Hadamard transform of one row of E*32 values held
// by a full warp, lane l owning elements [l*E, l*E+E).  Sylvester (natural)
// order: y_i = sum_j (-1)^popcount(i&j) x_j.
template <int E>
__device__ __forceinline__ void warp_fwht(float (&v)[E], int lane) {
#pragma unroll
    for (int h = 1; h < E; h <<= 1) {
#pragma unroll
        for (int i = 0; i < E; i++) {
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < E; i++) {
            float o = __shfl_xor_sync(0xffffffffu, v[i], m);
            v[i] = upper ? (o - v[i]) : (v[i] + o);
        }
    }
}

}  // namespace csa
