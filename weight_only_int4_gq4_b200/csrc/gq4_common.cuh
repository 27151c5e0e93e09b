// gq4_common.cuh -- small device helpers shared by the gq4 kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace gq4 {

constexpr int kGroup = 64;  // gs: weights per scale (colibri PR #298, fmt=4 gs=64)

// d = (b & (a ^ c)) | (~b & c): keep c outside mask b, and a^c inside it (LUT 0x6a).
__device__ __forceinline__ uint32_t lop3_sel_xor(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Two signed nibbles -> bf16x2 holding the exact integers q in -8..7.
// Input: the nibbles sit at bits 0-3 and 16-19 of `v` (two's complement).  The lop3
// flips each nibble's sign bit (n ^ 8 = q + 8) and plants it under the bf16 exponent of
// 128.0 (0x4300), whose mantissa unit is 1, giving 136 + q exactly; subtracting 136 in
// bf16 is exact as well.
__device__ __forceinline__ uint32_t nib2_to_bf16x2(uint32_t v) {
    const uint32_t t = lop3_sel_xor(v, 0x000F000Fu, 0x43084308u);
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(t), "r"(0x3F803F80u), "r"(0xC308C308u));
    return d;
}

// D = A(16x16 bf16) * B(16x8 bf16) + C, f32 accumulate (legacy warp-level tensor op,
// used here as the dot-product engine of the HBM-bound decode kernels).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1, const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1),
          "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

// Streaming 8-byte weight load: read-only path, no L1 allocation (each byte is read once).
__device__ __forceinline__ uint2 ldg_stream_u2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ float ldg_f32(const float *p) {
    float r;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float f) {
    // round-to-nearest-even f32 -> bf16 (NaN kept quiet)
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (u >> 16) | 0x40u;
    u += 0x7fffu + ((u >> 16) & 1u);
    return u >> 16;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + expf(-g)) * u;
}

// ---- checked build (GQ4_CHECKED) ------------------------------------------------------
// The bug class the pages report is an index outside its array: a scale read with a row
// index on an O*ng scale array (colibri PR #298, "fmt=4 CUDA attention crash -- root
// cause") and a shard's scale pointer offset by rows instead of rows*ng (the
// maintainer's oracle reply).  Built with GQ4_CHECKED, the kernels test every weight,
// scale and activation-row index they compute against the extent of its array before
// the access.  An index outside is not used -- the access reads zeros, or a copy that
// must still deliver its bytes reads row 0 instead -- and GQ4_ERR_BOUNDS is OR-ed into the
// library's bounds status word (gq4_bounds_status reads it).  Nothing traps.  Without the
// flag the tests compile away.
#ifdef GQ4_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif
constexpr int32_t kStatusBounds = 16;  // GQ4_ERR_BOUNDS
__device__ int32_t g_bounds_status;    // OR of kStatusBounds raised since the last clear

// True when 0 <= i < n (always true without GQ4_CHECKED).
__device__ __forceinline__ bool in_bounds(int64_t i, int64_t n) {
    if constexpr (!kChecked) {
        return true;
    } else {
        if (i >= 0 && i < n) return true;
        atomicOr(&g_bounds_status, kStatusBounds);
        return false;
    }
}

// Self-test of the mechanism: tests index i against extent n and accesses nothing.
__global__ void gq4_bounds_selftest_kernel(int64_t i, int64_t n) {
    if (threadIdx.x == 0) (void)in_bounds(i, n);
}

}  // namespace gq4
