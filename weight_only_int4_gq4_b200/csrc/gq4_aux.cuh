// gq4_aux.cuh -- the grouped-int4 kernels beside the expert FFN: quantisation of float
// weights, row dequantisation / gather, and a generic matvec for any group size that is
// a multiple of 8 (partial last groups included), over all rows or over selected rows.
//
// Sources (colibri PR #298, "cuda+engine: full fmt=4 (grouped int4 gs=64) support"):
//   * "What was implemented (CPU)": matmul_i4_grouped handles arbitrary gs (multiple of
//     16) and applies each group's scale once; detect_group_size derives gs from the
//     scale-array size;
//   * "implementation complete but blocked" / the gs=128 follow-up: embed_row, qt_addrow
//     and qt_matvec_rows need the fmt=4 (per-group scale) branch, group-size-generic;
//   * the maintainer's "data request": the converter quantises with --group-size 64.
// Device layout of the packed weights as everywhere in this library: rows of in/2 bytes;
// inside every 32-bit word (weights k = 8i..8i+7 of a row) the even-k nibbles sit in
// bits 0-15 (k0,k2,k4,k6) and the odd-k nibbles in bits 16-31 (k1,k3,k5,k7).
#pragma once
#include "gq4_common.cuh"

namespace gq4 {

// Nibble slot of weight j (0..7) of a device word: even j -> j/2, odd j -> 4 + j/2.
__device__ __forceinline__ int dev_slot(int j) { return (j & 1) ? 4 + (j >> 1) : (j >> 1); }

// Signed value of nibble slot i of a device word.
__device__ __forceinline__ int dev_q(uint32_t v, int i) {
    return (int)((v >> (4 * i)) & 15u) - (int)(((v >> (4 * i)) & 8u) << 1);
}

// ---------------------------------------------------------------- quantisation
// One group per SEG consecutive threads (SEG a power of two <= 32, a group's words split
// among them; a thread takes words sub, sub+SEG, ...).  Per group: amax = max |w|,
// s = amax / 7 (IEEE f32 division), q = round-half-even(w / s) clamped to [-8, 7];
// amax == 0 gives s = 0, q = 0.  Writes the device word order and one scale per group.
// Rows hold ng groups; threads of a row's padded group slots past `in` do nothing.
template <int SEG>
__global__ void __launch_bounds__(256) gq4_quantize_kernel(const float *w, int64_t O, int64_t I, int gs, int ng,
                                                           uint32_t *dw, float *ds) {
    const int64_t groups = O * ng;
    const int lane = threadIdx.x & 31, sub = lane & (SEG - 1);
    constexpr int kGpw = 32 / SEG;  // groups per warp and pass
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    // warp-uniform loop (the shuffles need every lane); lanes of a group slot past the
    // last group run with no words
    for (int64_t gw = warp * kGpw; gw < groups; gw += warps * kGpw) {
        const int64_t gi = gw + lane / SEG;
        const bool valid = gi < groups;
        const int64_t o = valid ? gi / ng : 0;
        const int g = valid ? (int)(gi - o * ng) : 0;
        const int64_t k0 = (int64_t)g * gs;
        const int words = valid ? (int)(min((int64_t)gs, I - k0) >> 3) : 0;  // I % 8 == 0
        const float *src = w + o * I + k0;
        float amax = 0.f;
        for (int wi = sub; wi < words; wi += SEG) {
            const float4 a = *(const float4 *)(src + 8 * wi);
            const float4 b = *(const float4 *)(src + 8 * wi + 4);
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
        }
        #pragma unroll
        for (int off = SEG >> 1; off > 0; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off, SEG));
        const float s = __fdiv_rn(amax, 7.0f);
        if (valid && sub == 0) ds[o * ng + g] = s;
        uint32_t *dst = dw + (o * I + k0) / 8;
        for (int wi = sub; wi < words; wi += SEG) {
            const float4 a = *(const float4 *)(src + 8 * wi);
            const float4 b = *(const float4 *)(src + 8 * wi + 4);
            const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t word = 0;
            #pragma unroll
            for (int j = 0; j < 8; ++j) {
                int q = 0;
                if (s > 0.f) {
                    float r = rintf(__fdiv_rn(v[j], s));
                    r = fminf(fmaxf(r, -8.f), 7.f);
                    q = (int)r;
                }
                word |= ((uint32_t)q & 15u) << (4 * dev_slot(j));
            }
            dst[wi] = word;
        }
    }
}

// ---------------------------------------------------------------- row dequantisation
// out[j][k] = (accumulate ? out[j][k] : 0) + alpha_j * s[idx_j][k/gs] * q[idx_j][k];
// one thread per (selected row, word); gs % 8 == 0, so a word lies in one group.  A listed
// row outside [0, n_weight_rows) is not read and gives NaN outputs.
// ODT: 0 = f32 out, 1 = bf16 out (round to nearest even; no accumulate).
template <int ODT>
__global__ void __launch_bounds__(256) gq4_dequant_rows_kernel(const uint32_t *dw, const float *ds, int64_t n_weight_rows,
                                                               int64_t I, int gs,
                                                               int ng, const int32_t *idx, int64_t n,
                                                               const float *alpha, int accumulate, void *out) {
    const int64_t wpr = I >> 3;  // words per row
    const int64_t total = n * wpr;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = t / wpr, wi = t - j * wpr;
        const int64_t row = idx[j];
        if (row < 0 || row >= n_weight_rows) {  // not read: NaN outputs
            const float nan = __uint_as_float(0x7fc00000u);
            if (ODT == 0) {
                float4 *o4 = (float4 *)((float *)out + j * I + wi * 8);
                o4[0] = make_float4(nan, nan, nan, nan);
                o4[1] = o4[0];
            } else {
                *(uint4 *)((uint16_t *)out + j * I + wi * 8) = make_uint4(0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u);
            }
            continue;
        }
        const int64_t wix = row * wpr + wi, six = row * ng + (wi * 8) / gs;
        const uint32_t v = in_bounds(wix, n_weight_rows * wpr) ? __ldg(dw + wix) : 0u;
        const float s = in_bounds(six, n_weight_rows * (int64_t)ng) ? __ldg(ds + six) : 0.f;
        const float a = alpha ? alpha[j] : 1.f;
        float r[8];
        #pragma unroll
        for (int i = 0; i < 8; ++i) r[i] = a * (s * (float)dev_q(v, dev_slot(i)));
        if (ODT == 0) {
            float4 *o4 = (float4 *)((float *)out + j * I + wi * 8);
            if (accumulate) {
                const float4 p0 = o4[0], p1 = o4[1];
                r[0] += p0.x; r[1] += p0.y; r[2] += p0.z; r[3] += p0.w;
                r[4] += p1.x; r[5] += p1.y; r[6] += p1.z; r[7] += p1.w;
            }
            o4[0] = make_float4(r[0], r[1], r[2], r[3]);
            o4[1] = make_float4(r[4], r[5], r[6], r[7]);
        } else {
            uint4 h;
            h.x = bf16_bits_rn(r[0]) | (bf16_bits_rn(r[1]) << 16);
            h.y = bf16_bits_rn(r[2]) | (bf16_bits_rn(r[3]) << 16);
            h.z = bf16_bits_rn(r[4]) | (bf16_bits_rn(r[5]) << 16);
            h.w = bf16_bits_rn(r[6]) | (bf16_bits_rn(r[7]) << 16);
            *(uint4 *)((uint16_t *)out + j * I + wi * 8) = h;
        }
    }
}

// ---------------------------------------------------------------- generic matvec
// One warp per output row (per gate/up row pair in MODE 1); lane L takes groups
// L, L+32, ...; within a group it walks the words, accumulates sum_k q * x[t][k] in f32
// and adds scale * partial once per group (the scale hoisted per group, as the pages'
// CPU kernel does); the lanes' sums are added by a fixed shuffle tree.
// Activations: staged in shared memory as f32 when stage_x (all T rows fit), else read
// from global memory.  rows: NULL (row r = warp's index) or a gather list; a listed row
// outside [0, n_weight_rows) is not read and gives NaN outputs.
// MODE: 0 = y[t][r] f32; 1 = gate+up: h[t][r] = silu(g) * u rounded to XDT.
constexpr int kGenMaxTok = 8;  // tokens per pass

template <int MODE, int XDT>
__global__ void __launch_bounds__(256) gq4_generic_kernel(const uint32_t *dw0, const float *ds0, const uint32_t *dw1,
                                                          const float *ds1, int64_t n_weight_rows, int64_t n_rows,
                                                          const int32_t *rows,
                                                          int64_t I, int gs, int ng, const void *x, int T,
                                                          int stage_x, void *out) {
    extern __shared__ float xs[];  // [T][I] f32 when stage_x
    const int64_t wpr = I >> 3;
    if (stage_x) {
        for (int64_t i = threadIdx.x; i < (int64_t)T * I; i += blockDim.x)
            xs[i] = XDT == 1 ? bf16_bits_to_f32(((const uint16_t *)x)[i]) : ((const float *)x)[i];
        __syncthreads();
    }
    auto xval = [&](int t, int64_t k) -> float {
        if (stage_x) return xs[(int64_t)t * I + k];
        return XDT == 1 ? bf16_bits_to_f32(((const uint16_t *)x)[(int64_t)t * I + k])
                        : ((const float *)x)[(int64_t)t * I + k];
    };
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int wpg = gs >> 3;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < n_rows; r += warps) {
        const int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= n_weight_rows) {  // warp-uniform
            for (int t = lane; t < T; t += 32) {
                const int64_t o = (int64_t)t * n_rows + r;
                if (MODE == 0 || XDT == 0) ((float *)out)[o] = __uint_as_float(0x7fc00000u);
                else ((uint16_t *)out)[o] = 0x7fc0u;
            }
            continue;
        }
        for (int t0 = 0; t0 < T; t0 += kGenMaxTok) {
            const int nt = min(kGenMaxTok, T - t0);
            float acc0[kGenMaxTok], acc1[kGenMaxTok];
            #pragma unroll
            for (int t = 0; t < kGenMaxTok; ++t) { acc0[t] = 0.f; acc1[t] = 0.f; }
            for (int g = lane; g < ng; g += 32) {
                const int64_t w0 = (int64_t)g * wpg;
                const int words = (int)min((int64_t)wpg, wpr - w0);
                float p0[kGenMaxTok], p1[kGenMaxTok];
                #pragma unroll
                for (int t = 0; t < kGenMaxTok; ++t) { p0[t] = 0.f; p1[t] = 0.f; }
                for (int wi = 0; wi < words; ++wi) {
                    const int64_t wix = row * wpr + w0 + wi;
                    const bool wok = in_bounds(wix, n_weight_rows * wpr);
                    const uint32_t v0 = wok ? __ldg(dw0 + wix) : 0u;
                    const uint32_t v1 = MODE == 1 && wok ? __ldg(dw1 + wix) : 0u;
                    const int64_t k = (w0 + wi) * 8;
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float q0 = (float)dev_q(v0, dev_slot(j));
                        const float q1 = MODE == 1 ? (float)dev_q(v1, dev_slot(j)) : 0.f;
                        #pragma unroll
                        for (int t = 0; t < kGenMaxTok; ++t) {
                            if (t < nt) {
                                const float xv = xval(t0 + t, k + j);
                                p0[t] = fmaf(q0, xv, p0[t]);
                                if (MODE == 1) p1[t] = fmaf(q1, xv, p1[t]);
                            }
                        }
                    }
                }
                const int64_t six = row * ng + g;
                const bool sok = in_bounds(six, n_weight_rows * (int64_t)ng);
                const float s0 = sok ? __ldg(ds0 + six) : 0.f;
                const float s1 = MODE == 1 && sok ? __ldg(ds1 + six) : 0.f;
                #pragma unroll
                for (int t = 0; t < kGenMaxTok; ++t) {
                    acc0[t] = fmaf(s0, p0[t], acc0[t]);
                    if (MODE == 1) acc1[t] = fmaf(s1, p1[t], acc1[t]);
                }
            }
            #pragma unroll
            for (int t = 0; t < kGenMaxTok; ++t) {
                #pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    acc0[t] += __shfl_xor_sync(0xffffffffu, acc0[t], off);
                    if (MODE == 1) acc1[t] += __shfl_xor_sync(0xffffffffu, acc1[t], off);
                }
            }
            if (lane == 0) {
                #pragma unroll
                for (int t = 0; t < kGenMaxTok; ++t) {
                    if (t >= nt) break;
                    const int64_t o = (int64_t)(t0 + t) * n_rows + r;
                    if (MODE == 0) {
                        ((float *)out)[o] = acc0[t];
                    } else {
                        const float h = silu_mul(acc0[t], acc1[t]);
                        if (XDT == 1) ((uint16_t *)out)[o] = (uint16_t)bf16_bits_rn(h);
                        else ((float *)out)[o] = h;
                    }
                }
            }
        }
    }
}

}  // namespace gq4
