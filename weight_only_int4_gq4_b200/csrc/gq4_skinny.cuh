// gq4_skinny.cuh -- decode-regime grouped-int4 kernels (few tokens per matrix).
//
// What they compute (colibri PR #298 "cuda+engine: full fmt=4 (grouped int4 gs=64)
// support"): y[c][o] = sum_g s[o][g] * sum_{k in group g} q[o][k] * x[c][k], with
// the per-group scale applied once per 64-wide group to an f32 partial (the maintainer's
// advice in "data request": hoist the scale per group instead of dividing k/gs per
// element), fp32 accumulation.
//
// Design (B200, HBM-bound):
//  * Weights: [O][I/2] bytes per matrix (rows as on the pages), nibbles of each 32-bit
//    word in the device order described below.  A warp takes
//    a 16-row x 64-column group tile (512 B): lane (g,t) reads 8 contiguous bytes of row
//    g and of row g+8 -- every 32-byte sector is used whole.
//  * The dot products run on the warp tensor op m16n8k16 (bf16 in, f32 out): the
//    nibbles become exact bf16 integers (one lop3 + one bf16x2 fma per two weights).
//    The device word order (even-k nibbles in the low half-word, odd-k in the high one,
//    written by gq4_upload) makes nibble slots i and i+4 of a word the bf16 pair of
//    columns (2i, 2i+1); the 16 contraction slots of one op are assigned so that a
//    lane's own 8 bytes are its A fragment (no shuffles) and its B fragment is 32
//    contiguous bytes of the activation row, staged once in shared memory.  The op is
//    only the dot-product engine: the bound is HBM, and this keeps the issue slots per
//    weight near 1.
//  * The f32 partial of each group is scaled by s[o][g] and added to the running sum.
//  * A CTA (8 warps) owns a 16-row tile (32 with gate+up) for all columns it serves;
//    its warps split the groups, and the eight partial tiles are summed in shared memory
//    in a fixed order (deterministic), then the epilogue of the mode runs.
//  * Persistent grid over units (matrix/expert, row tile); for the MoE modes the number
//    of units is read on the device (active experts x row tiles), so no host sync.
#pragma once
#include "gq4_common.cuh"

namespace gq4 {

enum SkinnyMode { kMatvec = 0, kGateUp = 1, kMoeGateUp = 2, kMoeDown = 3 };

struct SkinnyParams {
    const uint8_t *w0;  // matrix (or gate) packed nibbles, expert 0
    const float *s0;
    const uint8_t *w1;  // up (gate+up modes)
    const float *s1;
    int64_t estride_w;  // bytes between experts
    int64_t estride_s;  // floats between experts
    int O, I, ng;
    int row_tiles;      // ceil(O/16)
    // activations: matvec/gate-up: x [n_tok][I] (xdt); moe gate-up: x [T][I] bf16
    // (gathered through row_tok); moe down: h [T*K][I] bf16 in row-map order
    const void *x;
    int xdt;            // 0 f32, 1 bf16
    int n_tok;
    int xcols;          // staged columns the shared-memory buffer holds
    // outputs
    float *y;           // matvec [n_tok][O]; moe down [T][O] (accumulated)
    void *h;            // gate-up [n_tok][O] (xdt); moe gate-up [T*K][O] bf16
    // MoE tables (device)
    const int32_t *offs, *cnt, *row_tok, *row_slot, *n_active, *active;
    const float *wts;
    float *zero_ptr;    // moe gate-up: y zeroed here before the down kernel adds into it
    int64_t zero_n;     // floats (multiple of 4)
    // split-K kernel, plain matvec / gate+up only: a group size of 64 << gshift (scale of
    // 64-wide group G at column G >> gshift of a scale row of sng floats; 0 = ng), and an
    // optional gather list: output j < n_out is weight row rows[j]
    int gshift;
    int sng;
    const int32_t *rows;
    int n_out;
    // extents for the checked build (GQ4_CHECKED): bytes of the weight array (all experts),
    // floats of the scale array, rows of the activation array, experts of the call
    int64_t w_bytes, s_count, x_rows;
    int n_exp;
    // TMA-fed decode kernel, MoE modes: device counter of the (expert, band) units taken,
    // zero before the launch
    int32_t *unit_ctr;
};

template <int MODE>
struct ModeTraits {
    static constexpr int kPair = (MODE == kGateUp || MODE == kMoeGateUp) ? 2 : 1;
    static constexpr bool kMoe = (MODE == kMoeGateUp || MODE == kMoeDown);
};

// Bytes of one staged column: the I activations as bf16 plus 16 B of padding, which
// shifts consecutive columns by four banks (conflict-free 16-byte fragment reads).
__host__ __device__ inline int skinny_xstride(int I) { return I * 2 + 16; }

// Stage columns [c0, c0+nc) (nc <= xcols) of the activations into shared memory.
template <int MODE>
__device__ __forceinline__ void skinny_stage(const SkinnyParams &p, char *xs, int c0, int nc,
                                             int row0) {
    const int chunks = p.ng * 4;  // 16-activation pieces per column
    const int xstride = skinny_xstride(p.I);
    for (int i = threadIdx.x; i < nc * chunks; i += blockDim.x) {
        const int cl = i / chunks;
        const int piece = i - cl * chunks;
        const int c = c0 + cl;
        uint32_t w[8];
        if (MODE == kMoeGateUp || MODE == kMoeDown || p.xdt == 1) {
            const uint16_t *src;
            int64_t xr;
            if (MODE == kMoeGateUp) xr = p.row_tok[row0 + c];
            else if (MODE == kMoeDown) xr = row0 + c;
            else xr = c;
            if (!in_bounds(xr, p.x_rows)) xr = 0;
            src = (const uint16_t *)p.x + xr * p.I;
            const uint4 a = *((const uint4 *)(src + piece * 16));
            const uint4 b = *((const uint4 *)(src + piece * 16 + 8));
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        } else {
            // f32 activations: column c is split `c % 3` of token c / 3, where
            // x = hi + mid + lo with each term a bf16 (hi = rn(x), mid = rn(x - hi),
            // lo = rn(x - hi - mid); the differences are exact in f32).
            const int tok = c / 3, split = c - tok * 3;
            const float4 *src = (const float4 *)((const float *)p.x + (int64_t)tok * p.I + piece * 16);
            #pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 f = src[q];
                const float fv[4] = {f.x, f.y, f.z, f.w};
                uint32_t hb[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float r = fv[e];
                    uint32_t b = bf16_bits_rn(r);
                    for (int s = 0; s < split; ++s) {
                        r = r - bf16_bits_to_f32(b);
                        b = bf16_bits_rn(r);
                    }
                    hb[e] = b;
                }
                w[q * 2 + 0] = hb[0] | (hb[1] << 16);
                w[q * 2 + 1] = hb[2] | (hb[3] << 16);
            }
        }
        uint4 *dst = (uint4 *)(xs + (int64_t)cl * xstride + piece * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

template <int MODE, int NT, int UG>
__global__ void __launch_bounds__(256) gq4_skinny_kernel(const SkinnyParams p) {
    using TR = ModeTraits<MODE>;
    constexpr int PAIR = TR::kPair;
    constexpr int NCOL = NT * 8;
    extern __shared__ __align__(16) char smem[];
    const int xstride = skinny_xstride(p.I);
    char *xs = smem;
    float *red = (float *)(smem + (int64_t)p.xcols * xstride);  // [8][PAIR*16][NCOL]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rb = p.I >> 1;  // bytes per packed row

    if (MODE == kMoeGateUp && p.zero_ptr) {
        float4 *z = (float4 *)p.zero_ptr;
        const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_n / 4;
             i += (int64_t)gridDim.x * blockDim.x)
            z[i] = zero;
    }

    const int n_units = TR::kMoe ? (*p.n_active) * p.row_tiles : p.row_tiles;
    const int gb = (warp * p.ng) >> 3, ge = ((warp + 1) * p.ng) >> 3;
    const int sng = p.sng ? p.sng : p.ng;          // scales per weight row
    const int n_out = p.rows ? p.n_out : p.O;      // output rows
    int staged_e = -1, staged_c0 = -1;

    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        int e = 0, rt = u, row0 = 0, cols;
        if (TR::kMoe) {
            const int a = u / p.row_tiles;
            rt = u - a * p.row_tiles;
            e = p.active[a];
            if (!in_bounds(e, p.n_exp)) continue;  // uniform across the block
            row0 = p.offs[e];
            cols = p.cnt[e];
        } else {
            cols = (p.xdt == 0) ? 3 * p.n_tok : p.n_tok;
        }
        const uint8_t *W0 = p.w0 + (int64_t)e * p.estride_w;
        const float *S0 = p.s0 + (int64_t)e * p.estride_s;
        const uint8_t *W1 = PAIR == 2 ? p.w1 + (int64_t)e * p.estride_w : nullptr;
        const float *S1 = PAIR == 2 ? p.s1 + (int64_t)e * p.estride_s : nullptr;
        // output rows jA, jB of this lane; their weight rows (gathered or the same)
        const int jA = rt * 16 + g, jB = jA + 8;
        int rA = jA, rB = jB;
        if (!TR::kMoe && p.rows) {
            rA = jA < n_out ? p.rows[jA] : -1;
            rB = jB < n_out ? p.rows[jB] : -1;
        }
        const bool vA = jA < n_out && rA >= 0 && rA < p.O, vB = jB < n_out && rB >= 0 && rB < p.O;

        for (int c0 = 0; c0 < cols; c0 += p.xcols) {
            const int nc = min(p.xcols, cols - c0);
            if (e != staged_e || c0 != staged_c0) {
                __syncthreads();  // previous readers of xs are done
                skinny_stage<MODE>(p, xs, c0, nc, row0);
                __syncthreads();
                staged_e = e;
                staged_c0 = c0;
            }
            // f32 activations use three staged columns per token: a pass holds whole tokens
            const int pw = (!TR::kMoe && p.xdt == 0) ? (NCOL / 3) * 3 : NCOL;
            for (int cc = 0; cc < nc; cc += pw) {
                const int ncc = min(pw, nc - cc);
                float acc[PAIR][NT][4];
                #pragma unroll
                for (int m = 0; m < PAIR; ++m)
                    #pragma unroll
                    for (int n = 0; n < NT; ++n)
                        #pragma unroll
                        for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;

                for (int G0 = gb; G0 < ge; G0 += UG) {
                    uint2 wa[PAIR][UG], wb[PAIR][UG];
                    float sa[PAIR][UG], sb[PAIR][UG];
                    #pragma unroll
                    for (int q = 0; q < UG; ++q) {
                        const int G = G0 + q;
                        const bool ok = G < ge;
                        #pragma unroll
                        for (int m = 0; m < PAIR; ++m) {
                            const uint8_t *Wm = m ? W1 : W0;
                            const float *Sm = m ? S1 : S0;
                            const int64_t off = (int64_t)G * 32 + t * 8;
                            // byte and float offsets from the tensor's start (checked build)
                            const int64_t wbase = (int64_t)e * p.estride_w, sbase = (int64_t)e * p.estride_s;
                            const bool wA = ok && vA && in_bounds(wbase + (int64_t)rA * rb + off + 7, p.w_bytes);
                            const bool wB = ok && vB && in_bounds(wbase + (int64_t)rB * rb + off + 7, p.w_bytes);
                            const bool cA = ok && vA && in_bounds(sbase + (int64_t)rA * sng + (G >> p.gshift), p.s_count);
                            const bool cB = ok && vB && in_bounds(sbase + (int64_t)rB * sng + (G >> p.gshift), p.s_count);
                            wa[m][q] = wA ? ldg_stream_u2(Wm + (int64_t)rA * rb + off) : make_uint2(0, 0);
                            wb[m][q] = wB ? ldg_stream_u2(Wm + (int64_t)rB * rb + off) : make_uint2(0, 0);
                            sa[m][q] = cA ? ldg_f32(Sm + (int64_t)rA * sng + (G >> p.gshift)) : 0.f;
                            sb[m][q] = cB ? ldg_f32(Sm + (int64_t)rB * sng + (G >> p.gshift)) : 0.f;
                        }
                    }
                    #pragma unroll
                    for (int q = 0; q < UG; ++q) {
                        const int G = G0 + q;
                        if (G >= ge) break;
                        // A fragments: r[2j] / r[2j+1] are the two bf16x2 pairs of step j
                        uint32_t ra[PAIR][8], rbv[PAIR][8];
                        #pragma unroll
                        for (int m = 0; m < PAIR; ++m) {
                            #pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                ra[m][i] = nib2_to_bf16x2(wa[m][q].x >> (4 * i));
                                ra[m][4 + i] = nib2_to_bf16x2(wa[m][q].y >> (4 * i));
                                rbv[m][i] = nib2_to_bf16x2(wb[m][q].x >> (4 * i));
                                rbv[m][4 + i] = nib2_to_bf16x2(wb[m][q].y >> (4 * i));
                            }
                        }
                        #pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            if (n * 8 >= ncc) break;  // warp-uniform: no op for empty n-tiles
                            const int cl = cc + n * 8 + g;  // staged column this lane feeds
                            uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
                            if (n * 8 + g < ncc) {
                                const uint4 *src = (const uint4 *)(xs + (int64_t)cl * xstride + (G * 4 + t) * 32);
                                b0 = src[0];
                                b1 = src[1];
                            }
                            const uint32_t bf[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                            #pragma unroll
                            for (int m = 0; m < PAIR; ++m) {
                                float d[4] = {0.f, 0.f, 0.f, 0.f};
                                #pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const uint32_t a[4] = {ra[m][2 * j], rbv[m][2 * j], ra[m][2 * j + 1], rbv[m][2 * j + 1]};
                                    mma_bf16_16816(d, a, bf[2 * j], bf[2 * j + 1], d);
                                }
                                acc[m][n][0] = fmaf(sa[m][q], d[0], acc[m][n][0]);
                                acc[m][n][1] = fmaf(sa[m][q], d[1], acc[m][n][1]);
                                acc[m][n][2] = fmaf(sb[m][q], d[2], acc[m][n][2]);
                                acc[m][n][3] = fmaf(sb[m][q], d[3], acc[m][n][3]);
                            }
                        }
                    }
                }
                // cross-warp reduction of the 8 partial tiles (fixed order)
                #pragma unroll
                for (int m = 0; m < PAIR; ++m)
                    #pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        float *r0 = red + ((warp * PAIR + m) * 16 + g) * NCOL + n * 8 + 2 * t;
                        r0[0] = acc[m][n][0];
                        r0[1] = acc[m][n][1];
                        r0[8 * NCOL] = acc[m][n][2];
                        r0[8 * NCOL + 1] = acc[m][n][3];
                    }
                __syncthreads();
                if (!TR::kMoe && p.xdt == 0) {
                    // f32 activations: three staged columns per token
                    const int ntok = ncc / 3;
                    for (int i = threadIdx.x; i < 16 * ntok; i += blockDim.x) {
                        const int row = i & 15, tl = i >> 4;
                        const int o = rt * 16 + row;
                        if (o >= n_out) continue;
                        const int tok = (c0 + cc) / 3 + tl;
                        float v[PAIR];
                        #pragma unroll
                        for (int m = 0; m < PAIR; ++m) {
                            float s = 0.f;
                            for (int sp = 0; sp < 3; ++sp)
                                for (int w = 0; w < 8; ++w)
                                    s += red[((w * PAIR + m) * 16 + row) * NCOL + tl * 3 + sp];
                            v[m] = s;
                        }
                        if (p.rows && (p.rows[o] < 0 || p.rows[o] >= p.O)) v[0] = __uint_as_float(0x7fc00000u);
                        if (MODE == kMatvec)
                            p.y[(int64_t)tok * n_out + o] = v[0];
                        else
                            ((float *)p.h)[(int64_t)tok * n_out + o] = silu_mul(v[0], v[PAIR - 1]);
                    }
                } else {
                    for (int i = threadIdx.x; i < 16 * ncc; i += blockDim.x) {
                        const int row = i & 15, cl = i >> 4;
                        const int o = rt * 16 + row;
                        if (o >= n_out) continue;
                        float v[PAIR];
                        #pragma unroll
                        for (int m = 0; m < PAIR; ++m) {
                            float s = 0.f;
                            for (int w = 0; w < 8; ++w) s += red[((w * PAIR + m) * 16 + row) * NCOL + cl];
                            v[m] = s;
                        }
                        const int c = c0 + cc + cl;
                        if (!TR::kMoe && p.rows && (p.rows[o] < 0 || p.rows[o] >= p.O))
                            v[0] = __uint_as_float(0x7fc00000u);
                        if (MODE == kMatvec) {
                            p.y[(int64_t)c * n_out + o] = v[0];
                        } else if (MODE == kGateUp) {
                            ((uint16_t *)p.h)[(int64_t)c * n_out + o] = (uint16_t)bf16_bits_rn(silu_mul(v[0], v[1]));
                        } else if (MODE == kMoeGateUp) {
                            ((uint16_t *)p.h)[(int64_t)(row0 + c) * p.O + o] = (uint16_t)bf16_bits_rn(silu_mul(v[0], v[1]));
                        } else {  // kMoeDown: weighted scatter-add into y
                            const int r = row0 + c;
                            const float wt = p.wts[p.row_slot[r]];
                            const int tok = p.row_tok[r];
                            if (in_bounds(tok, p.n_tok)) atomicAdd(p.y + (int64_t)tok * p.O + o, wt * v[0]);
                        }
                    }
                }
                __syncthreads();  // red is rewritten by the next pass
            }
        }
    }
}

}  // namespace gq4

// ======================================================================================
// Row-band decode kernel (3 or more activation columns per matrix/expert).
//
// A CTA owns a band of 8 row tiles (one per warp; 128 rows, or 128 gate + 128 up rows)
// of one matrix/expert for all of K, so the activations of the expert's rows are read
// once per band instead of once per row tile, and no cross-warp reduction is needed:
//  * activations: chunks of kBandKC groups (512 columns) of the expert's rows, one bulk
//    copy per row (the copy's source does the token gather), double-buffered, completion
//    on an mbarrier with a transaction count;
//  * weights and scales: each warp streams its own 16-row tiles through a private
//    kBandDW-stage shared-memory ring with cp.async (rows past O are zero-filled), kBandDW-1
//    groups ahead of the tensor ops;
//  * products: the same nibble decode and m16n8k16 fragments as the split-K kernel.
// ======================================================================================
namespace gq4 {

constexpr int kBandKC = 8;      // groups per activation chunk
constexpr int kBandDW = 8;      // per-warp weight ring depth (groups)
constexpr int kBandMaxCols = 32;
__host__ __device__ inline int band_xstride() { return kBandKC * 64 * 2 + 16; }  // bytes per staged row
__host__ __device__ inline int band_wstage(int pair) { return pair * (16 * 32 + 16 * 4); }
__host__ __device__ inline size_t band_smem(int pair) {
    return (size_t)2 * kBandMaxCols * band_xstride() + (size_t)8 * kBandDW * band_wstage(pair) + 64;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
// Bounded wait (about two seconds of SM cycles); false if it gave up.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t ok;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
                     " selp.u32 %0, 1, 0, p;\n}\n" : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        if (ok) return true;
        if (clock64() - t0 > 4000000000ll) return false;
    }
}

template <int MODE, int NT>
__global__ void __launch_bounds__(256) gq4_band_kernel(const SkinnyParams p, int32_t *status) {
    using TR = ModeTraits<MODE>;
    constexpr int PAIR = TR::kPair;
    extern __shared__ __align__(128) uint8_t bsm[];
    const int xstride = band_xstride();
    uint8_t *xbuf = bsm;                                                   // [2][32 rows][xstride]
    uint8_t *wring = bsm + 2 * kBandMaxCols * xstride;                     // [8 warps][DW][stage]
    const uint32_t xbar = smem_addr(wring + 8 * kBandDW * band_wstage(PAIR)); // 2 mbarriers
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rb = p.I >> 1;
    const int wst = band_wstage(PAIR);
    uint8_t *myring = wring + warp * kBandDW * wst;
    const int bands = (p.row_tiles + 7) >> 3;
    const int nchunks = (p.ng + kBandKC - 1) / kBandKC;

    if (threadIdx.x == 0) {
        bar_init(xbar, 1);
        bar_init(xbar + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (MODE == kMoeGateUp && p.zero_ptr) {
        float4 *z = (float4 *)p.zero_ptr;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_n / 4;
             i += (int64_t)gridDim.x * blockDim.x)
            z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();

    const int n_units = TR::kMoe ? (*p.n_active) * bands : bands;
    uint32_t xphase[2] = {0u, 0u};
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        int e = 0, band = u, row0 = 0, cols = p.n_tok;
        if (TR::kMoe) {
            const int a = u / bands;
            band = u - a * bands;
            e = p.active[a];
            if (!in_bounds(e, p.n_exp)) continue;  // uniform across the block
            row0 = p.offs[e];
            cols = p.cnt[e];
        }
        const int rt = band * 8 + warp;          // this warp's row tile
        const bool tile_ok = rt < p.row_tiles;
        const uint8_t *W0 = p.w0 + (int64_t)e * p.estride_w;
        const float *S0 = p.s0 + (int64_t)e * p.estride_s;
        const uint8_t *W1 = PAIR == 2 ? p.w1 + (int64_t)e * p.estride_w : nullptr;
        const float *S1 = PAIR == 2 ? p.s1 + (int64_t)e * p.estride_s : nullptr;

        for (int c0 = 0; c0 < cols; c0 += kBandMaxCols) {
            const int nc = min(kBandMaxCols, cols - c0);
            // weight prefetch of group G into ring slot G % DW (one commit group per group)
            auto issue_w = [&](int G) {
                if (G < p.ng && tile_ok) {
                    uint8_t *st = myring + (G % kBandDW) * wst;
                    #pragma unroll
                    for (int m = 0; m < PAIR; ++m) {
                        const uint8_t *Wm = m ? W1 : W0;
                        const float *Sm = m ? S1 : S0;
                        const int row = rt * 16 + (lane >> 1);
                        const int64_t woff = (int64_t)row * rb + (int64_t)G * 32 + (lane & 1) * 16;
                        const bool rv = row < p.O && in_bounds((int64_t)e * p.estride_w + woff + 15, p.w_bytes);
                        const uint8_t *src = Wm + (rv ? woff : 0);
                        cp_async16(smem_addr(st + m * 576 + (lane >> 1) * 32 + (lane & 1) * 16), src, rv ? 16u : 0u);
                        if (lane < 16) {
                            const int srow = rt * 16 + lane;
                            const int64_t soff = (int64_t)srow * p.ng + G;
                            const bool sv = srow < p.O && in_bounds((int64_t)e * p.estride_s + soff, p.s_count);
                            cp_async4(smem_addr(st + m * 576 + 512 + lane * 4), Sm + (sv ? soff : 0), sv ? 4u : 0u);
                        }
                    }
                }
                cp_async_commit();  // possibly empty: keeps the group count uniform
            };
            // activation chunk c of rows [c0, c0+nc) into buffer c & 1
            auto issue_x = [&](int c) {
                if (c < nchunks && warp == 0) {
                    const int k0 = c * kBandKC * 64;
                    const int kn = min(kBandKC * 64, p.I - k0);
                    const uint32_t bar = xbar + 8 * (c & 1);
                    if (lane == 0) bar_expect_tx(bar, (uint32_t)(nc * kn * 2));
                    __syncwarp();
                    for (int r = lane; r < nc; r += 32) {
                        const int col = c0 + r;
                        int64_t xr;
                        if (MODE == kMoeGateUp) xr = p.row_tok[row0 + col];
                        else if (MODE == kMoeDown) xr = row0 + col;
                        else xr = col;
                        if (!in_bounds(xr, p.x_rows)) xr = 0;  // the copy must still deliver its bytes
                        const uint16_t *src = (const uint16_t *)p.x + xr * p.I + k0;
                        bulk_g2s(smem_addr(xbuf + ((c & 1) * kBandMaxCols + r) * xstride), src, kn * 2, bar);
                    }
                }
            };

            float acc[PAIR][NT][4];
            #pragma unroll
            for (int m = 0; m < PAIR; ++m)
                #pragma unroll
                for (int n = 0; n < NT; ++n)
                    #pragma unroll
                    for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;

            issue_x(0);
            #pragma unroll
            for (int G = 0; G < kBandDW - 1; ++G) issue_w(G);
            for (int c = 0; c < nchunks; ++c) {
                issue_x(c + 1);
                const uint32_t bar = xbar + 8 * (c & 1);
                const bool late = !bar_wait(bar, xphase[c & 1]);
                xphase[c & 1] ^= 1u;
                const uint8_t *xc = xbuf + (c & 1) * kBandMaxCols * xstride;
                const int gend = min(p.ng, (c + 1) * kBandKC);
                for (int G = c * kBandKC; G < gend; ++G) {
                    __syncwarp();                  // slot (G-1) % DW is read by every lane
                    issue_w(G + kBandDW - 1);
                    cp_async_wait<kBandDW - 1>();  // group G has landed (this thread's copies)
                    __syncwarp();                  // ... and every lane's
                    if (!tile_ok) continue;
                    const uint8_t *st = myring + (G % kBandDW) * wst;
                    const int gl = G - c * kBandKC;
                    uint32_t ra[PAIR][8], rbv[PAIR][8];
                    float sa[PAIR], sb[PAIR];
                    #pragma unroll
                    for (int m = 0; m < PAIR; ++m) {
                        const uint2 wa = *(const uint2 *)(st + m * 576 + g * 32 + t * 8);
                        const uint2 wb = *(const uint2 *)(st + m * 576 + (g + 8) * 32 + t * 8);
                        sa[m] = *(const float *)(st + m * 576 + 512 + g * 4);
                        sb[m] = *(const float *)(st + m * 576 + 512 + (g + 8) * 4);
                        #pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            ra[m][i] = nib2_to_bf16x2(wa.x >> (4 * i));
                            ra[m][4 + i] = nib2_to_bf16x2(wa.y >> (4 * i));
                            rbv[m][i] = nib2_to_bf16x2(wb.x >> (4 * i));
                            rbv[m][4 + i] = nib2_to_bf16x2(wb.y >> (4 * i));
                        }
                    }
                    #pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        if (n * 8 >= nc) break;  // warp-uniform
                        uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
                        if (n * 8 + g < nc) {
                            const uint4 *src = (const uint4 *)(xc + (n * 8 + g) * xstride + (gl * 4 + t) * 32);
                            b0 = src[0];
                            b1 = src[1];
                        }
                        const uint32_t bf[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        #pragma unroll
                        for (int m = 0; m < PAIR; ++m) {
                            float d[4] = {0.f, 0.f, 0.f, 0.f};
                            #pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint32_t a[4] = {ra[m][2 * j], rbv[m][2 * j], ra[m][2 * j + 1], rbv[m][2 * j + 1]};
                                mma_bf16_16816(d, a, bf[2 * j], bf[2 * j + 1], d);
                            }
                            acc[m][n][0] = fmaf(sa[m], d[0], acc[m][n][0]);
                            acc[m][n][1] = fmaf(sa[m], d[1], acc[m][n][1]);
                            acc[m][n][2] = fmaf(sb[m], d[2], acc[m][n][2]);
                            acc[m][n][3] = fmaf(sb[m], d[3], acc[m][n][3]);
                        }
                    }
                }
                // every warp is done with buffer c & 1; a wait that gave up anywhere ends
                // the CTA (GQ4_ERR_TIMEOUT) once the copies it issued have landed or timed out
                if (__syncthreads_or(late)) {
                    if (threadIdx.x == 0 && status) atomicOr(status, 8);
                    bar_wait(bar, xphase[c & 1] ^ 1u);
                    if (c + 1 < nchunks) bar_wait(xbar + 8 * ((c + 1) & 1), xphase[(c + 1) & 1]);
                    cp_async_wait<0>();
                    return;
                }
            }
            cp_async_wait<0>();
            // ---------------------------------------------------------------- epilogue
            if (tile_ok) {
                #pragma unroll
                for (int n = 0; n < NT; ++n) {
                    #pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int cl = n * 8 + 2 * t + (i & 1);
                        const int o = rt * 16 + g + ((i >> 1) << 3);
                        if (cl >= nc || o >= p.O) continue;
                        const int c = c0 + cl;
                        if (MODE == kMatvec) {
                            p.y[(int64_t)c * p.O + o] = acc[0][n][i];
                        } else if (MODE == kGateUp) {
                            ((uint16_t *)p.h)[(int64_t)c * p.O + o] =
                                (uint16_t)bf16_bits_rn(silu_mul(acc[0][n][i], acc[PAIR - 1][n][i]));
                        } else if (MODE == kMoeGateUp) {
                            ((uint16_t *)p.h)[(int64_t)(row0 + c) * p.O + o] =
                                (uint16_t)bf16_bits_rn(silu_mul(acc[0][n][i], acc[PAIR - 1][n][i]));
                        } else {
                            const int r = row0 + c;
                            const int tok = p.row_tok[r];
                            if (in_bounds(tok, p.n_tok))
                                atomicAdd(p.y + (int64_t)tok * p.O + o, p.wts[p.row_slot[r]] * acc[0][n][i]);
                        }
                    }
                }
            }
        }
    }
}

}  // namespace gq4
