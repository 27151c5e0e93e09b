// gq4_mla.cuh -- grouped-scale MLA absorb projections over the kv_b tensor.
//
// colibri PR #298, "fmt=4 CUDA attention crash — root cause": the two MLA attention
// absorb kernels multiply weights of the kv_b tensor (28,672 rows x 512 latent inputs,
// 8 groups of 64 per row) by their scale.  With fmt=4 the scale of weight (row, k) is
// scales[row*ng + k/gs], taken inside the accumulation loop; the fmt=2 rule (one scale
// per row, applied after the loop) indexed the O*ng buffer by row.  These kernels run the
// two projections on their own, outside attention:
//   Q absorb: q_lat[t][h][c] = sum_{d<dn} q_nope[t][h][d] * w(h*D + d, c),     c < R
//   V absorb: o[t][h][v]     = sum_{c<R}  lat[t][h][c]   * w(h*D + dn + v, c), v < dv
// with D = dn + dv: the rows of kv_b come in per-head blocks, dn key rows then dv value
// rows, and R (the latent width) is the tensor's input dimension.
// Both read each packed word once with coalesced 4-byte loads; the pages' tensor is
// 8.26 MB with its scales, so they are latency- more than bandwidth-bound.  fp32
// accumulation; each group's scale multiplies that group's partial (V) or the token's
// coefficient of that row and group (Q), never a rounded weight.
#pragma once
#include "gq4_aux.cuh"

namespace gq4 {

constexpr int kMlaTok = 4;        // tokens per block
constexpr int kMlaThreads = 256;
constexpr int kMlaVRowsPerWarp = 4;
constexpr int kMlaMaxR = 2048;    // latent width: the V kernel stages kMlaTok x R floats
constexpr int kMlaMaxDn = 1024;   // key rows per head: the Q kernel stages kMlaTok x dn floats

template <int XDT>  // 0: f32, 1: bf16
__device__ __forceinline__ float mla_act(const void *x, int64_t i) {
    if (XDT == 0) return ((const float *)x)[i];
    return __uint_as_float((uint32_t)((const uint16_t *)x)[i] << 16);
}

// Q absorb.  Block: one head, kMlaTok tokens and one slice of the head's key rows
// (blockIdx.z of gridDim.z slices; with more than one slice the block adds its partial
// sums into the zeroed output with atomics, in no fixed order).  With W = R/8 packed words
// per row, the block has W x nsplit threads (nsplit = 256 / W when W <= 256, else 256
// threads over the words in turn): thread (split, j) owns columns 8j..8j+7 (one device
// word, all in one group since gs % 8 == 0) and sums the slice's key rows d = d0 + split,
// d0 + split + nsplit, ...; the splits' partial sums are added in shared memory in split
// order.
template <int XDT>
__global__ void __launch_bounds__(kMlaThreads) gq4_mla_q_kernel(const uint32_t *__restrict__ w,
                                                              const float *__restrict__ s, int R, int ng,
                                                              int gs, int nh, int dn, int dv,
                                                              const void *__restrict__ q, int64_t T,
                                                              float *__restrict__ out) {
    extern __shared__ float mla_sm[];
    const int h = blockIdx.x;
    const int64_t t0 = (int64_t)blockIdx.y * kMlaTok;
    const int nt = (int)min((int64_t)kMlaTok, T - t0);
    const int W = R >> 3;
    const bool wide = W >= (int)blockDim.x;
    const int nsplit = wide ? 1 : (int)blockDim.x / W;
    const int split = wide ? 0 : (int)threadIdx.x / W;
    const int dper = (dn + gridDim.z - 1) / gridDim.z;
    const int d0 = blockIdx.z * dper, d1 = min(dn, d0 + dper);
    const bool atomic_out = gridDim.z > 1;
    float *qs = mla_sm;                 // [kMlaTok][dn]
    float *red = mla_sm + kMlaTok * dn; // [nsplit][kMlaTok][R] (nsplit > 1)
    for (int i = threadIdx.x; i < kMlaTok * dn; i += blockDim.x) {
        const int t = i / dn, d = i - t * dn;
        qs[i] = t < nt ? mla_act<XDT>(q, ((t0 + t) * nh + h) * (int64_t)dn + d) : 0.f;
    }
    __syncthreads();
    const int64_t D = dn + dv;
    const int jstep = wide ? (int)blockDim.x : W;
    for (int j = wide ? (int)threadIdx.x : (int)threadIdx.x % W; j < W && split < nsplit; j += jstep) {
        float acc[kMlaTok][8];
        #pragma unroll
        for (int t = 0; t < kMlaTok; ++t)
            #pragma unroll
            for (int m = 0; m < 8; ++m) acc[t][m] = 0.f;
        const int g = (8 * j) / gs;
        #pragma unroll 4
        for (int d = d0 + split; d < d1; d += nsplit) {
            const int64_t row = (int64_t)h * D + d;
            const int64_t wix = row * W + j, six = row * ng + g;
            const uint32_t v = in_bounds(wix, (int64_t)nh * D * W) ? __ldg(w + wix) : 0u;
            const float sc = in_bounds(six, (int64_t)nh * D * ng) ? __ldg(s + six) : 0.f;
            float qv[8];
            #pragma unroll
            for (int m = 0; m < 8; ++m) qv[m] = (float)dev_q(v, dev_slot(m));
            #pragma unroll
            for (int t = 0; t < kMlaTok; ++t) {
                const float a = qs[t * dn + d] * sc;
                #pragma unroll
                for (int m = 0; m < 8; ++m) acc[t][m] = fmaf(a, qv[m], acc[t][m]);
            }
        }
        if (nsplit == 1) {
            #pragma unroll
            for (int t = 0; t < kMlaTok; ++t) {
                if (t >= nt) break;
                float *o = out + ((t0 + t) * nh + h) * (int64_t)R + 8 * j;
                if (atomic_out) {
                    #pragma unroll
                    for (int m = 0; m < 8; ++m) atomicAdd(o + m, acc[t][m]);
                } else {
                    ((float4 *)o)[0] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
                    ((float4 *)o)[1] = make_float4(acc[t][4], acc[t][5], acc[t][6], acc[t][7]);
                }
            }
        } else {
            #pragma unroll
            for (int t = 0; t < kMlaTok; ++t) {
                float4 *o = (float4 *)(red + ((int64_t)split * kMlaTok + t) * R + 8 * j);
                o[0] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
                o[1] = make_float4(acc[t][4], acc[t][5], acc[t][6], acc[t][7]);
            }
        }
    }
    if (nsplit > 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < nt * R; i += blockDim.x) {
            const int t = i / R, c = i - t * R;
            float sum = 0.f;
            for (int sp = 0; sp < nsplit; ++sp) sum += red[((int64_t)sp * kMlaTok + t) * R + c];
            float *o = out + ((t0 + t) * nh + h) * (int64_t)R + c;
            if (atomic_out) atomicAdd(o, sum); else *o = sum;
        }
    }
}

// V absorb.  Block: one head, kMlaTok tokens (blockIdx.z) and 8 warps of kMlaVRowsPerWarp
// value rows each (blockIdx.y).  A warp's lanes take the words j = lane, lane+32, ... of
// all its rows at once (coalesced), form each word's partial against the staged latent
// values, scale it by the word's group scale, and the lanes' sums meet in a shuffle
// reduction per row and token.
template <int XDT>
__global__ void __launch_bounds__(kMlaThreads) gq4_mla_v_kernel(const uint32_t *__restrict__ w,
                                                              const float *__restrict__ s, int R, int ng,
                                                              int gs, int nh, int dn, int dv,
                                                              const void *__restrict__ lat, int64_t T,
                                                              float *__restrict__ out) {
    extern __shared__ float mla_sm[];  // [kMlaTok][R]
    const int h = blockIdx.x;
    const int64_t t0 = (int64_t)blockIdx.z * kMlaTok;
    const int nt = (int)min((int64_t)kMlaTok, T - t0);
    for (int i = threadIdx.x; i < kMlaTok * R; i += blockDim.x) {
        const int t = i / R, c = i - t * R;
        mla_sm[i] = t < nt ? mla_act<XDT>(lat, ((t0 + t) * nh + h) * (int64_t)R + c) : 0.f;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = R >> 3;
    const int64_t D = dn + dv;
    const int v0 = (blockIdx.y * (kMlaThreads / 32) + warp) * kMlaVRowsPerWarp;
    const int nv = min(kMlaVRowsPerWarp, dv - v0);  // rows of this warp (may be <= 0)
    // the warp's rows are walked together so their loads are in flight at the same time
    float acc[kMlaVRowsPerWarp][kMlaTok];
    #pragma unroll
    for (int r = 0; r < kMlaVRowsPerWarp; ++r)
        #pragma unroll
        for (int t = 0; t < kMlaTok; ++t) acc[r][t] = 0.f;
    for (int j = lane; j < W && nv > 0; j += 32) {
        uint32_t word[kMlaVRowsPerWarp];
        float sc[kMlaVRowsPerWarp];
        #pragma unroll
        for (int r = 0; r < kMlaVRowsPerWarp; ++r) {
            const int64_t row = (int64_t)h * D + dn + v0 + min(r, nv - 1);
            const int64_t wix = row * W + j, six = row * ng + (8 * j) / gs;
            word[r] = in_bounds(wix, (int64_t)nh * D * W) ? __ldg(w + wix) : 0u;
            sc[r] = in_bounds(six, (int64_t)nh * D * ng) ? __ldg(s + six) : 0.f;
        }
        float qv[kMlaVRowsPerWarp][8];  // the words decoded once, used by every token
        #pragma unroll
        for (int r = 0; r < kMlaVRowsPerWarp; ++r)
            #pragma unroll
            for (int m = 0; m < 8; ++m) qv[r][m] = (float)dev_q(word[r], dev_slot(m));
        #pragma unroll
        for (int t = 0; t < kMlaTok; ++t) {
            const float4 a = *(const float4 *)(mla_sm + t * R + 8 * j);
            const float4 b = *(const float4 *)(mla_sm + t * R + 8 * j + 4);
            #pragma unroll
            for (int r = 0; r < kMlaVRowsPerWarp; ++r) {
                float part = qv[r][0] * a.x;
                part = fmaf(qv[r][1], a.y, part);
                part = fmaf(qv[r][2], a.z, part);
                part = fmaf(qv[r][3], a.w, part);
                part = fmaf(qv[r][4], b.x, part);
                part = fmaf(qv[r][5], b.y, part);
                part = fmaf(qv[r][6], b.z, part);
                part = fmaf(qv[r][7], b.w, part);
                acc[r][t] = fmaf(sc[r], part, acc[r][t]);
            }
        }
    }
    #pragma unroll
    for (int r = 0; r < kMlaVRowsPerWarp; ++r)
        #pragma unroll
        for (int t = 0; t < kMlaTok; ++t)
            #pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], off);
    if (lane == 0) {
        #pragma unroll
        for (int r = 0; r < kMlaVRowsPerWarp; ++r)
            #pragma unroll
            for (int t = 0; t < kMlaTok; ++t)
                if (r < nv && t < nt) out[((t0 + t) * nh + h) * (int64_t)dv + v0 + r] = acc[r][t];
    }
}

}  // namespace gq4
