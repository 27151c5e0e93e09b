// gq4_tc.cuh -- many-tokens-per-expert grouped-int4 GEMM on the 5th-generation tensor
// cores (tcgen05 + TMEM), for the prefill regime of the routed-expert FFN.
//
// Per expert e with cnt rows (tokens) and an M tile of 128 weight rows:
//   D[row][n] = sum_g s[row][g] * sum_{k in g} q[row][k] * X[n][k]
// (colibri PR #298: w = scale[o*ng + k/gs] * q, gs = 64).  The per-group scale must not
// be folded into a bf16 weight (bf16(s*q) loses ~3 bits per weight), so:
//   * q is turned into bf16 exactly (integers -8..7) by the math warps and written to
//     shared memory in the 128-byte-swizzled K-major layout the MMA reads;
//   * for each 64-wide group the MMA warp issues four M=128 x N x K=16 tcgen05.mma into
//     one of two TMEM partial buffers (accumulate off for the first), then commits;
//   * the math warps load the partial (tcgen05.ld), multiply it by the row's scale of
//     that group and add it to running sums kept in registers ("promotion"), then free
//     the buffer -- the MMA of group g+1 overlaps the promotion of group g.
// TMEM lane = weight row, so the scale is one register per thread and group.
//
// Warp roles (320 threads, one CTA per SM, persistent over units):
//   warp 0      TMA producer: packed nibble tile (128 rows x 32 B) and the activation
//               tile (N <= 192 rows x 64 bf16, swizzle 128B) of each group into a 4-stage ring
//   warp 1      TMEM allocation and the MMA issuer (one thread)
//   warps 2-9   math: dequantise rows [16m, 16m+16) of the A tile, promote the TMEM
//               partials of their lane quarter / column half, epilogue
// Units: (large expert, M tile).  gate+up: an M tile is 64 gate rows + the same 64 up
// rows, interleaved (A row 2i = gate row i, 2i+1 = up row i), so g and u of one output
// sit in adjacent TMEM lanes of one warp and SiLU(g)*u needs one shuffle; down: 128 rows
// of the down matrix, then a weighted scatter-add into y.
// Every mbarrier wait is bounded (~2 s on the global timer): on expiry the kernel raises
// GQ4_ERR_TIMEOUT in the status word, all roles leave their loops, TMEM is freed.
#pragma once
#include <cuda.h>

#include "gq4_common.cuh"

namespace gq4 {

constexpr int kTcThreads = 320;
constexpr int kTcStages = 4;
constexpr int kTcAStages = 3;
constexpr int kTcMaxN = 192;                                   // rows per pass (TMEM, registers)
constexpr int kTcChunks = kTcMaxN / 64;                         // 32-column chunks per column half
constexpr int kTcPackedBytes = 128 * 32;                        // 128 rows x 64 nibbles
constexpr int kTcXBytes = kTcMaxN * 128;                        // N rows x 64 bf16
constexpr int kTcStageBytes = kTcPackedBytes + kTcXBytes;       // 36 KB, 1024-aligned
constexpr int kTcABytes = 128 * 128;                            // 128 rows x 64 bf16
constexpr int kTcOffA = kTcStages * kTcStageBytes;
constexpr int kTcOffBar = kTcOffA + kTcAStages * kTcABytes;
constexpr int kTcSmemBytes = kTcOffBar + 256 + 1024;            // + 1024 for alignment
constexpr int kTcTmemCols = 512;                                // two N<=192 partials (power of 2)
constexpr int kStatusTimeout = 8;                               // GQ4_ERR_TIMEOUT

struct TcParams {
    const float *s0;     // scales: gate (gate+up) or down, [E][O][ng]
    const float *s1;     // up scales (gate+up)
    int64_t estride_s;   // floats between experts
    int O, I, ng;        // rows per expert (F for gate+up, H for down), K, groups
    int m_tiles;         // M tiles per expert
    int estride_rows;    // packed rows between experts in the TMA view of the weights
    const int32_t *offs, *cnt, *n_large, *large, *row_tok, *row_slot;
    const float *wts;
    uint16_t *h;         // gate+up output, bf16 [T*K][O] in row-map order
    float *y;            // down output [T][O], accumulated
    int32_t *status;     // device status word
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `parity` to complete; false if the CTA aborted or ~2 s passed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > 2000000000ull) {
                *abort_flag = 1;
                atomicOr(status, kStatusTimeout);
                return false;
            }
        }
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor: bf16 x bf16 -> f32, both K-major, M = 128, N.
__device__ __forceinline__ uint32_t idesc_bf16_m128(int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- the kernel
template <int MODE>  // 0: gate+up with SiLU(g)*u -> h (bf16); 1: down -> y += w * D
__global__ void __launch_bounds__(kTcThreads, 1)
gq4_tc_kernel(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
              const __grid_constant__ CUtensorMap tm_x, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + kTcOffBar;
    auto full_bar = [&](int s) { return bar0 + 8 * s; };
    auto empty_bar = [&](int s) { return bar0 + 32 + 8 * s; };
    auto afull_bar = [&](int a) { return bar0 + 64 + 8 * a; };
    auto aempty_bar = [&](int a) { return bar0 + 88 + 8 * a; };
    auto pfull_bar = [&](int b) { return bar0 + 112 + 8 * b; };
    auto pempty_bar = [&](int b) { return bar0 + 128 + 8 * b; };
    uint32_t *tmem_slot = (uint32_t *)(smem + kTcOffBar + 160);
    volatile int *abort_flag = (volatile int *)(smem + kTcOffBar + 168);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1 + 8);
        }
        for (int a = 0; a < kTcAStages; ++a) {
            mbar_init(afull_bar(a), 8);
            mbar_init(aempty_bar(a), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(pfull_bar(b), 1);
            mbar_init(pempty_bar(b), 8);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTcTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_units = (*p.n_large) * p.m_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                const int a = u / p.m_tiles, mt = u - a * p.m_tiles;
                const int e = p.large[a];
                const int row0 = p.offs[e], cnt = p.cnt[e];
                const int wrow = e * p.estride_rows + (MODE == 0 ? mt * 64 : mt * 128);
                for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                    const int N = (min(kTcMaxN, cnt - n0) + 15) & ~15;
                    for (int G = 0; G < p.ng; ++G, ++it) {
                        const int s = it % kTcStages;
                        if (!(ok = mbar_wait(empty_bar(s), ((it / kTcStages) & 1) ^ 1, abort_flag, p.status)))
                            break;
                        const uint32_t dst = sb + s * kTcStageBytes;
                        mbar_expect_tx(full_bar(s), kTcPackedBytes + N * 128);
                        if (MODE == 0) {
                            tma_load_2d(dst, &tm_w0, G * 32, wrow, full_bar(s));
                            tma_load_2d(dst + 2048, &tm_w1, G * 32, wrow, full_bar(s));
                        } else {
                            tma_load_2d(dst, &tm_w0, G * 32, wrow, full_bar(s));
                            tma_load_2d(dst + 2048, &tm_w0, G * 32, wrow + 64, full_bar(s));
                        }
                        for (int r = 0; r < N; r += 16)
                            tma_load_2d(dst + kTcPackedBytes + r * 128, &tm_x, G * 64, row0 + n0 + r,
                                        full_bar(s));
                    }
                }
            }
            if (!ok) {  // let copies already issued land before the CTA leaves
                for (uint32_t j = it > kTcStages ? it - kTcStages : 0; j < it; ++j) {
                    const uint64_t t0 = global_ns();
                    while (!mbar_try_wait(full_bar(j % kTcStages), (j / kTcStages) & 1) &&
                           global_ns() - t0 < 100000000ull) {
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                const int a = u / p.m_tiles;
                const int e = p.large[a];
                const int cnt = p.cnt[e];
                for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                    const int N = (min(kTcMaxN, cnt - n0) + 15) & ~15;
                    const uint32_t idesc = idesc_bf16_m128(N);
                    for (int G = 0; G < p.ng; ++G, ++it) {
                        const int s = it % kTcStages, as = it % kTcAStages, b = it & 1;
                        ok = mbar_wait(full_bar(s), (it / kTcStages) & 1, abort_flag, p.status) &&
                             mbar_wait(afull_bar(as), (it / kTcAStages) & 1, abort_flag, p.status) &&
                             mbar_wait(pempty_bar(b), ((it >> 1) & 1) ^ 1, abort_flag, p.status);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t a_addr = sb + kTcOffA + as * kTcABytes;
                        const uint32_t x_addr = sb + s * kTcStageBytes + kTcPackedBytes;
                        #pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma(tmem + b * 256, sw128_desc(a_addr + kk * 32),
                                   sw128_desc(x_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
                        tc_commit(pfull_bar(b));
                        tc_commit(aempty_bar(as));
                        tc_commit(empty_bar(s));
                    }
                }
            }
            // the last commits must have arrived before the CTA's shared memory is released
            if (ok && it > 0) {
                const uint32_t j = it - 1;
                mbar_wait(empty_bar(j % kTcStages), (j / kTcStages) & 1, abort_flag, p.status);
                mbar_wait(aempty_bar(j % kTcAStages), (j / kTcAStages) & 1, abort_flag, p.status);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ math warps
        const int m = warp - 2;            // 0..7: A rows [16m, 16m+16)
        const int q = warp & 3;            // TMEM lane quarter this warp may access
        const int half = m >> 2;           // column half: 32-column chunks 2c + half
        const int lrow = 32 * q + lane;    // TMEM lane = A row owned in the promotion
        const int drow = 16 * m + (lane >> 1), dkh = lane & 1;  // dequant: A row, k half
        // packed tile rows: [0,64) first box, [64,128) second; gate+up interleaves them
        const int prow = MODE == 0 ? ((drow & 1) ? 64 + (drow >> 1) : (drow >> 1)) : drow;
        uint32_t it = 0;
        bool ok = true;
        float acc[kTcChunks][32];

        auto dequant = [&](uint32_t i) -> bool {
            const int s = i % kTcStages, as = i % kTcAStages;
            if (!mbar_wait(full_bar(s), (i / kTcStages) & 1, abort_flag, p.status)) return false;
            if (!mbar_wait(aempty_bar(as), ((i / kTcAStages) & 1) ^ 1, abort_flag, p.status)) return false;
            const uint4 w = *(const uint4 *)(smem + s * kTcStageBytes + prow * 32 + dkh * 16);
            uint8_t *arow = smem + kTcOffA + as * kTcABytes + drow * 128;
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = dkh * 4 + j;  // 16-byte chunk = columns 8c..8c+7
                uint4 o;
                o.x = nib2_to_bf16x2(wv[j]);
                o.y = nib2_to_bf16x2(wv[j] >> 4);
                o.z = nib2_to_bf16x2(wv[j] >> 8);
                o.w = nib2_to_bf16x2(wv[j] >> 12);
                *(uint4 *)(arow + ((c ^ (drow & 7)) << 4)) = o;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(afull_bar(as));
                mbar_arrive(empty_bar(s));
            }
            return true;
        };
        auto promote = [&](uint32_t i, float scale, int N) -> bool {
            const int b = i & 1;
            if (!mbar_wait(pfull_bar(b), (i >> 1) & 1, abort_flag, p.status)) return false;
            tc_fence_after();
            #pragma unroll
            for (int c = 0; c < kTcChunks; ++c) {
                const int col = 32 * (2 * c + half);
                if (col < N) {
                    uint32_t r[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + b * 256 + col, r);
                    tmem_wait_ld();
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) acc[c][j] = fmaf(scale, __uint_as_float(r[j]), acc[c][j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pempty_bar(b));
            return true;
        };

        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            const int a = u / p.m_tiles, mt = u - a * p.m_tiles;
            const int e = p.large[a];
            const int row0 = p.offs[e], cnt = p.cnt[e];
            // the scale row of this thread's TMEM lane
            const float *srow;
            if (MODE == 0)
                srow = ((lrow & 1) ? p.s1 : p.s0) + (int64_t)e * p.estride_s +
                       (int64_t)(mt * 64 + (lrow >> 1)) * p.ng;
            else
                srow = p.s0 + (int64_t)e * p.estride_s + (int64_t)(mt * 128 + lrow) * p.ng;
            for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                const int nrows = min(kTcMaxN, cnt - n0);
                const int N = (nrows + 15) & ~15;
                #pragma unroll
                for (int c = 0; c < kTcChunks; ++c)
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) acc[c][j] = 0.f;
                float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
                float prev_scale = 0.f;
                for (int G = 0; G < p.ng; ++G) {
                    if (!(ok = dequant(it + G))) break;
                    if ((G & 3) == 0) s4 = *(const float4 *)(srow + G);  // ng % 4 == 0
                    const float sc = (G & 3) == 0 ? s4.x : (G & 3) == 1 ? s4.y : (G & 3) == 2 ? s4.z : s4.w;
                    if (G > 0 && !(ok = promote(it + G - 1, prev_scale, N))) break;
                    prev_scale = sc;
                }
                if (ok) ok = promote(it + p.ng - 1, prev_scale, N);
                it += p.ng;
                if (!ok) break;
                // ---------------------------------------------------- epilogue
                if (MODE == 0) {
                    // even lane: gate row, odd lane: the up row of the same output f
                    const int f = mt * 64 + (lrow >> 1);
                    #pragma unroll
                    for (int c = 0; c < kTcChunks; ++c) {
                        const int col = 32 * (2 * c + half);
                        if (col < N) {
                            #pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const float uv = __shfl_xor_sync(0xffffffffu, acc[c][j], 1);
                                if (!(lane & 1) && col + j < nrows) {
                                    const float g = acc[c][j];
                                    const float hv = g / (1.0f + expf(-g)) * uv;
                                    p.h[(int64_t)(row0 + n0 + col + j) * p.O + f] = (uint16_t)bf16_bits_rn(hv);
                                }
                            }
                        }
                    }
                } else {
                    const int o = mt * 128 + lrow;
                    #pragma unroll
                    for (int c = 0; c < kTcChunks; ++c) {
                        const int col = 32 * (2 * c + half);
                        if (col < N) {
                            #pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                if (col + j < nrows) {
                                    const int r = row0 + n0 + col + j;
                                    const int tok = p.row_tok[r];
                                    const float wt = p.wts[p.row_slot[r]];
                                    atomicAdd(p.y + (int64_t)tok * p.O + o, wt * acc[c][j]);
                                }
                            }
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
    }
}

}  // namespace gq4
