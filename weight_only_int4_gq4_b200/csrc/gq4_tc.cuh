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
//     one of three TMEM partial buffers (accumulate off for the first), then commits;
//   * the math warps load the partial (tcgen05.ld), multiply it by the row's scale of
//     that group and add it to running sums kept in registers ("promotion"), then free
//     the buffer -- the MMAs of groups g+1 and g+2 overlap the promotion of group g.
// TMEM lane = weight row, so the scale is one register per thread and group.
//
// Warp roles (512 threads = 4 warpgroups, one CTA per SM, persistent over units):
//   WG0  warp 0  TMA producer of the packed nibble tiles: 128 rows x 128 B (four groups,
//                swizzle 128B) per stage in two 64-row boxes, 5-stage ring
//        warp 1  TMEM allocation and the MMA issuer (one elected lane of the warp)
//        warp 2  TMA producer of the activation tiles (N <= 160 rows x 64 bf16, swizzle
//                128B) as 128/64/32/16-row boxes, 4-stage ring; warp 3 idle
//   (TMA cost is per request more than per byte: few large boxes keep the rings fed)
//   WG1  warps 4-7   dequant: rows [32d, 32d+32) of the bf16 A tile, 3-slot ring
//   WG2-3 warps 8-15 promotion: TMEM lane quarter (warp % 4) x column half, running
//                sums in registers, epilogue
// setmaxnreg moves registers from WG0/WG1 (48 each) to the promotion warps (200 each):
// 256*48 + 256*200 = 63488 <= 65536 = 512 threads x 128 at launch.
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

constexpr int kTcThreads = 512;
constexpr int kTcWStages = 5;                                   // packed-weight ring, 4 groups/stage
constexpr int kTcXStages = 4;                                   // activation ring, 1 group/stage
constexpr int kTcAStages = 3;                                   // dequantised bf16 A tiles
constexpr int kTcMaxN = 160;                                   // rows per pass (TMEM, registers)
constexpr int kTcPBufs = 3;                                     // TMEM partial buffers of kTcMaxN columns
constexpr int kTcChunks = (kTcMaxN + 63) / 64;                  // 32-column chunks per column half
static_assert(kTcChunks == 3, "the promotion reads chunks 2c + half, c < 3");
constexpr int kTcWGroups = 4;                                   // groups per weight stage
constexpr int kTcWBytes = 128 * 32 * kTcWGroups;                // 128 rows x 256 nibbles
constexpr int kTcXBytes = kTcMaxN * 128;                        // N rows x 64 bf16
constexpr int kTcABytes = 128 * 128;                            // 128 rows x 64 bf16
constexpr int kTcOffX = 0;                                      // 1024-aligned tiles first
constexpr int kTcOffA = kTcOffX + kTcXStages * kTcXBytes;
constexpr int kTcOffW = kTcOffA + kTcAStages * kTcABytes;
constexpr int kTcOffBar = kTcOffW + kTcWStages * kTcWBytes;
constexpr int kTcSmemBytes = kTcOffBar + 512 + 1024;            // + 1024 for alignment
static_assert(kTcSmemBytes <= 232448, "shared memory per CTA");
constexpr int kTcTmemCols = 512;                                // power of 2 >= kTcPBufs * kTcMaxN
static_assert(kTcPBufs * kTcMaxN <= kTcTmemCols, "TMEM partial buffers");
constexpr int kTcRegsLow = 48, kTcRegsHigh = 200;               // setmaxnreg split
// registers the split needs from the launch: a launch with fewer per thread would leave
// setmaxnreg.inc waiting forever, so the host refuses it (cudaFuncAttributes::numRegs)
constexpr int kTcRegsNeeded = 256 * kTcRegsLow + 256 * kTcRegsHigh;
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
    // extents for the checked build (GQ4_CHECKED): floats of the scale arrays, experts
    // of the call, tokens (rows of y)
    int64_t s_count;
    int n_exp, n_tok;
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
// As above, but the warp may be suspended in hardware (up to ~0.1 ms) until the phase
// completes, instead of spinning on the issue slots the working warps need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(100000u) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `parity` to complete; false if the CTA aborted or ~2 s passed.
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                              int32_t *status, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if ((i & 7) == 0) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicOr(status, kStatusTimeout);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status) {
    return mbar_wait_for(bar, parity, abort_flag, status, 2000000000ull);
}

// Self-test of the bounded wait every kernel uses: one thread waits on an mbarrier that
// nothing arrives on, with a short limit; the wait gives up, raises GQ4_ERR_TIMEOUT in
// the status word and returns, and the kernel ends normally (no trap, no hang).
__global__ void gq4_wait_selftest_kernel(int32_t *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_for(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
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
// D (+)= A * B (both from shared memory, descriptors), issued by one lane elected from
// the converged calling warp.  ACC (accumulate into D) is a compile-time predicate.
template <bool ACC>
__device__ __forceinline__ void tc_mma_elect(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc) {
    asm volatile(
        "{\n .reg .pred e, p;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "n"(ACC ? 1 : 0) : "memory");
}
// tcgen05.commit (arrive on `bar` once this thread's MMAs are done) by the elected lane.
__device__ __forceinline__ void tc_commit_elect(uint32_t bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n"
        ::"r"(bar) : "memory");
}
// tcgen05.ld writes its destination registers asynchronously, until tcgen05.wait::ld.
// The compiler treats them as written by the load itself, so between a separate load and
// wait it may copy or spill them (saving values that have not arrived yet).  These
// helpers issue the loads and the wait in one asm statement, so nothing the compiler
// generates can sit between them.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld32x2_wait(uint32_t ta, uint32_t tb, uint32_t (&a)[32], uint32_t (&b)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]), "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]), "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
        : "r"(ta), "r"(tb)
        : "memory");
}
// (a0, a1) += s * (p0, p1) as one packed f32x2 FMA.
__device__ __forceinline__ void fma2(float &a0, float &a1, float p0, float p1, uint64_t ss) {
    asm("{\n .reg .b64 ra, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rc, {%0, %1};\n"
        " fma.rn.f32x2 rd, ra, %4, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
        : "+f"(a0), "+f"(a1) : "f"(p0), "f"(p1), "l"(ss));
}
__device__ __forceinline__ uint64_t splat2(float s) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(s));
    return r;
}

// Expert of large-list entry a; in the checked build an entry outside [0, n_exp) raises
// GQ4_ERR_BOUNDS and stands for expert 0, the same in every role of the CTA.
__device__ __forceinline__ int tc_expert(const int32_t *large, int n_exp, int a) {
    const int e = large[a];
    return in_bounds(e, n_exp) ? e : 0;
}

// ---------------------------------------------------------------- the kernel
template <int MODE>  // 0: gate+up with SiLU(g)*u -> h (bf16); 1: down -> y += w * D
__global__ void __launch_bounds__(kTcThreads, 1)
gq4_tc_kernel(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
              const __grid_constant__ CUtensorMap tm_x16, const __grid_constant__ CUtensorMap tm_x32,
              const __grid_constant__ CUtensorMap tm_x64, const __grid_constant__ CUtensorMap tm_x128,
              const TcParams p) {
    if (*p.n_large == 0) return;  // no expert with many rows: nothing to set up (uniform exit)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + kTcOffBar;
    auto wfull_bar = [&](int s) { return bar0 + 8 * s; };
    auto wempty_bar = [&](int s) { return bar0 + 96 + 8 * s; };
    auto xfull_bar = [&](int s) { return bar0 + 192 + 8 * s; };
    auto xempty_bar = [&](int s) { return bar0 + 232 + 8 * s; };
    auto afull_bar = [&](int a) { return bar0 + 272 + 8 * a; };
    auto aempty_bar = [&](int a) { return bar0 + 296 + 8 * a; };
    auto pfull_bar = [&](int b) { return bar0 + 320 + 8 * b; };
    auto pempty_bar = [&](int b) { return bar0 + 344 + 8 * b; };
    uint32_t *tmem_slot = (uint32_t *)(smem + kTcOffBar + 376);
    volatile int *abort_flag = (volatile int *)(smem + kTcOffBar + 384);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcWStages; ++s) {
            mbar_init(wfull_bar(s), 1);
            mbar_init(wempty_bar(s), 4);  // the four dequant warps
        }
        for (int s = 0; s < kTcXStages; ++s) {
            mbar_init(xfull_bar(s), 1);
            mbar_init(xempty_bar(s), 1);  // MMA commit
        }
        for (int a = 0; a < kTcAStages; ++a) {
            mbar_init(afull_bar(a), 4);
            mbar_init(aempty_bar(a), 1);
        }
        for (int b = 0; b < kTcPBufs; ++b) {
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

    if (warp < 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kTcRegsLow) : "memory");
      if (warp == 0 || warp == 2) {
        // ------------------------------------------------------------ TMA producers
        // warp 0: packed weights into the W ring; warp 2: activations into the X ring
        if (lane == 0) {
            const bool wprod = warp == 0;
            const int nst = wprod ? kTcWStages : kTcXStages;
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                const int a = u / p.m_tiles, mt = u - a * p.m_tiles;
                const int e = tc_expert(p.large, p.n_exp, a);
                const int row0 = p.offs[e], cnt = p.cnt[e];
                const int wrow = e * p.estride_rows + (MODE == 0 ? mt * 64 : mt * 128);
                for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                    const int N = (min(kTcMaxN, cnt - n0) + 15) & ~15;
                    if (wprod) {
                        for (int G = 0; G < p.ng; G += kTcWGroups, ++it) {
                            const int s = it % nst;
                            if (!(ok = mbar_wait(wempty_bar(s), ((it / nst) & 1) ^ 1, abort_flag, p.status))) break;
                            const uint32_t dst = sb + kTcOffW + s * kTcWBytes;
                            mbar_expect_tx(wfull_bar(s), kTcWBytes);
                            tma_load_2d(dst, &tm_w0, G * 32, wrow, wfull_bar(s));
                            if (MODE == 0)
                                tma_load_2d(dst + kTcWBytes / 2, &tm_w1, G * 32, wrow, wfull_bar(s));
                            else
                                tma_load_2d(dst + kTcWBytes / 2, &tm_w0, G * 32, wrow + 64, wfull_bar(s));
                        }
                    } else {
                        for (int G = 0; G < p.ng; ++G, ++it) {
                            const int s = it % nst;
                            if (!(ok = mbar_wait(xempty_bar(s), ((it / nst) & 1) ^ 1, abort_flag, p.status))) break;
                            const uint32_t dst = sb + kTcOffX + s * kTcXBytes;
                            mbar_expect_tx(xfull_bar(s), N * 128);
                            int r = 0;  // N (a multiple of 16) as 128/64/32/16-row boxes
                            if (N - r >= 128) { tma_load_2d(dst + r * 128, &tm_x128, G * 64, row0 + n0 + r, xfull_bar(s)); r += 128; }
                            if (N - r >= 64) { tma_load_2d(dst + r * 128, &tm_x64, G * 64, row0 + n0 + r, xfull_bar(s)); r += 64; }
                            if (N - r >= 32) { tma_load_2d(dst + r * 128, &tm_x32, G * 64, row0 + n0 + r, xfull_bar(s)); r += 32; }
                            if (N - r >= 16) { tma_load_2d(dst + r * 128, &tm_x16, G * 64, row0 + n0 + r, xfull_bar(s)); r += 16; }
                        }
                    }
                }
            }
            if (!ok) {  // let copies already issued land before the CTA leaves
                for (uint32_t j = it > (uint32_t)nst ? it - nst : 0; j < it; ++j) {
                    const uint32_t bar = wprod ? wfull_bar(j % nst) : xfull_bar(j % nst);
                    const uint64_t t0 = global_ns();
                    while (!mbar_try_wait(bar, (j / nst) & 1) && global_ns() - t0 < 100000000ull) {
                    }
                }
            }
        }
        __syncwarp();
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop (converged); lane 0 polls the barriers and one
        // elected lane issues each MMA and commit.  The accumulate flag of each MMA is a
        // compile-time predicate: computing it at run time just before the instruction
        // made every issue cost ~210 cycles on B200 (measured), a third of the pipe's rate.
        {
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
                const int a = u / p.m_tiles;
                const int e = tc_expert(p.large, p.n_exp, a);
                const int cnt = p.cnt[e];
                for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                    const int N = (min(kTcMaxN, cnt - n0) + 15) & ~15;
                    const uint32_t idesc = idesc_bf16_m128(N);
                    for (int G = 0; G < p.ng; ++G, ++it) {
                        const int xs = it % kTcXStages, as = it % kTcAStages, b = it % kTcPBufs;
                        if (lane == 0)
                            ok = mbar_wait(xfull_bar(xs), (it / kTcXStages) & 1, abort_flag, p.status) &&
                                 mbar_wait(afull_bar(as), (it / kTcAStages) & 1, abort_flag, p.status) &&
                                 mbar_wait(pempty_bar(b), ((it / kTcPBufs) & 1) ^ 1, abort_flag, p.status);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t a_addr = sb + kTcOffA + as * kTcABytes;
                        const uint32_t x_addr = sb + kTcOffX + xs * kTcXBytes;
                        const uint64_t ad = sw128_desc(a_addr), xd = sw128_desc(x_addr);
                        tc_mma_elect<false>(tmem + b * kTcMaxN, ad, xd, idesc);
                        tc_mma_elect<true>(tmem + b * kTcMaxN, ad + 2, xd + 2, idesc);
                        tc_mma_elect<true>(tmem + b * kTcMaxN, ad + 4, xd + 4, idesc);
                        tc_mma_elect<true>(tmem + b * kTcMaxN, ad + 6, xd + 6, idesc);
                        tc_commit_elect(pfull_bar(b));
                        tc_commit_elect(aempty_bar(as));
                        tc_commit_elect(xempty_bar(xs));
                    }
                }
            }
            // the last commits must have arrived before the CTA's shared memory is released
            if (lane == 0 && ok && it > 0) {
                const uint32_t j = it - 1;
                mbar_wait(xempty_bar(j % kTcXStages), (j / kTcXStages) & 1, abort_flag, p.status);
                mbar_wait(aempty_bar(j % kTcAStages), (j / kTcAStages) & 1, abort_flag, p.status);
            }
        }
        __syncwarp();
      } else if (warp >= 4) {
        // ------------------------------------------------------------ dequant warps
        // A row written by this lane.  Lanes l and rows pair up so that the eight lanes
        // of a shared-memory phase hit eight distinct 16-byte swizzle slots both when
        // reading the packed tile (slot = prow & 7) and when writing the A row (r & 7).
        const int l16 = lane & 15;
        const int r16 = l16 < 8 ? 2 * l16 + (l16 >> 2) : 2 * (l16 - 8) + 1 - ((l16 - 8) >> 2);
        const int r = 32 * (warp - 4) + 16 * (lane >> 4) + r16;
        // packed tile rows: [0,64) first box, [64,128) second; gate+up interleaves them
        const int prow = MODE == 0 ? ((r & 1) ? 64 + (r >> 1) : (r >> 1)) : r;
        uint32_t it = 0, wit = 0;  // group counter, weight-stage counter
        bool ok = true;
        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            const int e = tc_expert(p.large, p.n_exp, u / p.m_tiles);
            const int cnt = p.cnt[e];
            for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                for (int G = 0; G < p.ng; ++G, ++it) {
                    const uint32_t wi = wit + (G >> 2);  // weight stage of this group
                    const int ws = wi % kTcWStages, as = it % kTcAStages;
                    if ((G & 3) == 0 &&
                        !(ok = mbar_wait(wfull_bar(ws), (wi / kTcWStages) & 1, abort_flag, p.status)))
                        break;
                    if (!(ok = mbar_wait(aempty_bar(as), ((it / kTcAStages) & 1) ^ 1, abort_flag, p.status)))
                        break;
                    // packed tile (128B-swizzled): row pr at pr*128, its 16-byte chunk c at
                    // (c ^ (pr & 7)) * 16; group G%4 is chunks 2(G%4), 2(G%4)+1; rows
                    // [64,128) in the second half
                    const uint8_t *wrow_p = smem + kTcOffW + ws * kTcWBytes + (prow >> 6) * (kTcWBytes / 2) +
                                            (prow & 63) * 128;
                    const int c0 = 2 * (G & 3), swz = prow & 7;
                    const uint4 w0 = *(const uint4 *)(wrow_p + ((c0 ^ swz) << 4));
                    const uint4 w1 = *(const uint4 *)(wrow_p + (((c0 + 1) ^ swz) << 4));
                    if ((G & 3) == 3) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(wempty_bar(ws));  // all four groups read
                    }
                    uint8_t *arow = smem + kTcOffA + as * kTcABytes + r * 128;
                    const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    #pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = columns 8c..8c+7
                        uint4 o;
                        o.x = nib2_to_bf16x2(wv[c]);
                        o.y = nib2_to_bf16x2(wv[c] >> 4);
                        o.z = nib2_to_bf16x2(wv[c] >> 8);
                        o.w = nib2_to_bf16x2(wv[c] >> 12);
                        *(uint4 *)(arow + ((c ^ (r & 7)) << 4)) = o;
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(afull_bar(as));
                }
                wit += p.ng / kTcWGroups;
            }
        }
      }
    } else {
        // ------------------------------------------------------------ promotion warps
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kTcRegsHigh) : "memory");
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int half = (warp - 8) >> 2;    // column half: 32-column chunks 2c + half
        const int lrow = 32 * q + lane;      // TMEM lane = A row
        uint32_t it = 0;
        bool ok = true;
        float acc[kTcChunks][32];

        for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            const int a = u / p.m_tiles, mt = u - a * p.m_tiles;
            const int e = tc_expert(p.large, p.n_exp, a);
            const int row0 = p.offs[e], cnt = p.cnt[e];
            // the scale row of this thread's TMEM lane (offset in floats from the array start)
            const int64_t soff = (int64_t)e * p.estride_s +
                                 (int64_t)(MODE == 0 ? mt * 64 + (lrow >> 1) : mt * 128 + lrow) * p.ng;
            const float *srow = ((MODE == 0 && (lrow & 1)) ? p.s1 : p.s0) + soff;
            const int64_t s_count = p.s_count;
            auto scales4 = [srow, soff, s_count](int k) {  // scales of groups k..k+3
                return in_bounds(soff + k + 3, s_count) ? *(const float4 *)(srow + k)
                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            };
            for (int n0 = 0; ok && n0 < cnt; n0 += kTcMaxN) {
                const int nrows = min(kTcMaxN, cnt - n0);
                const int N = (nrows + 15) & ~15;
                #pragma unroll
                for (int c = 0; c < kTcChunks; ++c)
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) acc[c][j] = 0.f;
                // scales four groups at a time, prefetched one float4 ahead (ng % 4 == 0)
                float4 s_cur = scales4(0);
                float4 s_next = p.ng > 4 ? scales4(4) : s_cur;
                for (int G = 0; G < p.ng; ++G, ++it) {
                    const int gq = G & 3;
                    const float sc = gq == 0 ? s_cur.x : gq == 1 ? s_cur.y : gq == 2 ? s_cur.z : s_cur.w;
                    if (gq == 3) {
                        s_cur = s_next;
                        if (G + 5 < p.ng) s_next = scales4(G + 5);
                    }
                    const int b = it % kTcPBufs;
                    if (!(ok = mbar_wait(pfull_bar(b), (it / kTcPBufs) & 1, abort_flag, p.status))) break;
                    tc_fence_after();
                    const uint64_t ss = splat2(sc);
                    const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + b * kTcMaxN;
                    // chunks 2c + half of 32 columns; the first two are loaded together
                    const int col0 = 32 * half, col1 = 32 * (2 + half), col2 = 32 * (4 + half);
                    if (col0 < N) {
                        uint32_t r0[32], r1[32];
                        if (col1 < N) tmem_ld32x2_wait(tbase + col0, tbase + col1, r0, r1);
                        else tmem_ld32_wait(tbase + col0, r0);
                        if (col2 >= N) {  // nothing else to read: the buffer may be reused
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(pempty_bar(b));
                        }
                        #pragma unroll
                        for (int j = 0; j < 32; j += 2)
                            fma2(acc[0][j], acc[0][j + 1], __uint_as_float(r0[j]), __uint_as_float(r0[j + 1]), ss);
                        if (col1 < N) {
                            #pragma unroll
                            for (int j = 0; j < 32; j += 2)
                                fma2(acc[1][j], acc[1][j + 1], __uint_as_float(r1[j]), __uint_as_float(r1[j + 1]), ss);
                        }
                    }
                    if (col2 < N) {
                        uint32_t r2[32];
                        tmem_ld32_wait(tbase + col2, r2);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(pempty_bar(b));
                        #pragma unroll
                        for (int j = 0; j < 32; j += 2)
                            fma2(acc[2][j], acc[2][j + 1], __uint_as_float(r2[j]), __uint_as_float(r2[j + 1]), ss);
                    }
                    if (half == 1 && N <= 32) {  // this warp owns no chunk of this pass
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(pempty_bar(b));
                    }
                }
                if (!ok) break;
                // ---------------------------------------------------- epilogue
                if (MODE == 0) {
                    // even lane: gate row, odd lane: the up row of the same output f.  Per
                    // pair of columns (j, j+1) the even lane finishes column j and the odd
                    // lane column j+1: each sends its partner the value the partner lacks
                    const int f = mt * 64 + (lrow >> 1);
                    const bool odd = lane & 1;
                    #pragma unroll
                    for (int c = 0; c < kTcChunks; ++c) {
                        const int col = 32 * (2 * c + half);
                        if (col < N) {
                            #pragma unroll
                            for (int j = 0; j < 32; j += 2) {
                                const float send = odd ? acc[c][j] : acc[c][j + 1];
                                const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                                const float g = odd ? recv : acc[c][j];
                                const float uv = odd ? acc[c][j + 1] : recv;
                                const int jj = col + j + (odd ? 1 : 0);
                                if (jj < nrows) {
                                    const float hv = g / (1.0f + expf(-g)) * uv;
                                    p.h[(int64_t)(row0 + n0 + jj) * p.O + f] = (uint16_t)bf16_bits_rn(hv);
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
                            // token and weight of the 32 columns: one coalesced load per lane
                            int tok_l = 0;
                            float wt_l = 0.f;
                            if (col + lane < nrows) {
                                const int rr = row0 + n0 + col + lane;
                                tok_l = p.row_tok[rr];
                                wt_l = p.wts[p.row_slot[rr]];
                                if (!in_bounds(tok_l, p.n_tok)) tok_l = -1;
                            }
                            #pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int tok = __shfl_sync(0xffffffffu, tok_l, j);
                                const float wt = __shfl_sync(0xffffffffu, wt_l, j);
                                if (col + j < nrows && tok >= 0) atomicAdd(p.y + (int64_t)tok * p.O + o, wt * acc[c][j]);
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
