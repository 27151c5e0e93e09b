// gq4_stream.cuh -- TMA-fed decode kernel for grouped-int4 products with few activation
// columns (1..32 per matrix or expert): the HBM-bound regime of the routed-expert FFN.
//
// What it computes (colibri PR #298, "cuda+engine: full fmt=4 (grouped int4 gs=64)
// support"): y[c][o] = sum_g s[o][g] * sum_{k in group g} q[o][k] * x[c][k], the group
// scale applied once per 64-wide group to an f32 partial, fp32 accumulation; for gate+up
// h = bf16(silu(g) * u); for the MoE down projection a weighted scatter-add into y.
//
// Design (B200, HBM-bound):
//  * A CTA (one per SM, persistent) owns a band of BR = 16*RW rows of one matrix or
//    expert (for gate+up: BR gate rows and the same BR up rows) for all of K.
//  * One producer warp streams the band through a ring of shared-memory stages, four
//    64-wide groups per stage: the packed nibble tile of each matrix (BR rows x 128 B,
//    one 2-D TMA copy, 128-byte swizzle), the f32 scales of those rows and groups (BR x
//    16 B, one TMA copy) and the stage's 256 activations of every column (one bulk copy
//    per column; the source address does the token gather).  Completion is an mbarrier
//    with a transaction count; no thread spends instructions on weight addresses.
//  * Sixteen consumer warps: row warps x k-warps.  The 16 accumulator rows of a warp's
//    m16n8k16 tensor ops are 16 band rows of one matrix, or, for gate+up, 8 band rows of
//    the gate matrix and the same 8 rows of the up matrix, so that one thread holds
//    gate and up of the same outputs and the SiLU product needs no exchange.  When the
//    band has fewer rows than the warps cover, k-warps split the stage's groups.  Each
//    item (16 accumulator rows x one 64-wide group) is one tensor op chain per 8
//    columns: the nibbles become exact bf16 integers (one lop3 + one bf16x2 fma per two
//    weights), the f32 partial of the group is scaled by its row's s[o][g] and added to
//    the running sum.  The integer pipe is the scarce one (the nibble decode lives there),
//    so every address, slot and phase is computed incrementally or once per warp.
//  * With k-warps, their sums are added at the end of a band in a fixed order through
//    shared memory (deterministic); then the mode's epilogue runs.
//  * Routed experts (MoE modes): the (expert, band) units are taken from a counter in the
//    order of the expert list, which the row map sorts by rows per expert, most first, so
//    the costliest units start first and the CTAs finish together.  The producer passes
//    each pass's band, column offset, column count and first row to the consumers in a
//    small shared-memory queue beside the ring; a band of -1 ends the kernel.  The
//    down projection's token indices and routing weights are read at the start of a
//    pass, one column per lane, so their latency hides behind the pass's stages.
// Every wait is bounded (~2 s): on expiry GQ4_ERR_TIMEOUT is raised in the status word
// and the other waits return at once.  Warps that share a barrier (the k-warps of the
// dense modes) still pass it; the queue-fed consumers of routed experts, which share
// none, leave at their next failed wait.  The producer lets its copies in flight land
// before the CTA leaves.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "gq4_common.cuh"
#include "gq4_skinny.cuh"
#include "gq4_tc.cuh"

namespace gq4 {

constexpr int kStConsumerWarps = 16;
constexpr int kStThreads = (kStConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kStMaxCols = 32;                            // columns per pass
constexpr int kStXStride = 528;  // bytes per staged activation row: 256 bf16 + 16 B pad
constexpr int kStGroups = 4;     // groups per stage (128 packed bytes per row)
constexpr int kStQueue = 9;      // pass queue entries: ring depth (<= 8) + 1

struct StreamArgs {
    int nstages;       // ring depth
    int stage_bytes;   // bytes per stage (multiple of 1024)
    int wrows;         // rows per expert in the weight tensor maps
    int srows;         // rows per expert in the scale tensor maps
    int32_t *status;   // device status word (GQ4_ERR_TIMEOUT), may be NULL
};

// Warp split of a band of 16*RW rows (of each matrix) over the 16 consumer warps.
template <int PAIR, int RW>
struct StreamSplit {
    static constexpr int kRowsPerWarp = 16 / PAIR;            // band rows per row warp
    static constexpr int kRowWarps = RW * PAIR;               // 16*RW / kRowsPerWarp
    static constexpr int kKWarps = kStConsumerWarps / kRowWarps;
    static constexpr int kGroupsPerWarp = kStGroups / kKWarps;  // per stage
};

__host__ __device__ inline int stream_stage_bytes(int pair, int br, int ncols) {
    const int b = pair * br * 128 + pair * br * 16 + ncols * kStXStride;
    return (b + 1023) & ~1023;
}
__host__ __device__ inline int stream_xch_bytes(int pair, int rw, int nt) {
    const int row_warps = rw * pair;
    return row_warps * (kStConsumerWarps / row_warps - 1) * nt * 4 * 32 * 4;
}
// ring + exchange buffer + 2 mbarriers per stage + abort flag + pass queue + 1024 for
// alignment
__host__ __device__ inline int stream_smem_bytes(int nstages, int stage_bytes, int pair, int rw, int nt) {
    return nstages * stage_bytes + stream_xch_bytes(pair, rw, nt) + 16 * nstages + 16 + 16 * kStQueue + 1024;
}

// Four bf16x2 pairs of one device word (nibble slots i and i+4 -> columns 2i, 2i+1).
__device__ __forceinline__ void word_to_bf16x4(uint32_t v, uint32_t *r) {
    r[0] = nib2_to_bf16x2(v);
    r[1] = nib2_to_bf16x2(v >> 4);
    r[2] = nib2_to_bf16x2(v >> 8);
    r[3] = nib2_to_bf16x2(v >> 12);
}

// Bounded wait for the phase of `parity`; false once the CTA has aborted or ~2 s passed
// (then GQ4_ERR_TIMEOUT is raised in *status when a status word was given).
__device__ __forceinline__ bool st_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                        int32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if ((i & 7) == 0) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > 2000000000ull) {
                *abort_flag = 1;
                if (status) atomicOr(status, kStatusTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void named_bar_consumers() {
    asm volatile("bar.sync 1, %0;" ::"r"(kStConsumerWarps * 32) : "memory");
}

// The items of one stage for one consumer warp: groups GL0 .. GL0+IPW-1.
//   a_row: the packed tile row of accumulator rows 0-7 (this lane: row g), A1 bytes on
//   the tile row of rows 8-15; s_row: the four scales of the first, S1 bytes on those of
//   the second; x_lane: the activation bytes this lane feeds for n-tile 0, group 0.
// Columns past nc hold stale values: they only reach accumulator columns that are never
// stored, so they need no zeroing.
template <int NT, int NTA, int IPW, int GL0, int A1, int S1>
__device__ __forceinline__ void stream_items_n(const uint8_t *a_row, const uint8_t *s_row, const uint8_t *x_lane,
                                             const int (&aoff)[kStGroups], float (&acc)[NT][4]) {
    const float4 sva = *(const float4 *)s_row;
    const float4 svb = *(const float4 *)(s_row + S1);
    #pragma unroll
    for (int q = 0; q < IPW; ++q) {
        const int gl = GL0 + q;
        const uint2 wa = *(const uint2 *)(a_row + aoff[gl]);
        const uint2 wb = *(const uint2 *)(a_row + A1 + aoff[gl]);
        const float sa = gl == 0 ? sva.x : gl == 1 ? sva.y : gl == 2 ? sva.z : sva.w;
        const float sb = gl == 0 ? svb.x : gl == 1 ? svb.y : gl == 2 ? svb.z : svb.w;
        const uint64_t ssa = splat2(sa), ssb = splat2(sb);
        uint32_t ra[8], rb[8];
        word_to_bf16x4(wa.x, ra);
        word_to_bf16x4(wa.y, ra + 4);
        word_to_bf16x4(wb.x, rb);
        word_to_bf16x4(wb.y, rb + 4);
        #pragma unroll
        for (int n = 0; n < NTA; ++n) {
            const uint4 *src = (const uint4 *)(x_lane + n * 8 * kStXStride + gl * 128);
            const uint4 b0 = src[0], b1 = src[1];
            const uint32_t bf[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t af[4] = {ra[2 * j], rb[2 * j], ra[2 * j + 1], rb[2 * j + 1]};
                mma_bf16_16816(d, af, bf[2 * j], bf[2 * j + 1], d);
            }
            fma2(acc[n][0], acc[n][1], d[0], d[1], ssa);
            fma2(acc[n][2], acc[n][3], d[2], d[3], ssb);
        }
    }
}

template <int MODE, int NT, int RW>
__global__ void __launch_bounds__(kStThreads, 1)
gq4_stream_kernel(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                  const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_s1,
                  const SkinnyParams p, const StreamArgs a) {
    using TR = ModeTraits<MODE>;
    using SP = StreamSplit<TR::kPair, RW>;
    constexpr int PAIR = TR::kPair;
    constexpr int BR = 16 * RW;                 // band rows of each matrix
    constexpr int RPW = SP::kRowsPerWarp;
    constexpr int NRW = SP::kRowWarps;
    constexpr int KW = SP::kKWarps;
    constexpr int IPW = SP::kGroupsPerWarp;
    static_assert(NRW * KW == kStConsumerWarps && IPW * KW == kStGroups, "warp split");
    constexpr int WBOX = BR * 128, SBOX = BR * 16;
    constexpr int XOFF = PAIR * (WBOX + SBOX);
    // tile and scale offsets of accumulator rows 8-15: the up matrix's rows for gate+up,
    // else band rows R+8
    constexpr int A1 = PAIR == 2 ? WBOX : 8 * 128;
    constexpr int S1 = PAIR == 2 ? SBOX : 8 * 16;
    constexpr int PW = NT * 8 < kStMaxCols ? NT * 8 : kStMaxCols;  // columns per pass (x rows a stage holds)
    // routed experts take their units from a counter; the other modes walk them statically
    constexpr bool kDyn = TR::kMoe;
    static_assert(!kDyn || KW == 1, "a queue-fed consumer runs no exchange barrier");

    extern __shared__ uint8_t st_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)st_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int NS = a.nstages, SB = a.stage_bytes;
    constexpr int XCH = (NRW * (KW - 1) * NT * 4 * 32 * 4);
    float *xch = (float *)(sm + NS * SB);
    const uint32_t bar0 = sbase + NS * SB + XCH;
    auto full_bar = [&](int s) { return bar0 + 8 * s; };
    auto empty_bar = [&](int s) { return bar0 + 8 * (NS + s); };
    volatile int *abort_flag = (volatile int *)(sm + NS * SB + XCH + 16 * NS);
    // pass queue: {band (-1: end), first column, columns, first row}; its entries are
    // ordered by the ring's mbarriers (the asm statements clobber memory)
    int4 *queue = (int4 *)(sm + NS * SB + XCH + 16 * NS + 16);
    int32_t *status = a.status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kStConsumerWarps);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (MODE == kMoeGateUp && p.zero_ptr) {  // y is accumulated into by the down kernel
        float4 *z = (float4 *)p.zero_ptr;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_n / 4;
             i += (int64_t)gridDim.x * blockDim.x)
            z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if constexpr (TR::kMoe) {
        // MoE launches may start before the kernel ahead of them in the stream has
        // finished (programmatic dependent launch): the prologue above touches nothing that
        // kernel writes; everything below reads its results, so wait for it here
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // and let the next MoE kernel start its own prologue
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    __syncthreads();

    const int bands = (p.O + BR - 1) / BR;
    const int n_units = TR::kMoe ? (*p.n_active) * bands : bands;
    const int nst = p.ng / kStGroups;  // stages per pass

    uint32_t issued = 0;  // ring entries the producer warp filled (stages and the end marker)
    if (warp == kStConsumerWarps) {
        // ------------------------------------------------------------ producer warp
        int s = 0, seq = 0;
        uint32_t ph = 0;
        bool ok = true;
        // expert, first row and columns of unit uu (routed experts: two dependent loads)
        auto unit_info = [&](int uu, int &e, int &row0, int &cols) {
            e = 0; row0 = 0; cols = p.n_tok;
            if (TR::kMoe) {
                e = p.active[uu / bands];
                if (!in_bounds(e, p.n_exp)) e = 0;  // the stages must still be delivered
                row0 = p.offs[e];
                cols = p.cnt[e];
            }
        };
        int u = blockIdx.x;
        if (kDyn) {
            int v = 0;
            if (lane == 0) v = atomicAdd(p.unit_ctr, 1);
            u = __shfl_sync(0xffffffffu, v, 0);
        }
        int e = 0, row0 = 0, cols = 0;
        if (u < n_units) unit_info(u, e, row0, cols);
        while (u < n_units) {
            const int band = TR::kMoe ? u % bands : u;
            // the next unit is claimed now and its expert read at this unit's second ring
            // entry, so that neither latency falls between two units
            int u_nx = u + gridDim.x, e_nx = 0, row0_nx = 0, cols_nx = 0;
            bool have_nx = false;
            if (kDyn && lane == 0) u_nx = atomicAdd(p.unit_ctr, 1);
            int entry = 0;
            const int wrow = e * a.wrows + band * BR, srow = e * a.srows + band * BR;
            for (int c0 = 0; c0 < cols; c0 += PW) {
                const int nc = min(PW, cols - c0);
                const uint16_t *xrow = nullptr;  // this lane's activation row
                if (lane < nc) {
                    int64_t xr;
                    if (MODE == kMoeGateUp) xr = p.row_tok[row0 + c0 + lane];
                    else if (MODE == kMoeDown) xr = row0 + c0 + lane;
                    else xr = c0 + lane;
                    if (!in_bounds(xr, p.x_rows)) xr = 0;  // the copy must still deliver its bytes
                    xrow = (const uint16_t *)p.x + xr * p.I;
                }
                const uint32_t tx = (uint32_t)(XOFF + nc * 512);
                for (int k = 0; k < nst; ++k, ++entry) {
                    if (kDyn && entry == 1) {
                        u_nx = __shfl_sync(0xffffffffu, u_nx, 0);
                        if (u_nx < n_units) unit_info(u_nx, e_nx, row0_nx, cols_nx);
                        have_nx = true;
                    }
                    if (ok && lane == 0) ok = st_wait(empty_bar(s), ph ^ 1u, abort_flag, status) && !*abort_flag;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (ok) {
                        const uint32_t stg = sbase + s * SB;
                        if (lane == 0) {
                            // the queue entry is published by the arrive below (release)
                            if (kDyn && k == 0) queue[seq % kStQueue] = make_int4(band, c0, nc, row0);
                            mbar_expect_tx(full_bar(s), tx);
                            tma_load_2d(stg, &tm_w0, k * 128, wrow, full_bar(s));
                            if (PAIR == 2) tma_load_2d(stg + WBOX, &tm_w1, k * 128, wrow, full_bar(s));
                            tma_load_2d(stg + PAIR * WBOX, &tm_s0, k * kStGroups, srow, full_bar(s));
                            if (PAIR == 2)
                                tma_load_2d(stg + PAIR * WBOX + SBOX, &tm_s1, k * kStGroups, srow, full_bar(s));
                        }
                        __syncwarp();
                        if (lane < nc)
                            bulk_g2s(stg + XOFF + lane * kStXStride, xrow + k * 256, 512u, full_bar(s));
                        ++issued;
                    }
                    if (++s == NS) { s = 0; ph ^= 1u; }
                }
                ++seq;
            }
            if (kDyn && !ok) break;  // the consumers leave at their next failed wait
            if (kDyn) u_nx = __shfl_sync(0xffffffffu, u_nx, 0);
            if (!have_nx && u_nx < n_units) unit_info(u_nx, e_nx, row0_nx, cols_nx);
            u = u_nx; e = e_nx; row0 = row0_nx; cols = cols_nx;
        }
        if (kDyn && ok) {
            // end marker: a ring entry with no copies whose queue entry has band -1
            if (lane == 0) ok = st_wait(empty_bar(s), ph ^ 1u, abort_flag, status) && !*abort_flag;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) {
                if (lane == 0) {
                    queue[seq % kStQueue] = make_int4(-1, 0, 0, 0);
                    mbar_arrive(full_bar(s));
                }
                ++issued;
            }
        }
    } else {
        // ------------------------------------------------------------ consumer warps
        const int g = lane >> 2, t = lane & 3;
        const int rw = warp % NRW, kw = warp / NRW;
        const int gl0 = kw * IPW;   // this warp's first group in a stage
        const int R = RPW * rw + g; // band row of accumulator slots 0,1 (and of 2,3 for gate+up)
        // 128B swizzle: 16-byte chunk c of tile row r sits at chunk c ^ (r & 7), and
        // (R & 7) == ((R + 8) & 7) == g; lane t reads bytes 8t..8t+7 of each group
        int aoff[kStGroups];
        #pragma unroll
        for (int gl = 0; gl < kStGroups; ++gl) aoff[gl] = (((2 * gl + (t >> 1)) ^ g) << 4) | ((t & 1) << 3);
        const int a_base = R * 128;
        const int s_base = PAIR * WBOX + R * 16;
        const int x_base = XOFF + g * kStXStride + t * 32;
        int s = 0, seq = 0;
        uint32_t ph = 0;
        int su = blockIdx.x, sc0 = 0;  // static walk: unit and first column of the next pass
        for (;;) {
            int band, c0, nc, row0;
            bool waited = false;  // the pass's first stage has been waited for
            if constexpr (kDyn) {
                if (!st_wait(full_bar(s), ph, abort_flag, status)) break;
                const int4 q = queue[seq % kStQueue];
                if (q.x < 0) break;
                band = q.x; c0 = q.y; nc = q.z; row0 = q.w;
                waited = true;
            } else {
                if (su >= n_units || p.n_tok <= 0) break;
                band = su; c0 = sc0; row0 = 0;
                nc = min(PW, p.n_tok - c0);
                if (sc0 + PW < p.n_tok) sc0 += PW;
                else { sc0 = 0; su += gridDim.x; }
            }
            // down projection: token and routing weight of column `lane` of this pass
            int tok_l = -1;
            float wt_l = 0.f;
            if (MODE == kMoeDown && lane < nc) {
                const int r = row0 + c0 + lane;
                tok_l = p.row_tok[r];
                wt_l = p.wts[p.row_slot[r]];
            }
            float acc[NT][4];
            #pragma unroll
            for (int n = 0; n < NT; ++n)
                #pragma unroll
                for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;

            bool aborted = false;
            // the pass's stages with the active n-tile count fixed for the whole pass
            auto run_pass = [&](auto nta_c) {
                constexpr int NTA = decltype(nta_c)::value;
                for (int k = 0; k < nst; ++k) {
                    const bool have = (k == 0 && waited) || st_wait(full_bar(s), ph, abort_flag, status);
                    if (have) {
                        const uint8_t *stg = sm + s * SB;
                        const uint8_t *ar = stg + a_base, *sr = stg + s_base, *xl = stg + x_base;
                        if constexpr (IPW == 4) {
                            stream_items_n<NT, NTA, 4, 0, A1, S1>(ar, sr, xl, aoff, acc);
                        } else if constexpr (IPW == 2) {
                            if (gl0 == 0) stream_items_n<NT, NTA, 2, 0, A1, S1>(ar, sr, xl, aoff, acc);
                            else stream_items_n<NT, NTA, 2, 2, A1, S1>(ar, sr, xl, aoff, acc);
                        } else {
                            if (gl0 == 0) stream_items_n<NT, NTA, 1, 0, A1, S1>(ar, sr, xl, aoff, acc);
                            else if (gl0 == 1) stream_items_n<NT, NTA, 1, 1, A1, S1>(ar, sr, xl, aoff, acc);
                            else if (gl0 == 2) stream_items_n<NT, NTA, 1, 2, A1, S1>(ar, sr, xl, aoff, acc);
                            else stream_items_n<NT, NTA, 1, 3, A1, S1>(ar, sr, xl, aoff, acc);
                        }
                    } else if (kDyn) {
                        aborted = true;  // no barrier below needs this warp: leave
                        break;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty_bar(s));
                    if (++s == NS) { s = 0; ph ^= 1u; }
                }
            };
            if (NT >= 3 && nc > 16) run_pass(std::integral_constant<int, (NT >= 3 ? 3 : 1)>{});
            else if (NT >= 2 && nc > 8) run_pass(std::integral_constant<int, (NT >= 2 ? 2 : 1)>{});
            else run_pass(std::integral_constant<int, 1>{});
            if (aborted) break;
            ++seq;

            // ---- add the k-warps' sums (fixed order) and run the epilogue
            float v[NT][4];
            if constexpr (KW > 1) {
                if (kw != 0) {
                    float *dst = xch + (rw * (KW - 1) + kw - 1) * NT * 4 * 32 + lane;
                    #pragma unroll
                    for (int n = 0; n < NT; ++n)
                        #pragma unroll
                        for (int i = 0; i < 4; ++i) dst[(n * 4 + i) * 32] = acc[n][i];
                }
                named_bar_consumers();
                if (kw == 0) {
                    #pragma unroll
                    for (int n = 0; n < NT; ++n)
                        #pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            float sum = acc[n][i];
                            #pragma unroll
                            for (int w = 1; w < KW; ++w)
                                sum += xch[((rw * (KW - 1) + w - 1) * NT * 4 + n * 4 + i) * 32 + lane];
                            v[n][i] = sum;
                        }
                }
                named_bar_consumers();  // the exchange buffer may be rewritten
            } else {
                #pragma unroll
                for (int n = 0; n < NT; ++n)
                    #pragma unroll
                    for (int i = 0; i < 4; ++i) v[n][i] = acc[n][i];
            }
            if (kw == 0 && !*abort_flag) {
                #pragma unroll
                for (int n = 0; n < NT; ++n) {
                    if constexpr (PAIR == 2) {
                        // slots 0,1: gate of row R, columns 2t, 2t+1; slots 2,3: up of the same
                        #pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int cl = n * 8 + 2 * t + i;
                            const int o = band * BR + R;
                            if (cl >= nc || o >= p.O) continue;
                            const int c = c0 + cl;
                            const uint16_t hv = (uint16_t)bf16_bits_rn(silu_mul(v[n][i], v[n][i + 2]));
                            if (MODE == kGateUp) ((uint16_t *)p.h)[(int64_t)c * p.O + o] = hv;
                            else ((uint16_t *)p.h)[(int64_t)(row0 + c) * p.O + o] = hv;
                        }
                    } else {
                        #pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int cl = n * 8 + 2 * t + (i & 1);
                            const int o = band * BR + R + ((i >> 1) << 3);
                            if (MODE == kMoeDown) {
                                // every lane takes part in the shuffles
                                const int tok = __shfl_sync(0xffffffffu, tok_l, cl & 31);
                                const float wt = __shfl_sync(0xffffffffu, wt_l, cl & 31);
                                if (cl >= nc || o >= p.O) continue;
                                if (in_bounds(tok, p.n_tok)) atomicAdd(p.y + (int64_t)tok * p.O + o, wt * v[n][i]);
                            } else {
                                if (cl >= nc || o >= p.O) continue;
                                p.y[(int64_t)(c0 + cl) * p.O + o] = v[n][i];
                            }
                        }
                    }
                }
            }
        }
    }
    // copies still in flight (only after an abort) must land before the CTA leaves
    if (warp == kStConsumerWarps && lane == 0) {
        const uint32_t first = issued > (uint32_t)NS ? issued - NS : 0;
        for (uint32_t j = first; j < issued; ++j) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(full_bar(j % NS), (j / NS) & 1) && global_ns() - t0 < 100000000ull) {
            }
        }
    }
    __syncthreads();
}

}  // namespace gq4
