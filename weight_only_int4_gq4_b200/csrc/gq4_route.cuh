// gq4_route.cuh -- router top-K and the on-device token -> expert row map.
//
// Router (colibri PR #298, "implementation complete but blocked": router top-K with a
// taken-flag array, K passes): per token, K passes each take the largest logit among the
// experts not yet taken; among equal logits the lower index wins.  Weights: softmax over
// all E renormalised over the K chosen, i.e. exp(l_j - l_max) / sum_sel exp(l - l_max).
// One warp per token; lane i holds experts i, i+32, ...
//
// Row map (pxq_llama.cpp release notes 2026-09-02, "Device-side MoE row map": histogram,
// scan and fill on the device, bit-identical to the host table).  Rows of an expert are
// ordered by ascending flat slot f = t*K + j.  Slots are cut into chunks of 1024:
//   count: per chunk, a histogram of experts           -> chunk_cnt[c][e]
//   scan : per expert, offsets of each chunk's rows     -> base[c][e], offs, active list
//   fill : per chunk, a slot's rank among earlier slots of the same expert in the chunk
//          (warp match + per-warp counts) added to base[c][e]
// Every step is integer counting in a fixed order, so the table is deterministic.
#pragma once
#include "gq4_common.cuh"

namespace gq4 {

constexpr int kChunk = 1024;        // slots per row-map chunk (one per thread)
constexpr int kMaxExperts = 1024;
constexpr int kStatusNonFinite = 9; // GQ4_ERR_NONFINITE_LOGIT

// Order-preserving key of a float (larger float -> larger unsigned key; NaN excluded).
// Key 0 (below every float's key) marks an expert that is absent or already taken.
__device__ __forceinline__ uint32_t route_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float route_key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Route one token with one warp.  EPL = experts per lane (>= ceil(E/32)); lane i holds
// experts i, i+32, ...  Each of the K passes takes the largest remaining logit, the lower
// expert index among equal logits: a warp-wide max of the lanes' best keys (redux.sync),
// then a warp-wide min of the expert index among the lanes holding that key; only the
// winning lane rescans its experts for its next best.
template <int EPL>
__device__ __forceinline__ void route_token_warp(const float *lg, int E, int K, int32_t *idx,
                                                 float *wts, int32_t *status) {
    const int lane = threadIdx.x & 31;
    uint32_t key[EPL];
    bool bad = false;
    #pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        const float v = e < E ? lg[e] : 0.f;
        if (e < E && (isnan(v) || (isinf(v) && v > 0.f))) bad = true;
        // -0 and +0 compare equal: give them one key so the lower index wins their tie
        key[i] = (e < E && !isnan(v)) ? route_key(v == 0.f ? 0.f : v) : 0u;
    }
    bad = __any_sync(0xffffffffu, bad);
    // this lane's best remaining expert: the largest key, the lowest slot among equals
    uint32_t bk = 0u;
    int bi = 0;
    #pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (key[i] > bk) { bk = key[i]; bi = i; }
    float my_v[EPL];  // pick j is kept by lane j % 32 in slot j / 32 (K <= E <= 32*EPL)
    int my_e[EPL];
    #pragma unroll
    for (int i = 0; i < EPL; ++i) { my_v[i] = -INFINITY; my_e[i] = 0; }
    float vmax = -INFINITY;
    for (int j = 0; j < K; ++j) {
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const int we = __reduce_min_sync(0xffffffffu, (bk == wk && wk != 0u) ? (lane + 32 * bi) : 0x7fffffff);
        const float wv = route_key_value(wk);
        if (we != 0x7fffffff && (we & 31) == lane) {  // the winner drops its pick
            #pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i == bi) key[i] = 0u;
            bk = 0u;
            bi = 0;
            #pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (key[i] > bk) { bk = key[i]; bi = i; }
        }
        if (j == 0) vmax = wv;
        if ((j & 31) == lane) {
            #pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i == (j >> 5)) { my_v[i] = wv; my_e[i] = we; }
        }
    }
    if (!bad && isinf(vmax)) bad = true;  // no finite maximum
    float p[EPL];
    float z = 0.f;
    #pragma unroll
    for (int i = 0; i < EPL; ++i) {
        p[i] = (lane + 32 * i < K) ? expf(my_v[i] - vmax) : 0.f;
        z += p[i];
    }
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    #pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int j = lane + 32 * i;
        if (j < K) {
            if (bad) {
                idx[j] = j;
                wts[j] = __uint_as_float(0x7fc00000u);
            } else {
                idx[j] = my_e[i];
                wts[j] = p[i] / z;
            }
        }
    }
    if (bad && lane == 0) atomicOr(status, kStatusNonFinite);
}

template <int EPL>
__global__ void __launch_bounds__(256) gq4_route_kernel(const float *logits, int T, int E, int K,
                                                        int32_t *idx, float *wts, int32_t *status) {
    const int tok = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (tok >= T) return;
    route_token_warp<EPL>(logits + (int64_t)tok * E, E, K, idx + (int64_t)tok * K,
                          wts + (int64_t)tok * K, status);
}

// ---- row map, chunked -------------------------------------------------------------
// count: block c histograms slots [c*1024, (c+1)*1024) into chunk_cnt[c][E].
// An index outside [0, E) is not counted and raises GQ4_ERR_SHAPE (3) in *status.
__global__ void __launch_bounds__(1024) gq4_rowmap_count_kernel(const int32_t *idx, int n, int E,
                                                                int32_t *chunk_cnt, int32_t *status) {
    __shared__ int32_t h[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int f = blockIdx.x * kChunk + threadIdx.x;
    if (f < n) {
        const int e = idx[f];
        if (e >= 0 && e < E) atomicAdd(&h[e], 1);
        else atomicOr(status, 3);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_cnt[(int64_t)blockIdx.x * E + e] = h[e];
}

// Block-wide exclusive scan of one value per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_excl_scan_1024(int v, int *sh /*[32]*/, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = sh[lane];
        #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        sh[lane] = s;  // inclusive per-warp totals
    }
    __syncthreads();
    const int before = (warp ? sh[warp - 1] : 0) + x - v;
    *total = sh[31];
    __syncthreads();
    return before;
}

// Expert lists for the two GEMM regimes: small (0 < cnt < thr: the decode kernels) and
// large (cnt >= thr: the tensor-core kernels).  The large list is ascending.  The small
// list is ordered by row count, most rows first (counts from 63 up share one place; the
// order among equal counts is not fixed): the decode kernels take their work in list
// order, so the units that cost most start first.  Null pointers: skipped.
struct ExpertLists {
    int32_t *n_small, *small, *n_large, *large;
    int thr;
};

constexpr int kCountBins = 64;

// Called by all 1024 threads of the block; thread e = expert e with c rows.
__device__ __forceinline__ void classify_experts(int e, int E, int c, int *sh, const ExpertLists &L) {
    __shared__ int bin_cnt[kCountBins], bin_base[kCountBins];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool is_small = e < E && c > 0 && c < L.thr, is_large = e < E && c >= L.thr;
    // bin 0 holds the most rows
    const int b = is_small ? kCountBins - 1 - min(c, kCountBins - 1) : -1;
    if (threadIdx.x < kCountBins) bin_cnt[threadIdx.x] = 0;
    __syncthreads();
    if (b >= 0) atomicAdd(&bin_cnt[b], 1);
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of the bin counts, in bin order
        const int t0 = bin_cnt[lane], t1 = bin_cnt[lane + 32];
        int x0 = t0, x1 = t1;
        #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
            if (lane >= o) { x0 += y0; x1 += y1; }
        }
        const int total0 = __shfl_sync(0xffffffffu, x0, 31);
        bin_base[lane] = x0 - t0;
        bin_base[lane + 32] = total0 + x1 - t1;
        if (lane == 31 && L.n_small) *L.n_small = total0 + x1;
    }
    __syncthreads();
    if (b >= 0 && L.small) L.small[atomicAdd(&bin_base[b], 1)] = e;
    if (L.thr >= (1 << 30)) {  // no expert can reach the threshold
        if (e == 0 && L.n_large) *L.n_large = 0;
        return;
    }
    int tot;
    const int lb = block_excl_scan_1024(is_large ? 1 : 0, sh, &tot);
    if (is_large && L.large) L.large[lb] = e;
    if (e == 0 && L.n_large) *L.n_large = tot;
}

// scan: one block of 1024 threads, thread e = expert e (E <= 1024).
__global__ void __launch_bounds__(1024) gq4_rowmap_scan_kernel(int32_t *chunk_cnt /*in: counts,
                                                               out: bases*/, int nchunks, int E,
                                                               int32_t *cnt, int32_t *offs,
                                                               int32_t *n_active, int32_t *active,
                                                               ExpertLists lists) {
    __shared__ int sh[32];
    const int e = threadIdx.x;
    int total_e = 0;
    if (e < E)
        for (int c = 0; c < nchunks; ++c) {
            const int v = chunk_cnt[(int64_t)c * E + e];
            chunk_cnt[(int64_t)c * E + e] = total_e;  // rows of e in earlier chunks
            total_e += v;
        }
    int tot;
    const int off = block_excl_scan_1024(e < E ? total_e : 0, sh, &tot);
    const int act_before = block_excl_scan_1024((e < E && total_e > 0) ? 1 : 0, sh, &tot);
    if (e < E) {
        cnt[e] = total_e;
        offs[e] = off;
        if (total_e > 0) active[act_before] = e;
        for (int c = 0; c < nchunks; ++c) chunk_cnt[(int64_t)c * E + e] += off;
    }
    if (e == 0) *n_active = tot;
    if (e == E - 1) offs[E] = off + total_e;
    classify_experts(e, E, total_e, sh, lists);
}

// Rank of each slot of one chunk among the earlier slots of the same expert in the
// chunk: per-warp counts (warp match) in shared memory wcnt[32][E], then a prefix over
// the earlier warps.  `base` gives the first row of expert e for this chunk.  Called by
// all 1024 threads; thread i owns slot f = chunk_start + i (e < 0: no slot).
__device__ __forceinline__ void rowmap_fill_chunk(int f, int e, int K, int E, int32_t *wcnt,
                                                  const int32_t *base, int32_t *row_tok,
                                                  int32_t *row_slot, int32_t *slot_row) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
        int r = base[e] + __popc(peers & ((1u << lane) - 1u));
        for (int w = 0; w < warp; ++w) r += wcnt[w * E + e];
        row_slot[r] = f;
        row_tok[r] = f / K;
        slot_row[f] = r;
    }
}

// fill: block c writes the rows of slots [c*1024, (c+1)*1024).  Dynamic shared memory:
// 32*E ints.
__global__ void __launch_bounds__(1024) gq4_rowmap_fill_kernel(const int32_t *idx, int n, int K, int E,
                                                               const int32_t *base /*[nchunks][E]*/,
                                                               int32_t *row_tok, int32_t *row_slot,
                                                               int32_t *slot_row) {
    extern __shared__ int32_t wcnt_dyn[];
    const int f = blockIdx.x * kChunk + threadIdx.x;
    int e = f < n ? idx[f] : -1;
    if (e >= E) e = -1;
    rowmap_fill_chunk(f, e, K, E, wcnt_dyn, base + (int64_t)blockIdx.x * E, row_tok, row_slot,
                      slot_row);
}

// Decode path: router and the whole row map in one block of 1024 threads (T*K <= 1024).
// The block first clears the four-word status block (the layer's first kernel: nothing
// else has written it yet).  Dynamic shared memory: (32 + 1) * E ints.
template <int EPL>
__global__ void __launch_bounds__(1024) gq4_route_rowmap_small_kernel(
    const float *logits, int T, int E, int K, int32_t *idx, float *wts, int32_t *status,
    int32_t *cnt, int32_t *offs, int32_t *n_active, int32_t *active, int32_t *row_tok,
    int32_t *row_slot, int32_t *slot_row, ExpertLists lists) {
    extern __shared__ int32_t sm_dyn[];
    int32_t *hist = sm_dyn;        // [E] counts, then offsets
    int32_t *wcnt = sm_dyn + E;    // [32][E]
    __shared__ int sh[32];
    const int warp = threadIdx.x >> 5;
    // the expert kernels after this one may start their prologues now; they wait for
    // this kernel's results (griddepcontrol.wait) before reading them
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x < 4) status[threadIdx.x] = 0;
    __syncthreads();
    for (int t = warp; t < T; t += 32)
        route_token_warp<EPL>(logits + (int64_t)t * E, E, K, idx + (int64_t)t * K,
                              wts + (int64_t)t * K, status);
    for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
    __syncthreads();  // idx written by this block is visible to the block from here
    const int n = T * K;
    const int f = threadIdx.x;
    const int e = f < n ? idx[f] : -1;
    if (e >= 0) atomicAdd(&hist[e], 1);
    __syncthreads();
    const int ex = threadIdx.x;
    const int c = ex < E ? hist[ex] : 0;
    int tot;
    const int off = block_excl_scan_1024(c, sh, &tot);
    const int act_before = block_excl_scan_1024((ex < E && c > 0) ? 1 : 0, sh, &tot);
    if (ex < E) {
        cnt[ex] = c;
        offs[ex] = off;
        if (c > 0) active[act_before] = ex;
        hist[ex] = off;  // now the first row of each expert
    }
    if (ex == 0) *n_active = tot;
    if (ex == E - 1) offs[E] = off + c;
    classify_experts(ex, E, c, sh, lists);
    __syncthreads();
    rowmap_fill_chunk(f, e, K, E, wcnt, hist, row_tok, row_slot, slot_row);
}

}  // namespace gq4

namespace gq4 {
// Gather the activation rows of the experts with many rows into row-map order:
// xg[r] = x[row_tok[r]] for every row r of an expert in the `large` list (the tensor-core
// kernels read only those rows).  One warp per (large expert, row) pair.
__global__ void gq4_gather_rows_kernel(const uint4 *x, const int32_t *row_tok, const int32_t *offs,
                                       const int32_t *cnt, const int32_t *n_large, const int32_t *large,
                                       int chunks_per_row, uint4 *xg, int64_t x_rows, int n_exp) {
    const int nl = *n_large;
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    for (int a = 0; a < nl; ++a) {
        const int e = large[a];
        if (!in_bounds(e, n_exp)) continue;  // the same for every warp
        const int r0 = offs[e], n = cnt[e];
        for (; w < n; w += warps) {
            const int r = r0 + w;
            const int64_t xr = row_tok[r];
            const uint4 *src = x + (in_bounds(xr, x_rows) ? xr : 0) * chunks_per_row;
            uint4 *dst = xg + (int64_t)r * chunks_per_row;
            for (int c = lane; c < chunks_per_row; c += 32) dst[c] = src[c];
        }
        w -= n;  // continue the warp's stride in the next expert's rows
    }
}
}  // namespace gq4
