// gq4_host.cu -- the C ABI of libgq4 (declared in include/gq4.h): argument checks,
// workspace layout and kernel launches.  Every compute step runs in the kernels of
// gq4_skinny.cuh / gq4_route.cuh / gq4_tc.cuh; this file only validates, lays out the
// workspace, encodes TMA descriptors and launches.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "gq4.h"
#include "gq4_aux.cuh"
#include "gq4_common.cuh"
#include "gq4_mla.cuh"
#include "gq4_route.cuh"
#include "gq4_skinny.cuh"
#include "gq4_stream.cuh"
#include "gq4_tc.cuh"

using namespace gq4;

namespace {

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;
};
inline Range rng(const void *p, size_t bytes) { return {(uintptr_t)p, (uintptr_t)p + bytes}; }
inline bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

inline cudaStream_t S(gq4_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Checks of one tensor descriptor for the GPU kernels.
gq4_status check_tensor(const gq4_tensor *t, int n_experts_min) {
    if (!t || !t->w || !t->s) return GQ4_ERR_NULL;
    if (t->out < 1 || t->in < 1 || t->n_experts < n_experts_min) return GQ4_ERR_SHAPE;
    if (t->gs <= 0 || t->ng != (t->in + t->gs - 1) / t->gs) return GQ4_ERR_SHAPE;
    if (t->gs != kGroup || t->in % kGroup != 0) return GQ4_ERR_UNSUPPORTED;
    if (t->out > (int64_t)1 << 30 || t->in > (int64_t)1 << 20) return GQ4_ERR_SHAPE;
    if (!aligned16(t->w) || !aligned16(t->s)) return GQ4_ERR_ALIGN;
    if (t->n_experts > 1) {
        if (t->expert_stride_w < t->out * (t->in / 2) || t->expert_stride_s < t->out * t->ng)
            return GQ4_ERR_SHAPE;
        if (t->expert_stride_w % 16 || t->expert_stride_s % 4) return GQ4_ERR_ALIGN;
    }
    return GQ4_OK;
}

// Checks of one tensor descriptor for the generic kernels: any group size that is a
// multiple of 8 (a device word of 8 weights lies in one group), in % 8 == 0.
gq4_status check_tensor_generic(const gq4_tensor *t, int n_experts_min) {
    if (!t || !t->w || !t->s) return GQ4_ERR_NULL;
    if (t->out < 1 || t->in < 1 || t->n_experts < n_experts_min) return GQ4_ERR_SHAPE;
    if (t->gs <= 0 || t->ng != (t->in + t->gs - 1) / t->gs) return GQ4_ERR_SHAPE;
    if (t->gs % 8 != 0 || t->in % 8 != 0) return GQ4_ERR_UNSUPPORTED;
    if (t->out > (int64_t)1 << 30 || t->in > (int64_t)1 << 20) return GQ4_ERR_SHAPE;
    if (!aligned16(t->w) || !aligned16(t->s)) return GQ4_ERR_ALIGN;
    return GQ4_OK;
}

inline size_t tensor_w_bytes(const gq4_tensor *t) {
    return (size_t)(t->n_experts - 1) * t->expert_stride_w + (size_t)t->out * (t->in / 2);
}
inline size_t tensor_s_bytes(const gq4_tensor *t) {
    return ((size_t)(t->n_experts - 1) * t->expert_stride_s + (size_t)t->out * t->ng) * 4;
}

// Array extents the checked build tests indexes against: the weight and scale arrays of
// t0 (and t1, the smaller of the two), the rows of the activation array, the experts.
void set_extents(SkinnyParams &p, const gq4_tensor *t0, const gq4_tensor *t1, int64_t x_rows, int n_exp) {
    size_t wb = tensor_w_bytes(t0), sb = tensor_s_bytes(t0);
    if (t1) {
        wb = std::min(wb, tensor_w_bytes(t1));
        sb = std::min(sb, tensor_s_bytes(t1));
    }
    p.w_bytes = (int64_t)wb;
    p.s_count = (int64_t)(sb / 4);
    p.x_rows = x_rows;
    p.n_exp = n_exp;
}

int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Opt a kernel into more than 48 KB of dynamic shared memory (once per process; the
// attribute applies to the function in every context of the process).
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)std::min<size_t>(bytes, 227 * 1024));
}

constexpr size_t kMaxSmem = 227 * 1024;

// ---- skinny launches -----------------------------------------------------------------
size_t skinny_smem(int mode_pair, int NT, int xcols, int I) {
    return (size_t)xcols * skinny_xstride(I) + (size_t)8 * mode_pair * 16 * NT * 8 * 4;
}

template <int MODE, int NT>
gq4_status launch_skinny_nt(const SkinnyParams &p, int units_upper, cudaStream_t st) {
    constexpr int PAIR = ModeTraits<MODE>::kPair;
    constexpr int UG = PAIR == 2 ? 2 : 4;
    auto kern = gq4_skinny_kernel<MODE, NT, UG>;
    const size_t smem = skinny_smem(PAIR, NT, p.xcols, p.I);
    if (smem > kMaxSmem) return GQ4_ERR_UNSUPPORTED;
    if (allow_smem(kern, smem) != cudaSuccess) return GQ4_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess)
        return GQ4_ERR_CUDA;
    per_sm = std::max(per_sm, 1);
    const int grid = std::max(1, std::min(units_upper, per_sm * sm_count()));
    kern<<<grid, 256, smem, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

// Choose the n-tile count and the staged-column budget for `cols` columns per unit.
template <int MODE>
gq4_status launch_skinny(SkinnyParams p, int max_cols, bool f32x, int units_upper, cudaStream_t st) {
    constexpr int PAIR = ModeTraits<MODE>::kPair;
    int NT = max_cols <= 8 ? 1 : (max_cols <= 16 ? 2 : 4);
    // staged columns: as many as fit next to the reduction buffer (at most ~96 KB so two
    // CTAs share an SM), a multiple of 3 for f32 activations, at least one pass
    const size_t red = (size_t)8 * PAIR * 16 * NT * 8 * 4;
    const size_t xs = skinny_xstride(p.I);
    size_t budget = 96 * 1024 > red ? 96 * 1024 - red : 0;
    int fit = (int)std::min<size_t>(budget / xs, 1 << 20);
    int xcols = std::min(max_cols, std::max(fit, f32x ? 3 : 1));
    if (f32x) xcols = std::max(3, xcols / 3 * 3);
    if ((size_t)xcols * xs + red > kMaxSmem) return GQ4_ERR_UNSUPPORTED;
    p.xcols = xcols;
    switch (NT) {
        case 1: return launch_skinny_nt<MODE, 1>(p, units_upper, st);
        case 2: return launch_skinny_nt<MODE, 2>(p, units_upper, st);
        default: return launch_skinny_nt<MODE, 4>(p, units_upper, st);
    }
}

// Row-band kernel for 3..32 (or more, in passes) bf16 activation columns.
template <int MODE, int NT>
gq4_status launch_band_nt(const SkinnyParams &p, int units_upper, int32_t *status, cudaStream_t st) {
    auto kern = gq4_band_kernel<MODE, NT>;
    const size_t smem = band_smem(ModeTraits<MODE>::kPair);
    if (allow_smem(kern, smem) != cudaSuccess) return GQ4_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess)
        return GQ4_ERR_CUDA;
    per_sm = std::max(per_sm, 1);
    const int grid = std::max(1, std::min(units_upper, per_sm * sm_count()));
    kern<<<grid, 256, smem, st>>>(p, status);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

template <int MODE>
gq4_status launch_band(const SkinnyParams &p, int max_cols, int units_upper, int32_t *status,
                       cudaStream_t st) {
    const int c = std::min(max_cols, kBandMaxCols);
    if (c <= 8) return launch_band_nt<MODE, 1>(p, units_upper, status, st);
    if (c <= 16) return launch_band_nt<MODE, 2>(p, units_upper, status, st);
    if (c <= 24) return launch_band_nt<MODE, 3>(p, units_upper, status, st);
    return launch_band_nt<MODE, 4>(p, units_upper, status, st);
}

// Decode-path dispatch: the row-band kernel from 3 bf16 columns on, the split-K kernel
// for one or two columns (where bands would leave most SMs idle) and for f32 columns.
constexpr int kBandMinCols = 3;

// ---- MoE workspace layout --------------------------------------------------------------
struct MoeLayout {
    size_t status, idx, wts, cnt, offs, row_tok, row_slot, slot_row, n_active, active, chunk,
        h, lists, xg, total;
};

// Experts with at least this many rows go to the tensor-core (tcgen05) kernels, the
// others to the decode kernels.
constexpr int kLargeMin = GQ4_MOE_LARGE_MIN_ROWS;

inline size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

MoeLayout moe_layout(int64_t T, int32_t E, int32_t K, int64_t H, int64_t F) {
    MoeLayout L{};
    const size_t n = (size_t)T * K;
    const size_t nchunks = (n + kChunk - 1) / kChunk;
    size_t o = 0;
    L.status = o; o = al256(o + 16);
    L.idx = o; o = al256(o + n * 4);
    L.wts = o; o = al256(o + n * 4);
    L.cnt = o; o = al256(o + (size_t)E * 4);
    L.offs = o; o = al256(o + (size_t)(E + 1) * 4);
    L.row_tok = o; o = al256(o + n * 4);
    L.row_slot = o; o = al256(o + n * 4);
    L.slot_row = o; o = al256(o + n * 4);
    L.n_active = o; o = al256(o + 16);
    L.active = o; o = al256(o + (size_t)E * 4);
    L.chunk = o; o = al256(o + nchunks * (size_t)E * 4);
    L.h = o; o = al256(o + n * (size_t)F * 2);
    L.lists = o; o = al256(o + (size_t)(2 * E + 8) * 4);  // n_small, n_large, small[E], large[E]
    L.xg = o; o = al256(o + (T >= kLargeMin ? n * (size_t)H * 2 : 0));
    L.total = o;
    return L;
}

template <typename T>
inline T *at(void *ws, size_t off) { return reinterpret_cast<T *>((char *)ws + off); }

ExpertLists moe_lists(void *ws, const MoeLayout &L, int E, int thr) {
    int32_t *b = at<int32_t>(ws, L.lists);
    return ExpertLists{b, b + 8, b + 1, b + 8 + E, thr};
}

int epl_for(int E) {
    int epl = 1;
    while (epl * 32 < E) epl *= 2;
    return epl;
}

gq4_status launch_route(const float *logits, int T, int E, int K, int32_t *idx, float *wts,
                        int32_t *status, cudaStream_t st) {
    const int grid = (T + 7) / 8;
    switch (epl_for(E)) {
#define ROUTE_CASE(N) case N: gq4_route_kernel<N><<<grid, 256, 0, st>>>(logits, T, E, K, idx, wts, status); break;
        ROUTE_CASE(1) ROUTE_CASE(2) ROUTE_CASE(4) ROUTE_CASE(8) ROUTE_CASE(16) ROUTE_CASE(32)
#undef ROUTE_CASE
        default: return GQ4_ERR_SHAPE;
    }
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

gq4_status launch_rowmap(const int32_t *idx, int n, int K, int E, int32_t *cnt, int32_t *offs,
                         int32_t *row_tok, int32_t *row_slot, int32_t *slot_row, int32_t *n_active,
                         int32_t *active, int32_t *chunk, int32_t *status, ExpertLists lists,
                         cudaStream_t st) {
    const int nchunks = (n + kChunk - 1) / kChunk;
    gq4_rowmap_count_kernel<<<nchunks, kChunk, 0, st>>>(idx, n, E, chunk, status);
    gq4_rowmap_scan_kernel<<<1, 1024, 0, st>>>(chunk, nchunks, E, cnt, offs, n_active, active, lists);
    const size_t smem = (size_t)32 * E * 4;
    if (allow_smem(gq4_rowmap_fill_kernel, smem) != cudaSuccess) return GQ4_ERR_CUDA;
    gq4_rowmap_fill_kernel<<<nchunks, kChunk, smem, st>>>(idx, n, K, E, chunk, row_tok, row_slot,
                                                          slot_row);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

gq4_status launch_route_rowmap_small(const float *logits, int T, int E, int K, void *ws,
                                     const MoeLayout &L, ExpertLists lists, cudaStream_t st) {
    const size_t smem = (size_t)33 * E * 4;
    int32_t *status = at<int32_t>(ws, L.status);
#define SMALL_ARGS logits, T, E, K, at<int32_t>(ws, L.idx), at<float>(ws, L.wts), status,      \
                   at<int32_t>(ws, L.cnt), at<int32_t>(ws, L.offs), at<int32_t>(ws, L.n_active), \
                   at<int32_t>(ws, L.active), at<int32_t>(ws, L.row_tok),                        \
                   at<int32_t>(ws, L.row_slot), at<int32_t>(ws, L.slot_row), lists
    switch (epl_for(E)) {
#define SMALL_CASE(N)                                                                    \
    case N:                                                                              \
        if (allow_smem(gq4_route_rowmap_small_kernel<N>, smem) != cudaSuccess) return GQ4_ERR_CUDA; \
        gq4_route_rowmap_small_kernel<N><<<1, 1024, smem, st>>>(SMALL_ARGS);             \
        break;
        SMALL_CASE(1) SMALL_CASE(2) SMALL_CASE(4) SMALL_CASE(8) SMALL_CASE(16) SMALL_CASE(32)
#undef SMALL_CASE
#undef SMALL_ARGS
        default: return GQ4_ERR_SHAPE;
    }
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

// Upload repack: host rows hold the weights of k = 8i..8i+7 in one little-endian 32-bit
// word as nibbles k0..k7 (low nibble first).  The device word holds the even-k nibbles
// (k0,k2,k4,k6) in its low 16 bits and the odd-k nibbles (k1,k3,k5,k7) in its high 16
// bits, so one lop3 turns nibble slots i and i+4 into the bf16 pair (k_2i, k_2i+1) of
// consecutive columns.  With offset-binary input every nibble's top bit is flipped
// first (XOR 0x88 per byte).
__device__ __forceinline__ uint32_t compact_nibbles(uint32_t v) {  // nibbles at bits 0,8,16,24
    v = (v | (v >> 4)) & 0x00FF00FFu;
    return (v | (v >> 8)) & 0x0000FFFFu;
}

__global__ void gq4_repack_kernel(uint32_t *w, size_t nwords, uint32_t flip) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nwords;
         i += (size_t)gridDim.x * blockDim.x) {
        const uint32_t v = w[i] ^ flip;
        w[i] = compact_nibbles(v & 0x0F0F0F0Fu) | (compact_nibbles((v >> 4) & 0x0F0F0F0Fu) << 16);
    }
}

// ---- TMA descriptors (driver entry point, no libcuda link) ------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

// 2-D map over a row-major [rows][cols] array; box = box_cols x box_rows.
bool make_tmap_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, size_t esz, uint64_t cols,
                  uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * esz};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activation maps with 16/32/64/128-row boxes over a row-major bf16 [rows][cols] array.
bool make_act_maps(CUtensorMap (&m)[4], const void *base, uint64_t cols, uint64_t rows) {
    const uint32_t box_rows[4] = {16, 32, 64, 128};
    for (int i = 0; i < 4; ++i)
        if (!make_tmap_2d(&m[i], base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cols, rows, 64, box_rows[i],
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    return true;
}

// ---- TMA-fed decode kernel (gq4_stream.cuh) ------------------------------------------
// The matrices (or expert stacks) it reads: packed weights and scales of matrix 0 and,
// for gate+up, matrix 1, with their expert strides in rows.
struct StreamMats {
    const uint8_t *w0, *w1;
    const float *s0, *s1;
    int64_t n_experts, wrows, srows;  // expert strides in rows of the packed / scale arrays
};

// The kernel streams whole four-group stages and addresses experts by row: bf16
// activations, ng % 4 == 0, and expert strides that are whole rows.
bool stream_usable(const gq4_tensor *t) {
    if (t->ng % kStGroups) return false;
    if (t->n_experts > 1 && (t->expert_stride_w % (t->in / 2) || t->expert_stride_s % t->ng)) return false;
    return true;
}

StreamMats stream_mats(const gq4_tensor *t0, const gq4_tensor *t1) {
    StreamMats m{};
    m.w0 = t0->w; m.s0 = t0->s;
    m.w1 = t1 ? t1->w : t0->w; m.s1 = t1 ? t1->s : t0->s;
    m.n_experts = t0->n_experts;
    m.wrows = t0->n_experts > 1 ? t0->expert_stride_w / (t0->in / 2) : t0->out;
    m.srows = t0->n_experts > 1 ? t0->expert_stride_s / t0->ng : t0->out;
    return m;
}

template <int MODE, int NT, int RW>
gq4_status launch_stream_k(const StreamMats &m, const SkinnyParams &p, int units_upper, int32_t *status,
                           cudaStream_t st) {
    constexpr int PAIR = ModeTraits<MODE>::kPair;
    constexpr int BR = 16 * RW;
    auto kern = gq4_stream_kernel<MODE, NT, RW>;
    StreamArgs a{};
    a.stage_bytes = stream_stage_bytes(PAIR, BR, std::min(kStMaxCols, NT * 8));
    if (ModeTraits<MODE>::kMoe && !p.unit_ctr) return GQ4_ERR_NULL;
    const int budget = (int)kMaxSmem - stream_xch_bytes(PAIR, RW, NT) - 16 - 16 * kStQueue - 1024;
    a.nstages = std::min(8, budget / (a.stage_bytes + 16));
    if (a.nstages < 2) return GQ4_ERR_UNSUPPORTED;
    a.wrows = (int)m.wrows;
    a.srows = (int)m.srows;
    a.status = status;
    const size_t smem = stream_smem_bytes(a.nstages, a.stage_bytes, PAIR, RW, NT);
    if (smem > kMaxSmem) return GQ4_ERR_UNSUPPORTED;
    CUtensorMap tm[4];
    const uint64_t rows_w = (uint64_t)(m.n_experts - 1) * m.wrows + p.O;
    const uint64_t rows_s = (uint64_t)(m.n_experts - 1) * m.srows + p.O;
    for (int i = 0; i < 2; ++i) {
        if (!make_tmap_2d(&tm[i], i ? m.w1 : m.w0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.I / 2, rows_w, 128, BR,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_2d(&tm[2 + i], i ? m.s1 : m.s0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.ng, rows_s,
                          kStGroups, BR, CU_TENSOR_MAP_SWIZZLE_NONE))
            return GQ4_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GQ4_ERR_CUDA;
    const int grid = std::max(1, std::min(units_upper, sm_count()));
    if constexpr (ModeTraits<MODE>::kMoe) {
        // programmatic dependent launch: the kernel may start while the one ahead of it
        // finishes, and waits for that kernel's results inside (griddepcontrol.wait)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(kStThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, tm[0], tm[1], tm[2], tm[3], p, a) != cudaSuccess) return GQ4_ERR_CUDA;
    } else {
        kern<<<grid, kStThreads, smem, st>>>(tm[0], tm[1], tm[2], tm[3], p, a);
    }
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

// Band height.  MoE modes: the tallest band (gate+up 128 rows of each matrix, down 256):
// the expert count is only an upper bound on the host, and large stages keep more bytes
// in flight per SM (one token's eight experts ran 11 % faster than with 64-row bands).
// Dense matvec: the tallest band whose unit count gives every SM at least two bands
// (256, 128 or 64 rows), else the smallest.  (32-row gate+up bands balance one token's
// experts better on paper but ran slower: their TMA boxes and stages are too small.)
// The n-tile count covers the columns of one pass.  `mats` = matrices (experts) the
// call may touch.
template <int MODE, int NT>
gq4_status launch_stream_nt(const StreamMats &m, const SkinnyParams &p, int mats, int32_t *status,
                            cudaStream_t st) {
    auto units = [&](int br) { return mats * ((p.O + br - 1) / br); };
    const int want = 2 * sm_count();
    if constexpr (ModeTraits<MODE>::kMoe) {
        return launch_stream_k<MODE, NT, ModeTraits<MODE>::kPair == 2 ? 8 : 16>(m, p, units(ModeTraits<MODE>::kPair == 2 ? 128 : 256),
                                                                                 status, st);
    } else if constexpr (ModeTraits<MODE>::kPair == 2) {
        if (units(128) >= want) return launch_stream_k<MODE, NT, 8>(m, p, units(128), status, st);
        return launch_stream_k<MODE, NT, 4>(m, p, units(64), status, st);
    } else {
        if (units(256) >= want) return launch_stream_k<MODE, NT, 16>(m, p, units(256), status, st);
        if (units(128) >= want) return launch_stream_k<MODE, NT, 8>(m, p, units(128), status, st);
        return launch_stream_k<MODE, NT, 4>(m, p, units(64), status, st);
    }
}

// At most three n-tiles (24 columns) per pass: the four-tile variant needs more registers
// than the 16 consumer warps have and spills; a matrix with more columns takes passes.
// Routed experts take at most two (16 columns): the smaller stage leaves room for a fifth
// ring stage, which gained more than the second pass of the few experts with 17-24 rows
// cost (32-token decode, 64 or 32 experts: 4-8 % less time).
template <int MODE>
gq4_status launch_stream(const StreamMats &m, const SkinnyParams &p, int max_cols, int mats, int32_t *status,
                         cudaStream_t st) {
    const int c = std::min(max_cols, kStMaxCols);
    if (c <= 8) return launch_stream_nt<MODE, 1>(m, p, mats, status, st);
    if constexpr (ModeTraits<MODE>::kMoe) {
        return launch_stream_nt<MODE, 2>(m, p, mats, status, st);
    } else {
        if (c <= 16) return launch_stream_nt<MODE, 2>(m, p, mats, status, st);
        return launch_stream_nt<MODE, 3>(m, p, mats, status, st);
    }
}

template <int MODE>
gq4_status launch_tc(const CUtensorMap &w0, const CUtensorMap &w1, const CUtensorMap (&x)[4],
                     const TcParams &p, int units_upper, cudaStream_t st) {
    auto kern = gq4_tc_kernel<MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes) != cudaSuccess)
        return GQ4_ERR_CUDA;
    // the kernel's register split (setmaxnreg) must fit in what the launch allocates
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return GQ4_ERR_CUDA;
    if ((int64_t)fa.numRegs * kTcThreads < kTcRegsNeeded) return GQ4_ERR_UNSUPPORTED;
    const int grid = std::max(1, std::min(units_upper, sm_count()));
    kern<<<grid, kTcThreads, kTcSmemBytes, st>>>(w0, w1, x[0], x[1], x[2], x[3], p);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

}  // namespace

// Group sizes the mma.sync split-K kernel also takes: 64 << k with in % 64 == 0 (a group
// is 2^k consecutive 64-wide groups sharing one scale).  -1 when not of that form.
int wide_group_shift(const gq4_tensor *t) {
    if (t->in % 64) return -1;
    for (int k = 0; k < 15; ++k)
        if (t->gs == (64 << k)) return k;
    return -1;
}

// ---- generic kernels (gq4_aux.cuh) ----------------------------------------------------
// Matvec / gate+up over all rows or selected rows, any group size that is a multiple of 8.
template <int MODE>
gq4_status launch_generic(const gq4_tensor *W0, const gq4_tensor *W1, int64_t n_rows, const int32_t *rows,
                          const void *x, gq4_dtype xdt, int64_t n_tok, void *out, cudaStream_t st) {
    const size_t xbytes = (size_t)n_tok * W0->in * 4;
    const int stage = xbytes <= 96 * 1024 ? 1 : 0;
    const size_t smem = stage ? xbytes : 0;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n_rows + 7) / 8, (int64_t)sm_count() * 8));
#define GEN_LAUNCH(XDT)                                                                                    \
    {                                                                                                      \
        auto kern = gq4_generic_kernel<MODE, XDT>;                                                         \
        if (allow_smem(kern, smem) != cudaSuccess) return GQ4_ERR_CUDA;                                    \
        kern<<<blocks, 256, smem, st>>>((const uint32_t *)W0->w, W0->s,                                    \
                                        (const uint32_t *)(W1 ? W1->w : W0->w), W1 ? W1->s : W0->s,        \
                                        W0->out, n_rows, rows, W0->in, W0->gs, W0->ng, x, (int)n_tok,      \
                                        stage, out);                                                       \
    }
    if (xdt == GQ4_BF16) GEN_LAUNCH(1) else GEN_LAUNCH(0)
#undef GEN_LAUNCH
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

// =====================================================================================
extern "C" {

uint32_t gq4_abi_version(void) { return GQ4_ABI_VERSION; }

const char *gq4_status_string(int status) {
    switch (status) {
        case GQ4_OK: return "ok";
        case GQ4_ERR_NULL: return "a required pointer is NULL";
        case GQ4_ERR_ALIGN: return "a device pointer or stride is not 16-byte aligned";
        case GQ4_ERR_SHAPE: return "inconsistent or out-of-range sizes";
        case GQ4_ERR_UNSUPPORTED: return "format or size not supported by the GPU kernels";
        case GQ4_ERR_ALIAS: return "an output overlaps an input";
        case GQ4_ERR_WORKSPACE: return "workspace too small";
        case GQ4_ERR_CUDA: return "CUDA runtime error";
        case GQ4_ERR_TIMEOUT: return "a bounded device wait gave up";
        case GQ4_ERR_NONFINITE_LOGIT: return "router logits hold NaN/+inf or no finite maximum";
        case GQ4_ERR_BOUNDS: return "an index fell outside its array (checked build)";
        default: return "unknown status";
    }
}

gq4_status gq4_pack(const int8_t *q, int64_t out, int64_t in, int32_t gs,
                    int32_t src_offset_binary, uint8_t *packed_host) {
    if (!q || !packed_host) return GQ4_ERR_NULL;
    if (out < 0 || in < 0 || gs <= 0) return GQ4_ERR_SHAPE;
    const int64_t rb = (in + 1) / 2;
    for (int64_t o = 0; o < out; ++o) {
        const int8_t *qr = q + o * in;
        uint8_t *dst = packed_host + o * rb;
        for (int64_t b = 0; b < rb; ++b) {
            int lo = qr[2 * b], hi = (2 * b + 1 < in) ? qr[2 * b + 1] : 0;
            if (src_offset_binary) {
                if (lo < 0 || lo > 15 || hi < 0 || hi > 15) return GQ4_ERR_SHAPE;
                lo -= 8;
                hi = (2 * b + 1 < in) ? hi - 8 : 0;
            } else if (lo < -8 || lo > 7 || hi < -8 || hi > 7) {
                return GQ4_ERR_SHAPE;
            }
            dst[b] = (uint8_t)((lo & 15) | ((hi & 15) << 4));
        }
    }
    return GQ4_OK;
}

gq4_status gq4_device_bytes(int64_t out, int64_t in, int32_t gs, int32_t n_experts,
                            size_t *w_bytes, size_t *s_bytes) {
    if (!w_bytes || !s_bytes) return GQ4_ERR_NULL;
    if (out < 1 || in < 1 || gs <= 0 || n_experts < 1) return GQ4_ERR_SHAPE;
    *w_bytes = (size_t)n_experts * out * ((in + 1) / 2);
    *s_bytes = (size_t)n_experts * out * ((in + gs - 1) / gs) * 4;
    return GQ4_OK;
}

gq4_status gq4_tensor_init(const void *d_w, const float *d_s, int64_t out, int64_t in,
                           int32_t gs, int32_t n_experts, gq4_tensor *desc) {
    if (!d_w || !d_s || !desc) return GQ4_ERR_NULL;
    if (out < 1 || in < 1 || gs <= 0 || n_experts < 1) return GQ4_ERR_SHAPE;
    gq4_tensor t{};
    t.out = out;
    t.in = in;
    t.gs = gs;
    t.ng = (int32_t)((in + gs - 1) / gs);
    t.n_experts = n_experts;
    t.w = (const uint8_t *)d_w;
    t.s = d_s;
    t.expert_stride_w = out * ((in + 1) / 2);
    t.expert_stride_s = out * t.ng;
    *desc = t;
    return GQ4_OK;
}

gq4_status gq4_upload(const uint8_t *packed_host, const float *scales_host, int64_t out,
                      int64_t in, int32_t gs, int32_t n_experts, int32_t src_offset_binary,
                      void *d_w, size_t d_w_bytes, float *d_s, size_t d_s_bytes,
                      gq4_stream_t stream, gq4_tensor *desc) {
    if (!packed_host || !scales_host || !d_w || !d_s || !desc) return GQ4_ERR_NULL;
    size_t wb = 0, sb = 0;
    gq4_status st = gq4_device_bytes(out, in, gs, n_experts, &wb, &sb);
    if (st != GQ4_OK) return st;
    if (d_w_bytes < wb || d_s_bytes < sb) return GQ4_ERR_SHAPE;
    if (in % 8) return GQ4_ERR_UNSUPPORTED;  // device words hold 8 weights of one row
    if (!aligned16(d_w) || !aligned16(d_s)) return GQ4_ERR_ALIGN;
    if (overlap(rng(d_w, wb), rng(d_s, sb))) return GQ4_ERR_ALIAS;
    cudaStream_t s = S(stream);
    if (cudaMemcpyAsync(d_w, packed_host, wb, cudaMemcpyHostToDevice, s) != cudaSuccess) return GQ4_ERR_CUDA;
    if (cudaMemcpyAsync(d_s, scales_host, sb, cudaMemcpyHostToDevice, s) != cudaSuccess) return GQ4_ERR_CUDA;
    {
        const size_t nwords = wb / 4;
        const unsigned grid = (unsigned)std::min<size_t>((nwords + 255) / 256, (size_t)sm_count() * 8);
        gq4_repack_kernel<<<std::max(grid, 1u), 256, 0, s>>>((uint32_t *)d_w, nwords,
                                                           src_offset_binary ? 0x88888888u : 0u);
        if (cudaGetLastError() != cudaSuccess) return GQ4_ERR_CUDA;
    }
    return gq4_tensor_init(d_w, d_s, out, in, gs, n_experts, desc);
}

gq4_status gq4_matvec(const gq4_tensor *W, const void *x, gq4_dtype xdt, int64_t n_tok,
                      float *y, gq4_stream_t stream) {
    gq4_status st = check_tensor_generic(W, 1);
    if (st != GQ4_OK) return st;
    if (!x || !y) return GQ4_ERR_NULL;
    if (xdt != GQ4_F32 && xdt != GQ4_BF16) return GQ4_ERR_UNSUPPORTED;
    if (n_tok < 1 || n_tok > (1 << 20)) return GQ4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(y)) return GQ4_ERR_ALIGN;
    const size_t xb = (size_t)n_tok * W->in * (xdt == GQ4_F32 ? 4 : 2);
    const Range yr = rng(y, (size_t)n_tok * W->out * 4);
    if (overlap(yr, rng(x, xb)) || overlap(yr, rng(W->w, tensor_w_bytes(W))) ||
        overlap(yr, rng(W->s, tensor_s_bytes(W))))
        return GQ4_ERR_ALIAS;
    SkinnyParams p{};
    p.w0 = W->w; p.s0 = W->s;
    p.O = (int)W->out; p.I = (int)W->in; p.ng = W->ng;
    p.row_tiles = (int)((W->out + 15) / 16);
    p.x = x; p.xdt = (int)xdt; p.n_tok = (int)n_tok;
    p.y = y;
    set_extents(p, W, nullptr, n_tok, 1);
    const int cols = (int)(xdt == GQ4_F32 ? 3 * n_tok : n_tok);
    if (check_tensor(W, 1) != GQ4_OK) {  // another group size or a partial last group
        const int sh = wide_group_shift(W);
        if (sh < 0) return launch_generic<0>(W, nullptr, W->out, nullptr, x, xdt, n_tok, y, S(stream));
        p.ng = (int)(W->in / 64);  // 64-wide groups; the scale of group G is column G >> sh
        p.sng = W->ng;
        p.gshift = sh;
        return launch_skinny<kMatvec>(p, cols, xdt == GQ4_F32, p.row_tiles, S(stream));
    }
    if (xdt == GQ4_BF16 && stream_usable(W) && (n_tok >= kBandMinCols || (W->out + 63) / 64 >= sm_count()))
        return launch_stream<kMatvec>(stream_mats(W, nullptr), p, cols, 1, nullptr, S(stream));
    if (xdt == GQ4_BF16 && n_tok >= kBandMinCols)
        return launch_band<kMatvec>(p, cols, (p.row_tiles + 7) / 8, nullptr, S(stream));
    return launch_skinny<kMatvec>(p, cols, xdt == GQ4_F32, p.row_tiles, S(stream));
}

gq4_status gq4_gate_up_silu(const gq4_tensor *Wg, const gq4_tensor *Wu, const void *x,
                            gq4_dtype xdt, int64_t n_tok, void *h, gq4_stream_t stream) {
    gq4_status st = check_tensor_generic(Wg, 1);
    if (st != GQ4_OK) return st;
    st = check_tensor_generic(Wu, 1);
    if (st != GQ4_OK) return st;
    if (Wg->out != Wu->out || Wg->in != Wu->in || Wg->gs != Wu->gs) return GQ4_ERR_SHAPE;
    if (!x || !h) return GQ4_ERR_NULL;
    if (xdt != GQ4_F32 && xdt != GQ4_BF16) return GQ4_ERR_UNSUPPORTED;
    if (n_tok < 1 || n_tok > (1 << 20)) return GQ4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(h)) return GQ4_ERR_ALIGN;
    const size_t esz = xdt == GQ4_F32 ? 4 : 2;
    const Range hr = rng(h, (size_t)n_tok * Wg->out * esz);
    if (overlap(hr, rng(x, (size_t)n_tok * Wg->in * esz)) ||
        overlap(hr, rng(Wg->w, tensor_w_bytes(Wg))) || overlap(hr, rng(Wg->s, tensor_s_bytes(Wg))) ||
        overlap(hr, rng(Wu->w, tensor_w_bytes(Wu))) || overlap(hr, rng(Wu->s, tensor_s_bytes(Wu))))
        return GQ4_ERR_ALIAS;
    SkinnyParams p{};
    p.w0 = Wg->w; p.s0 = Wg->s; p.w1 = Wu->w; p.s1 = Wu->s;
    p.O = (int)Wg->out; p.I = (int)Wg->in; p.ng = Wg->ng;
    p.row_tiles = (int)((Wg->out + 15) / 16);
    p.x = x; p.xdt = (int)xdt; p.n_tok = (int)n_tok;
    p.h = h;
    set_extents(p, Wg, Wu, n_tok, 1);
    const int cols = (int)(xdt == GQ4_F32 ? 3 * n_tok : n_tok);
    if (check_tensor(Wg, 1) != GQ4_OK || check_tensor(Wu, 1) != GQ4_OK) {  // general group size
        const int sh = wide_group_shift(Wg);
        if (sh < 0) return launch_generic<1>(Wg, Wu, Wg->out, nullptr, x, xdt, n_tok, h, S(stream));
        p.ng = (int)(Wg->in / 64);
        p.sng = Wg->ng;
        p.gshift = sh;
        return launch_skinny<kGateUp>(p, cols, xdt == GQ4_F32, p.row_tiles, S(stream));
    }
    if (xdt == GQ4_BF16 && stream_usable(Wg) && stream_usable(Wu) &&
        (n_tok >= kBandMinCols || (Wg->out + 63) / 64 >= sm_count()))
        return launch_stream<kGateUp>(stream_mats(Wg, Wu), p, cols, 1, nullptr, S(stream));
    if (xdt == GQ4_BF16 && n_tok >= kBandMinCols)
        return launch_band<kGateUp>(p, cols, (p.row_tiles + 7) / 8, nullptr, S(stream));
    return launch_skinny<kGateUp>(p, cols, xdt == GQ4_F32, p.row_tiles, S(stream));
}

gq4_status gq4_route(const float *logits, int64_t T, int32_t E, int32_t K, int32_t *idx,
                     float *wts, int32_t *status, gq4_stream_t stream) {
    if (!logits || !idx || !wts || !status) return GQ4_ERR_NULL;
    if (T < 1 || T > (1 << 24) || E < 1 || E > kMaxExperts || K < 1 || K > E) return GQ4_ERR_SHAPE;
    if (!aligned16(logits) || !aligned16(idx) || !aligned16(wts) || !aligned16(status)) return GQ4_ERR_ALIGN;
    const Range lr = rng(logits, (size_t)T * E * 4);
    const Range ir = rng(idx, (size_t)T * K * 4), wr = rng(wts, (size_t)T * K * 4), sr = rng(status, 4);
    if (overlap(lr, ir) || overlap(lr, wr) || overlap(lr, sr) || overlap(ir, wr) || overlap(ir, sr) ||
        overlap(wr, sr))
        return GQ4_ERR_ALIAS;
    return launch_route(logits, (int)T, E, K, idx, wts, status, S(stream));
}

size_t gq4_rowmap_scratch_bytes(int64_t T, int32_t K, int32_t E) {
    if (T < 1 || K < 1 || E < 1) return 0;
    const size_t n = (size_t)T * K;
    return al256(16) + ((n + kChunk - 1) / kChunk) * (size_t)E * 4;
}

gq4_status gq4_rowmap(const int32_t *idx, int64_t T, int32_t K, int32_t E, int32_t *cnt,
                      int32_t *offs, int32_t *row_tok, int32_t *row_slot, int32_t *slot_row,
                      int32_t *n_active, int32_t *active, void *scratch, size_t scratch_bytes,
                      gq4_stream_t stream) {
    if (!idx || !cnt || !offs || !row_tok || !row_slot || !slot_row || !n_active || !active || !scratch)
        return GQ4_ERR_NULL;
    if (T < 1 || E < 1 || E > kMaxExperts || K < 1 || K > E || T * (int64_t)K > (1 << 26))
        return GQ4_ERR_SHAPE;
    if (scratch_bytes < gq4_rowmap_scratch_bytes(T, K, E)) return GQ4_ERR_WORKSPACE;
    const void *ptrs[] = {idx, cnt, offs, row_tok, row_slot, slot_row, n_active, active, scratch};
    for (const void *q : ptrs)
        if (!aligned16(q)) return GQ4_ERR_ALIGN;
    const size_t n = (size_t)T * K;
    const Range rs[] = {rng(idx, n * 4), rng(cnt, E * 4), rng(offs, (E + 1) * 4), rng(row_tok, n * 4),
                        rng(row_slot, n * 4), rng(slot_row, n * 4), rng(n_active, 4),
                        rng(active, E * 4), rng(scratch, scratch_bytes)};
    for (int i = 0; i < 9; ++i)
        for (int j = i + 1; j < 9; ++j)
            if (overlap(rs[i], rs[j])) return GQ4_ERR_ALIAS;
    cudaStream_t s = S(stream);
    int32_t *status = (int32_t *)scratch;
    int32_t *chunk = (int32_t *)((char *)scratch + al256(16));
    if (cudaMemsetAsync(status, 0, 16, s) != cudaSuccess) return GQ4_ERR_CUDA;
    return launch_rowmap(idx, (int)n, K, E, cnt, offs, row_tok, row_slot, slot_row, n_active,
                         active, chunk, status, ExpertLists{nullptr, nullptr, nullptr, nullptr, 1 << 30}, s);
}

size_t moe_expert_ffn_workspace_bytes(int64_t T, int32_t E, int32_t K, int64_t H, int64_t F) {
    if (T < 1 || E < 1 || K < 1 || H < 1 || F < 1) return 0;
    return moe_layout(T, E, K, H, F).total;
}

gq4_status moe_expert_ffn_routing(void *ws, size_t ws_bytes, int64_t T, int32_t E, int32_t K,
                                  int64_t H, int64_t F, gq4_routing *out) {
    if (!ws || !out) return GQ4_ERR_NULL;
    if (T < 1 || E < 1 || K < 1 || K > E || H < 1 || F < 1) return GQ4_ERR_SHAPE;
    const MoeLayout L = moe_layout(T, E, K, H, F);
    if (ws_bytes < L.total) return GQ4_ERR_WORKSPACE;
    out->idx = at<int32_t>(ws, L.idx);
    out->wts = at<float>(ws, L.wts);
    out->cnt = at<int32_t>(ws, L.cnt);
    out->offs = at<int32_t>(ws, L.offs);
    out->row_tok = at<int32_t>(ws, L.row_tok);
    out->row_slot = at<int32_t>(ws, L.row_slot);
    out->slot_row = at<int32_t>(ws, L.slot_row);
    out->n_active = at<int32_t>(ws, L.n_active);
    out->active = at<int32_t>(ws, L.active);
    out->status = at<int32_t>(ws, L.status);
    out->h = at<uint16_t>(ws, L.h);
    return GQ4_OK;
}

gq4_status moe_expert_ffn_status(const void *ws, size_t ws_bytes, int64_t T, int32_t E, int32_t K,
                                 int64_t H, int64_t F, gq4_stream_t stream, int32_t *status) {
    if (!ws || !status) return GQ4_ERR_NULL;
    if (T < 1 || E < 1 || K < 1 || H < 1 || F < 1) return GQ4_ERR_SHAPE;
    const MoeLayout L = moe_layout(T, E, K, H, F);
    if (ws_bytes < L.total) return GQ4_ERR_WORKSPACE;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, (const char *)ws + L.status, 4, cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
        return GQ4_ERR_CUDA;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return GQ4_ERR_CUDA;
    *status = v;
    return GQ4_OK;
}

gq4_status moe_expert_ffn(const gq4_tensor *Wg, const gq4_tensor *Wu, const gq4_tensor *Wd,
                          const float *logits, const void *x, gq4_dtype xdt, int64_t T,
                          int32_t E, int32_t K, float *y, void *ws, size_t ws_bytes,
                          gq4_event_t const *stage_events, gq4_stream_t stream) {
    gq4_status st;
    if ((st = check_tensor(Wg, 1)) != GQ4_OK) return st;
    if ((st = check_tensor(Wu, 1)) != GQ4_OK) return st;
    if ((st = check_tensor(Wd, 1)) != GQ4_OK) return st;
    if (!logits || !x || !y || !ws) return GQ4_ERR_NULL;
    if (xdt != GQ4_BF16) return GQ4_ERR_UNSUPPORTED;
    if (T < 1 || T > (1 << 20) || E < 1 || E > kMaxExperts || K < 1 || K > E) return GQ4_ERR_SHAPE;
    const int64_t H = Wg->in, F = Wg->out;
    if (Wu->out != F || Wu->in != H || Wd->out != H || Wd->in != F) return GQ4_ERR_SHAPE;
    if (Wg->n_experts < E || Wu->n_experts < E || Wd->n_experts < E) return GQ4_ERR_SHAPE;
    if (!aligned16(logits) || !aligned16(x) || !aligned16(y) || !aligned16(ws)) return GQ4_ERR_ALIGN;
    const MoeLayout L = moe_layout(T, E, K, H, F);
    if (ws_bytes < L.total) return GQ4_ERR_WORKSPACE;
    const Range yr = rng(y, (size_t)T * H * 4), wr = rng(ws, L.total);
    const Range ins[] = {rng(logits, (size_t)T * E * 4), rng(x, (size_t)T * H * 2),
                         rng(Wg->w, tensor_w_bytes(Wg)), rng(Wg->s, tensor_s_bytes(Wg)),
                         rng(Wu->w, tensor_w_bytes(Wu)), rng(Wu->s, tensor_s_bytes(Wu)),
                         rng(Wd->w, tensor_w_bytes(Wd)), rng(Wd->s, tensor_s_bytes(Wd))};
    for (const Range &r : ins)
        if (overlap(yr, r) || overlap(wr, r)) return GQ4_ERR_ALIAS;
    if (overlap(yr, wr)) return GQ4_ERR_ALIAS;

    cudaStream_t s = S(stream);
    bool marks_ok = true;  // a failed event record is reported after the launches
    auto mark = [&](int i) {
        if (!stage_events || !stage_events[i]) return;
        // inside a stream capture the record must be external to become a timestamped
        // graph node; outside a capture the flag is not accepted
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        cudaStreamIsCapturing(s, &cap);
        const cudaError_t e = cap == cudaStreamCaptureStatusActive
                                  ? cudaEventRecordWithFlags((cudaEvent_t)stage_events[i], s, cudaEventRecordExternal)
                                  : cudaEventRecord((cudaEvent_t)stage_events[i], s);
        if (e != cudaSuccess) {
            marks_ok = false;
            cudaGetLastError();  // do not let it be read as a failed launch
        }
    };
    const int n = (int)(T * K);
    mark(0);
    // the one-block decode router clears the status word itself; the chunked path needs a memset
    if (n > kChunk && cudaMemsetAsync(at<int32_t>(ws, L.status), 0, 16, s) != cudaSuccess) return GQ4_ERR_CUDA;
    // an expert can reach kLargeMin rows only if T does; the tensor-core kernels tile the
    // down rows by 128 and load scales four groups at a time
    const bool tc = T >= kLargeMin && H % 128 == 0 && F % 64 == 0 && Wg->ng % 4 == 0 && Wd->ng % 4 == 0 &&
                    Wg->expert_stride_w % (H / 2) == 0 && Wu->expert_stride_w == Wg->expert_stride_w &&
                    Wd->expert_stride_w % (F / 2) == 0;
    const ExpertLists lists = moe_lists(ws, L, E, tc ? kLargeMin : (1 << 30));
    // router + row map
    if (n <= kChunk) {
        st = launch_route_rowmap_small(logits, (int)T, E, K, ws, L, lists, s);
    } else {
        st = launch_route(logits, (int)T, E, K, at<int32_t>(ws, L.idx), at<float>(ws, L.wts),
                          at<int32_t>(ws, L.status), s);
        if (st == GQ4_OK)
            st = launch_rowmap(at<int32_t>(ws, L.idx), n, K, E, at<int32_t>(ws, L.cnt),
                               at<int32_t>(ws, L.offs), at<int32_t>(ws, L.row_tok),
                               at<int32_t>(ws, L.row_slot), at<int32_t>(ws, L.slot_row),
                               at<int32_t>(ws, L.n_active), at<int32_t>(ws, L.active),
                               at<int32_t>(ws, L.chunk), at<int32_t>(ws, L.status), lists, s);
    }
    if (st != GQ4_OK) return st;
    mark(1);

    // expert gate+up (h in row-map order) and down with the weighted scatter-add
    SkinnyParams p{};
    p.offs = at<int32_t>(ws, L.offs);
    p.cnt = at<int32_t>(ws, L.cnt);
    p.row_tok = at<int32_t>(ws, L.row_tok);
    p.row_slot = at<int32_t>(ws, L.row_slot);
    p.n_active = lists.n_small;  // the decode kernels take the experts with few rows
    p.active = lists.small;
    p.wts = at<float>(ws, L.wts);
    const int max_active = (int)std::min<int64_t>(E, (int64_t)T * K);
    const int max_cols = (int)std::min<int64_t>(T, 1 << 20);

    SkinnyParams pg = p;
    pg.w0 = Wg->w; pg.s0 = Wg->s; pg.w1 = Wu->w; pg.s1 = Wu->s;
    pg.estride_w = Wg->expert_stride_w; pg.estride_s = Wg->expert_stride_s;
    if (Wu->expert_stride_w != Wg->expert_stride_w || Wu->expert_stride_s != Wg->expert_stride_s)
        return GQ4_ERR_SHAPE;
    pg.O = (int)F; pg.I = (int)H; pg.ng = Wg->ng;
    pg.row_tiles = (int)((F + 15) / 16);
    pg.x = x; pg.xdt = 1; pg.n_tok = (int)T;
    pg.h = at<void>(ws, L.h);
    pg.zero_ptr = y; pg.zero_n = T * H;
    set_extents(pg, Wg, Wu, T, E);
    if ((T * H) % 4) return GQ4_ERR_SHAPE;
    const int small_cols = (int)std::min<int64_t>(max_cols, tc ? kLargeMin - 1 : max_cols);
    const bool band = small_cols >= kBandMinCols;
    int32_t *status = at<int32_t>(ws, L.status);
    // words 1 and 2 of the status block (cleared with it by the router or a memset) count
    // the units the two decode kernels have taken
    pg.unit_ctr = status + 1;
    const bool stream_gu = stream_usable(Wg) && stream_usable(Wu) && Wu->expert_stride_s == Wg->expert_stride_s;
    if (stream_gu)
        st = launch_stream<kMoeGateUp>(stream_mats(Wg, Wu), pg, small_cols, max_active, status, s);
    else
        st = band ? launch_band<kMoeGateUp>(pg, small_cols, max_active * ((pg.row_tiles + 7) / 8), status, s)
                  : launch_skinny<kMoeGateUp>(pg, small_cols, false, max_active * pg.row_tiles, s);
    if (st != GQ4_OK) return st;
    mark(2);

    // experts with many rows: gathered activations, tensor-core gate+up and down
    CUtensorMap tm_g, tm_u, tm_d, tm_x[4], tm_h[4];
    TcParams tp{};
    if (tc) {
        const int max_large = std::max(1, std::min<int>(E, (int)(T * K / kLargeMin)));
        const int chunks = (int)(H / 8);
        gq4_gather_rows_kernel<<<sm_count() * 4, 256, 0, s>>>((const uint4 *)x, at<int32_t>(ws, L.row_tok),
                                                             at<int32_t>(ws, L.offs), at<int32_t>(ws, L.cnt),
                                                             lists.n_large, lists.large, chunks,
                                                             at<uint4>(ws, L.xg), T, E);
        if (cudaGetLastError() != cudaSuccess) return GQ4_ERR_CUDA;
        const uint64_t rows_gu = (uint64_t)(Wg->n_experts - 1) * (Wg->expert_stride_w / (H / 2)) + F;
        const uint64_t rows_d = (uint64_t)(Wd->n_experts - 1) * (Wd->expert_stride_w / (F / 2)) + H;
        // packed weights: 64-row boxes of 128 B (four groups), 128B-swizzled
        if (!make_tmap_2d(&tm_g, Wg->w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H / 2, rows_gu, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_2d(&tm_u, Wu->w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H / 2, rows_gu, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_2d(&tm_d, Wd->w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, F / 2, rows_d, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_act_maps(tm_x, at<void>(ws, L.xg), H, n) || !make_act_maps(tm_h, at<void>(ws, L.h), F, n))
            return GQ4_ERR_CUDA;
        tp.offs = at<int32_t>(ws, L.offs);
        tp.cnt = at<int32_t>(ws, L.cnt);
        tp.n_large = lists.n_large;
        tp.large = lists.large;
        tp.row_tok = at<int32_t>(ws, L.row_tok);
        tp.row_slot = at<int32_t>(ws, L.row_slot);
        tp.wts = at<float>(ws, L.wts);
        tp.status = at<int32_t>(ws, L.status);
        tp.h = at<uint16_t>(ws, L.h);
        tp.y = y;
        tp.n_exp = E;
        tp.n_tok = (int)T;
        TcParams tg = tp;
        tg.s0 = Wg->s; tg.s1 = Wu->s; tg.estride_s = Wg->expert_stride_s;
        tg.O = (int)F; tg.I = (int)H; tg.ng = Wg->ng; tg.m_tiles = (int)(F / 64);
        tg.estride_rows = (int)(Wg->expert_stride_w / (H / 2));
        tg.s_count = (int64_t)(std::min(tensor_s_bytes(Wg), tensor_s_bytes(Wu)) / 4);
        st = launch_tc<0>(tm_g, tm_u, tm_x, tg, max_large * tg.m_tiles, s);
        if (st != GQ4_OK) return st;
    }
    mark(3);

    SkinnyParams pd = p;
    pd.w0 = Wd->w; pd.s0 = Wd->s;
    pd.estride_w = Wd->expert_stride_w; pd.estride_s = Wd->expert_stride_s;
    pd.O = (int)H; pd.I = (int)F; pd.ng = Wd->ng;
    pd.row_tiles = (int)((H + 15) / 16);
    pd.x = at<void>(ws, L.h); pd.xdt = 1; pd.n_tok = (int)T;
    pd.y = y;
    pd.unit_ctr = status + 2;
    set_extents(pd, Wd, nullptr, T * K, E);
    if (stream_usable(Wd))
        st = launch_stream<kMoeDown>(stream_mats(Wd, nullptr), pd, small_cols, max_active, status, s);
    else
        st = band ? launch_band<kMoeDown>(pd, small_cols, max_active * ((pd.row_tiles + 7) / 8), status, s)
                  : launch_skinny<kMoeDown>(pd, small_cols, false, max_active * pd.row_tiles, s);
    if (st != GQ4_OK) return st;
    mark(4);
    if (tc) {
        const int max_large = std::max(1, std::min<int>(E, (int)(T * K / kLargeMin)));
        TcParams td = tp;
        td.s0 = Wd->s; td.s1 = Wd->s; td.estride_s = Wd->expert_stride_s;
        td.O = (int)H; td.I = (int)F; td.ng = Wd->ng; td.m_tiles = (int)(H / 128);
        td.estride_rows = (int)(Wd->expert_stride_w / (F / 2));
        td.s_count = (int64_t)(tensor_s_bytes(Wd) / 4);
        st = launch_tc<1>(tm_d, tm_d, tm_h, td, max_large * td.m_tiles, s);
    }
    mark(5);
    return st != GQ4_OK ? st : (marks_ok ? GQ4_OK : GQ4_ERR_CUDA);
}

}  // extern "C"

// ---- allocation-free variant of moe_expert_ffn ------------------------------------------
// For callers that may not allocate device memory, the workspace lives in this one
// library-owned array.  In host code its name stands for a host-side shadow, not for
// device memory: the device address is looked up per device with cudaGetSymbolAddress
// and only that address is handed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GQ4_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kNoallocMaxDevices];  // device address of the array, per device

// Device address of the array on the current device (looked up on first use).
gq4_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ4_ERR_CUDA;
    if (dev < 0 || dev >= kNoallocMaxDevices) return GQ4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQ4_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return GQ4_OK;
}
}  // namespace

extern "C" gq4_status moe_expert_ffn_noalloc(const gq4_tensor *Wg, const gq4_tensor *Wu,
                                             const gq4_tensor *Wd, const float *logits,
                                             const void *x, gq4_dtype xdt, int64_t T, int32_t E,
                                             int32_t K, float *y, int32_t *status_out,
                                             gq4_stream_t stream) {
    if (!Wg || !Wu || !Wd) return GQ4_ERR_NULL;
    if (T < 1 || E < 1 || K < 1 || K > E || Wg->in < 1 || Wg->out < 1) return GQ4_ERR_SHAPE;
    if (status_out && !aligned16(status_out)) return GQ4_ERR_ALIGN;
    const MoeLayout L = moe_layout(T, E, K, Wg->in, Wg->out);
    if (L.total > GQ4_NOALLOC_SCRATCH_BYTES) return GQ4_ERR_WORKSPACE;
    if (!logits || !x || !y) return GQ4_ERR_NULL;
    gq4_status st = GQ4_OK;
    if (status_out) {
        // the status word is written after the layer: it must not sit inside any input
        // or output (weights and scales included), or the copy would overwrite them
        if ((st = check_tensor(Wg, 1)) != GQ4_OK || (st = check_tensor(Wu, 1)) != GQ4_OK ||
            (st = check_tensor(Wd, 1)) != GQ4_OK)
            return st;
        const Range sr = rng(status_out, 4);
        const Range others[] = {rng(y, (size_t)T * Wg->in * 4), rng(logits, (size_t)T * E * 4),
                                rng(x, (size_t)T * Wg->in * 2),
                                rng(Wg->w, tensor_w_bytes(Wg)), rng(Wg->s, tensor_s_bytes(Wg)),
                                rng(Wu->w, tensor_w_bytes(Wu)), rng(Wu->s, tensor_s_bytes(Wu)),
                                rng(Wd->w, tensor_w_bytes(Wd)), rng(Wd->s, tensor_s_bytes(Wd))};
        for (const Range &r : others)
            if (overlap(sr, r)) return GQ4_ERR_ALIAS;
    }
    void *ws = nullptr;
    if ((st = noalloc_scratch(&ws)) != GQ4_OK) return st;
    // moe_expert_ffn validates everything else and clears the status word itself
    st = moe_expert_ffn(Wg, Wu, Wd, logits, x, xdt, T, E, K, y, ws, GQ4_NOALLOC_SCRATCH_BYTES, nullptr,
                        stream);
    if (st != GQ4_OK || !status_out) return st;
    if (cudaMemcpyAsync(status_out, (const char *)ws + L.status, 4, cudaMemcpyDeviceToDevice, S(stream)) !=
        cudaSuccess)
        return GQ4_ERR_CUDA;
    return GQ4_OK;
}

// ---- group-size detection, quantisation, row dequantisation, matvec over rows ----------
extern "C" gq4_status gq4_detect_group_size(int64_t out, int64_t in, size_t scale_bytes, int32_t *gs_out) {
    if (!gs_out) return GQ4_ERR_NULL;
    if (out < 1 || in < 1) return GQ4_ERR_SHAPE;
    static const int32_t cand[8] = {16, 32, 48, 64, 96, 128, 192, 256};
    int32_t found = 0;
    for (int c = 0; c < 8; ++c) {
        const int64_t ng = (in + cand[c] - 1) / cand[c];
        if ((size_t)(out * ng * 4) != scale_bytes) continue;
        if (found) return GQ4_ERR_UNSUPPORTED;  // two candidates give the same size
        found = cand[c];
    }
    if (!found) return GQ4_ERR_SHAPE;
    *gs_out = found;
    return GQ4_OK;
}

extern "C" gq4_status gq4_quantize(const float *w, int64_t out, int64_t in, int32_t gs, void *d_w,
                                   size_t d_w_bytes, float *d_s, size_t d_s_bytes, gq4_stream_t stream,
                                   gq4_tensor *desc) {
    if (!w || !d_w || !d_s || !desc) return GQ4_ERR_NULL;
    if (out < 1 || in < 1 || gs < 1 || out > ((int64_t)1 << 30) || in > ((int64_t)1 << 20)) return GQ4_ERR_SHAPE;
    if (in % 8 || gs % 8) return GQ4_ERR_UNSUPPORTED;
    size_t wb = 0, sb = 0;
    gq4_status st = gq4_device_bytes(out, in, gs, 1, &wb, &sb);
    if (st != GQ4_OK) return st;
    if (d_w_bytes < wb || d_s_bytes < sb) return GQ4_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(d_w) || !aligned16(d_s)) return GQ4_ERR_ALIGN;
    const Range wr = rng(w, (size_t)out * in * 4), dwr = rng(d_w, wb), dsr = rng(d_s, sb);
    if (overlap(wr, dwr) || overlap(wr, dsr) || overlap(dwr, dsr)) return GQ4_ERR_ALIAS;
    const int ng = (int)((in + gs - 1) / gs);
    const int words = (int)std::min<int64_t>(gs / 8, 32);
    const int64_t groups = out * ng;
    const cudaStream_t s = S(stream);
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((groups * 32 / std::max(words, 1) + 255) / 256,
                                                                   (int64_t)sm_count() * 16));
#define QLAUNCH(SEG) gq4_quantize_kernel<SEG><<<blocks, 256, 0, s>>>(w, out, in, gs, ng, (uint32_t *)d_w, d_s)
    if (words <= 1) QLAUNCH(1);
    else if (words <= 2) QLAUNCH(2);
    else if (words <= 4) QLAUNCH(4);
    else if (words <= 8) QLAUNCH(8);
    else if (words <= 16) QLAUNCH(16);
    else QLAUNCH(32);
#undef QLAUNCH
    if (cudaGetLastError() != cudaSuccess) return GQ4_ERR_CUDA;
    return gq4_tensor_init(d_w, d_s, out, in, gs, 1, desc);
}

extern "C" gq4_status gq4_dequant_rows(const gq4_tensor *W, const int32_t *idx, int64_t n, const float *alpha,
                                       int32_t accumulate, void *out, gq4_dtype odt, gq4_stream_t stream) {
    gq4_status st = check_tensor_generic(W, 1);
    if (st != GQ4_OK) return st;
    if (!idx || !out) return GQ4_ERR_NULL;
    if (n < 1 || n > ((int64_t)1 << 30)) return GQ4_ERR_SHAPE;
    if (odt != GQ4_F32 && odt != GQ4_BF16) return GQ4_ERR_UNSUPPORTED;
    if (odt == GQ4_BF16 && accumulate) return GQ4_ERR_UNSUPPORTED;
    if (!aligned16(out) || !aligned16(idx) || (alpha && !aligned16(alpha))) return GQ4_ERR_ALIGN;
    const Range orr = rng(out, (size_t)n * W->in * (odt == GQ4_F32 ? 4 : 2));
    if (overlap(orr, rng(idx, (size_t)n * 4)) || overlap(orr, rng(W->w, tensor_w_bytes(W))) ||
        overlap(orr, rng(W->s, tensor_s_bytes(W))) || (alpha && overlap(orr, rng(alpha, (size_t)n * 4))))
        return GQ4_ERR_ALIAS;
    const cudaStream_t s = S(stream);
    const int64_t total = n * (W->in / 8);
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 16));
    if (odt == GQ4_F32)
        gq4_dequant_rows_kernel<0><<<blocks, 256, 0, s>>>((const uint32_t *)W->w, W->s, W->out, W->in, W->gs, W->ng,
                                                          idx, n, alpha, accumulate, out);
    else
        gq4_dequant_rows_kernel<1><<<blocks, 256, 0, s>>>((const uint32_t *)W->w, W->s, W->out, W->in, W->gs, W->ng,
                                                          idx, n, alpha, 0, out);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

extern "C" gq4_status gq4_matvec_rows(const gq4_tensor *W, const int32_t *idx, int64_t n_sel, const void *x,
                                      gq4_dtype xdt, int64_t n_tok, float *y, gq4_stream_t stream) {
    gq4_status st = check_tensor_generic(W, 1);
    if (st != GQ4_OK) return st;
    if (!idx || !x || !y) return GQ4_ERR_NULL;
    if (xdt != GQ4_F32 && xdt != GQ4_BF16) return GQ4_ERR_UNSUPPORTED;
    if (n_sel < 1 || n_sel > ((int64_t)1 << 30) || n_tok < 1 || n_tok > (1 << 20)) return GQ4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(y) || !aligned16(idx)) return GQ4_ERR_ALIGN;
    const Range yr = rng(y, (size_t)n_tok * n_sel * 4);
    if (overlap(yr, rng(x, (size_t)n_tok * W->in * (xdt == GQ4_F32 ? 4 : 2))) || overlap(yr, rng(idx, (size_t)n_sel * 4)) ||
        overlap(yr, rng(W->w, tensor_w_bytes(W))) || overlap(yr, rng(W->s, tensor_s_bytes(W))))
        return GQ4_ERR_ALIAS;
    const int sh = wide_group_shift(W);
    if (sh < 0) return launch_generic<0>(W, nullptr, n_sel, idx, x, xdt, n_tok, y, S(stream));
    // group sizes 64 << sh: the mma.sync split-K kernel over 16-row tiles of the gathered rows
    SkinnyParams p{};
    p.w0 = W->w; p.s0 = W->s;
    p.O = (int)W->out; p.I = (int)W->in; p.ng = (int)(W->in / 64);
    p.sng = W->ng;
    p.gshift = sh;
    p.rows = idx;
    p.n_out = (int)n_sel;
    p.row_tiles = (int)((n_sel + 15) / 16);
    p.x = x; p.xdt = (int)xdt; p.n_tok = (int)n_tok;
    p.y = y;
    set_extents(p, W, nullptr, n_tok, 1);
    const int cols = (int)(xdt == GQ4_F32 ? 3 * n_tok : n_tok);
    return launch_skinny<kMatvec>(p, cols, xdt == GQ4_F32, p.row_tiles, S(stream));
}

// ---------------------------------------------------------------------------------------
// Grouped-scale MLA absorb projections over the kv_b tensor
// ---------------------------------------------------------------------------------------
namespace {
gq4_status mla_check(const gq4_tensor *W, int32_t nh, int32_t dn, int32_t dv, int64_t T, const void *in,
                     gq4_dtype dt, const float *out) {
    gq4_status st = check_tensor_generic(W, 1);
    if (st != GQ4_OK) return st;
    if (!in || !out) return GQ4_ERR_NULL;
    if (dt != GQ4_F32 && dt != GQ4_BF16) return GQ4_ERR_UNSUPPORTED;
    if (nh < 1 || dn < 1 || dv < 1 || T < 1) return GQ4_ERR_SHAPE;
    if ((int64_t)nh * ((int64_t)dn + dv) != W->out) return GQ4_ERR_SHAPE;
    if ((T + kMlaTok - 1) / kMlaTok > 65535) return GQ4_ERR_SHAPE;
    if (W->in > kMlaMaxR || dn > kMlaMaxDn) return GQ4_ERR_UNSUPPORTED;
    if (!aligned16(in) || !aligned16(out)) return GQ4_ERR_ALIGN;
    return GQ4_OK;
}
}  // namespace

extern "C" gq4_status gq4_mla_absorb_q(const gq4_tensor *W, int32_t n_heads, int32_t d_nope, int32_t d_v,
                                       const void *q_nope, gq4_dtype qdt, int64_t T, float *q_lat,
                                       gq4_stream_t stream) {
    gq4_status st = mla_check(W, n_heads, d_nope, d_v, T, q_nope, qdt, q_lat);
    if (st != GQ4_OK) return st;
    const int R = (int)W->in;
    const Range o = rng(q_lat, (size_t)T * n_heads * R * 4);
    if (overlap(o, rng(q_nope, (size_t)T * n_heads * d_nope * (qdt == GQ4_F32 ? 4 : 2))) ||
        overlap(o, rng(W->w, tensor_w_bytes(W))) || overlap(o, rng(W->s, tensor_s_bytes(W))))
        return GQ4_ERR_ALIAS;
    const int words = R / 8;
    const int nsplit = words >= kMlaThreads ? 1 : kMlaThreads / words;
    const int threads = words >= kMlaThreads ? kMlaThreads : words * nsplit;
    const size_t smem = ((size_t)kMlaTok * d_nope + (nsplit > 1 ? (size_t)nsplit * kMlaTok * R : 0)) * 4;
    // key rows of a head split over blockIdx.z until the grid covers about two waves of
    // SMs (at least 16 rows per slice); the slices add into a zeroed output
    const int64_t tblocks = (T + kMlaTok - 1) / kMlaTok;
    int zs = (int)std::max<int64_t>(1, (2 * sm_count()) / ((int64_t)n_heads * tblocks));
    zs = std::max(1, std::min(zs, d_nope / 16));
    const dim3 grid((unsigned)n_heads, (unsigned)tblocks, (unsigned)zs);
    cudaStream_t s = S(stream);
    if (zs > 1 && cudaMemsetAsync(q_lat, 0, (size_t)T * n_heads * R * 4, s) != cudaSuccess) return GQ4_ERR_CUDA;
    if (qdt == GQ4_F32)
        gq4_mla_q_kernel<0><<<grid, threads, smem, s>>>((const uint32_t *)W->w, W->s, R, W->ng, W->gs, n_heads,
                                                        d_nope, d_v, q_nope, T, q_lat);
    else
        gq4_mla_q_kernel<1><<<grid, threads, smem, s>>>((const uint32_t *)W->w, W->s, R, W->ng, W->gs, n_heads,
                                                        d_nope, d_v, q_nope, T, q_lat);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

extern "C" gq4_status gq4_mla_absorb_v(const gq4_tensor *W, int32_t n_heads, int32_t d_nope, int32_t d_v,
                                       const void *lat, gq4_dtype ldt, int64_t T, float *o,
                                       gq4_stream_t stream) {
    gq4_status st = mla_check(W, n_heads, d_nope, d_v, T, lat, ldt, o);
    if (st != GQ4_OK) return st;
    const int R = (int)W->in;
    const Range orng = rng(o, (size_t)T * n_heads * d_v * 4);
    if (overlap(orng, rng(lat, (size_t)T * n_heads * R * (ldt == GQ4_F32 ? 4 : 2))) ||
        overlap(orng, rng(W->w, tensor_w_bytes(W))) || overlap(orng, rng(W->s, tensor_s_bytes(W))))
        return GQ4_ERR_ALIAS;
    const int rows_per_block = (kMlaThreads / 32) * kMlaVRowsPerWarp;
    const dim3 grid((unsigned)n_heads, (unsigned)((d_v + rows_per_block - 1) / rows_per_block),
                    (unsigned)((T + kMlaTok - 1) / kMlaTok));
    if (grid.y > 65535) return GQ4_ERR_SHAPE;
    const size_t smem = (size_t)kMlaTok * R * 4;
    cudaStream_t s = S(stream);
    if (ldt == GQ4_F32)
        gq4_mla_v_kernel<0><<<grid, kMlaThreads, smem, s>>>((const uint32_t *)W->w, W->s, R, W->ng, W->gs,
                                                            n_heads, d_nope, d_v, lat, T, o);
    else
        gq4_mla_v_kernel<1><<<grid, kMlaThreads, smem, s>>>((const uint32_t *)W->w, W->s, R, W->ng, W->gs,
                                                            n_heads, d_nope, d_v, lat, T, o);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Self-test of the bounded device wait
// ---------------------------------------------------------------------------------------
extern "C" gq4_status gq4_selftest_wait_timeout(uint32_t limit_us, int32_t *status, gq4_stream_t stream) {
    if (!status) return GQ4_ERR_NULL;
    if (!aligned16(status)) return GQ4_ERR_ALIGN;
    if (limit_us < 1 || limit_us > 1000000) return GQ4_ERR_SHAPE;
    gq4_wait_selftest_kernel<<<1, 32, 0, S(stream)>>>(status, (uint64_t)limit_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Reading a device status word
// ---------------------------------------------------------------------------------------
extern "C" gq4_status gq4_sync_status(const int32_t *status_dev, gq4_stream_t stream, int32_t *status_host) {
    if (!status_dev || !status_host) return GQ4_ERR_NULL;
    if (!aligned16(status_dev)) return GQ4_ERR_ALIGN;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, status_dev, 4, cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess) return GQ4_ERR_CUDA;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return GQ4_ERR_CUDA;
    *status_host = v;
    return GQ4_OK;
}

// ---------------------------------------------------------------------------------------
// Checked build: bounds status word and its self-test
// ---------------------------------------------------------------------------------------
extern "C" int32_t gq4_build_checked(void) { return kChecked ? 1 : 0; }

extern "C" gq4_status gq4_bounds_status(int32_t clear, gq4_stream_t stream, int32_t *status_host) {
    if (!status_host) return GQ4_ERR_NULL;
    int32_t v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_bounds_status, 4, 0, cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
        return GQ4_ERR_CUDA;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return GQ4_ERR_CUDA;
    if (clear) {
        const int32_t zero = 0;
        if (cudaMemcpyToSymbolAsync(g_bounds_status, &zero, 4, 0, cudaMemcpyHostToDevice, S(stream)) != cudaSuccess ||
            cudaStreamSynchronize(S(stream)) != cudaSuccess)
            return GQ4_ERR_CUDA;
    }
    *status_host = v;
    return GQ4_OK;
}

extern "C" gq4_status gq4_selftest_bounds(int64_t index, int64_t extent, gq4_stream_t stream) {
    if (extent < 0) return GQ4_ERR_SHAPE;
    gq4_bounds_selftest_kernel<<<1, 32, 0, S(stream)>>>(index, extent);
    return cudaGetLastError() == cudaSuccess ? GQ4_OK : GQ4_ERR_CUDA;
}
