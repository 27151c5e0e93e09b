/*
 * gq4.h -- C ABI of libgq4: grouped-int4 (fmt=4, gs=64) weight-only products for the
 * routed experts of a mixture-of-experts FFN, on one NVIDIA B200 (sm_100a).
 *
 * Format (colibri PR #298 "cuda+engine: full fmt=4 (grouped int4 gs=64) support",
 * sections "Changes" and "CUDA fmt=4 support ... implementation complete but blocked"):
 *   - a matrix of `out` rows and `in` columns stores signed 4-bit weights q in -8..7,
 *     two per byte, row-major, ceil(in/2) bytes per row; the even column sits in the low
 *     nibble; nibbles are two's complement on the device (offset-binary host data is
 *     converted by XOR 0x88 per byte at upload);
 *   - one f32 scale per `gs` consecutive inputs of each row: scales[o*ng + k/gs] with
 *     ng = ceil(in/gs), so w[o][k] = scales[o*ng + k/gs] * q[o][k].
 * Device layout: rows and scales as above; inside every 32-bit word (the 8 weights
 * k = 8i..8i+7 of a row) the nibbles are reordered to k0,k2,k4,k6 in bits 0-15 and
 * k1,k3,k5,k7 in bits 16-31 (each group ascending from the low bits).  gq4_upload
 * writes this order; gq4_tensor_init expects data already in it.
 *
 * Conventions shared by every call:
 *   - The caller owns all memory.  Device buffers are passed as raw device pointers and
 *     host buffers as raw host pointers; nothing here allocates or frees device memory.
 *   - Compute calls are asynchronous on the given stream (NULL = the legacy default
 *     stream) and return after the launches are queued.
 *   - Arguments are validated on the host before anything is launched; a call that
 *     returns an error has launched nothing and written no output.
 *   - Device pointers must be 16-byte aligned.  Inputs and outputs must not overlap
 *     (pxq_llama.cpp release notes 2026-09-02, "Host-overhead cuts": the router aliasing
 *     barrier; "Correctness fixes": a fused path that did not check 16-byte base
 *     alignment faulted instead of declining -- here the call declines).
 *   - The fast kernels take gs = 64 and in % 64 == 0; the matvec, gate+up, row and
 *     quantisation calls also take any gs that is a multiple of 8 with in % 8 == 0
 *     (partial last groups included) on generic kernels; moe_expert_ffn needs gs = 64.
 *     Other shapes return GQ4_ERR_UNSUPPORTED (the host packer accepts any shape).
 *   - No call reads environment variables or throws.  No call keeps global mutable
 *     state, with two exceptions: moe_expert_ffn_noalloc uses a library-owned device
 *     array per GPU and caches that array's device address per device (see its entry),
 *     and the checked build keeps one bounds status word (gq4_bounds_status).
 */
#ifndef GQ4_H
#define GQ4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GQ4_ABI_VERSION 7u

typedef struct CUstream_st *gq4_stream_t; /* binary-compatible with cudaStream_t */
typedef struct CUevent_st *gq4_event_t;   /* binary-compatible with cudaEvent_t */

typedef enum {
    GQ4_OK = 0,
    GQ4_ERR_NULL = 1,        /* a required pointer is NULL */
    GQ4_ERR_ALIGN = 2,       /* a device pointer or stride is not 16-byte aligned */
    GQ4_ERR_SHAPE = 3,       /* inconsistent or out-of-range sizes */
    GQ4_ERR_UNSUPPORTED = 4, /* valid format the GPU kernels do not take (gs != 64 ...) */
    GQ4_ERR_ALIAS = 5,       /* an output overlaps an input */
    GQ4_ERR_WORKSPACE = 6,   /* workspace too small */
    GQ4_ERR_CUDA = 7,        /* a CUDA runtime call failed */
    GQ4_ERR_TIMEOUT = 8,     /* a bounded device wait gave up (see gq4_selftest_wait_timeout) */
    GQ4_ERR_NONFINITE_LOGIT = 9, /* a router row held NaN/+inf, or no finite maximum */
    GQ4_ERR_BOUNDS = 16      /* an index fell outside its array (checked build only) */
} gq4_status;

typedef enum { GQ4_F32 = 0, GQ4_BF16 = 1 } gq4_dtype;

/* Non-owning descriptor of one grouped-int4 matrix, or of n_experts matrices of the
 * same shape stacked in memory (expert e at w + e*expert_stride_w bytes and
 * s + e*expert_stride_s floats).  `w` and `s` are device pointers. */
typedef struct {
    int64_t out;             /* rows O */
    int64_t in;              /* columns I (the contraction length) */
    int32_t gs;              /* group size (64) */
    int32_t ng;              /* ceil(in/gs) */
    int32_t n_experts;       /* 1 for a plain matrix */
    int32_t reserved;
    const uint8_t *w;        /* packed nibbles [n_experts][out][ceil(in/2)] */
    const float *s;          /* scales [n_experts][out][ng] */
    int64_t expert_stride_w; /* bytes between experts (>= out*ceil(in/2), multiple of 16) */
    int64_t expert_stride_s; /* floats between experts (>= out*ng, multiple of 4) */
} gq4_tensor;

/* Device views into a moe_expert_ffn workspace (see moe_expert_ffn_routing). */
typedef struct {
    int32_t *idx;      /* [T][K] expert of slot (t,j), logit-descending */
    float *wts;        /* [T][K] routing weight of slot (t,j) */
    int32_t *cnt;      /* [E] rows per expert */
    int32_t *offs;     /* [E+1] first row of each expert; offs[E] = T*K */
    int32_t *row_tok;  /* [T*K] token of row r */
    int32_t *row_slot; /* [T*K] flat slot t*K+j of row r */
    int32_t *slot_row; /* [T*K] row of flat slot f */
    int32_t *n_active; /* [1] number of experts with cnt > 0 */
    int32_t *active;   /* [E] those experts, ascending */
    int32_t *status;   /* [1] device status word (gq4_status bits, see moe_expert_ffn) */
    uint16_t *h;       /* [T*K][F] bf16 gate+up output silu(g)*u, row r = row-map row r */
} gq4_routing;

/* ABI version of the loaded library (GQ4_ABI_VERSION at build time).  The Python
 * binding refuses a library whose version differs (colibri PR #298, "fmt=4 CUDA
 * attention crash": a DLL and an engine built from different branches resolved the
 * same symbol with different signatures). */
uint32_t gq4_abi_version(void);

/* Static, NUL-terminated description of a status code. */
const char *gq4_status_string(int status);

/* ---------------------------------------------------------------- host packing
 * gq4_pack: q[out][in] (int8, each in -8..7 unless src_offset_binary, then 0..15
 * offset-binary nibbles u = q+8) -> packed_host[out][ceil(in/2)], even column in the
 * low nibble, two's complement, the pad nibble of an odd `in` written as 0.
 * Host pointers; gs only checked (> 0).  GQ4_ERR_SHAPE on a value out of range
 * (nothing is guaranteed written then). */
gq4_status gq4_pack(const int8_t *q, int64_t out, int64_t in, int32_t gs,
                    int32_t src_offset_binary, uint8_t *packed_host);

/* Bytes a device copy needs: w_bytes = n_experts*out*ceil(in/2), s_bytes =
 * n_experts*out*ceil(in/gs)*4 (colibri PR #298: qt_bytes counts O*ng*4 scale bytes). */
gq4_status gq4_device_bytes(int64_t out, int64_t in, int32_t gs, int32_t n_experts,
                            size_t *w_bytes, size_t *s_bytes);

/* Copy packed weights and scales of n_experts matrices from host memory into
 * caller-owned device buffers, reorder the nibbles of each 32-bit word into the device
 * layout (on the device), and fill *desc (expert strides = the tight sizes).  With
 * src_offset_binary = 1 each byte is XORed with 0x88 first (offset_to_signed_s4).
 * `in` must be a multiple of 8 (GQ4_ERR_UNSUPPORTED otherwise).  Asynchronous on `stream`; the host buffers must stay valid
 * until the stream reaches this point.  Device buffers must be at least the sizes from
 * gq4_device_bytes and 16-byte aligned. */
gq4_status gq4_upload(const uint8_t *packed_host, const float *scales_host, int64_t out,
                      int64_t in, int32_t gs, int32_t n_experts, int32_t src_offset_binary,
                      void *d_w, size_t d_w_bytes, float *d_s, size_t d_s_bytes,
                      gq4_stream_t stream, gq4_tensor *desc);

/* Fill *desc for device data already laid out as above (no copy).  The descriptor
 * carries gs and ng with the pointers so that every launch site indexes the O*ng scale
 * array by group (colibri PR #298, "fmt=4 CUDA attention crash -- root cause": the fix
 * threaded w->gs and w->ng, which the uploaded tensor already carried, through every
 * launch; "Summary / Changes": tensor_upload allocates O*ng scales for fmt=4).  Expert
 * strides are set to the tight sizes; a caller with padded experts edits them after. */
gq4_status gq4_tensor_init(const void *d_w, const float *d_s, int64_t out, int64_t in,
                           int32_t gs, int32_t n_experts, gq4_tensor *desc);

/* ---------------------------------------------------------------- compute
 * gq4_matvec: y[t][o] = sum_k w[o][k] * x[t][k] for t < n_tok, fp32 accumulation
 * (colibri PR #298, "Changes": quant_matmul with per-group scales; the maintainer's
 * reply: matmul_i4_grouped against a double reference).
 *   W: one matrix (n_experts == 1); x: device [n_tok][W->in] of xdt; y: device f32
 *   [n_tok][W->out].  f32 x is taken exactly (split into three bf16 terms).
 *   Any n_tok >= 1; the kernel is built for few tokens (decode). */
gq4_status gq4_matvec(const gq4_tensor *W, const void *x, gq4_dtype xdt, int64_t n_tok,
                      float *y, gq4_stream_t stream);

/* gq4_gate_up_silu: g = Wg x, u = Wu x in one pass over x (x read once), then
 * h = silu(g) * u = g * sigmoid(g) * u, rounded to xdt (bf16 round-to-nearest-even, or
 * f32).  colibri PR #298, "Changes": matmul_i4_grouped_pair, "fused gate+up for fmt=4
 * -- reads x once instead of twice".
 *   Wg, Wu: one matrix each, same shape [F][H]; x device [n_tok][H] xdt; h device
 *   [n_tok][F] xdt. */
gq4_status gq4_gate_up_silu(const gq4_tensor *Wg, const gq4_tensor *Wu, const void *x,
                            gq4_dtype xdt, int64_t n_tok, void *h, gq4_stream_t stream);

/* gq4_route: router top-K and weights, per token (colibri PR #298, "implementation
 * complete but blocked": K passes over a taken-flag array; ties go to the lower expert
 * index).  wts = softmax over all E renormalised over the K chosen.
 *   logits device f32 [T][E]; idx device int32 [T][K]; wts device f32 [T][K];
 *   status device int32 [1]: GQ4_ERR_NONFINITE_LOGIT is OR-ed in when a row holds NaN or
 *   +inf or has no finite maximum (that row gets experts 0..K-1 and NaN weights).
 *   1 <= K <= E <= 1024. */
gq4_status gq4_route(const float *logits, int64_t T, int32_t E, int32_t K, int32_t *idx,
                     float *wts, int32_t *status, gq4_stream_t stream);

/* gq4_rowmap: on-device token -> expert table (pxq_llama.cpp release notes 2026-09-02,
 * "Device-side MoE row map": histogram, scan and fill with no host round trip).
 * Rows of an expert are ordered by ascending flat slot f = t*K + j.  Writes cnt [E],
 * offs [E+1], row_tok / row_slot / slot_row [T*K], n_active [1], active [E] (device).
 * `scratch` is device memory of gq4_rowmap_scratch_bytes(T, K, E) bytes; its first
 * int32 is the call's status word: GQ4_ERR_SHAPE is OR-ed in when an idx entry lies
 * outside [0, E), and the tables are then not valid (read it with gq4_sync_status). */
size_t gq4_rowmap_scratch_bytes(int64_t T, int32_t K, int32_t E);
gq4_status gq4_rowmap(const int32_t *idx, int64_t T, int32_t K, int32_t E, int32_t *cnt,
                      int32_t *offs, int32_t *row_tok, int32_t *row_slot, int32_t *slot_row,
                      int32_t *n_active, int32_t *active, void *scratch, size_t scratch_bytes,
                      gq4_stream_t stream);

/* moe_expert_ffn: one routed-expert FFN layer.
 *   y[t] = sum_j wts[t][j] * Wd_e (silu(Wg_e x_t) * (Wu_e x_t)),  e = idx[t][j]
 * with the router, the on-device row map, the fused gate+up (h rounded to bf16), the
 * down projection and the weighted scatter-add all on the GPU, no host round trip.
 * Sources: colibri PR #298, "Summary / Changes" (the fmt=4 expert matmuls and the fused
 * grouped gate+up pair, matmul_i4_grouped_pair, which halved expert-matmul time) and
 * "implementation complete but blocked" (top-K by K passes over taken flags, the grouped
 * down projection); pxq_llama.cpp release notes 2026-09-02, "Device-side MoE row map"
 * (the token -> expert table built on the device with histogram, scan and fill, because
 * a host-built table forced a device-to-host sync per layer).  The top-K softmax
 * renormalised over the chosen experts, SiLU(gate)*up and the weighted sum of the K
 * expert outputs complete the layer as the method statement gives it.
 *   Wg, Wu: E stacked [F][H]; Wd: E stacked [H][F]; logits device f32 [T][E];
 *   x device bf16 [T][H]; y device f32 [T][H] (overwritten); ws device workspace of
 *   moe_expert_ffn_workspace_bytes(T, E, K, H, F) bytes; 1 <= K <= E <= 1024.
 * Experts are split by their row count: with T >= GQ4_MOE_LARGE_MIN_ROWS, H % 128 == 0,
 * F % 64 == 0 and expert strides that are whole rows, an expert with at least
 * GQ4_MOE_LARGE_MIN_ROWS rows runs on the tensor-core kernels, the others (and every
 * expert otherwise) on the decode kernels.  The split changes speed, not results
 * beyond rounding.
 * Data-dependent errors (non-finite logits) are reported through the workspace status
 * word: read it with moe_expert_ffn_status.  The order in which the K slot
 * contributions are added into y is not fixed (float atomics); results agree within
 * rounding.
 *   stage_events: NULL, or GQ4_MOE_STAGE_EVENTS (6) CUDA events (created by the caller)
 *   recorded on `stream` at: [0] the start, [1] after the router and row map, [2] after
 *   gate+up of the experts with few rows (decode kernels), [3] after gate+up of the
 *   experts with many rows (row gather + tensor-core kernel), [4] after down of the
 *   experts with few rows, [5] after down of the experts with many rows.  Where a stage
 *   launches nothing its two events are recorded back to back.  A caller times the
 *   stages with cudaEventElapsedTime.  Inside a stream capture the events are recorded
 *   as external events, so a call captured in a CUDA graph records them at every replay.
 *   An event that cannot be recorded makes the call return GQ4_ERR_CUDA after its
 *   launches. */
#define GQ4_MOE_STAGE_EVENTS 6
#define GQ4_MOE_LARGE_MIN_ROWS 33
size_t moe_expert_ffn_workspace_bytes(int64_t T, int32_t E, int32_t K, int64_t H, int64_t F);
gq4_status moe_expert_ffn(const gq4_tensor *Wg, const gq4_tensor *Wu, const gq4_tensor *Wd,
                          const float *logits, const void *x, gq4_dtype xdt, int64_t T,
                          int32_t E, int32_t K, float *y, void *ws, size_t ws_bytes,
                          gq4_event_t const *stage_events, gq4_stream_t stream);

/* Device pointers of the routing tables and of h (the bf16 gate+up output, in row-map
 * order) inside a workspace used by moe_expert_ffn with the same (T, E, K, H, F).  h is
 * computed in a fixed order on every path, so repeated calls on the same inputs give
 * the same h bit for bit (y is not: its K contributions meet through float atomics). */
gq4_status moe_expert_ffn_routing(void *ws, size_t ws_bytes, int64_t T, int32_t E, int32_t K,
                                  int64_t H, int64_t F, gq4_routing *out);

/* Synchronise `stream` and read the workspace status word into *status (GQ4_OK when no
 * data error was seen).  Returns GQ4_ERR_CUDA when the synchronisation fails. */
gq4_status moe_expert_ffn_status(const void *ws, size_t ws_bytes, int64_t T, int32_t E,
                                 int32_t K, int64_t H, int64_t F, gq4_stream_t stream,
                                 int32_t *status);

/* ---------------------------------------------------------------- general group sizes,
 * quantisation and row operations (any gs that is a multiple of 8; in % 8 == 0)
 *
 * gq4_matvec and gq4_gate_up_silu above take these shapes too: a tensor with gs != 64
 * or a partial last group runs on a generic CUDA-core kernel (one warp per row, the
 * scale applied once per group), colibri PR #298 "What was implemented (CPU)":
 * matmul_i4_grouped "handles arbitrary gs (multiple of 16)".  Only moe_expert_ffn still
 * requires gs = 64 and in % 64 == 0.
 *
 * gq4_detect_group_size: host only.  The group size of a matrix from the byte count of
 * its scale array (PR #298, same section: detect_group_size() tries
 * {16,32,48,64,96,128,192,256}): *gs_out = the one candidate with
 * out*ceil(in/gs)*4 == scale_bytes.  GQ4_ERR_SHAPE when none matches,
 * GQ4_ERR_UNSUPPORTED when two or more match (their groups differ; the size alone
 * cannot decide). */
gq4_status gq4_detect_group_size(int64_t out, int64_t in, size_t scale_bytes, int32_t *gs_out);

/* gq4_quantize: float weights -> grouped int4 in the device layout, on the GPU (the
 * converter step, PR #298 maintainer's "data request": convert_fp8_to_int4.py
 * --group-size 64).  Per group of gs consecutive inputs of a row (the last group of a
 * row may be partial; gs >= in gives one scale per row, the fmt=2 case):
 *   s = max|w| / 7 (f32 division), q = round-half-to-even(w / s) in f32, clamped to
 *   [-8, 7]; an all-zero group gets s = 0 and q = 0.
 * The pages name the group size, not the rounding: this absmax rule is the reading.
 *   w: device f32 [out][in], 16-byte aligned, finite; d_w: device, >= out*in/2 bytes;
 *   d_s: device f32 [out][ceil(in/gs)]; *desc filled as gq4_tensor_init does.
 *   gs % 8 == 0 and in % 8 == 0 (GQ4_ERR_UNSUPPORTED otherwise). */
gq4_status gq4_quantize(const float *w, int64_t out, int64_t in, int32_t gs, void *d_w,
                        size_t d_w_bytes, float *d_s, size_t d_s_bytes, gq4_stream_t stream,
                        gq4_tensor *desc);

/* gq4_dequant_rows: row dequantisation / gather (PR #298: embed_row, qt_addrow and
 * qt_matvec_rows needed the fmt=4 per-group-scale branch).
 *   out[j][k] = (accumulate ? out[j][k] : 0) + alpha[j] * w[idx[j]][k], k < in,
 * alpha = NULL meaning 1.  embed_row is accumulate = 0, qt_addrow accumulate = 1.
 *   idx: device int32 [n]; alpha: NULL or device f32 [n]; out: device [n][in] of odt
 *   (GQ4_F32, or GQ4_BF16 rounded to nearest even, which takes no accumulate).
 *   An index outside [0, W->out) is not read: that row of out becomes NaN. */
gq4_status gq4_dequant_rows(const gq4_tensor *W, const int32_t *idx, int64_t n,
                            const float *alpha, int32_t accumulate, void *out, gq4_dtype odt,
                            gq4_stream_t stream);

/* gq4_matvec_rows: matvec over selected rows (qt_matvec_rows):
 *   y[t][j] = sum_k w[idx[j]][k] * x[t][k], fp32 accumulation.
 *   idx: device int32 [n_sel]; x: device [n_tok][W->in] of xdt; y: device f32
 *   [n_tok][n_sel].  An index outside [0, W->out) gives NaN in its column of y. */
gq4_status gq4_matvec_rows(const gq4_tensor *W, const int32_t *idx, int64_t n_sel,
                           const void *x, gq4_dtype xdt, int64_t n_tok, float *y,
                           gq4_stream_t stream);

/* ---- grouped-scale MLA absorb projections over the kv_b tensor
 * colibri PR #298, "fmt=4 CUDA attention crash — root cause": the Q- and V-projection
 * loops of the MLA attention absorb kernels multiply kv_b weights by their scale, and
 * with fmt=4 the scale of weight (row, k) is scales[row*ng + k/gs], looked up inside the
 * accumulation loop (one scale per row, the fmt=2 rule, reads the wrong entries of the
 * O*ng scale array).  These calls run the two projections on their own.
 *   W: the kv_b tensor, out = n_heads * (d_nope + d_v) rows in per-head blocks (d_nope
 *      key rows, then d_v value rows), in = R latent channels; any gs % 8 == 0 with
 *      R % 8 == 0, R <= 2048, d_nope <= 1024 (GQ4_ERR_UNSUPPORTED beyond); the first
 *      expert of a stacked tensor is used.  With D = d_nope + d_v:
 * gq4_mla_absorb_q: q_lat[t][h][c] = sum_{d < d_nope} q_nope[t][h][d] * w(h*D + d, c)
 *      q_nope: device [T][n_heads][d_nope] of qdt (GQ4_F32 or GQ4_BF16);
 *      q_lat: device f32 [T][n_heads][R].
 * gq4_mla_absorb_v: o[t][h][v] = sum_{c < R} lat[t][h][c] * w(h*D + d_nope + v, c)
 *      lat: device [T][n_heads][R] of ldt; o: device f32 [T][n_heads][d_v].
 * fp32 accumulation.  T <= 262140.  Outputs must not overlap the inputs or W.  The Q
 * projection may split a head's key rows over several blocks whose sums meet through
 * float atomics, so its last bits can differ from call to call. */
gq4_status gq4_mla_absorb_q(const gq4_tensor *W, int32_t n_heads, int32_t d_nope, int32_t d_v,
                            const void *q_nope, gq4_dtype qdt, int64_t T, float *q_lat,
                            gq4_stream_t stream);
gq4_status gq4_mla_absorb_v(const gq4_tensor *W, int32_t n_heads, int32_t d_nope, int32_t d_v,
                            const void *lat, gq4_dtype ldt, int64_t T, float *o,
                            gq4_stream_t stream);

/* gq4_sync_status: waits for `stream` and reads a device status word written by the
 * library's kernels -- the status output of gq4_route / gq4_rowmap, the status word of
 * gq4_selftest_wait_timeout or of moe_expert_ffn_noalloc -- into *status_host (0, or the
 * OR of GQ4_ERR_NONFINITE_LOGIT, GQ4_ERR_TIMEOUT, ... the kernels raised).  Synchronous:
 * it returns after all work queued on `stream` before it has finished.
 * Data-dependent errors stay on the device so that no compute call has to synchronise
 * (pxq_llama.cpp release notes 2026-09-02, "Device-side MoE row map": a device-to-host
 * sync inside the per-layer loop was the cost the on-device table removed); the caller
 * reads the word with this call when it chooses.  An out-of-range index becomes a status
 * bit rather than a fault (colibri PR #298, "fmt=4 CUDA attention crash -- root cause":
 * a wrong scale index became a GPU memory fault and a system crash).
 *   status_dev: 16-byte aligned device int32; status_host: host int32.
 *   Returns GQ4_ERR_CUDA when the copy or the synchronisation fails (for example after an
 *   earlier launch failed on the stream). */
gq4_status gq4_sync_status(const int32_t *status_dev, gq4_stream_t stream, int32_t *status_host);

/* ---- self-test of the bounded device wait
 * Every wait of the library's kernels (on an mbarrier that a TMA copy, a tensor-core
 * commit or another warp completes) gives up after a time limit (2 s in the kernels),
 * raises GQ4_ERR_TIMEOUT in the call's status word and lets the kernel end, so a stuck
 * producer never hangs the GPU.  This call runs that wait on a barrier nothing arrives
 * on, with a limit of limit_us microseconds (1 .. 1,000,000), so that the path can be
 * tested without a fault.
 *   status: 16-byte aligned device int32, OR-ed with GQ4_ERR_TIMEOUT when the wait
 *   gives up (the caller clears it first).  Asynchronous on `stream`. */
gq4_status gq4_selftest_wait_timeout(uint32_t limit_us, int32_t *status, gq4_stream_t stream);

/* moe_expert_ffn_noalloc: the same layer as moe_expert_ffn, for callers that cannot
 * allocate device memory -- a plug-in whose host program owns every device allocation
 * and hands it only the tensors, or a decode loop that must not call cudaMalloc because
 * cudaMalloc can synchronise the device.  It has no counterpart on the source pages: it
 * exists only so that such callers need no workspace.
 *   Instead of a caller workspace it uses one library-owned device array of
 *   GQ4_NOALLOC_SCRATCH_BYTES (16 MiB), which every GPU that loads this library holds
 *   until the process exits.  A shape whose workspace
 *   (moe_expert_ffn_workspace_bytes(T, E, K, H, F)) exceeds that returns
 *   GQ4_ERR_WORKSPACE before anything is launched; 16 MiB covers decode batches up to
 *   about 120 tokens at H = 6144, F = 2048, K = 8, E = 256.
 *   Arguments as for moe_expert_ffn (no stage events); status_out is NULL or a 16-byte
 *   aligned device int32 that receives the data-error status word of this call
 *   (GQ4_ERR_NONFINITE_LOGIT ...), copied on `stream` after the layer.
 *   The first call on a device looks up that device's address of the array (with the
 *   device current); make that first call before any stream capture.  The call itself
 *   calls no cudaMalloc, cudaFree or other allocating routine.
 *   Every call, on every stream, shares the one array per device and it keeps the last
 *   call's contents; the call clears what must start at zero (the status word).  Calls
 *   that overlap on the GPU -- on two streams, or from two host threads -- race on the
 *   array and corrupt each other's results: serialise them. */
#define GQ4_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
gq4_status moe_expert_ffn_noalloc(const gq4_tensor *Wg, const gq4_tensor *Wu,
                                  const gq4_tensor *Wd, const float *logits, const void *x,
                                  gq4_dtype xdt, int64_t T, int32_t E, int32_t K, float *y,
                                  int32_t *status_out, gq4_stream_t stream);

/* ---- checked build
 * The bug class the source pages report is an index outside its array: the MLA absorb
 * kernels read the O*ng scale array of a grouped tensor with a bare row index (colibri
 * PR #298, "fmt=4 CUDA attention crash -- root cause"), and a shard's scale pointer was
 * offset by rows instead of rows*ng (the maintainer's oracle reply).  A library built with
 * GQ4_CHECKED defined (libgq4_checked.so) tests every weight, scale and activation-row
 * index its kernels compute against the extent of its array -- taken from the tensor
 * descriptors and the call's sizes -- before the access.  An index outside is not used:
 * the access reads zeros (a copy that must deliver its bytes reads row 0 instead), the
 * results are then not valid, and GQ4_ERR_BOUNDS is OR-ed into one library-wide bounds
 * status word.  Nothing traps.  Outputs written through a valid index are unchanged.
 * gq4_build_checked: 1 for a checked library, 0 otherwise.
 * gq4_bounds_status: waits for `stream`, reads the bounds status word into *status_host
 *   (0 or GQ4_ERR_BOUNDS; always 0 in an unchecked library) and clears it when `clear` is
 *   non-zero.  The word is shared by every call on every stream of the process.
 * gq4_selftest_bounds: launches, on `stream`, a test of `index` against `extent` that
 *   accesses no memory, so that the reporting path can be tested without an out-of-range
 *   access; in a checked library index outside [0, extent) raises GQ4_ERR_BOUNDS.
 *   GQ4_ERR_SHAPE for a negative extent. */
int32_t gq4_build_checked(void);
gq4_status gq4_bounds_status(int32_t clear, gq4_stream_t stream, int32_t *status_host);
gq4_status gq4_selftest_bounds(int64_t index, int64_t extent, gq4_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* GQ4_H */
