/*
 * gq4_oracle.c -- the CPU oracle for the grouped-int4 (fmt=4, gs=64) expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or calls
 * this file; only the tests, the package's smoke entry and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with the CUDA
 * path.
 *
 * Plain C99, fp64 arithmetic, no SIMD intrinsics, no blocking, no fusion: every
 * function is the written-out definition, in the order the sources state it, so a
 * reader can check it by eye.  OpenMP (when enabled at compile time) only spreads
 * independent outputs over threads; the arithmetic of each output element is the same
 * sequential loop either way.
 *
 * Sources (web pages, cited by title and section):
 *   [PR298]  colibri pull request #298, "cuda+engine: full fmt=4 (grouped int4 gs=64)
 *            support + diagnostic harness", and its review thread.
 *   [PXQ]    pxq_llama.cpp release notes 2026-09-02.
 * Where the pages are silent the reading is stated at the function.
 *
 * Pins (tests/test_oracle.py, tests/test_oracle_next.py): every function here is checked
 * against hand-worked nibble and rounding tables, closed forms, the fmt=2 identity,
 * exact integer arithmetic, brute-force sorting, an independent numpy decode and the
 * worked size examples of the kv_b tensor and the expert; none of its results is
 * compared with itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_SHAPE 3
#define ORC_ERR_NONFINITE_LOGIT 9

/* ---------------------------------------------------------------------------------
 * a1. Nibble decode.
 * [PR298] "Summary / Changes": fmt=4 uses the same packed int4 layout as fmt=2, i.e.
 * (I+1)/2 bytes per row, two weights per byte.  Reading: the even k sits in the low
 * nibble of byte k/2, the odd k in the high nibble.  The signed value is the 4-bit two's
 * complement of the nibble (the pages' host files hold offset-binary nibbles u = q+8 and
 * turn them into two's complement by XOR 0x88 per byte at upload, section "CUDA fmt=4
 * support ... implementation complete but blocked", "offset_to_signed_s4").
 * ------------------------------------------------------------------------------- */
int orc_nibble_to_q(int nibble, int offset_binary)
{
    nibble &= 15;
    if (offset_binary) return nibble - 8;
    return nibble >= 8 ? nibble - 16 : nibble;
}

int orc_unpack(const uint8_t *packed, int64_t row_bytes, int64_t o, int64_t k,
               int offset_binary)
{
    uint8_t b = packed[o * row_bytes + (k >> 1)];
    int nib = (k & 1) ? (b >> 4) : (b & 15);
    return orc_nibble_to_q(nib, offset_binary);
}

/* The oracle's own packer: q[o][k] in -8..7 -> packed rows of (I+1)/2 bytes, even k in
 * the low nibble, the pad nibble of an odd I written as 0.  offset_binary=1 writes
 * u = q+8 instead of two's complement. */
void orc_pack(const int8_t *q, int64_t O, int64_t I, int offset_binary, uint8_t *out)
{
    int64_t rb = (I + 1) / 2;
    memset(out, 0, (size_t)(O * rb));
    for (int64_t o = 0; o < O; o++)
        for (int64_t k = 0; k < I; k++) {
            int v = q[o * I + k];
            int nib = offset_binary ? (v + 8) : (v & 15);
            if (k & 1) out[o * rb + k / 2] |= (uint8_t)(nib << 4);
            else       out[o * rb + k / 2] |= (uint8_t)nib;
        }
}

/* ---------------------------------------------------------------------------------
 * Sizes.  [PR298] "implementation complete but blocked": qt_bytes counts O*ng*4 scale
 * bytes; "Summary": tensors allocate O*ng scales with ng = ceil(I/gs).
 * ------------------------------------------------------------------------------- */
int64_t orc_ngroups(int64_t I, int64_t gs) { return (I + gs - 1) / gs; }
int64_t orc_weight_bytes(int64_t O, int64_t I) { return O * ((I + 1) / 2); }
int64_t orc_scale_bytes(int64_t O, int64_t I, int64_t gs) { return O * orc_ngroups(I, gs) * 4; }

/* ---------------------------------------------------------------------------------
 * a1 (scale). w(o,k) = scale[o*ng + k/gs] * q(o,k).
 * [PR298] "CUDA fmt=4 support": scale_at() looks up scales[o*ng + i/gs]; the attention
 * crash write-up restates it as wscale[row*ng + k/gs].  The last group may be partial
 * (the maintainer's oracle covers "partial last group" and "gs > I").
 * ------------------------------------------------------------------------------- */
double orc_weight(const uint8_t *packed, const float *scales, int64_t O, int64_t I,
                  int64_t gs, int64_t o, int64_t k)
{
    (void)O;
    int64_t ng = orc_ngroups(I, gs);
    int q = orc_unpack(packed, (I + 1) / 2, o, k, 0);
    return (double)scales[o * ng + k / gs] * (double)q;
}

/* Activation element at its stored value: dtype 0 = f32, 1 = bf16 (widened exactly). */
static double orc_x(const void *x, int xdt, int64_t idx)
{
    if (xdt == 1) {
        uint16_t h = ((const uint16_t *)x)[idx];
        uint32_t bits = (uint32_t)h << 16;
        float f;
        memcpy(&f, &bits, 4);
        return (double)f;
    }
    return (double)((const float *)x)[idx];
}

/* ---------------------------------------------------------------------------------
 * a2. matvec: y[t][o] = sum_k w(o,k) * x[t][k], natural k order, fp64.
 * [PR298] "implementation complete but blocked": matmul_i4_grouped accumulates per
 * group and applies the group's scale; mathematically the same sum.  The maintainer's
 * oracle reply: a plain dequant reference in double.
 * y is returned in fp64; the caller compares it with the GPU's f32.
 * bound[t][o] = sum_k |w(o,k)| * max_k |x[t][k]|  (the Sigma|terms| scale of the
 * acceptance test: "compare against the sum of |terms|", maintainer's oracle reply).
 * ------------------------------------------------------------------------------- */
void orc_matvec(const uint8_t *packed, const float *scales, int64_t O, int64_t I,
                int64_t gs, const void *x, int xdt, int64_t T, double *y, double *bound)
{
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < O; o++) {
        double l1 = 0.0;
        for (int64_t k = 0; k < I; k++) l1 += fabs(orc_weight(packed, scales, O, I, gs, o, k));
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0, xmax = 0.0;
            for (int64_t k = 0; k < I; k++) {
                double xv = orc_x(x, xdt, t * I + k);
                acc += orc_weight(packed, scales, O, I, gs, o, k) * xv;
                if (fabs(xv) > xmax) xmax = fabs(xv);
            }
            y[t * O + o] = acc;
            if (bound) bound[t * O + o] = l1 * xmax;
        }
    }
}

/* L1 norm of each dequantised row: ||w_row||_1. */
void orc_row_l1(const uint8_t *packed, const float *scales, int64_t O, int64_t I,
                int64_t gs, double *l1)
{
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < O; o++) {
        double s = 0.0;
        for (int64_t k = 0; k < I; k++) s += fabs(orc_weight(packed, scales, O, I, gs, o, k));
        l1[o] = s;
    }
}

/* ---------------------------------------------------------------------------------
 * Rounding of a double to the activation dtype (round to nearest, ties to even).
 * bf16 = the upper 16 bits of an IEEE binary32 with an 8-bit significand.  Rounding
 * is done from the fp64 value directly (one rounding), by scaling to the bf16 ulp.
 * ------------------------------------------------------------------------------- */
double orc_round_bf16(double v)
{
    if (v == 0.0 || isnan(v) || isinf(v)) return v;
    int e;
    frexp(v, &e);                /* |v| = m * 2^e, m in [0.5, 1) */
    if (e < -125) e = -125;      /* below the binary32 normal range: fixed ulp 2^-133 */
    double ulp = ldexp(1.0, e - 8); /* 8 significant bits */
    double r = nearbyint(v / ulp) * ulp; /* default rounding mode is to nearest even */
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, v); /* past max bf16 */
    return r;
}

double orc_round_f32(double v) { return (double)(float)v; }

/* ---------------------------------------------------------------------------------
 * a3. Fused gate+up with SiLU: g = Wg x, u = Wu x, h = g * sigmoid(g) * u.
 * [PR298] "Summary / Changes": matmul_i4_grouped_pair is the fused gate+up that
 * "reads x once"; the maintainer's reply fixes its invariant pair(g,u) == grouped(g),
 * grouped(u).  SiLU(gate)*up is the stated activation of the expert FFN.
 * h is rounded to hdt (0 = f32, 1 = bf16 RNE).
 * ------------------------------------------------------------------------------- */
void orc_gate_up_silu(const uint8_t *pg, const float *sg, const uint8_t *pu,
                      const float *su, int64_t F, int64_t H, int64_t gs, const void *x,
                      int xdt, int64_t T, int hdt, double *h, double *g_out, double *u_out)
{
    double *g = (double *)malloc(sizeof(double) * (size_t)(T * F));
    double *u = (double *)malloc(sizeof(double) * (size_t)(T * F));
    orc_matvec(pg, sg, F, H, gs, x, xdt, T, g, NULL);
    orc_matvec(pu, su, F, H, gs, x, xdt, T, u, NULL);
    for (int64_t i = 0; i < T * F; i++) {
        double gv = g[i];
        double v = gv / (1.0 + exp(-gv)) * u[i];
        h[i] = hdt == 1 ? orc_round_bf16(v) : orc_round_f32(v);
        if (g_out) g_out[i] = gv;
        if (u_out) u_out[i] = u[i];
    }
    free(g);
    free(u);
}

/* ---------------------------------------------------------------------------------
 * a4. Router.  Per token: top-K of E logits, softmax over all E, renormalised over the
 * K chosen.
 * Selection follows [PR298] "implementation complete but blocked", router top-K with a
 * taken-flag array: K passes, each takes the largest logit among experts not yet
 * taken.  Reading: the comparison is strict '>', scanned in ascending expert index, so
 * among equal logits the lower index wins.  Slot j = the j-th pick.
 * Reading on non-finite input: a NaN or +inf logit, or a row whose largest logit is
 * -inf, makes the token invalid (returned in bad[t] = 1); its picks are then experts
 * 0..K-1 and its weights NaN.
 * ------------------------------------------------------------------------------- */
int orc_route(const float *logits, int64_t T, int64_t E, int64_t K, int32_t *idx,
              double *wts, int32_t *bad)
{
    if (K < 1 || K > E) return ORC_ERR_SHAPE;
    int any_bad = 0;
    char *taken = (char *)malloc((size_t)E);
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    for (int64_t t = 0; t < T; t++) {
        const float *l = logits + t * E;
        int invalid = 0;
        double lmax = -INFINITY;
        for (int64_t e = 0; e < E; e++) {
            if (isnan(l[e]) || (isinf(l[e]) && l[e] > 0)) invalid = 1;
            if ((double)l[e] > lmax) lmax = (double)l[e];
        }
        if (!invalid && isinf(lmax)) invalid = 1;
        bad[t] = invalid;
        if (invalid) {
            any_bad = 1;
            for (int64_t j = 0; j < K; j++) {
                idx[t * K + j] = (int32_t)j;
                wts[t * K + j] = NAN;
            }
            continue;
        }
        /* selection: K passes over the not-yet-taken experts */
        memset(taken, 0, (size_t)E);
        for (int64_t j = 0; j < K; j++) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            idx[t * K + j] = (int32_t)best;
        }
        /* softmax over all E ... */
        double z = 0.0;
        for (int64_t e = 0; e < E; e++) {
            p[e] = exp((double)l[e] - lmax);
            z += p[e];
        }
        for (int64_t e = 0; e < E; e++) p[e] /= z;
        /* ... then renormalised over the K selected */
        double zs = 0.0;
        for (int64_t j = 0; j < K; j++) zs += p[idx[t * K + j]];
        for (int64_t j = 0; j < K; j++) wts[t * K + j] = p[idx[t * K + j]] / zs;
    }
    free(taken);
    free(p);
    return any_bad ? ORC_ERR_NONFINITE_LOGIT : ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * a5. Row map (token -> expert table).
 * [PXQ] "Device-side MoE row map": a histogram, a scan and a fill; the device table must
 * equal the host table bit for bit.  Reading of the order the pages leave open: rows
 * of an expert are ordered by ascending flat slot f = t*K + j.
 *   cnt[e]   = #{f : idx[f] == e}
 *   offs     = exclusive prefix sum of cnt, offs[E] = T*K
 *   row r of expert e (offs[e] <= r < offs[e+1]) holds slot row_slot[r] = f,
 *   token row_tok[r] = f / K, and slot_row[f] = r.
 * ------------------------------------------------------------------------------- */
int orc_rowmap(const int32_t *idx, int64_t T, int64_t K, int64_t E, int32_t *cnt,
               int32_t *offs, int32_t *row_tok, int32_t *row_slot, int32_t *slot_row)
{
    int64_t n = T * K;
    for (int64_t e = 0; e < E; e++) cnt[e] = 0;
    for (int64_t f = 0; f < n; f++) {
        if (idx[f] < 0 || idx[f] >= E) return ORC_ERR_SHAPE;
        cnt[idx[f]]++;
    }
    offs[0] = 0;
    for (int64_t e = 0; e < E; e++) offs[e + 1] = offs[e] + cnt[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int64_t e = 0; e < E; e++) fill[e] = offs[e];
    for (int64_t f = 0; f < n; f++) {
        int32_t r = fill[idx[f]]++;
        row_slot[r] = (int32_t)f;
        row_tok[r] = (int32_t)(f / K);
        slot_row[f] = r;
    }
    free(fill);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * a6-a8. MoE expert FFN for a set of sampled tokens.
 * For token t and each of its K slots j (expert e = idx[t][j], weight wts[t][j]):
 *   h = round_hdt( silu(Wg_e x_t) * (Wu_e x_t) )          (a3 on the gathered row)
 *   D = Wd_e h                                             (fp64)
 *   y[t] = sum_j wts[t][j] * D_j, summed in slot order     (a8)
 * Expert e's packed matrices sit at pg + e*wstride_gu etc.; the strides are in bytes
 * for packed weights and in floats for scales.  Gate/up are [F][H], down is [H][F].
 * bound[s][o] = sum_j |wts_j| * ||Wd_e[o]||_1 * max|h_j| (the Sigma|terms| scale).
 * The slot results are independent of how tokens group into experts, so the oracle
 * evaluates them token by token; the row map is checked separately.
 * ------------------------------------------------------------------------------- */
void orc_moe_tokens(const uint8_t *pg, const float *sg, const uint8_t *pu, const float *su,
                    const uint8_t *pd, const float *sd, int64_t wstride_gu,
                    int64_t sstride_gu, int64_t wstride_d, int64_t sstride_d, int64_t H,
                    int64_t F, int64_t gs, const void *x, int xdt, int hdt,
                    const int32_t *idx, const double *wts, int64_t K,
                    const int64_t *tokens, int64_t n_tokens, double *y, double *bound)
{
    for (int64_t i = 0; i < n_tokens * H; i++) { y[i] = 0.0; if (bound) bound[i] = 0.0; }
    double *h = (double *)malloc(sizeof(double) * (size_t)F);
    double *Dall = (double *)malloc(sizeof(double) * (size_t)(K * H));
    double *hmax = (double *)malloc(sizeof(double) * (size_t)K);
    double *l1 = (double *)malloc(sizeof(double) * (size_t)H);
    for (int64_t s = 0; s < n_tokens; s++) {
        int64_t t = tokens[s];
        const void *xt = xdt == 1 ? (const void *)((const uint16_t *)x + t * H)
                                  : (const void *)((const float *)x + t * H);
        for (int64_t j = 0; j < K; j++) {
            int64_t e = idx[t * K + j];
            orc_gate_up_silu(pg + e * wstride_gu, sg + e * sstride_gu, pu + e * wstride_gu,
                             su + e * sstride_gu, F, H, gs, xt, xdt, 1, hdt, h, NULL, NULL);
            double m = 0.0;
            for (int64_t f = 0; f < F; f++) if (fabs(h[f]) > m) m = fabs(h[f]);
            hmax[j] = m;
            /* D = Wd_e h, with h as a double vector (already rounded to hdt) */
            const uint8_t *pde = pd + e * wstride_d;
            const float *sde = sd + e * sstride_d;
#pragma omp parallel for schedule(static)
            for (int64_t o = 0; o < H; o++) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; f++) acc += orc_weight(pde, sde, H, F, gs, o, f) * h[f];
                Dall[j * H + o] = acc;
            }
            if (bound) {
                orc_row_l1(pde, sde, H, F, gs, l1);
                for (int64_t o = 0; o < H; o++)
                    bound[s * H + o] += fabs(wts[t * K + j]) * l1[o] * hmax[j];
            }
        }
        for (int64_t o = 0; o < H; o++) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; j++) acc += wts[t * K + j] * Dall[j * H + o];
            y[s * H + o] = acc;
        }
    }
    free(h);
    free(Dall);
    free(hmax);
    free(l1);
}

/* ---------------------------------------------------------------------------------
 * NEXT rows: group-size detection, quantisation, row dequantisation / gather and the
 * matvec over selected rows.
 * ------------------------------------------------------------------------------- */

/* detect_group_size.  [PR298] "What was implemented (CPU)": detect_group_size() derives
 * gs from the byte count of the scale array, trying {16,32,48,64,96,128,192,256}.
 * Reading: a candidate matches when O*ceil(I/gs)*4 equals the byte count; the answer is
 * the single matching candidate.  Returns the group size, 0 when none matches, -1 when
 * more than one matches (their groups differ, so the size cannot decide). */
int64_t orc_detect_group_size(int64_t O, int64_t I, int64_t scale_bytes)
{
    static const int64_t cand[8] = {16, 32, 48, 64, 96, 128, 192, 256};
    int64_t found = 0;
    for (int c = 0; c < 8; c++) {
        if (orc_scale_bytes(O, I, cand[c]) != scale_bytes) continue;
        if (found) return -1;
        found = cand[c];
    }
    return found;
}

/* Quantisation of float weights into the grouped format (the converter step before
 * packing: [PR298] maintainer's "data request", "convert_fp8_to_int4.py --group-size 64").
 * The pages name the group-size option, not the rounding.  Reading: a symmetric
 * absmax scale per group, s = max|w| / 7, so the largest magnitude maps to +-7;
 * q = round-half-to-even(w / s), clamped to [-8, 7]; an all-zero group gets s = 0 and
 * q = 0.  The code is an integer decided by floating point, so the decision is taken in
 * f32 (single-precision division and rounding), the precision the GPU kernel uses.
 * Weights must be finite.  Output: q int8 [O][I] and scales f32 [O][ceil(I/gs)]; the
 * last group may be partial; gs >= I gives one group per row (the per-row fmt=2 case). */
void orc_quantize(const float *w, int64_t O, int64_t I, int64_t gs, int8_t *q, float *scales)
{
    int64_t ng = orc_ngroups(I, gs);
    for (int64_t o = 0; o < O; o++)
        for (int64_t g = 0; g < ng; g++) {
            int64_t k0 = g * gs, k1 = k0 + gs < I ? k0 + gs : I;
            float amax = 0.0f;
            for (int64_t k = k0; k < k1; k++) {
                float a = fabsf(w[o * I + k]);
                if (a > amax) amax = a;
            }
            volatile float s = amax / 7.0f;  /* f32 division, no contraction */
            scales[o * ng + g] = s;
            for (int64_t k = k0; k < k1; k++) {
                int v = 0;
                if (s > 0.0f) {
                    volatile float r = w[o * I + k] / s;
                    float rq = rintf(r);  /* round half to even (default rounding mode) */
                    if (rq > 7.0f) rq = 7.0f;
                    if (rq < -8.0f) rq = -8.0f;
                    v = (int)rq;
                }
                q[o * I + k] = (int8_t)v;
            }
        }
}

/* Row dequantisation / gather ([PR298] "embed_row, qt_addrow, qt_matvec_rows: fmt=4
 * branches"): out[j][k] = (accumulate ? out[j][k] : 0) + alpha_j * w(idx[j], k), fp64,
 * alpha_j = 1 when alpha is NULL.  embed_row is accumulate = 0 (a gather of dequantised
 * rows), qt_addrow is accumulate = 1. */
void orc_dequant_rows(const uint8_t *packed, const float *scales, int64_t O, int64_t I,
                      int64_t gs, const int32_t *idx, int64_t n, const double *alpha,
                      int accumulate, double *out)
{
    for (int64_t j = 0; j < n; j++) {
        double a = alpha ? alpha[j] : 1.0;
        for (int64_t k = 0; k < I; k++) {
            double v = a * orc_weight(packed, scales, O, I, gs, idx[j], k);
            out[j * I + k] = accumulate ? out[j * I + k] + v : v;
        }
    }
}

/* Matvec over selected rows (qt_matvec_rows): y[t][j] = sum_k w(idx[j], k) * x[t][k],
 * natural k order, fp64; bound[t][j] = ||w_row||_1 * max_k |x[t][k]| as for orc_matvec. */
void orc_matvec_rows(const uint8_t *packed, const float *scales, int64_t O, int64_t I,
                     int64_t gs, const int32_t *idx, int64_t n, const void *x, int xdt,
                     int64_t T, double *y, double *bound)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; j++) {
        int64_t o = idx[j];
        double l1 = 0.0;
        for (int64_t k = 0; k < I; k++) l1 += fabs(orc_weight(packed, scales, O, I, gs, o, k));
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0, xmax = 0.0;
            for (int64_t k = 0; k < I; k++) {
                double xv = orc_x(x, xdt, t * I + k);
                acc += orc_weight(packed, scales, O, I, gs, o, k) * xv;
                if (fabs(xv) > xmax) xmax = fabs(xv);
            }
            y[t * n + j] = acc;
            if (bound) bound[t * n + j] = l1 * xmax;
        }
    }
}

/* ---------------------------------------------------------------------------------
 * Grouped-scale MLA absorb projections over the kv_b tensor.
 * [PR298] "fmt=4 CUDA attention crash — root cause": the Q- and V-projection loops of
 * the two MLA attention absorb kernels multiply weights of the kv_b tensor (28,672 rows
 * x 512 inputs, 8 groups of 64 per row) by their scale.  With fmt=4 the scale of weight
 * (row, k) is scales[row*ng + k/gs], looked up inside the accumulation loop; one scale
 * per row applied after the loop is the fmt=2 rule and is wrong here.
 * Reading (the pages name the kernels, not their shapes): the rows of kv_b come in
 * per-head blocks of dn + dv rows, the first dn the key part and the last dv the value
 * part; the inputs are the R latent channels.  With D = dn + dv:
 *   Q absorb: q_lat[t][h][c] = sum_{d<dn} q_nope[t][h][d] * w(h*D + d, c),      c < R
 *   V absorb: o[t][h][v]     = sum_{c<R}  lat[t][h][c]   * w(h*D + dn + v, c),  v < dv
 * fp64, natural summation order.  bound = sum |w| * max |input| over the summed index
 * (the Sigma|terms| scale of the acceptance test).
 * ------------------------------------------------------------------------------- */
void orc_mla_absorb_q(const uint8_t *packed, const float *scales, int64_t R, int64_t gs,
                      int64_t nh, int64_t dn, int64_t dv, const void *q, int qdt, int64_t T,
                      double *out, double *bound)
{
    int64_t D = dn + dv, O = nh * D;
#pragma omp parallel for schedule(static)
    for (int64_t th = 0; th < T * nh; th++) {
        int64_t h = th % nh;
        for (int64_t c = 0; c < R; c++) {
            double acc = 0.0, l1 = 0.0, qmax = 0.0;
            for (int64_t d = 0; d < dn; d++) {
                double w = orc_weight(packed, scales, O, R, gs, h * D + d, c);
                double qv = orc_x(q, qdt, th * dn + d);
                acc += qv * w;
                l1 += fabs(w);
                if (fabs(qv) > qmax) qmax = fabs(qv);
            }
            out[th * R + c] = acc;
            if (bound) bound[th * R + c] = l1 * qmax;
        }
    }
}

void orc_mla_absorb_v(const uint8_t *packed, const float *scales, int64_t R, int64_t gs,
                      int64_t nh, int64_t dn, int64_t dv, const void *lat, int ldt, int64_t T,
                      double *out, double *bound)
{
    int64_t D = dn + dv, O = nh * D;
#pragma omp parallel for schedule(static)
    for (int64_t th = 0; th < T * nh; th++) {
        int64_t h = th % nh;
        for (int64_t v = 0; v < dv; v++) {
            double acc = 0.0, l1 = 0.0, xmax = 0.0;
            for (int64_t c = 0; c < R; c++) {
                double w = orc_weight(packed, scales, O, R, gs, h * D + dn + v, c);
                double xv = orc_x(lat, ldt, th * R + c);
                acc += xv * w;
                l1 += fabs(w);
                if (fabs(xv) > xmax) xmax = fabs(xv);
            }
            out[th * dv + v] = acc;
            if (bound) bound[th * dv + v] = l1 * xmax;
        }
    }
}

/* Threads the OpenMP loops above may use (test and baseline infrastructure: the CPU
 * baseline reports an all-core and a single-thread figure).  Returns the previous count
 * (1 when the oracle was built without OpenMP). */
int orc_set_threads(int n)
{
#ifdef _OPENMP
    int prev = omp_get_max_threads();
    if (n > 0) omp_set_num_threads(n);
    return prev;
#else
    (void)n;
    return 1;
#endif
}
