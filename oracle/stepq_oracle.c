/*
 * stepq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of the STEPQuant decode step
 * for gated Delta-rule recurrent states.  Only the tests, the smoke check and
 * the CPU-baseline leg of the benchmark may load it; the product path never
 * does.  It shares no code with the CUDA library: its own half-precision
 * conversion, its own byte layout code, its own loops.
 *
 * Arithmetic: IEEE binary32 (`float`) throughout, as the workloads fix ("fp32
 * state math"), round-to-nearest-even, compiled with -ffp-contract=off so no
 * multiply-add is fused unless written as fmaf().  Every sum runs over
 * ascending index, except the column-fit objective, whose order is stated in
 * objective().  Code and scale decisions are taken in that same binary32
 * arithmetic.
 *
 * Sources (the pages, cited by title and part):
 *   [P1] hyper.ai summary of "STEPQuant: When and Where Errors Matter in
 *        Delta-Rule Recurrent State Quantization", section "Method"
 *        (symmetric uniform quantisation; lifetime-aware allocation with FP16
 *        pivots; row-impact scores; key-row-aware dual-axis fitting; packed
 *        state kernels in the recurrent-state pool).
 *   [P3] rcap.io post on the same paper, the decode-step pseudocode (unpack,
 *        gated Delta update, readout before requantisation, row scales from
 *        sqrt(row magnitude)/sqrt(row impact), column scales by weighted
 *        least squares with squared impact weights, quantise X/(r c)).
 *   The deterministic column fit (8 candidates alpha * max_i|X_ij/r_i| / qmax,
 *   alpha = 1.0 .. 0.65, ties to the larger alpha), the round-half-even codes
 *   and the per-unit widths {4,6,8} are the concrete form taken here of
 *   [P3]'s `fit_weighted_lsq` and `quantize`, which the pages leave open.
 *
 * Readings where the pages are silent:
 *   - row magnitude = max_j |X_ij|; objective weight = w_i^2 (w as given).
 *   - per-row widths inside one head (key-row units): the row factor absorbs
 *     the width, rho_i = r_i * qmax_hi / qmax_i, so each row's codes span its
 *     own range; for a head of one width this is exactly r_i.
 *   - scales are stored as IEEE half (RNE, saturating at 65504, and a
 *     positive scale never rounds to zero: it is raised to 2^-24).
 *   - codes are stored offset-binary (code + 2^(b-1)), b bits each, LSB-first
 *     within a row's little-endian byte string.
 *   - a zero row (max |X_ij| = 0) stores rho = 0 and codes 0 and takes no part
 *     in the column fit; a zero column stores c = 0; a row holding a NaN or an
 *     infinity is stored as a zero row and raises STATUS_NONFINITE.
 *   - the column-fit objective sum_i w_i^2 (X_ij - r_i c code_ij)^2 is
 *     evaluated in one stated binary32 order (see objective()), because the
 *     argmin it feeds is an integer decision that the CUDA kernels must
 *     reproduce exactly for multi-step rollouts to agree; likewise the column
 *     maximum max_i |X_ij / r_i| takes the quotient as |X_ij| times the
 *     correctly rounded 1/r_i (times qmax_hi/qmax_i for rows of other widths).
 *     That order is itself pinned to the definition: oracle/definition.py
 *     evaluates the whole requantisation in float64 with no order, and
 *     tests/test_oracle_fullsize_fit.py holds this file's factors,
 *     candidates, objectives, argmin and codes to it on full-size heads of
 *     every workload (differences only within derived rounding bounds).
 *
 * Parity status of each function is stated in its comment ("pinned by ...").
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_INVALID 1
#define ORC_STATUS_NONFINITE 2
#define ORC_STATUS_BAD_SLOT 1

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16, written from the format's definition.                  */
/* Pinned by tests/test_oracle_half.py against numpy's float16 conversion.   */
/* ------------------------------------------------------------------------ */

float orc_half_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(m + 1024), e - 25);   /* (1024 + m) * 2^(e-15-10) */
    return sign ? -v : v;
}

/* Round to the nearest binary16 value, ties to even; values whose rounding
 * would exceed the largest finite half (65504) saturate to it; NaN -> 0. */
uint16_t orc_float_to_half(float x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    float a = fabsf(x);
    float r;
    int e;
    if (isnan(x))
        return 0;
    if (a >= 65504.0f)
        return sign | 0x7bff;
    if (a < 0x1p-14f) {
        r = rintf(a * 0x1p24f) * 0x1p-24f;       /* subnormal grid: 2^-24 */
    } else {
        float step;
        frexpf(a, &e);                           /* a in [2^(e-1), 2^e) */
        step = ldexpf(1.0f, e - 1 - 10);         /* 10 fraction bits */
        r = rintf(a / step) * step;
    }
    if (r == 0.0f)
        return sign;
    if (r < 0x1p-14f)
        return sign | (uint16_t)(r * 0x1p24f);
    frexpf(r, &e);                               /* r in [2^(e-1), 2^e) */
    {
        int ex = e - 1 + 15;
        int m = (int)(ldexpf(r, -(e - 1)) * 1024.0f) - 1024;
        return sign | (uint16_t)(ex << 10) | (uint16_t)m;
    }
}

/* A positive scale: half of x, but never zero for x > 0. */
static uint16_t scale_half(float x)
{
    uint16_t h = orc_float_to_half(x);
    if (x > 0.0f && h == 0)
        h = 1;                                    /* 2^-24 */
    return h;
}

/* ------------------------------------------------------------------------ */
/* Plan and byte layout                                                     */
/* ------------------------------------------------------------------------ */

typedef struct {
    int dk, dv, H;
    int gate_kind;      /* 0 scalar per head, 1 one gate per key row       */
    int unit_kind;      /* 0 head, 1 key row                                */
    int mode;           /* 0 STEPQuant dual-axis fit, 1 uniform per-row     */
    uint8_t *row_bits;  /* [H*dk]: 4, 6, 8 or 16 (FP16 pivot)              */
    float *w;           /* [H*dk]                                           */
    int *head_pivot;    /* [H]: 1 when the whole head is an FP16 pivot     */
    size_t *head_off;   /* [H]: byte offset of the head blob in a slot     */
    size_t *head_bytes; /* [H]                                              */
    size_t *row_off;    /* [H*dk]: byte offset of row i inside its blob    */
    size_t *scale_off;  /* [H]: offset of rho[dk] (c[dv] follows)          */
    size_t slot_bytes;
} orc_plan;

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static size_t row_bytes(int dv, int b) { return b == 16 ? (size_t)dv * 2 : (size_t)dv * b / 8; }

void orc_plan_free(void *p)
{
    orc_plan *pl = (orc_plan *)p;
    if (!pl)
        return;
    free(pl->row_bits); free(pl->w); free(pl->head_pivot); free(pl->head_off);
    free(pl->head_bytes); free(pl->row_off); free(pl->scale_off); free(pl);
}

/* bits: H entries (unit_kind 0) or H*dk entries (unit_kind 1). */
int orc_plan_new(int dk, int dv, int H, int gate_kind, int unit_kind, int mode,
                 const uint8_t *bits, const float *w, void **out)
{
    orc_plan *pl;
    size_t off = 0;
    int h, i;
    *out = NULL;
    if (dk <= 0 || dv <= 0 || H <= 0 || (gate_kind & ~1) || (unit_kind & ~1) || (mode & ~1))
        return ORC_ERR_INVALID;
    pl = (orc_plan *)calloc(1, sizeof(orc_plan));
    pl->dk = dk; pl->dv = dv; pl->H = H;
    pl->gate_kind = gate_kind; pl->unit_kind = unit_kind; pl->mode = mode;
    pl->row_bits = (uint8_t *)malloc((size_t)H * dk);
    pl->w = (float *)malloc(sizeof(float) * H * dk);
    pl->head_pivot = (int *)calloc(H, sizeof(int));
    pl->head_off = (size_t *)calloc(H, sizeof(size_t));
    pl->head_bytes = (size_t *)calloc(H, sizeof(size_t));
    pl->row_off = (size_t *)calloc((size_t)H * dk, sizeof(size_t));
    pl->scale_off = (size_t *)calloc(H, sizeof(size_t));
    for (h = 0; h < H; h++) {
        for (i = 0; i < dk; i++) {
            int b = unit_kind == 0 ? bits[h] : bits[h * dk + i];
            float wi = w[h * dk + i];
            if (!(b == 4 || b == 6 || b == 8 || b == 16) || (b != 16 && (dv * b) % 8) ||
                !(wi > 0.0f) || isinf(wi)) {
                orc_plan_free(pl);
                return ORC_ERR_INVALID;
            }
            pl->row_bits[h * dk + i] = (uint8_t)b;
            pl->w[h * dk + i] = wi;
        }
    }
    for (h = 0; h < H; h++) {
        size_t hb = 0;
        pl->head_pivot[h] = (unit_kind == 0 && bits[h] == 16);
        pl->head_off[h] = off;
        if (pl->head_pivot[h]) {
            hb = (size_t)dk * dv * 2;            /* raw halves, row-major */
        } else {
            for (i = 0; i < dk; i++) {
                pl->row_off[h * dk + i] = hb;
                hb += row_bytes(dv, pl->row_bits[h * dk + i]);
            }
            pl->scale_off[h] = hb;
            hb += (size_t)dk * 2 + (size_t)dv * 2; /* rho[dk] then c[dv], halves */
        }
        pl->head_bytes[h] = round_up(hb, 16);
        off += pl->head_bytes[h];
    }
    pl->slot_bytes = round_up(off, 256);
    *out = pl;
    return ORC_OK;
}

size_t orc_slot_bytes(const void *p) { return ((const orc_plan *)p)->slot_bytes; }

void orc_head_layout(const void *p, int h, size_t *off, size_t *bytes)
{
    const orc_plan *pl = (const orc_plan *)p;
    *off = pl->head_off[h];
    *bytes = pl->head_bytes[h];
}

/* ------------------------------------------------------------------------ */
/* Code packing: b-bit offset-binary codes, LSB-first in a row's bytes.      */
/* Pinned by tests/test_oracle_pack.py (hand-derived byte strings and a     */
/* round trip over every code of every width).                               */
/* ------------------------------------------------------------------------ */

static void put_bits(uint8_t *row, int pos, int nbits, uint32_t val)
{
    int t;
    for (t = 0; t < nbits; t++) {
        int bit = pos + t;
        if ((val >> t) & 1u)
            row[bit / 8] |= (uint8_t)(1u << (bit % 8));
        else
            row[bit / 8] &= (uint8_t)~(1u << (bit % 8));
    }
}

static uint32_t get_bits(const uint8_t *row, int pos, int nbits)
{
    uint32_t v = 0;
    int t;
    for (t = 0; t < nbits; t++) {
        int bit = pos + t;
        v |= (uint32_t)((row[bit / 8] >> (bit % 8)) & 1u) << t;
    }
    return v;
}

static void put_half(uint8_t *p, uint16_t h) { p[0] = (uint8_t)(h & 0xff); p[1] = (uint8_t)(h >> 8); }
static uint16_t get_half(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Write one head blob from its codes [dk*dv] (ignored on pivot rows), pivot
 * halves [dk*dv] (used on pivot rows / pivot heads), rho[dk] and c[dv]. */
void orc_pack_codes(const void *p, int h, const int16_t *codes, const uint16_t *piv,
                    const uint16_t *rho, const uint16_t *c, uint8_t *blob)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, i, j;
    memset(blob, 0, pl->head_bytes[h]);
    if (pl->head_pivot[h]) {
        for (i = 0; i < dk * dv; i++)
            put_half(blob + 2 * (size_t)i, piv[i]);
        return;
    }
    for (i = 0; i < dk; i++) {
        int b = pl->row_bits[h * dk + i];
        uint8_t *row = blob + pl->row_off[h * dk + i];
        for (j = 0; j < dv; j++) {
            if (b == 16)
                put_half(row + 2 * j, piv[i * dv + j]);
            else
                put_bits(row, j * b, b, (uint32_t)(codes[i * dv + j] + (1 << (b - 1))));
        }
        put_half(blob + pl->scale_off[h] + 2 * i, rho[i]);
    }
    for (j = 0; j < dv; j++)
        put_half(blob + pl->scale_off[h] + 2 * dk + 2 * j, c[j]);
}

/* Read a head blob back into codes / pivot halves / rho / c. */
void orc_unpack_codes(const void *p, int h, const uint8_t *blob, int16_t *codes,
                      uint16_t *piv, uint16_t *rho, uint16_t *c)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, i, j;
    if (pl->head_pivot[h]) {
        for (i = 0; i < dk * dv; i++) {
            piv[i] = get_half(blob + 2 * (size_t)i);
            codes[i] = 0;
        }
        for (i = 0; i < dk; i++) rho[i] = 0;
        for (j = 0; j < dv; j++) c[j] = 0;
        return;
    }
    for (i = 0; i < dk; i++) {
        int b = pl->row_bits[h * dk + i];
        const uint8_t *row = blob + pl->row_off[h * dk + i];
        for (j = 0; j < dv; j++) {
            if (b == 16) {
                piv[i * dv + j] = get_half(row + 2 * j);
                codes[i * dv + j] = 0;
            } else {
                piv[i * dv + j] = 0;
                codes[i * dv + j] = (int16_t)((int)get_bits(row, j * b, b) - (1 << (b - 1)));
            }
        }
        rho[i] = get_half(blob + pl->scale_off[h] + 2 * i);
    }
    for (j = 0; j < dv; j++)
        c[j] = get_half(blob + pl->scale_off[h] + 2 * dk + 2 * j);
}

/* ------------------------------------------------------------------------ */
/* Reconstruction: S_prev = codes (.) (r c^T), FP16 pivots raw.  [P3]        */
/* Pinned by the round-trip and per-entry error tests.                       */
/* ------------------------------------------------------------------------ */

void orc_dequantize_head(const void *p, int h, const uint8_t *blob, float *S)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, i, j;
    int16_t *codes = (int16_t *)malloc(sizeof(int16_t) * dk * dv);
    uint16_t *piv = (uint16_t *)malloc(sizeof(uint16_t) * dk * dv);
    uint16_t *rho = (uint16_t *)malloc(sizeof(uint16_t) * dk);
    uint16_t *c = (uint16_t *)malloc(sizeof(uint16_t) * dv);
    orc_unpack_codes(p, h, blob, codes, piv, rho, c);
    for (i = 0; i < dk; i++) {
        int b = pl->head_pivot[h] ? 16 : pl->row_bits[h * dk + i];
        for (j = 0; j < dv; j++) {
            if (b == 16)
                S[i * dv + j] = orc_half_to_float(piv[i * dv + j]);
            else
                S[i * dv + j] = (float)codes[i * dv + j] *
                                (orc_half_to_float(rho[i]) * orc_half_to_float(c[j]));
        }
    }
    free(codes); free(piv); free(rho); free(c);
}

/* ------------------------------------------------------------------------ */
/* The quantiser on an updated state X (one head).                           */
/*   row factor   r_i = sqrt(max_j|X_ij|) / sqrt(w_i)             [P3][P1]   */
/*   column scale c_j = argmin over alpha of sum_i w_i^2 (X_ij -               */
/*                r_i c_j code_ij)^2, c = alpha max_i|X_ij/r_i| / qmax [P3]    */
/*   codes        clamp(rne(X_ij / (r_i c_j)), +-qmax_i)                [P3]  */
/* Uniform mode (the pages' INT-b comparator): per-row absmax scale          */
/* s_i = max_j|X_ij| / qmax_i, c = 1.                                        */
/* Pinned by tests/test_oracle_quant.py: exact rational brute force of the   */
/* candidate objective on small heads, closed forms of r and M, per-entry    */
/* error bounds.                                                             */
/* ------------------------------------------------------------------------ */

static const float ALPHA[8] = {1.0f, 0.95f, 0.9f, 0.85f, 0.8f, 0.75f, 0.7f, 0.65f};

/* The weighted least-squares objective of one candidate column scale c,
 * E = sum_i w_i^2 (X_ij - r_i c code_i)^2, evaluated in units of each row's
 * quantisation step: with z_i = |X_ij| * (1/r_i) and t_i = z_i * (1/c),
 *     E = c^2 * sum_i A_i (t_i - code_i)^2,   A_i = (w_i r_i)^2,
 * code_i = min(rne(t_i), qmax_i).  binary32, in this order:
 *   - 1/r_i and 1/c correctly rounded; z_i = |X_ij| * (1/r_i) rounded;
 *   - q = fmaf(z_i, 1/c, 2^23) rounds t_i to an integer (exact product,
 *     one rounding); clamp q to 2^23 + qmax_i; d_i = fmaf(z_i, 1/c, 2^23 - q);
 *   - four partial sums P_g over the rows i = g, g+4, g+8, ... (ascending),
 *     P_g = fmaf(A_i * d_i, d_i, P_g);
 *   - E = (c * c) * ((P_0 + P_1) + (P_2 + P_3)).
 * Rows that are zero, non-finite or FP16 pivots take no part. */
static float objective(const float *X, int dv, int j, int dk, const int *active,
                       const float *irho, const float *A, const int *qmax, float c)
{
    const float two23 = 8388608.0f;
    float ic = 1.0f / c;
    float P[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    int i;
    for (i = 0; i < dk; i++) {
        float z, q, d;
        if (!active[i])
            continue;
        z = fabsf(X[i * dv + j]) * irho[i];
        q = fmaf(z, ic, two23);
        if (q > two23 + (float)qmax[i])
            q = two23 + (float)qmax[i];
        d = fmaf(z, ic, two23 - q);
        P[i & 3] = fmaf(A[i] * d, d, P[i & 3]);
    }
    return (c * c) * ((P[0] + P[1]) + (P[2] + P[3]));
}

static int code_of(float x, float P, int qmax)
{
    float t = x / P;                              /* X / (r c), one rounding */
    float r = rintf(t);                           /* round half to even */
    if (r > (float)qmax) r = (float)qmax;
    if (r < -(float)qmax) r = -(float)qmax;
    return (int)r;
}

/* Codes of one column under a given column scale c (half bits); rows that are
 * pivots or zero get code 0.  Exposed so a test can re-derive the codes of a
 * column under any candidate. */
void orc_column_codes(const void *p, int h, const float *X, const uint16_t *rho, int j,
                      uint16_t c_bits, int16_t *codes_col)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, i;
    float cj = orc_half_to_float(c_bits);
    for (i = 0; i < dk; i++) {
        int b = pl->row_bits[h * dk + i];
        float ri = orc_half_to_float(rho[i]);
        if (b == 16 || ri == 0.0f || cj == 0.0f)
            codes_col[i] = 0;
        else
            codes_col[i] = (int16_t)code_of(X[i * dv + j], ri * cj, (1 << (b - 1)) - 1);
    }
}

/* Quantise X [dk*dv] of head h into blob.  Optional diagnostics (may be NULL):
 *   E [dv*8]  objective of each candidate, cand [dv*8] candidate scales (half
 *   bits), best [dv] chosen candidate.  Returns a status bit mask. */
int orc_quantize_head(const void *p, int h, const float *X, uint8_t *blob,
                      float *E_diag, uint16_t *cand_diag, int8_t *best_diag)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, i, j, a;
    int status = 0;
    int16_t *codes = (int16_t *)calloc((size_t)dk * dv, sizeof(int16_t));
    uint16_t *piv = (uint16_t *)calloc((size_t)dk * dv, sizeof(uint16_t));
    uint16_t *rho = (uint16_t *)calloc(dk, sizeof(uint16_t));
    uint16_t *c = (uint16_t *)calloc(dv, sizeof(uint16_t));
    int *active = (int *)calloc(dk, sizeof(int));
    int *qmax = (int *)calloc(dk, sizeof(int));
    float *kappa = (float *)calloc(dk, sizeof(float));
    int16_t *col = (int16_t *)calloc(dk, sizeof(int16_t));
    float *irho = (float *)calloc(dk, sizeof(float));
    float *ikap = (float *)calloc(dk, sizeof(float));
    float *Aw = (float *)calloc(dk, sizeof(float));
    int qhi = 0;

    if (E_diag) for (a = 0; a < dv * 8; a++) E_diag[a] = 0.0f;
    if (cand_diag) for (a = 0; a < dv * 8; a++) cand_diag[a] = 0;
    if (best_diag) for (j = 0; j < dv; j++) best_diag[j] = 0;

    for (i = 0; i < dk; i++) {
        int b = pl->head_pivot[h] ? 16 : pl->row_bits[h * dk + i];
        if (b == 16) {
            /* FP16 pivot unit: stored raw [P1] */
            for (j = 0; j < dv; j++) {
                float x = X[i * dv + j];
                if (!isfinite(x))
                    status |= ORC_STATUS_NONFINITE;
                piv[i * dv + j] = orc_float_to_half(x);
            }
            continue;
        }
        qmax[i] = (1 << (b - 1)) - 1;
        if (qmax[i] > qhi)
            qhi = qmax[i];
    }
    if (!pl->head_pivot[h]) {
        /* row factors */
        for (i = 0; i < dk; i++) {
            float m = 0.0f;
            int bad = 0;
            if (pl->row_bits[h * dk + i] == 16)
                continue;
            for (j = 0; j < dv; j++) {
                float ax = fabsf(X[i * dv + j]);
                if (!isfinite(ax))
                    bad = 1;
                else if (ax > m)
                    m = ax;
            }
            if (bad) {
                status |= ORC_STATUS_NONFINITE;
                m = 0.0f;
            }
            if (m == 0.0f)
                continue;                         /* zero row: rho 0, codes 0 */
            active[i] = 1;
            if (pl->mode == 0) {
                float r = sqrtf(m) / sqrtf(pl->w[h * dk + i]);
                kappa[i] = (float)qhi / (float)qmax[i];
                rho[i] = scale_half(r * kappa[i]);
            } else {
                rho[i] = scale_half(m / (float)qmax[i]);
            }
        }
        if (pl->mode == 1) {
            for (j = 0; j < dv; j++)
                c[j] = 0x3c00;                    /* 1.0 */
        } else {
            for (i = 0; i < dk; i++) {
                if (!active[i])
                    continue;
                irho[i] = 1.0f / orc_half_to_float(rho[i]);
                ikap[i] = irho[i] * kappa[i];
                Aw[i] = (pl->w[h * dk + i] * orc_half_to_float(rho[i])) *
                        (pl->w[h * dk + i] * orc_half_to_float(rho[i]));
            }
            for (j = 0; j < dv; j++) {
                float M = 0.0f, Ebest = 0.0f;
                int best = 0;
                for (i = 0; i < dk; i++) {
                    float z;
                    if (!active[i])
                        continue;
                    /* max_i |X_ij / r_i| (times kappa_i), the quotient taken as a
                     * product with the correctly rounded 1/r_i, as in the objective */
                    z = fabsf(X[i * dv + j]) * ikap[i];
                    if (z > M)
                        M = z;
                }
                if (M == 0.0f) {
                    c[j] = 0;
                    continue;
                }
                for (a = 0; a < 8; a++) {
                    uint16_t ca = scale_half((ALPHA[a] * M) / (float)qhi);
                    float E = objective(X, dv, j, dk, active, irho, Aw, qmax,
                                        orc_half_to_float(ca));
                    if (E_diag) E_diag[j * 8 + a] = E;
                    if (cand_diag) cand_diag[j * 8 + a] = ca;
                    if (a == 0 || E < Ebest) {    /* strict: ties keep the larger alpha */
                        Ebest = E;
                        best = a;
                        c[j] = ca;
                    }
                }
                if (best_diag) best_diag[j] = (int8_t)best;
            }
        }
        for (j = 0; j < dv; j++) {
            orc_column_codes(p, h, X, rho, j, c[j], col);
            for (i = 0; i < dk; i++)
                codes[i * dv + j] = active[i] ? col[i] : 0;
        }
    }
    orc_pack_codes(p, h, codes, piv, rho, c, blob);
    free(codes); free(piv); free(rho); free(c); free(active); free(qmax); free(kappa); free(col);
    free(irho); free(ikap); free(Aw);
    return status;
}

/* ------------------------------------------------------------------------ */
/* The gated Delta update and readout (one head).                [P3][P1]     */
/*   X = D S + beta k (v^T - k^T D S),  y = X^T q  (before requantisation)   */
/* D = g I (scalar gate) or diag(g) (one gate per key row).                  */
/* Pinned by tests/test_oracle_step.py: g=1,beta=0 leaves S unchanged        */
/* bit-exactly; g=1,beta=1,|k|=1 writes k^T X = v^T; the matrix form         */
/* evaluated by numpy in float64.                                            */
/* ------------------------------------------------------------------------ */

/* As orc_delta_update, also storing delta [dv] when delta_out is not NULL. */
void orc_delta_update_d(int dk, int dv, const float *S, const float *q, const float *k,
                        const float *v, float beta, const float *gate, int gate_kind,
                        float *X, float *y, float *delta_out)
{
    int i, j;
    for (j = 0; j < dv; j++) {
        float u = 0.0f, delta;
        for (i = 0; i < dk; i++) {
            float g = gate_kind ? gate[i] : gate[0];
            u = u + k[i] * (g * S[i * dv + j]);   /* (k^T D S)_j */
        }
        delta = beta * (v[j] - u);
        if (delta_out)
            delta_out[j] = delta;
        for (i = 0; i < dk; i++) {
            float g = gate_kind ? gate[i] : gate[0];
            X[i * dv + j] = g * S[i * dv + j] + k[i] * delta;
        }
    }
    for (j = 0; j < dv; j++) {
        float acc = 0.0f;
        for (i = 0; i < dk; i++)
            acc = acc + q[i] * X[i * dv + j];     /* (X^T q)_j */
        y[j] = acc;
    }
}

void orc_delta_update(int dk, int dv, const float *S, const float *q, const float *k,
                      const float *v, float beta, const float *gate, int gate_kind,
                      float *X, float *y)
{
    orc_delta_update_d(dk, dv, S, q, k, v, beta, gate, gate_kind, X, y, NULL);
}

/* One quantised decode step of one head in place on its blob. */
int orc_step_head(const void *p, int h, uint8_t *blob, const float *q, const float *k,
                  const float *v, float beta, const float *gate, float *y, float *X_out)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, st;
    float *S = (float *)malloc(sizeof(float) * dk * dv);
    float *X = X_out ? X_out : (float *)malloc(sizeof(float) * dk * dv);
    orc_dequantize_head(p, h, blob, S);
    orc_delta_update(dk, dv, S, q, k, v, beta, gate, pl->gate_kind, X, y);
    st = orc_quantize_head(p, h, X, blob, NULL, NULL, NULL);
    free(S);
    if (!X_out)
        free(X);
    return st;
}

/* ------------------------------------------------------------------------ */
/* Pool-level calls over n requests (slot-indexed pool of packed states).    */
/* Arrays are dense: q,k,v,y [n][H][d], beta [n][H], gate [n][H] or          */
/* [n][H][dk], X/S [n][H][dk][dv].                                           */
/* ------------------------------------------------------------------------ */

int orc_pack(const void *p, uint8_t *pool, int64_t num_slots, const int32_t *slot_idx,
             int64_t n, const float *X)
{
    const orc_plan *pl = (const orc_plan *)p;
    int64_t r;
    int h, st = 0;
    size_t hs = (size_t)pl->dk * pl->dv;
    for (r = 0; r < n; r++) {
        if (slot_idx[r] < 0 || slot_idx[r] >= num_slots) {
            st |= ORC_STATUS_BAD_SLOT;
            continue;
        }
        for (h = 0; h < pl->H; h++)
            st |= orc_quantize_head(p, h, X + ((size_t)r * pl->H + h) * hs,
                                    pool + (size_t)slot_idx[r] * pl->slot_bytes + pl->head_off[h],
                                    NULL, NULL, NULL);
    }
    return st;
}

int orc_unpack(const void *p, const uint8_t *pool, int64_t num_slots, const int32_t *slot_idx,
               int64_t n, float *S)
{
    const orc_plan *pl = (const orc_plan *)p;
    int64_t r;
    int h, st = 0;
    size_t hs = (size_t)pl->dk * pl->dv;
    for (r = 0; r < n; r++) {
        if (slot_idx[r] < 0 || slot_idx[r] >= num_slots) {
            st |= ORC_STATUS_BAD_SLOT;
            continue;
        }
        for (h = 0; h < pl->H; h++)
            orc_dequantize_head(p, h, pool + (size_t)slot_idx[r] * pl->slot_bytes + pl->head_off[h],
                                S + ((size_t)r * pl->H + h) * hs);
    }
    return st;
}

int orc_decode_step(const void *p, uint8_t *pool, int64_t num_slots, const int32_t *slot_idx,
                    int64_t n, const float *q, const float *k, const float *v,
                    const float *beta, const float *gate, float *y)
{
    const orc_plan *pl = (const orc_plan *)p;
    int64_t r;
    int h, st = 0;
    int d = pl->dk, dv = pl->dv, H = pl->H;
    for (r = 0; r < n; r++) {
        if (slot_idx[r] < 0 || slot_idx[r] >= num_slots) {
            st |= ORC_STATUS_BAD_SLOT;
            continue;
        }
        for (h = 0; h < H; h++) {
            size_t rh = (size_t)r * H + h;
            const float *g = pl->gate_kind ? gate + rh * d : gate + rh;
            st |= orc_step_head(p, h, pool + (size_t)slot_idx[r] * pl->slot_bytes + pl->head_off[h],
                                q + rh * d, k + rh * d, v + rh * dv, beta[rh], g, y + rh * dv, NULL);
        }
    }
    return st;
}

/* ------------------------------------------------------------------------ */
/* Per-unit reconstruction distortion, the input of the lifetime-aware bit   */
/* allocation ([P1], section "Method": the distortion of every state unit    */
/* at each candidate width is measured on calibration states).               */
/*   D_u = sum over the unit's entries of (X_ij - S_ij)^2,                   */
/* S the dequantised packed state; each difference taken in double from the  */
/* binary32 values, squares summed in double over rows then columns, in      */
/* ascending order.  A unit is a head (unit_kind 0) or one key row           */
/* (unit_kind 1); dist is [n][units], units = H or H*dk.  Rows of slots out  */
/* of range are skipped (status BAD_SLOT, their entries left untouched).     */
/* Pinned by tests/test_oracle_alloc.py: zero for states that the quantiser  */
/* represents exactly, and equal to the squared Frobenius error of          */
/* orc_unpack's reconstruction computed independently.                       */
/* ------------------------------------------------------------------------ */

int orc_unit_distortion(const void *p, const uint8_t *pool, int64_t num_slots,
                        const int32_t *slot_idx, int64_t n, const float *X, double *dist)
{
    const orc_plan *pl = (const orc_plan *)p;
    int dk = pl->dk, dv = pl->dv, H = pl->H, h, i, j, st = 0;
    int64_t r;
    size_t hs = (size_t)dk * dv;
    size_t units = pl->unit_kind ? (size_t)H * dk : (size_t)H;
    float *S = (float *)malloc(sizeof(float) * hs);
    for (r = 0; r < n; r++) {
        if (slot_idx[r] < 0 || slot_idx[r] >= num_slots) {
            st |= ORC_STATUS_BAD_SLOT;
            continue;
        }
        for (h = 0; h < H; h++) {
            const float *Xh = X + ((size_t)r * H + h) * hs;
            double head = 0.0;
            orc_dequantize_head(p, h, pool + (size_t)slot_idx[r] * pl->slot_bytes + pl->head_off[h], S);
            for (i = 0; i < dk; i++) {
                double row = 0.0;
                for (j = 0; j < dv; j++) {
                    double e = (double)Xh[i * dv + j] - (double)S[i * dv + j];
                    row += e * e;
                }
                if (pl->unit_kind)
                    dist[(size_t)r * units + (size_t)h * dk + i] = row;
                head += row;
            }
            if (!pl->unit_kind)
                dist[(size_t)r * units + h] = head;
        }
    }
    free(S);
    return st;
}

/* The unquantised baseline: the same update on an fp32 state, in place. */
void orc_fp32_step_head(int dk, int dv, float *S, const float *q, const float *k,
                        const float *v, float beta, const float *gate, int gate_kind, float *y)
{
    float *X = (float *)malloc(sizeof(float) * dk * dv);
    orc_delta_update(dk, dv, S, q, k, v, beta, gate, gate_kind, X, y);
    memcpy(S, X, sizeof(float) * dk * dv);
    free(X);
}

int orc_fp32_step(int dk, int dv, int H, int gate_kind, float *S, int64_t num_slots,
                  const int32_t *slot_idx, int64_t n, const float *q, const float *k,
                  const float *v, const float *beta, const float *gate, float *y)
{
    int64_t r;
    int h, st = 0;
    size_t hs = (size_t)dk * dv;
    for (r = 0; r < n; r++) {
        if (slot_idx[r] < 0 || slot_idx[r] >= num_slots) {
            st |= ORC_STATUS_BAD_SLOT;
            continue;
        }
        for (h = 0; h < H; h++) {
            size_t rh = (size_t)r * H + h;
            const float *g = gate_kind ? gate + rh * dk : gate + rh;
            orc_fp32_step_head(dk, dv, S + ((size_t)slot_idx[r] * H + h) * hs, q + rh * dk,
                               k + rh * dk, v + rh * dv, beta[rh], g, gate_kind, y + rh * dv);
        }
    }
    return st;
}
