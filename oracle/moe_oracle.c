/*
 * CPU oracle for the block-quantized, top-k routed MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA path is checked against.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the library's own code path never
 * calls it, and it shares no code, header or constant with that path.
 *
 * Everything is computed in fp64 from the exact stored inputs (bf16 hidden
 * states, fp32 router weights, fp16 scales, integer codes), one token at a
 * time, with every sum taken sequentially in index order.  The only rounding
 * the method itself defines is the final bf16 output of the layer.
 *
 * What the source pages fix, and where this code follows them:
 *  - "Strata Coder deep-dive" page, section 1: a layer has 512 experts (256 in
 *    the pruned Coder variant, section 2) and each token is routed to 10 of
 *    them -> oracle_topk with k = 10.
 *  - same page, sections 2-3: an expert is three projections, gate, up and
 *    down, stored block-quantized at low bit width, gate/up at lower precision
 *    than down -> oracle_dequant, oracle_expert_ffn (per-matrix bit widths).
 *  - "Coder benchmark record" page, "expert profile file" section: a ranking
 *    of every (layer, expert) pair built from routing counts -> oracle_hist_add,
 *    oracle_rank.
 * Readings where the pages are silent (listed again in the design notes):
 *  - SwiGLU expert: h = silu(W_g x) * (W_u x), y = W_d h.
 *  - gate weights: softmax over the selected k logits (equal to a softmax over
 *    all E followed by renormalisation over the k); ties broken by the lower
 *    expert index, which also fixes the order of a token's k slots.
 *  - block-32 codes with an fp16 scale: w = scale * (code - 2^(bits-1)).
 *  - out = (residual ? x : 0) + sum_j w_j * y_j, rounded once to bf16 (RNE).
 *  - a selected expert whose slot is -1 or >= n_slots contributes 0 and the
 *    call reports it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_SLOT (-6)

/* Same memory layout as the library's arena descriptor; defined here on its own. */
typedef struct {
    int32_t H, I, block;
    int32_t bits_gate, bits_up, bits_down;
    int64_t slot_bytes;
    int64_t off_codes[3];
    int64_t off_scales[3];
    int32_t n_slots;
    int32_t reserved;
} orc_desc;

/* ---------------------------------------------------------------- numbers */

/* bf16 bits -> value: the bf16 pattern is the top half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* IEEE binary16 bits -> value, decoded field by field. */
double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)mant, -24);                 /* subnormal: mant * 2^-24 */
    else if (expo == 31)
        v = mant ? NAN : INFINITY;
    else
        v = ldexp((double)(mant | 0x400), expo - 25); /* 1.mant * 2^(expo-15) */
    return sign ? -v : v;
}

/* Round a double to the nearest bf16 (ties to even) and return its bits.
 * bf16: 8 significant bits, binary32 exponent range, subnormal quantum 2^-133. */
uint16_t oracle_double_to_bf16(double v) {
    if (isnan(v)) return 0x7fc0;
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v), r;
    if (a == 0.0) return neg ? 0x8000 : 0;
    if (a < ldexp(1.0, -126)) {
        r = ldexp(nearbyint(ldexp(a, 133)), -133);     /* subnormal range */
    } else {
        int e;
        double m = frexp(a, &e);                       /* a = m * 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);      /* keep 8 significant bits */
    }
    float f = (float)r;                                /* exact: r is a bf16 value or inf */
    if (r > 3.3895313892515355e38) f = INFINITY;       /* above the largest finite bf16 */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t b = (uint16_t)(u >> 16);
    return neg ? (uint16_t)(b | 0x8000) : b;
}

/* ---------------------------------------------------------------- arena */

static void mat_shape(const orc_desc* d, int m, int* rows, int* K) {
    if (m < 2) { *rows = d->I; *K = d->H; } else { *rows = d->H; *K = d->I; }
}

static int mat_bits(const orc_desc* d, int m) {
    return m == 0 ? d->bits_gate : (m == 1 ? d->bits_up : d->bits_down);
}

/* Stored code of element (row, c) of matrix m: bits LSB-first, row-major. */
int oracle_code(const uint8_t* slot, const orc_desc* d, int m, int row, int c) {
    int rows, K;
    mat_shape(d, m, &rows, &K);
    int b = mat_bits(d, m);
    int64_t row_bytes = (int64_t)K * b / 8;
    int64_t bit = (int64_t)c * b;
    uint8_t byte = slot[d->off_codes[m] + row * row_bytes + bit / 8];
    return (byte >> (bit % 8)) & ((1 << b) - 1);
}

/* Dequantised weight: scale[row][c/32] * (code - 2^(bits-1)). */
double oracle_dequant(const uint8_t* slot, const orc_desc* d, int m, int row, int c) {
    int rows, K;
    mat_shape(d, m, &rows, &K);
    int b = mat_bits(d, m);
    const uint8_t* sp = slot + d->off_scales[m] + 2 * ((int64_t)row * (K / d->block) + c / d->block);
    uint16_t sbits = (uint16_t)(sp[0] | (sp[1] << 8));
    int q = oracle_code(slot, d, m, row, c);
    return oracle_half_to_double(sbits) * (double)(q - (1 << (b - 1)));
}

/* ---------------------------------------------------------------- expert FFN */

double oracle_silu(double g) { return g / (1.0 + exp(-g)); }

/* y = W_d (silu(W_g x) * (W_u x)) for one token; h (length I) is optional. */
void oracle_expert_ffn(const uint8_t* slot, const orc_desc* d, const double* x, double* y, double* h_out) {
    int H = d->H, I = d->I;
    double* h = (double*)malloc(sizeof(double) * I);
    for (int r = 0; r < I; r++) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; c++) g += oracle_dequant(slot, d, 0, r, c) * x[c];
        for (int c = 0; c < H; c++) u += oracle_dequant(slot, d, 1, r, c) * x[c];
        h[r] = oracle_silu(g) * u;
    }
    for (int c = 0; c < H; c++) {
        double s = 0.0;
        for (int r = 0; r < I; r++) s += oracle_dequant(slot, d, 2, c, r) * h[r];
        y[c] = s;
    }
    if (h_out) memcpy(h_out, h, sizeof(double) * I);
    free(h);
}

/* ---------------------------------------------------------------- router */

/* logits[t][e] = (sum over h, in order, of x[t][h] * W[e][h]) + b[e], all fp64.
 * Each bf16 x fp32 product is exact in fp64; the sum is rounded in index order. */
void oracle_router_logits(const uint16_t* x, int T, int H, const float* W, const float* b,
                          int E, double* logits) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; t++) {
        for (int e = 0; e < E; e++) {
            double s = 0.0;
            for (int h = 0; h < H; h++)
                s += oracle_bf16_to_double(x[(int64_t)t * H + h]) * (double)W[(int64_t)e * H + h];
            if (b) s += (double)b[e];
            logits[(int64_t)t * E + e] = s;
        }
    }
}

/* A logit as it takes part in the selection and the weights: NaN counts as
 * -infinity (the pages fix nothing for non-finite values; this makes the order
 * total, so a NaN logit ranks below every number and, if selected, weighs 0). */
static double orc_ord(double v) { return isnan(v) ? -INFINITY : v; }

/* Top-k by repeated selection: the j-th pick is the largest logit not yet
 * chosen, the lower expert index winning an exact tie.  Weights are the
 * softmax of the k chosen logits: w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0). */
void oracle_topk(const double* logits, int T, int E, int k, int32_t* idx, double* w) {
    char* taken = (char*)malloc(E);
    for (int t = 0; t < T; t++) {
        const double* l = logits + (int64_t)t * E;
        memset(taken, 0, E);
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || orc_ord(l[e]) > orc_ord(l[best])) best = e;   /* strict '>' keeps the lower index */
            }
            taken[best] = 1;
            idx[(int64_t)t * k + j] = best;
        }
        double l0 = orc_ord(l[idx[(int64_t)t * k]]), z = 0.0;
        for (int j = 0; j < k; j++) z += exp(orc_ord(l[idx[(int64_t)t * k + j]]) - l0);
        for (int j = 0; j < k; j++) w[(int64_t)t * k + j] = exp(orc_ord(l[idx[(int64_t)t * k + j]]) - l0) / z;
    }
    free(taken);
}

/* ---------------------------------------------------------------- grouping */

/* Pair p = t*k + j routes token t to expert idx[p].  counts[e] = number of
 * pairs on e; offsets = exclusive prefix sum (E+1 entries); perm lists the
 * pairs grouped by expert, ascending pair id inside a group; inv[perm[i]] = i. */
void oracle_permutation(const int32_t* idx, int T, int k, int E, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv) {
    int64_t P = (int64_t)T * k;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int64_t p = 0; p < P; p++) counts[idx[p]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    for (int e = 0; e < E; e++) {
        int32_t pos = offsets[e];
        for (int64_t p = 0; p < P; p++)
            if (idx[p] == e) { perm[pos] = (int32_t)p; inv[p] = pos; pos++; }
    }
}

/* hist[layer][e] += counts[e] */
void oracle_hist_add(const int32_t* counts, int E, int layer, uint32_t* hist) {
    for (int e = 0; e < E; e++) hist[(int64_t)layer * E + e] += (uint32_t)counts[e];
}

/* ---------------------------------------------------------------- ranking */

static const uint32_t* g_rank_hist;
static int g_rank_E;

static int rank_cmp(const void* a, const void* b) {
    int32_t i = *(const int32_t*)a, j = *(const int32_t*)b;
    uint32_t ci = g_rank_hist[i], cj = g_rank_hist[j];
    if (ci != cj) return ci > cj ? -1 : 1;      /* more routed first */
    return i < j ? -1 : (i > j ? 1 : 0);        /* then (layer, expert) ascending */
}

/* Rank every (layer, expert) pair by routing count; pairs[2r] = layer,
 * pairs[2r+1] = expert of rank r.  The comparison is a total order, so the
 * result does not depend on the sort algorithm. */
void oracle_rank(const uint32_t* hist, int L, int E, uint16_t* pairs) {
    int32_t n = L * E;
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * n);
    for (int32_t i = 0; i < n; i++) order[i] = i;
    g_rank_hist = hist;
    g_rank_E = E;
    qsort(order, n, sizeof(int32_t), rank_cmp);
    for (int32_t r = 0; r < n; r++) {
        pairs[2 * r] = (uint16_t)(order[r] / E);
        pairs[2 * r + 1] = (uint16_t)(order[r] % E);
    }
    free(order);
}

/* ---------------------------------------------------------------- layer */

/* Steering projection of the "Coder benchmark record" page, section on the
 * steering vector: after the layer, the component of the residual stream h
 * along a unit direction v is removed, h - (h . v) v.  The dot product is
 * summed in index order in fp64; v is used as given (its unit length is the
 * caller's).  h has H entries and is updated in place. */
void oracle_steer(double* h, const float* v, int H) {
    double dot = 0.0;
    for (int c = 0; c < H; c++) dot += h[c] * (double)v[c];
    for (int c = 0; c < H; c++) h[c] -= dot * (double)v[c];
}

/* One MoE layer for the tokens listed in `tokens` (all T when tokens == NULL).
 *  x        [T][H] bf16 bits          W [E][H] fp32, b [E] fp32 or NULL
 *  arena    n_slots * slot_bytes       slot_table [L][E] int32
 *  steer    [H] fp32 unit direction removed from each output row before its
 *           rounding (oracle_steer), or NULL
 *  out      [T][H] bf16 bits (rows of listed tokens written)
 *  out_f64  [T][H] fp64 before rounding, optional
 *  idx, w   [T][k] routing of the listed tokens, optional
 * Returns ORC_ERR_SLOT when a selected expert has no valid slot (it then
 * contributes 0), ORC_ERR_ARG on bad arguments, else ORC_OK. */
int oracle_moe_layer(const orc_desc* d, const uint8_t* arena, const int32_t* slot_table,
                     int L, int layer, const uint16_t* x, int T, const float* W, const float* b,
                     int E, int k, int residual, const float* steer, uint16_t* out, double* out_f64,
                     int32_t* idx_out, double* w_out, const int32_t* tokens, int n_tokens) {
    if (!d || !arena || !slot_table || !x || !W || !out) return ORC_ERR_ARG;
    if (layer < 0 || layer >= L || k < 1 || k > E || T < 0) return ORC_ERR_ARG;
    int H = d->H;
    int nt = tokens ? n_tokens : T;
    int64_t npair = (int64_t)nt * k;
    double* logit = (double*)malloc(sizeof(double) * (size_t)E * (nt ? nt : 1));
    uint16_t* xs = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)H * (nt ? nt : 1));
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(npair ? npair : 1));
    double* w = (double*)malloc(sizeof(double) * (size_t)(npair ? npair : 1));
    double* y = (double*)malloc(sizeof(double) * (size_t)H * (npair ? npair : 1));
    int bad_slot = 0;
    for (int i = 0; i < nt; i++) {
        int t = tokens ? tokens[i] : i;
        memcpy(xs + (int64_t)i * H, x + (int64_t)t * H, sizeof(uint16_t) * H);
    }
    oracle_router_logits(xs, nt, H, W, b, E, logit);
    oracle_topk(logit, nt, E, k, idx, w);

    /* every (token, slot j) pair's expert output, independently */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:bad_slot)
    for (int64_t p = 0; p < npair; p++) {
        int i = (int)(p / k);
        double* yp = y + p * H;
        int32_t s = slot_table[(int64_t)layer * E + idx[p]];
        if (s < 0 || s >= d->n_slots) {
            for (int c = 0; c < H; c++) yp[c] = 0.0;
            bad_slot = 1;
            continue;
        }
        double* xd = (double*)malloc(sizeof(double) * H);
        for (int c = 0; c < H; c++) xd[c] = oracle_bf16_to_double(xs[(int64_t)i * H + c]);
        oracle_expert_ffn(arena + (int64_t)s * d->slot_bytes, d, xd, yp, NULL);
        free(xd);
    }
    double* row = (double*)malloc(sizeof(double) * H);
    for (int i = 0; i < nt; i++) {
        int t = tokens ? tokens[i] : i;
        for (int c = 0; c < H; c++) {
            double acc = 0.0;
            for (int j = 0; j < k; j++) acc += w[(int64_t)i * k + j] * y[((int64_t)i * k + j) * H + c];
            row[c] = residual ? oracle_bf16_to_double(xs[(int64_t)i * H + c]) + acc : acc;
        }
        if (steer) oracle_steer(row, steer, H);
        for (int c = 0; c < H; c++) {
            if (out_f64) out_f64[(int64_t)t * H + c] = row[c];
            out[(int64_t)t * H + c] = oracle_double_to_bf16(row[c]);
        }
        if (idx_out) memcpy(idx_out + (int64_t)t * k, idx + (int64_t)i * k, sizeof(int32_t) * k);
        if (w_out) memcpy(w_out + (int64_t)t * k, w + (int64_t)i * k, sizeof(double) * k);
    }
    free(logit); free(xs); free(idx); free(w); free(y); free(row);
    return bad_slot ? ORC_ERR_SLOT : ORC_OK;
}

/* ---------------------------------------------------------------- threads */

/* Threads of the parallel loops over tokens and pairs (a timing control:
 * every value is computed by one thread in the same order either way). */
void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
