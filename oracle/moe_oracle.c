/*
 * moe_oracle.c -- plain fp64 CPU oracle of the routed Mixture-of-Experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file defines what the layer computes so that the
 * CUDA path can be checked against it.  Only the tests, the package entry's smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * table or constant with the CUDA library, and the CUDA library never calls it.
 *
 * Sources (page title, section):
 *  [P1] "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速" -- section "稀疏在哪裡：397B 參數、
 *       17B 啟動": 512 routed experts, top-10 chosen by softmax probability, plus one
 *       shared expert that runs for every token whatever the routing says.
 *  [P1] same page, section "Kernel 手術台：RPA、Grouped GEMM v2、GDN 融合": the expert FFN is
 *       a SwiGLU (gate and up projections, then down) over FP8 weights quantised with
 *       512-element sub-channels.
 *  [P1] same page, section "數值驗證：省下來的效能有沒有偷跑": the lowered path is audited
 *       against a high-precision reference; the gating weights must not deviate.
 *  [P2] "TPU推理外部化全面加速：InferenceX首份第三方性能數據發布" -- section "优化 MoE 路由与
 *       专家内核": tokens are gathered into contiguous per-expert groups; the sort key packs
 *       (expert id, token index); the combine is an un-permute weighted by the top-k weights.
 *  [P3] the NVIDIA model/hardware co-design commentary -- section "讀的時候記得這是廠商文":
 *       NVFP4 keeps two levels of scale factors.
 *  [P4] "设计 AI 芯片的硬件与软件" -- section "数值格式，或如何制造便宜的脉动阵列": FP8 means the
 *       E4M3 and E5M2 formats; products are accumulated at higher precision.
 *  [P5] "Flash-Next 在 GPU 上到底在算什麼" -- section "① 專家 FFN": each expert computes
 *       input x matrix A -> activation -> x matrix B, with 4/8-bit weights dequantised
 *       to 16-bit before the multiply-adds.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  R1/R2  top-k ties: equal logits -> the lower expert index wins; the k chosen experts
 *         are ordered by (logit descending, index ascending).
 *  R3     p_hat = softmax over the k selected logits (= full softmax renormalised over top-k).
 *  R4     permutation order = assignments sorted by the key (expert, token) ascending.
 *  R5/R6  activation quantiser per (row, 512-block): s = fl32(amax / 448), q = e4m3(fl32(x/s));
 *         amax == 0 -> s = 1, q = 0.
 *  R7     activations are quantised for every FP8 layer.
 *  R8     the shared expert has no gate; its output is added with weight 1.
 *  R9     gate is the first projection, up the second; h = silu(G) * U.
 *  R10    h is rounded to fp32 then quantised with the R5/R6 rule per 512-block of I.
 *  R10a   the h codes (bf16 values for 4-bit layers) that another valid fp32 evaluation of
 *         G and U could also produce: see the rounding budget before orc_h_window.
 *  R11    4-bit layers keep activations in bf16: h is rounded to bf16 (RNE).
 *  R12    outputs are summed in fp64 here and rounded to bf16 (RNE) once.
 *  R13    e4m3 = OCP FP8 E4M3: bias 7, no infinities, max finite 448, subnormal step 2^-9,
 *         round-to-nearest-even, finite values beyond 448 saturate to 448.
 *  R14    int4 weights are symmetric two's-complement nibbles, the even K index in the
 *         low nibble; the weight is q * s with one bf16 s per (row, 128-element K group).
 *  R20    MXFP4 weights ([P4] same section: MXFP4 spends 4.25 bits per number, i.e. one
 *         8-bit scale per 32 four-bit values) follow the OCP Microscaling format: each
 *         nibble is an E2M1 value (S.EE.M, bias 1, exponent field 0 = 0.M, no inf/NaN,
 *         largest 6), the even K index in the low nibble; each (row, 32-element K block)
 *         has one E8M0 byte c, the scale 2^(c-127) (c = 255 is NaN).  The weight is
 *         e2m1 * 2^(c-127); activations and h stay bf16 as in R11 (the same page calls
 *         4-bit activations far harder than 4-bit weights).
 *  R21    NVFP4 weights ([P3] section "讀的時候記得這是廠商文": NVFP4 reaches near-8-bit accuracy
 *         at 4-bit speed through two levels of scale factors): E2M1 nibbles as in R20; one
 *         E4M3 byte (R13) per (row, 16-element K block); one fp32 tensor scale per weight
 *         matrix (per expert and projection).  The weight is e2m1 * e4m3(s) * t; activations
 *         and h stay bf16.
 *
 * Every sum below is written out in the order the definition states; nothing is blocked,
 * fused or reordered beyond it.  Build: gcc -O2 -fno-fast-math -ffp-contract=off.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_FP8_SC512 1
#define ORC_INT4_G128 2
#define ORC_MXFP4_G32 3
#define ORC_NVFP4_G16 4

typedef struct {
    int T, H, E, I, k, Is; /* Is = 0: no shared expert */
    int wfmt;              /* ORC_FP8_SC512, ORC_INT4_G128, ORC_MXFP4_G32 or ORC_NVFP4_G16 */
} orc_dims;

typedef struct {
    /* FP8: codes [E,I,H], [E,I,H], [E,H,I]; scales fp32 [E,I,nb(H)], [E,I,nb(H)], [E,H,nb(I)]
     * int4: packed bytes [E,I,H/2], [E,I,H/2], [E,H,I/2]; scales bf16 [E,I,H/128] ...
     * MXFP4: packed bytes as int4; scales E8M0 bytes [E,I,H/32], [E,I,H/32], [E,H,I/32]
     * NVFP4: packed bytes as int4; scales E4M3 bytes [E,I,H/16], [E,I,H/16], [E,H,I/16] */
    const uint8_t *w_gate, *w_up, *w_down;
    const void *s_gate, *s_up, *s_down;
    /* shared expert, same formats with E = 1 and I -> Is (NULL when Is == 0) */
    const uint8_t *ws_gate, *ws_up, *ws_down;
    const void *ss_gate, *ss_up, *ss_down;
    /* NVFP4 tensor scales: fp32 [E] per projection, [1] for the shared expert (else NULL) */
    const float *t_gate, *t_up, *t_down;
    const float *ts_gate, *ts_up, *ts_down;
} orc_weights;

/* ------------------------------------------------------------------------------------ */
/* number formats                                                                       */
/* ------------------------------------------------------------------------------------ */

/* E4M3 decode from the format definition (R13): S.EEEE.MMM, bias 7; exponent field 0 is
 * subnormal (0.MMM x 2^-6); S.1111.111 is NaN; there is no infinity. */
double orc_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* E4M3 encode of an fp32 value, round-to-nearest-even with saturation of finite values
 * (R13).  Works on the exact value in fp64: the quantum of the binade is 2^(e-3) for
 * normal numbers (2^-6 <= |x|) and 2^-9 below, and rint() rounds half to even under the
 * default rounding mode. */
uint8_t orc_e4m3_encode(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(xf) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(xf)) return 0x7F;
    if (a > 448.0) a = 448.0; /* finite values and +-inf saturate to the largest finite */
    double quantum;
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);
    } else {
        int e2;
        frexp(a, &e2); /* a = f * 2^e2 with f in [0.5, 1): leading bit weight 2^(e2-1) */
        quantum = ldexp(1.0, (e2 - 1) - 3);
    }
    double r = rint(a / quantum) * quantum; /* exact: a/quantum and the product are exact */
    if (r > 448.0) r = 448.0;               /* cannot happen after the clamp, kept for clarity */
    /* encode r: exponent field 0 holds 0.MMM x 2^-6, field E >= 1 holds 1.MMM x 2^(E-7) */
    int code;
    if (r < ldexp(1.0, -6)) {
        code = (int)(r / ldexp(1.0, -9)); /* 0..7, exact */
    } else {
        int e2;
        double f = frexp(r, &e2); /* r = f * 2^e2, f in [0.5, 1) */
        int lead = e2 - 1;
        int mant = (int)((2.0 * f - 1.0) * 8.0); /* exact: r has at most 4 significant bits */
        code = ((lead + 7) << 3) | mant;
    }
    return (uint8_t)(sign | code);
}

void orc_e4m3_encode_n(int n, const float *x, uint8_t *q)
{
    for (int i = 0; i < n; ++i) q[i] = orc_e4m3_encode(x[i]);
}

/* E2M1 decode from the format definition (R20): S.EE.M, exponent bias 1; exponent field 0
 * holds 0.M (so 0 or 0.5); field E >= 1 holds 1.M x 2^(E-1). */
double orc_e2m1_decode(int nib)
{
    int sign = (nib >> 3) & 1;
    int e = (nib >> 1) & 3;
    int m = nib & 1;
    double v = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return sign ? -v : v;
}

/* E8M0 decode (R20): the byte is a biased exponent, 2^(c-127); 255 is NaN. */
double orc_e8m0_decode(uint8_t c)
{
    if (c == 255) return NAN;
    return ldexp(1.0, (int)c - 127);
}

double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp64 -> bf16 with one round-to-nearest-even (no double rounding through fp32).
 * bf16 carries 8 significant bits and fp32's exponent range; its subnormal step is 2^-133. */
uint16_t orc_double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    int neg = signbit(x) ? 1 : 0;
    double a = fabs(x);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        int e2;
        frexp(a, &e2);
        int lead = e2 - 1; /* exponent of the leading bit */
        if (lead < -126) lead = -126;
        double quantum = ldexp(1.0, lead - 7);
        r = rint(a / quantum) * quantum;
    }
    uint16_t bits;
    if (r >= ldexp(1.0, 128)) {
        bits = 0x7F80; /* overflow to infinity */
    } else {
        float f = (float)r; /* exact: r has at most 8 significant bits */
        uint32_t u;
        memcpy(&u, &f, 4);
        bits = (uint16_t)(u >> 16);
    }
    return neg ? (uint16_t)(bits | 0x8000) : bits;
}

/* ------------------------------------------------------------------------------------ */
/* A1: route -- [P1] top-k by softmax probability; R1-R3                                 */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    float v;
    int e;
} orc_cand;

static int orc_cand_cmp(const void *pa, const void *pb)
{
    const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->e < b->e) ? -1 : (a->e > b->e);
}

/* One token: sort all E logits by (value desc, index asc), keep the first k; p_hat is the
 * softmax over those k logits in fp64.  Selection uses the fp32 logits themselves: exp is
 * monotone, so the top-k by probability is the top-k by logit. */
static void orc_route_token(int E, int k, const float *L, int32_t *idx, double *w)
{
    orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)E);
    for (int e = 0; e < E; ++e) {
        c[e].v = L[e];
        c[e].e = e;
    }
    qsort(c, (size_t)E, sizeof(orc_cand), orc_cand_cmp);
    double lmax = (double)c[0].v;
    double denom = 0.0;
    for (int j = 0; j < k; ++j) denom += exp((double)c[j].v - lmax);
    for (int j = 0; j < k; ++j) {
        idx[j] = c[j].e;
        w[j] = exp((double)c[j].v - lmax) / denom;
    }
    free(c);
}

int orc_route(int T, int E, int k, const float *logits, int32_t *topk_idx, double *topk_w)
{
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    for (int t = 0; t < T; ++t)
        orc_route_token(E, k, logits + (size_t)t * E, topk_idx + (size_t)t * k,
                        topk_w + (size_t)t * k);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* router logits -- [P5] ② (the router is a dense 16-bit layer): logits = x . W_r^T       */
/* ------------------------------------------------------------------------------------ */

/* logits[t, e] = sum_i x[t, i] * w[e, i] with bf16 inputs, in fp64 (each product of two bf16
 * values is exact; the sum of H of them is exact to ~1e-16 relative).  bound[t, e] (optional)
 * receives sum_i |x[t, i] * w[e, i]|, the scale of the rounding error any other summation
 * order can make. */
int orc_router_logits(int T, int H, int E, const uint16_t *x, const uint16_t *w, double *logits, double *bound)
{
    if (T < 0 || H < 1 || E < 1) return -1;
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, mag = 0.0;
            for (int i = 0; i < H; ++i) {
                double p = orc_bf16_to_double(x[(size_t)t * H + i]) * orc_bf16_to_double(w[(size_t)e * H + i]);
                acc += p;
                mag += fabs(p);
            }
            logits[(size_t)t * E + e] = acc;
            if (bound) bound[(size_t)t * E + e] = mag;
        }
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* A3: permute -- [P2] contiguous per-expert groups, packed (expert, token) sort key; R4  */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    int32_t e, t, j;
} orc_asg;

static int orc_asg_cmp(const void *pa, const void *pb)
{
    const orc_asg *a = (const orc_asg *)pa, *b = (const orc_asg *)pb;
    if (a->e != b->e) return (a->e < b->e) ? -1 : 1;
    if (a->t != b->t) return (a->t < b->t) ? -1 : 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

/* counts[e] = number of assignments to e; offsets = exclusive prefix sum (E+1 entries);
 * perm_tok[r] = token of the r-th assignment in (expert, token) order; pos[t*k+j] = row r of
 * assignment (t, j). */
int orc_permute(int T, int E, int k, const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                int32_t *perm_tok, int32_t *pos)
{
    size_t n = (size_t)T * (size_t)k;
    orc_asg *a = (orc_asg *)malloc(sizeof(orc_asg) * (n ? n : 1));
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[(size_t)t * k + j];
            if (e < 0 || e >= E) {
                free(a);
                return -1;
            }
            counts[e] += 1;
            a[(size_t)t * k + j].e = e;
            a[(size_t)t * k + j].t = t;
            a[(size_t)t * k + j].j = j;
        }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    qsort(a, n, sizeof(orc_asg), orc_asg_cmp);
    for (size_t r = 0; r < n; ++r) {
        perm_tok[r] = a[r].t;
        pos[(size_t)a[r].t * k + a[r].j] = (int32_t)r;
    }
    free(a);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* A2: FP8 512-sub-channel quantiser -- [P1] Kernel section; R5, R6, R13                  */
/* ------------------------------------------------------------------------------------ */

/* x: K fp32 values of one row; q: K e4m3 codes; s: ceil(K/512) fp32 scales.  The last
 * block may be shorter than 512. */
void orc_quant_row_fp8(int K, const float *x, uint8_t *q, float *s)
{
    int nb = (K + 511) / 512;
    for (int kb = 0; kb < nb; ++kb) {
        int i0 = kb * 512, i1 = (kb + 1) * 512 < K ? (kb + 1) * 512 : K;
        float amax = 0.0f;
        for (int i = i0; i < i1; ++i) {
            float a = fabsf(x[i]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            s[kb] = 1.0f;
            for (int i = i0; i < i1; ++i) q[i] = 0;
            continue;
        }
        volatile float sc = amax / 448.0f; /* fp32 IEEE division */
        s[kb] = sc;
        for (int i = i0; i < i1; ++i) {
            volatile float v = x[i] / sc; /* fp32 IEEE division */
            q[i] = orc_e4m3_encode(v);
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* A4-A6: one expert on one activation row, FP8 weights -- [P1] Kernel section, [P5] ①    */
/* ------------------------------------------------------------------------------------ */

static double orc_dec_tab[256];
static double orc_e2m1_tab[16], orc_e8m0_tab[256]; /* memoised R20 decodes */
static pthread_once_t orc_tab_once = PTHREAD_ONCE_INIT;
static void orc_tab_init(void)
{
    for (int c = 0; c < 256; ++c) orc_dec_tab[c] = orc_e4m3_decode((uint8_t)c);
    for (int c = 0; c < 16; ++c) orc_e2m1_tab[c] = orc_e2m1_decode(c);
    for (int c = 0; c < 256; ++c) orc_e8m0_tab[c] = orc_e8m0_decode((uint8_t)c);
}

/* y[n] = sum_kb sx[kb] * sw[n,kb] * sum_{i in kb} dec(qx[i]) * dec(qw[n,i]),  n < N.
 * The inner sum is exact in fp64 (each product of two e4m3 values has at most 8
 * significant bits and lies in [2^-18, 2^18)).  yabs (optional) receives
 * sum_kb |sx[kb] * sw[n,kb]| * sum_{i in kb} |dec(qx[i]) * dec(qw[n,i])|, the magnitude that
 * scales the rounding error of any fp32 evaluation of the same sum (R10a). */
static void orc_proj_fp8(int N, int K, const uint8_t *qx, const float *sx, const uint8_t *qw,
                         const float *sw, double *y, double *yabs)
{
    int nb = (K + 511) / 512;
    for (int n = 0; n < N; ++n) {
        const uint8_t *row = qw + (size_t)n * K;
        double acc = 0.0, mag = 0.0;
        for (int kb = 0; kb < nb; ++kb) {
            int i0 = kb * 512, i1 = (kb + 1) * 512 < K ? (kb + 1) * 512 : K;
            double part = 0.0, apart = 0.0;
            for (int i = i0; i < i1; ++i) {
                double pr = orc_dec_tab[qx[i]] * orc_dec_tab[row[i]];
                part += pr;
                apart += fabs(pr);
            }
            acc += (double)sx[kb] * (double)sw[(size_t)n * nb + kb] * part;
            mag += fabs((double)sx[kb] * (double)sw[(size_t)n * nb + kb]) * apart;
        }
        y[n] = acc;
        if (yabs) yabs[n] = mag;
    }
}

static double orc_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

static double orc_silu(double z) { return z * (1.0 / (1.0 + exp(-z))); }

/* ---- R10a: the h codes (or bf16 values) that are not unique ------------------------------
 *
 * The layer holds h in fp32 and then rounds it to a coarse format (e4m3 codes per 512-block
 * for FP8 layers, bf16 for 4-bit layers).  fp32 results of G and U obtained in any other
 * valid summation order (R17) differ from the exact values, and where the exact h lies close
 * to a rounding boundary of the coarse format, the other side of that boundary is an equally
 * valid result.  The oracle bounds, per element, how far a valid fp32 h can lie from the
 * exact one, lists every coarse value a valid h can round to, and reports for each output
 * the largest move those alternatives allow through the down projection (the envelope).
 *
 * Rounding budget (a reading; the pages give none).  A valid fp32 G lies within
 * ORC_ROUND * S of the exact G, S = the sum of |every product| of the dot product (after its
 * scales), ORC_ROUND = 2^-22.  Measured on the B200 for this layer's projections (the fp32
 * outputs of the FP8 and int4 tensor-core GEMMs against exact fp64 sums of the same operands,
 * 2^18 elements each): the largest error was 1.0 * 2^-24 * S, so the budget keeps a margin of
 * 4.  (The worst case for a chain of n additions is about n * 2^-24 * S, hundreds of times
 * more; it would make almost every h code ambiguous.)  h = silu(G) * U then moves by at most
 *   dh = |silu'(G)| |U| dG + |silu(G)| dU + dG dU + (2^-20 + |G| 2^-23) |h|,
 * the last term covering the fp32 exponential (its argument's rounding grows with |G|), the
 * division, the product and the final fp32 rounding of h. */

#define ORC_U22 (1.0 / 4194304.0)
#define ORC_U23 (1.0 / 8388608.0)
#define ORC_ROUND ORC_U22

/* The largest distance of a valid fp32 h from the exact silu(G) * U, given the distances
 * dG, dU of valid fp32 G, U from the exact G, U. */
static double orc_h_window(double G, double U, double dG, double dU)
{
    double sg = orc_sigmoid(G);
    double dsilu = sg * (1.0 + G * (1.0 - sg));
    double h = G * sg * U;
    return fabs(dsilu) * fabs(U) * dG + fabs(G * sg) * dU + dG * dU +
           (1.0 / 1048576.0 + fabs(G) * ORC_U23) * fabs(h);
}

/* e4m3 code of the double v rounded toward -inf (dir < 0) or +inf (dir > 0) to fp32 first,
 * so that no value of the interval it bounds escapes through that rounding. */
static uint8_t orc_e4m3_encode_dir(double v, int dir)
{
    float f = (float)v;
    if (dir > 0 && (double)f < v) f = nextafterf(f, INFINITY);
    if (dir < 0 && (double)f > v) f = nextafterf(f, -INFINITY);
    return orc_e4m3_encode(f);
}

/* FP8 layers.  h: the exact h rounded to fp32 as the layer holds it; dh: its window; qh, sh:
 * the oracle's codes and scales (R10).  Per 512-block of I with scale s (amax / 448): a valid
 * amax differs by at most the block's largest window, so a valid scale differs by at most
 * that over amax (relative) plus one rounding; a valid h / s then lies in
 * v +- (|v| (ds/s + 2^-22) + dh / s) around the oracle's v = h / s, and every code between
 * the roundings of the two ends is valid (rounding is monotone).  D_i = the largest
 * |dec(code) - dec(q_i)| * s over those codes; env[n] += D_i * |Wd[n, i] * sd[n, block(i)]|. */
static void orc_h_ambiguity(int H, int I, const float *h, const double *dh, const uint8_t *qh,
                            const float *sh, const uint8_t *wd, const float *sd, double *env)
{
    int nbI = (I + 511) / 512;
    for (int kb = 0; kb < nbI; ++kb) {
        int i0 = kb * 512, i1 = (kb + 1) * 512 < I ? (kb + 1) * 512 : I;
        double amax = 0.0, dmax = 0.0;
        for (int i = i0; i < i1; ++i) {
            if (fabs((double)h[i]) > amax) amax = fabs((double)h[i]);
            if (dh[i] > dmax) dmax = dh[i];
        }
        if (amax == 0.0 && dmax == 0.0) continue;
        double s = (double)sh[kb];
        double ds = amax > 0.0 ? dmax / amax + ORC_U23 : 1.0;
        for (int i = i0; i < i1; ++i) {
            double v = (double)h[i] / s;
            double half = fabs(v) * (ds + ORC_U22) + dh[i] / s;
            if (half == 0.0) continue;
            double q = orc_dec_tab[qh[i]];
            double lo = orc_dec_tab[orc_e4m3_encode_dir(v - half, -1)];
            double hi = orc_dec_tab[orc_e4m3_encode_dir(v + half, +1)];
            double D = fabs(lo - q) > fabs(hi - q) ? fabs(lo - q) : fabs(hi - q);
            if (D == 0.0) continue;
            D *= s;
            for (int n = 0; n < H; ++n) {
                double wv = orc_dec_tab[wd[(size_t)n * I + i]] * (double)sd[(size_t)n * nbI + i / 512];
                env[n] += D * fabs(wv);
            }
        }
    }
}

/* One FP8 expert (gate/up/down already offset to that expert) on one quantised row.
 * h_out (optional, I values) receives h rounded to fp32 before its quantisation (R10);
 * env (optional, H values) is cleared and receives the R10a envelope. */
static void orc_expert_fp8(int H, int I, const uint8_t *qx, const float *sx, const uint8_t *wg,
                           const float *sg, const uint8_t *wu, const float *su, const uint8_t *wd,
                           const float *sd, double *y, float *h_out, double *env)
{
    double *G = (double *)malloc(sizeof(double) * (size_t)I);
    double *U = (double *)malloc(sizeof(double) * (size_t)I);
    double *SG = (double *)malloc(sizeof(double) * (size_t)I);
    double *SU = (double *)malloc(sizeof(double) * (size_t)I);
    float *h = (float *)malloc(sizeof(float) * (size_t)I);
    uint8_t *qh = (uint8_t *)malloc((size_t)I);
    float *sh = (float *)malloc(sizeof(float) * (size_t)((I + 511) / 512));
    orc_proj_fp8(I, H, qx, sx, wg, sg, G, SG);
    orc_proj_fp8(I, H, qx, sx, wu, su, U, SU);
    for (int n = 0; n < I; ++n) h[n] = (float)(orc_silu(G[n]) * U[n]);
    if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)I);
    orc_quant_row_fp8(I, h, qh, sh);
    orc_proj_fp8(H, I, qh, sh, wd, sd, y, NULL);
    if (env) {
        const double c = ORC_ROUND;
        double *dh = SG; /* reused: the window of each h */
        for (int n = 0; n < I; ++n) dh[n] = orc_h_window(G[n], U[n], c * SG[n], c * SU[n]);
        for (int n = 0; n < H; ++n) env[n] = 0.0;
        orc_h_ambiguity(H, I, h, dh, qh, sh, wd, sd, env);
    }
    free(G);
    free(U);
    free(SG);
    free(SU);
    free(h);
    free(qh);
    free(sh);
}

/* ------------------------------------------------------------------------------------ */
/* 4-bit experts -- [P5] ① (4-bit weights dequantised to 16-bit, then multiply-add);        */
/* R11, R14 (int4), R20 (MXFP4)                                                         */
/* ------------------------------------------------------------------------------------ */

static int orc_nib(const uint8_t *packed_row, int i)
{
    int b = packed_row[i >> 1];
    int v = (i & 1) ? (b >> 4) : (b & 0xF);
    return v >= 8 ? v - 16 : v;
}

/* The raw nibble (0..15) of element i of a packed row. */
static int orc_nib_raw(const uint8_t *packed_row, int i)
{
    int b = packed_row[i >> 1];
    return (i & 1) ? (b >> 4) : (b & 0xF);
}

/* Weight [n, i] of a 4-bit [N, K] matrix without its tensor scale: int4 q * s (R14),
 * e2m1 * 2^(c-127) (R20) or e2m1 * e4m3(s) (R21). */
static double orc_w4(int wfmt, int K, const uint8_t *qw, const void *sw, int n, int i)
{
    const uint8_t *row = qw + (size_t)n * (K / 2);
    if (wfmt == ORC_NVFP4_G16) {
        const uint8_t *sc = (const uint8_t *)sw;
        return orc_e2m1_tab[orc_nib_raw(row, i)] * orc_dec_tab[sc[(size_t)n * (K / 16) + i / 16]];
    }
    if (wfmt == ORC_MXFP4_G32) {
        const uint8_t *sc = (const uint8_t *)sw;
        return orc_e2m1_tab[orc_nib_raw(row, i)] * orc_e8m0_tab[sc[(size_t)n * (K / 32) + i / 32]];
    }
    const uint16_t *sc = (const uint16_t *)sw;
    return (double)orc_nib(row, i) * orc_bf16_to_double(sc[(size_t)n * (K / 128) + i / 128]);
}

/* The scale array of expert e of a 4-bit [E, N, K] weight set. */
static const void *orc_w4_scales(int wfmt, const void *sw, size_t e, int N, int K)
{
    if (wfmt == ORC_NVFP4_G16) return (const uint8_t *)sw + e * (size_t)N * (size_t)(K / 16);
    if (wfmt == ORC_MXFP4_G32) return (const uint8_t *)sw + e * (size_t)N * (size_t)(K / 32);
    return (const uint16_t *)sw + e * (size_t)N * (size_t)(K / 128);
}

/* y[n] = sum_i a[i] * (W[n, i] * t)  with a in fp64 (bf16 values, exact); t is the matrix's
 * tensor scale (1 except for NVFP4).  Every product is exact in fp64.  yabs (optional)
 * receives sum_i |a[i] * W[n, i] * t| (R10a). */
static void orc_proj_w4(int wfmt, int N, int K, const double *a, const uint8_t *qw, const void *sw,
                        double t, double *y, double *yabs)
{
    for (int n = 0; n < N; ++n) {
        double acc = 0.0, mag = 0.0;
        for (int i = 0; i < K; ++i) {
            double pr = a[i] * (orc_w4(wfmt, K, qw, sw, n, i) * t);
            acc += pr;
            mag += fabs(pr);
        }
        y[n] = acc;
        if (yabs) yabs[n] = mag;
    }
}

/* R10a for 4-bit layers: h is rounded to bf16 (R11).  A valid fp32 h lies in
 * hx +- dh around the exact hx; every bf16 value between the roundings of the two ends is a
 * valid result (rounding is monotone).  D_i = the largest |that value - bf16(hx_i)|;
 * env[n] += D_i * |W[n, i] * td| (td: the down matrix's tensor scale, 1 except for NVFP4). */
static void orc_h_ambiguity_bf16(int wfmt, int H, int I, const double *hx, const double *dh,
                                 const uint8_t *wd, const void *sd, double td, double *env)
{
    for (int i = 0; i < I; ++i) {
        if (dh[i] == 0.0) continue;
        double b = orc_bf16_to_double(orc_double_to_bf16(hx[i]));
        double lo = orc_bf16_to_double(orc_double_to_bf16(hx[i] - dh[i]));
        double hi = orc_bf16_to_double(orc_double_to_bf16(hx[i] + dh[i]));
        double D = fabs(lo - b) > fabs(hi - b) ? fabs(lo - b) : fabs(hi - b);
        if (D == 0.0) continue;
        for (int n = 0; n < H; ++n) env[n] += D * fabs(orc_w4(wfmt, I, wd, sd, n, i) * td);
    }
}

/* tg, tu, td: the three matrices' tensor scales (1 except for NVFP4). */
static void orc_expert_w4(int wfmt, int H, int I, const double *x, const uint8_t *wg, const void *sg,
                          double tg, const uint8_t *wu, const void *su, double tu, const uint8_t *wd,
                          const void *sd, double td, double *y, double *h_out, double *env)
{
    double *G = (double *)malloc(sizeof(double) * (size_t)I);
    double *U = (double *)malloc(sizeof(double) * (size_t)I);
    double *SG = (double *)malloc(sizeof(double) * (size_t)I);
    double *SU = (double *)malloc(sizeof(double) * (size_t)I);
    double *hx = (double *)malloc(sizeof(double) * (size_t)I);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    orc_proj_w4(wfmt, I, H, x, wg, sg, tg, G, SG);
    orc_proj_w4(wfmt, I, H, x, wu, su, tu, U, SU);
    for (int n = 0; n < I; ++n) {
        hx[n] = orc_silu(G[n]) * U[n];
        h[n] = orc_bf16_to_double(orc_double_to_bf16(hx[n]));
    }
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
    orc_proj_w4(wfmt, H, I, h, wd, sd, td, y, NULL);
    if (env) {
        const double c = ORC_ROUND;
        double *dh = SG; /* reused: the window of each h */
        for (int n = 0; n < I; ++n) dh[n] = orc_h_window(G[n], U[n], c * SG[n], c * SU[n]);
        for (int n = 0; n < H; ++n) env[n] = 0.0;
        orc_h_ambiguity_bf16(wfmt, H, I, hx, dh, wd, sd, td, env);
    }
    free(G);
    free(U);
    free(SG);
    free(SU);
    free(hx);
    free(h);
}

/* ------------------------------------------------------------------------------------ */
/* the layer on a chosen set of tokens -- route, quantise, experts, weighted combine       */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    const orc_dims *d;
    const orc_weights *w;
    const uint16_t *x;    /* [T,H] bf16 bits */
    const float *logits;  /* [T,E] */
    const int32_t *sel;   /* tokens to evaluate */
    int n_sel;
    double *out;          /* [n_sel,H] fp64 before the final rounding */
    uint16_t *out_bf16;   /* [n_sel,H] */
    double *amb;          /* [n_sel,H] R10a envelope, or NULL */
    int next;             /* next index of sel to take (guarded by mu) */
    pthread_mutex_t mu;
} orc_job;

static void orc_layer_token(const orc_dims *d, const orc_weights *w, const uint16_t *xrow,
                            const float *lrow, double *out, double *amb)
{
    int H = d->H, I = d->I, E = d->E, k = d->k, Is = d->Is;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    double *p = (double *)malloc(sizeof(double) * (size_t)k);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    double *env = amb ? (double *)malloc(sizeof(double) * (size_t)H) : NULL;
    orc_route_token(E, k, lrow, idx, p);
    for (int n = 0; n < H; ++n) out[n] = 0.0;
    if (amb)
        for (int n = 0; n < H; ++n) amb[n] = 0.0;

    if (d->wfmt == ORC_FP8_SC512) {
        int nbH = (H + 511) / 512, nbI = (I + 511) / 512, nbIs = (Is + 511) / 512;
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        uint8_t *qx = (uint8_t *)malloc((size_t)H);
        float *sx = (float *)malloc(sizeof(float) * (size_t)nbH);
        for (int i = 0; i < H; ++i) xf[i] = (float)orc_bf16_to_double(xrow[i]);
        orc_quant_row_fp8(H, xf, qx, sx);
        const float *sg = (const float *)w->s_gate, *su = (const float *)w->s_up,
                    *sd = (const float *)w->s_down;
        for (int j = 0; j < k; ++j) {
            size_t e = (size_t)idx[j];
            orc_expert_fp8(H, I, qx, sx, w->w_gate + e * I * H, sg + e * I * nbH,
                           w->w_up + e * I * H, su + e * I * nbH, w->w_down + e * H * I,
                           sd + e * H * nbI, y, NULL, env);
            for (int n = 0; n < H; ++n) out[n] += p[j] * y[n];
            if (amb)
                for (int n = 0; n < H; ++n) amb[n] += p[j] * env[n];
        }
        if (Is > 0) {
            orc_expert_fp8(H, Is, qx, sx, w->ws_gate, (const float *)w->ss_gate, w->ws_up,
                           (const float *)w->ss_up, w->ws_down, (const float *)w->ss_down, y, NULL,
                           env);
            for (int n = 0; n < H; ++n) out[n] += y[n];
            if (amb)
                for (int n = 0; n < H; ++n) amb[n] += env[n];
        }
        (void)nbIs;
        free(xf);
        free(qx);
        free(sx);
    } else {
        double *xd = (double *)malloc(sizeof(double) * (size_t)H);
        for (int i = 0; i < H; ++i) xd[i] = orc_bf16_to_double(xrow[i]);
        const int f = d->wfmt;
        const int nv = f == ORC_NVFP4_G16;
        for (int j = 0; j < k; ++j) {
            size_t e = (size_t)idx[j];
            orc_expert_w4(f, H, I, xd, w->w_gate + e * I * (H / 2), orc_w4_scales(f, w->s_gate, e, I, H),
                          nv ? (double)w->t_gate[e] : 1.0, w->w_up + e * I * (H / 2),
                          orc_w4_scales(f, w->s_up, e, I, H), nv ? (double)w->t_up[e] : 1.0,
                          w->w_down + e * H * (I / 2), orc_w4_scales(f, w->s_down, e, H, I),
                          nv ? (double)w->t_down[e] : 1.0, y, NULL, env);
            for (int n = 0; n < H; ++n) out[n] += p[j] * y[n];
            if (amb)
                for (int n = 0; n < H; ++n) amb[n] += p[j] * env[n];
        }
        if (Is > 0) {
            orc_expert_w4(f, H, Is, xd, w->ws_gate, w->ss_gate, nv ? (double)w->ts_gate[0] : 1.0, w->ws_up,
                          w->ss_up, nv ? (double)w->ts_up[0] : 1.0, w->ws_down, w->ss_down,
                          nv ? (double)w->ts_down[0] : 1.0, y, NULL, env);
            for (int n = 0; n < H; ++n) out[n] += y[n];
            if (amb)
                for (int n = 0; n < H; ++n) amb[n] += env[n];
        }
        free(xd);
    }
    free(idx);
    free(p);
    free(y);
    free(env);
}

static void *orc_worker(void *arg)
{
    orc_job *jb = (orc_job *)arg;
    pthread_once(&orc_tab_once, orc_tab_init);
    for (;;) {
        pthread_mutex_lock(&jb->mu);
        int i = jb->next++;
        pthread_mutex_unlock(&jb->mu);
        if (i >= jb->n_sel) break;
        int t = jb->sel[i];
        const orc_dims *d = jb->d;
        double *o = jb->out + (size_t)i * d->H;
        orc_layer_token(d, jb->w, jb->x + (size_t)t * d->H, jb->logits + (size_t)t * d->E, o,
                        jb->amb ? jb->amb + (size_t)i * d->H : NULL);
        for (int n = 0; n < d->H; ++n) jb->out_bf16[(size_t)i * d->H + n] = orc_double_to_bf16(o[n]);
    }
    return NULL;
}

/* The layer output for the tokens sel[0..n_sel): out (fp64, before rounding) and out_bf16
 * (R12); amb (optional) receives the R10a envelope per output (zero where no h value sits
 * at a rounding boundary).  Tokens are
 * independent, so any subset is exact; nthreads workers take tokens in turn.  Returns 0, or
 * -1 on bad dims. */
int orc_layer(const orc_dims *d, const orc_weights *w, const uint16_t *x, const float *logits,
              int n_sel, const int32_t *sel, double *out, uint16_t *out_bf16, double *amb,
              int nthreads)
{
    if (d->E < 1 || d->k < 1 || d->k > d->E || d->H < 1 || d->I < 1 || d->Is < 0) return -1;
    if (d->wfmt < ORC_FP8_SC512 || d->wfmt > ORC_NVFP4_G16) return -1;
    if (d->wfmt == ORC_NVFP4_G16 &&
        (!w->t_gate || !w->t_up || !w->t_down || (d->Is > 0 && (!w->ts_gate || !w->ts_up || !w->ts_down))))
        return -1;
    if (d->wfmt != ORC_FP8_SC512 && (d->H % 128 || d->I % 128 || d->Is % 128)) return -1;
    for (int i = 0; i < n_sel; ++i)
        if (sel[i] < 0 || sel[i] >= d->T) return -1;
    pthread_once(&orc_tab_once, orc_tab_init);
    orc_job jb;
    jb.d = d;
    jb.w = w;
    jb.x = x;
    jb.logits = logits;
    jb.sel = sel;
    jb.n_sel = n_sel;
    jb.out = out;
    jb.out_bf16 = out_bf16;
    jb.amb = amb;
    jb.next = 0;
    pthread_mutex_init(&jb.mu, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, orc_worker, &jb);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&jb.mu);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* single steps, exposed for step-by-step parity                                        */
/* ------------------------------------------------------------------------------------ */

/* x (bf16 bits) rows -> quantised rows, FP8 layers (A2). */
void orc_quant_rows_bf16(int R, int K, const uint16_t *x, uint8_t *q, float *s)
{
    int nb = (K + 511) / 512;
    float *xf = (float *)malloc(sizeof(float) * (size_t)K);
    for (int r = 0; r < R; ++r) {
        for (int i = 0; i < K; ++i) xf[i] = (float)orc_bf16_to_double(x[(size_t)r * K + i]);
        orc_quant_row_fp8(K, xf, q + (size_t)r * K, s + (size_t)r * nb);
    }
    free(xf);
}

/* One FP8 expert on one quantised row: y (H values, fp64) and h (I values, fp32 before
 * its quantisation). */
void orc_expert_fp8_row(int H, int I, const uint8_t *qx, const float *sx, const uint8_t *wg,
                        const float *sg, const uint8_t *wu, const float *su, const uint8_t *wd,
                        const float *sd, double *y, float *h)
{
    pthread_once(&orc_tab_once, orc_tab_init);
    orc_expert_fp8(H, I, qx, sx, wg, sg, wu, su, wd, sd, y, h, NULL);
}

/* One 4-bit expert (int4, MXFP4 or NVFP4; t = the tensor scales, 1 unless NVFP4) on one bf16
 * row: y (H values) and h (I values, bf16-rounded). */
void orc_expert_w4_row(int wfmt, int H, int I, const uint16_t *x, const uint8_t *wg, const void *sg,
                       const uint8_t *wu, const void *su, const uint8_t *wd, const void *sd, const double *t,
                       double *y, double *h)
{
    pthread_once(&orc_tab_once, orc_tab_init);
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    for (int i = 0; i < H; ++i) xd[i] = orc_bf16_to_double(x[i]);
    orc_expert_w4(wfmt, H, I, xd, wg, sg, t[0], wu, su, t[1], wd, sd, t[2], y, h, NULL);
    free(xd);
}

/* One int4 expert on one bf16 row: y (H values) and h (I values, bf16-rounded). */
void orc_expert_int4_row(int H, int I, const uint16_t *x, const uint8_t *wg, const uint16_t *sg,
                         const uint8_t *wu, const uint16_t *su, const uint8_t *wd,
                         const uint16_t *sd, double *y, double *h)
{
    const double ones[3] = {1.0, 1.0, 1.0};
    orc_expert_w4_row(ORC_INT4_G128, H, I, x, wg, sg, wu, su, wd, sd, ones, y, h);
}
