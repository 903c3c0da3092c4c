/*
 * moe_oracle.c -- plain, slow, single-threaded CPU oracle for the MoE
 * routing hot path: top-k gate -> layout -> dispatch -> combine.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is
 * compared against.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no source, header,
 * table or constant generator with the CUDA library, and the CUDA library
 * never calls it.
 *
 * Every routine states the definition it follows.  The pages cited are:
 *   [pplx]   "Efficient and portable mixture-of-experts communication"
 *            (Perplexity Research blog), sections Introduction, Dispatch,
 *            Combine.
 *   [EPv2]   "DeepSeek releases the open-source DeepEP library for MoE
 *            training and inference" (hi.news.hada.io summary of DeepEP V2),
 *            section "training / prefill / decoding usage patterns".
 *   [EPv1]   "DeepSeek, DeepEP 오픈소스 공개" (GeekNews), sections
 *            "Topic Body" and "성능 / 일반 커널" (normal kernels).
 *   [TK]     "DeepSeek Tile-Kernels / DeepEP V2" (deepinsightai.io), list
 *            "Funktionen der DeepSeek-Tile-Kernel".
 * Where the pages leave a rule open, the reading taken is written beside it.
 *
 * Arithmetic: fp32 with explicit rounding steps (compile with
 * -ffp-contract=off so no multiply-add is fused behind our back).  The pages
 * fix fp32 accumulation for combine and BF16 storage; gate selections and
 * FP8 codes are integers decided by floating point, so they are decided in
 * the kernels' precision (fp32) with one exp written out from its
 * definition below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_INVALID_ARG 1
#define ORC_ERR_BAD_INDEX 4

#define GATE_SOFTMAX 0
#define GATE_SOFTMAX_RENORM 1
#define GATE_SIGMOID_GROUP 2

#define DT_BF16 0
#define DT_FP8_E4M3 1
#define DT_FP8_E4M3_TOKEN 2
#define DT_MXFP8_E4M3 3
#define DT_NVFP4 4
#define DT_E5M6 5
#define DT_FP8_UE8M0 6

/* ------------------------------------------------------------------ */
/* bit helpers                                                         */
/* ------------------------------------------------------------------ */
static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bfloat16 -> fp32 is exact: the bf16 pattern is the top half of the fp32. */
float oracle_f32_from_bf16(uint16_t h) { return bits_f32(((uint32_t)h) << 16); }

/* fp32 -> bfloat16, round to nearest, ties to even (IEEE 754 default
 * rounding applied to an 8-bit significand).  NaN stays a quiet NaN. */
uint16_t oracle_bf16_from_f32(float f)
{
    uint32_t u = f32_bits(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    /* exactly representable, below half, half (tie), above half */
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------ */
/* exp written out from its definition (Cody & Waite argument reduction,
 * Taylor series).  e^y = 2^n * e^r with n = nearest integer to y/ln2 and
 * r = y - n*ln2, |r| <= ln2/2; e^r = sum_{i=0..7} r^i / i! by Horner.
 * ln2 is split into a head with 16 significant bits (so n*head is exact for
 * |n| < 256) and a tail; both terms are removed with one fused multiply-add
 * each.  The input is clamped to [-87, 88] so that 2^n stays a normal
 * float: below -87 the result saturates at about e^-87.
 * The constants are the mathematical ones rounded to fp32:
 *   log2(e), ln2 head = floor(ln2 * 2^16) / 2^16, ln2 tail = ln2 - head,
 *   1/i! for i = 2..7.                                                  */
/* ------------------------------------------------------------------ */
float oracle_dexp(float y)
{
    const float log2e = 1.44269504088896340736f;
    const float ln2_head = 45426.0f / 65536.0f; /* 0.693145751953125 */
    const float ln2_tail = 1.42860682030941723212e-6f;
    const float c2 = 1.0f / 2.0f, c3 = 1.0f / 6.0f, c4 = 1.0f / 24.0f;
    const float c5 = 1.0f / 120.0f, c6 = 1.0f / 720.0f, c7 = 1.0f / 5040.0f;

    /* clamp to [-87, 88] by comparisons: any NaN input (outside the gate's
     * contract; quiet or signalling) fails the first test and becomes -87,
     * so the routine is defined on every fp32 pattern */
    if (!(y > -87.0f)) y = -87.0f;
    if (y > 88.0f) y = 88.0f;
    float t = y * log2e;        /* one fp32 rounding */
    float n = rintf(t);         /* nearest integer, ties to even */
    float r = fmaf(-n, ln2_head, y);
    r = fmaf(-n, ln2_tail, r);
    float p = c7;
    p = fmaf(p, r, c6);
    p = fmaf(p, r, c5);
    p = fmaf(p, r, c4);
    p = fmaf(p, r, c3);
    p = fmaf(p, r, c2);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;            /* in [-126, 127] */
    float two_n = bits_f32((uint32_t)(ni + 127) << 23);
    return p * two_n;           /* one fp32 rounding */
}

/* logistic sigmoid 1 / (1 + e^-x), each operation rounded once in fp32 */
float oracle_sigmoid(float x)
{
    float e = oracle_dexp(-x);
    float d = 1.0f + e;
    return 1.0f / d;
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (OCP 8-bit floating point, "E4M3": 1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 holds the subnormals
 * m * 2^-9; S.1111.111 is NaN; no infinities; largest finite 448 =
 * S.1111.110).  Encoding rounds to nearest, ties to even mantissa, and
 * saturates every finite value (and infinity) beyond 448 to +-448.       */
/* ------------------------------------------------------------------ */
float oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

uint8_t oracle_e4m3_encode(float f)
{
    uint8_t sign = (f32_bits(f) >> 31) ? 0x80 : 0x00;
    if (isnan(f)) return sign | 0x7F;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;          /* saturate */
    if (a < ldexp(1.0, -6)) {                    /* subnormal range */
        double q = a * 512.0;                    /* in units of 2^-9, exact */
        double m = nearbyint(q);                 /* ties to even */
        return sign | (uint8_t)m;                /* m == 8 is the code of 2^-6 */
    }
    int ex;
    frexp(a, &ex);                               /* a = fr * 2^ex, fr in [0.5,1) */
    int unb = ex - 1;                            /* a in [2^unb, 2^(unb+1)) */
    double q = (ldexp(a, -unb) - 1.0) * 8.0;     /* mantissa in eighths, exact */
    double m = nearbyint(q);                     /* ties to even */
    int biased = unb + 7;
    if (m == 8.0) { m = 0.0; biased += 1; }
    if (biased > 15 || (biased == 15 && m == 7.0)) return sign | 0x7E;
    return sign | (uint8_t)((biased << 3) | (int)m);
}

void oracle_e4m3_encode_array(const float* in, uint8_t* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(in[i]);
}

/* ------------------------------------------------------------------ */
/* E5M6, a 12-bit float.  [TK] lists E5M6 conversion without a definition.
 * Reading: the IEEE-style binary format with 1 sign bit, 5 exponent bits
 * (bias 15) and 6 fraction bits -- FP16 with its 4 lowest fraction bits
 * dropped: exponent field 0 holds the subnormals m * 2^-20, field 31 the
 * infinities and NaNs, largest finite 2^15 * (1 + 63/64) = 65024.
 * Encoding rounds to nearest, ties to even, and saturates every finite value
 * (and infinity) beyond 65024 to +-65024, as the FP8 encoders here do.
 * Two codes are packed in three bytes, little endian: code 2i in bits
 * 0..11, code 2i+1 in bits 12..23.                                      */
/* ------------------------------------------------------------------ */
float oracle_e5m6_decode(uint16_t c)
{
    int s = (c >> 11) & 1, e = (c >> 6) & 31, m = c & 63;
    double v;
    if (e == 31) return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0) v = ldexp((double)m, -20);
    else v = ldexp(1.0 + m / 64.0, e - 15);
    return (float)(s ? -v : v);
}

uint16_t oracle_e5m6_encode(float f)
{
    uint16_t sign = (f32_bits(f) >> 31) ? 0x800 : 0x000;
    if (isnan(f)) return sign | 0x7FF;
    double a = fabs((double)f);
    if (a >= 65024.0) return sign | 0x7BF;       /* saturate */
    if (a < ldexp(1.0, -14)) {                   /* subnormal range */
        double m = nearbyint(a * 1048576.0);     /* units of 2^-20, exact; ties to even */
        return sign | (uint16_t)m;               /* m == 64 is the code of 2^-14 */
    }
    int ex;
    frexp(a, &ex);
    int unb = ex - 1;                            /* a in [2^unb, 2^(unb+1)) */
    double q = (ldexp(a, -unb) - 1.0) * 64.0;    /* fraction in 64ths, exact */
    double m = nearbyint(q);                     /* ties to even */
    int biased = unb + 15;
    if (m == 64.0) { m = 0.0; biased += 1; }
    if (biased >= 31) return sign | 0x7BF;
    return sign | (uint16_t)((biased << 6) | (int)m);
}

/* ------------------------------------------------------------------ */
/* FP4 E2M1 (the OCP MX element type that NVFP4 uses: 1 sign, 2 exponent
 * bits with bias 1, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
 * no infinity, no NaN).  Encoding rounds to nearest, ties to the even
 * mantissa, and saturates beyond 6 (infinity too) to +-6.  NaN inputs are
 * outside the contract.                                                */
/* ------------------------------------------------------------------ */
float oracle_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (float)(s ? -v : v);
}

uint8_t oracle_e2m1_encode(float f)
{
    uint8_t sign = (f32_bits(f) >> 31) ? 0x8 : 0x0;
    double a = fabs((double)f);
    if (!(a < 6.0)) return sign | 0x7;           /* saturate (and NaN) */
    if (a < 2.0) return sign | (uint8_t)nearbyint(a * 2.0);      /* steps of 0.5: codes 0..4 */
    if (a < 4.0) return sign | (uint8_t)(2 + nearbyint(a));      /* 2, 3, 4 -> codes 4, 5, 6 */
    return sign | (uint8_t)(4 + nearbyint(a * 0.5));              /* 4, 6 -> codes 6, 7 */
}

void oracle_dexp_array(const float* in, float* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_dexp(in[i]);
}

void oracle_sigmoid_array(const float* in, float* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = oracle_sigmoid(in[i]);
}

/* ------------------------------------------------------------------ */
/* top-k selection: k passes of arg-max over the candidates.  Order is by
 * key descending; equal keys go to the lower index (the reading taken for
 * ties).  -0.0 and +0.0 compare equal.  Output is in selection order.    */
/* ------------------------------------------------------------------ */
static int better(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

static void select_topk(const float* key, const unsigned char* cand, int n,
                        int k, int* sel)
{
    unsigned char* taken = (unsigned char*)calloc((size_t)n, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int i = 0; i < n; ++i) {
            if (!cand[i] || taken[i]) continue;
            if (best < 0 || better(key[i], i, key[best], best)) best = i;
        }
        sel[j] = best;
        if (best >= 0) taken[best] = 1;
    }
    free(taken);
}

/* ------------------------------------------------------------------ */
/* Gate.  [pplx] Introduction: the router turns the logits into a
 * probability distribution, the top-K experts are picked and the output is
 * the average of their outputs weighted by the router's probabilities.
 * [TK] list, "Gating" and "MoE-Routing ... Gewichtsnormalisierung": top-k
 * selection and scoring, with weight normalisation.
 *
 *  GATE_SOFTMAX:         p = softmax(logits); w_j = p_{sel j}.
 *  GATE_SOFTMAX_RENORM:  w_j = p_{sel j} / sum_{j'} p_{sel j'}.
 *  GATE_SIGMOID_GROUP:   DeepSeek-V3 group-limited gating, which [EPv1]
 *     Topic Body names and whose run uses top-4 groups and top-8 experts
 *     ([EPv1] normal kernels).  Reading taken: s = sigmoid(logit); the
 *     experts split into n_groups consecutive groups; a group's score is
 *     the sum of its group_topn largest s (added in descending order);
 *     the topk_groups best groups are kept; the top-k experts by s among
 *     the kept groups are chosen; w_j = s_{sel j} / sum_{j'} s_{sel j'}.
 *
 *  softmax: m = max logit; e_i = exp(l_i - m); Z = sum of e_i in ascending
 *  expert order; p_i = e_i / Z.  Softmax is strictly increasing, so the
 *  top-k of p is the top-k of the logits: selection uses the logits.
 *  Every sum over selected experts runs in slot order (selection order).
 */
/* ------------------------------------------------------------------ */
int oracle_topk_gate(const float* logits, int N, int E, int k, int kind,
                     int n_groups, int topk_groups, int group_topn,
                     int32_t* topk_idx, float* topk_w)
{
    if (N < 0 || E < 1 || k < 1 || k > E) return ORC_ERR_INVALID_ARG;
    if (kind == GATE_SIGMOID_GROUP) {
        if (n_groups < 1 || E % n_groups != 0) return ORC_ERR_INVALID_ARG;
        int eg = E / n_groups;
        if (topk_groups < 1 || topk_groups > n_groups) return ORC_ERR_INVALID_ARG;
        if (group_topn < 1 || group_topn > eg) return ORC_ERR_INVALID_ARG;
        if (topk_groups * eg < k) return ORC_ERR_INVALID_ARG;
    } else if (kind != GATE_SOFTMAX && kind != GATE_SOFTMAX_RENORM) {
        return ORC_ERR_INVALID_ARG;
    }
    float* key = (float*)malloc(sizeof(float) * (size_t)E);
    float* val = (float*)malloc(sizeof(float) * (size_t)E);
    unsigned char* cand = (unsigned char*)malloc((size_t)E);
    int* sel = (int*)malloc(sizeof(int) * (size_t)E);
    float* gscore = (float*)malloc(sizeof(float) * (size_t)(n_groups > 0 ? n_groups : 1));
    unsigned char* gcand = (unsigned char*)malloc((size_t)(n_groups > 0 ? n_groups : 1));
    int* gsel = (int*)malloc(sizeof(int) * (size_t)(n_groups > 0 ? n_groups : 1));

    for (int t = 0; t < N; ++t) {
        const float* l = logits + (size_t)t * E;
        int32_t* oi = topk_idx + (size_t)t * k;
        float* ow = topk_w + (size_t)t * k;
        if (kind == GATE_SOFTMAX || kind == GATE_SOFTMAX_RENORM) {
            float m = l[0];
            for (int i = 1; i < E; ++i) if (l[i] > m) m = l[i];
            float z = 0.0f;
            for (int i = 0; i < E; ++i) {
                val[i] = oracle_dexp(l[i] - m);
                z = z + val[i];
            }
            for (int i = 0; i < E; ++i) { key[i] = l[i]; cand[i] = 1; }
            select_topk(key, cand, E, k, sel);
            float ps = 0.0f;
            for (int j = 0; j < k; ++j) {
                float p = val[sel[j]] / z;
                oi[j] = sel[j];
                ow[j] = p;
                ps = (j == 0) ? p : ps + p;
            }
            if (kind == GATE_SOFTMAX_RENORM)
                for (int j = 0; j < k; ++j) ow[j] = ow[j] / ps;
        } else {
            int eg = E / n_groups;
            for (int i = 0; i < E; ++i) val[i] = oracle_sigmoid(l[i]);
            for (int g = 0; g < n_groups; ++g) {
                const float* gv = val + (size_t)g * eg;
                for (int i = 0; i < eg; ++i) cand[i] = 1;
                select_topk(gv, cand, eg, group_topn, gsel);
                float sum = gv[gsel[0]];
                for (int j = 1; j < group_topn; ++j) sum = sum + gv[gsel[j]];
                gscore[g] = sum;
                gcand[g] = 1;
            }
            select_topk(gscore, gcand, n_groups, topk_groups, gsel);
            for (int i = 0; i < E; ++i) cand[i] = 0;
            for (int j = 0; j < topk_groups; ++j)
                for (int i = 0; i < eg; ++i) cand[(size_t)gsel[j] * eg + i] = 1;
            select_topk(val, cand, E, k, sel);
            float ss = val[sel[0]];
            for (int j = 1; j < k; ++j) ss = ss + val[sel[j]];
            for (int j = 0; j < k; ++j) {
                oi[j] = sel[j];
                ow[j] = val[sel[j]] / ss;
            }
        }
    }
    free(key); free(val); free(cand); free(sel);
    free(gscore); free(gcand); free(gsel);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Layout.  [EPv2] usage patterns: the handle carries the routing metadata
 * combine needs and the per-expert received-token counts that size the
 * grouped GEMM.  [pplx] Dispatch: the receiver packs tokens into one
 * contiguous per-expert buffer and keeps, per received row, the source
 * token so that combine knows where each row goes back; the order on the
 * pages is not fixed -- the reading taken is ascending token id (then
 * top-k slot) inside each expert.  [pplx] Sharding: experts are sharded
 * over EP ranks; rank r owns experts [r*E/R, (r+1)*E/R).
 *
 * Entries equal to -1 are masked slots (no expert); any other id outside
 * [0, E) is skipped and reported as ORC_ERR_BAD_INDEX.  Skipped entries get
 * token_slot = -1 and fill the tail rows [expert_offset[E], N*k) of the
 * receive buffer, whose slot_token is -1.
 *
 * expert_count[e]   = #{(t,j) : idx[t,j] = e}
 * expert_offset[e]  = sum_{e' < e} expert_count[e'],  e = 0..E
 * token_slot[t,j]   = expert_offset[e] + #{(t',j') before (t,j) in
 *                     row-major order with idx[t',j'] = e}
 * slot_token[s]     = t for s = token_slot[t,j]; -1 for the tail rows
 * rank_count[r]     = sum of expert_count over rank r's experts
 * rank_offset[r]    = expert_offset[r*E/R], rank_offset[R] = expert_offset[E]
 * rank_tokens[r]    = #{t : some j has idx[t,j] in rank r}            */
/* ------------------------------------------------------------------ */
int oracle_get_layout(const int32_t* topk_idx, int N, int k, int E, int R,
                      int32_t* expert_count, int32_t* expert_offset,
                      int32_t* rank_count, int32_t* rank_offset,
                      int32_t* rank_tokens, int32_t* token_slot,
                      int32_t* slot_token)
{
    if (N < 0 || k < 1 || E < 1 || R < 1 || E % R != 0) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    int epr = E / R;
    int64_t S = (int64_t)N * k;
    for (int e = 0; e < E; ++e) expert_count[e] = 0;
    for (int64_t i = 0; i < S; ++i) {
        int32_t e = topk_idx[i];
        if (e >= 0 && e < E) expert_count[e] += 1;
        else if (e != -1) status = ORC_ERR_BAD_INDEX;
    }
    expert_offset[0] = 0;
    for (int e = 0; e < E; ++e) expert_offset[e + 1] = expert_offset[e] + expert_count[e];

    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = expert_offset[e];
    int64_t tail = expert_offset[E];
    for (int t = 0; t < N; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t i = (int64_t)t * k + j;
            int32_t e = topk_idx[i];
            if (e >= 0 && e < E) {
                int32_t s = cursor[e]++;
                token_slot[i] = s;
                slot_token[s] = t;
            } else {
                token_slot[i] = -1;
                slot_token[tail++] = -1;
            }
        }
    }
    free(cursor);

    for (int r = 0; r < R; ++r) {
        int32_t c = 0;
        for (int e = r * epr; e < (r + 1) * epr; ++e) c += expert_count[e];
        rank_count[r] = c;
        rank_offset[r] = expert_offset[r * epr];
        rank_tokens[r] = 0;
    }
    rank_offset[R] = expert_offset[E];
    for (int t = 0; t < N; ++t) {
        for (int r = 0; r < R; ++r) {
            int hit = 0;
            for (int j = 0; j < k; ++j) {
                int32_t e = topk_idx[(int64_t)t * k + j];
                if (e >= 0 && e < E && e / epr == r) hit = 1;
            }
            rank_tokens[r] += hit;
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* GEMM-aligned layout.  [EPv2] mentions a "new GEMM layout" without
 * defining it; the reading taken: each expert's rows start at a multiple of
 * `align` so a grouped GEMM can tile every expert by align rows.
 *   expert_offset[e] = sum_{e' < e} round_up(expert_count[e'], align)
 *   token_slot[t,j]  = expert_offset[e] + (rank of (t,j) inside e, as before)
 *   slot_token[s]    = the token of row s, -1 for every other row in
 *                      [0, num_rows) (padding, masked tail, spare capacity)
 *   rank_offset[r]   = expert_offset[r*E/R]; rank_count[r] = the rows of rank
 *                      r's region, padding included.
 * num_rows must be at least expert_offset[E] + (masked entries); N*k +
 * E*(align-1) always suffices.  align = 1 is the packed layout.          */
/* ------------------------------------------------------------------ */
int oracle_get_layout_aligned(const int32_t* topk_idx, int N, int k, int E, int R,
                              int align, int64_t num_rows, int32_t* expert_count,
                              int32_t* expert_offset, int32_t* rank_count,
                              int32_t* rank_offset, int32_t* rank_tokens,
                              int32_t* token_slot, int32_t* slot_token)
{
    if (N < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || align < 1) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    int epr = E / R;
    int64_t S = (int64_t)N * k;
    int64_t invalid = 0;
    for (int e = 0; e < E; ++e) expert_count[e] = 0;
    for (int64_t i = 0; i < S; ++i) {
        int32_t e = topk_idx[i];
        if (e >= 0 && e < E) expert_count[e] += 1;
        else { invalid += 1; if (e != -1) status = ORC_ERR_BAD_INDEX; }
    }
    expert_offset[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t padded = (expert_count[e] + align - 1) / align * align;
        expert_offset[e + 1] = expert_offset[e] + padded;
    }
    if ((int64_t)expert_offset[E] + invalid > num_rows) return ORC_ERR_INVALID_ARG;
    for (int64_t s = 0; s < num_rows; ++s) slot_token[s] = -1;
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = expert_offset[e];
    for (int t = 0; t < N; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t i = (int64_t)t * k + j;
            int32_t e = topk_idx[i];
            if (e >= 0 && e < E) {
                int32_t s = cursor[e]++;
                token_slot[i] = s;
                slot_token[s] = t;
            } else {
                token_slot[i] = -1;
            }
        }
    }
    free(cursor);
    for (int r = 0; r < R; ++r) {
        rank_offset[r] = expert_offset[r * epr];
        rank_count[r] = expert_offset[(r + 1) * epr] - expert_offset[r * epr];
        rank_tokens[r] = 0;
    }
    rank_offset[R] = expert_offset[E];
    for (int t = 0; t < N; ++t) {
        for (int r = 0; r < R; ++r) {
            int hit = 0;
            for (int j = 0; j < k; ++j) {
                int32_t e = topk_idx[(int64_t)t * k + j];
                if (e >= 0 && e < E && e / epr == r) hit = 1;
            }
            rank_tokens[r] += hit;
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* Dispatch.  [pplx] Dispatch: each token's activations (with block scaling
 * factors when quantised) are sent to every expert it was routed to and
 * unpacked into one contiguous buffer per expert.  [EPv2] usage patterns:
 * BF16 and FP8 inputs.  [TK] list, "Quantisierung ... pro Block".
 *
 * BF16: recv_x[token_slot[t,j], :] = x[t, :] for every valid slot.
 * FP8, per token t and block b of 128 channels (reading taken for the
 * block size and format: e4m3 with one fp32 scale per 128 channels):
 *   amax  = max_c |x[t,c]|                       (exact)
 *   inv   = 448 / amax,  scale = amax / 448      (IEEE fp32 divisions)
 *   q_c   = e4m3(x[t,c] * inv)  (fp32 product, RNE, saturating);
 *           an element equal to zero encodes as zero with its sign, which
 *           is what the product gives whenever inv is finite and defines
 *           the all-zero block (amax = 0, scale = 0).
 * The same codes and scale go to every slot of the token.
 * A slot outside [-1, num_rows) is skipped and reported (num_rows = N*k
 * for the packed layout, more for a padded one).                        */
/* ------------------------------------------------------------------ */
/* Quantisation variants ([TK] list, "Quantisierung ... pro Token, pro Block"):
 *  DT_FP8_E4M3_TOKEN: one fp32 scale per token row: amax over the whole row,
 *      scale = amax / 448, codes e4m3(x * (448 / amax)) as for the blocks;
 *      recv_scale is [S, 1].
 *  DT_MXFP8_E4M3: OCP Microscaling MXFP8 -- blocks of 32 elements share the
 *      scale X = 2^e with e = floor(log2(amax)) - 8 (8 = the largest exponent
 *      of e4m3), clamped to [-127, 127]; elements e4m3(x * 2^-e), RNE,
 *      saturating to 448 (x * 2^-e can reach 511.x); the scale is stored as
 *      the E8M0 byte e + 127 in recv_scale viewed as uint8 [S, H/32].  An
 *      all-zero block stores e = -127 (byte 0) and zero codes.               */
static int floor_log2_pos(float a)   /* a > 0, finite: exact from the bits */
{
    uint32_t u = f32_bits(a);
    int ex = (int)((u >> 23) & 0xFF);
    if (ex > 0) return ex - 127;
    int m = (int)(u & 0x7FFFFF), hb = 22;
    while (!((m >> hb) & 1)) --hb;
    return hb - 149;                 /* subnormal: 2^(hb - 23) * 2^-126 */
}

static int oracle_dispatch_variant(const uint16_t* x, int N, int H, int k,
                                   const int32_t* token_slot, int64_t num_rows, int dtype,
                                   uint8_t* recv_x, float* recv_scale)
{
    int status = ORC_OK;
    int64_t S = num_rows;
    int nb = dtype == DT_FP8_E4M3_TOKEN ? 1 : (dtype == DT_FP8_UE8M0 ? H / 128 : H / 32);
    uint8_t* q = (uint8_t*)malloc((size_t)H);
    float* fsc = (float*)malloc(sizeof(float));
    uint8_t* esc = (uint8_t*)malloc((size_t)nb);
    for (int t = 0; t < N; ++t) {
        const uint16_t* xr = x + (size_t)t * H;
        if (dtype == DT_FP8_E4M3_TOKEN) {
            float amax = 0.0f;
            for (int c = 0; c < H; ++c) {
                float v = fabsf(oracle_f32_from_bf16(xr[c]));
                if (v > amax) amax = v;
            }
            float inv = 448.0f / amax;
            fsc[0] = amax / 448.0f;
            for (int c = 0; c < H; ++c) {
                float v = oracle_f32_from_bf16(xr[c]);
                q[c] = oracle_e4m3_encode((v == 0.0f) ? v : v * inv);
            }
        } else if (dtype == DT_FP8_UE8M0) {
            /* 1x128 blocks, power-of-two scale 2^e with e = ceil(log2(amax/448)):
             * the smallest power of two not below the fp32 quotient */
            for (int b = 0; b < nb; ++b) {
                float amax = 0.0f;
                for (int c = b * 128; c < (b + 1) * 128; ++c) {
                    float v = fabsf(oracle_f32_from_bf16(xr[c]));
                    if (v > amax) amax = v;
                }
                int e = -127;
                if (amax > 0.0f) {
                    float qt = amax / 448.0f;
                    if (isinf(qt)) {
                        e = 127;   /* ceil(log2(+inf)) is +inf: clamped to the largest exponent */
                    } else {
                        int fe;
                        double fr = frexp((double)qt, &fe);     /* qt = fr * 2^fe, fr in [0.5, 1) */
                        e = (fr == 0.5) ? fe - 1 : fe;
                    }
                }
                if (e < -127) e = -127;
                if (e > 127) e = 127;
                esc[b] = (uint8_t)(e + 127);
                float down = ldexpf(1.0f, -e);    /* e <= 120 for bf16 input: 2^-e is a normal float */
                for (int c = b * 128; c < (b + 1) * 128; ++c) {
                    float v = oracle_f32_from_bf16(xr[c]);
                    q[c] = oracle_e4m3_encode((v == 0.0f) ? v : v * down);
                }
            }
        } else {
            for (int b = 0; b < nb; ++b) {
                float amax = 0.0f;
                for (int c = b * 32; c < (b + 1) * 32; ++c) {
                    float v = fabsf(oracle_f32_from_bf16(xr[c]));
                    if (v > amax) amax = v;
                }
                int e = (amax > 0.0f) ? floor_log2_pos(amax) - 8 : -127;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
                esc[b] = (uint8_t)(e + 127);
                float down = ldexpf(1.0f, -e);    /* e <= 119 for bf16 input: 2^-e is a normal float */
                for (int c = b * 32; c < (b + 1) * 32; ++c) {
                    float v = oracle_f32_from_bf16(xr[c]);
                    q[c] = oracle_e4m3_encode((v == 0.0f) ? v : v * down);
                }
            }
        }
        for (int j = 0; j < k; ++j) {
            int32_t s = token_slot[(int64_t)t * k + j];
            if (s == -1) continue;
            if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }
            memcpy(recv_x + (size_t)s * H, q, (size_t)H);
            if (dtype == DT_FP8_E4M3_TOKEN) recv_scale[s] = fsc[0];
            else memcpy((uint8_t*)recv_scale + (size_t)s * nb, esc, (size_t)nb);
        }
    }
    free(q); free(fsc); free(esc);
    return status;
}

int oracle_dispatch_rows(const uint16_t* x, int N, int H, int k,
                         const int32_t* token_slot, int64_t num_rows, int dtype, void* recv_x,
                         float* recv_scale);
int oracle_dispatch(const uint16_t* x, int N, int H, int k,
                    const int32_t* token_slot, int dtype, void* recv_x,
                    float* recv_scale)
{
    return oracle_dispatch_rows(x, N, H, k, token_slot, (int64_t)N * k, dtype, recv_x, recv_scale);
}

/* the receive buffer holds num_rows rows (N*k for the packed layout) */
int oracle_dispatch_rows(const uint16_t* x, int N, int H, int k,
                         const int32_t* token_slot, int64_t num_rows, int dtype, void* recv_x,
                         float* recv_scale)
{
    if (N < 0 || H < 1 || k < 1) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_FP8_E4M3 && H % 128 != 0) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_MXFP8_E4M3 && H % 32 != 0) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_FP8_E4M3_TOKEN && H % 8 != 0) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_FP8_UE8M0 && H % 128 != 0) return ORC_ERR_INVALID_ARG;
    if ((dtype < DT_BF16 || dtype > DT_MXFP8_E4M3) && dtype != DT_FP8_UE8M0) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_FP8_E4M3_TOKEN || dtype == DT_MXFP8_E4M3 || dtype == DT_FP8_UE8M0)
        return oracle_dispatch_variant(x, N, H, k, token_slot, num_rows, dtype, (uint8_t*)recv_x,
                                       recv_scale);
    int status = ORC_OK;
    int64_t S = num_rows;
    int nb = H / 128;
    uint8_t* q = (uint8_t*)malloc((size_t)H);
    float* sc = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    for (int t = 0; t < N; ++t) {
        const uint16_t* xr = x + (size_t)t * H;
        if (dtype == DT_FP8_E4M3) {
            for (int b = 0; b < nb; ++b) {
                float amax = 0.0f;
                for (int c = b * 128; c < (b + 1) * 128; ++c) {
                    float v = fabsf(oracle_f32_from_bf16(xr[c]));
                    if (v > amax) amax = v;
                }
                float inv = 448.0f / amax;
                sc[b] = amax / 448.0f;
                for (int c = b * 128; c < (b + 1) * 128; ++c) {
                    float v = oracle_f32_from_bf16(xr[c]);
                    float p = (v == 0.0f) ? v : v * inv;
                    q[c] = oracle_e4m3_encode(p);
                }
            }
        }
        for (int j = 0; j < k; ++j) {
            int32_t s = token_slot[(int64_t)t * k + j];
            if (s == -1) continue;
            if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }
            if (dtype == DT_BF16) {
                uint16_t* dst = (uint16_t*)recv_x + (size_t)s * H;
                for (int c = 0; c < H; ++c) dst[c] = xr[c];
            } else {
                uint8_t* dst = (uint8_t*)recv_x + (size_t)s * H;
                for (int c = 0; c < H; ++c) dst[c] = q[c];
                for (int b = 0; b < nb; ++b) recv_scale[(size_t)s * nb + b] = sc[b];
            }
        }
    }
    free(q); free(sc);
    return status;
}

/* ------------------------------------------------------------------ */
/* Scale layouts for a grouped GEMM.  [EPv2] names "a new GEMM layout"
 * without defining it and [TK] lists batched transposes; neither fixes
 * where the receive scales go.  Reading: the same values in one of three
 * places, for scale (s, b) of receive row s and scale block b, with B
 * blocks per row (H/128 per-block FP8, 1 per-token FP8, H/32 MXFP8):
 *   ROW_MAJOR   element s*B + b: what dispatch writes by default.
 *   MN_MAJOR    element b*ld + s, ld = num_rows rounded up to 16 bytes of
 *               scales (4 fp32 or 16 E8M0 bytes): each block's scales are
 *               contiguous over the rows (the transposed, M-major scale
 *               operand of a grouped GEMM), each column 16-byte aligned.
 *   MMA_TILED   E8M0 only, B % 4 == 0: the order in which the block-scaled
 *               tensor-core MMA takes its scale factors.  Rows are padded to
 *               a multiple of 128; 128-row x 4-block atoms of 512 bytes are
 *               stored row-major over (s / 128, b / 4); inside an atom,
 *               row s and block b sit at byte
 *               (s mod 32)*16 + ((s mod 128) / 32)*4 + (b mod 4).
 *   MN_MAJOR_PACK4  one-byte scales of 1x128 blocks (UE8M0): four
 *               consecutive blocks of a row form one 32-bit word (block
 *               4j+i in byte i), and the words are MN-major -- word (s, j)
 *               at word index j*ld + s, ld = num_rows rounded up to 4 --
 *               the packed power-of-two scale operand of a 1x128-scaled
 *               FP8 GEMM.
 * Positions of rows that no token lands in are not written.            */
/* ------------------------------------------------------------------ */
#define SL_ROW_MAJOR 0
#define SL_MN_MAJOR 1
#define SL_MMA_TILED 2
#define SL_MN_MAJOR_PACK4 3

static int scale_blocks(int H, int dtype)
{
    if (dtype == DT_FP8_E4M3) return H / 128;
    if (dtype == DT_FP8_E4M3_TOKEN) return 1;
    if (dtype == DT_MXFP8_E4M3) return H / 32;
    if (dtype == DT_NVFP4) return H / 16;
    if (dtype == DT_FP8_UE8M0) return H / 128;
    return 0;
}

static int scale_elem_bytes(int dtype)
{
    return (dtype == DT_MXFP8_E4M3 || dtype == DT_NVFP4 || dtype == DT_FP8_UE8M0) ? 1 : 4;
}

static int64_t round_up64(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

/* elements the scale buffer holds in this layout; -1 where the layout does
 * not apply to the payload type */
int64_t oracle_scale_elems(int64_t num_rows, int H, int dtype, int layout)
{
    int B = scale_blocks(H, dtype);
    if (num_rows < 0 || B < 1) return -1;
    if (layout == SL_ROW_MAJOR) return num_rows * B;
    if (layout == SL_MN_MAJOR) return (int64_t)B * round_up64(num_rows, 16 / scale_elem_bytes(dtype));
    if (layout == SL_MMA_TILED && (dtype == DT_MXFP8_E4M3 || dtype == DT_NVFP4) && B % 4 == 0)
        return round_up64(num_rows, 128) * B;
    if (layout == SL_MN_MAJOR_PACK4 && dtype == DT_FP8_UE8M0)
        return (int64_t)((B + 3) / 4) * 4 * round_up64(num_rows, 4);
    return -1;
}

/* element index of scale (s, b); the layout must apply (see above) */
int64_t oracle_scale_index(int layout, int64_t num_rows, int H, int dtype, int64_t s, int b)
{
    int B = scale_blocks(H, dtype);
    if (layout == SL_MN_MAJOR) return (int64_t)b * round_up64(num_rows, 16 / scale_elem_bytes(dtype)) + s;
    if (layout == SL_MMA_TILED) {
        int64_t atom = (s / 128) * (B / 4) + b / 4;
        return atom * 512 + (s % 32) * 16 + ((s % 128) / 32) * 4 + b % 4;
    }
    if (layout == SL_MN_MAJOR_PACK4)   /* 32-bit words of 4 blocks, the words MN-major */
        return (int64_t)(b / 4) * 4 * round_up64(num_rows, 4) + s * 4 + b % 4;
    return s * B + b;
}

/* dispatch with the receive scales in `layout`: the row-major dispatch,
 * then every landed row's scales moved to their place */
int oracle_dispatch_scaled(const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                           int64_t num_rows, int dtype, int layout, void* recv_x,
                           void* recv_scale)
{
    if (layout == SL_ROW_MAJOR)
        return oracle_dispatch_rows(x, N, H, k, token_slot, num_rows, dtype, recv_x,
                                    (float*)recv_scale);
    if (oracle_scale_elems(num_rows, H, dtype, layout) < 0) return ORC_ERR_INVALID_ARG;
    int B = scale_blocks(H, dtype), es = scale_elem_bytes(dtype);
    unsigned char* rows = (unsigned char*)calloc((size_t)(num_rows > 0 ? num_rows : 1) * B, (size_t)es);
    int st = oracle_dispatch_rows(x, N, H, k, token_slot, num_rows, dtype, recv_x, (float*)rows);
    if (st != ORC_ERR_INVALID_ARG) {
        for (int64_t i = 0; i < (int64_t)N * k; ++i) {
            int64_t s = token_slot[i];
            if (s < 0 || s >= num_rows) continue;
            for (int b = 0; b < B; ++b)
                memcpy((unsigned char*)recv_scale + oracle_scale_index(layout, num_rows, H, dtype, s, b) * es,
                       rows + (s * B + b) * es, (size_t)es);
        }
    }
    free(rows);
    return st;
}

/* ------------------------------------------------------------------ */
/* E5M6 dispatch: every element of the token's row encoded on its own (no
 * scale), the packed row copied to each of the token's receive rows
 * (3H/2 bytes).  H % 32 == 0.                                           */
/* ------------------------------------------------------------------ */
int oracle_dispatch_e5m6(const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                         int64_t num_rows, uint8_t* recv_x)
{
    if (N < 0 || H < 32 || H % 32 != 0 || k < 1 || num_rows < 0) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    size_t rb = (size_t)H / 2 * 3;
    uint8_t* q = (uint8_t*)malloc(rb);
    for (int t = 0; t < N; ++t) {
        const uint16_t* xr = x + (size_t)t * H;
        for (int c = 0; c < H; c += 2) {
            uint32_t c0 = oracle_e5m6_encode(oracle_f32_from_bf16(xr[c]));
            uint32_t c1 = oracle_e5m6_encode(oracle_f32_from_bf16(xr[c + 1]));
            uint32_t w = c0 | (c1 << 12);
            q[c / 2 * 3 + 0] = (uint8_t)(w & 0xFF);
            q[c / 2 * 3 + 1] = (uint8_t)((w >> 8) & 0xFF);
            q[c / 2 * 3 + 2] = (uint8_t)((w >> 16) & 0xFF);
        }
        for (int j = 0; j < k; ++j) {
            int32_t s = token_slot[(int64_t)t * k + j];
            if (s == -1) continue;
            if (s < -1 || s >= num_rows) { status = ORC_ERR_BAD_INDEX; continue; }
            memcpy(recv_x + (size_t)s * rb, q, rb);
        }
    }
    free(q);
    return status;
}

/* ------------------------------------------------------------------ */
/* NVFP4 dispatch.  [EPv2] feature list (Hybrid-EP: NVFP4 support) and [TK]
 * (FP4 conversion) name the format without its rule.  Reading, per token t
 * (the per-token mode of [TK]), the two-level NVFP4 scaling with the
 * token's row in place of the tensor:
 *   amax_t = max_c |x[t,c]|,  g_t = amax_t / 2688 (448 * 6, the largest
 *            e4m3 times the largest e2m1): the row's fp32 scale,
 *   inv_t  = 2688 / amax_t,
 *   per block b of 16 channels: sb = e4m3((amax_b / 6) * inv_t) if
 *            amax_b > 0, else 0 (an unsigned e4m3 code),
 *   r_b    = inv_t / e4m3_value(sb),
 *   q_c    = e2m1(x_c * r_b)  (a zero keeps its sign, as in FP8),
 * every operation in fp32 rounded once; x is recovered as
 * e2m1_value(q) * e4m3_value(sb) * g_t.  Two codes per byte, channel 2i in
 * the low nibble.  Block scales (one byte per 16 channels) in any layout of
 * oracle_scale_index; the row scales fp32 [num_rows].  H % 64 == 0.    */
/* ------------------------------------------------------------------ */
int oracle_dispatch_nvfp4(const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                          int64_t num_rows, int layout, uint8_t* recv_x, uint8_t* block_scale,
                          float* row_scale)
{
    if (N < 0 || H < 64 || H % 64 != 0 || k < 1 || num_rows < 0) return ORC_ERR_INVALID_ARG;
    if (oracle_scale_elems(num_rows, H, DT_NVFP4, layout) < 0) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    int B = H / 16;
    uint8_t* q = (uint8_t*)malloc((size_t)H / 2);
    uint8_t* sb = (uint8_t*)malloc((size_t)B);
    for (int t = 0; t < N; ++t) {
        const uint16_t* xr = x + (size_t)t * H;
        float amax_t = 0.0f;
        for (int c = 0; c < H; ++c) {
            float v = fabsf(oracle_f32_from_bf16(xr[c]));
            if (v > amax_t) amax_t = v;
        }
        float g = amax_t / 2688.0f;
        float inv = 2688.0f / amax_t;
        for (int b = 0; b < B; ++b) {
            float amax_b = 0.0f;
            for (int c = b * 16; c < (b + 1) * 16; ++c) {
                float v = fabsf(oracle_f32_from_bf16(xr[c]));
                if (v > amax_b) amax_b = v;
            }
            float sbf = (amax_b / 6.0f) * inv;
            sb[b] = amax_b > 0.0f ? oracle_e4m3_encode(sbf) : 0;
            float r = inv / oracle_e4m3_decode(sb[b]);
            for (int c = b * 16; c < (b + 1) * 16; c += 2) {
                float v0 = oracle_f32_from_bf16(xr[c]), v1 = oracle_f32_from_bf16(xr[c + 1]);
                uint8_t lo = oracle_e2m1_encode(v0 == 0.0f ? v0 : v0 * r);
                uint8_t hi = oracle_e2m1_encode(v1 == 0.0f ? v1 : v1 * r);
                q[c / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
        for (int j = 0; j < k; ++j) {
            int32_t s = token_slot[(int64_t)t * k + j];
            if (s == -1) continue;
            if (s < -1 || s >= num_rows) { status = ORC_ERR_BAD_INDEX; continue; }
            memcpy(recv_x + (size_t)s * (H / 2), q, (size_t)H / 2);
            for (int b = 0; b < B; ++b)
                block_scale[oracle_scale_index(layout, num_rows, H, DT_NVFP4, s, b)] = sb[b];
            row_scale[s] = g;
        }
    }
    free(q); free(sb);
    return status;
}

/* ------------------------------------------------------------------ */
/* Per-channel FP8 of the receive buffer.  [TK] lists FP8 quantisation "per
 * channel" (and batched transposes) without a formula.  Reading: an
 * expert's receive rows are the contracted dimension of its weight-gradient
 * GEMM (dW_e = X_e^T dY_e), so one scale per (expert, channel) factors out
 * of it.  Per expert e and channel c, over the rows
 * s in [expert_offset[e], expert_offset[e] + expert_count[e]):
 *   amax = max |x[s,c]|,  scale[e,c] = amax / 448,
 *   code = e4m3(x[s,c] * (448 / amax))   (zeros keep their sign)
 * -- the per-block FP8 rule with the block = one channel of one expert.
 * Codes are written row-major [num_rows, H] or transposed [H, num_rows]
 * (channel-major); rows outside every expert's landed range (padding of the
 * aligned layout) are not written.                                      */
/* ------------------------------------------------------------------ */
int oracle_quant_fp8_channel(const uint16_t* x, int64_t num_rows, int H, int E,
                             const int32_t* expert_offset, const int32_t* expert_count,
                             int transpose, uint8_t* out, float* scale)
{
    if (num_rows < 0 || H < 1 || E < 1 || expert_offset[0] < 0 || expert_offset[E] > num_rows)
        return ORC_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e)
        if (expert_count[e] < 0 || expert_offset[e] + expert_count[e] > expert_offset[e + 1])
            return ORC_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e) {
        int64_t r0 = expert_offset[e], r1 = r0 + expert_count[e];
        for (int c = 0; c < H; ++c) {
            float amax = 0.0f;
            for (int64_t s = r0; s < r1; ++s) {
                float v = fabsf(oracle_f32_from_bf16(x[(size_t)s * H + c]));
                if (v > amax) amax = v;
            }
            float inv = 448.0f / amax;
            scale[(size_t)e * H + c] = amax / 448.0f;
            for (int64_t s = r0; s < r1; ++s) {
                float v = oracle_f32_from_bf16(x[(size_t)s * H + c]);
                uint8_t q = oracle_e4m3_encode((v == 0.0f) ? v : v * inv);
                if (transpose) out[(size_t)c * num_rows + s] = q;
                else out[(size_t)s * H + c] = q;
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* SwiGLU fused with quantisation.  [TK] list: SwiGLU combined with the
 * quantisation operations.  Between an expert's two GEMMs the first one's
 * output row h = [gate | up] (bf16, 2I channels; reading: the gate half
 * first) becomes a = SiLU(gate) * up, quantised for the second GEMM.
 * Reading (fp32, every operation rounded once):
 *   silu(g) = g / (1 + dexp(-g))   (the textbook x * sigmoid(x), written
 *                                   as one division)
 *   a_c     = silu(g_c) * u_c
 * a is quantised the way dispatch quantises a row, with these fp32 values
 * in place of the bf16 ones: BF16 (a rounded to bf16), per-128-block FP8,
 * per-row FP8 or MXFP8, scales in any layout of oracle_scale_index over
 * num_rows rows.  Rows whose slot_token is -1 (padding of the aligned
 * layout) are skipped; slot_token may be NULL (every row).             */
/* ------------------------------------------------------------------ */
static float silu_f32(float g)
{
    float e = oracle_dexp(-g);
    float d = 1.0f + e;
    return g / d;
}

void oracle_silu_array(const float* in, float* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = silu_f32(in[i]);
}

/* quantise one fp32 row of n values: codes (or bf16) to out_row, fp32
 * scales to fsc or E8M0 bytes to esc, one per block */
static void quantize_f32_row(const float* a, int n, int dtype, void* out_row, float* fsc,
                             uint8_t* esc)
{
    if (dtype == DT_BF16) {
        for (int c = 0; c < n; ++c) ((uint16_t*)out_row)[c] = oracle_bf16_from_f32(a[c]);
        return;
    }
    uint8_t* q = (uint8_t*)out_row;
    int bw = dtype == DT_FP8_E4M3 ? 128 : (dtype == DT_MXFP8_E4M3 ? 32 : n);
    for (int b = 0; b * bw < n; ++b) {
        float amax = 0.0f;
        for (int c = b * bw; c < (b + 1) * bw; ++c)
            if (fabsf(a[c]) > amax) amax = fabsf(a[c]);
        if (dtype == DT_MXFP8_E4M3) {
            int e = (amax > 0.0f) ? floor_log2_pos(amax) - 8 : -127;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
            esc[b] = (uint8_t)(e + 127);
            float down = ldexpf(1.0f, -e);   /* e <= 119 for finite a: a normal float */
            for (int c = b * bw; c < (b + 1) * bw; ++c)
                q[c] = oracle_e4m3_encode((a[c] == 0.0f) ? a[c] : a[c] * down);
        } else {
            float inv = 448.0f / amax;
            fsc[b] = amax / 448.0f;
            for (int c = b * bw; c < (b + 1) * bw; ++c)
                q[c] = oracle_e4m3_encode((a[c] == 0.0f) ? a[c] : a[c] * inv);
        }
    }
}

int oracle_swiglu_quant(const uint16_t* h, int64_t num_rows, int I, const int32_t* slot_token,
                        int dtype, int layout, void* out, void* out_scale)
{
    if (num_rows < 0 || I < 1 || dtype < DT_BF16 || dtype > DT_MXFP8_E4M3) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_FP8_E4M3 && I % 128 != 0) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_MXFP8_E4M3 && I % 32 != 0) return ORC_ERR_INVALID_ARG;
    if (dtype == DT_BF16 ? layout != SL_ROW_MAJOR : oracle_scale_elems(num_rows, I, dtype, layout) < 0)
        return ORC_ERR_INVALID_ARG;
    int B = scale_blocks(I, dtype), es = scale_elem_bytes(dtype);
    int ob = dtype == DT_BF16 ? 2 : 1;
    float* a = (float*)malloc(sizeof(float) * (size_t)I);
    float* fsc = (float*)malloc(sizeof(float) * (size_t)(B > 0 ? B : 1));
    uint8_t* esc = (uint8_t*)malloc((size_t)(B > 0 ? B : 1));
    for (int64_t s = 0; s < num_rows; ++s) {
        if (slot_token && slot_token[s] < 0) continue;
        const uint16_t* hr = h + (size_t)s * 2 * I;
        for (int c = 0; c < I; ++c) {
            float g = oracle_f32_from_bf16(hr[c]);
            float u = oracle_f32_from_bf16(hr[I + c]);
            a[c] = silu_f32(g) * u;
        }
        quantize_f32_row(a, I, dtype, (uint8_t*)out + (size_t)s * I * ob, fsc, esc);
        for (int b = 0; b < B; ++b) {
            const void* src = dtype == DT_MXFP8_E4M3 ? (const void*)&esc[b] : (const void*)&fsc[b];
            memcpy((uint8_t*)out_scale + oracle_scale_index(layout, num_rows, I, dtype, s, b) * es,
                   src, (size_t)es);
        }
    }
    free(a); free(fsc); free(esc);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Combine.  [pplx] Introduction and Combine: the token's output is the
 * average of its experts' outputs weighted by the router weights; [EPv2]
 * usage patterns: combine reduces the expert outputs back to the token.
 *   out[t,c] = bf16_rne( acc ),  acc = +0.0f, then for j = 0..k-1 in slot
 *   order: acc = fma(w[t,j], y[token_slot[t,j], c], acc)   (fp32)
 * Masked slots (-1) contribute nothing; other out-of-range slots are
 * skipped and reported.                                                */
/* ------------------------------------------------------------------ */
int oracle_combine(const uint16_t* y, int64_t num_rows, int N, int H, int k,
                   const int32_t* token_slot, const float* topk_w,
                   uint16_t* out)
{
    if (N < 0 || H < 1 || k < 1) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    int64_t S = num_rows;   /* rows of y */
    for (int t = 0; t < N; ++t) {
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t s = token_slot[(int64_t)t * k + j];
                if (s == -1) continue;
                if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }
                float v = oracle_f32_from_bf16(y[(size_t)s * H + c]);
                acc = fmaf(topk_w[(int64_t)t * k + j], v, acc);
            }
            out[(size_t)t * H + c] = oracle_bf16_from_f32(acc);
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* Backward of dispatch and combine.  [EPv2] usage patterns: the backward
 * pass of dispatch is a combine and the backward pass of combine is a
 * dispatch.  Written out as the adjoints of the forward maps:
 *
 *  dispatch backward:  grad_x[t,c] = bf16_rne(acc), acc = +0.0f, then
 *      acc = acc + grad_recv[token_slot[t,j], c] for j = 0..k-1 (slot order,
 *      fp32, masked slots skipped).
 *  combine backward:   for every valid slot s = token_slot[t,j]
 *      grad_y[s,c]  = bf16_rne( fp32(topk_w[t,j] * grad_out[t,c]) )
 *      grad_w[t,j]  = sum_c grad_out[t,c] * y[s,c], accumulated in double
 *                     (exact products, 53-bit sum) and rounded to fp32;
 *      a masked slot gets grad_w = 0 and writes no grad_y row.
 * The kernels may sum grad_w in another order in fp32; their error bound
 * follows from the arithmetic and is stated with the tests.            */
/* ------------------------------------------------------------------ */
int oracle_dispatch_backward(const uint16_t* grad_recv, int64_t num_rows, int N, int H, int k,
                             const int32_t* token_slot, uint16_t* grad_x)
{
    if (N < 0 || H < 1 || k < 1) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    int64_t S = num_rows;   /* rows of grad_recv */
    for (int t = 0; t < N; ++t) {
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t s = token_slot[(int64_t)t * k + j];
                if (s == -1) continue;
                if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }
                acc = acc + oracle_f32_from_bf16(grad_recv[(size_t)s * H + c]);
            }
            grad_x[(size_t)t * H + c] = oracle_bf16_from_f32(acc);
        }
    }
    return status;
}

int oracle_combine_backward(const uint16_t* grad_out, const uint16_t* y, int64_t num_rows, int N,
                            int H, int k, const int32_t* token_slot, const float* topk_w,
                            uint16_t* grad_y, float* grad_w, double* grad_w_abs)
{
    if (N < 0 || H < 1 || k < 1) return ORC_ERR_INVALID_ARG;
    int status = ORC_OK;
    int64_t S = num_rows;   /* rows of y and grad_y */
    for (int t = 0; t < N; ++t) {
        const uint16_t* g = grad_out + (size_t)t * H;
        for (int j = 0; j < k; ++j) {
            int64_t i = (int64_t)t * k + j;
            int32_t s = token_slot[i];
            grad_w[i] = 0.0f;
            if (grad_w_abs) grad_w_abs[i] = 0.0;
            if (s == -1) continue;
            if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }
            const uint16_t* yr = y + (size_t)s * H;
            uint16_t* gy = grad_y + (size_t)s * H;
            double dot = 0.0, mag = 0.0;
            for (int c = 0; c < H; ++c) {
                float gc = oracle_f32_from_bf16(g[c]);
                float prod = topk_w[i] * gc;
                gy[c] = oracle_bf16_from_f32(prod);
                double term = (double)gc * (double)oracle_f32_from_bf16(yr[c]);
                dot += term;
                mag += fabs(term);
            }
            grad_w[i] = (float)dot;
            if (grad_w_abs) grad_w_abs[i] = mag;
        }
    }
    return status;
}

