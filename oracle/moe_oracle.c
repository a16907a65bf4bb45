/*
 * CPU oracle for the DeepSeek-V3 MoE layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant generator with the CUDA path.
 *
 * Plain, slow, obviously correct: token-major loops, fp64 accumulation, every
 * stage written out as the pages define it.  Sources (page title, box):
 *   - "DeepSeek-V3" (ainfra.dev llm-vis), boxes "MoE router", "Mixture-of-
 *     Experts FFN", "Routed experts", "Shared expert", "Expert combine",
 *     "SwiGLU MLP", "Residual add".
 *   - "DeepSeek V3" field guide (curiouscaliboi), cutaway 02 "Fine-grained
 *     expert routing": the group stage (two strongest bias-adjusted scores per
 *     group, top 4 groups eligible, top 8 experts inside them, weights from the
 *     unbiased sigmoid renormalised to 1, times 2.5, no token dropped).
 *   - "Teardown: DeepSeek-V3" (inside-the-model), section 6 "Mixture of
 *     experts" and section 10 "FP8 training" (E4M3, 1x128 activation tiles,
 *     128x128 weight blocks, router kept in high precision).
 *
 * Readings where the pages are silent (each restated in the design notes):
 *   - sigmoid arithmetic: sigmoid_spec below (Cody-Waite reduction + Taylor
 *     polynomial), so that selection can be compared bit for bit;
 *   - group score = fp32 sum of the two largest biased scores of the group;
 *   - ties: larger value first, then the lower index (groups and experts);
 *   - slot order: descending biased score, then ascending expert index;
 *   - weights: s[idx[j]] / S with S the fp32 sum of the selected s taken in
 *     ascending expert index, no epsilon;
 *   - h is stored in bf16 (FP8 config: e4m3 with 1x128 scales), everything
 *     else accumulates in fp64;
 *   - e4m3 = OCP E4M3 (bias 7, no infinities, max 448), round to nearest even
 *     with saturation; scale = amax / 448 (1 when amax is 0).
 *
 * Parity pins live in tests/ (brute force over group and expert subsets,
 * closed forms, exhaustive sigmoid and e4m3 sweeps, library cross-checks).
 * Parity unpinned: nothing in this file; the GPU's fp32 accumulation order is
 * covered by the output tolerance only.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -pthread -lm.
 * -ffp-contract=off is required: sigmoid_spec must not be contracted into
 * fused multiply-adds the definition does not name.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar formats                                                           */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the top half of an IEEE binary32. */
double orc_bf16_to_f64(uint16_t h) { return (double)f32_from_bits((uint32_t)h << 16); }

/* Round a double to the nearest bf16 (ties to even), in one rounding step.
 * bf16 keeps 8 significant bits; the smallest subnormal is 2^-133. */
uint16_t orc_bf16_from_f64(double v)
{
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                        /* a = m * 2^ex, m in [0.5, 1) */
    int qexp = ex - 8;                    /* quantum of an 8-bit significand */
    if (qexp < -133) qexp = -133;
    double q = ldexp(a, -qexp);           /* exact: power-of-two scaling */
    double r = rint(q);                   /* default mode: nearest, ties even */
    double res = ldexp(r, qexp);
    if (res >= 0x1p128) return sign | 0x7F80;   /* overflow to infinity */
    uint32_t u = bits_from_f32((float)res);     /* exact: res is a bf16 value */
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* OCP E4M3 (FN): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 * field 0 holds subnormals m * 2^-9; S.1111.111 is NaN; no infinities. */
double orc_e4m3_to_f64(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to nearest even on the E4M3 grid, saturating finite values at 448. */
uint8_t orc_e4m3_from_f32(float f)
{
    if (isnan(f)) return 0x7F;
    uint8_t sign = signbit(f) ? 0x80 : 0;
    double a = fabs((double)f);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                        /* a in [2^(ex-1), 2^ex) */
    int qexp = (ex - 1) - 3;              /* 3 mantissa bits */
    if (qexp < -9) qexp = -9;             /* subnormal quantum */
    double r = ldexp(rint(ldexp(a, -qexp)), qexp);
    if (r > 448.0) r = 448.0;             /* saturate (no infinities) */
    if (r == 0.0) return sign;
    /* encode the exact grid value r */
    int e2;
    frexp(r, &e2);
    int E = (e2 - 1) + 7;
    uint8_t code;
    if (E <= 0) {
        code = (uint8_t)(r / 0x1p-9);                   /* subnormal: m */
    } else {
        double m = r / ldexp(1.0, e2 - 1) - 1.0;        /* in [0, 1) */
        code = (uint8_t)((E << 3) | (int)(m * 8.0));
    }
    return sign | code;
}

/* ------------------------------------------------------------------------ */
/* sigmoid_spec: the fp32 sigmoid both sides compute (reading of the router  */
/* box's ".sigmoid()").  exp by Cody-Waite argument reduction z = n ln2 + r, */
/* ln2 split in a high part with trailing zeros and a low part, a degree-7   */
/* Taylor polynomial in r with coefficients 1/i!, and 2^n built from the     */
/* exponent bits.  Only correctly rounded fp32 operations appear: multiply,  */
/* add, fused multiply-add where written, divide, and rint.                  */
/* ------------------------------------------------------------------------ */

static float exp_spec(float z)
{
    const float inv_ln2 = 0x1.715476p+0f;
    const float ln2_hi  = 0x1.62e4p-1f;
    const float ln2_lo  = 0x1.7f7d1cp-20f;
    if (z > 88.0f) z = 88.0f;
    if (z < -87.0f) z = -87.0f;
    float n = rintf(z * inv_ln2);
    float r = fmaf(-n, ln2_hi, z);
    r = fmaf(-n, ln2_lo, r);
    /* exp(r) = 1 + (r + r^2 Q(r)), Q(r) = sum_{i=2..7} r^(i-2)/i!; the two
     * leading terms are added last so that the polynomial's own rounding
     * stays below the final rounding. */
    float r2 = r * r;
    float Q = 0x1.a01a02p-13f;            /* 1/7! */
    Q = fmaf(Q, r, 0x1.6c16c2p-10f);      /* 1/6! */
    Q = fmaf(Q, r, 0x1.111112p-7f);       /* 1/5! */
    Q = fmaf(Q, r, 0x1.555556p-5f);       /* 1/4! */
    Q = fmaf(Q, r, 0x1.555556p-3f);       /* 1/3! */
    Q = fmaf(Q, r, 0.5f);                 /* 1/2! */
    float q = fmaf(r2, Q, r);
    float p = 1.0f + q;
    int ni = (int)n;                      /* in [-126, 127] after clamping */
    float two_n = f32_from_bits((uint32_t)(ni + 127) << 23);
    return p * two_n;
}

float orc_sigmoid(float l)
{
    float e = exp_spec(-l);
    float den = 1.0f + e;
    return 1.0f / den;
}

void orc_sigmoid_array(const float* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_sigmoid(in[i]);
}

/* ------------------------------------------------------------------------ */
/* S1  router logits: l[t,e] = sum_c x[t,c] * Wr[e,c], fp64 accumulation,    */
/* rounded once to fp32 ("MoE router" box: gate(x.float())).                 */
/* x is fp32 (x_is_f32 = 1) or bf16; Wr is bf16 [E, d] (nn.Linear layout).   */
/* ------------------------------------------------------------------------ */

static double x_at(const void* x, int x_is_f32, int64_t i)
{
    return x_is_f32 ? (double)((const float*)x)[i] : orc_bf16_to_f64(((const uint16_t*)x)[i]);
}

void orc_router_logits(const void* x, int x_is_f32, const uint16_t* w_router,
                       int T, int d, int E, float* logits)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += x_at(x, x_is_f32, (int64_t)t * d + c) *
                       orc_bf16_to_f64(w_router[(int64_t)e * d + c]);
            logits[(int64_t)t * E + e] = (float)acc;
        }
}

/* ------------------------------------------------------------------------ */
/* S2  selection (router box + field-guide cutaway 02):                      */
/*   s = sigmoid(l); b = s + bias (selection only);                         */
/*   group score = b(1) + b(2), the two largest b in the group;             */
/*   keep the topk_groups best groups; pick the top k experts by b among    */
/*   them; w[j] = s[idx[j]] / sum_j s[idx[j]] (unbiased, renormalised).     */
/*   The sum runs over the selected experts in ascending index.             */
/* Returns 0, or -1 when a size is invalid.                                 */
/* ------------------------------------------------------------------------ */

/* "a ranks before b": larger value, then lower index. */
static int ranks_before(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

int orc_select(const float* logits, const float* bias, int T, int E, int G,
               int topk_groups, int k, int32_t* idx_out, float* w_out)
{
    if (E <= 0 || G <= 0 || E % G != 0) return -1;
    int gs = E / G;
    if (gs < 2 || topk_groups < 1 || topk_groups > G || k < 1 || k > topk_groups * gs) return -1;
    float* s = (float*)malloc(sizeof(float) * E);
    float* b = (float*)malloc(sizeof(float) * E);
    float* gscore = (float*)malloc(sizeof(float) * G);
    char* gsel = (char*)malloc(G);
    char* taken = (char*)malloc(E);
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (int64_t)t * E;
        for (int e = 0; e < E; ++e) {
            s[e] = orc_sigmoid(l[e]);
            b[e] = s[e] + bias[e];
            if (b[e] == 0.0f) b[e] = 0.0f;            /* -0 ranks as +0 */
        }
        /* group scores: the two strongest biased scores of each group */
        for (int g = 0; g < G; ++g) {
            int i1 = -1, i2 = -1;
            for (int e = g * gs; e < (g + 1) * gs; ++e) {
                if (i1 < 0 || ranks_before(b[e], e, b[i1], i1)) { i2 = i1; i1 = e; }
                else if (i2 < 0 || ranks_before(b[e], e, b[i2], i2)) { i2 = e; }
            }
            gscore[g] = b[i1] + b[i2];
            if (gscore[g] == 0.0f) gscore[g] = 0.0f;
            gsel[g] = 0;
        }
        /* the topk_groups best groups are eligible */
        for (int r = 0; r < topk_groups; ++r) {
            int best = -1;
            for (int g = 0; g < G; ++g)
                if (!gsel[g] && (best < 0 || ranks_before(gscore[g], g, gscore[best], best))) best = g;
            gsel[best] = 1;
        }
        /* top k experts by biased score inside the eligible groups, emitted
         * in rank order (slot j = j-th best) */
        memset(taken, 0, E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (gsel[e / gs] && !taken[e] && (best < 0 || ranks_before(b[e], e, b[best], best))) best = e;
            taken[best] = 1;
            idx_out[(int64_t)t * k + j] = best;
        }
        /* weights from the unbiased scores, renormalised to sum to one; S is
         * summed in ascending expert index, so that it depends on the selected
         * set only and a bias that reorders slots leaves the weights alone */
        float S = 0.0f;
        for (int e = 0; e < E; ++e)
            if (taken[e]) S = S + s[e];
        for (int j = 0; j < k; ++j) w_out[(int64_t)t * k + j] = s[idx_out[(int64_t)t * k + j]] / S;
    }
    free(s); free(b); free(gscore); free(gsel); free(taken);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* S3  permutation: group the (t, j) pairs by expert ("Routed experts" box,  */
/* grouped-GEMM dispatch), ascending t inside each expert.                   */
/*   counts[e]  = #{(t,j): idx[t,j] = e}                                    */
/*   offsets    = exclusive prefix sum of counts, offsets[E] = T*k           */
/*   src[row]   = t*k + j,   inv[t*k + j] = row                              */
/* Returns 0, or -1 when an expert id is out of range.                      */
/* ------------------------------------------------------------------------ */

int orc_permute(const int32_t* idx, int T, int k, int E, int32_t* counts,
                int32_t* offsets, int32_t* src, int32_t* inv)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < (int64_t)T * k; ++p) {
        if (idx[p] < 0 || idx[p] >= E) return -1;
        counts[idx[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)calloc(E, sizeof(int32_t));
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(int64_t)t * k + j];
            int32_t row = offsets[e] + fill[e]++;
            src[row] = t * k + j;
            inv[(int64_t)t * k + j] = row;
        }
    free(fill);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Bias controller ("MoE router" box, update_bias; teardown section 6: the   */
/* bias is lowered for overloaded experts and raised for underloaded ones    */
/* after each step):                                                         */
/*   mean = (sum of counts) / E                     (fp32, as counts.mean()) */
/*   bias[e] -= gamma  if counts[e] > mean   else  bias[e] += gamma  (fp32)   */
/* ------------------------------------------------------------------------ */

void orc_update_bias(const int32_t* counts, int E, float* bias, float gamma)
{
    int64_t sum = 0;
    for (int e = 0; e < E; ++e) sum += counts[e];
    float mean = (float)sum / (float)E;
    for (int e = 0; e < E; ++e) {
        if ((float)counts[e] > mean) bias[e] = bias[e] - gamma;
        else bias[e] = bias[e] + gamma;
    }
}

/* ------------------------------------------------------------------------ */
/* Pre-norm of the MoE sublayer ("DeepSeek-V3" llm-vis, "RMSNorm" box: each  */
/* token vector is rescaled to unit RMS over its features, eps 1e-6, the     */
/* normalised value is cast back to the activation dtype, then multiplied by */
/* the learned per-feature gain; "Residual add" box: y = h + ffn(norm2(h))): */
/*   r      = 1 / sqrt(mean_c h[c]^2 + eps)      (fp64 here; fp32 on the page)*/
/*   out[c] = bf16( bf16(h[c] * r) * g[c] )                                   */
/* ------------------------------------------------------------------------ */

void orc_rmsnorm(const uint16_t* h, const uint16_t* g, int T, int d, double eps, uint16_t* out)
{
    for (int t = 0; t < T; ++t) {
        const uint16_t* hr = h + (int64_t)t * d;
        double ss = 0.0;
        for (int c = 0; c < d; ++c) {
            double v = orc_bf16_to_f64(hr[c]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / (double)d + eps);
        for (int c = 0; c < d; ++c) {
            uint16_t v = orc_bf16_from_f64(orc_bf16_to_f64(hr[c]) * r);
            out[(int64_t)t * d + c] = orc_bf16_from_f64(orc_bf16_to_f64(v) * orc_bf16_to_f64(g[c]));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* S6  activation quantisation (teardown, section 10: activations scaled in  */
/* 1x128 tiles, E4M3).  Per token and 128-channel block, in fp32:            */
/*   sx = amax / 448 (1 when amax = 0);  q = e4m3_rn_sat(x / sx).            */
/* ------------------------------------------------------------------------ */

void orc_quant_act(const uint16_t* x, int T, int d, uint8_t* q, float* sx)
{
    int nb = d / 128;
    for (int t = 0; t < T; ++t)
        for (int bk = 0; bk < nb; ++bk) {
            const uint16_t* xr = x + (int64_t)t * d + bk * 128;
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i) {
                float v = fabsf(f32_from_bits((uint32_t)xr[i] << 16));
                if (v > amax) amax = v;
            }
            float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
            sx[(int64_t)t * nb + bk] = scale;
            for (int i = 0; i < 128; ++i)
                q[(int64_t)t * d + bk * 128 + i] =
                    orc_e4m3_from_f32(f32_from_bits((uint32_t)xr[i] << 16) / scale);
        }
}

/* ------------------------------------------------------------------------ */
/* S4 + S5  expert math and combine, token-major ("Mixture-of-Experts FFN"   */
/* forward, "Expert combine" box: y = 2.5 * sum_i w_i e_i(x) + shared(x)).   */
/* expert(x) = W_down (SiLU(W_gate x) * (W_up x)), SiLU(z) = z * sigmoid(z)  */
/* ("SwiGLU MLP" box; teardown section 6).                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    int d, E, H, Hs, k;
    int x_is_f32;         /* C0: fp32 x, rounded to bf16 for the experts */
    int fp8;              /* expert weights e4m3 with 128x128 block scales;
                             activations quantised per 1x128 tile */
    double routed_scale;
    /* E pointers each; bf16 (uint16) or e4m3 (uint8) elements */
    const void* const* w_gate;     /* [H, d] */
    const void* const* w_up;       /* [H, d] */
    const void* const* w_down;     /* [d, H] */
    const float* const* s_gate;    /* [H/128, d/128] (fp8 only) */
    const float* const* s_up;
    const float* const* s_down;    /* [d/128, H/128] */
    const void* ws_gate;           /* shared expert [Hs, d] */
    const void* ws_up;
    const void* ws_down;           /* [d, Hs] */
    const float* ss_gate, *ss_up, *ss_down;
} orc_layer;

/* weight element (r, c) of a [rows, cols] matrix */
static double w_at(const orc_layer* L, const void* w, const float* s, int cols, int64_t r, int64_t c)
{
    if (!L->fp8) return orc_bf16_to_f64(((const uint16_t*)w)[r * cols + c]);
    double code = orc_e4m3_to_f64(((const uint8_t*)w)[r * cols + c]);
    return code * (double)s[(r / 128) * (cols / 128) + (c / 128)];
}

/* o[0..d) = expert(xh); e < 0 selects the shared expert. h: scratch [H]. */
static void expert_eval(const orc_layer* L, int e, const double* xh, double* h, double* o)
{
    int d = L->d, H = e < 0 ? L->Hs : L->H;
    const void* wg = e < 0 ? L->ws_gate : L->w_gate[e];
    const void* wu = e < 0 ? L->ws_up : L->w_up[e];
    const void* wd = e < 0 ? L->ws_down : L->w_down[e];
    const float* sg = e < 0 ? L->ss_gate : (L->fp8 ? L->s_gate[e] : NULL);
    const float* su = e < 0 ? L->ss_up : (L->fp8 ? L->s_up[e] : NULL);
    const float* sd = e < 0 ? L->ss_down : (L->fp8 ? L->s_down[e] : NULL);
    for (int i = 0; i < H; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < d; ++c) {
            g += w_at(L, wg, sg, d, i, c) * xh[c];
            u += w_at(L, wu, su, d, i, c) * xh[c];
        }
        h[i] = g / (1.0 + exp(-g)) * u;          /* SiLU(g) * u */
    }
    /* h is stored before the down projection: bf16, or e4m3 with one scale
     * per 128 hidden channels */
    if (!L->fp8) {
        for (int i = 0; i < H; ++i) h[i] = orc_bf16_to_f64(orc_bf16_from_f64(h[i]));
    } else {
        for (int b0 = 0; b0 < H; b0 += 128) {
            double amax = 0.0;
            for (int i = b0; i < b0 + 128; ++i) if (fabs(h[i]) > amax) amax = fabs(h[i]);
            double scale = amax > 0.0 ? amax / 448.0 : 1.0;
            for (int i = b0; i < b0 + 128; ++i)
                h[i] = orc_e4m3_to_f64(orc_e4m3_from_f32((float)(h[i] / scale))) * scale;
        }
    }
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int i = 0; i < H; ++i) acc += w_at(L, wd, sd, H, c, i) * h[i];
        o[c] = acc;
    }
}

typedef struct {
    const orc_layer* L;
    const void* x;
    const int32_t* idx;
    const float* w;
    const int32_t* tokens;
    int n_tok, tid, nthreads;
    double* y;
    int status;
} worker_arg;

static void* worker(void* p)
{
    worker_arg* a = (worker_arg*)p;
    const orc_layer* L = a->L;
    int d = L->d, Hmax = L->H > L->Hs ? L->H : L->Hs;
    double* xh = (double*)malloc(sizeof(double) * d);
    double* h = (double*)malloc(sizeof(double) * Hmax);
    double* o = (double*)malloc(sizeof(double) * d);
    double* routed = (double*)malloc(sizeof(double) * d);
    uint16_t* xrow = (uint16_t*)malloc(sizeof(uint16_t) * d);
    uint8_t* q = (uint8_t*)malloc(d);
    float* sx = (float*)malloc(sizeof(float) * (d / 128 + 1));
    a->status = 0;
    for (int n = a->tid; n < a->n_tok; n += a->nthreads) {
        int t = a->tokens[n];
        /* x_hat: the value the experts see */
        for (int c = 0; c < d; ++c) {
            double v = x_at(a->x, L->x_is_f32, (int64_t)t * d + c);
            xrow[c] = orc_bf16_from_f64(v);
            xh[c] = orc_bf16_to_f64(xrow[c]);
        }
        if (L->fp8) {
            orc_quant_act(xrow, 1, d, q, sx);
            for (int c = 0; c < d; ++c) xh[c] = orc_e4m3_to_f64(q[c]) * (double)sx[c / 128];
        }
        for (int c = 0; c < d; ++c) routed[c] = 0.0;
        for (int j = 0; j < L->k; ++j) {
            int e = a->idx[(int64_t)t * L->k + j];
            if (e < 0 || e >= L->E || !L->w_gate[e]) { a->status = -1; continue; }
            expert_eval(L, e, xh, h, o);
            double wj = (double)a->w[(int64_t)t * L->k + j];
            for (int c = 0; c < d; ++c) routed[c] += wj * o[c];
        }
        expert_eval(L, -1, xh, h, o);
        double* yt = a->y + (int64_t)n * d;
        for (int c = 0; c < d; ++c) yt[c] = L->routed_scale * routed[c] + o[c];
    }
    free(xh); free(h); free(o); free(routed); free(xrow); free(q); free(sx);
    return NULL;
}

/* y[n, :] for token tokens[n]; idx/w are the routing of all tokens [T, k].
 * Runs on n_threads host threads (over tokens).  Returns 0, or -1 when a
 * routed expert id is out of range or its weights were not provided. */
int orc_expert_tokens(const orc_layer* L, const void* x, const int32_t* idx, const float* w,
                      const int32_t* tokens, int n_tok, int n_threads, double* y)
{
    if (n_threads < 1) n_threads = 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * n_threads);
    worker_arg* args = (worker_arg*)malloc(sizeof(worker_arg) * n_threads);
    for (int i = 0; i < n_threads; ++i) {
        worker_arg a = {L, x, idx, w, tokens, n_tok, i, n_threads, y, 0};
        args[i] = a;
        pthread_create(&th[i], NULL, worker, &args[i]);
    }
    int status = 0;
    for (int i = 0; i < n_threads; ++i) {
        pthread_join(th[i], NULL);
        if (args[i].status) status = args[i].status;
    }
    free(th); free(args);
    return status;
}

/* One routed expert or the shared expert (e < 0) on one input row, for the
 * closed-form pins: o = expert(x_hat) with x_hat given in fp64. */
void orc_expert_single(const orc_layer* L, int e, const double* xh, double* o)
{
    int Hmax = L->H > L->Hs ? L->H : L->Hs;
    double* h = (double*)malloc(sizeof(double) * Hmax);
    expert_eval(L, e, xh, h, o);
    free(h);
}
