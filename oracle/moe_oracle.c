/*
 * CPU oracle for the shared-experts-fused GLM4-MoE expert layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline do. It shares no code, header or table with the CUDA library.
 *
 * What it computes (the plain definition; slow and obviously correct):
 *
 *   "GLM4-MoE生产环境优化：SGLang降低65%首Token延迟" (intelliparadigm.com), section
 *   2.1 "Shared Experts Fusion", the pseudocode block: the unfused layer is
 *       out = shared_expert(x) + sum(route(x, top_k = 8))
 *   Same page, numbered list under the pseudocode, and the de/en pages,
 *   section 1 "Shared Experts Fusion": the shared expert becomes routed expert
 *   no. 161 (index 160); each token takes the top 9 of 161 experts, its 8 routed
 *   experts plus the shared expert forced into the 9th position, with its weight
 *   handled specially; all expert outputs are aggregated with weights.
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes):
 *   R1 router: logits L = x . Wr^T (+ b), softmax over the selected top-K,
 *      renormalised (renormalize = 0: full softmax over all routed experts
 *      evaluated at the selected ids).
 *   R2 the shared expert's "special handling": slot K holds (id E_r, weight
 *      shared_weight), shared_weight = 1.0 reproduces the unfused sum exactly.
 *   R3 ranking key (logit desc, id asc) on the fp32 logits; NaN ranks as -inf.
 *   R4 logits are fp32 in a fixed order so that routing is reproducible bit for
 *      bit: H is cut into segments of 256; inside a segment an fp32 fma chain
 *      from +0 over ascending h; the segment sums are added in ascending
 *      segment order to a running fp32 total that starts at +0; the bias (if
 *      any) is added last in fp32.
 *   R5 slot order in a token: slots 0..K-1 by R3, slot K the shared expert.
 *   R6 permutation: experts in id order, inside an expert stable by the flat
 *      slot index t*S + k.
 *   R7 expert FFN (SwiGLU): w13[e] rows [0, I) = gate, [I, 2I) = up;
 *      h = silu(gate . v) * (up . v), silu(g) = g / (1 + exp(-g));
 *      y = w2[e] . h.
 *   R8 E4M3 is the OCP "E4M3FN" format: bias 7, no infinities, 0x7F/0xFF NaN,
 *      largest finite 448, smallest subnormal 2^-9. E4M3 layers quantise x per
 *      token and h per (token, expert) row with scale = amax/448 computed in
 *      fp32, codes = E4M3_rn_satfinite(v / scale) with an fp32 divide, after h
 *      has been rounded to bf16.
 *   R9 roundings that are part of the layer's storage format: bf16 layers round
 *      h to bf16 and the output to bf16 once. Everything else is fp64.
 *   R15 routed scaling factor s (the de/en pages, section 1, mention that the
 *      shared expert's weight needs special handling): the routed slots weigh
 *      s * softmax and the shared slot keeps shared_weight, the same sum as an
 *      engine that scales the whole fused sum by s with the shared slot at 1/s.
 *   R16 bias for selection only: the bias enters the ranking key (R3, R4) but
 *      the softmax uses the logits without it.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2

/* ---------------------------------------------------------------- codecs */

double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 value (ties to even), directly, with no
 * intermediate rounding to fp32. Returns the bf16 bit pattern. */
uint16_t orc_round_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int ex;
    frexp(a, &ex);                  /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                 /* a in [2^E, 2^(E+1)) */
    int qexp = (E >= -126) ? E - 7 : -133;   /* spacing of bf16 values there */
    double r = nearbyint(ldexp(a, -qexp));    /* exact scaling, RNE */
    double q = ldexp(r, qexp);
    if (q >= ldexp(1.0, 128)) return sign | 0x7F80;   /* rounds past the largest */
    float f = (float)q;             /* exact: q is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);            /* subnormal: m/8 * 2^-6 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* fp32 -> E4M3, round to nearest even, saturating to +-448; the sign bit is
 * kept for values that round to zero; NaN -> 0x7F. */
uint8_t orc_e4m3_encode(float vf) {
    if (isnan(vf)) return 0x7F;
    uint8_t sign = signbit(vf) ? 0x80 : 0;
    double a = fabs((double)vf);
    if (a > 448.0) a = 448.0;
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);
    int E = ex - 1;
    int qexp = (E >= -6) ? E - 3 : -9;
    double r = nearbyint(ldexp(a, -qexp));
    double q = ldexp(r, qexp);                  /* q <= 448 because a <= 448 */
    if (q == 0.0) return sign;
    frexp(q, &ex);
    E = ex - 1;
    uint8_t code;
    if (E < -6) {
        code = (uint8_t)ldexp(q, 9);            /* subnormal mantissa 1..7 */
    } else {
        int mant = (int)(ldexp(q, -E) * 8.0 - 8.0);
        code = (uint8_t)(((E + 7) << 3) | mant);
    }
    return sign | code;
}

/* Per-row E4M3 quantisation (R8): scale = amax/448 in fp32 (amax = 0 -> 1),
 * codes = E4M3(v / scale) with an fp32 divide. */
float orc_quant_row_e4m3(int n, const float* v, uint8_t* codes) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    float scale = (amax > 0.0f) ? amax / 448.0f : 1.0f;
    for (int i = 0; i < n; ++i) {
        float q = v[i] / scale;
        codes[i] = orc_e4m3_encode(q);
    }
    return scale;
}

/* ---------------------------------------------------------------- router */

/* Router logits in the fixed fp32 order of R4. x holds the activations as fp32
 * values (bf16 inputs widen exactly). H must be a multiple of 256. */
void orc_router_logits(int T, int H, int E_r, const float* x, const float* wr,
                       const float* bias, float* L) {
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E_r; ++e) {
            const float* xv = x + (size_t)t * H;
            const float* wv = wr + (size_t)e * H;
            float total = 0.0f;
            for (int s0 = 0; s0 < H; s0 += 256) {
                float acc = 0.0f;
                for (int h = s0; h < s0 + 256; ++h) acc = fmaf(xv[h], wv[h], acc);
                total = total + acc;
            }
            if (bias) total = total + bias[e];
            L[(size_t)t * E_r + e] = total;
        }
    }
}

/* The same logits in fp64 (for reporting the fp32 rounding error only). */
void orc_router_logits_f64(int T, int H, int E_r, const float* x, const float* wr,
                           const float* bias, double* L) {
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E_r; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h) acc += (double)x[(size_t)t * H + h] * wr[(size_t)e * H + h];
            if (bias) acc += bias[e];
            L[(size_t)t * E_r + e] = acc;
        }
}

static double rank_key(float v) { return isnan(v) ? -INFINITY : (double)v; }

/* Top-K selection and weights for T tokens (R1-R3, R15, R16). L holds the
 * ranking keys; Lw the logits the weights use (NULL: the keys). Slots 0..K-1
 * hold the routed experts in rank order with weight routed_scale * softmax; if
 * shared_id >= 0, slot K holds (shared_id, shared_weight).
 * S = K + (shared_id >= 0). */
void orc_topk(int T, int E_r, int K, const float* L, const float* Lw, int renormalize, float routed_scale,
              int shared_id, float shared_weight, int32_t* ids, double* w) {
    int S = K + (shared_id >= 0 ? 1 : 0);
    char* taken = (char*)malloc((size_t)E_r);
    for (int t = 0; t < T; ++t) {
        const float* l = L + (size_t)t * E_r;
        const float* lw = (Lw ? Lw : L) + (size_t)t * E_r;
        int32_t* id = ids + (size_t)t * S;
        double* wt = w + (size_t)t * S;
        memset(taken, 0, (size_t)E_r);
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E_r; ++e) {
                if (taken[e]) continue;
                if (best < 0 || rank_key(l[e]) > rank_key(l[best])) best = e;
            }
            taken[best] = 1;
            id[k] = best;
        }
        /* softmax over the selected (renormalize) or all weight logits, taken
         * relative to their largest value */
        double m = -INFINITY, den = 0.0;
        if (renormalize) {
            for (int k = 0; k < K; ++k) if (rank_key(lw[id[k]]) > m) m = rank_key(lw[id[k]]);
            for (int k = 0; k < K; ++k) den += exp(rank_key(lw[id[k]]) - m);
        } else {
            for (int e = 0; e < E_r; ++e) if (rank_key(lw[e]) > m) m = rank_key(lw[e]);
            for (int e = 0; e < E_r; ++e) den += exp(rank_key(lw[e]) - m);
        }
        for (int k = 0; k < K; ++k) wt[k] = (double)routed_scale * (exp(rank_key(lw[id[k]]) - m) / den);
        if (shared_id >= 0) {
            id[K] = shared_id;
            wt[K] = (double)shared_weight;
        }
    }
    free(taken);
}

/* ---------------------------------------------------------------- QK-norm + partial RoPE */

/* "GLM4-MoE生产环境优化：SGLang降低65%首Token延迟", section 2.2 QK-Norm-RoPE
 * fusion, and the de/en pages, section 2 "Qknorm Fusion": the attention's q
 * and k heads are normalised head by head and rotated, and in GLM4-MoE only
 * half of each head's dimensions rotate. Readings (the pages give no formula):
 *   R17 the norm is RMSNorm over head_dim with a per-dimension weight (one for
 *       q heads, one for k heads): u = v / sqrt(mean(v^2) + eps) * w;
 *   R18 RoPE on the first rot dimensions, pairs (i, i + rot/2) for i < rot/2:
 *       (a, b) -> (a cos - b sin, b cos + a sin) with cos/sin of the token's
 *       position from the caller's table [max_pos][rot] (cos in [0, rot/2),
 *       sin in [rot/2, rot)); dimensions >= rot pass through;
 *   R19 the fused qkv row of a token is [q heads | k heads | v heads]; v is
 *       left alone. Everything here is fp64 (the output is not rounded).
 * out: [T][n_q + n_kv][d]. */
void orc_qk_norm_rope(int T, int n_q, int n_kv, int d, int rot, float eps, const uint16_t* qkv,
                      const int32_t* pos, const uint16_t* qw, const uint16_t* kw, const float* cos_sin,
                      double* out) {
    const int row = (n_q + 2 * n_kv) * d;
    const int half = rot / 2;
    double* u = (double*)malloc((size_t)d * sizeof(double));
    for (int t = 0; t < T; ++t) {
        const float* cs = cos_sin + (size_t)pos[t] * rot;
        for (int h = 0; h < n_q + n_kv; ++h) {
            const uint16_t* v = qkv + (size_t)t * row + (size_t)h * d;
            const uint16_t* w = h < n_q ? qw : kw;
            double ss = 0.0;
            for (int i = 0; i < d; ++i) {
                const double a = orc_bf16_to_double(v[i]);
                ss += a * a;
            }
            const double r = 1.0 / sqrt(ss / d + (double)eps);
            for (int i = 0; i < d; ++i) u[i] = orc_bf16_to_double(v[i]) * r * orc_bf16_to_double(w[i]);
            double* o = out + ((size_t)t * (n_q + n_kv) + h) * d;
            for (int i = 0; i < d; ++i) o[i] = u[i];
            for (int i = 0; i < half; ++i) {
                const double c = cs[i], s = cs[half + i];
                o[i] = u[i] * c - u[i + half] * s;
                o[i + half] = u[i + half] * c + u[i] * s;
            }
        }
    }
    free(u);
}

/* ---------------------------------------------------------------- permute */

/* Counting sort of the R = T*S slots by expert, stable by flat index (R6).
 * perm[row] = flat slot index; inv[flat] = row; offsets has E+1 entries.
 * Returns -1 if an id is out of [0, E). */
int orc_permute(int R, int E, const int32_t* ids, int32_t* counts, int32_t* offsets,
                int32_t* perm, int32_t* inv) {
    if (E <= 0 || R < 0) return -1;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int f = 0; f < R; ++f) {
        if (ids[f] < 0 || ids[f] >= E) return -1;
        counts[ids[f]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int f = 0; f < R; ++f) {
        int e = ids[f];
        int row = offsets[e] + fill[e]++;
        perm[row] = f;
        inv[f] = row;
    }
    free(fill);
    return 0;
}

/* ---------------------------------------------------------------- experts */

typedef struct {
    int T, H, I, E_r, K, shared_id;
    float shared_weight;
    int renormalize;
    int act_dtype;          /* ORC_F32 | ORC_BF16 */
    int w_dtype;            /* ORC_F32 | ORC_BF16 | ORC_E4M3 */
    float routed_scale;     /* R15 */
    int bias_select_only;   /* R16 */
    const void* x;          /* [T, H] fp32 or bf16 bits */
    const float* router_w;  /* [E_r, H] */
    const float* router_bias;  /* [E_r] or NULL */
    const void* w13;        /* [E, 2I, H] */
    const float* s13;       /* [E, 2I] (E4M3 only) */
    const void* w2;         /* [E, H, I] */
    const float* s2;        /* [E, H]  (E4M3 only) */
} orc_layer;

static double wval(int dt, const void* base, size_t i) {
    if (dt == ORC_F32) return (double)((const float*)base)[i];
    if (dt == ORC_BF16) return orc_bf16_to_double(((const uint16_t*)base)[i]);
    return orc_e4m3_decode(((const uint8_t*)base)[i]);
}

static double xval(const orc_layer* Ly, int t, int h) {
    size_t i = (size_t)t * Ly->H + h;
    if (Ly->act_dtype == ORC_F32) return (double)((const float*)Ly->x)[i];
    return orc_bf16_to_double(((const uint16_t*)Ly->x)[i]);
}

/* One expert applied to one token (R7, R8, R9). v: the token's activations as the
 * layer stores them (fp32 values). Writes y[H] in fp64, unrounded.
 * scratch: at least 2I + H doubles + H floats + H + I bytes. */
static void expert_ffn(const orc_layer* Ly, int e, const float* v, double* y, void* scratch) {
    const int H = Ly->H, I = Ly->I;
    double* xin = (double*)scratch;       /* [H] value the GEMM sees */
    double* hh = xin + H;                 /* [I] */
    float* hf = (float*)(hh + I);         /* [I] */
    uint8_t* codes = (uint8_t*)(hf + I);  /* [max(H, I)] */
    double sx = 1.0;
    if (Ly->w_dtype == ORC_E4M3) {
        float s = orc_quant_row_e4m3(H, v, codes);
        for (int h = 0; h < H; ++h) xin[h] = orc_e4m3_decode(codes[h]);
        sx = (double)s;
    } else {
        for (int h = 0; h < H; ++h) xin[h] = (double)v[h];
    }
    const size_t w13off = (size_t)e * 2 * I * H;
    for (int n = 0; n < I; ++n) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            g += xin[h] * wval(Ly->w_dtype, Ly->w13, w13off + (size_t)n * H + h);
            u += xin[h] * wval(Ly->w_dtype, Ly->w13, w13off + (size_t)(I + n) * H + h);
        }
        if (Ly->w_dtype == ORC_E4M3) {
            g = g * sx * (double)Ly->s13[(size_t)e * 2 * I + n];
            u = u * sx * (double)Ly->s13[(size_t)e * 2 * I + I + n];
        }
        double silu = g / (1.0 + exp(-g));
        hh[n] = silu * u;
    }
    double sh = 1.0;
    if (Ly->act_dtype == ORC_BF16) {
        for (int n = 0; n < I; ++n) hh[n] = orc_bf16_to_double(orc_round_bf16(hh[n]));
    }
    if (Ly->w_dtype == ORC_E4M3) {
        for (int n = 0; n < I; ++n) hf[n] = (float)hh[n];   /* exact: bf16 values */
        float s = orc_quant_row_e4m3(I, hf, codes);
        for (int n = 0; n < I; ++n) hh[n] = orc_e4m3_decode(codes[n]);
        sh = (double)s;
    }
    const size_t w2off = (size_t)e * H * I;
    for (int j = 0; j < H; ++j) {
        double acc = 0.0;
        for (int n = 0; n < I; ++n)
            acc += hh[n] * wval(Ly->w_dtype, Ly->w2, w2off + (size_t)j * I + n);
        if (Ly->w_dtype == ORC_E4M3) acc = acc * sh * (double)Ly->s2[(size_t)e * H + j];
        y[j] = acc;
    }
}

static size_t scratch_bytes(const orc_layer* Ly) {
    size_t H = Ly->H, I = Ly->I, n = H > I ? H : I;
    return (H + 2 * I) * sizeof(double) + I * sizeof(float) + n + 64;
}

/* Public single-expert entry (used by the tests' closed-form checks). */
void orc_expert_ffn(const orc_layer* Ly, int e, const float* v, double* y) {
    void* scratch = malloc(scratch_bytes(Ly));
    expert_ffn(Ly, e, v, y, scratch);
    free(scratch);
}

static double round_out(const orc_layer* Ly, double v) {
    if (Ly->act_dtype == ORC_BF16) return orc_bf16_to_double(orc_round_bf16(v));
    return (double)(float)v;
}

/* ---------------------------------------------------------------- forward */

typedef struct {
    const orc_layer* Ly;
    int n_tok;
    const int32_t* tok;
    int fuse_shared;
    double* out;        /* [n_tok, H] fp64, unrounded */
    double* out_rnd;    /* [n_tok, H] rounded to the output dtype */
    int32_t* ids;       /* [n_tok, S] (fused) or [n_tok, K] */
    double* w;
    int lo, hi;
} fwd_job;

static void forward_token(const orc_layer* Ly, int t, int fuse_shared, double* out,
                          double* out_rnd, int32_t* ids, double* w, void* scratch) {
    const int H = Ly->H, E_r = Ly->E_r, K = Ly->K;
    float* v = (float*)malloc((size_t)H * sizeof(float));
    float* L = (float*)malloc((size_t)E_r * sizeof(float));      /* ranking keys */
    float* Lw = (float*)malloc((size_t)E_r * sizeof(float));     /* logits without the bias */
    double* y = (double*)malloc((size_t)H * sizeof(double));
    for (int h = 0; h < H; ++h) v[h] = (float)xval(Ly, t, h);
    orc_router_logits(1, H, E_r, v, Ly->router_w, NULL, Lw);
    for (int e = 0; e < E_r; ++e) L[e] = Ly->router_bias ? Lw[e] + Ly->router_bias[e] : Lw[e];
    const float* Lweights = Ly->bias_select_only ? Lw : NULL;
    for (int j = 0; j < H; ++j) out[j] = 0.0;
    if (fuse_shared) {
        /* Fused: one pass over the S = K + 1 slots, shared expert in slot K. */
        int S = K + (Ly->shared_id >= 0 ? 1 : 0);
        orc_topk(1, E_r, K, L, Lweights, Ly->renormalize, Ly->routed_scale, Ly->shared_id, Ly->shared_weight,
                 ids, w);
        for (int k = 0; k < S; ++k) {
            expert_ffn(Ly, ids[k], v, y, scratch);
            for (int j = 0; j < H; ++j) out[j] += w[k] * y[j];
        }
    } else {
        /* Unfused: routed top-K sum, then the shared expert added on its own. */
        orc_topk(1, E_r, K, L, Lweights, Ly->renormalize, Ly->routed_scale, -1, 0.0f, ids, w);
        for (int k = 0; k < K; ++k) {
            expert_ffn(Ly, ids[k], v, y, scratch);
            for (int j = 0; j < H; ++j) out[j] += w[k] * y[j];
        }
        if (Ly->shared_id >= 0) {
            expert_ffn(Ly, Ly->shared_id, v, y, scratch);
            for (int j = 0; j < H; ++j) out[j] = (double)Ly->shared_weight * y[j] + out[j];
        }
    }
    for (int j = 0; j < H; ++j) out_rnd[j] = round_out(Ly, out[j]);
    free(v);
    free(L);
    free(Lw);
    free(y);
}

static void* fwd_worker(void* arg) {
    fwd_job* J = (fwd_job*)arg;
    const orc_layer* Ly = J->Ly;
    int S = Ly->K + ((J->fuse_shared && Ly->shared_id >= 0) ? 1 : 0);
    void* scratch = malloc(scratch_bytes(Ly));
    for (int i = J->lo; i < J->hi; ++i)
        forward_token(Ly, J->tok[i], J->fuse_shared, J->out + (size_t)i * Ly->H,
                      J->out_rnd + (size_t)i * Ly->H, J->ids + (size_t)i * S,
                      J->w + (size_t)i * S, scratch);
    free(scratch);
    return NULL;
}

/* The layer for the tokens listed in tok[0..n_tok) (a sample, or all of them),
 * on up to n_threads host threads. ids/w receive each token's slots:
 * S = K + 1 entries when fused with a shared expert, else K. Returns the number
 * of threads used. */
int orc_forward(const orc_layer* Ly, int n_tok, const int32_t* tok, int fuse_shared,
                double* out, double* out_rnd, int32_t* ids, double* w, int n_threads) {
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_tok) n_threads = n_tok > 0 ? n_tok : 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    fwd_job* jobs = (fwd_job*)malloc(sizeof(fwd_job) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i) {
        fwd_job j = {Ly, n_tok, tok, fuse_shared, out, out_rnd, ids, w,
                     (int)((long)n_tok * i / n_threads), (int)((long)n_tok * (i + 1) / n_threads)};
        jobs[i] = j;
        pthread_create(&th[i], NULL, fwd_worker, &jobs[i]);
    }
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    free(jobs);
    return n_threads;
}

/* Weighted combine given expert rows Y (R9's output rounding applied):
 * out[t] = sum_{k<S} w[t,k] * Y[inv[t*S+k]], fp64 in slot order. Y is fp32. */
void orc_combine(int T, int S, int H, const float* Y, const int32_t* inv, const double* w,
                 int act_dtype, double* out) {
    orc_layer tmp;
    memset(&tmp, 0, sizeof(tmp));
    tmp.act_dtype = act_dtype;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < H; ++j) {
            double acc = 0.0;
            for (int k = 0; k < S; ++k)
                acc += w[(size_t)t * S + k] * (double)Y[(size_t)inv[(size_t)t * S + k] * H + j];
            out[(size_t)t * H + j] = round_out(&tmp, acc);
        }
}
