/*
 * moe_oracle.c -- plain, slow CPU oracle of the calibration-free sparse
 * routed-expert reader.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and
 * the bench's CPU-baseline leg may call it; the product path never does.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What the pages fix (all cited by page title and section):
 *   "Channel Selection for Mixture-of-Experts Decoding Needs No Calibration
 *   Data" (arXiv:2610.37386 v1), abstract: routed-expert decoding at small
 *   batch is bound by loading expert weights; a per-token top-k keep rule
 *   needs no calibration data; the reader is built from the weights alone,
 *   screens channels with a ternary sketch and recovers skipped channels with
 *   a low-rank map.
 *   "KAIST: MoE Decoding Needs No Calibration Data", section "A reader that
 *   needs no data at all": the sketch is a rotated ternary sketch of the gate
 *   and up weights, resident on the GPU; the top-k is computed exactly from
 *   the native BF16 weights; skipped channels are recovered through a
 *   low-rank map of the down projections.
 *
 * Everything else is a reading the pages leave open; each function states the
 * reading it takes.  Compiled with -O2 -ffp-contract=off and no fast-math so
 * every float operation is one correctly rounded IEEE operation in the order
 * written.
 *
 * Parity status: every function here is pinned by the not-gpu tests
 * (closed forms, invariants, brute force); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 */

static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even,
 * with a single rounding.  Values are O(1) here; the subnormal bf16 range
 * is not needed and is flushed through the float path. */
uint16_t orc_double_to_bf16(double v) {
    if (v == 0.0 || isnan(v) || isinf(v)) {
        float f = (float)v;
        uint32_t u;
        memcpy(&u, &f, 4);
        return (uint16_t)(u >> 16);
    }
    int e;
    double m = frexp(fabs(v), &e);          /* |v| = m * 2^e, m in [0.5, 1) */
    double r = nearbyint(ldexp(m, 8));      /* 8 significant bits, half-even */
    double out = ldexp(r, e - 8);
    if (v < 0) out = -out;
    float f = (float)out;                   /* exact: 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

void orc_double_to_bf16_array(long n, const double* v, uint16_t* out) {
    for (long i = 0; i < n; i++) out[i] = orc_double_to_bf16(v[i]);
}

/* -------------------------------------------------------------- SplitMix64
 * Rotation signs are random numbers the method draws; both sides implement
 * the same counter-based generator from its published definition: SplitMix64
 * (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014).  Output j (0-based) of the stream seeded with `seed` is
 * mix(seed + (j+1)*gamma). */
uint64_t orc_splitmix64_at(uint64_t seed, uint64_t j) {
    uint64_t z = seed + (j + 1) * 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* s_j = +1 when the top bit of output j is 0, else -1. */
void orc_rot_signs(int d, uint64_t seed, int8_t* s) {
    for (int j = 0; j < d; j++)
        s[j] = (orc_splitmix64_at(seed, (uint64_t)j) >> 63) ? (int8_t)-1 : (int8_t)1;
}

/* ------------------------------------------------------------------- FWHT
 * Unnormalised fast Walsh-Hadamard transform in Sylvester order, fp32.
 * Reading: the pages say only "rotated"; the rotation here is the
 * randomized Hadamard x -> H (s . x).  The stage order is fixed (h = 1, 2,
 * 4, ...) so that any implementation doing the same butterflies per stage
 * produces the same bits. */
void orc_fwht(int d, float* v) {
    for (int h = 1; h < d; h *= 2)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; j++) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* ------------------------------------------------------------ exp and SiLU
 * exp_r: a self-contained exp so that both sides take the screening decisions
 * on identical bits.  Method: Cody & Waite argument reduction (Cody & Waite,
 * "Software Manual for the Elementary Functions", 1980) with ln 2 split into a
 * 16-significant-bit head (so n*LN2_HI is exact for |n| < 256) and a tail;
 * then the degree-7 Taylor polynomial of exp(r), |r| <= ln2/2, in Horner form
 * with correctly rounded fused multiply-adds; then an exact scale by 2^n.
 * The input is clamped to [-87, 88] so the result is always a normal float. */
static const float ORC_LOG2E  = 0x1.715476p+0f;     /* (float) 1/ln 2          */
static const float ORC_LN2_HI = 0x1.62e4p-1f;       /* ln 2 truncated, 16 bits */
static const float ORC_LN2_LO = 0x1.7f7d1cp-20f;    /* (float)(ln 2 - LN2_HI)  */
static const float ORC_INV_FACT[8] = {               /* (float)(1/k!)           */
    1.0f, 1.0f, 0.5f, 0x1.555556p-3f, 0x1.555556p-5f,
    0x1.111112p-7f, 0x1.6c16c2p-10f, 0x1.a01a02p-13f};

float orc_exp_r(float t) {
    if (t < -87.0f) t = -87.0f;
    if (t > 88.0f) t = 88.0f;
    float n = rintf(t * ORC_LOG2E);
    float r = fmaf(-n, ORC_LN2_HI, t);
    r = fmaf(-n, ORC_LN2_LO, r);
    float p = ORC_INV_FACT[7];
    for (int k = 6; k >= 0; k--) p = fmaf(p, r, ORC_INV_FACT[k]);
    int ni = (int)n;
    uint32_t bits = (uint32_t)(ni + 127) << 23;
    float two_n;
    memcpy(&two_n, &bits, 4);
    return p * two_n;
}

float orc_silu_r(float t) { return t / (1.0f + orc_exp_r(-t)); }

/* ------------------------------------------------- rotate + int8 quantize
 * v = FWHT(s . x) in fp32; amax = max |v_j|; q_j = rint((v_j * 127) / amax)
 * (round half to even, clamped to +-127); c_x = amax / (127 d).  The sketch
 * dot T.q times alpha*c_x estimates the exact dot w.x, since H^T H = d I.
 * Reading: int8 rotated activations (so sketch dots are exact int32) and
 * this operation order are choices the pages leave open. */
void orc_rotate_quantize(int d, const uint16_t* x, const int8_t* s,
                         float* v, int8_t* q, float* cx) {
    for (int j = 0; j < d; j++) v[j] = (float)s[j] * bf16_to_f32(x[j]);
    orc_fwht(d, v);
    float amax = 0.0f;
    for (int j = 0; j < d; j++)
        if (fabsf(v[j]) > amax) amax = fabsf(v[j]);
    if (amax == 0.0f) {
        for (int j = 0; j < d; j++) q[j] = 0;
        *cx = 0.0f;
        return;
    }
    for (int j = 0; j < d; j++) {
        float t = (v[j] * 127.0f) / amax;
        long n = lrintf(t);
        if (n > 127) n = 127;
        if (n < -127) n = -127;
        q[j] = (int8_t)n;
    }
    *cx = amax / (127.0f * (float)d);
}

/* ----------------------------------------------------------- ternary sketch
 * One gate or up row w (channel i of expert e): w' = FWHT(s . w) (fp32, as
 * above), then a TWN ternarisation (Li & Liu, "Ternary Weight Networks",
 * 2016): Delta = 0.7 * mean_j |w'_j|; T_j = sign(w'_j) where |w'_j| > Delta,
 * else 0; alpha = mean of |w'_j| over the nonzero T_j (0 when there are none).
 * Both sums are fp64 in index order.  Reading: TWN with 0.7 and a per-row
 * scale are the choices for the pages' "ternary sketch"; the fp64 index-order
 * sums make both builders agree bit for bit. */
void orc_twn_row(int d, const uint16_t* w, const int8_t* s, int8_t* trit,
                 float* alpha, float* wrot /* [d] scratch/out */) {
    for (int j = 0; j < d; j++) wrot[j] = (float)s[j] * bf16_to_f32(w[j]);
    orc_fwht(d, wrot);
    double sabs = 0.0;
    for (int j = 0; j < d; j++) sabs += fabs((double)wrot[j]);
    double delta = 0.7 * (sabs / (double)d);
    double snz = 0.0;
    int nnz = 0;
    for (int j = 0; j < d; j++) {
        double a = fabs((double)wrot[j]);
        if (a > delta) {
            trit[j] = wrot[j] > 0.0f ? 1 : -1;
            snz += a;
            nnz++;
        } else {
            trit[j] = 0;
        }
    }
    *alpha = nnz ? (float)(snz / (double)nnz) : 0.0f;
}

/* 2-bit packing, 16 trits per uint32 word; word m of a row holds positions
 * 16m .. 16m+15.  Position 16m + 4p + b (p, b in 0..3) sits at bits
 * [8b + 2p, 8b + 2p + 1] as the unsigned code T + 1 (00 = -1, 01 = 0,
 * 10 = +1; 11 is never written).  Reading: the pages fix no layout.  In this
 * one, masking a word with 0x03030303 << 2p leaves four byte lanes that a
 * byte-wise dot product multiplies with the int8 activations of positions
 * 16m + 4p .. 16m + 4p + 3; the code offset is removed once per row by
 * subtracting the sum of the activations. */
static int trit_shift(int n /* 0..15 */) { return 8 * (n % 4) + 2 * (n / 4); }

void orc_pack_trits(int d, const int8_t* trit, uint32_t* packed) {
    for (int k = 0; k < d / 16; k++) packed[k] = 0;
    for (int j = 0; j < d; j++) {
        uint32_t code = (uint32_t)(trit[j] + 1);
        packed[j / 16] |= code << trit_shift(j % 16);
    }
}

int orc_unpack_trit(const uint32_t* packed, int j) {
    uint32_t code = (packed[j / 16] >> trit_shift(j % 16)) & 3u;
    return (int)code - 1;
}

/* Base-3 packing of a ternary row, five trits per byte ("KAIST: MoE Decoding
 * Needs No Calibration Data", section "A reader that needs no data at all":
 * the resident sketch is about 7% of the BF16 weights; 2-bit codes give
 * 8.3%, base 3 with five trits per byte 6.7%).  Byte g holds trits 5g .. 5g+4
 * as sum over i of (t_{5g+i} + 1) * 3^i, at most 242; a row of d trits takes
 * ceil(d / 5) bytes, the last one padded with zero trits (digit 1). */
void orc_pack_trits_base3(int d, const int8_t* trit, uint8_t* packed) {
    const int nb = (d + 4) / 5;
    for (int g = 0; g < nb; g++) {
        int v = 0, pw = 1;
        for (int i = 0; i < 5; i++) {
            const int j = 5 * g + i;
            const int digit = j < d ? trit[j] + 1 : 1;
            v += digit * pw;
            pw *= 3;
        }
        packed[g] = (uint8_t)v;
    }
}

void orc_unpack_trits_base3(int d, const uint8_t* packed, int8_t* trit) {
    for (int j = 0; j < d; j++) {
        int v = packed[j / 5];
        for (int i = 0; i < j % 5; i++) v /= 3;
        trit[j] = (int8_t)(v % 3 - 1);
    }
}

/* Sketch of every gate and up row of E experts: sk[E, I, d/16], alpha[E, I]. */
void orc_build_sketch(int E, int I, int d, const uint16_t* w_gate, const uint16_t* w_up,
                      uint64_t rot_seed, int8_t* rot_sign, uint32_t* sk_gate,
                      uint32_t* sk_up, float* alpha_gate, float* alpha_up) {
    orc_rot_signs(d, rot_seed, rot_sign);
    int8_t* trit = (int8_t*)malloc((size_t)d);
    float* wrot = (float*)malloc(sizeof(float) * (size_t)d);
    for (int m = 0; m < 2; m++) {
        const uint16_t* W = m ? w_up : w_gate;
        uint32_t* SK = m ? sk_up : sk_gate;
        float* AL = m ? alpha_up : alpha_gate;
        for (long row = 0; row < (long)E * I; row++) {
            orc_twn_row(d, W + row * d, rot_sign, trit, &AL[row], wrot);
            orc_pack_trits(d, trit, SK + row * (d / 16));
        }
    }
    free(trit);
    free(wrot);
}

/* -------------------------------------------------------------------- router
 * Routed experts (abstract).  logit_e = sum_j W_r[e,j] x_j (+ b_e): every
 * bf16*bf16 product is exact in fp64 and the sum runs in index order in fp64.
 * Top-`top_e` by logit descending, ties to the lower expert id, slot 0 the
 * largest.  Weights: softmax over the chosen logits (fp64), stored fp32.
 * Reading: "top-8 softmax-renormalised" = softmax over all experts, keep the
 * top 8, renormalise -- identical to a softmax over the 8 chosen logits. */
static _Thread_local const double* g_sort_logits; /* qsort context, per thread */
static int cmp_logit_desc(const void* a, const void* b) {
    int ia = *(const int*)a, ib = *(const int*)b;
    double la = g_sort_logits[ia], lb = g_sort_logits[ib];
    if (la > lb) return -1;
    if (la < lb) return 1;
    return ia - ib;
}

void orc_route(int B, int E, int d, int top_e, const uint16_t* x, const uint16_t* w_router,
               const float* bias, double* logits, int32_t* ids, float* weights) {
    int* order = (int*)malloc(sizeof(int) * (size_t)E);
    for (int b = 0; b < B; b++) {
        double* L = logits + (long)b * E;
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int j = 0; j < d; j++)
                acc += (double)bf16_to_f32(w_router[(long)e * d + j]) *
                       (double)bf16_to_f32(x[(long)b * d + j]);
            if (bias) acc += (double)bias[e];
            L[e] = acc;
        }
        for (int e = 0; e < E; e++) order[e] = e;
        g_sort_logits = L;
        qsort(order, (size_t)E, sizeof(int), cmp_logit_desc);
        double mx = L[order[0]], den = 0.0;
        for (int s = 0; s < top_e; s++) den += exp(L[order[s]] - mx);
        for (int s = 0; s < top_e; s++) {
            ids[b * top_e + s] = order[s];
            weights[b * top_e + s] = (float)(exp(L[order[s]] - mx) / den);
        }
    }
    free(order);
}

/* ---------------------------------------------------------- top-n selection
 * Keep the n indices with the largest key; ties go to the lower index, i.e.
 * sort by (key descending, index ascending) and take the first n.  The result
 * is returned in ascending index order. */
static _Thread_local const float* g_sort_keys;    /* qsort context, per thread */
static int cmp_key_desc(const void* a, const void* b) {
    int ia = *(const int*)a, ib = *(const int*)b;
    float ka = g_sort_keys[ia], kb = g_sort_keys[ib];
    if (ka > kb) return -1;
    if (ka < kb) return 1;
    return ia - ib;
}
static int cmp_int_asc(const void* a, const void* b) {
    return *(const int*)a - *(const int*)b;
}

/* idx[0..m) are the eligible indices into key[]; writes the chosen n to out. */
void orc_top_n(int m, const int32_t* idx, const float* key, int n, int32_t* out) {
    int* tmp = (int*)malloc(sizeof(int) * (size_t)(m > 0 ? m : 1));
    for (int t = 0; t < m; t++) tmp[t] = idx[t];
    g_sort_keys = key;
    qsort(tmp, (size_t)m, sizeof(int), cmp_key_desc);
    for (int t = 0; t < n; t++) out[t] = tmp[t];
    qsort(out, (size_t)n, sizeof(int), cmp_int_asc);
    free(tmp);
}

/* Exact-stage dot of one BF16 row with x: fp64 sum in index order, rounded
 * once to fp32 (the products are exact in fp64). */
static float exact_dot(const uint16_t* row, const uint16_t* x, int d) {
    double s = 0.0;
    for (int j = 0; j < d; j++) s += (double)bf16_to_f32(row[j]) * (double)bf16_to_f32(x[j]);
    return (float)s;
}

/* -------------------------------------------- one (token, routed expert) pair
 * The reader, in the order the pages give it ("A reader that needs no data
 * at all"; abstract):
 *  1. screen: G_i = T^g_i . q, U_i = T^u_i . q (exact integers);
 *     ghat_i = ((float)G_i * alpha^g_i) * c_x, uhat_i likewise;
 *     ahat_i = silu_r(ghat_i) * uhat_i; sigma_i = |ahat_i|.
 *     Reading: the screening score is the exact-stage score evaluated on the
 *     sketch estimates.
 *  2. candidates: the c channels with the largest sigma (ties: lower i).
 *  3. exact: g_i = W_gate[i,:].x, u_i = W_up[i,:].x from the BF16 rows
 *     (fp64 sum, rounded once to fp32), a_i = silu_r(g_i) * u_i (fp32).
 *  4. keep: the k candidates with the largest |a_i| (ties: lower i) -- the
 *     per-token top-k rule of the abstract.
 *  5. read only the kept down rows and recover the skipped channels through
 *     the low-rank map W_down ~ Ubar V^T:
 *        y_e = sum_{i in K} a_i W_down[i,:] + V z,
 *        z   = sum_{i not in K} ahat_i Ubar[i,:].
 *     Reading: the map is applied to the sketch estimates of every skipped
 *     channel.  Accumulation is fp64.
 *     recovery_input == 1 is the variant that feeds the map the exact a_i
 *     of the candidates step 4 dropped (computed in step 3 anyway) and the
 *     sketch estimates only outside the candidate set:
 *        z = sum_{i in C, i not in K} a_i Ubar[i,:] + sum_{i not in C} ahat_i Ubar[i,:].
 * exact_mode != 0 replaces the sketch estimates by the exact g, u (a test
 * mode for the invariant "exact sketch + full-rank map = dense expert").
 * r == 0 or ubar == NULL disables recovery. */
void orc_expert_reader(int I, int d, int k, int c, int r, int exact_mode, int recovery_input,
                       const uint16_t* x, const int8_t* q, float cx,
                       const uint32_t* skg, const uint32_t* sku,
                       const float* ag, const float* au,
                       const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                       const uint16_t* ubar, const uint16_t* vmap,
                       double* y_e,
                       int32_t* dbg_G, int32_t* dbg_U, float* dbg_sigma,
                       int32_t* dbg_cand, int32_t* dbg_kept, float* dbg_a_kept) {
    const int words = d / 16;
    float* ahat = (float*)malloc(sizeof(float) * (size_t)I);
    float* sigma = (float*)malloc(sizeof(float) * (size_t)I);
    float* a = (float*)calloc((size_t)I, sizeof(float));
    float* absa = (float*)calloc((size_t)I, sizeof(float));
    int32_t* all = (int32_t*)malloc(sizeof(int32_t) * (size_t)I);
    int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * (size_t)c);
    int32_t* kept = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    char* is_kept = (char*)calloc((size_t)I, 1);


    for (int i = 0; i < I; i++) {
        float gh, uh;
        if (exact_mode) {
            gh = exact_dot(wg + (long)i * d, x, d);
            uh = exact_dot(wu + (long)i * d, x, d);
        } else {
            long G = 0, U = 0;
            for (int j = 0; j < d; j++) {
                G += (long)orc_unpack_trit(skg + (long)i * words, j) * q[j];
                U += (long)orc_unpack_trit(sku + (long)i * words, j) * q[j];
            }
            if (dbg_G) dbg_G[i] = (int32_t)G;
            if (dbg_U) dbg_U[i] = (int32_t)U;
            gh = ((float)G * ag[i]) * cx;
            uh = ((float)U * au[i]) * cx;
        }
        ahat[i] = orc_silu_r(gh) * uh;
        sigma[i] = fabsf(ahat[i]);
        if (dbg_sigma) dbg_sigma[i] = sigma[i];
        all[i] = i;
    }
    orc_top_n(I, all, sigma, c, cand);
    for (int t = 0; t < c; t++) {
        int i = cand[t];
        float g = exact_dot(wg + (long)i * d, x, d), u = exact_dot(wu + (long)i * d, x, d);
        a[i] = orc_silu_r(g) * u;
        absa[i] = fabsf(a[i]);
    }
    orc_top_n(c, cand, absa, k, kept);
    for (int t = 0; t < k; t++) is_kept[kept[t]] = 1;
    char* is_cand = (char*)calloc((size_t)I, 1);
    for (int t = 0; t < c; t++) is_cand[cand[t]] = 1;
    if (dbg_cand) memcpy(dbg_cand, cand, sizeof(int32_t) * (size_t)c);
    if (dbg_kept) memcpy(dbg_kept, kept, sizeof(int32_t) * (size_t)k);
    if (dbg_a_kept)
        for (int t = 0; t < k; t++) dbg_a_kept[t] = a[kept[t]];

    for (int j = 0; j < d; j++) y_e[j] = 0.0;
    for (int t = 0; t < k; t++) {
        int i = kept[t];
        for (int j = 0; j < d; j++)
            y_e[j] += (double)a[i] * (double)bf16_to_f32(wd[(long)i * d + j]);
    }
    if (r > 0 && ubar && vmap) {
        double* z = (double*)calloc((size_t)r, sizeof(double));
        for (int i = 0; i < I; i++) {
            if (is_kept[i]) continue;
            const double zi = (recovery_input == 1 && is_cand[i]) ? (double)a[i] : (double)ahat[i];
            for (int p = 0; p < r; p++)
                z[p] += zi * (double)bf16_to_f32(ubar[(long)i * r + p]);
        }
        for (int j = 0; j < d; j++) {
            double acc = 0.0;
            for (int p = 0; p < r; p++)
                acc += (double)bf16_to_f32(vmap[(long)j * r + p]) * z[p];
            y_e[j] += acc;
        }
        free(z);
    }
    free(ahat); free(sigma); free(a); free(absa); free(all);
    free(cand); free(kept); free(is_kept); free(is_cand);
}

/* ------------------------------------------------------------ whole forward
 * One MoE block over B tokens: route, rotate+quantize, reader per (token,
 * slot), then y_b = sum over slots (routing order) of w * y_e, fp64, rounded
 * once to bf16.  If `residual` is given, it is added before the rounding.
 * Debug arrays (any may be NULL) are laid out [B, top_e, ...].  `threads` > 1
 * runs the (token, slot) readers on that many OpenMP threads; every pair is
 * independent and the combine stays serial, so the result is the same bits
 * for any thread count. */
void orc_forward(int B, int E, int top_e, int I, int d, int k, int c, int r, int exact_mode, int recovery_input,
                 const uint16_t* x, const uint16_t* w_router, const float* bias,
                 const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                 const int8_t* rot_sign, const uint32_t* sk_gate, const uint32_t* sk_up,
                 const float* alpha_gate, const float* alpha_up,
                 const uint16_t* ubar, const uint16_t* vmap, const uint16_t* residual,
                 uint16_t* y, double* y_f64,
                 int32_t* dbg_ids, float* dbg_w, int32_t* dbg_G, int32_t* dbg_U,
                 float* dbg_sigma, int32_t* dbg_cand, int32_t* dbg_kept,
                 float* dbg_a_kept, double* dbg_y_expert, int threads) {
    double* logits = (double*)malloc(sizeof(double) * (size_t)B * E);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)B * top_e);
    float* w = (float*)malloc(sizeof(float) * (size_t)B * top_e);
    float* v = (float*)malloc(sizeof(float) * (size_t)d);
    int8_t* q = (int8_t*)malloc((size_t)B * d);
    float* cx = (float*)malloc(sizeof(float) * (size_t)B);
    double* ye = (double*)malloc(sizeof(double) * (size_t)B * top_e * d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    orc_route(B, E, d, top_e, x, w_router, bias, logits, ids, w);
    const long rowsz = (long)I * d, skrow = (long)I * (d / 16);
    for (int b = 0; b < B; b++) orc_rotate_quantize(d, x + (long)b * d, rot_sign, v, q + (long)b * d, &cx[b]);
    /* the reader of every (token, slot) pair */
    const long npairs = (long)B * top_e;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 1 ? threads : 1) if (threads > 1)
    for (long ps = 0; ps < npairs; ps++) {
        const int b = (int)(ps / top_e);
        const int e = ids[ps];
        orc_expert_reader(I, d, k, c, r, exact_mode, recovery_input, x + (long)b * d, q + (long)b * d, cx[b],
                          sk_gate + e * skrow, sk_up + e * skrow,
                          alpha_gate + (long)e * I, alpha_up + (long)e * I,
                          w_gate + e * rowsz, w_up + e * rowsz, w_down + e * rowsz,
                          ubar ? ubar + (long)e * I * r : NULL,
                          vmap ? vmap + (long)e * d * r : NULL, ye + ps * d,
                          dbg_G ? dbg_G + ps * I : NULL, dbg_U ? dbg_U + ps * I : NULL,
                          dbg_sigma ? dbg_sigma + ps * I : NULL,
                          dbg_cand ? dbg_cand + ps * c : NULL,
                          dbg_kept ? dbg_kept + ps * k : NULL,
                          dbg_a_kept ? dbg_a_kept + ps * k : NULL);
    }
    /* combine, slots in routing order */
    for (int b = 0; b < B; b++) {
        for (int j = 0; j < d; j++) acc[j] = 0.0;
        for (int s = 0; s < top_e; s++) {
            const long ps = (long)b * top_e + s;
            if (dbg_y_expert) memcpy(dbg_y_expert + ps * d, ye + ps * d, sizeof(double) * (size_t)d);
            for (int j = 0; j < d; j++) acc[j] += (double)w[ps] * ye[ps * d + j];
        }
        for (int j = 0; j < d; j++) {
            double o = acc[j] + (residual ? (double)bf16_to_f32(residual[(long)b * d + j]) : 0.0);
            if (y_f64) y_f64[(long)b * d + j] = o;
            y[(long)b * d + j] = orc_double_to_bf16(o);
        }
    }
    if (dbg_ids) memcpy(dbg_ids, ids, sizeof(int32_t) * (size_t)B * top_e);
    if (dbg_w) memcpy(dbg_w, w, sizeof(float) * (size_t)B * top_e);
    free(logits); free(ids); free(w); free(v); free(q); free(cx); free(ye); free(acc);
}

/* ------------------------------------------------------------ dense expert
 * The all-channel SwiGLU expert that the reader approximates:
 * y_e = sum_i silu(g_i) u_i W_down[i,:], with g, u, silu and the sums in
 * fp64 (libm exp).  Used for the dense block and for the invariants. */
void orc_forward_dense(int B, int E, int top_e, int I, int d,
                       const uint16_t* x, const uint16_t* w_router, const float* bias,
                       const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                       const uint16_t* residual, uint16_t* y, double* y_f64) {
    double* logits = (double*)malloc(sizeof(double) * (size_t)B * E);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)B * top_e);
    float* w = (float*)malloc(sizeof(float) * (size_t)B * top_e);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    orc_route(B, E, d, top_e, x, w_router, bias, logits, ids, w);
    const long rowsz = (long)I * d;
    for (int b = 0; b < B; b++) {
        const uint16_t* xb = x + (long)b * d;
        for (int j = 0; j < d; j++) acc[j] = 0.0;
        for (int s = 0; s < top_e; s++) {
            int e = ids[b * top_e + s];
            const uint16_t *wg = w_gate + e * rowsz, *wu = w_up + e * rowsz, *wd = w_down + e * rowsz;
            for (int i = 0; i < I; i++) {
                double g = 0.0, u = 0.0;
                for (int j = 0; j < d; j++) {
                    double xj = (double)bf16_to_f32(xb[j]);
                    g += (double)bf16_to_f32(wg[(long)i * d + j]) * xj;
                    u += (double)bf16_to_f32(wu[(long)i * d + j]) * xj;
                }
                double h = g / (1.0 + exp(-g)) * u * (double)w[b * top_e + s];
                for (int j = 0; j < d; j++) acc[j] += h * (double)bf16_to_f32(wd[(long)i * d + j]);
            }
        }
        for (int j = 0; j < d; j++) {
            double o = acc[j] + (residual ? (double)bf16_to_f32(residual[(long)b * d + j]) : 0.0);
            if (y_f64) y_f64[(long)b * d + j] = o;
            y[(long)b * d + j] = orc_double_to_bf16(o);
        }
    }
    free(logits); free(ids); free(w); free(acc);
}

/* ------------------------------------------------------------------ RMSNorm
 * Between the layers of the stacked block: h = x / sqrt(mean(x^2) + eps),
 * no learned gain, fp64, rounded once to bf16. */
void orc_rmsnorm(int B, int d, double eps, const uint16_t* x, uint16_t* h) {
    for (int b = 0; b < B; b++) {
        double ss = 0.0;
        for (int j = 0; j < d; j++) {
            double t = (double)bf16_to_f32(x[(long)b * d + j]);
            ss += t * t;
        }
        double inv = 1.0 / sqrt(ss / (double)d + eps);
        for (int j = 0; j < d; j++)
            h[(long)b * d + j] = orc_double_to_bf16((double)bf16_to_f32(x[(long)b * d + j]) * inv);
    }
}
