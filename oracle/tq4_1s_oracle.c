/*
 * TQ4_1S ("Config-I") CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar C implementation of what the TQ4_1S layer computes,
 * written from the Nemotron-TheHobbit-30B-A3B model card, section
 * "What Config-I means": a Walsh-Hadamard (RHT) rotation applied per
 * 32-element block, then 4-bit, 16-level Lloyd-Max quantization with two
 * half-block scales, about 5 bits per weight; section "Running it": the
 * quantized Linears dequantize on the fly; section "Performance": a sync-free
 * MoE with bf16 tensor-core matmuls; section "The model underneath": a
 * 128-expert, top-6 MoE.
 *
 * Only the test suite, the package's smoke entry and the bench's CPU-baseline
 * leg may load this library.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Readings of points the pages leave open (each is also listed in the design
 * notes):
 *  - Codebook: the Lloyd-Max quantizer of N(0,1) with 16 levels, computed by
 *    Lloyd iteration in double; fp32 tables are the round-to-nearest images
 *    of the double levels and of the double midpoints.
 *  - Signs: one 32-sign vector per tensor, bit i of the low 32 bits of the
 *    first SplitMix64 output for the tensor's seed; bit set => s_i = -1.
 *  - Hadamard: Sylvester (natural) order, scaled by r = fp32(1/sqrt(32)).
 *  - Quantize arithmetic: a fixed fp32 op sequence (butterfly stages
 *    h = 1,2,4,8,16; v = a*r; half-block mean square by a pairwise tree with
 *    strides 8,4,2,1; rms = sqrt; scale d = fp16(rms), saturating; code =
 *    number of fp32 thresholds strictly below v/d; d == 0 => codes 7).
 *  - Packing: codes plane [n][k/2] (even index in the low nibble) and scales
 *    plane [n][k/16] of fp16 bits.
 *  - Linear: y = bf16(sum_k x*W_hat) with the sum in fp64; no bias.
 *  - MoE: u = x*W_up^T, h = bf16(relu(u)^2), z = h*W_down^T,
 *    y = bf16(sum_j w_j z_j) over the top-k slots in slot order.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fexcess-precision=standard
 *        -shared -fPIC (no fast-math; every fp32 op rounds once).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 32
#define ORC_HALF 16
#define ORC_LEVELS 16

/* ------------------------------------------------------------------ */
/* Lloyd-Max codebook for N(0,1), 16 levels (model card, "What Config-I
 * means": "16-level Lloyd-Max").                                       */

static double orc_phi(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * M_PI); }

/* P(a < X < b) for X ~ N(0,1), written with erfc on the side that keeps the
 * subtraction away from cancellation. */
static double orc_mass(double a, double b) {
    const double s = 1.0 / sqrt(2.0);
    if (a >= 0.0) return 0.5 * (erfc(a * s) - erfc(b * s));
    if (b <= 0.0) return 0.5 * (erfc(-b * s) - erfc(-a * s));
    return 1.0 - 0.5 * erfc(-a * s) - 0.5 * erfc(b * s);
}

/* Returns the number of iterations used, or -1 if it did not converge.
 * c[16] levels, t[15] midpoints (double); c32/t32 their fp32 roundings. */
int orc_codebook(double *c, double *t, float *c32, float *t32) {
    double lv[ORC_LEVELS], th[ORC_LEVELS - 1];
    for (int j = 0; j < ORC_LEVELS; j++) lv[j] = -2.5 + 5.0 * j / (ORC_LEVELS - 1);
    int it;
    for (it = 1; it <= 200000; it++) {
        for (int j = 0; j < ORC_LEVELS - 1; j++) th[j] = 0.5 * (lv[j] + lv[j + 1]);
        double delta = 0.0;
        for (int j = 0; j < ORC_LEVELS; j++) {
            double a = (j == 0) ? -INFINITY : th[j - 1];
            double b = (j == ORC_LEVELS - 1) ? INFINITY : th[j];
            double pa = (j == 0) ? 0.0 : orc_phi(a);
            double pb = (j == ORC_LEVELS - 1) ? 0.0 : orc_phi(b);
            double nv = (pa - pb) / orc_mass(a, b);
            double d = fabs(nv - lv[j]);
            if (d > delta) delta = d;
            lv[j] = nv;
        }
        if (delta < 1e-13) break;
    }
    /* N(0,1) is symmetric and so is the start, so the exact fixed point is
     * odd-symmetric (c_{15-j} = -c_j, middle threshold 0); remove the
     * rounding noise that breaks this by averaging the two halves. */
    for (int j = 0; j < ORC_LEVELS / 2; j++) {
        double mag = 0.5 * (lv[ORC_LEVELS - 1 - j] - lv[j]);
        lv[ORC_LEVELS - 1 - j] = mag;
        lv[j] = -mag;
    }
    for (int j = 0; j < ORC_LEVELS - 1; j++) th[j] = 0.5 * (lv[j] + lv[j + 1]);
    for (int j = 0; j < ORC_LEVELS; j++) { c[j] = lv[j]; c32[j] = (float)lv[j]; }
    for (int j = 0; j < ORC_LEVELS - 1; j++) { t[j] = th[j]; t32[j] = (float)th[j]; }
    return it > 200000 ? -1 : it;
}

/* ------------------------------------------------------------------ */
/* Signs: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), first output for the given state.   */
uint64_t orc_splitmix64_first(uint64_t state) {
    uint64_t z = state + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint32_t orc_sign_mask(uint64_t seed) { return (uint32_t)(orc_splitmix64_first(seed) & 0xFFFFFFFFULL); }

/* Sylvester Hadamard matrix, natural order: H[i][j] = (-1)^popcount(i&j). */
void orc_hadamard32(int8_t *H) {
    for (int i = 0; i < ORC_BLOCK; i++)
        for (int j = 0; j < ORC_BLOCK; j++) {
            int p = __builtin_popcount((unsigned)(i & j)) & 1;
            H[i * ORC_BLOCK + j] = p ? -1 : 1;
        }
}

static float orc_r32(void) { return (float)(1.0 / sqrt(32.0)); }

/* ------------------------------------------------------------------ */
/* Number formats.                                                      */

float orc_f16_to_f32(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return (float)(s ? -v : v);
}

/* float -> fp16, round to nearest even, saturating to +-65504 (infinities
 * included), subnormals kept; any NaN -> 0x7E00 (the sign of a NaN is not
 * portable across processors, so it is dropped). */
uint16_t orc_f32_to_f16_sat(float f) {
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    if (isnan(f)) return 0x7E00;
    double a = fabs((double)f);
    if (a >= 65520.0) return sign | 0x7BFF;
    if (a < ldexp(1.0, -14)) {                 /* subnormal range: m * 2^-24 */
        double m = rint(a * ldexp(1.0, 24));   /* exact scaling, RNE */
        return sign | (uint16_t)m;             /* m == 1024 encodes 2^-14 */
    }
    int e;
    frexp(a, &e);                              /* a = f * 2^e, f in [0.5,1) */
    e -= 1;                                    /* a in [2^e, 2^(e+1)) */
    double q = rint(ldexp(a, 10 - e));         /* 1024 .. 2048 */
    if (q >= 2048.0) { q = 1024.0; e += 1; }
    if (e > 15) return sign | 0x7BFF;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

/* double -> bf16, one rounding to nearest even. */
uint16_t orc_f64_to_bf16(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return sign | 0x7FC0;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7F80;
    if (a < ldexp(1.0, -126)) {                /* bf16 subnormal: m * 2^-133 */
        double m = rint(ldexp(a, 133));
        return sign | (uint16_t)m;             /* m == 128 encodes 2^-126 */
    }
    int e;
    frexp(a, &e);
    e -= 1;
    double q = rint(ldexp(a, 7 - e));          /* 128 .. 256 */
    if (q >= 256.0) { q = 128.0; e += 1; }
    if (e > 127) return sign | 0x7F80;         /* overflow rounds to inf */
    return sign | (uint16_t)(((e + 127) << 7) | ((int)q - 128));
}

double orc_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* Block rotation in the fixed fp32 op order.                           */

/* In-place 32-point Hadamard butterfly, stages h = 1,2,4,8,16; each stage
 * maps (a_j, a_{j+h}) -> (a_j + a_{j+h}, a_j - a_{j+h}) for j with bit h
 * clear.  Computes H*a for the natural-order Sylvester matrix. */
void orc_fwht32_f32(float *a) {
    for (int h = 1; h < ORC_BLOCK; h <<= 1)
        for (int j = 0; j < ORC_BLOCK; j++)
            if (!(j & h)) {
                float x = a[j], y = a[j + h];
                a[j] = x + y;
                a[j + h] = x - y;
            }
}

/* v = r * H * diag(s) * w, fp32. */
void orc_rotate_block(const float *w, uint32_t mask, float *v) {
    float a[ORC_BLOCK];
    for (int i = 0; i < ORC_BLOCK; i++) a[i] = ((mask >> i) & 1u) ? -w[i] : w[i];
    orc_fwht32_f32(a);
    const float r = orc_r32();
    for (int i = 0; i < ORC_BLOCK; i++) v[i] = a[i] * r;
}

/* ------------------------------------------------------------------ */
/* Quantize: W[n][k] fp32 -> codes[n][k/2], scales[n][k/16] (fp16 bits).
 * Returns the number of 32-blocks that held a non-finite input.        */
int64_t orc_quantize(const float *W, int64_t n, int64_t k, uint64_t seed,
                     uint8_t *codes, uint16_t *scales) {
    double c[16], t[15];
    float c32[16], t32[15];
    orc_codebook(c, t, c32, t32);
    const uint32_t mask = orc_sign_mask(seed);
    int64_t bad = 0;
    for (int64_t row = 0; row < n; row++) {
        for (int64_t kb = 0; kb < k / ORC_BLOCK; kb++) {
            const float *w = W + row * k + kb * ORC_BLOCK;
            int finite = 1;
            for (int i = 0; i < ORC_BLOCK; i++) if (!isfinite(w[i])) finite = 0;
            if (!finite) bad++;
            float v[ORC_BLOCK];
            orc_rotate_block(w, mask, v);
            uint8_t q[ORC_BLOCK];
            for (int hh = 0; hh < 2; hh++) {
                const float *vh = v + hh * ORC_HALF;
                float p[ORC_HALF];
                for (int i = 0; i < ORC_HALF; i++) p[i] = vh[i] * vh[i];
                for (int s = 8; s >= 1; s >>= 1)
                    for (int i = 0; i < s; i++) p[i] = p[i] + p[i + s];
                float ms = p[0] * 0.0625f;
                float rms = sqrtf(ms);
                uint16_t dh = orc_f32_to_f16_sat(rms);
                scales[row * (k / ORC_HALF) + kb * 2 + hh] = dh;
                float d = orc_f16_to_f32(dh);
                for (int i = 0; i < ORC_HALF; i++) {
                    int code;
                    if (d == 0.0f) {
                        code = 7;
                    } else {
                        float u = vh[i] / d;
                        code = 0;
                        for (int j = 0; j < 15; j++) if (u > t32[j]) code++;
                    }
                    q[hh * ORC_HALF + i] = (uint8_t)code;
                }
            }
            uint8_t *cb = codes + row * (k / 2) + kb * (ORC_BLOCK / 2);
            for (int i = 0; i < ORC_BLOCK / 2; i++)
                cb[i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
        }
    }
    return bad;
}

/* Rotated-domain values of one 32-block: w_n_i = fp32(c32[code_i] * d_h). */
static void orc_block_levels(const uint8_t *cb, const uint16_t *sb, const float *c32, float *wn) {
    for (int i = 0; i < ORC_BLOCK; i++) {
        int code = (i & 1) ? (cb[i / 2] >> 4) : (cb[i / 2] & 0xF);
        float d = orc_f16_to_f32(sb[i / ORC_HALF]);
        wn[i] = c32[code] * d;
    }
}

/* Dequantize: W_hat = diag(s) * r * H * w_n per block (inverse rotation). */
void orc_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                    uint64_t seed, float *W) {
    double c[16], t[15];
    float c32[16], t32[15];
    orc_codebook(c, t, c32, t32);
    const uint32_t mask = orc_sign_mask(seed);
    const float r = orc_r32();
    for (int64_t row = 0; row < n; row++)
        for (int64_t kb = 0; kb < k / ORC_BLOCK; kb++) {
            float a[ORC_BLOCK];
            orc_block_levels(codes + row * (k / 2) + kb * 16, scales + row * (k / 16) + kb * 2, c32, a);
            orc_fwht32_f32(a);
            float *o = W + row * k + kb * ORC_BLOCK;
            for (int i = 0; i < ORC_BLOCK; i++) {
                float x = a[i] * r;
                o[i] = ((mask >> i) & 1u) ? -x : x;
            }
        }
}

/* Rotated-domain levels (no inverse rotation): w_n[n][k]. */
void orc_levels(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, float *wn) {
    double c[16], t[15];
    float c32[16], t32[15];
    orc_codebook(c, t, c32, t32);
    for (int64_t row = 0; row < n; row++)
        for (int64_t kb = 0; kb < k / ORC_BLOCK; kb++)
            orc_block_levels(codes + row * (k / 2) + kb * 16, scales + row * (k / 16) + kb * 2, c32,
                             wn + row * k + kb * ORC_BLOCK);
}

/* ------------------------------------------------------------------ */
/* Linear: y[m][n] = sum_k x[m][k] * W_hat[n][k] in fp64 (x bf16 bits).  */
void orc_linear(const uint16_t *x, int64_t m, int64_t k, const float *W, int64_t n, double *y) {
    for (int64_t i = 0; i < m; i++)
        for (int64_t j = 0; j < n; j++) {
            double s = 0.0;
            for (int64_t kk = 0; kk < k; kk++) s += orc_bf16_to_f64(x[i * k + kk]) * (double)W[j * k + kk];
            y[i * n + j] = s;
        }
}

void orc_round_bf16(const double *y, int64_t count, uint16_t *out) {
    for (int64_t i = 0; i < count; i++) out[i] = orc_f64_to_bf16(y[i]);
}

/* ------------------------------------------------------------------ */
/* MoE routing: bucket the (token, slot) pairs by expert, stable in
 * (token, slot) order.  offsets[e+1]; pairs[] holds t*topk + j.  Pairs with
 * an expert id outside [0, E) go to no bucket; their count is returned.  */
int64_t orc_moe_route(const int32_t *ids, int64_t m, int topk, int num_experts,
                      int32_t *offsets, int32_t *pairs) {
    int64_t bad = 0;
    for (int64_t p = 0; p < m * topk; p++)
        if (ids[p] < 0 || ids[p] >= num_experts) bad++;
    int32_t pos = 0;
    for (int e = 0; e < num_experts; e++) {
        offsets[e] = pos;
        for (int64_t p = 0; p < m * topk; p++)
            if (ids[p] == e) pairs[pos++] = (int32_t)p;
    }
    offsets[num_experts] = pos;
    return bad;
}

/* MoE router (model card, "The model underneath": each token is sent to 6 of
 * 128 experts; "Performance": the MoE runs without host syncs, so routing is
 * part of the layer).  Reading: the router's fp32 logits z [m][E] give the
 * softmax p_e = exp(z_e) / sum_i exp(z_i) over all E experts; the topk
 * experts of largest p are chosen and their p renormalised to sum to 1.
 * Softmax is monotone in z, so the choice is made on the fp32 z themselves
 * (equal z: the lower expert id first); selection order is descending.  The
 * softmax is taken in fp64 with the largest logit subtracted first (which
 * leaves p unchanged), the weights rounded to fp32 at the end.              */
void orc_router_topk(const float *z, int64_t m, int num_experts, int topk, int32_t *ids, float *w) {
    char *taken = (char *)malloc((size_t)num_experts);
    double *p = (double *)malloc(sizeof(double) * (size_t)num_experts);
    for (int64_t t = 0; t < m; t++) {
        const float *zt = z + t * num_experts;
        double zmax = -INFINITY;
        for (int e = 0; e < num_experts; e++)
            if ((double)zt[e] > zmax) zmax = (double)zt[e];
        double total = 0.0;
        for (int e = 0; e < num_experts; e++) {
            p[e] = exp((double)zt[e] - zmax);
            total += p[e];
        }
        for (int e = 0; e < num_experts; e++) p[e] /= total;
        memset(taken, 0, (size_t)num_experts);
        double sel = 0.0;
        for (int j = 0; j < topk; j++) {
            int best = -1;
            for (int e = 0; e < num_experts; e++) {
                if (taken[e]) continue;
                if (best < 0 || zt[e] > zt[best]) best = e;   /* strict: ties keep the lower id */
            }
            taken[best] = 1;
            ids[t * topk + j] = best;
            sel += p[best];
        }
        for (int j = 0; j < topk; j++) w[t * topk + j] = (float)(p[ids[t * topk + j]] / sel);
    }
    free(taken);
    free(p);
}

/* MoE layer.  x [m][H] bf16; ids/w [m][topk]; up codes/scales for E experts
 * of shape [I][H]; down codes/scales of shape [H][I].  Result y [m][H] in
 * fp64 before the final bf16 rounding.  Experts are dequantized one at a
 * time; each (token, slot) output z is computed on its own, and the slot sum
 * runs in slot order at the end.  Returns the number of pairs skipped for an
 * out-of-range expert id. */
int64_t orc_moe(const uint16_t *x, int64_t m, int64_t H, int64_t I,
                const int32_t *ids, const float *w, int topk, int num_experts,
                const uint8_t *up_codes, const uint16_t *up_scales, uint64_t up_seed,
                const uint8_t *dn_codes, const uint16_t *dn_scales, uint64_t dn_seed,
                double *y) {
    float *Wup = (float *)malloc(sizeof(float) * (size_t)(I * H));
    float *Wdn = (float *)malloc(sizeof(float) * (size_t)(H * I));
    double *z = (double *)calloc((size_t)(m * topk * H), sizeof(double));
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    int64_t bad = 0;
    for (int64_t p = 0; p < m * topk; p++)
        if (ids[p] < 0 || ids[p] >= num_experts) bad++;
    for (int e = 0; e < num_experts; e++) {
        int used = 0;
        for (int64_t p = 0; p < m * topk; p++) if (ids[p] == e) used = 1;
        if (!used) continue;
        orc_dequantize(up_codes + (size_t)e * I * (H / 2), up_scales + (size_t)e * I * (H / 16), I, H, up_seed, Wup);
        orc_dequantize(dn_codes + (size_t)e * H * (I / 2), dn_scales + (size_t)e * H * (I / 16), H, I, dn_seed, Wdn);
        for (int64_t p = 0; p < m * topk; p++) {
            if (ids[p] != e) continue;
            const uint16_t *xt = x + (p / topk) * H;
            for (int64_t i = 0; i < I; i++) {
                double s = 0.0;
                for (int64_t kk = 0; kk < H; kk++) s += orc_bf16_to_f64(xt[kk]) * (double)Wup[i * H + kk];
                u[i] = s;
            }
            for (int64_t i = 0; i < I; i++) {
                double r = u[i] > 0.0 ? u[i] : 0.0;
                hv[i] = orc_bf16_to_f64(orc_f64_to_bf16(r * r));
            }
            for (int64_t o = 0; o < H; o++) {
                double s = 0.0;
                for (int64_t i = 0; i < I; i++) s += hv[i] * (double)Wdn[o * I + i];
                z[p * H + o] = s;
            }
        }
    }
    for (int64_t t = 0; t < m; t++)
        for (int64_t o = 0; o < H; o++) {
            double s = 0.0;
            for (int j = 0; j < topk; j++) {
                int64_t p = t * topk + j;
                if (ids[p] < 0 || ids[p] >= num_experts) continue;
                s += (double)w[p] * z[p * H + o];
            }
            y[t * H + o] = s;
        }
    free(Wup); free(Wdn); free(z); free(u); free(hv);
    return bad;
}

/* ------------------------------------------------------------------ */
/* fp8-resident weight cache (model card "Nemotron-TheHobbit-30B-A3B",
 * section "Help wanted": dequantize once to fp8 and keep the weights
 * resident, ~63 GB, to remove the per-forward dequantization).  Reading:
 * fp8 = OCP E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, largest finite 448); one fp32 scale per output row n,
 * s_n = fp32(amax_n / 448) with amax_n = max_k |W_hat[n][k]|; codes
 * q = e4m3(fp32(W_hat / s_n)) rounded to nearest even, saturating at +-448;
 * a zero row has s_n = 0 and all codes 0.  The cached weight is s_n * q.  */

/* float -> E4M3 bits, round to nearest even, saturating to +-448; NaN -> 0x7F. */
uint8_t orc_f32_to_e4m3_sat(float f) {
    uint8_t sign = signbit(f) ? 0x80 : 0;
    if (isnan(f)) return 0x7F;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;            /* 1.75 * 2^8, the largest finite */
    if (a < ldexp(1.0, -6)) {                      /* subnormal range: m * 2^-9, m = 0..8 */
        double m = rint(ldexp(a, 9));
        return sign | (uint8_t)m;                  /* m == 8 encodes 2^-6 */
    }
    int e;
    frexp(a, &e);
    e -= 1;                                        /* a in [2^e, 2^(e+1)) */
    double q = rint(ldexp(a, 3 - e));              /* 8 .. 16 */
    if (q >= 16.0) { q = 8.0; e += 1; }
    if (e > 8 || (e == 8 && q > 14.0)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)q - 8));
}

double orc_e4m3_to_f64(uint8_t b) {
    int s = (b >> 7) & 1, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), e - 10);
    return s ? -v : v;
}

/* TQ4_1S weight [n][k] -> fp8 cache: codes q [n][k] and row scales s [n]. */
void orc_to_fp8(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, uint64_t seed,
                uint8_t *q, float *s) {
    float *W = (float *)malloc(sizeof(float) * (size_t)(n * k));
    orc_dequantize(codes, scales, n, k, seed, W);
    for (int64_t i = 0; i < n; i++) {
        float amax = 0.0f;
        for (int64_t j = 0; j < k; j++) {
            float a = fabsf(W[i * k + j]);
            if (a > amax) amax = a;
        }
        float sc = amax / 448.0f;
        s[i] = sc;
        for (int64_t j = 0; j < k; j++)
            q[i * k + j] = (sc == 0.0f) ? 0 : orc_f32_to_e4m3_sat(W[i * k + j] / sc);
    }
    free(W);
}

/* y = x * (s_n q[n][k])^T in fp64 (x bf16 [m][k]). */
void orc_linear_fp8(const uint16_t *x, int64_t m, int64_t k, const uint8_t *q, const float *s, int64_t n,
                    double *y) {
    for (int64_t i = 0; i < m; i++)
        for (int64_t j = 0; j < n; j++) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < k; kk++)
                acc += orc_bf16_to_f64(x[i * k + kk]) * ((double)s[j] * orc_e4m3_to_f64(q[j * k + kk]));
            y[i * n + j] = acc;
        }
}

/* ------------------------------------------------------------------ */
/* MLX-style affine group quantization ("Nemotron-Labs-TwoTower-30B-A3B --
 * MLX 6-bit", section "Quantization (6-bit, scheme mixed_v1)": the bulk of
 * the weights at 6 bits, embeddings and heads at >= 8 bits, the family at 4,
 * 6 and 8 bits).  Reading of what the README leaves open: groups of 64
 * consecutive weights of a row; scale = (max - min) / (2^b - 1) and
 * bias = min, both computed in fp32 and stored as bf16 (the checkpoint's
 * dtype); q = clamp(rint(fp32(fp32(w - bias) / scale)), 0, 2^b - 1) against
 * the stored bf16 values (a zero scale gives q = 0); codes of a row packed as
 * one little-endian bit stream, element i in bits [b i, b i + b).
 * Dequantized weight: fp32(fp32(scale * q) + bias).                       */

#define ORC_AFF_GROUP 64

static float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs). */
static uint16_t orc_f32_to_bf16(float f) { return orc_f64_to_bf16((double)f); }

void orc_affine_quantize(const float *W, int64_t n, int64_t k, int bits, uint8_t *codes, uint16_t *scales,
                         uint16_t *biases) {
    const int64_t ng = k / ORC_AFF_GROUP, row_bytes = k * bits / 8;
    const float qmax = (float)((1 << bits) - 1);
    memset(codes, 0, (size_t)(n * row_bytes));
    for (int64_t i = 0; i < n; i++)
        for (int64_t g = 0; g < ng; g++) {
            const float *w = W + i * k + g * ORC_AFF_GROUP;
            float lo = w[0], hi = w[0];
            for (int j = 1; j < ORC_AFF_GROUP; j++) {
                if (w[j] < lo) lo = w[j];
                if (w[j] > hi) hi = w[j];
            }
            const uint16_t sb = orc_f32_to_bf16((hi - lo) / qmax), bb = orc_f32_to_bf16(lo);
            scales[i * ng + g] = sb;
            biases[i * ng + g] = bb;
            const float sc = orc_bf16_to_f32(sb), bi = orc_bf16_to_f32(bb);
            for (int j = 0; j < ORC_AFF_GROUP; j++) {
                float q = 0.0f;
                if (sc != 0.0f) {
                    const float t = (w[j] - bi) / sc;
                    q = rintf(t);
                    if (q < 0.0f) q = 0.0f;
                    if (q > qmax) q = qmax;
                }
                const uint32_t v = (uint32_t)q;
                const int64_t bit = (g * ORC_AFF_GROUP + j) * bits;
                for (int b = 0; b < bits; b++)
                    if ((v >> b) & 1u) codes[i * row_bytes + (bit + b) / 8] |= (uint8_t)(1u << ((bit + b) % 8));
            }
        }
}

void orc_affine_dequantize(const uint8_t *codes, const uint16_t *scales, const uint16_t *biases, int64_t n,
                           int64_t k, int bits, float *W) {
    const int64_t ng = k / ORC_AFF_GROUP, row_bytes = k * bits / 8;
    for (int64_t i = 0; i < n; i++)
        for (int64_t e = 0; e < k; e++) {
            uint32_t v = 0;
            for (int b = 0; b < bits; b++) {
                const int64_t bit = e * bits + b;
                v |= (uint32_t)((codes[i * row_bytes + bit / 8] >> (bit % 8)) & 1u) << b;
            }
            const int64_t g = e / ORC_AFF_GROUP;
            const float sc = orc_bf16_to_f32(scales[i * ng + g]), bi = orc_bf16_to_f32(biases[i * ng + g]);
            const float t = sc * (float)v;
            W[i * k + e] = t + bi;
        }
}
