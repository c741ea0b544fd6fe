/*
 * Oracle for the routed mixture-of-experts FP8 blockwise (W8A8) prefill path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * CPU statement of what the path computes.  It is used by the tests, by the
 * package's smoke check and by the benchmark's CPU-baseline leg, and by
 * nothing else.  It shares no code, header, table or constant with the CUDA
 * library, and it includes nothing from it.
 *
 * Sources (web pages, cited by title and section):
 *   [KT-2244] "Full GLM-5.3 streamed FP8 GPU prefill on AVX2 / 2x32GiB SM120",
 *             section "Design": GPU W8A8 routed experts for prefill, unclamped
 *             SiLU, explicit rejection of unsupported inputs.
 *   [KT-2245] "Exact AVX2 FP8 arithmetic conversion avoids costly LUT gathers",
 *             section "Semantics and scope": E4M3 decode rules (normals by
 *             exponent/mantissa, subnormals = mantissa * 2^-9, signed zeros
 *             kept, NaN decodes to a signed zero); section "Real-checkpoint
 *             measurements": top-8 routes with normalised routing weights.
 *   [HPC-80]  "Integration for GLM-4.6-FP8 and performance tune on H20",
 *             gap table row 6: blockwise FP8 MoE, zero-padding of an
 *             intermediate width that is not a multiple of 128 (192 -> 256).
 *   [TF-2852] "GLM-5.3-Flash EXL3 on CUDA: a whole prompt pass routes its
 *             experts in one call", paragraph "Exactness" and the merged
 *             commit text: routed FP32 rows, whole-K accumulation, rows
 *             independent of how many rows share a call.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   R1  E4M3 encode is round-to-nearest, ties to the code with an even
 *       mantissa LSB, saturating to +-448; NaN encodes to 0x7F.
 *   R2  Group quantiser: s = fl32(amax / 448); s == 0 -> s = 1;
 *       code = enc(fl32(x / s)); a group holding NaN or Inf gets s = NaN and
 *       all codes 0x7F.  A partial trailing group uses its real columns only.
 *   R3  Routing: a logit is selectable unless it is NaN or -Inf; order by
 *       value descending then expert id ascending; weights are the softmax of
 *       the selected logits (equal to full softmax then renormalise).
 *       Unfilled slots carry id -1 and weight 0.
 *   R4  The intermediate h = SiLU(g) * u is rounded to FP32 and requantised
 *       with R2 per 128-column group before the down projection (W8A8).
 *   R5  routed_scaling multiplies the weighted slot sum.
 *
 * All floating-point arithmetic of the FFN is FP64.  The only FP32
 * operations are those R2 defines (the quantiser's divides), and the
 * rounding of h to FP32 in R4.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* E4M3 decode, by the format definition ([KT-2245] "Semantics and scope").  */
/* Byte b = s eeee mmm.  Bias 7.                                             */
/* ------------------------------------------------------------------------ */
ORACLE_API double oracle_e4m3_decode(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    double mag;
    if (e == 15 && m == 7) {
        mag = 0.0;                         /* NaN-to-signed-zero policy */
    } else if (e == 0) {
        mag = (double)m * ldexp(1.0, -9);  /* subnormal: mantissa * 2^-9 */
    } else {
        mag = (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
    }
    return sign ? -mag : mag;
}

/* ------------------------------------------------------------------------ */
/* E4M3 encode (reading R1): nearest finite code by explicit search.         */
/* ------------------------------------------------------------------------ */
/* Nearest finite E4M3 code to an exact (double) value, ties to the code with
 * an even mantissa LSB; magnitudes from 448 up (Inf included) saturate to the
 * code of 448; the sign is kept for +-0. */
static uint8_t e4m3_encode_exact(double v)
{
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    /* Saturation: every magnitude from the largest finite value (448) up to
     * and including Inf takes the code of 448. */
    if (a >= 448.0) return (uint8_t)(0x7E | (neg << 7));
    /* Candidates are the 127 non-negative finite codes 0x00..0x7E.  Keep the
     * closest; on an exact tie keep the code whose mantissa LSB is 0. */
    int best = 0;
    double best_d = a;  /* distance to code 0x00 (value +0) */
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | (neg << 7));
}

ORACLE_API uint8_t oracle_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    return e4m3_encode_exact((double)v);  /* every FP32 value is exact in double */
}

/* Encode n values (tests sweep large sets of FP32 inputs through this). */
ORACLE_API void oracle_e4m3_encode_n(const float* v, int64_t n, uint8_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------------ */
/* Group quantiser, reading R2.  n values (1..128) -> n codes and a scale.   */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_quant_group(const float* x, int n, uint8_t* codes, float* scale)
{
    int nonfinite = 0;
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(x[i])) nonfinite = 1;
        else if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    }
    if (nonfinite) {
        *scale = NAN;
        for (int i = 0; i < n; ++i) codes[i] = 0x7F;
        return;
    }
    volatile float s = amax / 448.0f;  /* one IEEE binary32 divide */
    float sv = s;
    if (sv == 0.0f) sv = 1.0f;
    for (int i = 0; i < n; ++i) {
        volatile float q = x[i] / sv;  /* one IEEE binary32 divide */
        codes[i] = oracle_e4m3_encode(q);
    }
    *scale = sv;
}

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Activation quantiser (path step "quantise activations"): x [T,H] BF16
 * bits -> codes [T,H], scales [T,H/128]. */
ORACLE_API void oracle_quant_act(const uint16_t* x, int64_t T, int64_t H,
                                 uint8_t* codes, float* scales)
{
    int64_t G = H / 128;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float buf[128];
        for (int64_t g = 0; g < G; ++g) {
            for (int i = 0; i < 128; ++i) buf[i] = bf16_to_float(x[t * H + g * 128 + i]);
            oracle_quant_group(buf, 128, codes + t * H + g * 128, scales + t * G + g);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Routing, reading R3.  logits [T,E] -> ids [T,k], weights [T,k] (FP64).    */
/* ------------------------------------------------------------------------ */
static int selectable(float v) { return !isnan(v) && !(isinf(v) && v < 0); }

ORACLE_API void oracle_route(const float* logits, int64_t T, int E, int k,
                             int32_t* ids, double* w)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        int32_t* id = ids + t * k;
        double* wt = w + t * k;
        int nsel = 0;
        /* Selection: k passes, each taking the largest remaining selectable
         * logit; ties go to the lower expert id. */
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (!selectable(l[e])) continue;
                int taken = 0;
                for (int q = 0; q < nsel; ++q) if (id[q] == e) taken = 1;
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;  /* strict: lower id wins ties */
            }
            if (best < 0) break;
            id[nsel++] = best;
        }
        for (int j = nsel; j < k; ++j) { id[j] = -1; wt[j] = 0.0; }
        if (nsel == 0) continue;
        double lmax = (double)l[id[0]];
        double den = 0.0;
        for (int j = 0; j < nsel; ++j) den += exp((double)l[id[j]] - lmax);
        for (int j = 0; j < nsel; ++j) wt[j] = exp((double)l[id[j]] - lmax) / den;
    }
}

/* ------------------------------------------------------------------------ */
/* Permutation: stable counting sort of the flat pairs p = t*k + j by expert.*/
/* offsets [E+1]; sorted_pairs [T*k], positions past offsets[E] hold -1.     */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_permute(const int32_t* ids, int64_t T, int k, int E,
                               int32_t* offsets, int32_t* sorted_pairs)
{
    int64_t P = T * (int64_t)k;
    int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    for (int64_t p = 0; p < P; ++p)
        if (ids[p] >= 0 && ids[p] < E) count[ids[p]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (int32_t)count[e];
    int64_t* next = (int64_t*)malloc((size_t)E * sizeof(int64_t));
    for (int e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t p = 0; p < P; ++p) {
        int e = ids[p];
        if (e < 0 || e >= E) continue;
        sorted_pairs[next[e]++] = (int32_t)p;
    }
    for (int64_t q = offsets[E]; q < P; ++q) sorted_pairs[q] = -1;
    free(count);
    free(next);
}

/* ------------------------------------------------------------------------ */
/* Expert FFN and combine (path steps gate/up, SiLU*up + requantise, down,  */
/* weighted combine).  Evaluated for the tokens listed in token_list.        */
/*                                                                           */
/*   codes [T,H], act_scales [T,H/128]             activation codes/scales   */
/*   ids [T,k], w [T,k] (FP64)                     routing                   */
/*   wg, wu [E,I,H]; sg, su [E,ceil(I/128),H/128]  gate / up weights+scales  */
/*   wd [E,H,I];     sd [E,H/128,ceil(I/128)]      down weights+scales       */
/*   out [n_tok,H] FP64                            routed output rows        */
/*   slot_out [n_tok,k,H] FP64 (nullable)          w_j * o_j per slot        */
/*   h_codes [n_tok,k,Ip], h_scales [n_tok,k,G_I] (nullable) intermediate;   */
/*   h_fp32 [n_tok,k,Ip] (nullable) the FP32 h before requantisation         */
/*   h_override_codes/h_override_scales (nullable): same layout as h_codes;  */
/*     when given, the down projection uses them instead of its own (used to */
/*     isolate the down-projection error of another implementation).         */
/* Slots with id -1 contribute nothing; a token with no valid slot gets 0.   */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_moe_ffn(const uint8_t* codes, const float* act_scales,
                               int64_t T, int64_t H,
                               const int32_t* ids, const double* w, int k,
                               int E, int64_t I,
                               const uint8_t* wg, const float* sg,
                               const uint8_t* wu, const float* su,
                               const uint8_t* wd, const float* sd,
                               double routed_scaling,
                               const int64_t* token_list, int64_t n_tok,
                               double* out, double* slot_out,
                               uint8_t* h_codes, float* h_scales, float* h_fp32,
                               const uint8_t* h_override_codes,
                               const float* h_override_scales,
                               int n_threads)
{
    (void)T;
    (void)E;
    const int64_t GH = H / 128;
    const int64_t GI = (I + 127) / 128;
    const int64_t Ip = GI * 128;
    double dec[256];
    for (int b = 0; b < 256; ++b) dec[b] = oracle_e4m3_decode((uint8_t)b);

#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif

#pragma omp parallel
    {
        double* xd = (double*)malloc((size_t)H * sizeof(double));
        double* o = (double*)malloc((size_t)H * sizeof(double));
        double* hd = (double*)malloc((size_t)Ip * sizeof(double));
        float* h32 = (float*)malloc((size_t)Ip * sizeof(float));
        uint8_t* hq = (uint8_t*)malloc((size_t)Ip);
        float* sh = (float*)malloc((size_t)GI * sizeof(float));

#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_tok; ++it) {
            int64_t t = token_list[it];
            double* orow = out + it * H;
            for (int64_t n = 0; n < H; ++n) orow[n] = 0.0;

            /* dequantised activation row: xd = dec(q) * s */
            for (int64_t kk = 0; kk < H; ++kk)
                xd[kk] = dec[codes[t * H + kk]] * (double)act_scales[t * GH + kk / 128];

            for (int j = 0; j < k; ++j) {
                int e = ids[t * k + j];
                double* srow = slot_out ? slot_out + (it * k + j) * H : NULL;
                if (srow) for (int64_t n = 0; n < H; ++n) srow[n] = 0.0;
                if (e < 0) continue;
                const uint8_t* Wg = wg + (int64_t)e * I * H;
                const uint8_t* Wu = wu + (int64_t)e * I * H;
                const float* Sg = sg + (int64_t)e * GI * GH;
                const float* Su = su + (int64_t)e * GI * GH;

                /* gate and up projections, then h = SiLU(g) * u (unclamped) */
                for (int64_t n = 0; n < I; ++n) {
                    double g = 0.0, u = 0.0;
                    for (int64_t kk = 0; kk < H; ++kk) {
                        double wgd = dec[Wg[n * H + kk]] * (double)Sg[(n / 128) * GH + kk / 128];
                        double wud = dec[Wu[n * H + kk]] * (double)Su[(n / 128) * GH + kk / 128];
                        g += xd[kk] * wgd;
                        u += xd[kk] * wud;
                    }
                    double h64 = g / (1.0 + exp(-g)) * u;
                    h32[n] = (float)h64;
                }

                /* requantise h per 128-column group (reading R4); the
                 * padding columns I..Ip-1 hold code 0 */
                for (int64_t n = I; n < Ip; ++n) hq[n] = 0;
                for (int64_t gi = 0; gi < GI; ++gi) {
                    int64_t c0 = gi * 128;
                    int64_t nc = (I - c0 < 128) ? (I - c0) : 128;
                    oracle_quant_group(h32 + c0, (int)nc, hq + c0, sh + gi);
                }
                if (h_fp32) {
                    memcpy(h_fp32 + (it * k + j) * Ip, h32, (size_t)I * sizeof(float));
                    for (int64_t n = I; n < Ip; ++n) h_fp32[(it * k + j) * Ip + n] = 0.0f;
                }
                if (h_codes) memcpy(h_codes + (it * k + j) * Ip, hq, (size_t)Ip);
                if (h_scales) memcpy(h_scales + (it * k + j) * GI, sh, (size_t)GI * sizeof(float));

                const uint8_t* hq_use = hq;
                const float* sh_use = sh;
                if (h_override_codes) {
                    hq_use = h_override_codes + (it * k + j) * Ip;
                    sh_use = h_override_scales + (it * k + j) * GI;
                }
                for (int64_t i = 0; i < I; ++i) hd[i] = dec[hq_use[i]] * (double)sh_use[i / 128];

                /* down projection and routing weight */
                const uint8_t* Wd = wd + (int64_t)e * H * I;
                const float* Sd = sd + (int64_t)e * GH * GI;
                double wj = w[t * k + j];
                for (int64_t n = 0; n < H; ++n) {
                    double acc = 0.0;
                    for (int64_t i = 0; i < I; ++i)
                        acc += hd[i] * (dec[Wd[n * I + i]] * (double)Sd[(n / 128) * GI + i / 128]);
                    o[n] = acc;
                }
                for (int64_t n = 0; n < H; ++n) {
                    orow[n] += wj * o[n];
                    if (srow) srow[n] = wj * o[n];
                }
            }
            for (int64_t n = 0; n < H; ++n) orow[n] *= routed_scaling;
        }
        free(xd);
        free(o);
        free(hd);
        free(h32);
        free(hq);
        free(sh);
    }
}

/* Number of OpenMP threads a parallel region of the oracle uses. */
ORACLE_API int oracle_num_threads(void)
{
#ifdef _OPENMP
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
#else
    return 1;
#endif
}

/* ======================================================================== */
/* MXFP8 variant (the pages name an MXFP8 MoE runtime as not yet qualified:   */
/* [KT-2245] "Real-checkpoint measurements", caveats).  E4M3 elements with    */
/* one UE8M0 (power-of-two) scale per 32 consecutive values along the         */
/* contraction dimension.  Readings (the pages give no definition; these      */
/* follow the OCP Microscaling Formats v1.0 rules):                           */
/*   M1  UE8M0 byte X decodes to 2^(X-127); X = 0xFF is NaN.                  */
/*   M2  Block quantiser over 32 values (fewer at a ragged end): amax =       */
/*       max|x|; e = floor(log2(amax)); shared exponent se = e - 8 (8 is the  */
/*       largest exponent of a normal E4M3 value, 448 = 1.75 * 2^8), clamped  */
/*       to [-127, 127]; X = se + 127; code_i = the E4M3 code nearest to the  */
/*       exact x_i / 2^se, ties to even, saturating at +-448.  amax = 0 ->    */
/*       X = 0 and codes +-0; a block holding NaN or Inf -> X = 0xFF and      */
/*       codes 0x7F.                                                          */
/*   M3  The FFN is the blockwise path of oracle_moe_ffn with these scales:   */
/*       activations and intermediate quantised by M2 per 32 columns,         */
/*       weights stored with one UE8M0 scale per (row, 32 columns).           */
/* ======================================================================== */

/* M1 */
ORACLE_API double oracle_ue8m0_decode(uint8_t x)
{
    if (x == 0xFF) return NAN;
    return ldexp(1.0, (int)x - 127);
}

/* M2: n values (1..32) -> n codes and one scale byte. */
ORACLE_API void oracle_mx_quant_block(const float* x, int n, uint8_t* codes, uint8_t* scale)
{
    int nonfinite = 0;
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(x[i])) nonfinite = 1;
        else if (fabs((double)x[i]) > amax) amax = fabs((double)x[i]);
    }
    if (nonfinite) {
        *scale = 0xFF;
        for (int i = 0; i < n; ++i) codes[i] = 0x7F;
        return;
    }
    int se;
    if (amax == 0.0) {
        se = -127;
    } else {
        int ex;
        frexp(amax, &ex);      /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
        se = (ex - 1) - 8;
        if (se < -127) se = -127;
        if (se > 127) se = 127;
    }
    *scale = (uint8_t)(se + 127);
    for (int i = 0; i < n; ++i) codes[i] = e4m3_encode_exact(ldexp((double)x[i], -se));
}

/* MX activation quantiser: x [T,H] BF16 bits -> codes [T,H], scales [T,H/32]. */
ORACLE_API void oracle_mx_quant_act(const uint16_t* x, int64_t T, int64_t H, uint8_t* codes, uint8_t* scales)
{
    int64_t G = H / 32;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float buf[32];
        for (int64_t g = 0; g < G; ++g) {
            for (int i = 0; i < 32; ++i) buf[i] = bf16_to_float(x[t * H + g * 32 + i]);
            oracle_mx_quant_block(buf, 32, codes + t * H + g * 32, scales + t * G + g);
        }
    }
}

/* M3: expert FFN and combine with MX operands, for the tokens listed.
 *   codes [T,H], act_scales [T,H/32] (UE8M0)          activations
 *   ids [T,k], w [T,k] (FP64)                          routing
 *   wg, wu [E,I,H]; sg, su [E,I,H/32] (UE8M0)           gate / up
 *   wd [E,H,I];     sd [E,H,I/32]   (UE8M0)             down
 *   out [n_tok,H] FP64; h_codes [n_tok,k,I], h_scales [n_tok,k,I/32],
 *   h_fp32 [n_tok,k,I] (nullable).  I % 32 == 0. */
ORACLE_API void oracle_mx_moe_ffn(const uint8_t* codes, const uint8_t* act_scales, int64_t T, int64_t H,
                                  const int32_t* ids, const double* w, int k, int E, int64_t I,
                                  const uint8_t* wg, const uint8_t* sg, const uint8_t* wu, const uint8_t* su,
                                  const uint8_t* wd, const uint8_t* sd, double routed_scaling,
                                  const int64_t* token_list, int64_t n_tok, double* out,
                                  uint8_t* h_codes, uint8_t* h_scales, float* h_fp32, int n_threads)
{
    (void)T;
    (void)E;
    const int64_t BH = H / 32, BI = I / 32;
    double dec[256], sdec[256];
    for (int b = 0; b < 256; ++b) {
        dec[b] = oracle_e4m3_decode((uint8_t)b);
        sdec[b] = oracle_ue8m0_decode((uint8_t)b);
    }
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double* xd = (double*)malloc((size_t)H * sizeof(double));
        double* hd = (double*)malloc((size_t)I * sizeof(double));
        float* h32 = (float*)malloc((size_t)I * sizeof(float));
        uint8_t* hq = (uint8_t*)malloc((size_t)I);
        uint8_t* sh = (uint8_t*)malloc((size_t)BI);
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_tok; ++it) {
            int64_t t = token_list[it];
            double* orow = out + it * H;
            for (int64_t n = 0; n < H; ++n) orow[n] = 0.0;
            for (int64_t kk = 0; kk < H; ++kk) xd[kk] = dec[codes[t * H + kk]] * sdec[act_scales[t * BH + kk / 32]];
            for (int j = 0; j < k; ++j) {
                int e = ids[t * k + j];
                if (e < 0) continue;
                const uint8_t* Wg = wg + (int64_t)e * I * H;
                const uint8_t* Wu = wu + (int64_t)e * I * H;
                const uint8_t* Sg = sg + (int64_t)e * I * BH;
                const uint8_t* Su = su + (int64_t)e * I * BH;
                for (int64_t n = 0; n < I; ++n) {
                    double g = 0.0, u = 0.0;
                    for (int64_t kk = 0; kk < H; ++kk) {
                        g += xd[kk] * (dec[Wg[n * H + kk]] * sdec[Sg[n * BH + kk / 32]]);
                        u += xd[kk] * (dec[Wu[n * H + kk]] * sdec[Su[n * BH + kk / 32]]);
                    }
                    h32[n] = (float)(g / (1.0 + exp(-g)) * u);
                }
                for (int64_t b = 0; b < BI; ++b) oracle_mx_quant_block(h32 + b * 32, 32, hq + b * 32, sh + b);
                if (h_fp32) memcpy(h_fp32 + (it * k + j) * I, h32, (size_t)I * sizeof(float));
                if (h_codes) memcpy(h_codes + (it * k + j) * I, hq, (size_t)I);
                if (h_scales) memcpy(h_scales + (it * k + j) * BI, sh, (size_t)BI);
                for (int64_t i = 0; i < I; ++i) hd[i] = dec[hq[i]] * sdec[sh[i / 32]];
                const uint8_t* Wd = wd + (int64_t)e * H * I;
                const uint8_t* Sd = sd + (int64_t)e * H * BI;
                double wj = w[t * k + j];
                for (int64_t n = 0; n < H; ++n) {
                    double acc = 0.0;
                    for (int64_t i = 0; i < I; ++i) acc += hd[i] * (dec[Wd[n * I + i]] * sdec[Sd[n * BI + i / 32]]);
                    orow[n] += wj * acc;
                }
            }
            for (int64_t n = 0; n < H; ++n) orow[n] *= routed_scaling;
        }
        free(xd);
        free(hd);
        free(h32);
        free(hq);
        free(sh);
    }
}
