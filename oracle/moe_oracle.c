/*
 * moe_oracle.c -- plain, slow CPU definition of the fused Mixture-of-Experts
 * layer.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the smoke
 * check and by the benchmark's CPU-baseline leg, never by the library.  It
 * shares no code, header, table or helper with the CUDA path.
 *
 * What it follows.  The layer is the "fused MoE" operation described on
 *   [A] "Az AWS új MoE-optimalizációkkal gyorsítja a SageMaker AI-t",
 *       § "A fused MoE a számítási folyamat több lépését egyesíti":
 *       token routing, data reordering and the experts' computation done as
 *       one batched GPU operation instead of a loop over experts;
 *   [B] "Ingénierie de kernels Mixture-of-Experts sur Amazon SageMaker AI":
 *       the expert GEMM is A[M,K] x B[K,N] with M = tokens, K = hidden size,
 *       N = the expert's output size;
 *   [C] "Amazon SageMaker AIにおけるMixture-of-Expertsカーネル最適化の深掘り",
 *       § "Mixture-of-Experts (MoE) モデルの原理と推論における課題":
 *       a router activates a few experts per input (sparse activation);
 *   [A] § "FP8 esetén a Triton backend bizonyult gyorsabbnak": FP8 per-tensor
 *       scaling, the GEMM and the aggregation of the experts' outputs.
 * The pages fix nothing finer.  The finer definition used here (softmax over
 * the top-k logits, SwiGLU experts, counting-sort permutation padded to the
 * MMA tile, amax/448 e4m3 scales) is the layer's specification; each reading
 * of a point the pages leave open is named R<n> below and listed with its
 * basis in the design notes.
 *
 * Precision: every floating-point step is done in double (inputs are exact
 * bf16 / f32 / e4m3 values widened to double).  Where a float decides an
 * integer (an e4m3 code), the decision is taken in float, the precision the
 * GPU path takes it in (x / s computed as an IEEE float division).
 *
 * Parity pins (tests/test_oracle_*.py): routing against brute force over all
 * C(E,k) subsets; the permutation against a stable sort; the layer against a
 * dense "every expert on every token, then mask" forward built from torch
 * fp64 matmuls, E = 1 (dense SwiGLU), k = E with equal logits (mean of the
 * experts), token-permutation equivariance and linearity in W_d; the e4m3
 * codec exhaustively against torch.float8_e4m3fn.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1 };

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* bf16 is the top half of an IEEE binary32: widening is exact. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double load(const void* p, int dtype, size_t i) {
    if (dtype == OR_BF16) return bf16_to_double(((const uint16_t*)p)[i]);
    return (double)((const float*)p)[i];
}

/* ---------------------------------------------------------------- routing
 * Router [C]: each token activates k of the E experts.  Readings:
 *  R1  select on the raw logits (softmax is monotone, so the set equals the
 *      top-k of the softmax), then weight the selected experts by a softmax
 *      over the selected logits only (= the full softmax renormalised);
 *  R2  order: larger logit first; equal logits (-0 == +0) lower index first;
 *      NaN ranks below every number, NaNs among themselves by index.
 */
static const float* g_sort_row; /* comparator context (single-threaded use) */

static int beats(float a, int ia, float b, int ib) {
    int na = isnan(a), nb = isnan(b);
    if (na && nb) return ia < ib;
    if (na) return 0;
    if (nb) return 1;
    if (a > b) return 1;
    if (a < b) return 0;
    return ia < ib;
}

static int cmp_expert(const void* pa, const void* pb) {
    int ia = *(const int*)pa, ib = *(const int*)pb;
    if (ia == ib) return 0;
    return beats(g_sort_row[ia], ia, g_sort_row[ib], ib) ? -1 : 1;
}

int oracle_route_topk(const float* logits, int T, int E, int k, int32_t* ids, double* w) {
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    int* order = (int*)malloc(sizeof(int) * (size_t)E);
    if (!order) return -2;
    for (int t = 0; t < T; ++t) {
        const float* row = logits + (size_t)t * E;
        for (int e = 0; e < E; ++e) order[e] = e;
        g_sort_row = row;
        qsort(order, (size_t)E, sizeof(int), cmp_expert); /* total order: any sort is stable */
        double m = (double)row[order[0]];
        double z = 0.0;
        for (int j = 0; j < k; ++j) z += exp((double)row[order[j]] - m);
        for (int j = 0; j < k; ++j) {
            ids[(size_t)t * k + j] = order[j];
            w[(size_t)t * k + j] = exp((double)row[order[j]] - m) / z;
        }
    }
    free(order);
    return 0;
}

/* ------------------------------------------------------------ permutation
 * "Data reordering" [A], [B]: the assignments (token t, slot j), flat index
 * f = t*k + j, are grouped by expert so each expert's GEMM reads a contiguous
 * block of rows.  Readings:
 *  R3  inside an expert the order is ascending f (a stable counting sort);
 *  R4  each expert's block is padded up to a multiple of block_m rows (empty
 *      experts take no rows); pad slots and the unused tail hold -1;
 *  tiles[b] names the expert owning rows [b*block_m, (b+1)*block_m).
 */
int oracle_permute_capacity(int T, int k, int E, int block_m) {
    long A = (long)T * k;
    long ne = A < E ? A : E;
    long c = A + ne * (block_m - 1);
    return (int)((c + block_m - 1) / block_m * block_m);
}

int oracle_align_permute(const int32_t* ids, int T, int k, int E, int block_m, int capacity,
                         int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                         int32_t* inv_perm, int32_t* tiles, int32_t* num_tiles) {
    long A = (long)T * k;
    if (block_m < 1 || capacity < 0) return -1;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long f = 0; f < A; ++f) {
        if (ids[f] < 0 || ids[f] >= E) return -3;
        counts[ids[f]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        long padded = (counts[e] + block_m - 1) / block_m * (long)block_m;
        offsets[e + 1] = offsets[e] + (int32_t)padded;
    }
    if (offsets[E] > capacity) return -4;
    for (int p = 0; p < capacity; ++p) sorted_ids[p] = -1;
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    if (!fill) return -2;
    for (long f = 0; f < A; ++f) {
        int e = ids[f];
        int32_t slot = offsets[e] + fill[e]++;
        sorted_ids[slot] = (int32_t)f;
        inv_perm[f] = slot;
    }
    free(fill);
    int nt = offsets[E] / block_m;
    for (int b = 0; b < capacity / block_m; ++b) tiles[b] = -1;
    for (int e = 0; e < E; ++e)
        for (int b = offsets[e] / block_m; b < offsets[e + 1] / block_m; ++b) tiles[b] = e;
    *num_tiles = nt;
    return 0;
}

/* ------------------------------------------------------------ expert FFN
 * Expert computation [B]: per assignment, A[M,K] x B[K,N] with M the tokens
 * routed to the expert and K = H.  Readings:
 *  R5  SwiGLU experts without bias: h = SiLU(x W_g) * (x W_u),
 *      SiLU(z) = z / (1 + e^-z); y = h W_d;
 *  R6  the routing weight multiplies each expert's output, then the top-k
 *      outputs are summed ("aggregation of the experts' results" [A]).
 * The output of token t is evaluated directly, token by token, with no
 * permutation at all:  out[t] = sum_j w[t,j] * FFN_{ids[t,j]}(x[t]).
 */
static double silu(double z) { return z / (1.0 + exp(-z)); }

static void ffn_one(int H, int I, const double* xt, const void* Wg, const void* Wu,
                    const void* Wd, int wdt, int e, double wgt, double* g, double* u,
                    double* out) {
    size_t hi = (size_t)H * I;
    for (int n = 0; n < I; ++n) { g[n] = 0.0; u[n] = 0.0; }
    for (int h = 0; h < H; ++h) {
        double xv = xt[h];
        size_t base = (size_t)e * hi + (size_t)h * I;
        for (int n = 0; n < I; ++n) {
            g[n] += xv * load(Wg, wdt, base + n);
            u[n] += xv * load(Wu, wdt, base + n);
        }
    }
    for (int n = 0; n < I; ++n) {
        double a = silu(g[n]) * u[n];
        size_t base = (size_t)e * hi + (size_t)n * H;
        for (int c = 0; c < H; ++c) out[c] += wgt * a * load(Wd, wdt, base + c);
    }
}

int oracle_moe_layer(int T, int H, int I, int E, int k,
                     const void* x, int x_dtype,
                     const int32_t* ids, const double* w,
                     const void* Wg, const void* Wu, const void* Wd, int w_dtype,
                     const int32_t* tokens, int n_tokens, double* out) {
    if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1 || k > E) return -1;
    int n = tokens ? n_tokens : T;
    int bad = 0;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)I);
        double* u = (double*)malloc(sizeof(double) * (size_t)I);
        double* xt = (double*)malloc(sizeof(double) * (size_t)H);
        if (!g || !u || !xt) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int i = 0; i < n; ++i) {
                int t = tokens ? tokens[i] : i;
                double* o = out + (size_t)i * H;
                for (int c = 0; c < H; ++c) o[c] = 0.0;
                if (t < 0 || t >= T) continue;
                for (int c = 0; c < H; ++c) xt[c] = load(x, x_dtype, (size_t)t * H + c);
                for (int j = 0; j < k; ++j) {
                    int e = ids[(size_t)t * k + j];
                    if (e < 0 || e >= E) continue;
                    ffn_one(H, I, xt, Wg, Wu, Wd, w_dtype, e, w[(size_t)t * k + j], g, u, o);
                }
            }
        }
        free(g); free(u); free(xt);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------ multi-LoRA
 * Multi-LoRA serving of MoE models ("Amazon SageMaker AIにおける
 * Mixture-of-Expertsカーネル最適化の深掘り", § "SageMakerを活用したMoEモデルの
 * デプロイと性能向上戦略"): several fine-tuned variants of one MoE model
 * ("adapters") share the GPU.  The pages name the technique only; readings:
 *  L1  token t carries an adapter index a_t in [0, n_adapters), or -1 for the
 *      base model alone;
 *  L2  adapter a holds, for every expert e and each of its three matrices, a
 *      rank-r pair: W_g[e] + s_a A_g[a,e] B_g[a,e] with A_g [H, r] and
 *      B_g [r, I]; W_u likewise; W_d[e] + s_a A_d[a,e] B_d[a,e] with
 *      A_d [I, r] and B_d [r, H] (the usual low-rank adaptation, applied to
 *      the weights the token actually meets);
 *  L3  s_a is the adapter's scale (alpha / r in the usual convention), an
 *      input;
 *  L4  so g = x W_g + s_a (x A_g) B_g and u likewise, h = SiLU(g) * u,
 *      y = h W_d + s_a (h A_d) B_d; routing and the weighted combine are
 *      unchanged.
 * Layouts: A_g, A_u [n_a][E][H][r], B_g, B_u [n_a][E][r][I], A_d [n_a][E][I][r],
 * B_d [n_a][E][r][H], all of one dtype (l_dtype).
 */
static void lora_shrink(int K, int r, const double* v, const void* A, int adt, size_t base,
                        double* t) {
    for (int q = 0; q < r; ++q) t[q] = 0.0;
    for (int c = 0; c < K; ++c) {
        double vc = v[c];
        for (int q = 0; q < r; ++q) t[q] += vc * load(A, adt, base + (size_t)c * r + q);
    }
}

int oracle_moe_layer_lora(int T, int H, int I, int E, int k,
                          const void* x, int x_dtype,
                          const int32_t* ids, const double* w,
                          const void* Wg, const void* Wu, const void* Wd, int w_dtype,
                          int n_adapters, int r, const int32_t* adapter,
                          const void* Ag, const void* Bg, const void* Au, const void* Bu,
                          const void* Ad, const void* Bd, int l_dtype, const double* scale,
                          const int32_t* tokens, int n_tokens, double* out) {
    if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1 || k > E || n_adapters < 0 || r < 1)
        return -1;
    int n = tokens ? n_tokens : T;
    int bad = 0;
    size_t hi = (size_t)H * I;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)I);
        double* u = (double*)malloc(sizeof(double) * (size_t)I);
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        double* xt = (double*)malloc(sizeof(double) * (size_t)H);
        double* tg = (double*)malloc(sizeof(double) * (size_t)r);
        double* tu = (double*)malloc(sizeof(double) * (size_t)r);
        double* td = (double*)malloc(sizeof(double) * (size_t)r);
        if (!g || !u || !h || !xt || !tg || !tu || !td) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int i = 0; i < n; ++i) {
                int t = tokens ? tokens[i] : i;
                double* o = out + (size_t)i * H;
                for (int c = 0; c < H; ++c) o[c] = 0.0;
                if (t < 0 || t >= T) continue;
                int a = adapter ? adapter[t] : -1;
                if (a >= n_adapters) a = -1;
                for (int c = 0; c < H; ++c) xt[c] = load(x, x_dtype, (size_t)t * H + c);
                for (int j = 0; j < k; ++j) {
                    int e = ids[(size_t)t * k + j];
                    if (e < 0 || e >= E) continue;
                    double wgt = w[(size_t)t * k + j];
                    /* base projections */
                    for (int m = 0; m < I; ++m) { g[m] = 0.0; u[m] = 0.0; }
                    for (int c = 0; c < H; ++c) {
                        size_t b = (size_t)e * hi + (size_t)c * I;
                        for (int m = 0; m < I; ++m) {
                            g[m] += xt[c] * load(Wg, w_dtype, b + m);
                            u[m] += xt[c] * load(Wu, w_dtype, b + m);
                        }
                    }
                    /* the adapter's low-rank deltas (L2, L4) */
                    size_t ae = 0;
                    if (a >= 0) {
                        ae = (size_t)a * E + (size_t)e;
                        lora_shrink(H, r, xt, Ag, l_dtype, ae * (size_t)H * r, tg);
                        lora_shrink(H, r, xt, Au, l_dtype, ae * (size_t)H * r, tu);
                        for (int q = 0; q < r; ++q) {
                            size_t b = ae * (size_t)r * I + (size_t)q * I;
                            for (int m = 0; m < I; ++m) {
                                g[m] += scale[a] * tg[q] * load(Bg, l_dtype, b + m);
                                u[m] += scale[a] * tu[q] * load(Bu, l_dtype, b + m);
                            }
                        }
                    }
                    for (int m = 0; m < I; ++m) h[m] = silu(g[m]) * u[m];
                    for (int m = 0; m < I; ++m) {
                        size_t b = (size_t)e * hi + (size_t)m * H;
                        for (int c = 0; c < H; ++c) o[c] += wgt * h[m] * load(Wd, w_dtype, b + c);
                    }
                    if (a >= 0) {
                        lora_shrink(I, r, h, Ad, l_dtype, ae * (size_t)I * r, td);
                        for (int q = 0; q < r; ++q) {
                            size_t b = ae * (size_t)r * H + (size_t)q * H;
                            for (int c = 0; c < H; ++c)
                                o[c] += wgt * scale[a] * td[q] * load(Bd, l_dtype, b + c);
                        }
                    }
                }
            }
        }
        free(g); free(u); free(h); free(xt); free(tg); free(tu); free(td);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------ FP8 e4m3
 * FP8 per-tensor quantisation [A] § "FP8 esetén…", [C] (FP8 量子化).
 * e4m3 "fn" encoding: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 * infinities, S.1111.111 = NaN, largest finite 448, subnormals m * 2^-9.
 * Readings:
 *  R7  scale s = amax / 448 (one per tensor; amax = 0 gives s = 1);
 *  R8  quantise: round to nearest, ties to even, saturating at +-448
 *      (+-inf saturates too, NaN stays NaN);
 *  R9  weights: one scale per expert matrix (W_g, W_u, W_d separately);
 *      x: one dynamic scale over the whole [T,H] input; h: one dynamic scale
 *      over all valid h rows; dequantised values are code * scale.
 */
float oracle_e4m3_decode(uint8_t c) {
    int sgn = c >> 7, ex = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (ex == 15 && m == 7) return sgn ? -NAN : NAN;
    if (ex == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, ex - 7);
    return (float)(sgn ? -v : v);
}

static double rne(double y) { /* y >= 0; round half to even */
    double r = floor(y), d = y - r;
    if (d > 0.5) return r + 1.0;
    if (d < 0.5) return r;
    return fmod(r, 2.0) == 0.0 ? r : r + 1.0;
}

uint8_t oracle_e4m3_encode(float xf) {
    if (isnan(xf)) return 0x7F;
    uint8_t sgn = signbit(xf) ? 0x80 : 0x00;
    double a = fabs((double)xf);
    if (a >= 448.0) return sgn | 0x7E;
    if (a < ldexp(1.0, -6)) {                 /* subnormal range: steps of 2^-9 */
        int m = (int)rne(a * 512.0);          /* m == 8 is the smallest normal */
        return sgn | (uint8_t)m;
    }
    int e2;
    double f = frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5, 1) */
    int eu = e2 - 1;                          /* a = (2f) * 2^eu, 2f in [1, 2) */
    int m = (int)rne((2.0 * f - 1.0) * 8.0);
    if (m == 8) { m = 0; eu += 1; }
    return sgn | (uint8_t)(((eu + 7) << 3) | m);
}

/* Scale and codes of one tensor (R7, R8).  The code decision divides in float. */
float oracle_fp8_quantize(const void* src, int dtype, size_t n, uint8_t* q) {
    double amax = 0.0;
    for (size_t i = 0; i < n; ++i) {
        double v = fabs(load(src, dtype, i));
        if (v > amax) amax = v;
    }
    float s = amax > 0.0 ? (float)amax / 448.0f : 1.0f;
    if (q)
        for (size_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode((float)load(src, dtype, i) / s);
    return s;
}

static void make_lut(float s, double* lut) {
    for (int c = 0; c < 256; ++c) lut[c] = (double)oracle_e4m3_decode((uint8_t)c) * (double)s;
}

/* The FP8 layer (R7-R9): weights and x quantise-dequantised with their own
 * scales; h is computed for every assignment (the h scale needs the amax of
 * all of them), quantise-dequantised, then the down projection, routing
 * weight and top-k sum follow as in the bf16 layer.
 * w_scales receives [E][3] = (s_g, s_u, s_d); act_scales receives (s_x, s_h). */
int oracle_moe_layer_fp8(int T, int H, int I, int E, int k,
                         const void* x, int x_dtype,
                         const int32_t* ids, const double* w,
                         const void* Wg, const void* Wu, const void* Wd, int w_dtype,
                         const int32_t* tokens, int n_tokens, double* out,
                         float* w_scales, float* act_scales) {
    if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1 || k > E) return -1;
    size_t hi = (size_t)H * I;
    size_t A = (size_t)T * k;
    uint8_t* qw = (uint8_t*)malloc(3 * (size_t)E * hi);
    double* lut = (double*)malloc(sizeof(double) * 256 * 3 * (size_t)E);
    uint8_t* qx = (uint8_t*)malloc((size_t)T * H + 1);
    double* h = (double*)malloc(sizeof(double) * (A * (size_t)I + 1));
    uint8_t* qh = (uint8_t*)malloc(A * (size_t)I + 1);
    if (!qw || !lut || !qx || !h || !qh) {
        free(qw); free(lut); free(qx); free(h); free(qh);
        return -2;
    }
    const void* mats[3] = {Wg, Wu, Wd};
    const size_t esz = (w_dtype == OR_BF16) ? 2 : 4;
#pragma omp parallel for schedule(dynamic, 1)
    for (int em = 0; em < 3 * E; ++em) {
        int e = em / 3, m = em % 3;
        const char* src = (const char*)mats[m] + (size_t)e * hi * esz;
        float s = oracle_fp8_quantize(src, w_dtype, hi, qw + (size_t)em * hi);
        w_scales[em] = s;
        make_lut(s, lut + (size_t)em * 256);
    }
    float sx = oracle_fp8_quantize(x, x_dtype, (size_t)T * H, qx);
    double lutx[256];
    make_lut(sx, lutx);

    /* h for every assignment */
#pragma omp parallel
    {
        double* xt = (double*)malloc(sizeof(double) * (size_t)H);
        double* u = (double*)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(dynamic, 1)
        for (long a = 0; a < (long)A; ++a) {
            int t = (int)(a / k);
            int e = ids[a];
            double* g = h + (size_t)a * I;
            for (int n = 0; n < I; ++n) { g[n] = 0.0; u[n] = 0.0; }
            if (!xt || !u || e < 0 || e >= E) continue;
            for (int c = 0; c < H; ++c) xt[c] = lutx[qx[(size_t)t * H + c]];
            const uint8_t* qg = qw + (size_t)(3 * e + 0) * hi;
            const uint8_t* qu = qw + (size_t)(3 * e + 1) * hi;
            const double* lg = lut + (size_t)(3 * e + 0) * 256;
            const double* lu = lut + (size_t)(3 * e + 1) * 256;
            for (int c = 0; c < H; ++c) {
                double xv = xt[c];
                for (int n = 0; n < I; ++n) {
                    g[n] += xv * lg[qg[(size_t)c * I + n]];
                    u[n] += xv * lu[qu[(size_t)c * I + n]];
                }
            }
            for (int n = 0; n < I; ++n) g[n] = silu(g[n]) * u[n];
        }
        free(xt); free(u);
    }
    double hmax = 0.0;
    for (size_t i = 0; i < A * (size_t)I; ++i) if (fabs(h[i]) > hmax) hmax = fabs(h[i]);
    float sh = hmax > 0.0 ? (float)hmax / 448.0f : 1.0f;
    for (size_t i = 0; i < A * (size_t)I; ++i) qh[i] = oracle_e4m3_encode((float)h[i] / sh);
    double luth[256];
    make_lut(sh, luth);
    act_scales[0] = sx;
    act_scales[1] = sh;

    int n = tokens ? n_tokens : T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; ++i) {
        int t = tokens ? tokens[i] : i;
        double* o = out + (size_t)i * H;
        for (int c = 0; c < H; ++c) o[c] = 0.0;
        if (t < 0 || t >= T) continue;
        for (int j = 0; j < k; ++j) {
            size_t a = (size_t)t * k + j;
            int e = ids[a];
            if (e < 0 || e >= E) continue;
            const uint8_t* qd = qw + (size_t)(3 * e + 2) * hi;
            const double* ld = lut + (size_t)(3 * e + 2) * 256;
            for (int nn = 0; nn < I; ++nn) {
                double av = w[a] * luth[qh[a * I + nn]];
                for (int c = 0; c < H; ++c) o[c] += av * ld[qd[(size_t)nn * H + c]];
            }
        }
    }
    free(qw); free(lut); free(qx); free(h); free(qh);
    return 0;
}
