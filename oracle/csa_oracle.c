/*
 * csa_oracle.c -- plain, slow, fp64 CPU oracle for the Compressed Sparse
 * Attention (CSA) / Heavily Compressed Attention (HCA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file or the library built from it: only the tests, the smoke
 * check of the package entry file and the CPU-baseline leg of the benchmark
 * use it.  It shares no code, header, table or constant with the CUDA
 * library; the two meet only through the seeded input generator.
 *
 * Sources of the method (page title, section):
 *   [P1] "DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" (gitcode issue),
 *        §3.2 (ratio 4 overlapping / ratio 128 non-overlapping compressor),
 *        §7.2 (two stage-1 compressors: main and indexer).
 *   [P3] "DS-V4 分析&学习", §1.2 (compress -> indexer -> top-k -> attend to
 *        k compressed + sliding window KV), §1.3 (each entry sees 2m adjacent
 *        positions, neighbouring blocks overlap), §1.4 (HCA, m'=128, dense),
 *        §1.5 (SWA), §4 (low-precision indexer QK).
 *   [P5] "百万上下文从「奢侈品」变「日用品」：DeepSeek V4 CSA/HCA 混合注意力架构深度解析",
 *        §3.2 (mean-pool + projection, floor(n/m) entries, indexer dot
 *        product + per-query top-k), §4.1 (HCA 128:1), §5.2 (sliding window
 *        [max(0, i-W+1), i], scale 1/sqrt(head_dim)).
 * Readings where the pages are silent are listed in the design notes and
 * restated at each function below.
 *
 * Floating point: everything is fp64 except the fp8 quantisation helpers,
 * which follow the fp32 procedure the kernels use (a quantised code is an
 * integer decided by floating point, so both sides decide it in fp32).
 * Build WITHOUT -ffast-math: the fp32 helpers rely on IEEE rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * FP8 E4M3 (OCP 8-bit floating point specification, E4M3 encoding):
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
 * holds subnormals M * 2^-9; S.1111.111 is NaN; there are no infinities, so
 * the largest finite magnitude is S.1111.110 = 1.75 * 2^8 = 448.
 * --------------------------------------------------------------------- */
double oracle_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int mant = code & 7;
    double v;
    if (e == 0xF && mant == 7) return NAN;
    if (e == 0)
        v = ldexp((double)mant, -9);
    else
        v = ldexp(1.0 + mant / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round x to the nearest E4M3 value, ties to even mantissa, saturating any
 * finite magnitude above 448 to 448 ("satfinite").  NaN maps to the NaN code.
 * Written from the encoding definition above: find the quantum (spacing of
 * representable values) of the binade that holds |x|, round |x|/quantum to
 * the nearest integer with ties to even, then re-encode the result. */
uint8_t oracle_e4m3_encode(float xf) {
    double x = (double)xf;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) -> binade 2^(e2-1) */
    int ub = e2 - 1;        /* unbiased exponent of the binade */
    double quantum = (ub < -6) ? ldexp(1.0, -9) : ldexp(1.0, ub - 3);
    double q = a / quantum; /* exact: a is an fp32 value, quantum a power of 2 */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double v = r * quantum;
    if (v > 448.0) v = 448.0;
    if (v == 0.0) return sign;
    /* re-encode the representable value v */
    if (v < ldexp(1.0, -6)) {
        int mant = (int)(v / ldexp(1.0, -9));
        return (uint8_t)(sign | mant);
    }
    frexp(v, &e2);
    ub = e2 - 1;
    int mant = (int)((v / ldexp(1.0, ub) - 1.0) * 8.0);
    return (uint8_t)(sign | ((ub + 7) << 3) | mant);
}

/* Per-row E4M3 quantisation with a per-row fp32 scale, in the kernels' fp32
 * arithmetic: scale = amax/448 (a zero row takes scale 1), code =
 * E4M3(x/scale).  x holds `rows` rows of `d` fp32 values. */
void oracle_quantize_rows_e4m3(const float* x, long rows, int d, uint8_t* codes, float* scales) {
    for (long r = 0; r < rows; ++r) {
        const float* row = x + r * (long)d;
        float amax = 0.0f;
        for (int c = 0; c < d; ++c) {
            float v = fabsf(row[c]);
            if (v > amax) amax = v;
        }
        float scale = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        scales[r] = scale;
        for (int c = 0; c < d; ++c) codes[r * (long)d + c] = oracle_e4m3_encode(row[c] / scale);
    }
}

/* ------------------------------------------------------------------------
 * Hadamard rotation of indexer rows before fp8 (a reading of the DSA-lineage
 * indexer that "DS-V4 分析&学习" §1.2 and the gitcode analysis name, which
 * print no formula for it: a rotation spreads outlier channels before E4M3, and dot
 * products are unchanged because the normalised Walsh-Hadamard matrix H_d is
 * orthonormal and symmetric).  In place, in fp32, in a fixed order that the
 * kernels reproduce exactly: for stride s = 1, 2, 4, ..., d/2 every pair
 * (i, i + s) with i & s == 0 becomes (x_i + x_{i+s}, x_i - x_{i+s}); then every
 * value is multiplied by fp32(1/sqrt(d)).  d is a power of two.
 * --------------------------------------------------------------------- */
void oracle_hadamard_rows_f32(float* x, long rows, int d) {
    const float norm = (float)(1.0 / sqrt((double)d));
    for (long r = 0; r < rows; ++r) {
        float* row = x + r * (long)d;
        for (int s = 1; s < d; s <<= 1) {
            for (int i = 0; i < d; ++i) {
                if (i & s) continue;
                const float a = row[i], b = row[i + s];
                row[i] = a + b;
                row[i + s] = a - b;
            }
        }
        for (int i = 0; i < d; ++i) row[i] = row[i] * norm;
    }
}

/* ------------------------------------------------------------------------
 * Stage 1: KV compression ([P5] §3.2 formula; [P3] §1.3; [P1] §3.2).
 *
 * out[b, i, :] = (mean over p in win(i) of x[b, p, :]) @ W,   i < floor(n/m)
 *   overlap = 1 (CSA, ratio m = 4): win(i) = [m(i-1), m(i+1)) ∩ [0, n):
 *     the entry's own block and the block before it, 2m positions ([P3]
 *     §1.3), causal, the mean taken over the positions that exist;
 *   overlap = 0 (HCA, ratio 128): win(i) = [m i, m(i+1)).
 * A trailing partial block yields no entry ([P5] §3.2 truncates to n//m).
 * W is stored [d_in, d_out] and applied as a row vector times W.
 * --------------------------------------------------------------------- */
long oracle_num_entries(long n, long m) { return (m > 0 && n > 0) ? n / m : 0; }

void oracle_compress(const double* x, int B, int n, int d_in, const double* W, int d_out,
                     int m, int overlap, double* out) {
    int N_c = (int)oracle_num_entries(n, m);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < N_c; ++i) {
            long lo = overlap ? (long)m * (i - 1) : (long)m * i;
            long hi = (long)m * (i + 1);
            if (lo < 0) lo = 0;
            if (hi > n) hi = n;
            double* pooled = (double*)malloc(sizeof(double) * (size_t)d_in);
            for (int c = 0; c < d_in; ++c) pooled[c] = 0.0;
            for (long p = lo; p < hi; ++p) {
                const double* row = x + ((long)b * n + p) * d_in;
                for (int c = 0; c < d_in; ++c) pooled[c] += row[c];
            }
            double cnt = (double)(hi - lo);
            for (int c = 0; c < d_in; ++c) pooled[c] /= cnt;
            double* o = out + ((long)b * N_c + i) * d_out;
            for (int j = 0; j < d_out; ++j) {
                double acc = 0.0;
                for (int c = 0; c < d_in; ++c) acc += pooled[c] * W[(long)c * d_out + j];
                o[j] = acc;
            }
            free(pooled);
        }
    }
}

/* ------------------------------------------------------------------------
 * Stage 1, learned variant: the gated-softmax compressor.  [P1] §3.2 lists
 * the production compressor's parts -- a KV projection (linear_wkv), a gate
 * projection (linear_wgate), softmax / split / reshape, and an APE parameter;
 * ratio 4 overlapping, ratio 128 not -- but prints no formula.  Reading:
 *
 *   c = 2 when overlapping, else 1; each position p projects to
 *     v_p = x_p @ W_kv                     (c * d_out values)
 *     z_p = x_p @ W_gate + ape[p mod m]    (c * d_out logits; ape is [m, c*d_out])
 *   Entry i < floor(n/m), channel e < d_out, is a softmax-weighted pool over
 *   the positions of its window, taken per channel:
 *     overlapping: block i-1 contributes (z_p[e], v_p[e]) -- the first half of
 *       the projected channels -- and block i contributes (z_p[d_out+e],
 *       v_p[d_out+e]) -- the second half ("split"); entry 0 has block 0 only;
 *     otherwise: block i contributes (z_p[e], v_p[e]).
 *   out[i, e] = sum_p exp(z - zmax) v / sum_p exp(z - zmax)  over those terms.
 * --------------------------------------------------------------------- */
void oracle_compress_gated(const double* x, int B, int n, int d_in, const double* W_kv,
                           const double* W_gate, const double* ape, int d_out, int m, int overlap,
                           double* out) {
    int N_c = (int)oracle_num_entries(n, m);
    int cw = overlap ? 2 * d_out : d_out;          /* projected width */
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < N_c; ++i) {
            /* the window's terms: (position, channel offset of its half) */
            long first = (overlap && i > 0) ? (long)m * (i - 1) : (long)m * i;
            long last = (long)m * (i + 1);          /* exclusive */
            long nt = last - first;
            double* z = (double*)malloc(sizeof(double) * (size_t)nt);
            double* v = (double*)malloc(sizeof(double) * (size_t)nt);
            double* o = out + ((long)b * N_c + i) * d_out;
            for (int e = 0; e < d_out; ++e) {
                for (long t = 0; t < nt; ++t) {
                    long p = first + t;
                    int half = (overlap && p >= (long)m * i) ? d_out : 0;
                    int ch = half + e;
                    const double* row = x + ((long)b * n + p) * d_in;
                    double zv = 0.0, vv = 0.0;
                    for (int k = 0; k < d_in; ++k) {
                        zv += row[k] * W_gate[(long)k * cw + ch];
                        vv += row[k] * W_kv[(long)k * cw + ch];
                    }
                    z[t] = zv + ape[(long)(p % m) * cw + ch];
                    v[t] = vv;
                }
                double zmax = -INFINITY;
                for (long t = 0; t < nt; ++t) if (z[t] > zmax) zmax = z[t];
                double num = 0.0, den = 0.0;
                for (long t = 0; t < nt; ++t) {
                    double w = exp(z[t] - zmax);
                    num += w * v[t];
                    den += w;
                }
                o[e] = num / den;
            }
            free(z);
            free(v);
        }
    }
}

/* ------------------------------------------------------------------------
 * Decode-time compression state ("DS-V4 分析&学习", opening summary: the KV
 * cache is the compressed cache plus a state cache and a tail state; §1.3:
 * an overlapping entry spans the previous and the current block, which makes
 * the decode-time state the part to maintain).
 *
 * state[b] holds two rows of d_in values: row 0 the sum of the last complete
 * block's m rows, row 1 the running sum of the current block.  The token at
 * absolute position pos[b] (negative: element b has no token this step) is
 * added to row 1.  When it completes block j = pos/m, entry j is the mean
 * over its window -- blocks j-1 and j (2m rows) when overlap and j > 0, block
 * j alone otherwise -- times W; it is written to out[b, j] when j < N_cap, and
 * done[b] = j.  Then row 0 takes row 1 and row 1 restarts at zero.  done[b]
 * is -1 when no entry completed.  Tokens must arrive in position order.
 * --------------------------------------------------------------------- */
void oracle_compress_append(double* state, const double* x_new, int B, int d_in, const double* W,
                            int d_out, int m, int overlap, const int* pos, double* out, int N_cap,
                            int* done) {
    for (int b = 0; b < B; ++b) {
        done[b] = -1;
        const long p = pos[b];
        if (p < 0) continue;
        double* prev = state + (long)b * 2 * d_in;
        double* cur = prev + d_in;
        const double* xr = x_new + (long)b * d_in;
        for (int c = 0; c < d_in; ++c) cur[c] += xr[c];
        if ((p + 1) % m != 0) continue;
        const long j = p / m;
        const int both = overlap && j > 0;
        const double cnt = both ? 2.0 * m : (double)m;
        if (j < N_cap) {
            double* o = out + ((long)b * N_cap + j) * d_out;
            for (int k = 0; k < d_out; ++k) {
                double acc = 0.0;
                for (int c = 0; c < d_in; ++c) {
                    const double pooled = ((both ? prev[c] : 0.0) + cur[c]) / cnt;
                    acc += pooled * W[(long)c * d_out + k];
                }
                o[k] = acc;
            }
        }
        done[b] = (int)j;
        for (int c = 0; c < d_in; ++c) {
            prev[c] = cur[c];
            cur[c] = 0.0;
        }
    }
}

/* ------------------------------------------------------------------------
 * Causal visibility of compressed entries.  Entry i covers positions up to
 * m(i+1)-1 and becomes visible to the query at absolute position t once its
 * block is complete: i < floor((t+1)/m), further clamped to the number of
 * valid entries of the batch element.
 * --------------------------------------------------------------------- */
long oracle_visible_entries(long t, int m, long n_entries) {
    if (t < 0) return 0;
    long v = (t + 1) / m;
    return v < n_entries ? v : n_entries;
}

/* ------------------------------------------------------------------------
 * Stage 2: Lightning-Indexer score ([P5] §3.2 stage two; [P3] §1.2, §4).
 * score[t, s] = sum_h w[t, h] * ReLU( qI[t, h, :] . kI[s, :] ),  s < V(t).
 * One shared indexer key row per entry (MQA-like); each indexer head passes
 * its dot product through a ReLU before the heads are summed.  The per-query,
 * per-head gate weights w (any sign) are the gated form of the DSA-lineage
 * indexer the pages name ([P3] §1.2; [P1] head) without printing it; w_rows
 * NULL means w = 1 (the plain sum).
 *
 * Query rows are given as a list: row rr has batch element row_b[rr],
 * absolute position row_t[rr] and query values qI_rows[rr, H_I, d_I] (fp64,
 * already dequantised), optional weights w_rows[rr, H_I].  Keys kI [B, N_cap, d_I] are given either as fp64
 * values (kI_f64) or as E4M3 codes with one fp32 scale per entry (kI_codes +
 * kI_scale), dequantised here in fp64.
 * scores receives n_rows x N_cap values, NaN where the entry is not visible.
 * --------------------------------------------------------------------- */
static void key_row(const double* kI_f64, const uint8_t* kI_codes, const float* kI_scale, int b,
                    long s, int N_cap, int d_I, double* out) {
    long base = ((long)b * N_cap + s) * d_I;
    if (kI_f64) {
        for (int c = 0; c < d_I; ++c) out[c] = kI_f64[base + c];
    } else {
        double sc = (double)kI_scale[(long)b * N_cap + s];
        for (int c = 0; c < d_I; ++c) out[c] = oracle_e4m3_decode(kI_codes[base + c]) * sc;
    }
}

static double score_one(const double* qrow, const double* wrow, int H_I, int d_I,
                        const double* krow) {
    double s = 0.0;
    for (int h = 0; h < H_I; ++h) {
        double dot = 0.0;
        for (int c = 0; c < d_I; ++c) dot += qrow[(long)h * d_I + c] * krow[c];
        if (dot > 0.0) s += (wrow ? wrow[h] : 1.0) * dot;
    }
    return s;
}

void oracle_indexer_scores(const double* qI_rows, const double* w_rows, const int* row_b,
                           const int* row_t, long n_rows,
                           int H_I, int d_I, const double* kI_f64, const uint8_t* kI_codes,
                           const float* kI_scale, int N_cap, const int* n_entries, int m,
                           double* scores) {
    #pragma omp parallel for schedule(dynamic, 4)
    for (long rr = 0; rr < n_rows; ++rr) {
        int b = row_b[rr];
        const double* qrow = qI_rows + rr * (long)H_I * d_I;
        const double* wrow = w_rows ? w_rows + rr * (long)H_I : NULL;
        long V = oracle_visible_entries(row_t[rr], m, n_entries[b]);
        double* out = scores + rr * (long)N_cap;
        double* krow = (double*)malloc(sizeof(double) * (size_t)d_I);
        for (long s = 0; s < N_cap; ++s) {
            if (s < V) {
                key_row(kI_f64, kI_codes, kI_scale, b, s, N_cap, d_I, krow);
                out[s] = score_one(qrow, wrow, H_I, d_I, krow);
            } else {
                out[s] = NAN;
            }
        }
        free(krow);
    }
}

/* ------------------------------------------------------------------------
 * Stage 2b: per-query top-k ([P5] §3.2 torch.topk over the indexer score).
 * The k largest visible scores; equal scores are ordered by lower entry
 * index first; with fewer than k visible entries all of them are taken and
 * the row is padded with -1.  idx_out rows are written in (score desc,
 * index asc) order.  kth[2*rr] / kth[2*rr+1] receive the k-th and (k+1)-th
 * largest scores (NaN where they do not exist); smax[rr] the largest |score|.
 * --------------------------------------------------------------------- */
typedef struct { double s; long i; } scored_t;

static int cmp_scored(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

void oracle_indexer_topk(const double* qI_rows, const double* w_rows, const int* row_b,
                         const int* row_t, long n_rows,
                         int H_I, int d_I, const double* kI_f64, const uint8_t* kI_codes,
                         const float* kI_scale, int N_cap, const int* n_entries, int m, int topk,
                         int* idx_out, double* kth, double* smax) {
    #pragma omp parallel for schedule(dynamic, 4)
    for (long rr = 0; rr < n_rows; ++rr) {
        int b = row_b[rr];
        const double* qrow = qI_rows + rr * (long)H_I * d_I;
        const double* wrow = w_rows ? w_rows + rr * (long)H_I : NULL;
        long V = oracle_visible_entries(row_t[rr], m, n_entries[b]);
        scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)(V > 0 ? V : 1));
        double* krow = (double*)malloc(sizeof(double) * (size_t)d_I);
        double amax = 0.0;
        for (long s = 0; s < V; ++s) {
            key_row(kI_f64, kI_codes, kI_scale, b, s, N_cap, d_I, krow);
            all[s].s = score_one(qrow, wrow, H_I, d_I, krow);
            all[s].i = s;
            if (fabs(all[s].s) > amax) amax = fabs(all[s].s);
        }
        qsort(all, (size_t)V, sizeof(scored_t), cmp_scored);
        int* out = idx_out + rr * (long)topk;
        for (int j = 0; j < topk; ++j) out[j] = (j < V) ? (int)all[j].i : -1;
        if (kth) {
            kth[2 * rr] = (topk >= 1 && topk <= V) ? all[topk - 1].s : NAN;
            kth[2 * rr + 1] = (topk < V) ? all[topk].s : NAN;
        }
        if (smax) smax[rr] = amax;
        free(krow);
        free(all);
    }
}

/* ------------------------------------------------------------------------
 * Stage 3: joint-softmax MQA attention over the selected compressed entries
 * plus the sliding window of raw KV ([P3] §1.2, §1.5; [P5] §5.2).
 *
 * Keys and values are the same vectors (shared-KV MQA: one KV head serves
 * every query head).  For query row rr (batch element row_b[rr], absolute
 * position t = row_t[rr], query q_rows[rr, H, D]) and head h:
 *   S_c(t) = the compressed entries listed for the row,
 *   S_w(t) = raw positions p with max(0, t-W+1) <= p <= t that the raw
 *            buffer holds (raw row j holds position raw_pos0[b] + j, rows
 *            0 <= j < raw_len[b], positions < 0 are never valid),
 *   z_s   = scale * q[t,h] . key_s,
 *   o     = sum_s exp(z_s - max z) key_s / sum_s exp(z_s - max z)
 * over the MULTISET S_c ∪ S_w (a compressed entry and a raw row are
 * different keys; nothing is de-duplicated; no sink term), lse = log sum
 * exp z.  An empty set gives o = 0 and lse = -inf.
 * --------------------------------------------------------------------- */
static void attend_row(const double* q, int H, int D, double scale, const double** keys, long nk,
                       double* o, double* lse, double* z) {
    for (int h = 0; h < H; ++h) {
        const double* qh = q + (long)h * D;
        double* oh = o + (long)h * D;
        for (int c = 0; c < D; ++c) oh[c] = 0.0;
        if (nk == 0) {
            if (lse) lse[h] = -INFINITY;
            continue;
        }
        double zmax = -INFINITY;
        for (long s = 0; s < nk; ++s) {
            double dot = 0.0;
            for (int c = 0; c < D; ++c) dot += qh[c] * keys[s][c];
            z[s] = dot * scale;
            if (z[s] > zmax) zmax = z[s];
        }
        double den = 0.0;
        for (long s = 0; s < nk; ++s) {
            double w = exp(z[s] - zmax);
            den += w;
            for (int c = 0; c < D; ++c) oh[c] += w * keys[s][c];
        }
        for (int c = 0; c < D; ++c) oh[c] /= den;
        if (lse) lse[h] = zmax + log(den);
    }
}

static long window_keys(const double* kv_raw, int b, int L_raw, int D, const int* raw_pos0,
                        const int* raw_len, int window, long t, const double** keys, long nk) {
    long lo = t - window + 1;
    if (lo < 0) lo = 0;
    for (long p = lo; p <= t && window > 0; ++p) {
        long j = p - raw_pos0[b];
        if (j < 0 || j >= raw_len[b] || j >= L_raw) continue;
        keys[nk++] = kv_raw + ((long)b * L_raw + j) * D;
    }
    return nk;
}

/* Sparse attention: S_c(t) = the non-negative entries of idx_rows[rr, :]
 * below N_cap (negative entries are padding; entries >= N_cap are ignored). */
void oracle_sparse_attn(const double* q_rows, const int* row_b, const int* row_t, long n_rows, int H,
                        int D, const double* kv_c, int N_cap, const int* idx_rows, int topk,
                        const double* kv_raw, int L_raw, const int* raw_pos0, const int* raw_len,
                        int window, double scale, double* out, double* lse) {
    #pragma omp parallel for schedule(dynamic, 4)
    for (long rr = 0; rr < n_rows; ++rr) {
        int b = row_b[rr];
        long t = row_t[rr];
        long cap = (long)topk + (window > 0 ? window : 0);
        const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(cap + 1));
        double* z = (double*)malloc(sizeof(double) * (size_t)(cap + 1));
        long nk = 0;
        for (int j = 0; j < topk; ++j) {
            int s = idx_rows[rr * (long)topk + j];
            if (s < 0 || s >= N_cap) continue;
            keys[nk++] = kv_c + ((long)b * N_cap + s) * D;
        }
        nk = window_keys(kv_raw, b, L_raw, D, raw_pos0, raw_len, window, t, keys, nk);
        attend_row(q_rows + rr * (long)H * D, H, D, scale, keys, nk, out + rr * (long)H * D,
                   lse ? lse + rr * (long)H : NULL, z);
        free(keys);
        free(z);
    }
}

/* HCA dense attention ([P3] §1.4; [P5] §4.3): S_c(t) = every entry
 * s < min(floor((t+1)/m), n_entries[b]) -- no top-k -- plus the window. */
void oracle_hca_attn(const double* q_rows, const int* row_b, const int* row_t, long n_rows, int H,
                     int D, const double* kv_c, int N_cap, const int* n_entries, int m,
                     const double* kv_raw, int L_raw, const int* raw_pos0, const int* raw_len,
                     int window, double scale, double* out, double* lse) {
    #pragma omp parallel for schedule(dynamic, 4)
    for (long rr = 0; rr < n_rows; ++rr) {
        int b = row_b[rr];
        long t = row_t[rr];
        long V = oracle_visible_entries(t, m, n_entries[b]);
        if (V > N_cap) V = N_cap;
        long cap = V + (window > 0 ? window : 0);
        const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(cap + 1));
        double* z = (double*)malloc(sizeof(double) * (size_t)(cap + 1));
        long nk = 0;
        for (long s = 0; s < V; ++s) keys[nk++] = kv_c + ((long)b * N_cap + s) * D;
        nk = window_keys(kv_raw, b, L_raw, D, raw_pos0, raw_len, window, t, keys, nk);
        attend_row(q_rows + rr * (long)H * D, H, D, scale, keys, nk, out + rr * (long)H * D,
                   lse ? lse + rr * (long)H : NULL, z);
        free(keys);
        free(z);
    }
}
