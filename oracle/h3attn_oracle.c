/*
 * h3attn_oracle.c -- plain, slow, fp64 CPU oracle of the h3attn hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (the method of the MiniMax-H3 denoiser's attention block):
 *   - per-head Q/K RMSNorm followed by rotary position embedding, the fused
 *     prologue the "H3 Runtime Current State" page lists as missing under
 *     Owned Performance Kernels ("Fused Q/K RMSNorm, RoPE, and layout work"),
 *     and that the "Buyer Questions: Current Evidence Status" block-24 profile books as
 *     "norm/RoPE" ahead of attention;
 *   - non-causal softmax(Q K^T * scale) V over a packed video+audio token
 *     sequence ("H3 Runtime Current State", Implemented And Validated: "H3
 *     packed denoising"; "Open-H3-Regenerate-2K", Forward table: dense cuDNN
 *     attention in standard_fwd), one sequence per cu_seqlens segment
 *     ("Ragged Ulysses sequence parallelism").
 *
 * The pages print no formula for either step.  The readings taken here:
 *   RMSNorm:  y = x / sqrt(mean(x^2) + eps) * gamma, over the head_dim values
 *             of one (token, head) row; gamma shared by all heads.
 *   RoPE:     adjacent pairs (x[2i], x[2i+1]) rotated by angle p * f_i:
 *               y[2i]   = x[2i] cos a - x[2i+1] sin a
 *               y[2i+1] = x[2i] sin a + x[2i+1] cos a
 *             3D tokens: dims [0,st) use t, [st,st+sh) use h, the rest use w;
 *             inside a section of width ds, pair i has f_i = theta^(-2i/ds).
 *             1D tokens: one position over all dims, f_i = theta^(-2i/d).
 *   Attention: s_j = scale * (q . k_j) over the keys of the query's sequence,
 *             p_j = exp(s_j - max_j s_j), o = sum_j p_j v_j / sum_j p_j,
 *             lse = max_j s_j + log(sum_j p_j).
 *   Order:    RMSNorm, then RoPE, then one rounding to bfloat16 (nearest,
 *             ties to even) -- the interface tensor attention consumes.
 *   Partials: attention of queries against one block of a split key set, and
 *             the combination of such partial results by their log-sum-exp
 *             (h3o_attention_kv, h3o_merge): the pieces a key-split schedule of
 *             the sequence-parallel attention ("H3 Runtime Current State",
 *             "Ragged Ulysses sequence parallelism", "Sequence-sharded 50-block
 *             execution") needs; the identity that the combined parts equal the
 *             attention over all keys is what pins them.
 *   Block-sparse: attention restricted to listed blocks of keys per block of
 *             queries (h3o_attention_block_sparse): the execution of a given
 *             pattern for the sparse backend of the "Open-H3-Regenerate-2K"
 *             refine table; the pages give no selection rule, so none is here.
 *   Projection: the Q/K/V projection followed by the same norm and rotation
 *             (h3o_qkv_norm_rope), for the prologue fused into its epilogue.
 *
 * Every loop below is the definition written out in double precision, in the
 * order stated, with no blocking, fusion or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

int h3o_version(void) { return 1; }

/* bfloat16 bit pattern -> double (exact). */
double h3o_bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> nearest bfloat16 (8 significant bits, float32 exponent range),
 * ties to even, rounded once from the double value. */
uint16_t h3o_bf16_from_double(double x) {
    if (isnan(x)) return (uint16_t)0x7FC0;
    uint16_t sign = signbit(x) ? (uint16_t)0x8000 : (uint16_t)0;
    double ax = fabs(x);
    /* largest finite bf16 is 255 * 2^120; the midpoint to 2^128 is 511 * 2^119
     * and ties go to the even neighbour, which is infinity. */
    if (ax >= ldexp(511.0, 119)) return (uint16_t)(sign | 0x7F80);
    double quantum;
    if (ax < ldexp(1.0, -126)) {
        quantum = ldexp(1.0, -133);            /* subnormal spacing */
    } else {
        int e;
        frexp(ax, &e);                         /* ax in [2^(e-1), 2^e) */
        quantum = ldexp(1.0, e - 1 - 7);       /* 7 stored mantissa bits */
    }
    double r = nearbyint(ax / quantum) * quantum; /* default mode: nearest-even */
    float f = (float)r;                        /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void h3o_bf16_round_array(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = h3o_bf16_from_double(x[i]);
}

/* Rotate the pair (row[i0], row[i0+1]) by angle a. */
static void rotate_pair(double* row, int i0, double a) {
    double c = cos(a), s = sin(a);
    double x0 = row[i0], x1 = row[i0 + 1];
    row[i0] = x0 * c - x1 * s;
    row[i0 + 1] = x0 * s + x1 * c;
}

/* Rotary embedding of one row of length d for a token of the given kind. */
static void rope_row(double* row, int d, int kind, const int32_t* p,
                     int sec_t, int sec_h, int sec_w, double theta) {
    if (kind == 1) {
        int start[3] = {0, sec_t, sec_t + sec_h};
        int width[3] = {sec_t, sec_h, sec_w};
        for (int axis = 0; axis < 3; ++axis) {
            for (int i = 0; i < width[axis] / 2; ++i) {
                double f = pow(theta, -2.0 * (double)i / (double)width[axis]);
                rotate_pair(row, start[axis] + 2 * i, (double)p[axis] * f);
            }
        }
    } else if (kind == 2) {
        for (int i = 0; i < d / 2; ++i) {
            double f = pow(theta, -2.0 * (double)i / (double)d);
            rotate_pair(row, 2 * i, (double)p[0] * f);
        }
    }
}

/*
 * RMSNorm (if gamma != NULL) then RoPE (if pos != NULL and kind[n] != 0) of
 * every (token, head) row of x.
 *   x:      bf16 bits, row (n, h) starts at x + n*s_tok + h*s_head (elements).
 *   gamma:  bf16 bits [d] or NULL.
 *   pos:    int32 [n_tokens][3] or NULL;  kind: uint8 [n_tokens] (0, 1 = 3D, 2 = 1D).
 *   y64:    double [n_tokens][n_heads][d] or NULL (unrounded result).
 *   y16:    bf16 bits [n_tokens][n_heads][d] or NULL (result rounded once).
 * Returns 0, or -1 on invalid arguments.
 */
int h3o_rmsnorm_rope(const uint16_t* x, int64_t n_tokens, int32_t n_heads, int32_t d,
                     int64_t s_tok, int64_t s_head, const uint16_t* gamma, double eps,
                     const int32_t* pos, const uint8_t* kind,
                     int32_t sec_t, int32_t sec_h, int32_t sec_w, double theta,
                     double* y64, uint16_t* y16) {
    if (!x || n_tokens < 0 || n_heads <= 0 || d <= 0 || d > 1024 || (d & 1)) return -1;
    if (pos && (!kind || sec_t < 0 || sec_h < 0 || sec_w < 0 || (sec_t & 1) || (sec_h & 1) ||
                (sec_w & 1) || sec_t + sec_h + sec_w != d))
        return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tokens; ++n) {
        double row[1024];
        for (int h = 0; h < n_heads; ++h) {
            const uint16_t* src = x + n * s_tok + (int64_t)h * s_head;
            for (int i = 0; i < d; ++i) row[i] = h3o_bf16_to_double(src[i]);
            if (gamma) {
                double ss = 0.0;
                for (int i = 0; i < d; ++i) ss += row[i] * row[i];
                double r = sqrt(ss / (double)d + eps);
                for (int i = 0; i < d; ++i) row[i] = row[i] / r * h3o_bf16_to_double(gamma[i]);
            }
            if (pos && kind[n] != 0)
                rope_row(row, d, kind[n], pos + 3 * n, sec_t, sec_h, sec_w, theta);
            int64_t o = (n * n_heads + h) * (int64_t)d;
            if (y64) for (int i = 0; i < d; ++i) y64[o + i] = row[i];
            if (y16) for (int i = 0; i < d; ++i) y16[o + i] = h3o_bf16_from_double(row[i]);
        }
    }
    return 0;
}

/*
 * Attention for selected query rows.
 *   q, k, v:    bf16 bits, packed [total][n_heads][d].
 *   cu_seqlens: int32 [nseq + 1], cu[0] = 0, non-decreasing, cu[nseq] = total.
 *   rows:       int64 [nrows] global query token indices (NULL = all tokens).
 *   o:          double [nrows][n_heads][d];  lse: double [nrows][n_heads] or NULL.
 * A query attends to every key of its own sequence, none of any other.
 * Returns 0, or -1 on invalid arguments.
 */
int h3o_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t total,
                  int32_t n_heads, int32_t d, const int32_t* cu_seqlens, int32_t nseq,
                  double scale, const int64_t* rows, int64_t nrows, double* o, double* lse) {
    if (!q || !k || !v || !o || !cu_seqlens || total <= 0 || n_heads <= 0 || d <= 0 || d > 1024 ||
        nseq <= 0)
        return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[nseq] != total) return -1;
    for (int s = 0; s < nseq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    if (!rows) nrows = total;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows ? rows[r] : r;
        if (t < 0 || t >= total) return -1;
    }
    double* kd = (double*)malloc(sizeof(double) * (size_t)total * (size_t)d);
    double* vd = (double*)malloc(sizeof(double) * (size_t)total * (size_t)d);
    if (!kd || !vd) { free(kd); free(vd); return -2; }
    for (int h = 0; h < n_heads; ++h) {
        /* this head's keys and values as doubles, [total][d] */
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < total; ++j) {
            for (int i = 0; i < d; ++i) {
                kd[j * d + i] = h3o_bf16_to_double(k[(j * n_heads + h) * (int64_t)d + i]);
                vd[j * d + i] = h3o_bf16_to_double(v[(j * n_heads + h) * (int64_t)d + i]);
            }
        }
        #pragma omp parallel for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t t = rows ? rows[r] : r;
            int s = 0;
            while (!(cu_seqlens[s] <= t && t < cu_seqlens[s + 1])) ++s;
            int64_t j0 = cu_seqlens[s], j1 = cu_seqlens[s + 1];
            double qd[1024];
            for (int i = 0; i < d; ++i) qd[i] = h3o_bf16_to_double(q[(t * n_heads + h) * (int64_t)d + i]);
            double* sc = (double*)malloc(sizeof(double) * (size_t)(j1 - j0));
            double mx = -INFINITY;
            for (int64_t j = j0; j < j1; ++j) {
                double dot = 0.0;
                for (int i = 0; i < d; ++i) dot += qd[i] * kd[j * d + i];
                sc[j - j0] = scale * dot;
                if (sc[j - j0] > mx) mx = sc[j - j0];
            }
            double acc[1024];
            for (int i = 0; i < d; ++i) acc[i] = 0.0;
            double den = 0.0;
            for (int64_t j = j0; j < j1; ++j) {
                double p = exp(sc[j - j0] - mx);
                den += p;
                for (int i = 0; i < d; ++i) acc[i] += p * vd[j * d + i];
            }
            double* out = o + (r * n_heads + h) * (int64_t)d;
            for (int i = 0; i < d; ++i) out[i] = acc[i] / den;
            if (lse) lse[r * n_heads + h] = mx + log(den);
            free(sc);
        }
    }
    free(kd);
    free(vd);
    return 0;
}

/*
 * Attention of each segment's query rows against a separate set of key/value
 * rows: segment s's queries [cu_q[s], cu_q[s+1]) of q attend to the keys
 * [cu_k[s], cu_k[s+1]) of k and v.  This is the partial attention a key-split
 * (context-parallel) schedule computes per key block; its (o, lse) pairs are
 * combined by h3o_merge.  The arithmetic is the definition above; an empty key
 * range is an empty sum: o = 0 and lse = -inf.
 *   q: bf16 bits [total_q][n_heads][d];  k, v: [total_k][n_heads][d].
 *   o: double [total_q][n_heads][d];     lse: double [total_q][n_heads] or NULL.
 * Returns 0, or -1 on invalid arguments.
 */
int h3o_attention_kv(const uint16_t* q, int64_t total_q, const uint16_t* k, const uint16_t* v,
                     int64_t total_k, int32_t n_heads, int32_t d, const int32_t* cu_q,
                     const int32_t* cu_k, int32_t nseq, double scale, double* o, double* lse) {
    if (!q || !o || !cu_q || !cu_k || total_q < 0 || total_k < 0 || n_heads <= 0 || d <= 0 ||
        d > 1024 || nseq <= 0)
        return -1;
    if (total_k > 0 && (!k || !v)) return -1;
    if (cu_q[0] != 0 || cu_q[nseq] != total_q || cu_k[0] != 0 || cu_k[nseq] != total_k) return -1;
    for (int s = 0; s < nseq; ++s)
        if (cu_q[s + 1] < cu_q[s] || cu_k[s + 1] < cu_k[s]) return -1;
    for (int h = 0; h < n_heads; ++h) {
        #pragma omp parallel for schedule(dynamic, 1)
        for (int64_t t = 0; t < total_q; ++t) {
            int seg = 0;
            while (!(cu_q[seg] <= t && t < cu_q[seg + 1])) ++seg;
            const int64_t kb = cu_k[seg], ke = cu_k[seg + 1];
            double* row_o = o + (t * n_heads + h) * (int64_t)d;
            if (ke == kb) {  /* no keys: the empty sum */
                for (int i = 0; i < d; ++i) row_o[i] = 0.0;
                if (lse) lse[t * n_heads + h] = -INFINITY;
                continue;
            }
            double qv[1024];
            for (int i = 0; i < d; ++i) qv[i] = h3o_bf16_to_double(q[(t * n_heads + h) * (int64_t)d + i]);
            double* s_row = (double*)malloc(sizeof(double) * (size_t)(ke - kb));
            double m = -INFINITY;
            for (int64_t j = kb; j < ke; ++j) {
                double qk = 0.0;
                for (int i = 0; i < d; ++i) qk += qv[i] * h3o_bf16_to_double(k[(j * n_heads + h) * (int64_t)d + i]);
                s_row[j - kb] = scale * qk;
                if (s_row[j - kb] > m) m = s_row[j - kb];
            }
            double num[1024];
            for (int i = 0; i < d; ++i) num[i] = 0.0;
            double z = 0.0;
            for (int64_t j = kb; j < ke; ++j) {
                const double w = exp(s_row[j - kb] - m);
                z += w;
                for (int i = 0; i < d; ++i) num[i] += w * h3o_bf16_to_double(v[(j * n_heads + h) * (int64_t)d + i]);
            }
            for (int i = 0; i < d; ++i) row_o[i] = num[i] / z;
            if (lse) lse[t * n_heads + h] = m + log(z);
            free(s_row);
        }
    }
    return 0;
}

/*
 * Combination of partial attention results over disjoint key sets, by their
 * log-sum-exp: with L = log(sum_p exp(lse_p)), o = sum_p exp(lse_p - L) o_p.
 * (Each o_p is its part's weighted mean of values with total weight exp(lse_p);
 * the whole mean weights each part by its share of the total.)  L is formed as
 * M + log(sum_p exp(lse_p - M)) with M = max_p lse_p.  Parts with lse = -inf
 * are empty and carry no weight; a row whose parts are all empty gives o = 0,
 * L = -inf.
 *   o_parts:   double [n_parts][n_rows][d];  lse_parts: double [n_parts][n_rows].
 *   o:         double [n_rows][d];           lse:       double [n_rows].
 * Returns 0, or -1 on invalid arguments.
 */
int h3o_merge(const double* o_parts, const double* lse_parts, int32_t n_parts, int64_t n_rows,
              int32_t d, double* o, double* lse) {
    if (!o_parts || !lse_parts || !o || !lse || n_parts <= 0 || n_rows < 0 || d <= 0) return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        double mx = -INFINITY;
        for (int p = 0; p < n_parts; ++p)
            if (lse_parts[p * n_rows + r] > mx) mx = lse_parts[p * n_rows + r];
        double* out = o + r * d;
        if (mx == -INFINITY) {
            for (int i = 0; i < d; ++i) out[i] = 0.0;
            lse[r] = -INFINITY;
            continue;
        }
        double den = 0.0;
        for (int p = 0; p < n_parts; ++p) den += exp(lse_parts[p * n_rows + r] - mx);
        const double L = mx + log(den);
        for (int i = 0; i < d; ++i) out[i] = 0.0;
        for (int p = 0; p < n_parts; ++p) {
            const double w = exp(lse_parts[p * n_rows + r] - L);
            const double* op = o_parts + (p * n_rows + r) * (int64_t)d;
            for (int i = 0; i < d; ++i) out[i] += w * op[i];
        }
        lse[r] = L;
    }
    return 0;
}

/*
 * The Q/K/V projection of the block followed by the per-head RMSNorm + RoPE of
 * Q and K: the prologue fused into the projection that produces its input
 * ("H3 Runtime Current State", Owned Performance Kernels: fused Q/K RMSNorm,
 * RoPE and layout work; "Buyer Questions: Current Evidence Status", block
 * composition: the projection output feeds norm/RoPE, and its strided NHD
 * layout is read in place).  The projection is not rounded before the norm:
 * the definition is the exact composition, rounded once at the end.
 *   x:     bf16 bits, token n's row at x + n*s_x, dim_in values.
 *   w:     bf16 bits [3*n_heads*d][dim_in] (one row per output feature).
 *   bias:  bf16 bits [3*n_heads*d] or NULL.
 *   Feature f = sum_c x[n][c] * w[f][c] (+ bias[f]); features [0, H*d) are Q
 *   (head f / d), [H*d, 2*H*d) K, [2*H*d, 3*H*d) V.  Q and K rows of length d go
 *   through RMSNorm (gamma_q / gamma_k when given, eps inside the root) and RoPE
 *   (when pos is given) exactly as h3o_rmsnorm_rope; V is the projection.
 *   rows:  int64 [nrows] token indices (NULL = every token).
 *   q64, k64, v64: double [nrows][n_heads][d] or NULL (unrounded);
 *   q16, k16, v16: bf16 bits, the same rounded once (NULL to skip).
 * Returns 0, or -1 on invalid arguments.
 */
int h3o_qkv_norm_rope(const uint16_t* x, int64_t n_tokens, int32_t dim_in, int64_t s_x,
                      const uint16_t* w, const uint16_t* bias, int32_t n_heads, int32_t d,
                      const uint16_t* gamma_q, const uint16_t* gamma_k, double eps,
                      const int32_t* pos, const uint8_t* kind, int32_t sec_t, int32_t sec_h,
                      int32_t sec_w, double theta, const int64_t* rows, int64_t nrows,
                      double* q64, double* k64, double* v64, uint16_t* q16, uint16_t* k16,
                      uint16_t* v16) {
    if (!x || !w || n_tokens < 0 || dim_in <= 0 || dim_in > 8192 || n_heads <= 0 || d <= 0 ||
        d > 1024 || (d & 1))
        return -1;
    if (pos && (!kind || sec_t < 0 || sec_h < 0 || sec_w < 0 || (sec_t & 1) || (sec_h & 1) ||
                (sec_w & 1) || sec_t + sec_h + sec_w != d))
        return -1;
    if (!rows) nrows = n_tokens;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows ? rows[r] : r;
        if (t < 0 || t >= n_tokens) return -1;
    }
    const int64_t hd = (int64_t)n_heads * d;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t n = rows ? rows[r] : r;
        double xin[8192];
        for (int c = 0; c < dim_in; ++c) xin[c] = h3o_bf16_to_double(x[n * s_x + c]);
        for (int part = 0; part < 3; ++part) {   /* 0 = Q, 1 = K, 2 = V */
            const uint16_t* g = part == 0 ? gamma_q : part == 1 ? gamma_k : NULL;
            double* out64 = part == 0 ? q64 : part == 1 ? k64 : v64;
            uint16_t* out16 = part == 0 ? q16 : part == 1 ? k16 : v16;
            for (int h = 0; h < n_heads; ++h) {
                double feat[1024];
                for (int i = 0; i < d; ++i) {
                    const int64_t f = part * hd + (int64_t)h * d + i;
                    double acc = 0.0;
                    for (int c = 0; c < dim_in; ++c) acc += xin[c] * h3o_bf16_to_double(w[f * dim_in + c]);
                    feat[i] = bias ? acc + h3o_bf16_to_double(bias[f]) : acc;
                }
                if (part < 2 && g) {
                    double sq = 0.0;
                    for (int i = 0; i < d; ++i) sq += feat[i] * feat[i];
                    const double rms = sqrt(sq / (double)d + eps);
                    for (int i = 0; i < d; ++i) feat[i] = feat[i] / rms * h3o_bf16_to_double(g[i]);
                }
                if (part < 2 && pos && kind[n] != 0)
                    rope_row(feat, d, kind[n], pos + 3 * n, sec_t, sec_h, sec_w, theta);
                const int64_t o = (r * n_heads + h) * (int64_t)d;
                if (out64) for (int i = 0; i < d; ++i) out64[o + i] = feat[i];
                if (out16) for (int i = 0; i < d; ++i) out16[o + i] = h3o_bf16_from_double(feat[i]);
            }
        }
    }
    return 0;
}

/*
 * Block-sparse attention over a dense batch.  The pages name a sparse attention
 * backend ("Open-H3-Regenerate-2K", refine timing table: "+ Sol-Attn sparse
 * attention", lossy and quality-gated per "H3 Runtime Current State", Next Work)
 * but not its selection rule, so only the execution of a given block pattern is
 * defined here: the n_q queries of a sequence are cut into query blocks of block_q
 * rows and its n_kv keys into key blocks of block_k keys; for every (batch b,
 * head h, query block qb) the list
 *     blk_idx[blk_off[c] .. blk_off[c + 1]),  c = (b * n_heads + h) * QB + qb,
 *     QB = ceil(n_q / block_q),
 * names the key blocks its queries see.  A query attends to exactly the keys of
 * the listed blocks (keys past n_kv in a listed last block do not exist; a block
 * listed twice counts once), with the arithmetic of h3o_attention on that key
 * set; no key at all is the empty sum, o = 0 and lse = -inf.
 *   q: bf16 bits [batch][n_q][n_heads][d];  k, v: [batch][n_kv][n_heads][d].
 *   rows: int64 [nrows] query rows b * n_q + t (NULL = all batch * n_q rows).
 *   o: double [nrows][n_heads][d];  lse: double [nrows][n_heads] or NULL.
 * Returns 0, or -1 on invalid arguments (offsets not starting at 0 or decreasing,
 * a block index outside [0, ceil(n_kv / block_k))).
 */
int h3o_attention_block_sparse(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               int32_t batch, int64_t n_q, int64_t n_kv, int32_t n_heads, int32_t d,
                               int32_t block_q, int32_t block_k, const int32_t* blk_off,
                               const int32_t* blk_idx, double scale, const int64_t* rows,
                               int64_t nrows, double* o, double* lse) {
    if (!q || !o || !blk_off || batch <= 0 || n_q < 0 || n_kv < 0 || n_heads <= 0 || d <= 0 ||
        d > 1024 || block_q <= 0 || block_k <= 0)
        return -1;
    if (n_kv > 0 && (!k || !v)) return -1;
    const int64_t n_qb = (n_q + block_q - 1) / block_q;
    const int64_t n_kb = (n_kv + block_k - 1) / block_k;
    const int64_t n_lists = (int64_t)batch * n_heads * n_qb;
    if (blk_off[0] != 0) return -1;
    for (int64_t c = 0; c < n_lists; ++c) {
        if (blk_off[c + 1] < blk_off[c]) return -1;
        for (int64_t e = blk_off[c]; e < blk_off[c + 1]; ++e)
            if (!blk_idx || blk_idx[e] < 0 || blk_idx[e] >= n_kb) return -1;
    }
    if (!rows) nrows = (int64_t)batch * n_q;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t g = rows ? rows[r] : r;
        if (g < 0 || g >= (int64_t)batch * n_q) return -1;
    }
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t g = rows ? rows[r] : r;
        const int64_t b = g / n_q, t = g % n_q;
        char* seen = (char*)calloc((size_t)(n_kb > 0 ? n_kb : 1), 1);
        double* s_row = (double*)malloc(sizeof(double) * (size_t)(n_kv > 0 ? n_kv : 1));
        for (int h = 0; h < n_heads; ++h) {
            const int64_t list = ((int64_t)b * n_heads + h) * n_qb + t / block_q;
            memset(seen, 0, (size_t)(n_kb > 0 ? n_kb : 1));
            for (int64_t e = blk_off[list]; e < blk_off[list + 1]; ++e) seen[blk_idx[e]] = 1;
            double qv[1024];
            for (int i = 0; i < d; ++i)
                qv[i] = h3o_bf16_to_double(q[((b * n_q + t) * n_heads + h) * (int64_t)d + i]);
            /* scores of the visible keys, and their maximum */
            double m = -INFINITY;
            int64_t n_vis = 0;
            for (int64_t j = 0; j < n_kv; ++j) {
                if (!seen[j / block_k]) continue;
                const int64_t kr = ((b * n_kv + j) * n_heads + h) * (int64_t)d;
                double qk = 0.0;
                for (int i = 0; i < d; ++i) qk += qv[i] * h3o_bf16_to_double(k[kr + i]);
                s_row[j] = scale * qk;
                if (s_row[j] > m) m = s_row[j];
                ++n_vis;
            }
            double* row_o = o + (r * n_heads + h) * (int64_t)d;
            if (n_vis == 0) {  /* no key: the empty sum */
                for (int i = 0; i < d; ++i) row_o[i] = 0.0;
                if (lse) lse[r * n_heads + h] = -INFINITY;
                continue;
            }
            double num[1024];
            for (int i = 0; i < d; ++i) num[i] = 0.0;
            double z = 0.0;
            for (int64_t j = 0; j < n_kv; ++j) {
                if (!seen[j / block_k]) continue;
                const int64_t vr = ((b * n_kv + j) * n_heads + h) * (int64_t)d;
                const double wgt = exp(s_row[j] - m);
                z += wgt;
                for (int i = 0; i < d; ++i) num[i] += wgt * h3o_bf16_to_double(v[vr + i]);
            }
            for (int i = 0; i < d; ++i) row_o[i] = num[i] / z;
            if (lse) lse[r * n_heads + h] = m + log(z);
        }
        free(seen);
        free(s_row);
    }
    return 0;
}
