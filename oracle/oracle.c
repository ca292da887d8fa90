/*
 * oracle.c -- plain fp64 CPU oracle for single-token paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, constant or helper with the CUDA library; it is deliberately slow
 * and written so that each line can be checked against the definitions on
 * the pages it cites:
 *
 *   [HEADS]  xuesongtap "attention-head" article (MHA/MQA/GQA, sliding
 *            window, MLA): §1 Attention equation and Bytes_KV equation,
 *            §2 group rule and §2.2 table, §3 sliding-window figure,
 *            §5.2 absorption identities, §5.3 MLA decode softmax,
 *            §5.4 Bytes_MLA equation.
 *   [EVOL]   toolsku "AI演算法注意力機制演進" article: GQA implementation
 *            (repeat_kv expansion, matmul, softmax, matmul).
 *
 * Every input is read in its stored precision (fp32, bf16 or fp64) and
 * widened to double exactly; all arithmetic is fp64.  No blocking, no
 * online softmax, no reordering: scores for the whole visible range are
 * materialised, the maximum subtracted, exponentiated, normalised and used
 * to weight the value rows, in that order.
 *
 * Cache layout read here (the library's documented storage format):
 *   K/V cache   [num_blocks][H_kv][block_size][d]
 *   MLA cache   [num_blocks][block_size][d_c + d_r]   (cols [0,d_c) = c_j,
 *                                                       cols [d_c,d_c+d_r) = k^R_j)
 *   block table [B][max_blocks]  logical block i of sequence b lives in
 *                                physical block block_table[b*max_blocks+i].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

enum { ORC_OK = 0, ORC_BAD_ARG = 1, ORC_NO_MEM = 2 };

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double orc_read(const void *base, size_t idx, int dtype) {
    if (dtype == ORC_F64) return ((const double *)base)[idx];
    if (dtype == ORC_F32) return (double)((const float *)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Visible key range of a decode query whose cache holds T tokens (the
 * current token included, at position T-1).  Full causal: [0, T).
 * Causal sliding window of width w > 0 covers the current position and the
 * w-1 before it ([HEADS] §3 figure: w=3, row 8 sees {6,7,8}): [max(0,T-w), T).
 */
void orc_visible_range(int T, int window, int *lo, int *hi) {
    int l = 0;
    if (window > 0 && T - window > 0) l = T - window;
    *lo = (T > 0) ? l : 0;
    *hi = (T > 0) ? T : 0;
}

/* Position j of sequence b -> element offset of the row in a paged cache. */
static size_t orc_row_offset(const int32_t *block_table, int max_blocks, int b,
                             int j, int block_size, int n_heads_cache, int head,
                             int row_width) {
    int logical = j / block_size;
    int in_block = j % block_size;
    int32_t phys = block_table[(size_t)b * max_blocks + logical];
    return (((size_t)phys * n_heads_cache + head) * block_size + in_block) *
           (size_t)row_width;
}

/*
 * GQA / MQA / MHA decode attention ([HEADS] §1 Attention equation, §2 group
 * rule; [EVOL] GQA implementation).  For every sequence b and query head h:
 *
 *   kvh   = floor(h / (H_q / H_kv))        contiguous equal groups ([HEADS] §2)
 *   s_j   = scale * sum_k q[b,h,k] K[b,kvh,j,k]        j in visible range
 *   p_j   = exp(s_j - max s) / sum_i exp(s_i - max s)  (softmax over keys)
 *   out[b,h,:] = sum_j p_j V[b,kvh,j,:]
 *
 * q   [B][H_q][d], out [B][H_q][d] (fp64).  probs (optional) receives p for
 * every (b, h) in a [B][H_q][max_T] array, zero outside the visible range.
 * seq_lens[b] = T_b tokens cached, the current one included; T_b = 0 gives
 * a zero output row.
 */
/*
 * Decode attention with global tokens and a ring-buffer table
 * (attention-head article, §3: sliding window; window plus global tokens G,
 * whose figure has G = {0, 5}: row 8 sees {0, 5, 6, 7, 8} with w = 3, and
 * the global query of row 5 sees all of 0..5).  Key j of sequence b
 * (T = seq_lens[b]; the query is position T - 1) is visible when j < T and
 * (window <= 0 or j >= T - window or j < sink or j in G_b or T - 1 in G_b).
 * G_b is row b of gpos [B][n_g] (n_g = 0: empty), read in order up to its
 * first entry that does not exceed the one before.  The row of key j sits in
 * the block of the table slot that holds logical block i = j / block_size:
 *   - no ring: slot i;
 *   - ring, no global set: block i < A = ceil(sink / block_size) keeps slot
 *     i, block i >= A goes to slot A + i % ring;
 *   - ring with a global set (a window layer that also keeps the positions
 *     of G, §3): slots [0, n_g) are the global slots, slot k holding the
 *     block of position G_b[k]; a key in a block before the window's first
 *     block (there only keys of G are visible) is read through the global
 *     slot of its own position, and block i from the window's first block
 *     (max(0, T - window) / block_size) on through ring slot n_g + i % ring.
 *     The ring no longer holds the history a global query (T - 1 in G_b)
 *     would need, so such a query with T > window is refused (ORC_BAD_ARG).
 * Softmax over the visible keys only.  Same arrays and dtypes as
 * orc_decode_gqa; probs (optional) [B][H_q][max_T].
 */
/* index k with row[k] == x in the (ascending, possibly padded) set, or -1 */
static int orc_set_index(const int32_t *row, int n, int x) {
    int prev = -1;
    for (int k = 0; k < n; ++k) {
        if (row[k] <= prev) break;
        if (row[k] == x) return k;
        prev = row[k];
    }
    return -1;
}

static int orc_in_set(const int32_t *row, int n, int x) {
    return orc_set_index(row, n, x) >= 0;
}

static int orc_slot(int i, int sink, int ring, int block_size) {
    if (ring <= 0) return i;
    const int a = sink > 0 ? (sink + block_size - 1) / block_size : 0;
    return i < a ? i : a + i % ring;
}

int orc_decode_gqa_vis(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seq_lens, const int32_t *block_table,
                       double *out, double *probs, int max_T, int B, int H_q,
                       int H_kv, int d, int block_size, int max_blocks,
                       double scale, int window, int sink, int ring, int dtype,
                       const int32_t *gpos, int n_g) {
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || d <= 0 || block_size <= 0 ||
        H_q % H_kv != 0 || sink < 0 || ring < 0 || n_g < 0 || (n_g > 0 && !gpos) ||
        (n_g > 0 && ring > 0 && sink > 0))
        return ORC_BAD_ARG;
    const int group = H_q / H_kv;
    int status = ORC_OK;

#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H_q; ++h) {
            double *o = out + ((size_t)b * H_q + h) * d;
            for (int k = 0; k < d; ++k) o[k] = 0.0;
            if (probs)
                for (int j = 0; j < max_T; ++j)
                    probs[((size_t)b * H_q + h) * max_T + j] = 0.0;
            const int T = seq_lens[b];
            if (T <= 0) continue;
            const int kvh = h / group;
            /* the visible keys, in increasing order */
            int *keys = (int *)malloc(sizeof(int) * (size_t)T);
            double *s = (double *)malloc(sizeof(double) * (size_t)T);
            if (!keys || !s) {
                free(keys); free(s);
#pragma omp atomic write
                status = ORC_NO_MEM;
                continue;
            }
            const int32_t *grow = n_g > 0 ? gpos + (size_t)b * n_g : NULL;
            const int q_global = grow && orc_in_set(grow, n_g, T - 1);
            if (q_global && ring > 0 && window > 0 && T > window) {
                free(keys); free(s);
#pragma omp atomic write
                status = ORC_BAD_ARG;
                continue;
            }
            /* first block of the window (global-set ring layout) */
            const int w0 = (window > 0 && T > window ? T - window : 0) / block_size;
            int n = 0;
            for (int j = 0; j < T; ++j)
                if (window <= 0 || j >= T - window || j < sink || q_global ||
                    (grow && orc_in_set(grow, n_g, j)))
                    keys[n++] = j;
            const size_t q_off = ((size_t)b * H_q + h) * d;
            for (int t = 0; t < n; ++t) {
                const int j = keys[t];
                const int slot = (grow && ring > 0)
                                     ? (j / block_size < w0 ? orc_set_index(grow, n_g, j)
                                                            : n_g + (j / block_size) % ring)
                                     : orc_slot(j / block_size, sink, ring, block_size);
                const int32_t phys = block_table[(size_t)b * max_blocks + slot];
                const size_t r = (((size_t)phys * H_kv + kvh) * block_size + j % block_size) * d;
                double dot = 0.0;
                for (int k = 0; k < d; ++k)
                    dot += orc_read(q, q_off + k, dtype) * orc_read(k_cache, r + k, dtype);
                s[t] = scale * dot;
            }
            double m = s[0];
            for (int t = 1; t < n; ++t)
                if (s[t] > m) m = s[t];
            double z = 0.0;
            for (int t = 0; t < n; ++t) {
                s[t] = exp(s[t] - m);
                z += s[t];
            }
            for (int t = 0; t < n; ++t) s[t] /= z;
            for (int t = 0; t < n; ++t) {
                const int j = keys[t];
                const int slot = (grow && ring > 0)
                                     ? (j / block_size < w0 ? orc_set_index(grow, n_g, j)
                                                            : n_g + (j / block_size) % ring)
                                     : orc_slot(j / block_size, sink, ring, block_size);
                const int32_t phys = block_table[(size_t)b * max_blocks + slot];
                const size_t r = (((size_t)phys * H_kv + kvh) * block_size + j % block_size) * d;
                for (int k = 0; k < d; ++k) o[k] += s[t] * orc_read(v_cache, r + k, dtype);
                if (probs && j < max_T) probs[((size_t)b * H_q + h) * max_T + j] = s[t];
            }
            free(keys);
            free(s);
        }
    }
    return status;
}

int orc_decode_gqa(const void *q, const void *k_cache, const void *v_cache,
                   const int32_t *seq_lens, const int32_t *block_table,
                   double *out, double *probs, int max_T, int B, int H_q,
                   int H_kv, int d, int block_size, int max_blocks,
                   double scale, int window, int dtype) {
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || d <= 0 || block_size <= 0 ||
        H_q % H_kv != 0)
        return ORC_BAD_ARG;
    const int group = H_q / H_kv;
    int status = ORC_OK;

#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H_q; ++h) {
            double *o = out + ((size_t)b * H_q + h) * d;
            for (int k = 0; k < d; ++k) o[k] = 0.0;
            int lo, hi;
            orc_visible_range(seq_lens[b], window, &lo, &hi);
            if (probs)
                for (int j = 0; j < max_T; ++j)
                    probs[((size_t)b * H_q + h) * max_T + j] = 0.0;
            if (hi <= lo) continue;
            const int kvh = h / group;
            const int n = hi - lo;
            double *s = (double *)malloc(sizeof(double) * (size_t)n);
            if (!s) {
#pragma omp atomic write
                status = ORC_NO_MEM;
                continue;
            }
            const size_t q_off = ((size_t)b * H_q + h) * d;
            /* scores */
            for (int j = lo; j < hi; ++j) {
                size_t r = orc_row_offset(block_table, max_blocks, b, j,
                                          block_size, H_kv, kvh, d);
                double dot = 0.0;
                for (int k = 0; k < d; ++k)
                    dot += orc_read(q, q_off + k, dtype) *
                           orc_read(k_cache, r + k, dtype);
                s[j - lo] = scale * dot;
            }
            /* softmax along key positions */
            double m = s[0];
            for (int i = 1; i < n; ++i)
                if (s[i] > m) m = s[i];
            double z = 0.0;
            for (int i = 0; i < n; ++i) {
                s[i] = exp(s[i] - m);
                z += s[i];
            }
            for (int i = 0; i < n; ++i) s[i] /= z;
            /* weighted sum of value rows */
            for (int j = lo; j < hi; ++j) {
                size_t r = orc_row_offset(block_table, max_blocks, b, j,
                                          block_size, H_kv, kvh, d);
                double p = s[j - lo];
                for (int k = 0; k < d; ++k)
                    o[k] += p * orc_read(v_cache, r + k, dtype);
                if (probs && j < max_T)
                    probs[((size_t)b * H_q + h) * max_T + j] = p;
            }
            free(s);
        }
    }
    return status;
}

/*
 * MLA decode with both up-projections absorbed ([HEADS] §5.2, §5.3).
 * Each head h of sequence b attends to the shared latent rows of its
 * sequence.  Row j of the latent cache holds c_j (d_c values) followed by
 * the already-rotated shared RoPE key k^R_j (d_r values):
 *
 *   s_j = scale * ( <q_lat[b,h], c_j> + <q_rope[b,h], k^R_j> )
 *   p   = softmax_j(s)            one softmax over the summed scores
 *   z[b,h,:] = sum_j p_j c_j      (d_c wide; the RoPE part only scores)
 *
 * q_lat [B][H][d_c] is the absorbed query q^C (U^K_h)^T, q_rope [B][H][d_r].
 * All keys j < T_b are visible (single-token causal decode, [HEADS] §5.3).
 */
int orc_decode_mla(const void *q_lat, const void *q_rope,
                   const void *latent_cache, const int32_t *seq_lens,
                   const int32_t *block_table, double *out, double *probs,
                   int max_T, int B, int H, int d_c, int d_r, int block_size,
                   int max_blocks, double scale, int dtype) {
    if (B <= 0 || H <= 0 || d_c <= 0 || d_r < 0 || block_size <= 0)
        return ORC_BAD_ARG;
    const int width = d_c + d_r;
    int status = ORC_OK;

#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *z = out + ((size_t)b * H + h) * d_c;
            for (int k = 0; k < d_c; ++k) z[k] = 0.0;
            if (probs)
                for (int j = 0; j < max_T; ++j)
                    probs[((size_t)b * H + h) * max_T + j] = 0.0;
            const int T = seq_lens[b];
            if (T <= 0) continue;
            double *s = (double *)malloc(sizeof(double) * (size_t)T);
            if (!s) {
#pragma omp atomic write
                status = ORC_NO_MEM;
                continue;
            }
            const size_t ql = ((size_t)b * H + h) * d_c;
            const size_t qr = ((size_t)b * H + h) * d_r;
            for (int j = 0; j < T; ++j) {
                size_t r = orc_row_offset(block_table, max_blocks, b, j,
                                          block_size, 1, 0, width);
                double content = 0.0, position = 0.0;
                for (int k = 0; k < d_c; ++k)
                    content += orc_read(q_lat, ql + k, dtype) *
                               orc_read(latent_cache, r + k, dtype);
                for (int k = 0; k < d_r; ++k)
                    position += orc_read(q_rope, qr + k, dtype) *
                                orc_read(latent_cache, r + d_c + k, dtype);
                s[j] = scale * (content + position);
            }
            double m = s[0];
            for (int j = 1; j < T; ++j)
                if (s[j] > m) m = s[j];
            double sum = 0.0;
            for (int j = 0; j < T; ++j) {
                s[j] = exp(s[j] - m);
                sum += s[j];
            }
            for (int j = 0; j < T; ++j) s[j] /= sum;
            for (int j = 0; j < T; ++j) {
                size_t r = orc_row_offset(block_table, max_blocks, b, j,
                                          block_size, 1, 0, width);
                for (int k = 0; k < d_c; ++k)
                    z[k] += s[j] * orc_read(latent_cache, r + k, dtype);
                if (probs && j < max_T)
                    probs[((size_t)b * H + h) * max_T + j] = s[j];
            }
            free(s);
        }
    }
    return status;
}

/*
 * MLA without absorption ([HEADS] §5.1, §5.3): expand every cached latent
 * into per-head keys and values, then run ordinary attention.  Test-only
 * counterpart that the absorbed form must equal (associativity, §5.2).
 *
 *   k_{j,h} = [ c_j U^K_h , k^R_j ]      (d_h + d_r wide)
 *   v_{j,h} =   c_j U^V_h                (d_v wide)
 *   q_h     = [ q^C_h , q^R_h ]
 *   o_h     = sum_j softmax_j(scale * <q_h, k_{j,h}>) v_{j,h}
 *
 * All arrays fp64.  q_c [B][H][d_h], q_rope [B][H][d_r],
 * U_K [H][d_c][d_h], U_V [H][d_c][d_v], out [B][H][d_v].
 */
int orc_mla_explicit(const double *q_c, const double *q_rope,
                     const double *latent_cache, const int32_t *seq_lens,
                     const int32_t *block_table, const double *U_K,
                     const double *U_V, double *out, int B, int H, int d_c,
                     int d_r, int d_h, int d_v, int block_size, int max_blocks,
                     double scale) {
    if (B <= 0 || H <= 0 || d_c <= 0 || d_h <= 0 || d_v <= 0 || d_r < 0)
        return ORC_BAD_ARG;
    const int width = d_c + d_r;
    int status = ORC_OK;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *o = out + ((size_t)b * H + h) * d_v;
            for (int k = 0; k < d_v; ++k) o[k] = 0.0;
            const int T = seq_lens[b];
            if (T <= 0) continue;
            double *s = (double *)malloc(sizeof(double) * (size_t)T);
            double *kc = (double *)malloc(sizeof(double) * (size_t)d_h);
            double *vv = (double *)malloc(sizeof(double) * (size_t)d_v);
            if (!s || !kc || !vv) {
                free(s); free(kc); free(vv);
                status = ORC_NO_MEM;
                continue;
            }
            const double *qc = q_c + ((size_t)b * H + h) * d_h;
            const double *qr = q_rope + ((size_t)b * H + h) * d_r;
            const double *UK = U_K + (size_t)h * d_c * d_h;
            const double *UV = U_V + (size_t)h * d_c * d_v;
            for (int j = 0; j < T; ++j) {
                const double *row = latent_cache +
                    orc_row_offset(block_table, max_blocks, b, j, block_size,
                                   1, 0, width);
                for (int i = 0; i < d_h; ++i) {
                    double acc = 0.0;
                    for (int c = 0; c < d_c; ++c) acc += row[c] * UK[(size_t)c * d_h + i];
                    kc[i] = acc;
                }
                double dot = 0.0;
                for (int i = 0; i < d_h; ++i) dot += qc[i] * kc[i];
                for (int i = 0; i < d_r; ++i) dot += qr[i] * row[d_c + i];
                s[j] = scale * dot;
            }
            double m = s[0];
            for (int j = 1; j < T; ++j)
                if (s[j] > m) m = s[j];
            double sum = 0.0;
            for (int j = 0; j < T; ++j) {
                s[j] = exp(s[j] - m);
                sum += s[j];
            }
            for (int j = 0; j < T; ++j) {
                const double *row = latent_cache +
                    orc_row_offset(block_table, max_blocks, b, j, block_size,
                                   1, 0, width);
                for (int i = 0; i < d_v; ++i) {
                    double acc = 0.0;
                    for (int c = 0; c < d_c; ++c) acc += row[c] * UV[(size_t)c * d_v + i];
                    vv[i] = acc;
                }
                double p = s[j] / sum;
                for (int i = 0; i < d_v; ++i) o[i] += p * vv[i];
            }
            free(s); free(kc); free(vv);
        }
    }
    return status;
}

/*
 * KV-cache size closed forms.
 *   Bytes_KV  = 2 * B * T * H_kv * d * s      ([HEADS] §1 Bytes_KV; factor 2 = K and V)
 *   Bytes_MLA = B * T * (r + d_R) * s         ([HEADS] §5.4; no factor 2)
 */
double orc_bytes_kv(double B, double T, double H_kv, double d, double s) {
    return 2.0 * B * T * H_kv * d * s;
}

double orc_bytes_mla(double B, double T, double r, double d_r, double s) {
    return B * T * (r + d_r) * s;
}

/*
 * Placement of a newly produced token's K/V (or latent row) in the paged
 * cache: position pos of sequence b lands in logical block pos / block_size,
 * slot pos % block_size.  Writes the element offset of that row (for head
 * `head` of a cache with n_heads heads per block) into *offset.
 */
int orc_slot_offset(const int32_t *block_table, int max_blocks, int b, int pos,
                    int block_size, int n_heads, int head, int row_width,
                    int64_t *offset) {
    if (pos < 0 || pos / block_size >= max_blocks) return ORC_BAD_ARG;
    *offset = (int64_t)orc_row_offset(block_table, max_blocks, b, pos,
                                      block_size, n_heads, head, row_width);
    return ORC_OK;
}

/*
 * OCP FP8 E4M3 (the fp8 KV-cache format): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); no
 * infinities; S.1111.111 is NaN; the largest finite magnitude is 448.
 */
double orc_e4m3_value(int code) {
    const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = (e == 0) ? (m / 8.0) * ldexp(1.0, -6)
                              : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -v : v;
}

/* Nearest finite E4M3 code to x, ties to the even code (mantissa bit 0),
 * magnitudes past 448 saturating to 448, the sign kept (so -0 -> 0x80). */
int orc_e4m3_encode(float x) {
    const double a = fabs((double)x);
    int best = 0;
    double best_err = a;                       /* code 0x00 has value 0 */
    for (int c = 1; c <= 0x7E; ++c) {
        const double err = fabs(orc_e4m3_value(c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return signbit(x) ? (best | 0x80) : best;
}

/* Row quantisation of the fp8 cache: amax = max |x| (fp32), scale = amax / 448,
 * codes = e4m3(x * (448 / amax)), all fp32 arithmetic rounded to nearest; a
 * zero row gets scale 0 and zero codes.  x [rows][d] fp32. */
void orc_quantize_rows_e4m3(const float *x, int rows, int d, uint8_t *codes, float *scales) {
    for (int r = 0; r < rows; ++r) {
        const float *xr = x + (size_t)r * d;
        float amax = 0.f;
        for (int i = 0; i < d; ++i) {
            const float v = fabsf(xr[i]);
            if (v > amax) amax = v;
        }
        const float inv = amax > 0.f ? 448.f / amax : 0.f;
        for (int i = 0; i < d; ++i) {
            const float y = xr[i] * inv;
            codes[(size_t)r * d + i] = (uint8_t)orc_e4m3_encode(y);
        }
        scales[r] = amax / 448.f;
    }
}
