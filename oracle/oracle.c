/*
 * Plain fp64 CPU oracle for fused multi-head attention with GQA and for
 * split-KV single-token decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the test suite, the smoke check of the entry module and
 * the CPU-baseline leg of the benchmark use it.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * What it computes, and where each piece is defined:
 *
 *   - Tylo.jl "Primitives" page, entry `attention!`: O = softmax(Q K^T scale +
 *     mask) V per (batch, query head), with GQA (Heads a multiple of
 *     Heads_KV, entry `flex_attention!`), `input_pos` = absolute position of
 *     the first query, `k_lengths`/`q_lengths` = per-batch valid lengths, and
 *     the softmax statistics M/L saved for the backward.  We export them as
 *     one number per row, LSE = M + ln L (natural log of the scaled scores).
 *   - mlx-arsenal "Attention" page, entries `causal_mask` and
 *     `sliding_window_mask`: additive masks of shape (1, 1, S, offset + S)
 *     whose masked entries are -inf; the sliding window lets a query see at
 *     most `window_size` previous positions, itself included.
 *   - Tylo.jl "Primitives" page, entry `CausalMask`: a query sees keys at or
 *     before its own position, positions being absolute (input_pos shifts the
 *     queries).
 *   - Tylo.jl "Primitives" page, entry `flex_attention!` with the score mods
 *     `SoftCapScore(cap)` (s -> cap * tanh(s / cap)) and `AliBiScore(slopes)`
 *     (adds slopes[h] * (q - kv), absolute positions) and the mask mod
 *     `DocumentMask(doc_q, doc_kv)` (a pair attends iff the document ids of
 *     the query and the key match), combined with the masks above.  The
 *     precomputed `BlockMask` only tells a kernel which tiles to skip; when it
 *     agrees with the mask mod (as the page requires) it changes nothing in
 *     the result, so the oracle ignores it.
 *   - vllm-mlx "attention" page, `MLXAttentionBackend.get_kv_cache_shape` and
 *     `MLXAttentionMetadata` (seq_lens, block_tables): a paged KV cache of
 *     shape (num_blocks, block_size, num_kv_heads, head_size); token j of
 *     sequence b sits in block block_tables[b][j / block_size], slot
 *     j % block_size.  Decoding from it is decode_attention! over the tokens
 *     the block table gathers.
 *   - mlx-arsenal "Radius-bounded block scores (RBS)" page: block centroids and
 *     radii, the base and rescue log block scores per (query block, key block),
 *     `relative_block_mask` and the recipe's union with a diagonal band; the
 *     block-sparse attention that follows is `flex_attention!` with those
 *     64x64 blocks masked.
 *   - Tylo.jl "Primitives" page, entry `∇attention!`: the input gradients of
 *     attention! from the output gradient: with P the softmax probabilities,
 *     dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dP * P)), dQ = scale dS K,
 *     dK = scale dS^T Q (GQA: a KV head collects the gradients of all the query
 *     heads it serves).  The oracle recomputes P from its definition; the GPU
 *     uses the saved LSE, which gives the same P up to rounding.
 *   - Tylo.jl "Primitives" page, entry `decode_attention!`: one query vector
 *     per head and sequence against the first lengths[b] cached keys.  The
 *     split into n_splits slices and their combine change only the rounding,
 *     so the oracle computes the plain softmax over all valid keys.  Its scale
 *     is the page's default qk_scale = 1/sqrt(Dk) (entry `flex_attention!`).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes with its reason):
 *   - GQA head map: query head h reads KV head h / (Hq / Hkv).
 *   - valid lengths are prefixes: key j is valid iff j < k_lengths[b], query
 *     row i is valid iff i < q_lengths[b].
 *   - window w > 0 (always causal): key j is visible from absolute query
 *     position p iff p - w < j <= p, i.e. at most w keys, itself included.
 *   - a row with no visible key (invalid row, empty length, or every key cut)
 *     has O = 0 and LSE = -inf.
 *   - score mods act on the scaled score s = scale * <q, k>; at most one of
 *     them per call (the page composes mods with ComposeScore, whose order a
 *     caller would fix; no such composition is built).  The ALiBi distance
 *     is (input_pos + i) - j, the absolute query position minus the key
 *     position, with the sign the page gives.
 *   - RBS quantiles (median, 90th percentile) interpolate linearly between the
 *     sorted radii (numpy's default); short last blocks average and score the
 *     tokens they have.
 *   - document ids: doc_q[i] belongs to local query row i (absolute position
 *     input_pos + i), doc_kv[j] to key j; both are shared by every batch
 *     entry and head.
 *
 * Precision: inputs are doubles (the harness widens the exact bf16 values),
 * every product, sum, exp and log is done in double.
 *
 * Layouts (row-major, C order):
 *   Q (B, Hq, n_rows, D)    -- n_rows query rows whose absolute row indices
 *                              within 0..Sq-1 are rows[0..n_rows-1] (NULL:
 *                              all Sq rows in order, n_rows == Sq)
 *   K, V (B, Hkv, Sk, D)
 *   O (B, Hq, n_rows, D), LSE (B, Hq, n_rows)
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of OpenMP threads an oracle call will use. */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * mlx-arsenal "Attention" page, `causal_mask(seq_len, offset)`: the
 * lower-triangular additive mask of shape (1, 1, seq_len, offset + seq_len);
 * query row i (at position offset + i in a KV cache of offset + seq_len
 * entries) sees keys 0..offset + i.  `out` holds seq_len * (offset + seq_len)
 * doubles, each 0.0 or -inf.
 */
void oracle_causal_mask(double *out, int seq_len, int offset) {
    const long n_kv = (long)offset + seq_len;
    for (long i = 0; i < seq_len; ++i)
        for (long j = 0; j < n_kv; ++j)
            out[i * n_kv + j] = (j <= offset + i) ? 0.0 : -INFINITY;
}

/*
 * mlx-arsenal "Attention" page, `sliding_window_mask(seq_len, window_size,
 * offset)`: causal, and each position sees at most window_size previous
 * positions including itself, i.e. keys offset+i-window_size+1 .. offset+i.
 * Same shape and values as the causal mask.
 */
void oracle_sliding_window_mask(double *out, int seq_len, int window_size, int offset) {
    const long n_kv = (long)offset + seq_len;
    for (long i = 0; i < seq_len; ++i) {
        const long pos = (long)offset + i;
        for (long j = 0; j < n_kv; ++j) {
            const int visible = (j <= pos) && (j > pos - window_size);
            out[i * n_kv + j] = visible ? 0.0 : -INFINITY;
        }
    }
}

/*
 * Additive mask row for absolute query row i of batch b: 0.0 where key j is
 * visible, -inf elsewhere.  Combines the causal rule (Tylo `CausalMask`,
 * absolute positions), the sliding window (mlx-arsenal
 * `sliding_window_mask`), and the per-batch valid lengths of `attention!`.
 */
static void mask_row(double *m, long i, int Sk, int causal, int window, int input_pos,
                     int k_len, int q_len) {
    const long pos = (long)input_pos + i;
    for (long j = 0; j < Sk; ++j) {
        int visible = (i < q_len) && (j < k_len);
        if (causal && j > pos) visible = 0;
        if (window > 0 && j <= pos - window) visible = 0;
        m[j] = visible ? 0.0 : -INFINITY;
    }
}

/*
 * Which keys each requested query row of `attention!` sees: out (B, n_rows, Sk)
 * uint8 holds 1 where the additive mask of oracle_attn_fwd's score row is 0.0
 * and 0 where it is -inf -- the same mask_row, so the visible set is exactly the
 * one whose keys oracle_attn_fwd weighs.  The mask does not depend on the head.
 * Rows as in oracle_attn_fwd (rows == NULL: all Sq rows).  With Sq = 1,
 * causal = 0 and k_lengths = the decode lengths it is the key set of
 * `decode_attention!` (the first lengths[b] cached keys).
 * Returns 0, or -1 on bad arguments.
 */
int oracle_attn_visible(unsigned char *out, int B, int Sq, int Sk, int causal, int window,
                        int input_pos, const int *k_lengths, const int *q_lengths,
                        const int *rows, int n_rows) {
    if (B < 0 || Sq < 0 || Sk < 0) return -1;
    if (window > 0 && !causal) return -1;
    if (rows == NULL) n_rows = Sq;
    const long total = (long)B * n_rows;
    int bad = 0;
#pragma omp parallel
    {
        double *mask = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        if (mask == NULL) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(static)
        for (long t = 0; t < total; ++t) {
            if (mask == NULL) continue;
            const long r = t % n_rows;
            const long b = t / n_rows;
            const long i = rows ? rows[r] : r;
            const int k_len = k_lengths ? k_lengths[b] : Sk;
            const int q_len = q_lengths ? q_lengths[b] : Sq;
            mask_row(mask, i, Sk, causal, window, input_pos, k_len, q_len);
            unsigned char *o = out + t * (long)Sk;
            for (long j = 0; j < Sk; ++j) o[j] = (mask[j] == 0.0) ? 1 : 0;
        }
        free(mask);
    }
    return bad ? -1 : 0;
}

/*
 * Tylo.jl "Primitives" page, `attention!` (+ GQA rule of `flex_attention!`).
 * For every batch b, query head hq and requested query row:
 *   s_j   = scale * <Q_i, K_j> + mask_j          (explicit score row)
 *   M     = max_j s_j,  L = sum_j exp(s_j - M)   (softmax statistics)
 *   O_i   = sum_j (exp(s_j - M) / L) V_j
 *   LSE_i = M + ln L
 * Returns 0, or -1 on bad arguments.
 */
int oracle_attn_fwd(double *O, double *LSE, const double *Q, const double *K, const double *V,
                    int B, int Hq, int Hkv, int Sq, int Sk, int D, double scale,
                    int causal, int window, int input_pos,
                    const int *k_lengths, const int *q_lengths,
                    const int *rows, int n_rows) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Sk < 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (window > 0 && !causal) return -1;
    if (rows == NULL) n_rows = Sq;
    const int group = Hq / Hkv;
    const long total = (long)B * Hq * n_rows;
    int bad = 0;

#pragma omp parallel
    {
        double *score = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        double *mask = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        if (score == NULL || mask == NULL) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (long t = 0; t < total; ++t) {
            if (score == NULL || mask == NULL) continue;
            const long r = t % n_rows;
            const long hq = (t / n_rows) % Hq;
            const long b = t / ((long)n_rows * Hq);
            const long i = rows ? rows[r] : r;
            const long hkv = hq / group;
            const int k_len = k_lengths ? k_lengths[b] : Sk;
            const int q_len = q_lengths ? q_lengths[b] : Sq;

            const double *q = Q + ((b * Hq + hq) * (long)n_rows + r) * D;
            const double *Kb = K + (b * Hkv + hkv) * (long)Sk * D;
            const double *Vb = V + (b * Hkv + hkv) * (long)Sk * D;
            double *o = O + ((b * Hq + hq) * (long)n_rows + r) * D;

            mask_row(mask, i, Sk, causal, window, input_pos, k_len, q_len);
            double mx = -INFINITY;
            for (long j = 0; j < Sk; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += q[d] * Kb[j * D + d];
                score[j] = scale * dot + mask[j];
                if (score[j] > mx) mx = score[j];
            }
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (mx == -INFINITY) {
                if (LSE) LSE[(b * Hq + hq) * (long)n_rows + r] = -INFINITY;
                continue;
            }
            double l = 0.0;
            for (long j = 0; j < Sk; ++j) {
                score[j] = exp(score[j] - mx);
                l += score[j];
            }
            for (long j = 0; j < Sk; ++j) {
                const double p = score[j] / l;
                if (p == 0.0) continue;
                for (int d = 0; d < D; ++d) o[d] += p * Vb[j * D + d];
            }
            if (LSE) LSE[(b * Hq + hq) * (long)n_rows + r] = mx + log(l);
        }
        free(score);
        free(mask);
    }
    return bad ? -1 : 0;
}

/*
 * Tylo.jl "Primitives" page, `flex_attention!`: the `attention!` rows above
 * with a score mod and a document mask.  For each requested row, every key j:
 *   s_j = scale * <Q_i, K_j>
 *   if softcap > 0:        s_j = softcap * tanh(s_j / softcap)   (SoftCapScore)
 *   else if alibi_slopes:  s_j += alibi_slopes[hq] * ((input_pos + i) - j)
 *                                                                (AliBiScore)
 *   visible_j = the causal / window / length rule of mask_row, and, if doc_q
 *               and doc_kv are given, doc_q[i] == doc_kv[j]       (DocumentMask)
 *               and, if block_keep is given, the 64x64 block of (i, j) is kept
 *               (block-sparse attention from a block mask per batch entry and head)
 *   then the softmax, O and LSE exactly as in oracle_attn_fwd.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_flex_fwd(double *O, double *LSE, const double *Q, const double *K, const double *V,
                    int B, int Hq, int Hkv, int Sq, int Sk, int D, double scale,
                    int causal, int window, int input_pos,
                    const int *k_lengths, const int *q_lengths,
                    const int *rows, int n_rows,
                    double softcap, const double *alibi_slopes,
                    const int *doc_q, const int *doc_kv,
                    const unsigned char *block_keep) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Sk < 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (window > 0 && !causal) return -1;
    if (softcap < 0.0) return -1;
    if (softcap > 0.0 && alibi_slopes != NULL) return -1; /* composition order not fixed */
    if ((doc_q == NULL) != (doc_kv == NULL)) return -1;
    if (rows == NULL) n_rows = Sq;
    const int group = Hq / Hkv;
    const long total = (long)B * Hq * n_rows;
    int bad = 0;

#pragma omp parallel
    {
        double *score = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        double *mask = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        if (score == NULL || mask == NULL) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (long t = 0; t < total; ++t) {
            if (score == NULL || mask == NULL) continue;
            const long r = t % n_rows;
            const long hq = (t / n_rows) % Hq;
            const long b = t / ((long)n_rows * Hq);
            const long i = rows ? rows[r] : r;
            const long kv_head = hq / group;
            const long row_id = (b * Hq + hq) * (long)n_rows + r;
            const int k_len = k_lengths ? k_lengths[b] : Sk;
            const int q_len = q_lengths ? q_lengths[b] : Sq;
            const double q_pos = (double)((long)input_pos + i);

            const double *q = Q + row_id * D;
            const double *Kb = K + (b * Hkv + kv_head) * (long)Sk * D;
            const double *Vb = V + (b * Hkv + kv_head) * (long)Sk * D;
            double *o = O + row_id * D;

            mask_row(mask, i, Sk, causal, window, input_pos, k_len, q_len);
            if (doc_q != NULL)
                for (long j = 0; j < Sk; ++j)
                    if (doc_q[i] != doc_kv[j]) mask[j] = -INFINITY;
            if (block_keep != NULL) {
                /* block-sparse attention: (B, Hq, ceil(Sq/64), ceil(Sk/64)) keep flags */
                const long nqb = (Sq + 63) / 64, nkb = (Sk + 63) / 64;
                const unsigned char *kr = block_keep + ((b * Hq + hq) * nqb + i / 64) * nkb;
                for (long j = 0; j < Sk; ++j)
                    if (!kr[j / 64]) mask[j] = -INFINITY;
            }
            double mx = -INFINITY;
            for (long j = 0; j < Sk; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += q[d] * Kb[j * D + d];
                double sj = scale * dot;
                if (softcap > 0.0) sj = softcap * tanh(sj / softcap);
                if (alibi_slopes != NULL) sj += alibi_slopes[hq] * (q_pos - (double)j);
                score[j] = sj + mask[j];
                if (score[j] > mx) mx = score[j];
            }
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (mx == -INFINITY) {
                if (LSE) LSE[row_id] = -INFINITY;
                continue;
            }
            double lsum = 0.0;
            for (long j = 0; j < Sk; ++j) {
                score[j] = exp(score[j] - mx);
                lsum += score[j];
            }
            for (long j = 0; j < Sk; ++j) {
                const double pj = score[j] / lsum;
                if (pj == 0.0) continue;
                for (int d = 0; d < D; ++d) o[d] += pj * Vb[j * D + d];
            }
            if (LSE) LSE[row_id] = mx + log(lsum);
        }
        free(score);
        free(mask);
    }
    return bad ? -1 : 0;
}

/*
 * Tylo.jl "Primitives" page, `decode_attention!`: one query per (sequence b,
 * query head hq) attends to cached keys 0..lengths[b]-1 of KV head
 * hq / (Hq / Hkv), with scale 1/sqrt(D).
 *   Q (B, Hq, D); K, V (B, Hkv, S_cap, D); O (B, Hq, D); LSE (B, Hq) or NULL.
 * A sequence with lengths[b] == 0 yields O = 0 and LSE = -inf.
 * Returns 0, or -1 on bad arguments (including a length above S_cap).
 */
int oracle_decode(double *O, double *LSE, const double *Q, const double *K, const double *V,
                  int B, int Hq, int Hkv, int S_cap, int D, const int *lengths) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || S_cap < 0 || D <= 0 || lengths == NULL) return -1;
    if (Hq % Hkv != 0) return -1;
    for (int b = 0; b < B; ++b)
        if (lengths[b] < 0 || lengths[b] > S_cap) return -1;
    const int group = Hq / Hkv;
    const double scale = 1.0 / sqrt((double)D);
    const long total = (long)B * Hq;
    int bad = 0;

#pragma omp parallel
    {
        double *score = (double *)malloc(sizeof(double) * (S_cap > 0 ? S_cap : 1));
        if (score == NULL) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long t = 0; t < total; ++t) {
            if (score == NULL) continue;
            const long hq = t % Hq;
            const long b = t / Hq;
            const long hkv = hq / group;
            const int len = lengths[b];
            const double *q = Q + (b * Hq + hq) * (long)D;
            const double *Kb = K + (b * Hkv + hkv) * (long)S_cap * D;
            const double *Vb = V + (b * Hkv + hkv) * (long)S_cap * D;
            double *o = O + (b * Hq + hq) * (long)D;

            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (len == 0) {
                if (LSE) LSE[b * Hq + hq] = -INFINITY;
                continue;
            }
            double mx = -INFINITY;
            for (long j = 0; j < len; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += q[d] * Kb[j * D + d];
                score[j] = scale * dot;
                if (score[j] > mx) mx = score[j];
            }
            double l = 0.0;
            for (long j = 0; j < len; ++j) {
                score[j] = exp(score[j] - mx);
                l += score[j];
            }
            for (long j = 0; j < len; ++j) {
                const double p = score[j] / l;
                for (int d = 0; d < D; ++d) o[d] += p * Vb[j * D + d];
            }
            if (LSE) LSE[b * Hq + hq] = mx + log(l);
        }
        free(score);
    }
    return bad ? -1 : 0;
}

/*
 * Paged decode (vllm-mlx "attention" page: KV cache shape (num_blocks,
 * block_size, num_kv_heads, head_size), metadata seq_lens and block_tables)
 * with the decode_attention! definition above: for sequence b and query head
 * hq, key j < seq_lens[b] is row block_tables[b * max_blocks + j / block_size],
 * slot j % block_size, KV head hq / (Hq / Hkv) of the cache; scale 1/sqrt(D).
 *   Q (B, Hq, D); K_cache, V_cache (num_blocks, block_size, Hkv, D);
 *   block_tables (B, max_blocks); O (B, Hq, D); LSE (B, Hq) or NULL.
 * Returns 0, or -1 on bad arguments (a length above max_blocks * block_size or
 * a referenced block outside 0 .. num_blocks-1).
 */
int oracle_decode_paged(double *O, double *LSE, const double *Q, const double *K_cache,
                        const double *V_cache, const int *block_tables, const int *seq_lens,
                        int B, int Hq, int Hkv, int num_blocks, int block_size, int max_blocks,
                        int D) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || num_blocks < 0 || block_size <= 0 || max_blocks < 0 ||
        D <= 0 || seq_lens == NULL || (B > 0 && block_tables == NULL))
        return -1;
    if (Hq % Hkv != 0) return -1;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || (long)seq_lens[b] > (long)max_blocks * block_size) return -1;
        for (long j = 0; j < seq_lens[b]; j += block_size) {
            const int blk = block_tables[(long)b * max_blocks + j / block_size];
            if (blk < 0 || blk >= num_blocks) return -1;
        }
    }
    const int group = Hq / Hkv;
    const double qk_scale = 1.0 / sqrt((double)D);
    const long total = (long)B * Hq;
    int bad = 0;

#pragma omp parallel
    {
        long cap = (long)max_blocks * block_size;
        double *score = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
        if (score == NULL) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long t = 0; t < total; ++t) {
            if (score == NULL) continue;
            const long hq = t % Hq;
            const long b = t / Hq;
            const long kvh = hq / group;
            const int n = seq_lens[b];
            const double *q = Q + (b * Hq + hq) * (long)D;
            double *o = O + (b * Hq + hq) * (long)D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (n == 0) {
                if (LSE) LSE[b * Hq + hq] = -INFINITY;
                continue;
            }
            double mx = -INFINITY;
            for (long j = 0; j < n; ++j) {
                const long blk = block_tables[b * max_blocks + j / block_size];
                const double *kr = K_cache + ((blk * block_size + j % block_size) * Hkv + kvh) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += q[d] * kr[d];
                score[j] = qk_scale * dot;
                if (score[j] > mx) mx = score[j];
            }
            double den = 0.0;
            for (long j = 0; j < n; ++j) {
                score[j] = exp(score[j] - mx);
                den += score[j];
            }
            for (long j = 0; j < n; ++j) {
                const long blk = block_tables[b * max_blocks + j / block_size];
                const double *vr = V_cache + ((blk * block_size + j % block_size) * Hkv + kvh) * D;
                const double w = score[j] / den;
                for (int d = 0; d < D; ++d) o[d] += w * vr[d];
            }
            if (LSE) LSE[b * Hq + hq] = mx + log(den);
        }
        free(score);
    }
    return bad ? -1 : 0;
}

/*
 * mlx-arsenal "Radius-bounded block scores (RBS)" page (sections "The idea" and
 * "What mlx-arsenal ships"): block scores of block-sparse prefill.  For KV head
 * h of batch b, key block kb (64 keys, the last one possibly shorter):
 *   centroid c = mean of its keys, radius r = max over its keys of |k - c|_2;
 *   r_low, r_high = median and 90th percentile of the head's block radii
 *                   (linear interpolation between order statistics);
 *   beta = clip((r - r_low) / (r_high - r_low), 0, 1), or, when r_high ==
 *          r_low, 1 for r > r_low and 0 otherwise.
 * For query head hq (KV head hq / (Hq/Hkv)) and query token t:
 *   l_base   = <q_t, c> / sqrt(D)
 *   l_rescue = (<q_t, c> + |q_t|_2 * r * beta) / sqrt(D)
 * and the block scores are log sum_t exp(l) over the tokens t of query block qb.
 *   Q (B, Hq, Sq, D); K (B, Hkv, Sk, D); base, rescue (B, Hq, nqb, nkb).
 * Returns 0, or -1 on bad arguments.
 */
static int cmp_double(const void *a, const void *b) {
    const double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

static double sorted_quantile(const double *v, int n, double q) {
    const double pos = q * (n - 1);
    const int lo = (int)floor(pos);
    const int hi = lo + 1 < n ? lo + 1 : lo;
    return v[lo] + (pos - lo) * (v[hi] - v[lo]);
}

int oracle_rbs_block_scores(double *base, double *rescue, const double *Q, const double *K,
                            int B, int Hq, int Hkv, int Sq, int Sk, int D) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Sk <= 0 || D <= 0 || Hq % Hkv != 0) return -1;
    const int BS = 64;
    const int nqb = (Sq + BS - 1) / BS, nkb = (Sk + BS - 1) / BS;
    const int group = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double *cent = (double *)malloc(sizeof(double) * (size_t)B * Hkv * nkb * D);
    double *rad = (double *)malloc(sizeof(double) * (size_t)B * Hkv * nkb);
    double *beta = (double *)malloc(sizeof(double) * (size_t)B * Hkv * nkb);
    if (!cent || !rad || !beta) {
        free(cent); free(rad); free(beta);
        return -1;
    }
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * Hkv; ++bh) {
        const double *Kh = K + bh * (long)Sk * D;
        for (int kb = 0; kb < nkb; ++kb) {
            const int j0 = kb * BS, j1 = (j0 + BS < Sk) ? j0 + BS : Sk;
            double *c = cent + (bh * nkb + kb) * (long)D;
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int j = j0; j < j1; ++j) acc += Kh[(long)j * D + d];
                c[d] = acc / (j1 - j0);
            }
            double rmax = 0.0;
            for (int j = j0; j < j1; ++j) {
                double ss = 0.0;
                for (int d = 0; d < D; ++d) {
                    const double e = Kh[(long)j * D + d] - c[d];
                    ss += e * e;
                }
                if (sqrt(ss) > rmax) rmax = sqrt(ss);
            }
            rad[bh * nkb + kb] = rmax;
        }
        double *sorted = (double *)malloc(sizeof(double) * nkb);
        if (!sorted) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        memcpy(sorted, rad + bh * nkb, sizeof(double) * nkb);
        qsort(sorted, nkb, sizeof(double), cmp_double);
        const double r_low = sorted_quantile(sorted, nkb, 0.5);
        const double r_high = sorted_quantile(sorted, nkb, 0.9);
        free(sorted);
        for (int kb = 0; kb < nkb; ++kb) {
            const double r = rad[bh * nkb + kb];
            double bt;
            if (r_high > r_low) {
                bt = (r - r_low) / (r_high - r_low);
                bt = bt < 0.0 ? 0.0 : (bt > 1.0 ? 1.0 : bt);
            } else {
                bt = r > r_low ? 1.0 : 0.0;
            }
            beta[bh * nkb + kb] = bt;
        }
    }
    if (!bad) {
#pragma omp parallel for schedule(dynamic, 1)
        for (long t = 0; t < (long)B * Hq * nqb; ++t) {
            const long qb = t % nqb, hq = (t / nqb) % Hq, b = t / ((long)nqb * Hq);
            const long bh = b * Hkv + hq / group;
            const int i0 = (int)qb * BS, i1 = (i0 + BS < Sq) ? i0 + BS : Sq;
            for (int kb = 0; kb < nkb; ++kb) {
                const double *c = cent + (bh * nkb + kb) * (long)D;
                const double rb = rad[bh * nkb + kb] * beta[bh * nkb + kb];
                double mb = -INFINITY, mr = -INFINITY;
                double lb[64], lr[64];
                for (int i = i0; i < i1; ++i) {
                    const double *q = Q + ((b * Hq + hq) * (long)Sq + i) * D;
                    double dot = 0.0, qq = 0.0;
                    for (int d = 0; d < D; ++d) {
                        dot += q[d] * c[d];
                        qq += q[d] * q[d];
                    }
                    lb[i - i0] = dot * inv_sqrt_d;
                    lr[i - i0] = (dot + sqrt(qq) * rb) * inv_sqrt_d;
                    if (lb[i - i0] > mb) mb = lb[i - i0];
                    if (lr[i - i0] > mr) mr = lr[i - i0];
                }
                double sb = 0.0, sr = 0.0;
                for (int i = 0; i < i1 - i0; ++i) {
                    sb += exp(lb[i] - mb);
                    sr += exp(lr[i] - mr);
                }
                base[t * nkb + kb] = mb + log(sb);
                rescue[t * nkb + kb] = mr + log(sr);
            }
        }
    }
    free(cent); free(rad); free(beta);
    return bad ? -1 : 0;
}

/*
 * mlx-arsenal RBS page, `relative_block_mask(log_scores, alpha)` and the recipe
 * `rbs_block_mask`: a block is kept when its summed exp over the query block
 * is at least alpha times the row maximum, i.e. log_score >= max_row + ln alpha;
 * the final mask is the union of the base branch (alpha_base), the rescue branch
 * (alpha_rescue) and the band |qb - kb| < diagonal.  keep: 1 / 0 per block,
 * rows = B * Hq * nqb rows of nkb blocks.
 */
int oracle_rbs_block_mask(unsigned char *keep, const double *base, const double *rescue,
                          long rows, int nqb, int nkb, double alpha_base, double alpha_rescue,
                          int diagonal) {
    if (rows < 0 || nqb <= 0 || nkb <= 0 || !(alpha_base > 0.0) || !(alpha_rescue > 0.0)) return -1;
    for (long r = 0; r < rows; ++r) {
        const double *sb = base + r * nkb, *sr = rescue + r * nkb;
        double mb = -INFINITY, mr = -INFINITY;
        for (int k = 0; k < nkb; ++k) {
            if (sb[k] > mb) mb = sb[k];
            if (sr[k] > mr) mr = sr[k];
        }
        const long qb = r % nqb;
        for (int k = 0; k < nkb; ++k) {
            const int band = (qb - k < diagonal) && (k - qb < diagonal);
            keep[r * nkb + k] = (sb[k] >= mb + log(alpha_base)) ||
                                (sr[k] >= mr + log(alpha_rescue)) || band;
        }
    }
    return 0;
}

/*
 * Tylo.jl "Primitives" page, `∇attention!`: gradients of the attention! rows
 * defined above (same masks and lengths) for the output gradient dO.
 *   per (b, hq, row i):  P_i = softmax(S_i + mask_i)      (explicit row)
 *                        dP_ij = <dO_i, V_j>
 *                        delta_i = sum_j P_ij dP_ij
 *                        dS_ij = P_ij (dP_ij - delta_i)
 *                        dQ_i  = scale sum_j dS_ij K_j
 *                        dK_j += scale dS_ij Q_i,  dV_j += P_ij dO_i
 * dK, dV accumulate over the query heads of a KV head.  Rows without a visible
 * key contribute nothing (their dQ row is 0).  All arrays row-major; dQ like Q,
 * dK / dV like K.  Returns 0, or -1 on bad arguments.
 */
int oracle_attn_bwd(double *dQ, double *dK, double *dV, const double *Q, const double *K,
                    const double *V, const double *dO, int B, int Hq, int Hkv, int Sq, int Sk,
                    int D, double scale, int causal, int window, int input_pos,
                    const int *k_lengths, const int *q_lengths) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Sk < 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (window > 0 && !causal) return -1;
    const int group = Hq / Hkv;
    memset(dQ, 0, sizeof(double) * (size_t)B * Hq * Sq * D);
    memset(dK, 0, sizeof(double) * (size_t)B * Hkv * Sk * D);
    memset(dV, 0, sizeof(double) * (size_t)B * Hkv * Sk * D);
    int bad = 0;
    /* one (b, KV head) per task: its dK / dV rows are written by this task only */
#pragma omp parallel
    {
        double *prob = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        double *mrow = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        double *dpr = (double *)malloc(sizeof(double) * (Sk > 0 ? Sk : 1));
        if (!prob || !mrow || !dpr) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < (long)B * Hkv; ++bh) {
            if (!prob || !mrow || !dpr) continue;
            const long b = bh / Hkv, hkv = bh % Hkv;
            const int k_len = k_lengths ? k_lengths[b] : Sk;
            const int q_len = q_lengths ? q_lengths[b] : Sq;
            const double *Kh = K + bh * (long)Sk * D, *Vh = V + bh * (long)Sk * D;
            double *dKh = dK + bh * (long)Sk * D, *dVh = dV + bh * (long)Sk * D;
            for (long hq = hkv * group; hq < (hkv + 1) * group; ++hq) {
                for (long i = 0; i < Sq; ++i) {
                    const double *q = Q + ((b * Hq + hq) * (long)Sq + i) * D;
                    const double *go = dO + ((b * Hq + hq) * (long)Sq + i) * D;
                    double *gq = dQ + ((b * Hq + hq) * (long)Sq + i) * D;
                    mask_row(mrow, i, Sk, causal, window, input_pos, k_len, q_len);
                    double mx = -INFINITY;
                    for (long j = 0; j < Sk; ++j) {
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d) dot += q[d] * Kh[j * D + d];
                        prob[j] = scale * dot + mrow[j];
                        if (prob[j] > mx) mx = prob[j];
                    }
                    if (mx == -INFINITY) continue;
                    double l = 0.0;
                    for (long j = 0; j < Sk; ++j) {
                        prob[j] = exp(prob[j] - mx);
                        l += prob[j];
                    }
                    double delta = 0.0;
                    for (long j = 0; j < Sk; ++j) {
                        prob[j] /= l;
                        double dp = 0.0;
                        for (int d = 0; d < D; ++d) dp += go[d] * Vh[j * D + d];
                        dpr[j] = dp;
                        delta += prob[j] * dp;
                    }
                    for (long j = 0; j < Sk; ++j) {
                        if (prob[j] == 0.0) continue;
                        const double ds = prob[j] * (dpr[j] - delta);
                        for (int d = 0; d < D; ++d) {
                            gq[d] += scale * ds * Kh[j * D + d];
                            dKh[j * D + d] += scale * ds * q[d];
                            dVh[j * D + d] += prob[j] * go[d];
                        }
                    }
                }
            }
        }
        free(prob);
        free(mrow);
        free(dpr);
    }
    return bad ? -1 : 0;
}
