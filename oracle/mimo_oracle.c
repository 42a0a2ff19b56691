/*
 * fp64 CPU oracle for the MiMo-V2-Flash hybrid attention layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do. It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Each function follows the pages' description step by step, in double
 * precision, with plain loops and no blocking, fusion or reordering:
 *
 *   [PR]  "Add Xiaomi MiMo-V2" (huggingface/transformers pull request 45144),
 *         section "Additional useful info" (the bullet list of architecture
 *         facts) and the PR body's "Important points" (sink vs. non-sink
 *         attention paths).
 *   [ISS] "feat(models): add Xiaomi MiMo v2 (mimo_v2_flash) text model
 *         support" (lablup/mlxcel issue 842), sections "Architecture,
 *         verified against upstream", "Architecture notes" and
 *         "Implementation plan".
 *
 * Readings taken where the pages are silent (each is pinned by a test in
 * tests/test_oracle_pins.py):
 *   - RoPE pairs element j with element j + r/2 inside the first r dims
 *     ("half-split", the non-interleaved form), frequency theta^(-2j/r),
 *     rotation (a, b) -> (a cos - b sin, b cos + a sin).
 *   - The sliding window holds W keys including the query itself:
 *     key j is visible from query i when 0 <= i - j < W.
 *   - Query head h reads KV head h / (Hq / Hkv) (contiguous grouping).
 *   - Softmax scale 1/sqrt(qk_dim) unless the caller gives another one.
 *   - The sink is one logit per query head that joins the softmax
 *     denominator only; it is not multiplied by the softmax scale and has
 *     no value vector.
 *   - The V rescale by sqrt(hidden / (heads * v_head_dim)) is a
 *     multiplication of V by that factor.
 *   - Decode: the new token sits at position L-1 where L counts it; a
 *     global cache keeps position p in slot p, a sliding-window ring of W
 *     slots keeps position p in slot p mod W.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>

/* Partial rotary embedding of n vectors (x and y are [n][dim], may alias).
 * [PR, Additional useful info, partial-RoPE bullet]: only the leading third
 * of the head dim rotates; [ISS, Architecture verified against upstream,
 * partial-RoPE item]: the rotated count is the integer part of
 * partial_rotary_factor * head_dim, which the caller passes as rotary_dim.
 * Dims >= rotary_dim are copied unchanged. pos[t] is the position of vector
 * t. [PR, Additional useful info, RoPE-theta bullet]: sliding and global
 * layers use different bases, so theta is the base of the layer at hand.
 * Returns 0, or -1 for an odd rotary_dim or one larger than dim. */
int oracle_rope(const double *x, double *y, int64_t n, int dim,
                int rotary_dim, double theta, const double *pos)
{
    if (rotary_dim < 0 || rotary_dim > dim || (rotary_dim % 2) != 0)
        return -1;
    int half = rotary_dim / 2;
    double *a_saved = (double *)malloc(sizeof(double) * (size_t)(half > 0 ? half : 1));
    double *b_saved = (double *)malloc(sizeof(double) * (size_t)(half > 0 ? half : 1));
    if (a_saved == NULL || b_saved == NULL) {
        free(a_saved);
        free(b_saved);
        return -1;
    }
    for (int64_t t = 0; t < n; ++t) {
        const double *xv = x + t * (int64_t)dim;
        double *yv = y + t * (int64_t)dim;
        for (int j = 0; j < half; ++j) {
            a_saved[j] = xv[j];
            b_saved[j] = xv[j + half];
        }
        for (int d = rotary_dim; d < dim; ++d)
            yv[d] = xv[d];
        for (int j = 0; j < half; ++j) {
            double inv_freq = pow(theta, -2.0 * (double)j / (double)rotary_dim);
            double phi = pos[t] * inv_freq;
            double c = cos(phi);
            double s = sin(phi);
            double a = a_saved[j];
            double b = b_saved[j];
            yv[j] = a * c - b * s;
            yv[j + half] = b * c + a * s;
        }
    }
    free(a_saved);
    free(b_saved);
    return 0;
}

/* First visible key of query index i.
 * [ISS, Architecture verified against upstream, interleave item]: a layer
 * whose hybrid_layer_pattern entry is 1 attends through a sliding window of
 * sliding_window_size keys; the other ("GA", global) layers are plain
 * causal. */
static int64_t first_visible(int64_t i, int layer_type, int64_t window)
{
    if (layer_type == 1) {
        int64_t lo = i - window + 1;
        return lo > 0 ? lo : 0;
    }
    return 0;
}

/* Attention output of one query against an explicit list of visible keys.
 * q: [qk_dim] rotated query; keys[t]/vals[t] point at rotated key / value t.
 * has_sink selects the gpt-oss-style sink logit, which [PR, Additional
 * useful info, sink bullet] puts on sliding-window layers only. v_scale
 * multiplies V: [PR, Additional useful info, V-rescale bullet] names the
 * factor sqrt(hidden_size / (num_attention_heads * v_head_dim)). */
static int attend(const double *q, const double *const *keys,
                  const double *const *vals, int64_t n_keys, int qk_dim,
                  int v_dim, double softmax_scale, int has_sink, double sink,
                  double v_scale, double *out)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
    if (x == NULL)
        return -1;
    /* scores x_t = scale * <q, k_t>, and their maximum (with the sink) */
    double m = -INFINITY;
    for (int64_t t = 0; t < n_keys; ++t) {
        double dot = 0.0;
        for (int d = 0; d < qk_dim; ++d)
            dot += q[d] * keys[t][d];
        x[t] = softmax_scale * dot;
        if (x[t] > m)
            m = x[t];
    }
    if (has_sink && sink > m)
        m = sink;
    /* softmax denominator: every visible key, plus the sink's own term */
    double denom = 0.0;
    for (int64_t t = 0; t < n_keys; ++t)
        denom += exp(x[t] - m);
    if (has_sink)
        denom += exp(sink - m);
    /* weighted sum of the rescaled values; the sink has no value */
    for (int e = 0; e < v_dim; ++e)
        out[e] = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) {
        double p = exp(x[t] - m) / denom;
        for (int e = 0; e < v_dim; ++e)
            out[e] += p * (v_scale * vals[t][e]);
    }
    free(x);
    return 0;
}

/* Prefill output rows for one batch element and one query head.
 * q_rot: [n_rows][qk_dim] rotated queries; rows[r] is the sequence index i
 * of row r. k_rot: [seq][qk_dim] rotated keys of the KV head this query head
 * reads; v: [seq][v_dim]. layer_type: 0 global (causal, no sink), 1 sliding
 * window (window keys including self, sink if has_sink). out: [n_rows][v_dim].
 * Returns 0, or -1 on a bad argument. */
int oracle_prefill_rows(const double *q_rot, const int64_t *rows, int64_t n_rows,
                        const double *k_rot, const double *v, int64_t seq,
                        int qk_dim, int v_dim, int layer_type, int64_t window,
                        double softmax_scale, int has_sink, double sink,
                        double v_scale, double *out)
{
    if (layer_type == 1 && window < 1)
        return -1;
    if (layer_type == 0 && has_sink)
        return -1; /* [PR, sink bullet]: global layers carry no sink */
    const double **keys = (const double **)malloc(sizeof(double *) * (size_t)(seq > 0 ? seq : 1));
    const double **vals = (const double **)malloc(sizeof(double *) * (size_t)(seq > 0 ? seq : 1));
    int rc = (keys == NULL || vals == NULL) ? -1 : 0;
    for (int64_t r = 0; rc == 0 && r < n_rows; ++r) {
        int64_t i = rows[r];
        if (i < 0 || i >= seq) {
            rc = -1;
            break;
        }
        int64_t lo = first_visible(i, layer_type, window);
        int64_t n = 0;
        for (int64_t j = lo; j <= i; ++j) {
            keys[n] = k_rot + j * (int64_t)qk_dim;
            vals[n] = v + j * (int64_t)v_dim;
            ++n;
        }
        rc = attend(q_rot + r * (int64_t)qk_dim, keys, vals, n, qk_dim, v_dim,
                    softmax_scale, has_sink, sink, v_scale, out + r * (int64_t)v_dim);
    }
    free(keys);
    free(vals);
    return rc;
}

/* One decode step for one batch element and one KV head.
 * The new token is at position L-1 (L counts it). Its key is rotated at that
 * position and, with its value, written into the cache: slot L-1 of a global
 * (linear) cache, slot (L-1) mod W of a sliding-window ring
 * ([ISS, Implementation plan]: sliding layers keep a rotating KV cache).
 * Cache entries already there
 * hold rotated keys. Every query head of the group (n_q of them, unrotated,
 * [n_q][qk_dim]) is rotated at position L-1 and attends to the visible
 * positions: 0..L-1 (global) or max(0, L-W)..L-1 (sliding window).
 * k_cache: [cap][qk_dim], v_cache: [cap][v_dim], updated in place.
 * sinks: [n_q] or NULL. out: [n_q][v_dim]. Returns 0 or -1. */
int oracle_decode(const double *q, int n_q, const double *k_new,
                  const double *v_new, double *k_cache, double *v_cache,
                  int64_t cap, int64_t L, int qk_dim, int v_dim, int rotary_dim,
                  double theta, int layer_type, int64_t window,
                  double softmax_scale, const double *sinks, double v_scale,
                  double *out)
{
    if (L < 1)
        return -1;
    if (layer_type == 1) {
        if (window < 1 || cap != window)
            return -1;
    } else {
        if (L > cap || sinks != NULL)
            return -1;
    }
    double pos = (double)(L - 1);
    int64_t slot_new = layer_type == 1 ? (L - 1) % window : L - 1;
    if (oracle_rope(k_new, k_cache + slot_new * (int64_t)qk_dim, 1, qk_dim,
                    rotary_dim, theta, &pos) != 0)
        return -1;
    for (int e = 0; e < v_dim; ++e)
        v_cache[slot_new * (int64_t)v_dim + e] = v_new[e];

    int64_t lo = first_visible(L - 1, layer_type, window);
    int64_t n = L - lo;
    const double **keys = (const double **)malloc(sizeof(double *) * (size_t)n);
    const double **vals = (const double **)malloc(sizeof(double *) * (size_t)n);
    double *q_rot = (double *)malloc(sizeof(double) * (size_t)qk_dim);
    int rc = (keys == NULL || vals == NULL || q_rot == NULL) ? -1 : 0;
    for (int64_t p = lo; rc == 0 && p <= L - 1; ++p) {
        int64_t slot = layer_type == 1 ? p % window : p;
        keys[p - lo] = k_cache + slot * (int64_t)qk_dim;
        vals[p - lo] = v_cache + slot * (int64_t)v_dim;
    }
    for (int h = 0; rc == 0 && h < n_q; ++h) {
        rc = oracle_rope(q + (int64_t)h * qk_dim, q_rot, 1, qk_dim, rotary_dim,
                         theta, &pos);
        if (rc == 0)
            rc = attend(q_rot, keys, vals, n, qk_dim, v_dim, softmax_scale,
                        sinks != NULL, sinks != NULL ? sinks[h] : 0.0, v_scale,
                        out + (int64_t)h * v_dim);
    }
    free(keys);
    free(vals);
    free(q_rot);
    return rc;
}
