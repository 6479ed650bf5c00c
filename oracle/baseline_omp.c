/*
 * baseline_omp.c -- the oracle's decode and chunk attention run over
 * independent (sequence, kv head) units on all host cores, for the timed
 * CPU baseline only.  TEST INFRASTRUCTURE ONLY, like kvq_oracle.c.
 *
 * Nothing here computes attention: every unit is one call of the pinned,
 * scalar oracle_decode_attn / oracle_chunk_attn (kvq_oracle.c) on a view of
 * one sequence and one kv head (its G query heads, its cache rows), so the
 * per-unit arithmetic and its results are exactly the oracle's.  Built with
 * -fopenmp into libkvq_oracle_omp.so together with kvq_oracle.c; the pinned
 * libkvq_oracle.so is built without OpenMP and does not contain this file.
 *
 * A paged arena [num_pages, Hk, page_size, D] is viewed, for kv head hk, as
 * an arena of num_pages * Hk one-head pages in which physical page p of head
 * hk is page p * Hk + hk; unit_tables holds those page ids ([B * Hk,
 * max_pages], -1 kept), written by the caller outside the timed region.
 */
#include <stdint.h>

int oracle_decode_attn(const uint16_t *q, int B, int Hq, int Hk, int D, int group,
                       const uint8_t *k, const uint8_t *v, const float *k_scale,
                       const float *v_scale, int max_seq, int page_size,
                       const int32_t *table, int max_pages, int num_pages,
                       const int32_t *seq_lens, double attn_scale, double *out);
int oracle_chunk_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D, int group,
                      const uint8_t *k, const uint8_t *v, const float *k_scale,
                      const float *v_scale, int max_seq, int page_size,
                      const int32_t *table, int max_pages, int num_pages,
                      const int32_t *seq_lens, double attn_scale, double *out);

/* T = 1 is decode (q [B, Hq, D]); T > 1 a chunk (q [B, Hq, T, D]). */
int oracle_attn_units(const uint16_t *q, int B, int Hq, int Hk, int T, int D, int group,
                      const uint8_t *k, const uint8_t *v, const float *k_scale,
                      const float *v_scale, int max_seq, int page_size,
                      const int32_t *unit_tables, int max_pages, int num_pages,
                      const int32_t *seq_lens, double attn_scale, double *out, int nthreads) {
    const int G = Hq / Hk, ng = D / group;
    const int64_t units = (int64_t)B * Hk;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : err)
    for (int64_t u = 0; u < units; ++u) {
        const int b = (int)(u / Hk), hk = (int)(u % Hk);
        const uint16_t *qu = q + ((int64_t)b * Hq + (int64_t)hk * G) * T * D;
        double *ou = out + ((int64_t)b * Hq + (int64_t)hk * G) * T * D;
        const uint8_t *ku = k, *vu = v;
        const float *ksu = k_scale, *vsu = v_scale;
        const int32_t *tu = 0;
        if (page_size > 0) {
            tu = unit_tables + u * max_pages;
        } else {
            const int64_t row = ((int64_t)b * Hk + hk) * max_seq;
            ku += row * D;
            vu += row * D;
            ksu += row * ng;
            vsu += row * ng;
        }
        const int npg = page_size > 0 ? num_pages * Hk : 0;
        if (T == 1)
            err |= oracle_decode_attn(qu, 1, G, 1, D, group, ku, vu, ksu, vsu, max_seq, page_size,
                                      tu, max_pages, npg, seq_lens + b, attn_scale, ou);
        else
            err |= oracle_chunk_attn(qu, 1, G, 1, T, D, group, ku, vu, ksu, vsu, max_seq,
                                     page_size, tu, max_pages, npg, seq_lens + b, attn_scale, ou);
    }
    return err;
}
