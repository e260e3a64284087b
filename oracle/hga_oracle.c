/*
 * Plain fp64 CPU oracle for the HGA per-segment attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; it shares no code, header, table or helper with the CUDA
 * path.  Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load it.
 *
 * Source of the method: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global
 * Attention and Segmented Backpropagation in Practice" (sns.style article; the
 * ja/de/ko editions carry the same text, the fr edition a rewrite):
 *   - Background (背景と概要 / Hintergrund / 배경): the sequence is split into
 *     segments; only the active segment is differentiable; history KV is
 *     detached and offloaded; each query block attends to a bounded, exact set
 *     of historical tokens instead of the dense history.
 *   - Deep analysis (深掘り分析 / Tiefenanalyse / 심층 분석): per-block summaries
 *     stay resident in VRAM.
 *   - fr edition, Contexte / Analyse approfondie: targeted loading of precise
 *     historical tokens per query block; the history is decoupled from the
 *     active graph.
 * The article does not say how a block summary is formed, how blocks are
 * scored, or how many are kept.  This oracle fixes the plainest reading that
 * the rest supports:
 *   summary  = mean of the block's keys, per KV head;
 *   score    = (mean of the query block's queries) . summary / sqrt(d),
 *              max over the query heads that share the KV head;
 *   top-K    = K largest scores, equal scores resolved to the lower block
 *              index, emitted in ascending block order (padding -1);
 *   attention= exact softmax over [selected history blocks] U [segment keys
 *              at positions <= the query's own], scale 1/sqrt(d);
 *   backward = gradients of <O, dO> with respect to Q, K_seg, V_seg only;
 *              the selection and the history are constants.
 * Block sizes: history blocks hold blk tokens (summaries, selection units);
 * query blocks hold qblk tokens (the rows that share one selection), qblk = blk
 * unless the dims say otherwise.  With qblk != blk nothing else changes: a
 * query block's mean is over its qblk rows, and a row attends to the blk
 * tokens of each block selected for its query block.
 *
 * Every function is a direct transcription of those definitions in double
 * precision: no blocking, no fusion, no reordering of sums.  OpenMP only
 * splits independent output rows between threads.
 *
 * Layouts (row-major, all double):
 *   q, d_o, o, dq        [B, S, Hq, d]
 *   k_seg, v_seg, dk, dv [B, S, Hkv, d]
 *   k_hist, v_hist       [B, nblk*blk, Hkv, d]
 *   summ                 [B, Hkv, nblk, d]
 *   qm                   [B, Hq, S/qblk, d]
 *   score                [B, Hkv, S/qblk, nblk]
 *   idx                  [B, Hkv, S/qblk, topk]  (int32)
 *   lse                  [B, Hq, S]
 * Query head hq belongs to KV head hq / (Hq/Hkv).
 */
#include "hga_oracle.h"

#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

/* Thread count of the OpenMP regions below (for timing the oracle on a given
 * number of host cores); the arithmetic does not depend on it. */
void ohga_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
int ohga_max_threads(void) { return omp_get_max_threads(); }

static size_t tok_off(int b, int t, int T, int h, int H, int d) {
  return (((size_t)b * T + t) * H + h) * (size_t)d;
}

/* Query-block size: qblk, or blk when the dims leave it 0. */
static int qb(const ohga_dims* D) { return D->qblk > 0 ? D->qblk : D->blk; }

static double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int k = 0; k < d; ++k) s += a[k] * b[k];
  return s;
}

/* summ[b,h,n,:] = (1/blk) * sum over the blk tokens of history block n. */
void ohga_block_summaries(const ohga_dims* D, const double* k_hist, double* summ) {
  const int T = D->nblk * D->blk;
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < D->B; ++b)
    for (int h = 0; h < D->Hkv; ++h)
      for (int n = 0; n < D->nblk; ++n) {
        double* out = summ + (((size_t)b * D->Hkv + h) * D->nblk + n) * D->d;
        for (int k = 0; k < D->d; ++k) {
          double s = 0.0;
          for (int t = 0; t < D->blk; ++t) s += k_hist[tok_off(b, n * D->blk + t, T, h, D->Hkv, D->d) + k];
          out[k] = s / D->blk;
        }
      }
}

/* qm[b,hq,i,:] = (1/qblk) * sum over the qblk queries of segment query block i. */
void ohga_query_means(const ohga_dims* D, const double* q, double* qm) {
  const int Q = qb(D);
  const int nqb = D->S / Q;
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < D->B; ++b)
    for (int hq = 0; hq < D->Hq; ++hq)
      for (int i = 0; i < nqb; ++i) {
        double* out = qm + (((size_t)b * D->Hq + hq) * nqb + i) * D->d;
        for (int k = 0; k < D->d; ++k) {
          double s = 0.0;
          for (int t = 0; t < Q; ++t) s += q[tok_off(b, i * Q + t, D->S, hq, D->Hq, D->d) + k];
          out[k] = s / Q;
        }
      }
}

/* score[b,h,i,n] = max over hq in group(h) of qm[b,hq,i] . summ[b,h,n] / sqrt(d). */
void ohga_block_scores(const ohga_dims* D, const double* qm, const double* summ, double* score) {
  const int nqb = D->S / qb(D);
  const int G = D->Hq / D->Hkv;
  const double inv_sqrt_d = 1.0 / sqrt((double)D->d);
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < D->B; ++b)
    for (int h = 0; h < D->Hkv; ++h)
      for (int i = 0; i < nqb; ++i)
        for (int n = 0; n < D->nblk; ++n) {
          const double* s = summ + (((size_t)b * D->Hkv + h) * D->nblk + n) * D->d;
          double best = -INFINITY;
          for (int g = 0; g < G; ++g) {
            const int hq = h * G + g;
            const double* m = qm + (((size_t)b * D->Hq + hq) * nqb + i) * D->d;
            const double v = dot(m, s, D->d) * inv_sqrt_d;
            if (v > best) best = v;
          }
          score[(((size_t)b * D->Hkv + h) * nqb + i) * D->nblk + n] = best;
        }
}

/* Order used by the selection: larger score first; equal scores (+0 == -0)
 * put the lower block index first. */
typedef struct { double s; int n; } ohga_cand;

static int cand_cmp(const void* pa, const void* pb) {
  const ohga_cand* a = (const ohga_cand*)pa;
  const ohga_cand* b = (const ohga_cand*)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->n < b->n) ? -1 : (a->n > b->n);
}

static int int_cmp(const void* pa, const void* pb) {
  const int a = *(const int*)pa, b = *(const int*)pb;
  return (a > b) - (a < b);
}

/* idx[b,h,i,:]: the min(topk, nblk) best blocks by the order above, listed in
 * ascending block index, padded with -1. */
void ohga_select_topk(const ohga_dims* D, const double* score, int32_t* idx) {
  const int nqb = D->S / qb(D);
  const int keff = D->topk < D->nblk ? D->topk : D->nblk;
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < D->B; ++b)
    for (int h = 0; h < D->Hkv; ++h)
      for (int i = 0; i < nqb; ++i) {
        const size_t row = ((size_t)b * D->Hkv + h) * nqb + i;
        ohga_cand* c = (ohga_cand*)malloc(sizeof(ohga_cand) * (D->nblk > 0 ? D->nblk : 1));
        int* chosen = (int*)malloc(sizeof(int) * (keff > 0 ? keff : 1));
        for (int n = 0; n < D->nblk; ++n) { c[n].s = score[row * D->nblk + n]; c[n].n = n; }
        qsort(c, D->nblk, sizeof(ohga_cand), cand_cmp);
        for (int r = 0; r < keff; ++r) chosen[r] = c[r].n;
        qsort(chosen, keff, sizeof(int), int_cmp);
        for (int r = 0; r < D->topk; ++r) idx[row * D->topk + r] = r < keff ? chosen[r] : -1;
        free(chosen);
        free(c);
      }
}

/* The key set of query row p (segment position) for KV head h, query block i:
 * every token of every selected history block, then segment tokens 0..p.
 * Returns the count; keys/vals receive pointers into the inputs. */
static int gather_keys(const ohga_dims* D, int b, int h, int i, int p, const double* k_seg, const double* v_seg,
                       const double* k_hist, const double* v_hist, const int32_t* idx, const double** keys,
                       const double** vals) {
  const int nqb = D->S / qb(D);
  const int T = D->nblk * D->blk;
  int nk = 0;
  const int32_t* sel = idx + (((size_t)b * D->Hkv + h) * nqb + i) * D->topk;
  for (int r = 0; r < D->topk; ++r) {
    const int n = sel[r];
    if (n < 0) continue;
    for (int t = 0; t < D->blk; ++t) {
      keys[nk] = k_hist + tok_off(b, n * D->blk + t, T, h, D->Hkv, D->d);
      vals[nk] = v_hist + tok_off(b, n * D->blk + t, T, h, D->Hkv, D->d);
      ++nk;
    }
  }
  for (int t = 0; t <= p; ++t) {
    keys[nk] = k_seg + tok_off(b, t, D->S, h, D->Hkv, D->d);
    vals[nk] = v_seg + tok_off(b, t, D->S, h, D->Hkv, D->d);
    ++nk;
  }
  return nk;
}

static int in_range(int h, int h0, int h1) { return h >= h0 && h < h1; }

/* Softmax attention of one query row over its key set, in fp64:
 * s_j = q.k_j/sqrt(d); m = max s; P_j = exp(s_j - m)/sum; O = sum P_j v_j;
 * LSE = m + log(sum exp(s_j - m)).  p_out (optional) receives P. */
static void row_attention(int d, const double* qrow, int nk, const double** keys, const double** vals, double* orow,
                          double* lse, double* s_buf, double* p_out) {
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  double m = -INFINITY;
  for (int j = 0; j < nk; ++j) {
    s_buf[j] = dot(qrow, keys[j], d) * inv_sqrt_d;
    if (s_buf[j] > m) m = s_buf[j];
  }
  double z = 0.0;
  for (int j = 0; j < nk; ++j) z += exp(s_buf[j] - m);
  for (int k = 0; k < d; ++k) orow[k] = 0.0;
  for (int j = 0; j < nk; ++j) {
    const double pj = exp(s_buf[j] - m) / z;
    if (p_out) p_out[j] = pj;
    for (int k = 0; k < d; ++k) orow[k] += pj * vals[j][k];
  }
  *lse = m + log(z);
}

/* row_mask (optional, length S): only segment positions p with row_mask[p]
 * != 0 are computed. */
void ohga_attn_fwd(const ohga_dims* D, const double* q, const double* k_seg, const double* v_seg,
                   const double* k_hist, const double* v_hist, const int32_t* idx, int h0, int h1,
                   const int8_t* row_mask, double* o, double* lse) {
  const int G = D->Hq / D->Hkv;
  const int maxk = D->topk * D->blk + D->S;
#pragma omp parallel
  {
    const double** keys = (const double**)malloc(sizeof(double*) * maxk);
    const double** vals = (const double**)malloc(sizeof(double*) * maxk);
    double* s_buf = (double*)malloc(sizeof(double) * maxk);
#pragma omp for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < D->B; ++b)
      for (int hq = 0; hq < D->Hq; ++hq)
        for (int p = 0; p < D->S; ++p) {
          const int h = hq / G;
          if (!in_range(h, h0, h1)) continue;
          if (row_mask && !row_mask[p]) continue;
          const int nk = gather_keys(D, b, h, p / qb(D), p, k_seg, v_seg, k_hist, v_hist, idx, keys, vals);
          row_attention(D->d, q + tok_off(b, p, D->S, hq, D->Hq, D->d), nk, keys, vals,
                        o + tok_off(b, p, D->S, hq, D->Hq, D->d), &lse[((size_t)b * D->Hq + hq) * D->S + p], s_buf,
                        NULL);
        }
    free(keys);
    free(vals);
    free(s_buf);
  }
}

/* Backward of L = <O, dO> with the selection held fixed and no gradient into
 * the history.  With P the softmax row, dP_j = dO.v_j, Dr = dO.O = sum_j P_j dP_j:
 *   dS_j = P_j (dP_j - Dr)            (softmax Jacobian applied to dP)
 *   dq   = sum_j dS_j k_j / sqrt(d)
 *   dk_j = sum over rows and heads of the group of dS_j q / sqrt(d)  (segment keys)
 *   dv_j = sum over rows and heads of the group of P_j dO            (segment keys)
 * dk/dv are accumulated per segment key position in a second, key-major pass so
 * that each output element is one plain sum. */
void ohga_attn_bwd(const ohga_dims* D, const double* q, const double* k_seg, const double* v_seg,
                   const double* k_hist, const double* v_hist, const int32_t* idx, const double* d_o, int h0, int h1,
                   double* dq, double* dk, double* dv) {
  const int G = D->Hq / D->Hkv;
  const int d = D->d;
  const int maxk = D->topk * D->blk + D->S;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  const size_t nrows = (size_t)D->B * D->Hq * D->S;
  double* lse = (double*)malloc(sizeof(double) * nrows);
  double* Dr = (double*)malloc(sizeof(double) * nrows);
  double* o = (double*)malloc(sizeof(double) * nrows * d);

  /* Pass 1: forward rows (O, LSE), Dr, and dq. */
#pragma omp parallel
  {
    const double** keys = (const double**)malloc(sizeof(double*) * maxk);
    const double** vals = (const double**)malloc(sizeof(double*) * maxk);
    double* s_buf = (double*)malloc(sizeof(double) * maxk);
    double* p_buf = (double*)malloc(sizeof(double) * maxk);
#pragma omp for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < D->B; ++b)
      for (int hq = 0; hq < D->Hq; ++hq)
        for (int p = 0; p < D->S; ++p) {
          const int h = hq / G;
          if (!in_range(h, h0, h1)) continue;
          const size_t r = ((size_t)b * D->Hq + hq) * D->S + p;
          const size_t off = tok_off(b, p, D->S, hq, D->Hq, d);
          const int nk = gather_keys(D, b, h, p / qb(D), p, k_seg, v_seg, k_hist, v_hist, idx, keys, vals);
          row_attention(d, q + off, nk, keys, vals, o + r * d, &lse[r], s_buf, p_buf);
          Dr[r] = dot(d_o + off, o + r * d, d);
          for (int k = 0; k < d; ++k) dq[off + k] = 0.0;
          for (int j = 0; j < nk; ++j) {
            const double dp = dot(d_o + off, vals[j], d);
            const double ds = p_buf[j] * (dp - Dr[r]);
            for (int k = 0; k < d; ++k) dq[off + k] += ds * keys[j][k] * inv_sqrt_d;
          }
        }
    free(keys);
    free(vals);
    free(s_buf);
    free(p_buf);
  }

  /* Pass 2: dk, dv for each segment key position j of each KV head in range.
   * Row p (p >= j) of head hq sees key j; its probability is
   * exp(q.k_j/sqrt(d) - LSE). */
#pragma omp parallel for collapse(3) schedule(dynamic, 4)
  for (int b = 0; b < D->B; ++b)
    for (int h = 0; h < D->Hkv; ++h)
      for (int j = 0; j < D->S; ++j) {
        if (!in_range(h, h0, h1)) continue;
        const size_t koff = tok_off(b, j, D->S, h, D->Hkv, d);
        const double* kj = k_seg + koff;
        const double* vj = v_seg + koff;
        for (int k = 0; k < d; ++k) { dk[koff + k] = 0.0; dv[koff + k] = 0.0; }
        for (int g = 0; g < G; ++g) {
          const int hq = h * G + g;
          for (int p = j; p < D->S; ++p) {
            const size_t r = ((size_t)b * D->Hq + hq) * D->S + p;
            const size_t qoff = tok_off(b, p, D->S, hq, D->Hq, d);
            const double pj = exp(dot(q + qoff, kj, d) * inv_sqrt_d - lse[r]);
            const double dp = dot(d_o + qoff, vj, d);
            const double ds = pj * (dp - Dr[r]);
            for (int k = 0; k < d; ++k) {
              dk[koff + k] += ds * q[qoff + k] * inv_sqrt_d;
              dv[koff + k] += pj * d_o[qoff + k];
            }
          }
        }
      }
  free(lse);
  free(Dr);
  free(o);
}

/* ---------------------------------------------------------------- decode
 * Decode step (article, Industry impact / fr Impact: HGA also serves
 * generation).  nq new query tokens (1 <= nq) at active-segment positions
 * t0 .. t0+nq-1 form the step's query group, a partial query block:
 *   qm[b,hq,:]  = (1/nq) * sum over the nq new queries of q_new[b,u,hq,:]
 *   score[b,h,n] = max over hq in group(h) of qm[b,hq] . summ[b,h,n] / sqrt(d)
 *   idx[b,h,:]  = the min(topk, nblk) best blocks (ties to the lower index),
 *                 ascending, padded with -1
 * and new query u attends to every token of the selected history blocks and
 * to the segment tokens at positions 0 .. t0+u.  Layouts:
 *   q_new, o     [B, nq, Hq, d]
 *   k_seg, v_seg [B, S, Hkv, d]   (S = capacity of the segment's KV buffer;
 *                                  positions >= t0+nq are never read)
 *   summ         [B, Hkv, nblk, d];  score [B, Hkv, nblk];  idx [B, Hkv, topk]
 *   lse          [B, Hq, nq]
 */
void ohga_decode_select(const ohga_dims* D, int nq, const double* q_new, const double* summ, double* score,
                        int32_t* idx) {
  const int G = D->Hq / D->Hkv;
  const int keff = D->topk < D->nblk ? D->topk : D->nblk;
  const double inv_sqrt_d = 1.0 / sqrt((double)D->d);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < D->B; ++b)
    for (int h = 0; h < D->Hkv; ++h) {
      double* qm = (double*)malloc(sizeof(double) * (size_t)G * D->d);
      for (int g = 0; g < G; ++g)
        for (int k = 0; k < D->d; ++k) {
          double s = 0.0;
          for (int u = 0; u < nq; ++u) s += q_new[tok_off(b, u, nq, h * G + g, D->Hq, D->d) + k];
          qm[(size_t)g * D->d + k] = s / nq;
        }
      double* row = score + ((size_t)b * D->Hkv + h) * D->nblk;
      for (int n = 0; n < D->nblk; ++n) {
        const double* sv = summ + (((size_t)b * D->Hkv + h) * D->nblk + n) * D->d;
        double best = -INFINITY;
        for (int g = 0; g < G; ++g) {
          const double v = dot(qm + (size_t)g * D->d, sv, D->d) * inv_sqrt_d;
          if (v > best) best = v;
        }
        row[n] = best;
      }
      ohga_cand* c = (ohga_cand*)malloc(sizeof(ohga_cand) * (D->nblk > 0 ? D->nblk : 1));
      int* chosen = (int*)malloc(sizeof(int) * (keff > 0 ? keff : 1));
      for (int n = 0; n < D->nblk; ++n) { c[n].s = row[n]; c[n].n = n; }
      qsort(c, D->nblk, sizeof(ohga_cand), cand_cmp);
      for (int r = 0; r < keff; ++r) chosen[r] = c[r].n;
      qsort(chosen, keff, sizeof(int), int_cmp);
      int32_t* out = idx + ((size_t)b * D->Hkv + h) * D->topk;
      for (int r = 0; r < D->topk; ++r) out[r] = r < keff ? chosen[r] : -1;
      free(chosen);
      free(c);
      free(qm);
    }
}

void ohga_decode_attn(const ohga_dims* D, int nq, int t0, const double* q_new, const double* k_seg,
                      const double* v_seg, const double* k_hist, const double* v_hist, const int32_t* idx, double* o,
                      double* lse) {
  const int G = D->Hq / D->Hkv;
  const int T = D->nblk * D->blk;
  const int maxk = D->topk * D->blk + t0 + nq;
#pragma omp parallel
  {
    const double** keys = (const double**)malloc(sizeof(double*) * maxk);
    const double** vals = (const double**)malloc(sizeof(double*) * maxk);
    double* s_buf = (double*)malloc(sizeof(double) * maxk);
#pragma omp for collapse(3) schedule(dynamic, 4)
    for (int b = 0; b < D->B; ++b)
      for (int hq = 0; hq < D->Hq; ++hq)
        for (int u = 0; u < nq; ++u) {
          const int h = hq / G;
          const int32_t* sel = idx + ((size_t)b * D->Hkv + h) * D->topk;
          int nk = 0;
          for (int r = 0; r < D->topk; ++r) {
            const int n = sel[r];
            if (n < 0) continue;
            for (int t = 0; t < D->blk; ++t) {
              keys[nk] = k_hist + tok_off(b, n * D->blk + t, T, h, D->Hkv, D->d);
              vals[nk] = v_hist + tok_off(b, n * D->blk + t, T, h, D->Hkv, D->d);
              ++nk;
            }
          }
          for (int t = 0; t <= t0 + u; ++t) {
            keys[nk] = k_seg + tok_off(b, t, D->S, h, D->Hkv, D->d);
            vals[nk] = v_seg + tok_off(b, t, D->S, h, D->Hkv, D->d);
            ++nk;
          }
          row_attention(D->d, q_new + tok_off(b, u, nq, hq, D->Hq, D->d), nk, keys, vals,
                        o + tok_off(b, u, nq, hq, D->Hq, D->d), &lse[((size_t)b * D->Hq + hq) * nq + u], s_buf, NULL);
        }
    free(keys);
    free(vals);
    free(s_buf);
  }
}

/* ---------------------------------------------------------------- sparse backward
 * Sparse segment backprop in the manner of SpaCO ("Training Long-Context
 * LLMs Efficiently via Chunk-wise Optimization", proposed method): only a
 * chosen subset of the segment's query blocks propagates gradient, and the
 * chosen ones are scaled by a correction factor.  With the HGA history
 * detached, a gradient path never leaves the segment, so the estimator is
 * the backward of L = scale * sum over the chosen blocks' rows of <O, dO>:
 * the plain backward (ohga_attn_bwd) with dO replaced by
 *   dO_eff[b, p] = scale * dO[b, p]  if qmask[b, p / qblk] != 0,  else 0.
 * qmask: [B, S/qblk] int8. */
void ohga_attn_bwd_sparse(const ohga_dims* D, const double* q, const double* k_seg, const double* v_seg,
                          const double* k_hist, const double* v_hist, const int32_t* idx, const double* d_o,
                          const int8_t* qmask, double scale, int h0, int h1, double* dq, double* dk, double* dv) {
  const size_t n = (size_t)D->B * D->S * D->Hq * D->d;
  const int nqb = D->S / qb(D);
  double* d_eff = (double*)malloc(sizeof(double) * (n > 0 ? n : 1));
  for (int b = 0; b < D->B; ++b)
    for (int p = 0; p < D->S; ++p) {
      const double f = qmask[(size_t)b * nqb + p / qb(D)] ? scale : 0.0;
      for (int hq = 0; hq < D->Hq; ++hq)
        for (int k = 0; k < D->d; ++k) {
          const size_t off = tok_off(b, p, D->S, hq, D->Hq, D->d) + k;
          d_eff[off] = f * d_o[off];
        }
    }
  ohga_attn_bwd(D, q, k_seg, v_seg, k_hist, v_hist, idx, d_eff, h0, h1, dq, dk, dv);
  free(d_eff);
}

/* Textbook dense causal attention over one whole sequence [B,T,H*,d] with
 * grouped KV heads: row t attends to keys 0..t.  Used only to check the
 * identity "every history block selected == dense causal attention". */
void ohga_dense_causal_fwd(int B, int T, int Hq, int Hkv, int d, const double* q, const double* k, const double* v,
                           double* o, double* lse) {
  const int G = Hq / Hkv;
#pragma omp parallel
  {
    const double** keys = (const double**)malloc(sizeof(double*) * T);
    const double** vals = (const double**)malloc(sizeof(double*) * T);
    double* s_buf = (double*)malloc(sizeof(double) * T);
#pragma omp for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
      for (int hq = 0; hq < Hq; ++hq)
        for (int t = 0; t < T; ++t) {
          for (int j = 0; j <= t; ++j) {
            keys[j] = k + tok_off(b, j, T, hq / G, Hkv, d);
            vals[j] = v + tok_off(b, j, T, hq / G, Hkv, d);
          }
          row_attention(d, q + tok_off(b, t, T, hq, Hq, d), t + 1, keys, vals, o + tok_off(b, t, T, hq, Hq, d),
                        &lse[((size_t)b * Hq + hq) * T + t], s_buf, NULL);
        }
    free(keys);
    free(vals);
    free(s_buf);
  }
}
