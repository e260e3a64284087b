/* Plain fp64 CPU oracle for the HGA per-segment attention step.
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the CPU
 * baseline of the benchmark; never by the product library.  See hga_oracle.c
 * for the definitions and layouts. */
#ifndef OHGA_ORACLE_H
#define OHGA_ORACLE_H
#include <stdint.h>

typedef struct {
  int B, Hq, Hkv, d, blk, S, nblk, topk;
  int qblk; /* query-block size; 0 = blk (the history block size) */
} ohga_dims;

void ohga_set_threads(int n);
int ohga_max_threads(void);
void ohga_block_summaries(const ohga_dims* D, const double* k_hist, double* summ);
void ohga_query_means(const ohga_dims* D, const double* q, double* qm);
void ohga_block_scores(const ohga_dims* D, const double* qm, const double* summ, double* score);
void ohga_select_topk(const ohga_dims* D, const double* score, int32_t* idx);
void ohga_attn_fwd(const ohga_dims* D, const double* q, const double* k_seg, const double* v_seg,
                   const double* k_hist, const double* v_hist, const int32_t* idx, int h0, int h1,
                   const int8_t* row_mask, double* o, double* lse);
void ohga_attn_bwd(const ohga_dims* D, const double* q, const double* k_seg, const double* v_seg,
                   const double* k_hist, const double* v_hist, const int32_t* idx, const double* d_o, int h0, int h1,
                   double* dq, double* dk, double* dv);
void ohga_attn_bwd_sparse(const ohga_dims* D, const double* q, const double* k_seg, const double* v_seg,
                          const double* k_hist, const double* v_hist, const int32_t* idx, const double* d_o,
                          const int8_t* qmask, double scale, int h0, int h1, double* dq, double* dk, double* dv);
void ohga_decode_select(const ohga_dims* D, int nq, const double* q_new, const double* summ, double* score,
                        int32_t* idx);
void ohga_decode_attn(const ohga_dims* D, int nq, int t0, const double* q_new, const double* k_seg,
                      const double* v_seg, const double* k_hist, const double* v_hist, const int32_t* idx, double* o,
                      double* lse);
void ohga_dense_causal_fwd(int B, int T, int Hq, int Hkv, int d, const double* q, const double* k, const double* v,
                           double* o, double* lse);
#endif
