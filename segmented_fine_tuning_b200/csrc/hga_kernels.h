// Internal launch interface between the C-ABI layer (hga_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hga {

// Bits of the per-device error flag.
enum : int { kDevErrIndex = 1, kDevErrTimeout = 2 };

struct Shape {
  int B, Hq, Hkv, d, blk, S, nblk, topk;
  bool bf16;
  int qblk;  // query-block size (blk when the dims leave it 0)
  int G() const { return Hq / Hkv; }
  int nqb() const { return S / qblk; }  // query blocks of the segment
  int nsb() const { return S / blk; }   // history blocks the finished segment becomes
};

// Largest K and history length the selection kernel handles in one CTA.
constexpr int kMaxTopk = 64;
constexpr int kMaxSelectBlocks = 4096;
// Longest segment (in query blocks) the tensor-core kernels handle.
constexpr int kMaxQueryBlocks = 128;

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes), called
// for a (kernel, device) pair only when `bytes` exceeds what was already set
// there: the attribute persists, and setting it on every launch costs host
// time that small kernels cannot hide.
cudaError_t smem_limit(const void* kernel, size_t bytes);

// Summaries of `nblocks` blocks: source blocks src_b0.. of k_src (T_src tokens
// per batch) -> destination blocks dst_b0.. of summ [B, s.nblk, Hkv, d].
cudaError_t launch_block_summaries(const Shape& s, const void* k_src, int T_src, int src_b0, int dst_b0, int nblocks,
                                   float* summ, cudaStream_t st);
// A finished segment enters the history in one pass over k_seg/v_seg [B,S,Hkv,d]:
// summaries of its S/blk blocks -> summ blocks dst_b0.. of [B, s.nblk, Hkv, d],
// and (pool_k != nullptr) block t of K and V -> pool slot slots[t] of
// pool_k/pool_v [B, pool_slots*blk, Hkv, d].  S/blk <= kMaxQueryBlocks.
cudaError_t launch_append_segment(const Shape& s, const void* k_seg, const void* v_seg, int dst_b0, float* summ,
                                  void* pool_k, void* pool_v, int pool_slots, const int32_t* slots, cudaStream_t st);
cudaError_t launch_select_topk(const Shape& s, const void* q, const float* summ, int32_t* idx, float* scores,
                               cudaStream_t st);
// idx_pool = slot_of_block[idx] on the device (-1 kept; absent or out-of-range
// blocks flag kDevErrIndex and give -1).
cudaError_t launch_remap_idx(const Shape& s, const int32_t* idx, const int32_t* slot_of_block, int32_t* idx_pool,
                             int* err, cudaStream_t st);
// Decode selection: keys of every history block (scored in parallel over the
// blocks) into ws (B*Hkv*nblk 64-bit keys), then top-K per (b, KV head) into
// idx [B, Hkv, topk] (and optional scores).
cudaError_t launch_decode_select(const Shape& s, int nq, const void* q_new, const float* summ, int32_t* idx,
                                 float* scores, void* ws, cudaStream_t st);
// Zero-copy gather: the distinct blocks of idx from a mapped pinned host tier
// (device addresses host_*_dev of [B, host_cap*blk, Hkv, d]) into a compact
// pool (slot = rank among the selected blocks), idx_pool = idx rewritten to
// slots; blocks without a slot (rank >= pool_slots) flag kDevErrIndex and give
// -1.  s.nblk <= gather_max_blocks().
int gather_max_blocks();
cudaError_t launch_gather_mapped(const Shape& s, const int32_t* idx, const void* host_k_dev, const void* host_v_dev,
                                 int host_cap, void* pool_k, void* pool_v, int pool_slots, int32_t* idx_pool,
                                 int* err, int n_sm, cudaStream_t st);
// dst_dev_view[0..n) = src[0..n) (int32), dst being pinned host memory seen
// through its device mapping: a device-to-host transfer by SM stores.
cudaError_t launch_store_mapped_i32(const int32_t* src, int32_t* dst_dev_view, size_t n, cudaStream_t st);
// D[b,hq,p] = sum_k dO[b,p,hq,k] * O[b,p,hq,k]  (fp32)
cudaError_t launch_bwd_preprocess(const Shape& s, const void* o, const void* d_o, float* Dr, cudaStream_t st);

// Backward parts (bit mask): dQ and dK/dV are independent once Dr exists.
enum : int { kBwdDq = 1, kBwdDkdv = 2 };

// CUDA-core attention (any supported shape, fp32 or bf16).
cudaError_t launch_attn_fwd_simt(const Shape& s, const void* q, const void* k_seg, const void* v_seg,
                                 const void* k_hist, const void* v_hist, int nkv, const int32_t* idx, void* o,
                                 float* lse, int* err, cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const Shape& s, const void* q, const void* k_seg, const void* v_seg,
                                 const void* k_hist, const void* v_hist, int nkv, const int32_t* idx,
                                 const float* lse, const float* Dr, const void* d_o, float* dq, float* dk,
                                 float* dv, int parts, int* err, cudaStream_t st, const uint8_t* qmask = nullptr,
                                 float gscale = 1.0f);

// Tensor-core attention (bf16, d in {64, 128}, block = 128, even G).  Tensor
// maps: q/d_o [B,S,Hq,d], k/v seg [B,S,Hkv,d], k/v hist [B,nkv*128,Hkv,d],
// all with a 64 x 1 x 128 x 1 box and 128-byte swizzle.
struct TcMaps {
  CUtensorMap q, d_o, ks, vs, kh, vh;
};
bool tc_supported(const Shape& s);
// withhold_kv (self test only): the producer issues no K/V tile loads, so the
// MMA warp's pipeline wait expires and the CTA takes its timeout path.
// heads_per_cta: 2 (a CTA serves a pair of query heads sharing its K/V tiles)
// or 1 (one head per CTA: twice the CTAs, for launches whose pairs would leave
// SMs idle).
cudaError_t launch_attn_fwd_tc(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, void* o, float* lse,
                               int* err, cudaStream_t st, int heads_per_cta, bool withhold_kv = false);
// qmask/gscale (sparse backward): only query blocks i with qmask[b*nqb + i] != 0
// propagate gradient, and every gradient is multiplied by gscale; nullptr / 1
// give the plain backward.
cudaError_t launch_attn_bwd_tc(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, const float* lse,
                               const float* Dr, float* dq, float* dk, float* dv, int parts, int* err,
                               cudaStream_t st, const uint8_t* qmask = nullptr, float gscale = 1.0f);

// Decode step: split-key attention of nq new queries (segment positions
// t0..t0+nq-1) over the selected history blocks idx [B,Hkv,topk] and the
// segment prefix; partial softmax states go to ws (decode_workspace_floats
// floats), then a merge kernel writes o [B,nq,Hq,d] and lse [B,Hq,nq].
// s.S is the segment buffer's capacity.
size_t decode_workspace_floats(const Shape& s, int nq);
cudaError_t launch_decode_attn(const Shape& s, int nq, int t0, const void* q_new, const void* k_seg,
                               const void* v_seg, const void* k_hist, const void* v_hist, int nkv,
                               const int32_t* idx, void* o, float* lse, float* ws, int* err, cudaStream_t st);

// Tensor-core operand-layout self test (see hga_selftest.h).
cudaError_t launch_selftest_umma(int form, const CUtensorMap& ma, const CUtensorMap& mb, const void* a_raw,
                                 float* d, int* err, cudaStream_t st);

}  // namespace hga
