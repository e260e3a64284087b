// CUDA-core kernels of the HGA attention step: forward and segment-only
// backward for every supported shape, in fp32 or bf16 storage with fp32
// arithmetic.  They serve the fp32 configuration (which tensor cores cannot
// meet at 1e-4: TF32 rounding alone is ~1e-3) and shapes outside the tcgen05
// kernels' tiling.
//
// Article: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global Attention
// and Segmented Backpropagation in Practice", Background: per query block, exact
// attention over a bounded set of history tokens plus the active segment; only
// the active segment is differentiable, the history is detached.
//
// One warp per output row (query row for O/dQ, segment key for dK/dV); the d
// components of a row are spread over the 32 lanes (d/32 each) and dot
// products are finished with warp shuffles.  fp32 throughout; the softmax
// uses the online (running max) form with accurate expf.
#include <float.h>

#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void st(T* p, float v);
template <>
__device__ __forceinline__ void st<float>(float* p, float v) {
  *p = v;
}
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct SimtArgs {
  int B, Hq, Hkv, d, blk, S, nkv, topk, nqb, G;
  int qblk;     // query-block size (rows sharing one selection); blk = history block size
  float scale;  // 1/sqrt(d)
  const int32_t* idx;
  int* err;
  const uint8_t* qmask;  // sparse backward: query blocks that propagate gradient (nullptr: all)
  float gscale;          // sparse backward: factor on every gradient (1: plain backward)
};

__device__ __forceinline__ bool block_on(const SimtArgs& a, int b, int p) {
  return !a.qmask || a.qmask[(size_t)b * a.nqb + p / a.qblk];
}

// Key j of query block i: either history token (block idx, offset) or a
// segment token.  Enumerates history tokens of valid selected blocks first,
// then segment tokens 0..p.
template <int DPL, typename T, typename F>
__device__ __forceinline__ void for_each_key(const SimtArgs& a, int b, int h, int p, const T* ks, const T* kh,
                                             F&& f) {
  const int i = p / a.qblk;
  const int32_t* sel = a.idx + (((size_t)b * a.Hkv + h) * a.nqb + i) * a.topk;
  const size_t hist_T = (size_t)a.nkv * a.blk;
  for (int r = 0; r < a.topk; ++r) {
    const int n = sel[r];
    if (n < 0 || n >= a.nkv) {
      if (n != -1 && (threadIdx.x & 31) == 0) flag_error(a.err, kDevErrIndex);
      continue;
    }
    for (int t = 0; t < a.blk; ++t) {
      const size_t tok = (size_t)n * a.blk + t;
      f(kh + (((size_t)b * hist_T + tok) * a.Hkv + h) * a.d, true, tok);
    }
  }
  for (int t = 0; t <= p; ++t) f(ks + (((size_t)b * a.S + t) * a.Hkv + h) * a.d, false, (size_t)t);
}

// Forward: warp = (b, hq, p).
template <int DPL, typename T>
__global__ void __launch_bounds__(256) fwd_simt_kernel(SimtArgs a, const T* __restrict__ q, const T* __restrict__ ks,
                                                       const T* __restrict__ vs, const T* __restrict__ kh,
                                                       const T* __restrict__ vh, T* __restrict__ o,
                                                       float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.B * a.Hq * a.S) return;
  const int p = row % a.S, hq = (row / a.S) % a.Hq, b = row / (a.S * a.Hq);
  const int h = hq / a.G;
  const size_t qoff = (((size_t)b * a.S + p) * a.Hq + hq) * a.d;
  float qv[DPL], acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    qv[e] = ld(q + qoff + lane + 32 * e) * a.scale;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const size_t hist_T = (size_t)a.nkv * a.blk;
  for_each_key<DPL>(a, b, h, p, ks, kh, [&](const T* kp, bool hist, size_t tok) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) s += qv[e] * ld(kp + lane + 32 * e);
    s = warp_sum(s);
    const T* vp = hist ? vh + (((size_t)b * hist_T + tok) * a.Hkv + h) * a.d
                       : vs + (((size_t)b * a.S + tok) * a.Hkv + h) * a.d;
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn);
    const float pj = expf(s - mn);
    l = l * corr + pj;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = acc[e] * corr + pj * ld(vp + lane + 32 * e);
    m = mn;
  });
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < DPL; ++e) st(o + qoff + lane + 32 * e, acc[e] * inv);
  if (lane == 0) lse[((size_t)b * a.Hq + hq) * a.S + p] = m + logf(l);
}

// dQ: warp = (b, hq, p).  dS_j = P_j (dP_j - D), dq = scale * sum dS_j k_j.
template <int DPL, typename T>
__global__ void __launch_bounds__(256) dq_simt_kernel(SimtArgs a, const T* __restrict__ q, const T* __restrict__ ks,
                                                      const T* __restrict__ vs, const T* __restrict__ kh,
                                                      const T* __restrict__ vh, const T* __restrict__ d_o,
                                                      const float* __restrict__ lse, const float* __restrict__ Dr,
                                                      float* __restrict__ dq) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.B * a.Hq * a.S) return;
  const int p = row % a.S, hq = (row / a.S) % a.Hq, b = row / (a.S * a.Hq);
  const int h = hq / a.G;
  const size_t qoff = (((size_t)b * a.S + p) * a.Hq + hq) * a.d;
  if (!block_on(a, b, p)) {
#pragma unroll
    for (int e = 0; e < DPL; ++e) dq[qoff + lane + 32 * e] = 0.f;
    return;
  }
  const size_t r = ((size_t)b * a.Hq + hq) * a.S + p;
  const float L = lse[r], Dv = Dr[r];
  float qv[DPL], dov[DPL], acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    qv[e] = ld(q + qoff + lane + 32 * e) * a.scale;
    dov[e] = ld(d_o + qoff + lane + 32 * e);
    acc[e] = 0.f;
  }
  const size_t hist_T = (size_t)a.nkv * a.blk;
  for_each_key<DPL>(a, b, h, p, ks, kh, [&](const T* kp, bool hist, size_t tok) {
    const T* vp = hist ? vh + (((size_t)b * hist_T + tok) * a.Hkv + h) * a.d
                       : vs + (((size_t)b * a.S + tok) * a.Hkv + h) * a.d;
    float s = 0.f, dp = 0.f;
    float kv[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      kv[e] = ld(kp + lane + 32 * e);
      s += qv[e] * kv[e];
      dp += dov[e] * ld(vp + lane + 32 * e);
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float pj = expf(s - L);
    const float ds = pj * (dp - Dv);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] += ds * kv[e];
  });
#pragma unroll
  for (int e = 0; e < DPL; ++e) dq[qoff + lane + 32 * e] = acc[e] * (a.scale * a.gscale);
}

// dK/dV: warp = (b, h, segment key j); sums over the G heads and rows p >= j.
template <int DPL, typename T>
__global__ void __launch_bounds__(256) dkdv_simt_kernel(SimtArgs a, const T* __restrict__ q,
                                                        const T* __restrict__ ks, const T* __restrict__ vs,
                                                        const T* __restrict__ d_o, const float* __restrict__ lse,
                                                        const float* __restrict__ Dr, float* __restrict__ dk,
                                                        float* __restrict__ dv) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.B * a.Hkv * a.S) return;
  const int j = row % a.S, h = (row / a.S) % a.Hkv, b = row / (a.S * a.Hkv);
  const size_t koff = (((size_t)b * a.S + j) * a.Hkv + h) * a.d;
  float kv[DPL], vv[DPL], gk[DPL], gv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    kv[e] = ld(ks + koff + lane + 32 * e) * a.scale;
    vv[e] = ld(vs + koff + lane + 32 * e);
    gk[e] = 0.f;
    gv[e] = 0.f;
  }
  for (int g = 0; g < a.G; ++g) {
    const int hq = h * a.G + g;
    for (int p = j; p < a.S; ++p) {
      if (!block_on(a, b, p)) continue;
      const size_t qoff = (((size_t)b * a.S + p) * a.Hq + hq) * a.d;
      const size_t r = ((size_t)b * a.Hq + hq) * a.S + p;
      float qv[DPL], dov[DPL];
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        qv[e] = ld(q + qoff + lane + 32 * e);
        dov[e] = ld(d_o + qoff + lane + 32 * e);
        s += qv[e] * kv[e];
        dp += dov[e] * vv[e];
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      const float pj = expf(s - lse[r]);
      const float ds = pj * (dp - Dr[r]);
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        gk[e] += ds * qv[e];
        gv[e] += pj * dov[e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    dk[koff + lane + 32 * e] = gk[e] * (a.scale * a.gscale);
    dv[koff + lane + 32 * e] = gv[e] * a.gscale;
  }
}

SimtArgs make_args(const Shape& s, int nkv, const int32_t* idx, int* err) {
  SimtArgs a;
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.d = s.d; a.blk = s.blk; a.S = s.S; a.nkv = nkv; a.topk = s.topk;
  a.nqb = s.nqb(); a.G = s.G(); a.qblk = s.qblk; a.scale = 1.0f / sqrtf((float)s.d); a.idx = idx; a.err = err;
  a.qmask = nullptr; a.gscale = 1.0f;
  return a;
}

template <int DPL, typename T>
void fwd_simt(const SimtArgs& a, const void* q, const void* ks, const void* vs, const void* kh, const void* vh,
              void* o, float* lse, cudaStream_t st) {
  const int rows = a.B * a.Hq * a.S;
  fwd_simt_kernel<DPL, T><<<(rows + 7) / 8, 256, 0, st>>>(a, (const T*)q, (const T*)ks, (const T*)vs, (const T*)kh,
                                                          (const T*)vh, (T*)o, lse);
}

template <int DPL, typename T>
void bwd_simt(const SimtArgs& a, const void* q, const void* ks, const void* vs, const void* kh, const void* vh,
              const float* lse, const float* Dr, const void* d_o, float* dq, float* dk, float* dv, int parts,
              cudaStream_t st) {
  if (parts & kBwdDq) {
    const int rows = a.B * a.Hq * a.S;
    dq_simt_kernel<DPL, T><<<(rows + 7) / 8, 256, 0, st>>>(a, (const T*)q, (const T*)ks, (const T*)vs,
                                                           (const T*)kh, (const T*)vh, (const T*)d_o, lse, Dr, dq);
  }
  if (parts & kBwdDkdv) {
    const int krows = a.B * a.Hkv * a.S;
    dkdv_simt_kernel<DPL, T><<<(krows + 7) / 8, 256, 0, st>>>(a, (const T*)q, (const T*)ks, (const T*)vs,
                                                              (const T*)d_o, lse, Dr, dk, dv);
  }
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Shape& s, const void* q, const void* k_seg, const void* v_seg,
                                 const void* k_hist, const void* v_hist, int nkv, const int32_t* idx, void* o,
                                 float* lse, int* err, cudaStream_t st) {
  const SimtArgs a = make_args(s, nkv, idx, err);
  if (s.d == 64) {
    if (s.bf16) fwd_simt<2, __nv_bfloat16>(a, q, k_seg, v_seg, k_hist, v_hist, o, lse, st);
    else fwd_simt<2, float>(a, q, k_seg, v_seg, k_hist, v_hist, o, lse, st);
  } else {
    if (s.bf16) fwd_simt<4, __nv_bfloat16>(a, q, k_seg, v_seg, k_hist, v_hist, o, lse, st);
    else fwd_simt<4, float>(a, q, k_seg, v_seg, k_hist, v_hist, o, lse, st);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_simt(const Shape& s, const void* q, const void* k_seg, const void* v_seg,
                                 const void* k_hist, const void* v_hist, int nkv, const int32_t* idx,
                                 const float* lse, const float* Dr, const void* d_o, float* dq, float* dk,
                                 float* dv, int parts, int* err, cudaStream_t st, const uint8_t* qmask,
                                 float gscale) {
  SimtArgs a = make_args(s, nkv, idx, err);
  a.qmask = qmask;
  a.gscale = gscale;
  if (s.d == 64) {
    if (s.bf16) bwd_simt<2, __nv_bfloat16>(a, q, k_seg, v_seg, k_hist, v_hist, lse, Dr, d_o, dq, dk, dv, parts, st);
    else bwd_simt<2, float>(a, q, k_seg, v_seg, k_hist, v_hist, lse, Dr, d_o, dq, dk, dv, parts, st);
  } else {
    if (s.bf16) bwd_simt<4, __nv_bfloat16>(a, q, k_seg, v_seg, k_hist, v_hist, lse, Dr, d_o, dq, dk, dv, parts, st);
    else bwd_simt<4, float>(a, q, k_seg, v_seg, k_hist, v_hist, lse, Dr, d_o, dq, dk, dv, parts, st);
  }
  return cudaGetLastError();
}

}  // namespace hga
