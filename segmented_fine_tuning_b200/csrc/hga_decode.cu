// Decode step of HGA attention: a few new query tokens per step attend to the
// top-K history blocks picked for them and to the active segment's prefix.
//
// Article: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global Attention
// and Segmented Backpropagation in Practice", Industry impact (fr edition,
// Impact): the scheme also serves generation and retrieval.  The step's n_q
// new queries (segment positions t0 .. t0+n_q-1) form one partial query
// block: their mean is scored against the resident block summaries exactly as
// a whole query block is in the prefill (hga_select_topk's kernel, run with a
// query block of n_q rows), and new query u attends to the selected history
// blocks plus segment positions 0 .. t0+u.
//
// Attention is split over the key axis (flash-decoding): one CTA per (chunk of
// `block` keys, group of up to 16 query rows, batch x KV head).  The chunks are
// the K selected history blocks and the segment prefix cut into blocks.  Each
// CTA stages its K and V chunk in shared memory once (cp.async, 16-byte
// vectors, rows padded by 16 bytes so that the per-key reads are conflict
// free), forms the scores of its rows, and writes the chunk's partial softmax
// state (running max m, sum l, unnormalised O) to the caller's workspace.  A
// second kernel merges the chunks of every row: M = max m_c, L = sum l_c
// 2^(m_c - M), O = sum O_c 2^(m_c - M) / L, LSE = (M + log2 L) ln 2.
// For bf16 with at most 8 rows per KV head a streaming form of the chunk
// kernel (decode_stream_kernel, below) takes the chunks instead.
// The work is bound by HBM: the selected K/V blocks and the segment prefix
// are read once.
#include <float.h>

#include <type_traits>

#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

constexpr int kDecThreads = 128;
constexpr int kDecRows = 16;  // query rows per CTA

template <typename T>
struct DecElem;
template <>
struct DecElem<float> {
  static constexpr int E = 4;  // elements per 16 bytes
  __device__ static float at(const float* p) { return *p; }
  __device__ static void unpack(uint4 v, float* out) {
    out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
  }
};
template <>
struct DecElem<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ static float at(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ static void unpack(uint4 v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[2 * k] = __uint_as_float(w[k] << 16);
      out[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};


struct DecArgs {
  int Hq, Hkv, S, d, blk, nq, t0, topk, nkv, n_chunks, G, R;
  float sl2;             // log2(e) / sqrt(d)
  const int32_t* idx;    // [B, Hkv, topk]
  float* part_ml;        // [B, Hkv, n_chunks, R, 2]
  float* part_o;         // [B, Hkv, n_chunks, R, d]
  int* err;
};

// Shared memory: K and V chunk [blk][d + pad] of T, Q rows [16][d] fp32 (pre-
// scaled to log2 units), scores / probabilities [16][blk] fp32, row max and sum.
template <typename T>
size_t dec_smem_bytes(int blk, int d) {
  const size_t row = (size_t)d * sizeof(T) + 16;
  return 2 * blk * row + (size_t)kDecRows * d * 4 + (size_t)kDecRows * blk * 4 + 2 * kDecRows * 4;
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_partial_kernel(const T* __restrict__ q_new,
                                                                     const T* __restrict__ k_seg,
                                                                     const T* __restrict__ v_seg,
                                                                     const T* __restrict__ k_hist,
                                                                     const T* __restrict__ v_hist, const DecArgs a) {
  constexpr int E = DecElem<T>::E;
  extern __shared__ __align__(16) uint8_t dec_smem[];
  const int d = a.d, blk = a.blk;
  const int row_bytes = d * (int)sizeof(T) + 16;
  uint8_t* sK = dec_smem;
  uint8_t* sV = sK + (size_t)blk * row_bytes;
  float* sQ = reinterpret_cast<float*>(sV + (size_t)blk * row_bytes);  // [16][d]
  float* sS = sQ + kDecRows * d;                                        // [16][blk]
  float* sM = sS + kDecRows * blk;
  float* sL = sM + kDecRows;

  const int c = blockIdx.x, rg = blockIdx.y;
  const int b = blockIdx.z / a.Hkv, h = blockIdx.z % a.Hkv;
  const int tid = threadIdx.x;
  const int r0 = rg * kDecRows;
  const int nr = min(kDecRows, a.R - r0);

  // The chunk: a selected history block, or a stretch of the segment prefix.
  const bool hist = c < a.topk;
  const T* kb;
  const T* vb;
  int nk, pos0 = 0;
  if (hist) {
    int n = __ldg(a.idx + ((size_t)b * a.Hkv + h) * a.topk + c);
    if (n < -1 || n >= a.nkv) {
      if (tid == 0) flag_error(a.err, kDevErrIndex);
      n = -1;
    }
    nk = n >= 0 ? blk : 0;
    const size_t off = (((size_t)b * a.nkv * blk + (size_t)(n >= 0 ? n : 0) * blk) * a.Hkv + h) * d;
    kb = k_hist + off;
    vb = v_hist + off;
  } else {
    pos0 = (c - a.topk) * blk;
    nk = min(blk, a.t0 + a.nq - pos0);
    const size_t off = (((size_t)b * a.S + pos0) * a.Hkv + h) * d;
    kb = k_seg + off;
    vb = v_seg + off;
  }
  const size_t key_stride = (size_t)a.Hkv * d;  // elements between consecutive tokens

  // 1. stage K, then V (16-byte vectors, two copy groups: the scores only
  //    wait for K), and this CTA's query rows
  const int vpr = d / E;  // vectors per row
  for (int x = tid; x < nk * vpr; x += kDecThreads) {
    const int j = x / vpr, v = x % vpr;
    cp_async16(sK + (size_t)j * row_bytes + v * 16, kb + j * key_stride + v * E);
  }
  cp_async_commit();
  for (int x = tid; x < nk * vpr; x += kDecThreads) {
    const int j = x / vpr, v = x % vpr;
    cp_async16(sV + (size_t)j * row_bytes + v * 16, vb + j * key_stride + v * E);
  }
  cp_async_commit();
  for (int x = tid; x < nr * d; x += kDecThreads) {
    const int r = x / d, k = x % d;
    const int rr = r0 + r, g = rr / a.nq, u = rr % a.nq;
    const T* src = q_new + (((size_t)b * a.nq + u) * a.Hq + h * a.G + g) * d + k;
    sQ[r * d + k] = DecElem<T>::at(src) * a.sl2;
  }
  cp_async_wait_group<1>();  // this thread's K copies have landed
  __syncthreads();

  // 2. scores (log2 units), one key per thread, rows in groups of four (a
  //    group's products are only formed for rows that exist)
  for (int j = tid; j < blk; j += kDecThreads) {
    const uint8_t* krow = sK + (size_t)j * row_bytes;
    for (int rq = 0; rq < nr; rq += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (j < nk) {
        for (int v = 0; v < vpr; ++v) {
          float kv[E];
          DecElem<T>::unpack(*reinterpret_cast<const uint4*>(krow + v * 16), kv);
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4) {
            const float4* qr = reinterpret_cast<const float4*>(sQ + (rq + r4) * d + v * E);
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4) {
              const float4 q4 = qr[e4];  // same address in every lane: broadcast
              acc[r4] = fmaf(q4.x, kv[4 * e4], acc[r4]);
              acc[r4] = fmaf(q4.y, kv[4 * e4 + 1], acc[r4]);
              acc[r4] = fmaf(q4.z, kv[4 * e4 + 2], acc[r4]);
              acc[r4] = fmaf(q4.w, kv[4 * e4 + 3], acc[r4]);
            }
          }
        }
      }
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) {
        const int r = rq + r4;
        if (r < nr) {
          const int u = (r0 + r) % a.nq;
          const bool visible = j < nk && (hist || pos0 + j <= a.t0 + u);
          sS[r * blk + j] = visible ? acc[r4] : -INFINITY;
        }
      }
    }
  }
  __syncthreads();

  // 3. per row: max, probabilities 2^(s - m), sum (one warp per row)
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < nr; r += kDecThreads / 32) {
    float m = -INFINITY;
    for (int j = lane; j < blk; j += 32) m = fmaxf(m, sS[r * blk + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int j = lane; j < blk; j += 32) {
      const float p = (m == -INFINITY) ? 0.f : ex2_approx(sS[r * blk + j] - m);
      sS[r * blk + j] = p;
      l += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      sM[r] = m;
      sL[r] = l;
    }
  }
  cp_async_wait_group<0>();  // this thread's V copies have landed
  __syncthreads();

  // 4. unnormalised O of the chunk: thread = (column, row phase), rows in
  //    groups of four
  const int phases = kDecThreads / d;  // 1 (d = 128) or 2 (d = 64)
  const int col = tid % d, ph = tid / d;
  const size_t base = (((size_t)b * a.Hkv + h) * a.n_chunks + c) * a.R + r0;
  for (int rq = 4 * ph; rq < nr; rq += 4 * phases) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < nk; ++j) {
      const float vj = DecElem<T>::at(reinterpret_cast<const T*>(sV + (size_t)j * row_bytes) + col);
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) acc[r4] = fmaf(sS[(rq + r4) * blk + j], vj, acc[r4]);
    }
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4)
      if (rq + r4 < nr) a.part_o[(base + rq + r4) * d + col] = acc[r4];
  }
  if (tid < nr) {
    a.part_ml[(base + tid) * 2] = sM[tid];
    a.part_ml[(base + tid) * 2 + 1] = sL[tid];
  }
}

// One CTA per (batch x KV head, row), four warps.  The chunks' (m, l) pairs
// are staged in shared memory and turned into merge weights 2^(m_c - M) once;
// warp w then sums the unnormalised O partials of chunks w, w+4, ... with lane
// L owning channels L, L+32, ... (each chunk's row is one coalesced read per
// warp, and a warp's loads for four chunks are in flight together), and the
// four warp sums meet in shared memory.
constexpr int kMaxChunks = 512;
constexpr int kMaxHeadDim = 128;
template <typename T>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecArgs a, T* __restrict__ o,
                                                             float* __restrict__ lse) {
  __shared__ float w_s[kMaxChunks];
  __shared__ float l_s[kMaxChunks];
  __shared__ float red[4];
  __shared__ float osum[4][kMaxHeadDim];
  const int rr = blockIdx.x % a.R;
  const int bh = blockIdx.x / a.R;
  const int b = bh / a.Hkv, h = bh % a.Hkv;
  const int g = rr / a.nq, u = rr % a.nq;
  const int hq = h * a.G + g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = a.d, cpl = d >> 5;  // channels per lane: 2 or 4
  const float* ml = a.part_ml + ((size_t)bh * a.n_chunks * a.R + rr) * 2;
  float mloc = -INFINITY;
  for (int c = tid; c < a.n_chunks; c += 128) {
    const float mc = ml[(size_t)c * a.R * 2];
    w_s[c] = mc;
    l_s[c] = ml[(size_t)c * a.R * 2 + 1];
    mloc = fmaxf(mloc, mc);
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, k));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  for (int c = tid; c < a.n_chunks; c += 128) {
    const float mc = w_s[c];
    w_s[c] = (mc == -INFINITY) ? 0.f : ex2_approx(mc - M);
  }
  __syncthreads();
  const float* po = a.part_o + ((size_t)bh * a.n_chunks * a.R + rr) * d + lane;
  const size_t cstride = (size_t)a.R * d;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int c = warp;
  for (; c + 12 < a.n_chunks; c += 16) {
    float v[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int m = 0; m < 4; ++m) v[k][m] = m < cpl ? po[(size_t)(c + 4 * k) * cstride + 32 * m] : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float wk = w_s[c + 4 * k];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = fmaf(v[k][m], wk, acc[m]);
    }
  }
  for (; c < a.n_chunks; c += 4) {
    const float wk = w_s[c];
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (m < cpl) acc[m] = fmaf(po[(size_t)c * cstride + 32 * m], wk, acc[m]);
  }
#pragma unroll
  for (int m = 0; m < 4; ++m)
    if (m < cpl) osum[warp][lane + 32 * m] = acc[m];
  // L = sum_c l_c w_c, by warp 0 while the sums land
  float L = 0.f;
  if (warp == 0) {
    for (int k = lane; k < a.n_chunks; k += 32) L = fmaf(l_s[k], w_s[k], L);
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) L += __shfl_xor_sync(0xffffffffu, L, k);
    if (lane == 0) red[0] = L;
  }
  __syncthreads();
  L = red[0];
  if (tid < d) {
    const float sum = (osum[0][tid] + osum[1][tid]) + (osum[2][tid] + osum[3][tid]);
    o[(((size_t)b * a.nq + u) * a.Hq + hq) * d + tid] = (T)(sum / L);
  }
  if (tid == 0) lse[((size_t)b * a.Hq + hq) * a.nq + u] = (M + log2f(L)) * 0.6931471805599453f;
}

// Streaming form of the chunk kernel for bf16 and at most kR (4 or 8) query
// rows per KV head, the usual decode shape (G x n_q rows): one CTA of 8 warps
// per (chunk, batch x KV head).  Half-warp w (0..15) takes keys w, w+16, ...
// of the chunk; its 16 lanes split the head dimension (lane l holds channels
// [l*D/16, (l+1)*D/16)).  K comes straight from global memory into registers
// (all of a lane's pieces in flight at once) and meets the query rows held in
// registers; a row's score is reduced over the 16 lanes by shuffles.  V is
// staged in shared memory by cp.async from the start, so it lands while the
// scores are formed.  After the chunk's softmax each half-warp accumulates
// P V over its keys and the 16 half-warp partials are summed in shared
// memory.  The chunk's (m, l, O) go to the same workspace as the general
// kernel's, for the same merge.
constexpr int kStreamThreads = 256;
constexpr int kStreamKeysPerLane = 8;  // keys of a 128-key chunk per half-warp

template <int KD, int kR>
size_t stream_smem_bytes(int blk) {
  return (size_t)blk * KD * 2 + (size_t)kR * blk * 4 + 2 * kR * 4 + (size_t)8 * kR * KD * 4;
}

template <int KD, int kR>
__global__ void __launch_bounds__(kStreamThreads) decode_stream_kernel(const __nv_bfloat16* __restrict__ q_new,
                                                                       const __nv_bfloat16* __restrict__ k_seg,
                                                                       const __nv_bfloat16* __restrict__ v_seg,
                                                                       const __nv_bfloat16* __restrict__ k_hist,
                                                                       const __nv_bfloat16* __restrict__ v_hist,
                                                                       const DecArgs a) {
  constexpr int EL = KD / 16;  // channels per lane: 8 (16 bytes) or 4 (8 bytes)
  extern __shared__ __align__(16) uint8_t dec_smem[];
  const int blk = a.blk;
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(dec_smem);            // [blk][KD]
  float* sS = reinterpret_cast<float*>(dec_smem + (size_t)blk * KD * 2);      // [kR][blk]
  float* sM = sS + kR * blk;
  float* sL = sM + kR;
  float* sRed = sL + kR;                                                      // [8][kR][KD]

  // KV head fastest in the grid: the Hkv CTAs of a chunk read its tokens'
  // rows (all heads side by side in memory) together
  const int c = blockIdx.y;
  const int b = blockIdx.x / a.Hkv, h = blockIdx.x % a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hw = warp * 2 + (lane >> 4), hl = lane & 15;
  const int R = a.R;

  const bool hist = c < a.topk;
  const __nv_bfloat16* kb;
  const __nv_bfloat16* vb;
  int nk, pos0 = 0;
  if (hist) {
    int n = __ldg(a.idx + ((size_t)b * a.Hkv + h) * a.topk + c);
    if (n < -1 || n >= a.nkv) {
      if (tid == 0) flag_error(a.err, kDevErrIndex);
      n = -1;
    }
    nk = n >= 0 ? blk : 0;
    const size_t off = (((size_t)b * a.nkv * blk + (size_t)(n >= 0 ? n : 0) * blk) * a.Hkv + h) * KD;
    kb = k_hist + off;
    vb = v_hist + off;
  } else {
    pos0 = (c - a.topk) * blk;
    nk = min(blk, a.t0 + a.nq - pos0);
    const size_t off = (((size_t)b * a.S + pos0) * a.Hkv + h) * KD;
    kb = k_seg + off;
    vb = v_seg + off;
  }
  const size_t key_stride = (size_t)a.Hkv * KD;

  // 1. V into shared memory (16-byte cp.async), K pieces into registers
  for (int x = tid; x < nk * (KD / 8); x += kStreamThreads) {
    const int j = x / (KD / 8), v = x % (KD / 8);
    cp_async16(sV + (size_t)j * KD + v * 8, vb + j * key_stride + v * 8);
  }
  cp_async_commit();
  using Piece = typename std::conditional<EL == 8, uint4, uint2>::type;
  Piece kp[kStreamKeysPerLane];
#pragma unroll
  for (int kk = 0; kk < kStreamKeysPerLane; ++kk) {
    const int j = hw + 16 * kk;
    if (j < nk) kp[kk] = __ldg(reinterpret_cast<const Piece*>(kb + j * key_stride + hl * EL));
    else kp[kk] = Piece{};
  }
  // this lane's channels of the query rows, in log2 units (rows >= R are zero)
  float q[kR][EL];
#pragma unroll
  for (int r = 0; r < kR; ++r) {
    const int g = r / a.nq, u = r % a.nq;
    const __nv_bfloat16* src = q_new + (((size_t)b * a.nq + u) * a.Hq + h * a.G + g) * KD + hl * EL;
#pragma unroll
    for (int e = 0; e < EL; ++e) q[r][e] = r < R ? __bfloat162float(src[e]) * a.sl2 : 0.f;
  }

  // 2. scores: a half-warp per key, reduced over its 16 lanes
#pragma unroll
  for (int kk = 0; kk < kStreamKeysPerLane; ++kk) {
    const int j = hw + 16 * kk;
    float kv[EL];
    if constexpr (EL == 8) {
      DecElem<__nv_bfloat16>::unpack(kp[kk], kv);
    } else {
      const uint2 w = kp[kk];
      kv[0] = __uint_as_float(w.x << 16); kv[1] = __uint_as_float(w.x & 0xFFFF0000u);
      kv[2] = __uint_as_float(w.y << 16); kv[3] = __uint_as_float(w.y & 0xFFFF0000u);
    }
    float sc[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < EL; ++e) acc = fmaf(q[r][e], kv[e], acc);
      sc[r] = acc;
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int r = 0; r < kR; ++r) sc[r] += __shfl_xor_sync(0xffffffffu, sc[r], o);
    if (hl == 0 && j < blk) {
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        if (r < R) {
          const int u = r % a.nq;
          const bool visible = j < nk && (hist || pos0 + j <= a.t0 + u);
          sS[r * blk + j] = visible ? sc[r] : -INFINITY;
        }
      }
    }
  }
  __syncthreads();

  // 3. per row: max, probabilities 2^(s - m), sum (one warp per row)
  for (int r = warp; r < R; r += kStreamThreads / 32) {
    float m = -INFINITY;
    for (int j = lane; j < blk; j += 32) m = fmaxf(m, sS[r * blk + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int j = lane; j < blk; j += 32) {
      const float p = (m == -INFINITY) ? 0.f : ex2_approx(sS[r * blk + j] - m);
      sS[r * blk + j] = p;
      l += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      sM[r] = m;
      sL[r] = l;
    }
  }
  cp_async_wait_group<0>();  // this thread's V copies have landed
  __syncthreads();

  // 4. P V over the half-warp's keys, then the two half-warps of a warp by a
  //    shuffle and the 8 warps in shared memory
  float o[kR][EL];
#pragma unroll
  for (int r = 0; r < kR; ++r)
#pragma unroll
    for (int e = 0; e < EL; ++e) o[r][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < kStreamKeysPerLane; ++kk) {
    const int j = hw + 16 * kk;
    if (j < nk) {
      float vv[EL];
      const Piece w = *reinterpret_cast<const Piece*>(sV + (size_t)j * KD + hl * EL);
      if constexpr (EL == 8) {
        DecElem<__nv_bfloat16>::unpack(w, vv);
      } else {
        vv[0] = __uint_as_float(w.x << 16); vv[1] = __uint_as_float(w.x & 0xFFFF0000u);
        vv[2] = __uint_as_float(w.y << 16); vv[3] = __uint_as_float(w.y & 0xFFFF0000u);
      }
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const float pr = r < R ? sS[r * blk + j] : 0.f;  // the same address in all 16 lanes
#pragma unroll
        for (int e = 0; e < EL; ++e) o[r][e] = fmaf(pr, vv[e], o[r][e]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kR; ++r)
#pragma unroll
    for (int e = 0; e < EL; ++e) o[r][e] += __shfl_xor_sync(0xffffffffu, o[r][e], 16);
  if (lane < 16) {
#pragma unroll
    for (int r = 0; r < kR; ++r)
#pragma unroll
      for (int e = 0; e < EL; ++e) sRed[((size_t)warp * kR + r) * KD + hl * EL + e] = o[r][e];
  }
  __syncthreads();
  const size_t base = (((size_t)b * a.Hkv + h) * a.n_chunks + c) * a.R;
  for (int x = tid; x < R * KD; x += kStreamThreads) {
    const int r = x / KD, col = x % KD;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += sRed[((size_t)w * kR + r) * KD + col];
    a.part_o[(base + r) * KD + col] = sum;
  }
  if (tid < R) {
    a.part_ml[(base + tid) * 2] = sM[tid];
    a.part_ml[(base + tid) * 2 + 1] = sL[tid];
  }
}

}  // namespace

size_t decode_workspace_floats(const Shape& s, int nq) {
  const int n_chunks = s.topk + (s.S + s.blk - 1) / s.blk;
  const size_t rows = (size_t)s.B * s.Hkv * n_chunks * s.G() * nq;
  return rows * (2 + s.d);
}

cudaError_t launch_decode_attn(const Shape& s, int nq, int t0, const void* q_new, const void* k_seg,
                               const void* v_seg, const void* k_hist, const void* v_hist, int nkv,
                               const int32_t* idx, void* o, float* lse, float* ws, int* err, cudaStream_t st) {
  DecArgs a;
  a.Hq = s.Hq; a.Hkv = s.Hkv; a.S = s.S; a.d = s.d; a.blk = s.blk; a.nq = nq; a.t0 = t0; a.topk = s.topk;
  a.nkv = nkv; a.G = s.G(); a.R = s.G() * nq;
  a.n_chunks = s.topk + (t0 + nq + s.blk - 1) / s.blk;
  if (a.n_chunks > kMaxChunks || s.d > kMaxHeadDim || s.d % 32 != 0) return cudaErrorInvalidValue;
  a.sl2 = 1.4426950408889634f / sqrtf((float)s.d);
  a.idx = idx; a.err = err;
  a.part_ml = ws;
  a.part_o = ws + (size_t)s.B * s.Hkv * a.n_chunks * a.R * 2;
  const dim3 grid(a.n_chunks, (a.R + kDecRows - 1) / kDecRows, s.B * s.Hkv);
  cudaError_t e;
  if (s.bf16 && a.R <= 8 && (s.d == 128 || s.d == 64) && s.blk <= 16 * kStreamKeysPerLane) {
    // the usual decode shape: the streaming chunk kernel
    const dim3 sgrid(s.B * s.Hkv, a.n_chunks);
    const bool r4 = a.R <= 4;
    const void* fn = s.d == 128 ? (r4 ? reinterpret_cast<const void*>(decode_stream_kernel<128, 4>)
                                      : reinterpret_cast<const void*>(decode_stream_kernel<128, 8>))
                                : (r4 ? reinterpret_cast<const void*>(decode_stream_kernel<64, 4>)
                                      : reinterpret_cast<const void*>(decode_stream_kernel<64, 8>));
    const size_t smem = s.d == 128 ? (r4 ? stream_smem_bytes<128, 4>(s.blk) : stream_smem_bytes<128, 8>(s.blk))
                                   : (r4 ? stream_smem_bytes<64, 4>(s.blk) : stream_smem_bytes<64, 8>(s.blk));
    if ((e = smem_limit(fn, smem)) != cudaSuccess) return e;
    const __nv_bfloat16* qn = static_cast<const __nv_bfloat16*>(q_new);
    const __nv_bfloat16* ks = static_cast<const __nv_bfloat16*>(k_seg);
    const __nv_bfloat16* vs = static_cast<const __nv_bfloat16*>(v_seg);
    const __nv_bfloat16* kh = static_cast<const __nv_bfloat16*>(k_hist);
    const __nv_bfloat16* vh = static_cast<const __nv_bfloat16*>(v_hist);
    if (s.d == 128 && r4)
      decode_stream_kernel<128, 4><<<sgrid, kStreamThreads, smem, st>>>(qn, ks, vs, kh, vh, a);
    else if (s.d == 128)
      decode_stream_kernel<128, 8><<<sgrid, kStreamThreads, smem, st>>>(qn, ks, vs, kh, vh, a);
    else if (r4)
      decode_stream_kernel<64, 4><<<sgrid, kStreamThreads, smem, st>>>(qn, ks, vs, kh, vh, a);
    else
      decode_stream_kernel<64, 8><<<sgrid, kStreamThreads, smem, st>>>(qn, ks, vs, kh, vh, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_combine_kernel<__nv_bfloat16><<<s.B * s.Hkv * a.R, 128, 0, st>>>(a, static_cast<__nv_bfloat16*>(o), lse);
  } else if (s.bf16) {
    const size_t smem = dec_smem_bytes<__nv_bfloat16>(s.blk, s.d);
    auto kp = decode_partial_kernel<__nv_bfloat16>;
    if ((e = smem_limit(reinterpret_cast<const void*>(kp), smem)) != cudaSuccess)
      return e;
    kp<<<grid, kDecThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(q_new),
                                        static_cast<const __nv_bfloat16*>(k_seg),
                                        static_cast<const __nv_bfloat16*>(v_seg),
                                        static_cast<const __nv_bfloat16*>(k_hist),
                                        static_cast<const __nv_bfloat16*>(v_hist), a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_combine_kernel<__nv_bfloat16><<<s.B * s.Hkv * a.R, 128, 0, st>>>(a, static_cast<__nv_bfloat16*>(o), lse);
  } else {
    const size_t smem = dec_smem_bytes<float>(s.blk, s.d);
    auto kp = decode_partial_kernel<float>;
    if ((e = smem_limit(reinterpret_cast<const void*>(kp), smem)) != cudaSuccess)
      return e;
    kp<<<grid, kDecThreads, smem, st>>>(static_cast<const float*>(q_new), static_cast<const float*>(k_seg),
                                        static_cast<const float*>(v_seg), static_cast<const float*>(k_hist),
                                        static_cast<const float*>(v_hist), a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_combine_kernel<float><<<s.B * s.Hkv * a.R, 128, 0, st>>>(a, static_cast<float*>(o), lse);
  }
  return cudaGetLastError();
}

}  // namespace hga
