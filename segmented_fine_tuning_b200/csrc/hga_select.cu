// HBM-bound kernels of the HGA step: block summaries, per-query-block
// selection (scores + top-K), and the backward preprocessing row dot.
//
// Article: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global Attention and
// Segmented Backpropagation in Practice" -- Deep analysis (resident per-block
// summaries), Background (bounded exact history set per query block).  The
// summary is the mean of a block's keys, the score the group-max of
// query-block-mean . summary / sqrt(d), ties to the lower block index.
#include <float.h>

#include <algorithm>

#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

template <typename T>
struct Vec;  // 16-byte vector of T, widened to float
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float* out) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
  __device__ static void unpack(uint4 v, float* out) {
    out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float* out) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), out);
  }
  __device__ static void unpack(uint4 v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[2 * k] = __uint_as_float(w[k] << 16);
      out[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};

// ------------------------------------------------------------ summaries
// CTA = (block n, column chunk of 32 vectors, batch b).  Each warp reads whole
// 32-vector stretches of token rows (coalesced 512 B for bf16), 8 warps cover
// 8 rows per pass; partials are combined in shared memory.  Source block
// src_b0 + n of k (T_src tokens per batch) -> destination block dst_b0 + n of
// summ [B, nblk_dst, Hkv, d].
template <typename T>
__global__ void __launch_bounds__(256) summaries_kernel(const T* __restrict__ k, int T_src, int Hkv, int d, int blk,
                                                        int src_b0, int dst_b0, int nblk_dst,
                                                        float* __restrict__ summ) {
  constexpr int V = Vec<T>::N;
  const int n = blockIdx.x;
  const int b = blockIdx.z;
  const int cols = Hkv * d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = (blockIdx.y * 32 + lane) * V;
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  if (col < cols) {
    const T* base = k + ((size_t)b * T_src + (size_t)(src_b0 + n) * blk) * cols + col;
    int t = warp;
    // up to 16 rows per warp (blk <= 128): all loads in flight at once
#pragma unroll 16
    for (; t < blk; t += 8) {
      float x[V];
      Vec<T>::load(base + (size_t)t * cols, x);
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] += x[e];
    }
  }
  __shared__ float part[8][32 * 8];
#pragma unroll
  for (int e = 0; e < V; ++e) part[warp][lane * V + e] = acc[e];
  __syncthreads();
  for (int x = threadIdx.x; x < 32 * V; x += 256) {
    float sacc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sacc += part[w][x];
    const int c = blockIdx.y * 32 * V + x;  // = h*d + channel: contiguous in the block-major layout
    if (c < cols) summ[((size_t)b * nblk_dst + dst_b0 + n) * cols + c] = sacc * (1.0f / blk);
  }
}

// ------------------------------------------------------------ segment append
// A finished segment entering the history, in one pass over its K and V:
// summaries of its blocks (as summaries_kernel) and, when a device block
// cache is given, the block copies of K and V into their pool slots.  CTA =
// (segment block t, column chunk of 32 vectors, batch b); each thread moves
// its column's 16-byte vector of every 8th row of the block.  Article: Deep
// analysis (summaries resident and growing), fr edition Analyse approfondie
// (finished segments leave the active window right away).
struct AppendSlots {
  int32_t slot[kMaxQueryBlocks];  // pool slot of segment block t
};

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(const T* __restrict__ k_seg, const T* __restrict__ v_seg, int S,
                                                     int Hkv, int d, int blk, int dst_b0, int nblk_dst,
                                                     float* __restrict__ summ, T* __restrict__ pool_k,
                                                     T* __restrict__ pool_v, int pool_slots, const AppendSlots slots) {
  constexpr int V = Vec<T>::N;
  const int t = blockIdx.x;
  const int b = blockIdx.z;
  const int cols = Hkv * d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = (blockIdx.y * 32 + lane) * V;
  const bool copy = pool_k != nullptr;
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  if (col < cols) {
    const size_t src0 = ((size_t)b * S + (size_t)t * blk) * cols + col;
    const size_t dst0 = copy ? ((size_t)b * pool_slots * blk + (size_t)slots.slot[t] * blk) * cols + col : 0;
    // K: every row is summed and, with a cache, stored to its slot
#pragma unroll 16
    for (int r = warp; r < blk; r += 8) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(k_seg + src0 + (size_t)r * cols));
      float x[V];
      Vec<T>::unpack(raw, x);
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] += x[e];
      if (copy) *reinterpret_cast<uint4*>(pool_k + dst0 + (size_t)r * cols) = raw;
    }
    if (copy) {
#pragma unroll 16
      for (int r = warp; r < blk; r += 8)
        *reinterpret_cast<uint4*>(pool_v + dst0 + (size_t)r * cols) =
            __ldg(reinterpret_cast<const uint4*>(v_seg + src0 + (size_t)r * cols));
    }
  }
  __shared__ float part[8][32 * 8];
#pragma unroll
  for (int e = 0; e < V; ++e) part[warp][lane * V + e] = acc[e];
  __syncthreads();
  for (int x = threadIdx.x; x < 32 * V; x += 256) {
    float sacc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sacc += part[w][x];
    const int c = blockIdx.y * 32 * V + x;
    if (c < cols) summ[((size_t)b * nblk_dst + dst_b0 + t) * cols + c] = sacc * (1.0f / blk);
  }
}

// ------------------------------------------------------------ selection
// Ordered 64-bit key: larger score first, then lower block index first.
__device__ __forceinline__ unsigned long long sel_key(float s, int n) {
  uint32_t u = __float_as_uint(s + 0.0f);  // -0 -> +0 so that they tie
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)n);
}

// The keff largest of keys[0..n) (distinct 64-bit keys, n >= keff >= 1) into
// chosen (block index) / chosen_key, in no particular order.  The keff-th
// largest key is found one byte at a time from the most significant end: per
// pass, a histogram of the next byte of the keys that still match the prefix
// found so far, and one warp walks it from the top to the byte where the count
// reaches the number of keys still to take.  Then every key at or above that
// threshold is taken.  Up to eight passes of three barriers each.  One pass
// first forms the bitwise AND and OR of all keys: the leading bytes on which
// every key agrees (one selection's scores often share their sign and
// exponent byte, and the index bytes above the largest index are constant)
// are taken as they are, without a histogram pass whose counts would all fall
// in one bin.
__device__ void topk_radix(const unsigned long long* keys, int n, int keff, int* chosen,
                           unsigned long long* chosen_key) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_need;
  __shared__ int s_count;
  __shared__ unsigned long long red_and[32], red_or[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned long long k_and = ~0ull, k_or = 0ull;
  for (int x = tid; x < n; x += blockDim.x) {
    const unsigned long long k = keys[x];
    k_and &= k;
    k_or |= k;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
    k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
  }
  if (lane == 0) {
    red_and[warp] = k_and;
    red_or[warp] = k_or;
  }
  __syncthreads();
  k_and = ~0ull;
  k_or = 0ull;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    k_and &= red_and[w];
    k_or |= red_or[w];
  }
  unsigned long long prefix = 0ull, mask = 0ull;
  int need = keff;
  for (int shift = 56; shift >= 0; shift -= 8) {
    if ((((k_and ^ k_or) >> shift) & 0xFFull) == 0ull) {
      // every key has this byte: so has the keff-th largest
      prefix |= k_and & (0xFFull << shift);
      mask |= 0xFFull << shift;
      continue;
    }
    for (int x = tid; x < 256; x += blockDim.x) hist[x] = 0u;
    __syncthreads();
    for (int x = tid; x < n; x += blockDim.x) {
      const unsigned long long k = keys[x];
      if ((k & mask) == prefix) atomicAdd(&hist[(unsigned)(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l holds the counts of bytes 255-8l down to 248-8l
      unsigned int c[8], sum = 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        c[k] = hist[255 - 8 * tid - k];
        sum += c[k];
      }
      unsigned int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const unsigned int excl = incl - sum;
      if (excl < (unsigned)need && incl >= (unsigned)need) {  // exactly one lane
        unsigned int cum = excl;
        int digit = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (cum + c[k] >= (unsigned)need) {
            digit = 255 - 8 * tid - k;
            break;
          }
          cum += c[k];
        }
        s_prefix = prefix | ((unsigned long long)digit << shift);
        s_need = need - (int)cum;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 0xFFull << shift;
  }
  // prefix is now the keff-th largest key
  if (tid == 0) s_count = 0;
  __syncthreads();
  for (int x = tid; x < n; x += blockDim.x) {
    const unsigned long long k = keys[x];
    if (k >= prefix) {
      const int slot = atomicAdd(&s_count, 1);
      chosen[slot] = x;
      chosen_key[slot] = k;
    }
  }
  __syncthreads();
}

// Writes one selection row: the chosen blocks in ascending order, then -1
// padding; scores (optional) recovered from the keys.  Threads 0..topk-1.
__device__ void write_selection(const int* chosen, const unsigned long long* chosen_key, int keff, int topk,
                                int32_t* idx_row, float* scores_row) {
  const int tid = threadIdx.x;
  if (tid >= topk) return;
  if (tid < keff) {
    const int n = chosen[tid];
    int rank = 0;
    for (int u = 0; u < keff; ++u) rank += chosen[u] < n;
    idx_row[rank] = n;
    if (scores_row) {
      // recover the score from the key (inverse of the ordering map)
      uint32_t u = (uint32_t)(chosen_key[tid] >> 32);
      u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
      scores_row[rank] = __uint_as_float(u);
    }
  } else {
    idx_row[tid] = -1;
    if (scores_row) scores_row[tid] = -INFINITY;
  }
}

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelU = 4;  // blocks per warp per scoring round
constexpr int kSelRankMax = 256;  // largest padded block count ranked by counting

// Scores of all nblk blocks for one selection, when the group size G divides
// 32: a warp takes U = 32/G blocks per round, every lane forms the partial dot
// products of its channels for all U*G (block, head) pairs, and one transposing
// butterfly (31 shuffles) leaves lane L with the full product of pair L --
// instead of 5 shuffles per product.  The group maximum is then log2(G) more
// shuffles, and lanes L with L % G == 0 write the keys.
template <int G>
__device__ void score_blocks_transposed(const float* qm, const float* __restrict__ summ, int b, int h, int Hkv, int d,
                                        int nblk, float inv_sqrt_d, unsigned long long* keys) {
  constexpr int U = 32 / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cpl = d >> 5;  // channels per lane: 2 or 4
  for (int n0 = warp * U; n0 < nblk; n0 += kSelWarps * U) {
    float sv[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int n = n0 + u;
      const float* src = summ + (((size_t)b * nblk + (n < nblk ? n : 0)) * Hkv + h) * d + lane;
#pragma unroll
      for (int m = 0; m < 4; ++m) sv[u][m] = (n < nblk && m < cpl) ? __ldg(src + 32 * m) : 0.f;
    }
    float v[32];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float qv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) qv[m] = m < cpl ? qm[g * d + lane + 32 * m] : 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u)
        v[u * G + g] = (qv[0] * sv[u][0] + qv[1] * sv[u][1]) + (qv[2] * sv[u][2] + qv[3] * sv[u][3]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int k = 0; k < off; ++k) {
        const float send = upper ? v[k] : v[k + off];
        const float keep = upper ? v[k + off] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    float best = v[0];  // pair index = lane = u * G + g
#pragma unroll
    for (int off = 1; off < G; off <<= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, off));
    const int n = n0 + lane / G;
    if ((lane % G) == 0 && n < nblk) keys[n] = sel_key(best * inv_sqrt_d, n);
  }
}

// CTA = (query block i, KV head h, batch b).  512 threads.
//  1. qm[g][:] = mean of the block's rows of Q for the G query heads of h
//     (the G heads of a KV head are contiguous in a token row).
//  2. score[n] = max_g qm[g] . summ[b,n,h] / sqrt(d): for G = 4 (the GQA
//     group of the Qwen3-8B shapes) with one transposing warp reduction per
//     32 (block, head) products;
//     otherwise a warp scores kSelU blocks per round, their summary channels
//     loaded before any arithmetic, the G * kSelU products reduced together.
//  3. top K_eff of the (score, index) keys by rank counting (up to 256
//     blocks) or a byte-wise radix select, then listed in ascending order.
template <typename T>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const T* __restrict__ q, const float* __restrict__ summ,
                                                             int S, int Hq, int Hkv, int d, int blk, int nblk, int topk,
                                                             float inv_sqrt_d, int32_t* __restrict__ idx,
                                                             float* __restrict__ scores) {
  constexpr int V = Vec<T>::N;
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv;
  const int nqb = S / blk;
  const int cols = G * d;
  float* qm = reinterpret_cast<float*>(sel_smem);                                        // [G*d]
  float* part = qm + cols + (cols & 1);                                                  // [kSelThreads*V]
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(part + kSelThreads * V);  // [nblk]
  __shared__ int chosen[kMaxTopk];
  __shared__ unsigned long long chosen_key[kMaxTopk];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int cpl = d >> 5;  // summary channels per lane (d is 64 or 128)

  // first scoring round's summary channels, in flight during step 1
  float sv[kSelU][4], sn[kSelU][4];
  auto load_round = [&](float (&dst)[kSelU][4], int n0) {
#pragma unroll
    for (int u = 0; u < kSelU; ++u) {
      const int n = n0 + u;
      const float* src = summ + (((size_t)b * nblk + (n < nblk ? n : 0)) * Hkv + h) * d + lane;
#pragma unroll
      for (int m = 0; m < 4; ++m) dst[u][m] = (n < nblk && m < cpl) ? __ldg(src + 32 * m) : 0.f;
    }
  };
  const bool transposed = (G == 4);
  if (!transposed) load_round(sv, warp * kSelU);

  // 1. query means: thread = (row phase r0, vector vt); rows r0, r0+rpp, ...
  //    are summed per thread, the rpp partials are then combined.
  const int tpr = cols / V;  // vectors per row (d is a multiple of 8)
  for (int c0 = 0; c0 < tpr; c0 += kSelThreads) {
    const int width = min(kSelThreads, tpr - c0);
    const int rpp = kSelThreads / width;
    const int vt = c0 + tid % width, r0 = tid / width;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    if (r0 < rpp) {
      const T* base = q + (((size_t)b * S + (size_t)i * blk) * Hq + (size_t)h * G) * d + (size_t)vt * V;
      const size_t rs = (size_t)Hq * d;
#pragma unroll 16
      for (int t = r0; t < blk; t += rpp) {
        float x[V];
        Vec<T>::load(base + t * rs, x);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += x[e];
      }
#pragma unroll
      for (int e = 0; e < V; ++e) part[r0 * width * V + (vt - c0) * V + e] = acc[e];
    }
    __syncthreads();
    for (int x = tid; x < width * V; x += kSelThreads) {
      float s = 0.f;
      for (int r = 0; r < rpp; ++r) s += part[r * width * V + x];
      qm[c0 * V + x] = s * (1.0f / blk);
    }
    __syncthreads();
  }

  // 2. scores -> keys.  G = 4: transposed reduction (above).
  //    Otherwise a warp scores kSelU blocks per round, the next round's
  //    summary channels loaded before this round's arithmetic.
  if (G == 4) score_blocks_transposed<4>(qm, summ, b, h, Hkv, d, nblk, inv_sqrt_d, keys);
  for (int n0 = warp * kSelU; !transposed && n0 < nblk; n0 += kSelWarps * kSelU) {
    const int n1 = n0 + kSelWarps * kSelU;
    if (n1 < nblk) load_round(sn, n1);
    float best[kSelU];
#pragma unroll
    for (int u = 0; u < kSelU; ++u) best[u] = -FLT_MAX;
    for (int g = 0; g < G; ++g) {
      float qv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) qv[m] = m < cpl ? qm[g * d + lane + 32 * m] : 0.f;
      float dot[kSelU];
#pragma unroll
      for (int u = 0; u < kSelU; ++u)
        dot[u] = (qv[0] * sv[u][0] + qv[1] * sv[u][1]) + (qv[2] * sv[u][2] + qv[3] * sv[u][3]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int u = 0; u < kSelU; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], o);
      }
#pragma unroll
      for (int u = 0; u < kSelU; ++u) best[u] = fmaxf(best[u], dot[u]);
    }
#pragma unroll
    for (int u = 0; u < kSelU; ++u) {
      const int n = n0 + u;
      if (lane == u && n < nblk) keys[n] = sel_key(best[u] * inv_sqrt_d, n);
    }
#pragma unroll
    for (int u = 0; u < kSelU; ++u)
#pragma unroll
      for (int m = 0; m < 4; ++m) sv[u][m] = sn[u][m];
  }
  __syncthreads();

  // 3. top K_eff.  Up to kSelRankMax blocks: every block counts the keys
  //    above its own (keys are distinct), no sort needed; beyond that the
  //    radix select above.
  const int keff = topk < nblk ? topk : nblk;
  if (nblk <= kSelRankMax) {
    for (int n = tid; n < nblk; n += kSelThreads) {
      const unsigned long long kn = keys[n];
      int rank = 0;
      for (int m = 0; m < nblk; ++m) rank += keys[m] > kn;
      if (rank < keff) {
        chosen[rank] = n;
        chosen_key[rank] = kn;
      }
    }
  } else if (keff > 0) {
    topk_radix(keys, nblk, keff, chosen, chosen_key);
  }
  __syncthreads();
  const size_t row = (((size_t)b * Hkv + h) * nqb + i) * topk;
  write_selection(chosen, chosen_key, keff, topk, idx + row, scores ? scores + row : nullptr);
}

// ------------------------------------------------------------ decode selection
// A decode step has one (partial) query block per (b, KV head), so one CTA per
// selection would leave the GPU nearly idle while it walks a long history.
// The scoring is therefore spread over the blocks: decode_score_kernel, CTA =
// (32 history blocks, KV head, batch), forms the mean of the n_q new queries
// of the G heads and writes each block's (score, index) key to the
// workspace; decode_topk_kernel, one CTA per (b, KV head), selects from them.
constexpr int kDecBlocksPerWarp = 4;
constexpr int kDecScoreWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kDecScoreWarps * 32)
    decode_score_kernel(const T* __restrict__ q_new, const float* __restrict__ summ, int nq, int Hq, int Hkv, int d,
                        int nblk, float inv_sqrt_d, unsigned long long* __restrict__ keys_out) {
  extern __shared__ __align__(16) float dsc_qm[];  // [G*d]
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv, cols = G * d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cpl = d >> 5;
  const int n_base = blockIdx.x * kDecScoreWarps * kDecBlocksPerWarp + warp * kDecBlocksPerWarp;
  // this warp's summary channels, in flight while the query mean is formed
  float sv[kDecBlocksPerWarp][4];
#pragma unroll
  for (int u = 0; u < kDecBlocksPerWarp; ++u) {
    const int n = n_base + u;
    const float* src = summ + (((size_t)b * nblk + (n < nblk ? n : 0)) * Hkv + h) * d + lane;
#pragma unroll
    for (int m = 0; m < 4; ++m) sv[u][m] = (n < nblk && m < cpl) ? __ldg(src + 32 * m) : 0.f;
  }
  // mean of the new queries of the G heads of KV head h (contiguous in a token row)
  const float inv_nq = 1.0f / nq;
  for (int c = tid; c < cols; c += blockDim.x) {
    const T* src = q_new + ((size_t)b * nq * Hq + (size_t)h * G) * d + c;
    float acc = 0.f;
    for (int u = 0; u < nq; ++u) acc += (float)src[(size_t)u * Hq * d];
    dsc_qm[c] = acc * inv_nq;
  }
  __syncthreads();
  float best[kDecBlocksPerWarp];
#pragma unroll
  for (int u = 0; u < kDecBlocksPerWarp; ++u) best[u] = -FLT_MAX;
  for (int g = 0; g < G; ++g) {
    float qv[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) qv[m] = m < cpl ? dsc_qm[g * d + lane + 32 * m] : 0.f;
    float dot[kDecBlocksPerWarp];
#pragma unroll
    for (int u = 0; u < kDecBlocksPerWarp; ++u)
      dot[u] = (qv[0] * sv[u][0] + qv[1] * sv[u][1]) + (qv[2] * sv[u][2] + qv[3] * sv[u][3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < kDecBlocksPerWarp; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], o);
    }
#pragma unroll
    for (int u = 0; u < kDecBlocksPerWarp; ++u) best[u] = fmaxf(best[u], dot[u]);
  }
#pragma unroll
  for (int u = 0; u < kDecBlocksPerWarp; ++u) {
    const int n = n_base + u;
    if (lane == u && n < nblk) keys_out[((size_t)b * Hkv + h) * nblk + n] = sel_key(best[u] * inv_sqrt_d, n);
  }
}

__global__ void __launch_bounds__(kSelThreads) decode_topk_kernel(const unsigned long long* __restrict__ keys_in,
                                                                  int Hkv, int nblk, int topk,
                                                                  int32_t* __restrict__ idx, float* __restrict__ scores) {
  extern __shared__ __align__(16) unsigned long long dtk_keys[];  // [nblk]
  __shared__ int chosen[kMaxTopk];
  __shared__ unsigned long long chosen_key[kMaxTopk];
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const unsigned long long* src = keys_in + ((size_t)b * Hkv + h) * nblk;
  for (int n = tid; n < nblk; n += kSelThreads) dtk_keys[n] = src[n];
  __syncthreads();
  const int keff = topk < nblk ? topk : nblk;
  if (nblk <= kSelRankMax) {
    for (int n = tid; n < nblk; n += kSelThreads) {
      const unsigned long long kn = dtk_keys[n];
      int rank = 0;
      for (int m = 0; m < nblk; ++m) rank += dtk_keys[m] > kn;
      if (rank < keff) {
        chosen[rank] = n;
        chosen_key[rank] = kn;
      }
    }
  } else if (keff > 0) {
    topk_radix(dtk_keys, nblk, keff, chosen, chosen_key);
  }
  __syncthreads();
  const size_t row = ((size_t)b * Hkv + h) * topk;
  write_selection(chosen, chosen_key, keff, topk, idx + row, scores ? scores + row : nullptr);
}

// ------------------------------------------------------------ bwd preprocess
// D = sum_k dO * O in fp32 per (b, p, hq) row.  A row is read by d/V lanes
// (16-byte vectors), so a warp covers 32V/d rows per pass; kPreRows passes are
// loaded before any arithmetic to keep enough bytes in flight.
// Dr[b, hq, p] = sum_k dO[b,p,hq,k] * O[b,p,hq,k].  Rows (token, head) are
// taken by the warps in a grid-stride loop, kPreRows rows per thread and pass
// with all their 16-byte loads in flight (kept as raw vectors, widened only
// at the multiply), lpr = d / V lanes per row, combined by shuffles.
constexpr int kPreRows = 8;
template <typename T>
__global__ void __launch_bounds__(256) preprocess_kernel(const T* __restrict__ o, const T* __restrict__ d_o, int S,
                                                         int Hq, int d, int rows, float* __restrict__ Dr) {
  constexpr int V = Vec<T>::N;
  const int lpr = d / V;    // lanes per row
  const int rpw = 32 / lpr;  // rows per warp per pass
  const int lane = threadIdx.x & 31;
  const int sub = lane / lpr, cl = lane % lpr;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; gw * rpw * kPreRows < rows; gw += warps) {
    const int row0 = gw * rpw * kPreRows + sub;
    uint4 xr[kPreRows], yr[kPreRows];
#pragma unroll
    for (int r = 0; r < kPreRows; ++r) {
      const int row = row0 + r * rpw;
      if (row < rows) {
        // rows are enumerated token-major: row = (b*S + p)*Hq + hq
        xr[r] = __ldg(reinterpret_cast<const uint4*>(o + (size_t)row * d + cl * V));
        yr[r] = __ldg(reinterpret_cast<const uint4*>(d_o + (size_t)row * d + cl * V));
      } else {
        xr[r] = yr[r] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float acc[kPreRows];
#pragma unroll
    for (int r = 0; r < kPreRows; ++r) {
      float x[V], y[V];
      Vec<T>::unpack(xr[r], x);
      Vec<T>::unpack(yr[r], y);
      acc[r] = 0.f;
#pragma unroll
      for (int e = 0; e < V; ++e) acc[r] = fmaf(x[e], y[e], acc[r]);
    }
    for (int k = lpr >> 1; k > 0; k >>= 1) {
#pragma unroll
      for (int r = 0; r < kPreRows; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], k);
    }
    if (cl == 0) {
#pragma unroll
      for (int r = 0; r < kPreRows; ++r) {
        const int row = row0 + r * rpw;
        if (row < rows) {
          const int hq = row % Hq;
          const int bp = row / Hq;
          const int b = bp / S, p = bp % S;
          Dr[((size_t)b * Hq + hq) * S + p] = acc[r];
        }
      }
    }
  }
}

// ------------------------------------------------------------ idx -> pool slots
// idx_pool[k] = slot_of_block[idx[k]] (-1 kept).  A block outside
// [0, nblk) or not resident (slot -1) flags the device error and yields -1.
__global__ void __launch_bounds__(256) remap_kernel(const int32_t* __restrict__ idx,
                                                    const int32_t* __restrict__ slot_of_block, int nblk, size_t n,
                                                    int32_t* __restrict__ idx_pool, int* err) {
  const size_t k = (size_t)blockIdx.x * 256 + threadIdx.x;
  if (k >= n) return;
  const int b = idx[k];
  int slot = -1;
  if (b >= 0) {
    if (b < nblk) slot = slot_of_block[b];
    if (slot < 0) flag_error(err, kDevErrIndex);
  }
  idx_pool[k] = slot;
}

}  // namespace

cudaError_t launch_block_summaries(const Shape& s, const void* k_src, int T_src, int src_b0, int dst_b0, int nblocks,
                                   float* summ, cudaStream_t st) {
  if (nblocks <= 0) return cudaSuccess;
  const int V = s.bf16 ? 8 : 4;
  const int cols = s.Hkv * s.d;
  dim3 grid(nblocks, (cols + 32 * V - 1) / (32 * V), s.B);
  if (s.bf16)
    summaries_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k_src), T_src, s.Hkv,
                                                          s.d, s.blk, src_b0, dst_b0, s.nblk, summ);
  else
    summaries_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(k_src), T_src, s.Hkv, s.d, s.blk, src_b0,
                                                  dst_b0, s.nblk, summ);
  return cudaGetLastError();
}

cudaError_t launch_append_segment(const Shape& s, const void* k_seg, const void* v_seg, int dst_b0, float* summ,
                                  void* pool_k, void* pool_v, int pool_slots, const int32_t* slots, cudaStream_t st) {
  const int nqb = s.nsb();  // the segment's blocks
  if (nqb <= 0) return cudaSuccess;
  AppendSlots sl;
  for (int t = 0; t < kMaxQueryBlocks; ++t) sl.slot[t] = (pool_k && t < nqb) ? slots[t] : 0;
  const int V = s.bf16 ? 8 : 4;
  const int cols = s.Hkv * s.d;
  dim3 grid(nqb, (cols + 32 * V - 1) / (32 * V), s.B);
  if (s.bf16)
    append_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k_seg), static_cast<const __nv_bfloat16*>(v_seg), s.S, s.Hkv, s.d, s.blk,
        dst_b0, s.nblk, summ, static_cast<__nv_bfloat16*>(pool_k), static_cast<__nv_bfloat16*>(pool_v), pool_slots, sl);
  else
    append_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(k_seg), static_cast<const float*>(v_seg), s.S,
                                               s.Hkv, s.d, s.blk, dst_b0, s.nblk, summ, static_cast<float*>(pool_k),
                                               static_cast<float*>(pool_v), pool_slots, sl);
  return cudaGetLastError();
}

cudaError_t launch_select_topk(const Shape& s, const void* q, const float* summ, int32_t* idx, float* scores,
                               cudaStream_t st) {
  const int cols = s.G() * s.d;
  const size_t smem = (size_t)(cols + (cols & 1) + kSelThreads * (s.bf16 ? 8 : 4)) * sizeof(float) +
                      (size_t)(s.nblk > 0 ? s.nblk : 1) * 8;
  dim3 grid(s.nqb(), s.Hkv, s.B);
  const float isd = 1.0f / sqrtf((float)s.d);
  cudaError_t e;
  if (s.bf16) {
    auto kern = select_kernel<__nv_bfloat16>;
    if ((e = smem_limit(reinterpret_cast<const void*>(kern), smem)) != cudaSuccess)
      return e;
    kern<<<grid, kSelThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(q), summ, s.S, s.Hq, s.Hkv, s.d, s.qblk, s.nblk,
                                  s.topk, isd, idx, scores);
  } else {
    auto kern = select_kernel<float>;
    if ((e = smem_limit(reinterpret_cast<const void*>(kern), smem)) != cudaSuccess)
      return e;
    kern<<<grid, kSelThreads, smem, st>>>(static_cast<const float*>(q), summ, s.S, s.Hq, s.Hkv, s.d, s.qblk, s.nblk, s.topk,
                                  isd, idx, scores);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_select(const Shape& s, int nq, const void* q_new, const float* summ, int32_t* idx,
                                 float* scores, void* ws, cudaStream_t st) {
  unsigned long long* keys = static_cast<unsigned long long*>(ws);
  const float isd = 1.0f / sqrtf((float)s.d);
  cudaError_t e;
  if (s.nblk > 0) {
    const int per_cta = kDecScoreWarps * kDecBlocksPerWarp;
    const dim3 grid((s.nblk + per_cta - 1) / per_cta, s.Hkv, s.B);
    const size_t smem = (size_t)s.G() * s.d * sizeof(float);
    if (s.bf16) {
      if ((e = smem_limit(reinterpret_cast<const void*>(decode_score_kernel<__nv_bfloat16>), smem)) != cudaSuccess)
        return e;
      decode_score_kernel<__nv_bfloat16><<<grid, kDecScoreWarps * 32, smem, st>>>(
          static_cast<const __nv_bfloat16*>(q_new), summ, nq, s.Hq, s.Hkv, s.d, s.nblk, isd, keys);
    } else {
      if ((e = smem_limit(reinterpret_cast<const void*>(decode_score_kernel<float>), smem)) != cudaSuccess)
        return e;
      decode_score_kernel<float><<<grid, kDecScoreWarps * 32, smem, st>>>(static_cast<const float*>(q_new), summ,
                                                                          nq, s.Hq, s.Hkv, s.d, s.nblk, isd, keys);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t smem = (size_t)(s.nblk > 0 ? s.nblk : 1) * 8;
  if ((e = smem_limit(reinterpret_cast<const void*>(decode_topk_kernel), smem)) !=
      cudaSuccess)
    return e;
  decode_topk_kernel<<<dim3(s.Hkv, s.B), kSelThreads, smem, st>>>(keys, s.Hkv, s.nblk, s.topk, idx, scores);
  return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(const Shape& s, const void* o, const void* d_o, float* Dr, cudaStream_t st) {
  const int rows = s.B * s.S * s.Hq;
  const int rows_per_cta = 8 * (32 * (s.bf16 ? 8 : 4) / s.d) * kPreRows;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  // at most the CTAs that are resident at once (4 per SM); the warps then stride over the rows
  const int grid = std::max(1, std::min((rows + rows_per_cta - 1) / rows_per_cta, 4 * n_sm));
  if (s.bf16)
    preprocess_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                           static_cast<const __nv_bfloat16*>(d_o), s.S, s.Hq, s.d,
                                                           rows, Dr);
  else
    preprocess_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(o), static_cast<const float*>(d_o), s.S,
                                                   s.Hq, s.d, rows, Dr);
  return cudaGetLastError();
}

}  // namespace hga

namespace hga {
cudaError_t launch_remap_idx(const Shape& s, const int32_t* idx, const int32_t* slot_of_block, int32_t* idx_pool,
                             int* err, cudaStream_t st) {
  const size_t n = (size_t)s.B * s.Hkv * s.nqb() * s.topk;
  if (n == 0) return cudaSuccess;
  remap_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(idx, slot_of_block, s.nblk, n, idx_pool, err);
  return cudaGetLastError();
}
}  // namespace hga

// ------------------------------------------------------------ zero-copy gather
// The distinct blocks selected in idx, copied from a pinned host tier mapped
// into the device's address space straight into a compact pool (slot k = the
// k-th smallest selected block), with idx rewritten to slots: the whole fetch
// runs on the device, ordered on the stream, with no host round trip.  Every
// CTA derives the same plan from idx (a bitmap of the selected blocks in
// shared memory and its prefix counts), then copies its share of (slot,
// 16 KB piece) work items with 16-byte loads from host memory; CTA 0 also
// writes idx_pool.  Blocks ranked at or beyond pool_slots get no slot: their
// entries become -1 and the device error flag is raised.
namespace hga {
namespace {

constexpr int kGatherThreads = 512;
constexpr int kGatherPiece = 16384;  // bytes per work item

__global__ void __launch_bounds__(kGatherThreads) gather_mapped_kernel(
    const int32_t* __restrict__ idx, size_t n_idx, int nblk, int B, size_t blk_bytes, int host_cap,
    const uint8_t* __restrict__ host_k, const uint8_t* __restrict__ host_v, uint8_t* __restrict__ pool_k,
    uint8_t* __restrict__ pool_v, int pool_slots, int32_t* __restrict__ idx_pool, int* err) {
  extern __shared__ uint32_t gbits[];  // [W] bitmap, then [W] exclusive prefix counts
  const int W = (nblk + 31) / 32;
  uint32_t* pre = gbits + W;
  __shared__ int s_total;
  const int tid = threadIdx.x;
  for (int w = tid; w < W; w += kGatherThreads) gbits[w] = 0u;
  __syncthreads();
  for (size_t k = tid; k < n_idx; k += kGatherThreads) {
    const int n = idx[k];
    if (n >= 0 && n < nblk) atomicOr(&gbits[n >> 5], 1u << (n & 31));
  }
  __syncthreads();
  if (tid == 0) {  // W <= 1024 words: a plain scan by one thread
    uint32_t run = 0;
    for (int w = 0; w < W; ++w) {
      pre[w] = run;
      run += __popc(gbits[w]);
    }
    s_total = (int)run;
  }
  __syncthreads();
  const int n_unique = s_total;
  if (blockIdx.x == 0) {
    for (size_t k = tid; k < n_idx; k += kGatherThreads) {
      const int n = idx[k];
      int slot = -1;
      if (n >= 0) {
        if (n < nblk) {
          slot = (int)(pre[n >> 5] + __popc(gbits[n >> 5] & ((1u << (n & 31)) - 1u)));
          if (slot >= pool_slots) slot = -1;
        }
        if (slot < 0) flag_error(err, kDevErrIndex);
      }
      idx_pool[k] = slot;
    }
  }
  // work items: (slot, batch, tensor, piece)
  const int pieces = (int)((blk_bytes + kGatherPiece - 1) / kGatherPiece);
  const int n_copy = n_unique < pool_slots ? n_unique : pool_slots;
  const long long items = (long long)n_copy * B * 2 * pieces;
  for (long long it = blockIdx.x; it < items; it += gridDim.x) {
    const int piece = (int)(it % pieces);
    const int tensor = (int)((it / pieces) % 2);
    const int b = (int)((it / pieces / 2) % B);
    const int slot = (int)(it / pieces / 2 / B);
    // block of this slot: the slot-th set bit (binary search over the prefix counts)
    int lo = 0, hi = W - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int)pre[mid] <= slot) lo = mid; else hi = mid - 1;
    }
    uint32_t word = gbits[lo];
    for (int r = slot - (int)pre[lo]; r > 0; --r) word &= word - 1u;  // drop the lower set bits
    const int n = lo * 32 + (__ffs(word) - 1);
    const size_t off = (size_t)piece * kGatherPiece;
    const size_t len = blk_bytes - off < (size_t)kGatherPiece ? blk_bytes - off : (size_t)kGatherPiece;
    const uint4* src = reinterpret_cast<const uint4*>((tensor ? host_v : host_k) +
                                                      ((size_t)b * host_cap + n) * blk_bytes + off);
    uint4* dst = reinterpret_cast<uint4*>((tensor ? pool_v : pool_k) + ((size_t)b * pool_slots + slot) * blk_bytes + off);
    const int nv = (int)(len / 16);
    // every load of the piece in flight before the stores
    uint4 v[kGatherPiece / 16 / kGatherThreads];
#pragma unroll
    for (int x = 0; x < kGatherPiece / 16 / kGatherThreads; ++x) {
      const int e = tid + x * kGatherThreads;
      if (e < nv) v[x] = src[e];
    }
#pragma unroll
    for (int x = 0; x < kGatherPiece / 16 / kGatherThreads; ++x) {
      const int e = tid + x * kGatherThreads;
      if (e < nv) dst[e] = v[x];
    }
  }
}

}  // namespace

int gather_max_blocks() { return 1024 * 32; }

cudaError_t launch_gather_mapped(const Shape& s, const int32_t* idx, const void* host_k_dev, const void* host_v_dev,
                                 int host_cap, void* pool_k, void* pool_v, int pool_slots, int32_t* idx_pool,
                                 int* err, int n_sm, cudaStream_t st) {
  const size_t n_idx = (size_t)s.B * s.Hkv * s.nqb() * s.topk;
  if (n_idx == 0) return cudaSuccess;
  const int W = (s.nblk + 31) / 32;
  const size_t smem = (size_t)2 * (W > 0 ? W : 1) * sizeof(uint32_t);
  const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * (s.bf16 ? 2 : 4);
  cudaError_t e = smem_limit(reinterpret_cast<const void*>(gather_mapped_kernel), smem);
  if (e != cudaSuccess) return e;
  gather_mapped_kernel<<<2 * n_sm, kGatherThreads, smem, st>>>(
      idx, n_idx, s.nblk, s.B, blk_bytes, host_cap, static_cast<const uint8_t*>(host_k_dev),
      static_cast<const uint8_t*>(host_v_dev), static_cast<uint8_t*>(pool_k), static_cast<uint8_t*>(pool_v), pool_slots,
      idx_pool, err);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- idx to host
// n int32 words from device memory into pinned host memory mapped into the
// device (dst is the device view), by SM stores.  A transfer this small then
// never waits in a copy engine's queue behind large copies of the same
// direction (a finished segment's K/V going to the host tier).  Each thread
// fences at system scope before it exits, so the words are visible to the host
// once the stream has passed the kernel.
__global__ void __launch_bounds__(256) store_mapped_i32_kernel(const int32_t* __restrict__ src, int32_t* dst,
                                                               size_t n) {
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (size_t)gridDim.x * blockDim.x)
    dst[k] = __ldg(src + k);
  __threadfence_system();
}

cudaError_t launch_store_mapped_i32(const int32_t* src, int32_t* dst_dev_view, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int blocks = (int)std::min<size_t>((n + 255) / 256, 32);
  store_mapped_i32_kernel<<<blocks, 256, 0, st>>>(src, dst_dev_view, n);
  return cudaGetLastError();
}

}  // namespace hga
