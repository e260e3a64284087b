// Tensor-core (tcgen05) backward of the HGA attention step for the active
// segment, bf16 in, fp32 accumulate, d = 128, 128-token blocks.
//
// Article: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global Attention
// and Segmented Backpropagation in Practice", Background and (fr edition)
// Analyse approfondie: only the active segment is differentiable; the KV of
// earlier segments is decoupled from the active graph.  So the history gets
// no gradient, and dK/dV exist only for segment keys; dQ sums over the
// history tiles and the causal segment tiles.
//
// With P recomputed from the forward's log-sum-exp and Dr = rowsum(dO * O):
//   dS = P * (dO V^T - Dr),  dQ = dS K / sqrt(d),
//   dK = dS^T Q / sqrt(d),   dV = P^T dO   (segment keys, summed over heads)
//
// Kernel 1 (dq_tc_kernel), one CTA per (b, query head, query block i), walks
// the same tile list as the forward (selected history blocks, then segment
// blocks 0..i).  Tensor memory: S double buffer | dP | dQ.  Per tile:
// S = Q K^T, dP = dO V^T (tensor core); dS (CUDA cores, two warpgroups, 64
// key columns each) is written as bf16 over the S columns it came from;
// dQ += dS K with dS read from tensor memory.  S runs two tiles ahead and dP
// one tile ahead of the dS pass.
//
// Kernel 2 (dkdv_tc_kernel), one CTA per (b, KV head, segment key block jb,
// query head of the group), walks query blocks i >= jb.  It computes the
// transposed products (keys in tensor-memory lanes): S^T = K Q^T,
// dP^T = V dO^T, then P^T and dS^T in place as bf16, and accumulates
// dV += P^T dO, dK += dS^T Q in tensor memory.  Each CTA adds its head's
// partial dK/dV to the fp32 outputs with vector atomics.
#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

constexpr int kB = 128;  // rows / keys per tile
constexpr int kD = 128;
constexpr int kTileBytes = kB * kD * 2;
constexpr int kHalf = kTileBytes / 2;
constexpr int kMaxTiles = kMaxTopk + kMaxQueryBlocks;
constexpr float kLog2e = 1.4426950408889634f;

// ============================================================== dQ kernel
constexpr int kKStages = 3, kVStages = 2;

struct DqCtl {
  uint64_t qdo_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t sdp_full, ds_full, dq_full, mma_done;
  uint32_t tmem;
  int abort;
  int nt;
  int tiles[kMaxTiles];
};
constexpr size_t kDqSmem = 1024 + (2 + kKStages + kVStages) * kTileBytes + sizeof(DqCtl);
static_assert(kDqSmem <= 232448, "shared memory budget");

struct BwdArgs {
  int B, Hq, Hkv, S, nkv, topk, nqb, G;
  float sl2;    // log2(e)/sqrt(d)
  float scale;  // 1/sqrt(d)
  const int32_t* idx;
  const float* lse;
  const float* Dr;
  float* dq;
  float* dk;
  float* dv;
  int* err;
};

__global__ void __launch_bounds__(320, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                 const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_vh,
                 const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;
  uint8_t* sDO = sm + kTileBytes;
  uint8_t* sK = sm + 2 * kTileBytes;
  uint8_t* sV = sK + kKStages * kTileBytes;
  DqCtl* ctl = reinterpret_cast<DqCtl*>(sV + kVStages * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_i = a.B * a.Hq;
  const int i = a.nqb - 1 - (int)(blockIdx.x / per_i);
  const int rem = (int)(blockIdx.x % per_i);
  const int b = rem / a.Hq, hq = rem % a.Hq;
  const int kvh = hq / a.G;

  if (warp == 0) {
    const int32_t* row = a.idx + (((size_t)b * a.Hkv + kvh) * a.nqb + i) * a.topk;
    int nh = 0;
    for (int base = 0; base < a.topk; base += 32) {
      const int r = base + lane;
      const int n = (r < a.topk) ? __ldg(row + r) : -1;
      const bool ok = (n >= 0 && n < a.nkv);
      if (r < a.topk && !ok && n != -1) flag_error(a.err, kDevErrIndex);
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      if (ok) ctl->tiles[nh + __popc(m & ((1u << lane) - 1u))] = n;
      nh += __popc(m);
    }
    for (int jb = lane; jb <= i; jb += 32) ctl->tiles[nh + jb] = -(jb + 1);
    if (lane == 0) {
      ctl->nt = nh + i + 1;
      ctl->abort = 0;
      mbar_init(&ctl->qdo_full, 1);
      for (int s = 0; s < kKStages; ++s) { mbar_init(&ctl->k_full[s], 1); mbar_init(&ctl->k_empty[s], 1); }
      for (int s = 0; s < kVStages; ++s) { mbar_init(&ctl->v_full[s], 1); mbar_init(&ctl->v_empty[s], 1); }
      mbar_init(&ctl->sdp_full, 1);
      mbar_init(&ctl->ds_full, 256);
      mbar_init(&ctl->dq_full, 1);
      mbar_init(&ctl->mma_done, 1);
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(&ctl->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  const int nt = ctl->nt;
  volatile int* abort = &ctl->abort;

  if (warp == 8) {
    if (lane == 0) {
      mbar_expect_tx(&ctl->qdo_full, 2 * kTileBytes);
      for (int hh = 0; hh < 2; ++hh) {
        tma_load_4d(&tm_q, &ctl->qdo_full, sQ + hh * kHalf, hh * 64, hq, i * kB, b);
        tma_load_4d(&tm_do, &ctl->qdo_full, sDO + hh * kHalf, hh * 64, hq, i * kB, b);
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int tile = ctl->tiles[j];
        const bool hist = tile >= 0;
        const int row0 = (hist ? tile : (-tile - 1)) * kB;
        const int ks = j % kKStages, vs = j % kVStages;
        if (!mbar_wait(&ctl->k_empty[ks], ((j / kKStages) & 1) ^ 1, abort, a.err)) break;
        mbar_expect_tx(&ctl->k_full[ks], kTileBytes);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_4d(hist ? &tm_kh : &tm_ks, &ctl->k_full[ks], sK + ks * kTileBytes + hh * kHalf, hh * 64, kvh,
                      row0, b);
        k_issued = j + 1;
        if (!mbar_wait(&ctl->v_empty[vs], ((j / kVStages) & 1) ^ 1, abort, a.err)) break;
        mbar_expect_tx(&ctl->v_full[vs], kTileBytes);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_4d(hist ? &tm_vh : &tm_vs, &ctl->v_full[vs], sV + vs * kTileBytes + hh * kHalf, hh * 64, kvh,
                      row0, b);
        v_issued = j + 1;
      }
      volatile int no_abort = 0;
      mbar_wait(&ctl->qdo_full, 0, &no_abort, a.err);
      for (int j = k_issued > kKStages ? k_issued - kKStages : 0; j < k_issued; ++j)
        mbar_wait(&ctl->k_full[j % kKStages], (j / kKStages) & 1, &no_abort, a.err);
      for (int j = v_issued > kVStages ? v_issued - kVStages : 0; j < v_issued; ++j)
        mbar_wait(&ctl->v_full[j % kVStages], (j / kVStages) & 1, &no_abort, a.err);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(kB, kB, false, false);
      constexpr uint32_t kIdQ = idesc_bf16(kB, kD, false, true);
      const uint32_t sq = smem_u32(sQ), sdo = smem_u32(sDO), sk = smem_u32(sK), sv = smem_u32(sV);
      auto kmajor = [&](uint32_t A, uint32_t Bm, uint32_t d_col) {
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + d_col, sdesc_sw128(A + off, 16, 1024), sdesc_sw128(Bm + off, 16, 1024), kIdS, kk > 0);
        }
      };
      auto wait_k = [&](int j) { return mbar_wait(&ctl->k_full[j % kKStages], (j / kKStages) & 1, abort, a.err); };
      auto wait_v = [&](int j) { return mbar_wait(&ctl->v_full[j % kVStages], (j / kVStages) & 1, abort, a.err); };
      bool ok = mbar_wait(&ctl->qdo_full, 0, abort, a.err) && wait_k(0) && wait_v(0);
      if (ok) {
        tc_fence_after();
        kmajor(sq, sk, 0);                       // S(0) -> buffer 0
        kmajor(sdo, sv, 256);                    // dP(0)
        umma_commit(&ctl->sdp_full);
        umma_commit(&ctl->v_empty[0]);
        if (nt > 1) {
          ok = wait_k(1);
          if (ok) {
            tc_fence_after();
            kmajor(sq, sk + (1 % kKStages) * kTileBytes, 128);  // S(1) -> buffer 1
          }
        }
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (!mbar_wait(&ctl->ds_full, j & 1, abort, a.err)) break;
        tc_fence_after();
        const uint32_t sb = (uint32_t)(j & 1) * 128;
        const uint32_t kslot = sk + (j % kKStages) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kB / 16; ++kk) {
          const uint32_t pcol = (kk >> 1) * 32 + (kk & 1) * 8;
          umma_ts(tmem + 384, tmem + sb + pcol, sdesc_sw128(kslot + kk * 2048, kHalf, 1024), kIdQ,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&ctl->k_empty[j % kKStages]);
        if (j + 1 < nt) {
          if (!wait_v(j + 1)) break;
          tc_fence_after();
          kmajor(sdo, sv + ((j + 1) % kVStages) * kTileBytes, 256);
          umma_commit(&ctl->sdp_full);
          umma_commit(&ctl->v_empty[(j + 1) % kVStages]);
        }
        if (j + 2 < nt) {
          if (!wait_k(j + 2)) break;
          tc_fence_after();
          kmajor(sq, sk + ((j + 2) % kKStages) * kTileBytes, sb);
        }
        if (j == nt - 1) umma_commit(&ctl->dq_full);
      }
      umma_commit(&ctl->mma_done);
      volatile int no_abort = 0;
      mbar_wait(&ctl->mma_done, 0, &no_abort, a.err);
    }
  } else {
    // ------------------------------------------------------------ dS pass
    const int e = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;
    const int p = i * kB + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const size_t rrow = ((size_t)b * a.Hq + hq) * a.S + p;
    const float lse2 = __ldg(a.lse + rrow) * kLog2e;
    const float Dv = __ldg(a.Dr + rrow);
    const float sl2 = a.sl2;
    bool ok = true;
    uint32_t sv[32], dv[32];
    for (int j = 0; j < nt; ++j) {
      // tcgen05.ld/st are warp-collective: branches around them are warp-uniform.
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl->sdp_full, j & 1, abort, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = (j == nt - 1);
      const uint32_t sb = (uint32_t)(j & 1) * 128;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * e + cc;
        HGA_TMEM_LD32_WAIT(tmem + lane_off + sb + c * 32, sv);
        HGA_TMEM_LD32_WAIT(tmem + lane_off + 256 + c * 32, dv);
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const bool k0 = !diag || c * 32 + x <= r;
          const bool k1 = !diag || c * 32 + x + 1 <= r;
          const float p0 = k0 ? ex2_approx(fmaf(__uint_as_float(sv[x]), sl2, -lse2)) : 0.f;
          const float p1 = k1 ? ex2_approx(fmaf(__uint_as_float(sv[x + 1]), sl2, -lse2)) : 0.f;
          pk[x >> 1] = pack_bf16x2(p0 * (__uint_as_float(dv[x]) - Dv), p1 * (__uint_as_float(dv[x + 1]) - Dv));
        }
        HGA_TMEM_ST16(tmem + lane_off + sb + c * 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl->ds_full);
    }
    if (__all_sync(0xffffffffu, ok && mbar_wait(&ctl->dq_full, 0, abort, a.err))) {
      tc_fence_after();
      float* out = a.dq + (((size_t)b * a.S + p) * a.Hq + hq) * kD + 64 * e;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        HGA_TMEM_LD32_WAIT(tmem + lane_off + 384 + 64 * e + 32 * cc, sv);
        float4* dst = reinterpret_cast<float4*>(out + 32 * cc);
#pragma unroll
        for (int x = 0; x < 8; ++x)
          dst[x] = make_float4(__uint_as_float(sv[4 * x]) * a.scale, __uint_as_float(sv[4 * x + 1]) * a.scale,
                               __uint_as_float(sv[4 * x + 2]) * a.scale, __uint_as_float(sv[4 * x + 3]) * a.scale);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== dK/dV kernel
constexpr int kQStages = 2;

struct DkvCtl {
  uint64_t kv_full;
  uint64_t qd_full[kQStages], qd_empty[kQStages];
  uint64_t sdp_full, pds_full, dkv_full, mma_done;
  uint32_t tmem;
  int abort;
};
struct __align__(16) RowStats {
  float lse[kB];
  float D[kB];
};
constexpr size_t kDkvSmem = 1024 + (2 + 2 * kQStages) * kTileBytes + kQStages * sizeof(RowStats) + sizeof(DkvCtl);
static_assert(kDkvSmem <= 232448, "shared memory budget");

__global__ void __launch_bounds__(320, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                   const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sK = sm;
  uint8_t* sV = sm + kTileBytes;
  uint8_t* sQ = sm + 2 * kTileBytes;                         // kQStages tiles
  uint8_t* sDO = sQ + kQStages * kTileBytes;                 // kQStages tiles
  RowStats* stats = reinterpret_cast<RowStats*>(sDO + kQStages * kTileBytes);
  DkvCtl* ctl = reinterpret_cast<DkvCtl*>(stats + kQStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Longest first: key block jb ascending (it sees nqb - jb query blocks).
  const int per_jb = a.B * a.Hq;
  const int jb = (int)(blockIdx.x / per_jb);
  const int rem = (int)(blockIdx.x % per_jb);
  const int b = rem / a.Hq, hq = rem % a.Hq;
  const int kvh = hq / a.G;
  const int n = a.nqb - jb;  // query blocks jb..nqb-1

  if (warp == 0) {
    if (lane == 0) {
      ctl->abort = 0;
      mbar_init(&ctl->kv_full, 1);
      for (int s = 0; s < kQStages; ++s) { mbar_init(&ctl->qd_full[s], 1); mbar_init(&ctl->qd_empty[s], 1); }
      mbar_init(&ctl->sdp_full, 1);
      mbar_init(&ctl->pds_full, 256);
      mbar_init(&ctl->dkv_full, 1);
      mbar_init(&ctl->mma_done, 1);
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(&ctl->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem;
  volatile int* abort = &ctl->abort;

  if (warp == 8) {
    if (lane == 0) {
      mbar_expect_tx(&ctl->kv_full, 2 * kTileBytes);
      for (int hh = 0; hh < 2; ++hh) {
        tma_load_4d(&tm_ks, &ctl->kv_full, sK + hh * kHalf, hh * 64, kvh, jb * kB, b);
        tma_load_4d(&tm_vs, &ctl->kv_full, sV + hh * kHalf, hh * 64, kvh, jb * kB, b);
      }
      int issued = 0;
      for (int it = 0; it < n; ++it) {
        const int s = it % kQStages;
        const int i = jb + it;
        if (!mbar_wait(&ctl->qd_empty[s], ((it / kQStages) & 1) ^ 1, abort, a.err)) break;
        mbar_expect_tx(&ctl->qd_full[s], 2 * kTileBytes + sizeof(RowStats));
        for (int hh = 0; hh < 2; ++hh) {
          tma_load_4d(&tm_q, &ctl->qd_full[s], sQ + s * kTileBytes + hh * kHalf, hh * 64, hq, i * kB, b);
          tma_load_4d(&tm_do, &ctl->qd_full[s], sDO + s * kTileBytes + hh * kHalf, hh * 64, hq, i * kB, b);
        }
        const size_t r0 = ((size_t)b * a.Hq + hq) * a.S + (size_t)i * kB;
        bulk_load(stats[s].lse, a.lse + r0, kB * 4, &ctl->qd_full[s]);
        bulk_load(stats[s].D, a.Dr + r0, kB * 4, &ctl->qd_full[s]);
        issued = it + 1;
      }
      volatile int no_abort = 0;
      mbar_wait(&ctl->kv_full, 0, &no_abort, a.err);
      for (int it = issued > kQStages ? issued - kQStages : 0; it < issued; ++it)
        mbar_wait(&ctl->qd_full[it % kQStages], (it / kQStages) & 1, &no_abort, a.err);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t kIdT = idesc_bf16(kB, kB, false, false);  // K Q^T, V dO^T
      constexpr uint32_t kIdG = idesc_bf16(kB, kD, false, true);   // P^T dO, dS^T Q
      const uint32_t sk = smem_u32(sK), sv = smem_u32(sV), sq = smem_u32(sQ), sdo = smem_u32(sDO);
      auto kmajor = [&](uint32_t A, uint32_t Bm, uint32_t d_col) {
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + d_col, sdesc_sw128(A + off, 16, 1024), sdesc_sw128(Bm + off, 16, 1024), kIdT, kk > 0);
        }
      };
      auto tsmma = [&](uint32_t a_col, uint32_t Bm, uint32_t d_col, bool acc) {
#pragma unroll
        for (int kk = 0; kk < kB / 16; ++kk) {
          const uint32_t pcol = (kk >> 1) * 32 + (kk & 1) * 8;
          umma_ts(tmem + d_col, tmem + a_col + pcol, sdesc_sw128(Bm + kk * 2048, kHalf, 1024), kIdG,
                  (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&ctl->kv_full, 0, abort, a.err) && mbar_wait(&ctl->qd_full[0], 0, abort, a.err);
      if (ok) {
        tc_fence_after();
        kmajor(sk, sq, 0);
        kmajor(sv, sdo, 128);
        umma_commit(&ctl->sdp_full);
      }
      for (int it = 0; ok && it < n; ++it) {
        const int s = it % kQStages;
        if (!mbar_wait(&ctl->pds_full, it & 1, abort, a.err)) break;
        tc_fence_after();
        tsmma(0, sdo + s * kTileBytes, 384, it > 0);    // dV += P^T dO
        tsmma(128, sq + s * kTileBytes, 256, it > 0);   // dK += dS^T Q
        umma_commit(&ctl->qd_empty[s]);
        if (it + 1 < n) {
          const int s1 = (it + 1) % kQStages;
          if (!mbar_wait(&ctl->qd_full[s1], ((it + 1) / kQStages) & 1, abort, a.err)) break;
          tc_fence_after();
          kmajor(sk, sq + s1 * kTileBytes, 0);
          kmajor(sv, sdo + s1 * kTileBytes, 128);
          umma_commit(&ctl->sdp_full);
        } else {
          umma_commit(&ctl->dkv_full);
        }
      }
      umma_commit(&ctl->mma_done);
      volatile int no_abort = 0;
      mbar_wait(&ctl->mma_done, 0, &no_abort, a.err);
    }
  } else {
    // ------------------------------------------------------------ P^T / dS^T pass
    const int e = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // key row within block jb
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float sl2 = a.sl2;
    bool ok = true;
    uint32_t sv[32], dv[32];
    for (int it = 0; it < n; ++it) {
      const int s = it % kQStages;
      // The row statistics arrive with the Q/dO stage: observe that stage's
      // barrier directly (its phase is complete by now) before reading them.
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl->sdp_full, it & 1, abort, a.err) &&
                                       mbar_wait(&ctl->qd_full[s], (it / kQStages) & 1, abort, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = (it == 0);
      const RowStats& rs = stats[s];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * e + cc;
        HGA_TMEM_LD32_WAIT(tmem + lane_off + c * 32, sv);
        HGA_TMEM_LD32_WAIT(tmem + lane_off + 128 + c * 32, dv);
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const int q0 = c * 32 + x;  // query column within block i
          const bool k0 = !diag || q0 >= r;
          const bool k1 = !diag || q0 + 1 >= r;
          const float p0 = k0 ? ex2_approx(fmaf(__uint_as_float(sv[x]), sl2, -rs.lse[q0] * kLog2e)) : 0.f;
          const float p1 = k1 ? ex2_approx(fmaf(__uint_as_float(sv[x + 1]), sl2, -rs.lse[q0 + 1] * kLog2e)) : 0.f;
          pp[x >> 1] = pack_bf16x2(p0, p1);
          pd[x >> 1] = pack_bf16x2(p0 * (__uint_as_float(dv[x]) - rs.D[q0]),
                                   p1 * (__uint_as_float(dv[x + 1]) - rs.D[q0 + 1]));
        }
        HGA_TMEM_ST16(tmem + lane_off + c * 32, pp);
        HGA_TMEM_ST16(tmem + lane_off + 128 + c * 32, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl->pds_full);
    }
    if (__all_sync(0xffffffffu, ok && mbar_wait(&ctl->dkv_full, 0, abort, a.err))) {
      tc_fence_after();
      const size_t off = (((size_t)b * a.S + (size_t)jb * kB + r) * a.Hkv + kvh) * kD + 64 * e;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        HGA_TMEM_LD32_WAIT(tmem + lane_off + 256 + 64 * e + 32 * cc, sv);
        HGA_TMEM_LD32_WAIT(tmem + lane_off + 384 + 64 * e + 32 * cc, dv);
        float4* gk = reinterpret_cast<float4*>(a.dk + off + 32 * cc);
        float4* gv = reinterpret_cast<float4*>(a.dv + off + 32 * cc);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          atomicAdd(gk + x, make_float4(__uint_as_float(sv[4 * x]) * a.scale, __uint_as_float(sv[4 * x + 1]) * a.scale,
                                        __uint_as_float(sv[4 * x + 2]) * a.scale,
                                        __uint_as_float(sv[4 * x + 3]) * a.scale));
          atomicAdd(gv + x, make_float4(__uint_as_float(dv[4 * x]), __uint_as_float(dv[4 * x + 1]),
                                        __uint_as_float(dv[4 * x + 2]), __uint_as_float(dv[4 * x + 3])));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, const float* lse,
                               const float* Dr, float* dq, float* dk, float* dv, int parts, int* err,
                               cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDqSmem)) !=
      cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDkvSmem)) !=
      cudaSuccess)
    return e;
  BwdArgs a;
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.S = s.S; a.nkv = nkv; a.topk = s.topk; a.nqb = s.nqb(); a.G = s.G();
  a.scale = 1.0f / sqrtf((float)kD);
  a.sl2 = kLog2e * a.scale;
  a.idx = idx; a.lse = lse; a.Dr = Dr; a.dq = dq; a.dk = dk; a.dv = dv; a.err = err;
  if (parts & kBwdDkdv) {
    // Per-head partials are added into the outputs: start from zero.
    const size_t kv_bytes = (size_t)s.B * s.S * s.Hkv * kD * sizeof(float);
    if ((e = cudaMemsetAsync(dk, 0, kv_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dv, 0, kv_bytes, st)) != cudaSuccess) return e;
    dkdv_tc_kernel<<<s.B * s.Hq * s.nqb(), 320, kDkvSmem, st>>>(m.q, m.d_o, m.ks, m.vs, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (parts & kBwdDq) {
    dq_tc_kernel<<<s.B * s.Hq * s.nqb(), 320, kDqSmem, st>>>(m.q, m.d_o, m.ks, m.vs, m.kh, m.vh, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hga
