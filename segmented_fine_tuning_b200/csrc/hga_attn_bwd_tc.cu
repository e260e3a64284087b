// Tensor-core (tcgen05) backward of the HGA attention step for the active
// segment, bf16 in, fp32 accumulate, d in {64, 128}, 128-row query blocks
// over history blocks of 128, 64, 32 or 16 tokens.
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
// the forward's tile list (selected history blocks, then segment blocks
// 0..i).  Tensor memory: S double buffer | dP | dQ (128 columns each).  Per
// tile: S = Q K^T and dP = dO V^T (M 128 queries, N 128 keys); dS (two
// warpgroups, 64 key columns each) is written as bf16 over the S columns it
// came from; dQ += dS K takes dS from tensor memory.  S runs two tiles ahead;
// dP's buffer is released as soon as the dS pass has loaded it, so dP(j+1)
// overlaps the dS math of tile j.  Each thread's dQ half row leaves through
// shared memory as one bulk copy.
//
// Kernel 2 works in 64-query sub-tiles so that tensor memory holds two
// sub-tiles of S^T and dP^T at once: while the CUDA cores turn sub-tile u into
// P^T and dS^T, the tensor core finishes the products of sub-tile u-1 and
// computes S^T and dP^T of sub-tile u+1.
//
// Kernel 2 (dkdv_tc_kernel), one CTA per (b, KV head, segment key block jb,
// query head of the group), walks query blocks i >= jb, each as two 64-query
// halves, with the transposed products (keys in tensor-memory lanes):
// S^T = K Q^T, dP^T = V dO^T (M 128 keys, N 64 queries), P^T and dS^T in
// place as bf16, dV += P^T dO and dK += dS^T Q (K = 64 queries) accumulated
// in tensor memory.  Each CTA adds its head's partial dK/dV to the zeroed fp32
// outputs: the rows go through shared memory and each thread adds its half
// rows with bulk reduce-adds (cp.reduce.async.bulk .add.f32).
#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

constexpr int kB = 128;  // rows / keys per tile
constexpr int kHalf = kB * 128;              // one 64-channel TMA box: 128 rows x 128 B
constexpr int kSubRows = 64;                 // rows of a sub-tile
constexpr int kSubOff = kSubRows * 128;      // byte offset of the second 64-row half inside a box
// History tiles of 64-token blocks hold two blocks: tile = n0 | (n1 << 16),
// n1 = kNoBlock when the tile's upper 64 keys have no block (an odd count).
constexpr int kNoBlock = 0x7FFF;
// History blocks of 32 or 16 tokens run in the grouped instantiation of the
// dQ kernel (kGrp): a tile holds g = 128 / block of them (four or eight), its
// entry is s | (c << 16), the tile's blocks are hb[s .. s+c) with c <= g, and
// the keys after the first c*block of a short last tile get P = 0.  Blocks of
// 128 and 64 tokens keep the plain kernel.
constexpr int kMaxTiles = kMaxTopk + kMaxQueryBlocks;
constexpr float kLog2e = 1.4426950408889634f;
// Pairs k (bit k) of every 32-column chunk whose 2^x goes to the FMA pipe
// (exp2_poly2) instead of the ex2 unit.  Measured on B200 with this
// kernel's two warps per scheduler: every split tried (4, 6 or 8 of 16
// pairs) was slower than none, so all pairs use the ex2 unit.
#ifndef HGA_BWD_POLY
#define HGA_BWD_POLY 0x0u
#endif
constexpr uint32_t kBwdPolyPairs = HGA_BWD_POLY;

// A bf16 chunk of 32 elements packed as 16 columns sits at the first 16 of
// the 32 fp32 columns it was computed from; k-step kk (16 elements) of a
// 64-element sub-tile therefore starts at column (kk / 2) * 32 + (kk % 2) * 8.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8); }

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
  // Sparse backward (SpaCO-style): only query blocks i with qmask[b*nqb + i]
  // != 0 propagate gradient, and every gradient is multiplied by gscale.
  // qmask == nullptr and gscale == 1: the plain backward.
  const uint8_t* qmask;
  float gscale;
  int hblk;  // history block tokens: 128 (one block per tile), 64 (two), 32 or 16 (grouped)
};

// ============================================================== dQ kernel
constexpr int kKStages = 3, kVStages = 2;

template <bool kGrp>
struct DqCtl {
  uint64_t qdo_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t sdp_full[2], ds_full[2];
  uint64_t dp_free;
  uint64_t dq_full, mma_done;
  uint32_t tmem;
  int abort;
  int nt;
  int tiles[kMaxTiles];  // >= 0: history block, pair or group; < 0: segment block -(t+1)
  int hb[kGrp ? kMaxTopk : 1];  // grouped: the valid selected history blocks, in idx order
};
// Head dim d in {64, 128}: a tile is 128 rows x d bf16 (d/64 TMA boxes).
template <bool kGrp>
constexpr size_t dq_smem_bytes(int d) {
  return 1024 + (2 + kKStages + kVStages) * (kB * d * 2) + sizeof(DqCtl<kGrp>);
}
static_assert(dq_smem_bytes<true>(128) <= 232448, "shared memory budget");

// Tensor-memory columns of the dQ kernel: S double buffer, dP, dQ.
constexpr uint32_t kDqS = 0, kDqP = 256, kDqAcc = 384;
// The dQ epilogue stages 2 x 128 half rows of d/2 + 4 floats in the tile buffers.
static_assert(2 * kB * (128 / 2 + 4) * 4 <= (2 + kKStages + kVStages) * kB * 128 * 2, "dQ stage fits");
static_assert(2 * kB * (64 / 2 + 4) * 4 <= (2 + kKStages + kVStages) * kB * 64 * 2, "dQ stage fits");

// dQ kernel: full 128-key tiles (N = 128 products: half the shared-memory
// re-reads of A per FLOP compared with 64-key halves).  S is double-buffered
// and runs two tiles ahead.  dP has one buffer, but the dS pass releases it as
// soon as it has loaded its columns (dp_free), so dP(j+1) is computed while
// dS(j) is being formed; dQ(j) follows dS(j).
template <int KD, bool kGrp>
__global__ void __launch_bounds__(320, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                 const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_vh,
                 const BwdArgs a) {
  constexpr int kD = KD;
  constexpr int kTileBytes = kB * kD * 2;
  constexpr int kBoxes = kD / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;
  uint8_t* sDO = sm + kTileBytes;
  uint8_t* sK = sm + 2 * kTileBytes;
  uint8_t* sV = sK + kKStages * kTileBytes;
  DqCtl<kGrp>* ctl = reinterpret_cast<DqCtl<kGrp>*>(sV + kVStages * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_i = a.B * a.Hq;
  const int i = a.nqb - 1 - (int)(blockIdx.x / per_i);  // longest tile lists first
  const int rem = (int)(blockIdx.x % per_i);
  const int b = rem / a.Hq, hq = rem % a.Hq;
  const int kvh = hq / a.G;
  if (a.qmask && !a.qmask[(size_t)b * a.nqb + i]) {
    // a query block that propagates no gradient: its dQ rows are zero
    for (int x = threadIdx.x; x < kB * kD / 4; x += blockDim.x) {
      const int r = x / (kD / 4), c4 = x % (kD / 4);
      reinterpret_cast<float4*>(a.dq + (((size_t)b * a.S + (size_t)i * kB + r) * a.Hq + hq) * kD)[c4] =
          make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }

  if (warp == 0) {
    const int32_t* row = a.idx + (((size_t)b * a.Hkv + kvh) * a.nqb + i) * a.topk;
    int nh = 0;
    for (int base = 0; base < a.topk; base += 32) {
      const int r = base + lane;
      const int n = (r < a.topk) ? __ldg(row + r) : -1;
      const bool ok = (n >= 0 && n < a.nkv);
      if (r < a.topk && !ok && n != -1) flag_error(a.err, kDevErrIndex);
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      if (ok) (kGrp ? ctl->hb : ctl->tiles)[nh + __popc(m & ((1u << lane) - 1u))] = n;
      nh += __popc(m);
    }
    if (kGrp) {
      // g consecutive list entries per tile (the last one may be short)
      const int g = kB / a.hblk;
      const int nht = (nh + g - 1) / g;
      for (int j = lane; j < nht; j += 32) ctl->tiles[j] = (j * g) | (min(g, nh - j * g) << 16);
      nh = nht;
    } else if (a.hblk == 64) {
      // 64-token history blocks: two per 128-key tile (nh <= 64, so one pass)
      __syncwarp();
      const int np = (nh + 1) >> 1;
      int packed = 0;
      if (lane < np) {
        const int n1 = (2 * lane + 1 < nh) ? ctl->tiles[2 * lane + 1] : kNoBlock;
        packed = ctl->tiles[2 * lane] | (n1 << 16);
      }
      __syncwarp();
      if (lane < np) ctl->tiles[lane] = packed;
      nh = np;
    }
    for (int jb = lane; jb <= i; jb += 32) ctl->tiles[nh + jb] = -(jb + 1);
    if (lane == 0) {
      ctl->nt = nh + i + 1;
      ctl->abort = 0;
      mbar_init(&ctl->qdo_full, 1);
      for (int s = 0; s < kKStages; ++s) { mbar_init(&ctl->k_full[s], 1); mbar_init(&ctl->k_empty[s], 1); }
      for (int s = 0; s < kVStages; ++s) { mbar_init(&ctl->v_full[s], 1); mbar_init(&ctl->v_empty[s], 1); }
      for (int x = 0; x < 2; ++x) { mbar_init(&ctl->sdp_full[x], 1); mbar_init(&ctl->ds_full[x], 256); }
      mbar_init(&ctl->dp_free, 256);
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
    // ------------------------------------------------------------ producer
    if (kGrp) {
      // Grouped history tiles: the whole warp.  Lane 0 waits for each slot
      // and arms it; lanes q < g then load block q of a history tile at once
      // (lane 0 alone a segment tile).
      const int g = kB / a.hblk;
      if (lane == 0) {
        mbar_expect_tx(&ctl->qdo_full, 2 * kTileBytes);
        for (int hh = 0; hh < kBoxes; ++hh) {
          tma_load_4d(&tm_q, &ctl->qdo_full, sQ + hh * kHalf, hh * 64, hq, i * kB, b);
          tma_load_4d(&tm_do, &ctl->qdo_full, sDO + hh * kHalf, hh * 64, hq, i * kB, b);
        }
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int tile = ctl->tiles[j];
        const bool hist = tile >= 0;
        // this lane's block of a history tile: a short tile repeats its last
        // block (finite values; those keys get P = 0 in the dS pass)
        const int row = hist ? ctl->hb[(tile & 0xFFFF) + min(lane, (tile >> 16) - 1)] * a.hblk : (-tile - 1) * kB;
        const bool loads = hist ? lane < g : lane == 0;
        const int sub = hist ? lane * a.hblk * 128 : 0;
        const int ks = j % kKStages, vs = j % kVStages;
        if (!mbar_wait_w(&ctl->k_empty[ks], ((j / kKStages) & 1) ^ 1, abort, a.err)) break;
        if (lane == 0) mbar_expect_tx(&ctl->k_full[ks], kTileBytes);
        __syncwarp();
        if (loads)
          for (int hh = 0; hh < kBoxes; ++hh)
            tma_load_4d(hist ? &tm_kh : &tm_ks, &ctl->k_full[ks], sK + ks * kTileBytes + hh * kHalf + sub, hh * 64,
                        kvh, row, b);
        k_issued = j + 1;
        if (!mbar_wait_w(&ctl->v_empty[vs], ((j / kVStages) & 1) ^ 1, abort, a.err)) break;
        if (lane == 0) mbar_expect_tx(&ctl->v_full[vs], kTileBytes);
        __syncwarp();
        if (loads)
          for (int hh = 0; hh < kBoxes; ++hh)
            tma_load_4d(hist ? &tm_vh : &tm_vs, &ctl->v_full[vs], sV + vs * kTileBytes + hh * kHalf + sub, hh * 64,
                        kvh, row, b);
        v_issued = j + 1;
      }
      if (lane == 0) {
        // Never leave the CTA with copies in flight (the slots' barriers
        // count every lane's bytes).
        volatile int no_abort = 0;
        mbar_wait(&ctl->qdo_full, 0, &no_abort, a.err);
        for (int j = k_issued > kKStages ? k_issued - kKStages : 0; j < k_issued; ++j)
          mbar_wait(&ctl->k_full[j % kKStages], (j / kKStages) & 1, &no_abort, a.err);
        for (int j = v_issued > kVStages ? v_issued - kVStages : 0; j < v_issued; ++j)
          mbar_wait(&ctl->v_full[j % kVStages], (j / kVStages) & 1, &no_abort, a.err);
      }
    } else if (lane == 0) {
      mbar_expect_tx(&ctl->qdo_full, 2 * kTileBytes);
      for (int hh = 0; hh < kBoxes; ++hh) {
        tma_load_4d(&tm_q, &ctl->qdo_full, sQ + hh * kHalf, hh * 64, hq, i * kB, b);
        tma_load_4d(&tm_do, &ctl->qdo_full, sDO + hh * kHalf, hh * 64, hq, i * kB, b);
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int tile = ctl->tiles[j];
        const bool hist = tile >= 0;
        const bool pair = hist && a.hblk == 64;
        const int row0 = pair ? (tile & 0xFFFF) * 64 : (hist ? tile : (-tile - 1)) * kB;
        // the upper half of a lone block's tile repeats it (finite values; its
        // keys get P = 0 in the dS pass)
        const int row1 = pair ? ((tile >> 16) == kNoBlock ? row0 : (tile >> 16) * 64) : 0;
        const int ks = j % kKStages, vs = j % kVStages;
        if (!mbar_wait(&ctl->k_empty[ks], ((j / kKStages) & 1) ^ 1, abort, a.err)) break;
        mbar_expect_tx(&ctl->k_full[ks], kTileBytes);
        for (int hh = 0; hh < kBoxes; ++hh) {
          uint8_t* dst = sK + ks * kTileBytes + hh * kHalf;
          tma_load_4d(hist ? &tm_kh : &tm_ks, &ctl->k_full[ks], dst, hh * 64, kvh, row0, b);
          if (pair) tma_load_4d(&tm_kh, &ctl->k_full[ks], dst + kSubOff, hh * 64, kvh, row1, b);
        }
        k_issued = j + 1;
        if (!mbar_wait(&ctl->v_empty[vs], ((j / kVStages) & 1) ^ 1, abort, a.err)) break;
        mbar_expect_tx(&ctl->v_full[vs], kTileBytes);
        for (int hh = 0; hh < kBoxes; ++hh) {
          uint8_t* dst = sV + vs * kTileBytes + hh * kHalf;
          tma_load_4d(hist ? &tm_vh : &tm_vs, &ctl->v_full[vs], dst, hh * 64, kvh, row0, b);
          if (pair) tma_load_4d(&tm_vh, &ctl->v_full[vs], dst + kSubOff, hh * 64, kvh, row1, b);
        }
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
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp: one elected lane issues
      constexpr uint32_t kIdS = idesc_bf16(kB, kB, false, false);  // [128 q x 128 keys] = Q K^T, dO V^T
      constexpr uint32_t kIdQ = idesc_bf16(kB, kD, false, true);   // dQ += dS (tmem) K (MN-major)
      // Descriptors built once; k-steps and ring slots are constant adds.
      const uint64_t dQd = sdesc_sw128(smem_u32(sQ), 16, 1024), dOd = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dKk = sdesc_sw128(smem_u32(sK), 16, 1024), dVk = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dKmn = sdesc_sw128(smem_u32(sK), kHalf, 1024);  // K as the MN-major B of dQ += dS K
      auto wait_k = [=](int j) { return mbar_wait_w(&ctl->k_full[j % kKStages], (j / kKStages) & 1, abort, a.err); };
      auto wait_v = [=](int j) { return mbar_wait_w(&ctl->v_full[j % kVStages], (j / kVStages) & 1, abort, a.err); };
      auto issue_s = [=](int j) {  // S(j) = Q K_j^T into buffer j % 2
        const uint64_t kb = dKk + sdesc_units((j % kKStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = sdesc_units((kk >> 2) * kHalf + (kk & 3) * 32);
          umma_ss_w(tmem + kDqS + (j & 1) * 128, dQd + off, kb + off, kIdS, kk > 0);
        }
      };
      auto issue_dp = [=](int j) {  // dP(j) = dO V_j^T
        const uint64_t vb = dVk + sdesc_units((j % kVStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = sdesc_units((kk >> 2) * kHalf + (kk & 3) * 32);
          umma_ss_w(tmem + kDqP, dOd + off, vb + off, kIdS, kk > 0);
        }
        umma_commit_w(&ctl->sdp_full[j & 1]);           // S(j) was issued earlier: both ready
        umma_commit_w(&ctl->v_empty[j % kVStages]);     // V_j's only reader
      };
      bool ok = mbar_wait_w(&ctl->qdo_full, 0, abort, a.err) && wait_k(0) && wait_v(0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        if (nt > 1) {
          ok = wait_k(1);
          if (ok) {
            tc_fence_after();
            issue_s(1);
          }
        }
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          // dP(j+1) as soon as the dS pass has read dP(j)
          if (!mbar_wait_w(&ctl->dp_free, j & 1, abort, a.err) || !wait_v(j + 1)) break;
          tc_fence_after();
          issue_dp(j + 1);
        }
        if (!mbar_wait_w(&ctl->ds_full[j & 1], (j >> 1) & 1, abort, a.err)) break;
        tc_fence_after();
        const uint64_t kb = dKmn + sdesc_units((j % kKStages) * kTileBytes);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kB / 16; ++kk)
          umma_ts_w(tmem + kDqAcc, tmem + kDqS + (j & 1) * 128 + packed_col(kk), kb + sdesc_units(kk * 2048), kIdQ,
                  kk > 0 ? 1u : acc0);
        umma_commit_w(&ctl->k_empty[j % kKStages]);  // K_j's last reader
        if (j + 2 < nt) {
          if (!wait_k(j + 2)) break;
          tc_fence_after();
          issue_s(j + 2);  // into buffer j % 2, after dQ(j) read dS(j) from it
        }
        if (j == nt - 1) umma_commit_w(&ctl->dq_full);
      }
      // All issued MMAs must finish before tensor memory is released.
      umma_commit_w(&ctl->mma_done);
      volatile int no_abort = 0;
      mbar_wait_w(&ctl->mma_done, 0, &no_abort, a.err);
    }
  } else {
    // ------------------------------------------------------------ dS pass
    const int e = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // query row within block i
    const int p = i * kB + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const size_t rrow = ((size_t)b * a.Hq + hq) * a.S + p;
    const float lse2 = __ldg(a.lse + rrow) * kLog2e;
    const float Dv = __ldg(a.Dr + rrow);
    const float2 s2 = make_float2(a.sl2, a.sl2), nl = make_float2(-lse2, -lse2), D2 = make_float2(Dv, Dv);
    bool ok = true;
    uint32_t sd[128];  // S columns [64e, 64e+64) of this row, then dP columns [64e, 64e+64)
    for (int j = 0; j < nt; ++j) {
      const int x = j & 1;
      // tcgen05.ld/st are warp-collective: branches around them are warp-uniform.
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl->sdp_full[x], (j >> 1) & 1, abort, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld64x2_wait(tmem + lane_off + kDqS + x * 128 + 64 * e, tmem + lane_off + kDqP + 64 * e, sd);
      tc_fence_before();
      mbar_arrive(&ctl->dp_free);  // dP(j) is in registers: the tensor core may overwrite it
      // keys above `lim` get P = 0: the diagonal segment tile masks keys after
      // the row's own position; a history tile holding one 64-token block
      // masks its upper 64 keys, a short grouped tile the keys after its blocks
      int lim = 127;
      if (j == nt - 1) lim = r;
      else if (!kGrp && a.hblk == 64 && ctl->tiles[j] >= 0 && (ctl->tiles[j] >> 16) == kNoBlock) lim = 63;
      else if (kGrp && ctl->tiles[j] >= 0) lim = (ctl->tiles[j] >> 16) * a.hblk - 1;
      const bool diag = lim < 127;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int xx = 0; xx < 32; xx += 2) {
          const int key = 64 * e + 32 * cc + xx;  // key column within the tile
          const float2 x = fma2(make_float2(__uint_as_float(sd[32 * cc + xx]), __uint_as_float(sd[32 * cc + xx + 1])),
                                s2, nl);
          float2 pr = exp2_pair(x, (kBwdPolyPairs >> (xx >> 1)) & 1u);
          if (diag) {
            pr.x = key <= lim ? pr.x : 0.f;
            pr.y = key + 1 <= lim ? pr.y : 0.f;
          }
          const float2 ds = mul2(pr, sub2(make_float2(__uint_as_float(sd[64 + 32 * cc + xx]),
                                                      __uint_as_float(sd[64 + 32 * cc + xx + 1])),
                                          D2));
          pk[xx >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        HGA_TMEM_ST16(tmem + lane_off + kDqS + x * 128 + 64 * e + 32 * cc, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl->ds_full[x]);
    }
    if (__all_sync(0xffffffffu, ok && mbar_wait(&ctl->dq_full, 0, abort, a.err))) {
      tc_fence_after();
      const float osc = a.scale * a.gscale;
      // Warpgroup e's half row (head-dim columns [e*d/2, (e+1)*d/2)) goes
      // through the freed tile buffers, rows padded to d/2 + 4 floats so that
      // a warp's 32 rows fall in distinct banks, and out as one bulk copy
      // (a warp's direct stores would each touch 32 rows).
      float* stage = reinterpret_cast<float*>(sm) + (size_t)(e * kB + r) * (kD / 2 + 4);
#pragma unroll
      for (int cc = 0; cc < kD / 64; ++cc) {
        uint32_t v[32];
        HGA_TMEM_LD32_WAIT(tmem + lane_off + kDqAcc + (kD / 2) * e + 32 * cc, v);
        float4* dst = reinterpret_cast<float4*>(stage + 32 * cc);
#pragma unroll
        for (int xx = 0; xx < 8; ++xx)
          dst[xx] = make_float4(__uint_as_float(v[4 * xx]) * osc, __uint_as_float(v[4 * xx + 1]) * osc,
                                __uint_as_float(v[4 * xx + 2]) * osc, __uint_as_float(v[4 * xx + 3]) * osc);
      }
      fence_proxy_async_smem();
      bulk_store(a.dq + (((size_t)b * a.S + p) * a.Hq + hq) * kD + (kD / 2) * e, stage, (kD / 2) * 4);
      bulk_commit();
      bulk_wait_read_all();  // the shared-memory source outlives the copy
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
  uint64_t sdp_full[2], pds_full[2];
  uint64_t dkv_full, mma_done;
  uint32_t tmem;
  int abort;
  int qblocks[kMaxQueryBlocks];  // query blocks i >= jb that propagate gradient, ascending
};
struct __align__(16) RowStats {
  float lse[kB];
  float D[kB];
};
constexpr size_t dkdv_smem_bytes(int d) {
  return 1024 + (2 + 2 * kQStages) * (kB * d * 2) + kQStages * sizeof(RowStats) + sizeof(DkvCtl);
}
static_assert(dkdv_smem_bytes(128) <= 232448, "shared memory budget");

// Tensor-memory columns of the dK/dV kernel.
constexpr uint32_t kKvS = 0, kKvP = 128, kKvDK = 256, kKvDV = 384;
// Row pitch (floats) of the fp32 dK/dV partials staged for the bulk
// reduction; the two [128 x pitch] partials reuse the kernel's tile buffers.
template <int KD>
constexpr int kv_pad() { return KD + 4; }
static_assert(2 * kB * kv_pad<128>() * 4 <= (2 + 2 * kQStages) * kB * 128 * 2, "partials fit the tile buffers");
static_assert(2 * kB * kv_pad<64>() * 4 <= (2 + 2 * kQStages) * kB * 64 * 2, "partials fit the tile buffers");

template <int KD>
__global__ void __launch_bounds__(320, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                   const BwdArgs a) {
  constexpr int kD = KD;
  constexpr int kTileBytes = kB * kD * 2;
  constexpr int kBoxes = kD / 64;
  constexpr int kPad = kv_pad<KD>();
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
  // query blocks jb..nqb-1 that propagate gradient (all of them unless sparse)
  int n = 0;
  for (int i = jb; i < a.nqb; ++i) n += (!a.qmask || a.qmask[(size_t)b * a.nqb + i]) ? 1 : 0;
  if (n == 0) return;  // no gradient reaches this key block from head hq (outputs start at zero)
  const int nsub = 2 * n;

  if (warp == 0) {
    if (lane == 0) {
      int c = 0;
      for (int i = jb; i < a.nqb; ++i)
        if (!a.qmask || a.qmask[(size_t)b * a.nqb + i]) ctl->qblocks[c++] = i;
      ctl->abort = 0;
      mbar_init(&ctl->kv_full, 1);
      for (int s = 0; s < kQStages; ++s) { mbar_init(&ctl->qd_full[s], 1); mbar_init(&ctl->qd_empty[s], 1); }
      for (int x = 0; x < 2; ++x) { mbar_init(&ctl->sdp_full[x], 1); mbar_init(&ctl->pds_full[x], 256); }
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(&ctl->kv_full, 2 * kTileBytes);
      for (int hh = 0; hh < kBoxes; ++hh) {
        tma_load_4d(&tm_ks, &ctl->kv_full, sK + hh * kHalf, hh * 64, kvh, jb * kB, b);
        tma_load_4d(&tm_vs, &ctl->kv_full, sV + hh * kHalf, hh * 64, kvh, jb * kB, b);
      }
      int issued = 0;
      for (int it = 0; it < n; ++it) {
        const int s = it % kQStages;
        const int i = ctl->qblocks[it];
        if (!mbar_wait(&ctl->qd_empty[s], ((it / kQStages) & 1) ^ 1, abort, a.err)) break;
        mbar_expect_tx(&ctl->qd_full[s], 2 * kTileBytes + sizeof(RowStats));
        for (int hh = 0; hh < kBoxes; ++hh) {
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
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp: one elected lane issues
      constexpr uint32_t kIdT = idesc_bf16(kB, kSubRows, false, false);  // [128 keys x 64 queries]
      constexpr uint32_t kIdG = idesc_bf16(kB, kD, false, true);         // dV += P^T dO_half, dK += dS^T Q_half
      // Descriptors built once; k-steps, query halves and stages are constant adds.
      const uint64_t dKd = sdesc_sw128(smem_u32(sK), 16, 1024), dVd = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024), dOk = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dQmn = sdesc_sw128(smem_u32(sQ), kHalf, 1024), dOmn = sdesc_sw128(smem_u32(sDO), kHalf, 1024);
      // S^T and dP^T of sub-tile u (query block jb + u/2, query half u%2) into buffer u%2.
      auto issue_sdp = [=](int u) -> bool {
        const int it = u >> 1, h = u & 1, s = it % kQStages;
        if (h == 0) {
          if (!mbar_wait_w(&ctl->qd_full[s], (it / kQStages) & 1, abort, a.err)) return false;
          tc_fence_after();
        }
        const uint32_t so = sdesc_units(s * kTileBytes + h * kSubOff);
        const uint64_t qb = dQk + so, ob = dOk + so;
        const uint32_t ts = tmem + kKvS + h * 64, tp = tmem + kKvP + h * 64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = sdesc_units((kk >> 2) * kHalf + (kk & 3) * 32);
          umma_ss_w(ts, dKd + off, qb + off, kIdT, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = sdesc_units((kk >> 2) * kHalf + (kk & 3) * 32);
          umma_ss_w(tp, dVd + off, ob + off, kIdT, kk > 0);
        }
        umma_commit_w(&ctl->sdp_full[h]);
        return true;
      };
      bool ok = mbar_wait_w(&ctl->kv_full, 0, abort, a.err);
      if (ok) {
        tc_fence_after();
        ok = issue_sdp(0) && issue_sdp(1);
      }
      for (int u = 0; ok && u < nsub; ++u) {
        const int it = u >> 1, h = u & 1, s = it % kQStages;
        if (!mbar_wait_w(&ctl->pds_full[h], (u >> 1) & 1, abort, a.err)) break;
        tc_fence_after();
        const uint32_t so = sdesc_units(s * kTileBytes + h * kSubOff);
        const uint64_t qb = dQmn + so, ob = dOmn + so;
        const uint32_t acc0 = u > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kSubRows / 16; ++kk)  // dV += P^T dO_half
          umma_ts_w(tmem + kKvDV, tmem + kKvS + h * 64 + packed_col(kk), ob + sdesc_units(kk * 2048), kIdG,
                  kk > 0 ? 1u : acc0);
#pragma unroll
        for (int kk = 0; kk < kSubRows / 16; ++kk)  // dK += dS^T Q_half
          umma_ts_w(tmem + kKvDK, tmem + kKvP + h * 64 + packed_col(kk), qb + sdesc_units(kk * 2048), kIdG,
                  kk > 0 ? 1u : acc0);
        if (h == 1) umma_commit_w(&ctl->qd_empty[s]);
        if (u + 2 < nsub) {
          if (!issue_sdp(u + 2)) break;
        }
        if (u == nsub - 1) umma_commit_w(&ctl->dkv_full);
      }
      umma_commit_w(&ctl->mma_done);
      volatile int no_abort = 0;
      mbar_wait_w(&ctl->mma_done, 0, &no_abort, a.err);
    }
  } else {
    // ------------------------------------------------------------ P^T / dS^T pass
    const int e = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // key row within block jb
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float2 s2 = make_float2(a.sl2, a.sl2), nlog2e = make_float2(-kLog2e, -kLog2e);
    bool ok = true;
    uint32_t sd[64];  // 32 S^T columns then 32 dP^T columns of this thread's key row
    for (int u = 0; u < nsub; ++u) {
      const int it = u >> 1, h = u & 1, s = it % kQStages;
      // The row statistics arrive with the Q/dO stage: observe that stage's
      // barrier directly (its phase is complete by now) before reading them.
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl->sdp_full[h], (u >> 1) & 1, abort, a.err) &&
                                       mbar_wait(&ctl->qd_full[s], (it / kQStages) & 1, abort, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = (ctl->qblocks[it] == jb);
      const RowStats& rs = stats[s];
      tmem_ld32x2_wait(tmem + lane_off + kKvS + h * 64 + 32 * e, tmem + lane_off + kKvP + h * 64 + 32 * e, sd);
      const int q0 = 64 * h + 32 * e;  // query column of sd[0] within block i
      uint32_t pp[16], pd[16];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        const int q = q0 + x;
        const float2 lq = *reinterpret_cast<const float2*>(&rs.lse[q]);  // same for every key row: broadcast
        const float2 dq2 = *reinterpret_cast<const float2*>(&rs.D[q]);
        const float2 arg = fma2(make_float2(__uint_as_float(sd[x]), __uint_as_float(sd[x + 1])), s2,
                                mul2(lq, nlog2e));
        float2 pr = exp2_pair(arg, (kBwdPolyPairs >> (x >> 1)) & 1u);
        if (diag) {
          pr.x = q >= r ? pr.x : 0.f;
          pr.y = q + 1 >= r ? pr.y : 0.f;
        }
        pp[x >> 1] = pack_bf16x2(pr.x, pr.y);
        const float2 ds = mul2(pr, sub2(make_float2(__uint_as_float(sd[32 + x]), __uint_as_float(sd[33 + x])), dq2));
        pd[x >> 1] = pack_bf16x2(ds.x, ds.y);
      }
      HGA_TMEM_ST16(tmem + lane_off + kKvS + h * 64 + 32 * e, pp);
      HGA_TMEM_ST16(tmem + lane_off + kKvP + h * 64 + 32 * e, pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl->pds_full[h]);
    }
    const bool done = __all_sync(0xffffffffu, ok && mbar_wait(&ctl->dkv_full, 0, abort, a.err));
    float* part = reinterpret_cast<float*>(sm);
    if (done) {
      tc_fence_after();
      // This head's scaled dK, dV into the tile buffers (no copy or MMA reads
      // them any more): part[t][row][col], rows padded to kPad floats so that
      // the 32 rows of a warp fall in distinct banks; warpgroup e writes
      // head-dim columns [e*d/2, (e+1)*d/2) of key row r.
      const float ks = a.scale * a.gscale, vsc = a.gscale;
#pragma unroll
      for (int cc = 0; cc < kD / 64; ++cc) {
        uint32_t gk[32], gv[32];
        HGA_TMEM_LD32_WAIT(tmem + lane_off + kKvDK + (kD / 2) * e + 32 * cc, gk);
        HGA_TMEM_LD32_WAIT(tmem + lane_off + kKvDV + (kD / 2) * e + 32 * cc, gv);
        float4* pk4 = reinterpret_cast<float4*>(part + r * kPad + (kD / 2) * e + 32 * cc);
        float4* pv4 = reinterpret_cast<float4*>(part + (kB + r) * kPad + (kD / 2) * e + 32 * cc);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          pk4[x] = make_float4(__uint_as_float(gk[4 * x]) * ks, __uint_as_float(gk[4 * x + 1]) * ks,
                               __uint_as_float(gk[4 * x + 2]) * ks, __uint_as_float(gk[4 * x + 3]) * ks);
          pv4[x] = make_float4(__uint_as_float(gv[4 * x]) * vsc, __uint_as_float(gv[4 * x + 1]) * vsc,
                               __uint_as_float(gv[4 * x + 2]) * vsc, __uint_as_float(gv[4 * x + 3]) * vsc);
        }
      }
    }
    if (done) {
      // Thread (e, r) adds the half rows it wrote into the zeroed outputs on
      // the bulk-copy engine.
      fence_proxy_async_smem();
      const size_t off = (((size_t)b * a.S + (size_t)jb * kB + r) * a.Hkv + kvh) * kD + (kD / 2) * e;
      bulk_reduce_add_f32(a.dk + off, part + r * kPad + (kD / 2) * e, (kD / 2) * 4);
      bulk_reduce_add_f32(a.dv + off, part + (kB + r) * kPad + (kD / 2) * e, (kD / 2) * 4);
      bulk_commit();
      bulk_wait_read_all();  // the shared-memory source outlives the copies
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

template <int KD, bool kGrp>
cudaError_t launch_bwd(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, const float* lse,
                       const float* Dr, float* dq, float* dk, float* dv, int parts, int* err, cudaStream_t st,
                       const uint8_t* qmask, float gscale) {
  constexpr size_t dq_smem = dq_smem_bytes<kGrp>(KD), kv_smem = dkdv_smem_bytes(KD);
  cudaError_t e;
  if ((e = smem_limit(reinterpret_cast<const void*>(dq_tc_kernel<KD, kGrp>), dq_smem)) !=
      cudaSuccess)
    return e;
  if ((e = smem_limit(reinterpret_cast<const void*>(dkdv_tc_kernel<KD>), kv_smem)) !=
      cudaSuccess)
    return e;
  BwdArgs a;
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.S = s.S; a.nkv = nkv; a.topk = s.topk; a.nqb = s.nqb(); a.G = s.G();
  a.scale = 1.0f / sqrtf((float)KD);
  a.sl2 = kLog2e * a.scale;
  a.idx = idx; a.lse = lse; a.Dr = Dr; a.dq = dq; a.dk = dk; a.dv = dv; a.err = err;
  a.qmask = qmask; a.gscale = gscale; a.hblk = s.blk;
  if (parts & kBwdDkdv) {
    // Per-head partials are added into the outputs: start from zero.
    const size_t kv_bytes = (size_t)s.B * s.S * s.Hkv * KD * sizeof(float);
    if ((e = cudaMemsetAsync(dk, 0, kv_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dv, 0, kv_bytes, st)) != cudaSuccess) return e;
    dkdv_tc_kernel<KD><<<s.B * s.Hq * s.nqb(), 320, kv_smem, st>>>(m.q, m.d_o, m.ks, m.vs, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (parts & kBwdDq) {
    dq_tc_kernel<KD, kGrp><<<s.B * s.Hq * s.nqb(), 320, dq_smem, st>>>(m.q, m.d_o, m.ks, m.vs, m.kh, m.vh, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_attn_bwd_tc(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, const float* lse,
                               const float* Dr, float* dq, float* dk, float* dv, int parts, int* err,
                               cudaStream_t st, const uint8_t* qmask, float gscale) {
  if (s.blk < 64)
    return s.d == 64 ? launch_bwd<64, true>(s, m, nkv, idx, lse, Dr, dq, dk, dv, parts, err, st, qmask, gscale)
                     : launch_bwd<128, true>(s, m, nkv, idx, lse, Dr, dq, dk, dv, parts, err, st, qmask, gscale);
  return s.d == 64 ? launch_bwd<64, false>(s, m, nkv, idx, lse, Dr, dq, dk, dv, parts, err, st, qmask, gscale)
                   : launch_bwd<128, false>(s, m, nkv, idx, lse, Dr, dq, dk, dv, parts, err, st, qmask, gscale);
}

}  // namespace hga
