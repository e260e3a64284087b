// Tensor-core (tcgen05) forward of the HGA attention step, bf16 in, fp32
// accumulate, for d in {64, 128}, 128-row query blocks and history blocks of
// 128, 64, 32 or 16 tokens.
//
// Article: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global Attention
// and Segmented Backpropagation in Practice", Background: each query block
// attends, exactly, to a bounded set of history tokens (the top-K blocks picked
// by summary score) plus the causal part of the active segment.
//
// Work unit (one CTA): batch b, KV head h, query block i, and a PAIR of query
// heads of h.  Both heads share the KV head and the query block, hence the
// same tile list: the K_eff selected history blocks followed by segment blocks
// 0..i (the last one, the diagonal, is causally masked).  Every K/V tile that
// TMA brings into shared memory feeds two 128x128x128 products.  Launches
// whose pairs would leave SMs idle use the split form instead: one head per
// CTA, its tiles alternating between the two softmax warpgroups (t takes
// tiles 2j + t), which merge their partial states at the end.
//
// Roles (384 threads, 1 CTA per SM):
//   warps 0-3   softmax for head 0 of the pair (split form: the even tiles),
//               one query row per thread
//   warps 4-7   softmax for head 1 (split form: the odd tiles)
//   warp  8     TMA producer: Q tiles once, then K_j, V_j into a 5-slot ring
//   warp  9     MMA issuer (one elected lane): S_t = Q_t K_j^T, O_t += P_t V_j
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1, 128 columns each, fp32.
// The softmax writes P (bf16) back into the S columns it has just read, and
// the PV product takes P straight from tensor memory.
//
// Online softmax in base 2 with a lazily updated reference maximum: the
// running reference m only moves (and O is rescaled in tensor memory) when a
// row's new maximum exceeds it by more than 8, so that P <= 2^8 stays exact
// in fp32/bf16 range while most tiles skip the rescale.
// MMA order per tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1).  Because tcgen05
// operations of one thread complete in order, the commit that announces
// S_t(j+1) also guarantees that PV_t(j) is done, which frees P_t and makes O_t
// safe to rescale.
#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

constexpr int kBM = 128;                      // query rows per tile
constexpr int kBN = 128;                      // keys per tile
constexpr int kHalf = kBM * 128;              // one 64-column TMA box: 128 rows x 128 bytes
constexpr int kRowHalf = 64 * 128;            // byte offset of row 64 inside a box
// History tiles of 64-token blocks hold two blocks: tile = n0 | (n1 << 16),
// n1 = kNoBlock when the tile's upper 64 keys have no block (an odd count).
constexpr int kNoBlock = 0x7FFF;
// History blocks of 32 or 16 tokens run in the grouped instantiation
// (kGrp): a tile holds g = 128 / block of them (four or eight), its entry is
// s | (c << 16), the tile's blocks are hb[s .. s+c) with c <= g, and the keys
// after the first c*block of a short last tile are masked.  Blocks of 128 and
// 64 tokens keep the plain kernel.
constexpr int kStages = 5;                    // K/V ring slots
constexpr int kMaxTiles = kMaxTopk + kMaxQueryBlocks;
constexpr float kRescaleThreshold = 8.0f;     // log2 units
// Pairs k (bit k) of every 32-column chunk whose 2^x goes to the FMA pipe
// (exp2_poly2) instead of the ex2 unit.  Measured on B200 with this
// kernel's two warps per scheduler: every split tried (4, 6 or 8 of 16
// pairs) was slower than none, so all pairs use the ex2 unit.
#ifndef HGA_FWD_POLY
#define HGA_FWD_POLY 0x0u
#endif
constexpr uint32_t kFwdPolyPairs = HGA_FWD_POLY;

template <bool kGrp>
struct FwdCtl {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t mma_done;
  uint64_t x_full;  // split form: warpgroup 1's row statistics are in shared memory
  uint32_t tmem;
  int abort;
  int nt;
  int tiles[kMaxTiles];  // >= 0: history block, pair or group; < 0: segment block -(t+1)
  int hb[kGrp ? kMaxTopk : 1];  // grouped: the valid selected history blocks, in idx order
};

// Head dim d in {64, 128}: a Q, K or V tile is 128 rows x d bf16 (d/64 boxes).
template <bool kGrp>
constexpr size_t fwd_smem_bytes(int d) {
  return 1024 + 2 * (kBM * d * 2) + kStages * (kBM * d * 2) + sizeof(FwdCtl<kGrp>);
}
static_assert(fwd_smem_bytes<true>(128) <= 232448, "shared memory budget");
// The O epilogue stages 2 x 128 rows of 2d + 16 bytes inside the Q tiles and ring slot 0.
static_assert(2 * kBM * (2 * 128 + 16) <= 3 * kBM * 128 * 2, "O stage fits");
static_assert(2 * kBM * (2 * 64 + 16) <= 3 * kBM * 64 * 2, "O stage fits");

struct FwdArgs {
  int B, Hq, Hkv, S, nkv, topk, nqb, G;
  float sl2;  // log2(e) / sqrt(d)
  const int32_t* idx;
  __nv_bfloat16* o;
  float* lse;
  int* err;
  int withhold_kv;  // self test of the timeout path: the producer issues no K/V loads
  int hblk;         // history block tokens: 128 (one block per tile), 64 (two), 32 or 16 (grouped)
};

template <int KD, bool kGrp, bool kTwo>
__global__ void __launch_bounds__(384, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ks,
                  const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ CUtensorMap tm_kh,
                  const __grid_constant__ CUtensorMap tm_vh, const FwdArgs a) {
  constexpr int kD = KD;                      // head dim
  constexpr int kTileBytes = kBM * kD * 2;    // bf16 tile: 32 KB at d = 128
  constexpr int kBoxes = kD / 64;             // 64-column TMA boxes per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;                                // 2 Q tiles
  uint8_t* sRing = sm + 2 * kTileBytes;            // kStages K/V tiles
  FwdCtl<kGrp>* ctl = reinterpret_cast<FwdCtl<kGrp>*>(sRing + kStages * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // kTwo: a CTA serves a pair of query heads; otherwise one head (launches
  // whose pairs would leave SMs idle), with the head-1 warps and products idle.
  constexpr int kHeads = kTwo ? 2 : 1;
  // Longest work first: query block i descending with blockIdx.
  const int nunit = a.G / kHeads;
  const int per_i = a.B * a.Hkv * nunit;
  const int i = a.nqb - 1 - (int)(blockIdx.x / per_i);
  const int rem = (int)(blockIdx.x % per_i);
  const int b = rem / (a.Hkv * nunit);
  const int kvh = (rem / nunit) % a.Hkv;
  const int hq0 = kvh * a.G + kHeads * (rem % nunit);

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
      const int g = kBN / a.hblk;
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
      mbar_init(&ctl->q_full, 1);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&ctl->kv_full[s], 1);
        mbar_init(&ctl->kv_empty[s], 1);
      }
      for (int t = 0; t < 2; ++t) {
        mbar_init(&ctl->s_full[t], 1);
        mbar_init(&ctl->p_full[t], 128);
        mbar_init(&ctl->o_full[t], 1);
      }
      mbar_init(&ctl->mma_done, 1);
      mbar_init(&ctl->x_full, 128);
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
      const int g = kBN / a.hblk;
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kh);
        prefetch_tmap(&tm_vh);
        prefetch_tmap(&tm_ks);
        prefetch_tmap(&tm_vs);
        mbar_expect_tx(&ctl->q_full, kHeads * kTileBytes);
        for (int t = 0; t < kHeads; ++t)
          for (int hh = 0; hh < kBoxes; ++hh)
            tma_load_4d(&tm_q, &ctl->q_full, sQ + t * kTileBytes + hh * kHalf, hh * 64, hq0 + t, i * kBM, b);
      }
      int issued = 0;
      for (int j = 0; j < (a.withhold_kv ? 0 : nt); ++j) {
        const int tile = ctl->tiles[j];
        const bool hist = tile >= 0;
        // this lane's block of a history tile: a short tile repeats its last
        // block (finite values; those keys are masked in the softmax)
        const int row = hist ? ctl->hb[(tile & 0xFFFF) + min(lane, (tile >> 16) - 1)] * a.hblk : (-tile - 1) * kBN;
        const bool loads = hist ? lane < g : lane == 0;
        const int sub = hist ? lane * a.hblk * 128 : 0;
        bool ok = true;
        for (int w = 0; w < 2; ++w) {
          const int pos = 2 * j + w;
          const int s = pos % kStages;
          if (!mbar_wait_w(&ctl->kv_empty[s], ((pos / kStages) & 1) ^ 1, abort, a.err)) {
            ok = false;
            break;
          }
          const CUtensorMap* m = hist ? (w ? &tm_vh : &tm_kh) : (w ? &tm_vs : &tm_ks);
          if (lane == 0) mbar_expect_tx(&ctl->kv_full[s], kTileBytes);
          __syncwarp();
          if (loads)
            for (int hh = 0; hh < kBoxes; ++hh)
              tma_load_4d(m, &ctl->kv_full[s], sRing + s * kTileBytes + hh * kHalf + sub, hh * 64, kvh, row, b);
          issued = pos + 1;
        }
        if (!ok) break;
      }
      if (lane == 0) {
        // Never leave the CTA with copies in flight (the slots' barriers
        // count every lane's bytes).
        volatile int no_abort = 0;
        mbar_wait(&ctl->q_full, 0, &no_abort, a.err);
        for (int pos = issued - kStages > 0 ? issued - kStages : 0; pos < issued; ++pos)
          mbar_wait(&ctl->kv_full[pos % kStages], (pos / kStages) & 1, &no_abort, a.err);
      }
    } else if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kh);
      prefetch_tmap(&tm_vh);
      prefetch_tmap(&tm_ks);
      prefetch_tmap(&tm_vs);
      mbar_expect_tx(&ctl->q_full, kHeads * kTileBytes);
      for (int t = 0; t < kHeads; ++t)
        for (int hh = 0; hh < kBoxes; ++hh)
          tma_load_4d(&tm_q, &ctl->q_full, sQ + t * kTileBytes + hh * kHalf, hh * 64, hq0 + t, i * kBM, b);
      int issued = 0;
      for (int j = 0; j < (a.withhold_kv ? 0 : nt); ++j) {
        const int tile = ctl->tiles[j];
        const bool hist = tile >= 0;
        const bool pair = hist && a.hblk == 64;
        const int row0 = pair ? (tile & 0xFFFF) * 64 : (hist ? tile : (-tile - 1)) * kBN;
        // the upper half of a lone block's tile repeats it (finite values; its
        // keys are masked in the softmax)
        const int row1 = pair ? ((tile >> 16) == kNoBlock ? row0 : (tile >> 16) * 64) : 0;
        bool ok = true;
        for (int w = 0; w < 2 && ok; ++w) {
          const int pos = 2 * j + w;
          const int s = pos % kStages;
          if (!mbar_wait(&ctl->kv_empty[s], ((pos / kStages) & 1) ^ 1, abort, a.err)) {
            ok = false;
            break;
          }
          const CUtensorMap* m = hist ? (w ? &tm_vh : &tm_kh) : (w ? &tm_vs : &tm_ks);
          mbar_expect_tx(&ctl->kv_full[s], kTileBytes);
          for (int hh = 0; hh < kBoxes; ++hh) {
            uint8_t* dst = sRing + s * kTileBytes + hh * kHalf;
            tma_load_4d(m, &ctl->kv_full[s], dst, hh * 64, kvh, row0, b);
            if (pair) tma_load_4d(m, &ctl->kv_full[s], dst + kRowHalf, hh * 64, kvh, row1, b);
          }
          issued = pos + 1;
        }
        if (!ok) break;
      }
      // Never leave the CTA with copies in flight: wait (bounded) for the
      // last loads issued into each slot and for Q.
      volatile int no_abort = 0;
      mbar_wait(&ctl->q_full, 0, &no_abort, a.err);
      for (int pos = issued - kStages > 0 ? issued - kStages : 0; pos < issued; ++pos)
        mbar_wait(&ctl->kv_full[pos % kStages], (pos / kStages) & 1, &no_abort, a.err);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp: one elected lane issues
      constexpr uint32_t kIdS = idesc_bf16(kBM, kBN, false, false);  // Q, K both K-major
      constexpr uint32_t kIdO = idesc_bf16(kBM, kD, false, true);    // P (tmem) x V (MN-major)
      // Descriptors are built once; every k-step and ring slot is a constant
      // add to the start-address field, so the issuing thread spends a few
      // cycles per tcgen05.mma instead of rebuilding descriptors.
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);          // Q tiles, K-major
      const uint64_t dK = sdesc_sw128(smem_u32(sRing), 16, 1024);       // ring as K tiles, K-major
      const uint64_t dV = sdesc_sw128(smem_u32(sRing), kHalf, 1024);    // ring as V tiles, MN-major
      auto issue_S = [=](int t, int s) {  // split form: both S buffers take the one Q tile
        const uint64_t a0 = dQ + sdesc_units((kTwo ? t : 0) * kTileBytes), b0 = dK + sdesc_units(s * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = sdesc_units((kk >> 2) * kHalf + (kk & 3) * 32);
          umma_ss_w(tmem + t * 128, a0 + off, b0 + off, kIdS, kk > 0);
        }
      };
      auto issue_PV = [=](int t, int s, bool acc) {
        const uint64_t b0 = dV + sdesc_units(s * kTileBytes);
        const uint32_t acc0 = acc ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // P chunk c (keys 32c..32c+31) sits at S columns [32c, 32c+16).
          const uint32_t pcol = (kk >> 1) * 32 + (kk & 1) * 8;
          umma_ts_w(tmem + 256 + t * 128, tmem + t * 128 + pcol, b0 + sdesc_units(kk * 2048), kIdO,
                  kk > 0 ? 1u : acc0);
        }
      };
      auto wait_full = [=](int pos) {
        return mbar_wait_w(&ctl->kv_full[pos % kStages], (pos / kStages) & 1, abort, a.err);
      };
      bool ok = mbar_wait_w(&ctl->q_full, 0, abort, a.err) && wait_full(0);
      if (ok && kTwo) {
        tc_fence_after();
        issue_S(0, 0);
        umma_commit_w(&ctl->s_full[0]);
        issue_S(1, 0);
        umma_commit_w(&ctl->s_full[1]);
        umma_commit_w(&ctl->kv_empty[0]);
        for (int j = 0; j < nt; ++j) {
          const int sV = (2 * j + 1) % kStages;
          const int sK = (2 * j + 2) % kStages;
          const bool more = j + 1 < nt;
          if (!wait_full(2 * j + 1)) break;
          if (!mbar_wait_w(&ctl->p_full[0], j & 1, abort, a.err)) break;
          tc_fence_after();
          issue_PV(0, sV, j > 0);
          if (more) {
            if (!wait_full(2 * j + 2)) break;
            tc_fence_after();
            issue_S(0, sK);
            umma_commit_w(&ctl->s_full[0]);
          } else {
            umma_commit_w(&ctl->o_full[0]);
          }
          if (!mbar_wait_w(&ctl->p_full[1], j & 1, abort, a.err)) break;
          tc_fence_after();
          issue_PV(1, sV, j > 0);
          umma_commit_w(&ctl->kv_empty[sV]);
          if (more) {
            issue_S(1, sK);
            umma_commit_w(&ctl->s_full[1]);
            umma_commit_w(&ctl->kv_empty[sK]);
          } else {
            umma_commit_w(&ctl->o_full[1]);
          }
        }
      } else if (ok) {
        // Split form: warpgroup t takes tiles g = 2j + t of the one head (tile
        // g's K at ring position 2g, V at 2g + 1); each slot is released after
        // its one product.  Same order as the pair form: PV_0(j), S_0(j+1),
        // PV_1(j), S_1(j+1).
        const int n0 = (nt + 1) / 2, n1 = nt / 2;
        tc_fence_after();
        issue_S(0, 0);
        umma_commit_w(&ctl->s_full[0]);
        umma_commit_w(&ctl->kv_empty[0]);
        if (n1 > 0) {
          if (!wait_full(2)) ok = false;
          if (ok) {
            tc_fence_after();
            issue_S(1, 2 % kStages);
            umma_commit_w(&ctl->s_full[1]);
            umma_commit_w(&ctl->kv_empty[2 % kStages]);
          }
        }
        for (int j = 0; ok && j < n0; ++j) {
          const int g0 = 2 * j, g1 = 2 * j + 1;
          if (!wait_full(2 * g0 + 1)) break;
          if (!mbar_wait_w(&ctl->p_full[0], j & 1, abort, a.err)) break;
          tc_fence_after();
          issue_PV(0, (2 * g0 + 1) % kStages, j > 0);
          umma_commit_w(&ctl->kv_empty[(2 * g0 + 1) % kStages]);
          if (j + 1 < n0) {
            if (!wait_full(2 * (g0 + 2))) break;
            tc_fence_after();
            issue_S(0, (2 * (g0 + 2)) % kStages);
            umma_commit_w(&ctl->s_full[0]);
            umma_commit_w(&ctl->kv_empty[(2 * (g0 + 2)) % kStages]);
          } else {
            umma_commit_w(&ctl->o_full[0]);
          }
          if (j < n1) {
            if (!wait_full(2 * g1 + 1)) break;
            if (!mbar_wait_w(&ctl->p_full[1], j & 1, abort, a.err)) break;
            tc_fence_after();
            issue_PV(1, (2 * g1 + 1) % kStages, j > 0);
            umma_commit_w(&ctl->kv_empty[(2 * g1 + 1) % kStages]);
            if (j + 1 < n1) {
              if (!wait_full(2 * (g1 + 2))) break;
              tc_fence_after();
              issue_S(1, (2 * (g1 + 2)) % kStages);
              umma_commit_w(&ctl->s_full[1]);
              umma_commit_w(&ctl->kv_empty[(2 * (g1 + 2)) % kStages]);
            } else {
              umma_commit_w(&ctl->o_full[1]);
            }
          }
        }
      }
      // All issued MMAs must finish before tensor memory is released.
      umma_commit_w(&ctl->mma_done);
      volatile int no_abort = 0;
      mbar_wait_w(&ctl->mma_done, 0, &no_abort, a.err);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    const float sl2 = a.sl2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t v[128];
    // pair form: every tile for head t; split form: tiles g = 2j + t of the one head
    const int ntt = kTwo ? nt : (nt + 1 - t) / 2;
    for (int j = 0; j < ntt; ++j) {
      const int g = kTwo ? j : 2 * j + t;  // the tile's position in the tile list
      // tcgen05.ld/st are warp-collective: every branch around them is
      // decided for the whole warp.
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl->s_full[t], j & 1, abort, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // The whole S row in one pass: 128 columns, one wait.
      tmem_ld128_wait(tS, v);
      if (g == nt - 1) {
        // diagonal segment tile: keys after the query's own position are masked
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e > r) v[e] = 0xFF800000u;  // -inf
      } else if (!kGrp && a.hblk == 64 && ctl->tiles[g] >= 0 && (ctl->tiles[g] >> 16) == kNoBlock) {
        // a history tile holding one 64-token block: its upper 64 keys are masked
#pragma unroll
        for (int e = 64; e < 128; ++e) v[e] = 0xFF800000u;
      } else if (kGrp && ctl->tiles[g] >= 0 && (ctl->tiles[g] >> 16) * a.hblk < kBN) {
        // a short grouped history tile: the keys after its blocks are masked
        const int nk = (ctl->tiles[g] >> 16) * a.hblk;
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e >= nk) v[e] = 0xFF800000u;
      }
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 128; e += 2)
        m4[(e >> 1) & 3] = max3f(m4[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
      const float mx = max3f(m4[0], m4[1], fmaxf(m4[2], m4[3])) * sl2;
      const bool need = mx > m_ref + kRescaleThreshold;
      const bool any_need = __any_sync(0xffffffffu, need);
      float alpha = 1.0f;  // rows that keep their reference use alpha = 1
      if (need) {
        alpha = ex2_approx(m_ref - mx);
        l *= alpha;
        m_ref = mx;
      }
      const float2 s2 = make_float2(sl2, sl2), nm = make_float2(-m_ref, -m_ref);
      float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 x = fma2(make_float2(__uint_as_float(v[c * 32 + e]), __uint_as_float(v[c * 32 + e + 1])), s2, nm);
          const float2 p = exp2_pair(x, (kFwdPolyPairs >> (e >> 1)) & 1u);
          l2[(e >> 1) & 1] = add2(l2[(e >> 1) & 1], p);
          pk[e >> 1] = pack_bf16x2(p.x, p.y);
        }
        HGA_TMEM_ST16(tS + c * 32, pk);
      }
      l += (l2[0].x + l2[0].y) + (l2[1].x + l2[1].y);
      if (any_need && j > 0) {
        // O_t holds the sum up to tile j-1 (PV_t(j-1) completed before S_t(j)
        // was announced): bring it to the new reference.
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t ov[32];
          HGA_TMEM_LD32_WAIT(tO + c * 32, ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          HGA_TMEM_ST32(tO + c * 32, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl->p_full[t]);
    }
    // split form: warpgroup 1's row statistics go to the unused second Q tile
    float* xs = reinterpret_cast<float*>(sm + 2 * kTileBytes - 1024);
    if (!kTwo && t == 1) {
      // Publish this row's (m, l) for warpgroup 0's merge (every thread
      // arrives once, whatever happened; -inf / 0 when it has nothing).
      const bool v1 = __all_sync(0xffffffffu, ok && (ntt == 0 || mbar_wait(&ctl->o_full[1], 0, abort, a.err)));
      xs[r] = v1 && ntt > 0 ? m_ref : -INFINITY;
      xs[kBM + r] = v1 && ntt > 0 ? l : 0.f;
      mbar_arrive(&ctl->x_full);
    } else if (!kTwo) {
      // Warpgroup 0 merges the two partial states of the head:
      // O = (a0 O_0 + a1 O_1) / (a0 l0 + a1 l1), a_t = 2^(m_t - max(m_0, m_1)).
      const bool with1 = nt / 2 > 0;
      if (__all_sync(0xffffffffu, ok && mbar_wait(&ctl->o_full[0], 0, abort, a.err) &&
                                      (!with1 || mbar_wait(&ctl->o_full[1], 0, abort, a.err)) &&
                                      mbar_wait(&ctl->x_full, 0, abort, a.err))) {
        tc_fence_after();
        const float m1 = xs[r], l1 = xs[kBM + r];
        const float mm = fmaxf(m_ref, m1);
        const float a0 = ex2_approx(m_ref - mm), a1 = l1 > 0.f ? ex2_approx(m1 - mm) : 0.f;
        const float lt = l * a0 + l1 * a1;
        const float s0 = a0 / lt, s1 = a1 / lt;
        const int p = i * kBM + r;
        // staged and written as in the pair form (head 0's rows)
        uint8_t* stage = sm + (size_t)r * (2 * kD + 16);
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t ov[32], ow[32];
          HGA_TMEM_LD32_WAIT(tO + c * 32, ov);
          if (with1) {
            HGA_TMEM_LD32_WAIT(tO + 128 + c * 32, ow);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ow[e] = 0u;
          }
          uint4* dst = reinterpret_cast<uint4*>(stage + c * 64);
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] = __uint_as_float(ov[8 * qd + e]) * s0 + __uint_as_float(ow[8 * qd + e]) * s1;
            uint4 w;
            w.x = pack_bf16x2(f[0], f[1]);
            w.y = pack_bf16x2(f[2], f[3]);
            w.z = pack_bf16x2(f[4], f[5]);
            w.w = pack_bf16x2(f[6], f[7]);
            dst[qd] = w;
          }
        }
        fence_proxy_async_smem();
        bulk_store(a.o + (((size_t)b * a.S + p) * a.Hq + hq0) * kD, stage, kD * 2);
        bulk_commit();
        a.lse[((size_t)b * a.Hq + hq0) * a.S + p] = (mm + log2f(lt)) * 0.6931471805599453f;
        bulk_wait_read_all();  // the shared-memory source outlives the copy
      }
    } else if (__all_sync(0xffffffffu, ok && mbar_wait(&ctl->o_full[t], 0, abort, a.err))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int p = i * kBM + r;
      const int hq = hq0 + t;
      // The row goes through shared memory, rows padded to 2d + 16 bytes so
      // that a warp's 32 rows fall in distinct banks, and out as one bulk copy
      // (a warp's direct stores would each touch 32 rows).  Head 0 stages in
      // bytes [0, 128 (2d + 16)) -- the Q tiles, free once S_1 of the last
      // tile is done, which o_full[0] implies; head 1 in the next 128 rows,
      // reaching into ring slot 0 only after every MMA has finished.
      uint8_t* stage = sm + (size_t)(t * kBM + r) * (2 * kD + 16);
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t ov[32];
        HGA_TMEM_LD32_WAIT(tO + c * 32, ov);
        uint4* dst = reinterpret_cast<uint4*>(stage + c * 64);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(ov[8 * qd + 0]) * inv_l, __uint_as_float(ov[8 * qd + 1]) * inv_l);
          w.y = pack_bf16x2(__uint_as_float(ov[8 * qd + 2]) * inv_l, __uint_as_float(ov[8 * qd + 3]) * inv_l);
          w.z = pack_bf16x2(__uint_as_float(ov[8 * qd + 4]) * inv_l, __uint_as_float(ov[8 * qd + 5]) * inv_l);
          w.w = pack_bf16x2(__uint_as_float(ov[8 * qd + 6]) * inv_l, __uint_as_float(ov[8 * qd + 7]) * inv_l);
          dst[qd] = w;
        }
      }
      fence_proxy_async_smem();
      bulk_store(a.o + (((size_t)b * a.S + p) * a.Hq + hq) * kD, stage, kD * 2);
      bulk_commit();
      a.lse[((size_t)b * a.Hq + hq) * a.S + p] = (m_ref + log2f(l)) * 0.6931471805599453f;
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

}  // namespace

bool tc_supported(const Shape& s) {
  return s.bf16 && (s.d == 128 || s.d == 64) && (s.blk == 128 || s.blk == 64 || s.blk == 32 || s.blk == 16) &&
         s.qblk == kBM && (s.G() % 2) == 0 &&
         s.topk <= kMaxTopk &&
         s.nqb() <= kMaxQueryBlocks;
}

template <int KD, bool kGrp, bool kTwo>
cudaError_t launch_fwd(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, void* o, float* lse, int* err,
                       cudaStream_t st, bool withhold_kv) {
  constexpr size_t smem = fwd_smem_bytes<kGrp>(KD);
  cudaError_t e = smem_limit(reinterpret_cast<const void*>(fwd_tc_kernel<KD, kGrp, kTwo>), smem);
  if (e != cudaSuccess) return e;
  FwdArgs a;
  a.B = s.B; a.Hq = s.Hq; a.Hkv = s.Hkv; a.S = s.S; a.nkv = nkv; a.topk = s.topk; a.nqb = s.nqb(); a.G = s.G();
  a.sl2 = 1.4426950408889634f / sqrtf((float)KD);
  a.idx = idx; a.o = static_cast<__nv_bfloat16*>(o); a.lse = lse; a.err = err; a.hblk = s.blk;
  a.withhold_kv = withhold_kv ? 1 : 0;
  const int grid = s.B * s.Hkv * (s.G() / (kTwo ? 2 : 1)) * s.nqb();
  fwd_tc_kernel<KD, kGrp, kTwo><<<grid, 384, smem, st>>>(m.q, m.ks, m.vs, m.kh, m.vh, a);
  return cudaGetLastError();
}

template <bool kGrp, bool kTwo>
cudaError_t launch_fwd_d(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, void* o, float* lse, int* err,
                         cudaStream_t st, bool withhold_kv) {
  return s.d == 64 ? launch_fwd<64, kGrp, kTwo>(s, m, nkv, idx, o, lse, err, st, withhold_kv)
                   : launch_fwd<128, kGrp, kTwo>(s, m, nkv, idx, o, lse, err, st, withhold_kv);
}

cudaError_t launch_attn_fwd_tc(const Shape& s, const TcMaps& m, int nkv, const int32_t* idx, void* o, float* lse,
                               int* err, cudaStream_t st, int heads_per_cta, bool withhold_kv) {
  const bool two = heads_per_cta != 1;
  if (s.blk < 64)
    return two ? launch_fwd_d<true, true>(s, m, nkv, idx, o, lse, err, st, withhold_kv)
               : launch_fwd_d<true, false>(s, m, nkv, idx, o, lse, err, st, withhold_kv);
  return two ? launch_fwd_d<false, true>(s, m, nkv, idx, o, lse, err, st, withhold_kv)
             : launch_fwd_d<false, false>(s, m, nkv, idx, o, lse, err, st, withhold_kv);
}

}  // namespace hga
