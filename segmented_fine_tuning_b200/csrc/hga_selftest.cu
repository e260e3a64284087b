// Self test of the tcgen05 operand layouts used by the attention kernels: a
// single 128x128x128 bf16 product computed with exactly the descriptor and
// tensor-memory arrangements of hga_attn_fwd_tc.cu / hga_attn_bwd_tc.cu.
//   form 0: D = A B^T, A and B from shared memory, both K-major (S = Q K^T)
//   form 1: D = A B,   A K-major, B MN-major from shared memory
//   form 2: D = A B,   A from tensor memory (packed bf16), B MN-major (P V)
//   form 3: D = A B^T, A from tensor memory, B K-major
// A and B are 128x128 row-major bf16 (A: M x K; B: N x K for forms 0/3,
// K x N for forms 1/2); D is 128x128 row-major fp32.
#include "hga_kernels.h"
#include "hga_ptx.cuh"

namespace hga {
namespace {

constexpr int kTile = 128 * 128 * 2;
constexpr int kHalf = kTile / 2;

struct StCtl {
  uint64_t full, done;
  uint32_t tmem;
  int abort;
};

__global__ void __launch_bounds__(160, 1) selftest_umma_kernel(const __grid_constant__ CUtensorMap ma,
                                                               const __grid_constant__ CUtensorMap mb,
                                                               const __nv_bfloat16* a_raw, float* d, int form,
                                                               int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sA = sm;
  uint8_t* sB = sm + kTile;
  StCtl* ctl = reinterpret_cast<StCtl*>(sm + 2 * kTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    if (lane == 0) {
      ctl->abort = 0;
      mbar_init(&ctl->full, 1);
      mbar_init(&ctl->done, 1);
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
  const bool a_in_tmem = (form >= 2);
  if (warp < 4 && a_in_tmem) {
    // Row r of A into tensor memory: K chunk c (32 elements) -> 16 packed
    // columns at column 32c, the arrangement the attention kernels use.
    const int r = warp * 32 + lane;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(a_raw + (size_t)r * 128);
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
      for (int x = 0; x < 16; ++x) pk[x] = src[c * 16 + x];
      HGA_TMEM_ST16(tmem + ((uint32_t)(warp * 32) << 16) + c * 32, pk);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort = &ctl->abort;
  if (warp == 4 && lane == 0) {
    mbar_expect_tx(&ctl->full, a_in_tmem ? kTile : 2 * kTile);
    for (int hh = 0; hh < 2; ++hh) {
      if (!a_in_tmem) tma_load_4d(&ma, &ctl->full, sA + hh * kHalf, hh * 64, 0, 0, 0);
      tma_load_4d(&mb, &ctl->full, sB + hh * kHalf, hh * 64, 0, 0, 0);
    }
    if (mbar_wait(&ctl->full, 0, abort, err)) {
      tc_fence_after();
      const bool b_mn = (form == 1 || form == 2);
      const uint32_t id = idesc_bf16(128, 128, false, b_mn);
      const uint32_t sa = smem_u32(sA), sb = smem_u32(sB);
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * kHalf + (kk & 3) * 32;
        const uint64_t bd = b_mn ? sdesc_sw128(sb + kk * 2048, kHalf, 1024) : sdesc_sw128(sb + koff, 16, 1024);
        if (a_in_tmem)
          umma_ts(tmem + 256, tmem + (kk >> 1) * 32 + (kk & 1) * 8, bd, id, kk > 0);
        else
          umma_ss(tmem + 256, sdesc_sw128(sa + koff, 16, 1024), bd, id, kk > 0);
      }
    }
    umma_commit(&ctl->done);
  }
  if (warp < 4) {
    volatile int no_abort = 0;
    if (__all_sync(0xffffffffu, mbar_wait(&ctl->done, 0, &no_abort, err))) {
      tc_fence_after();
      const int r = warp * 32 + lane;
      uint32_t v[32];
      for (int c = 0; c < 4; ++c) {
        HGA_TMEM_LD32_WAIT(tmem + ((uint32_t)(warp * 32) << 16) + 256 + c * 32, v);
        for (int x = 0; x < 32; ++x) d[(size_t)r * 128 + c * 32 + x] = __uint_as_float(v[x]);
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

cudaError_t launch_selftest_umma(int form, const CUtensorMap& ma, const CUtensorMap& mb, const void* a_raw,
                                 float* d, int* err, cudaStream_t st) {
  const int smem = 1024 + 2 * kTile + (int)sizeof(StCtl);
  cudaError_t e = cudaFuncSetAttribute(selftest_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  selftest_umma_kernel<<<1, 160, smem, st>>>(ma, mb, static_cast<const __nv_bfloat16*>(a_raw), d, form, err);
  return cudaGetLastError();
}

}  // namespace hga
