// C ABI of libhga.so: argument checks, tensor-map encoding, kernel dispatch,
// and the host side of the history tier (fetch of selected blocks, segment
// offload).  Declarations and the method's definition: include/hga.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <chrono>
#include <memory>
#include <mutex>
#include <thread>
#include <vector>

#include "../../include/hga.h"
#include "../../include/hga_selftest.h"
#include "hga_kernels.h"

namespace hga {
cudaError_t smem_limit(const void* kernel, size_t bytes) {
  struct Set {
    const void* kernel;
    int device;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Set> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Set& x : done)
      if (x.kernel == kernel && x.device == dev && x.bytes >= bytes) return cudaSuccess;
  }
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes)) != cudaSuccess)
    return e;
  std::lock_guard<std::mutex> lock(mu);
  for (Set& x : done)
    if (x.kernel == kernel && x.device == dev) {
      x.bytes = std::max(x.bytes, bytes);
      return cudaSuccess;
    }
  done.push_back({kernel, dev, bytes});
  return cudaSuccess;
}
}  // namespace hga

namespace {

thread_local char g_last_error[512] = "";

hga_status fail(hga_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

hga_status cuda_fail(cudaError_t e, const char* where) {
  return fail(HGA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Per-device error flag written by the kernels (see hga_device_status).
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_mu;

hga_status device_err_ptr(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HGA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error flag)");
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_err_ptr[dev];
  return HGA_OK;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

hga_status get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return fail(HGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *fn = cached;
  return HGA_OK;
}

// bf16 tensor [B, T, H, d] (d in {64, 128}) with a {64, 1, rows, 1} box (rows
// tokens x 64 channels = 128-byte rows; rows 128, or 64 for the history when
// its blocks hold 64 tokens), 128-byte swizzle.
hga_status encode_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int d, int rows = 128) {
  EncodeTiledFn enc = nullptr;
  hga_status s = get_encoder(&enc);
  if (s != HGA_OK) return s;
  const cuuint64_t D = (cuuint64_t)d;
  const cuuint64_t dims[4] = {D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HGA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HGA_OK;
}

// ---------------------------------------------------------------- checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hga_status check_dims(const hga_dims* d, hga::Shape* out) {
  if (!d) return fail(HGA_ERR_INVALID_ARG, "dims is NULL");
  if (d->dtype != HGA_F32 && d->dtype != HGA_BF16) return fail(HGA_ERR_INVALID_ARG, "bad dtype %d", (int)d->dtype);
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->S < 1 || d->n_hist_blocks < 0 || d->topk < 1)
    return fail(HGA_ERR_SHAPE, "non-positive dimension");
  if (d->Hq % d->Hkv) return fail(HGA_ERR_SHAPE, "Hq (%d) not a multiple of Hkv (%d)", d->Hq, d->Hkv);
  if (d->d != 64 && d->d != 128) return fail(HGA_ERR_SHAPE, "head dim %d not in {64,128}", d->d);
  if (d->block != 16 && d->block != 32 && d->block != 64 && d->block != 128)
    return fail(HGA_ERR_SHAPE, "block %d not in {16,32,64,128}", d->block);
  if (d->S % d->block) return fail(HGA_ERR_SHAPE, "S (%d) not a multiple of block (%d)", d->S, d->block);
  if (d->q_block != 0 && d->q_block != 16 && d->q_block != 32 && d->q_block != 64 && d->q_block != 128)
    return fail(HGA_ERR_SHAPE, "q_block %d not in {0,16,32,64,128}", d->q_block);
  const int qblk = d->q_block ? d->q_block : d->block;
  if (d->S % qblk) return fail(HGA_ERR_SHAPE, "S (%d) not a multiple of q_block (%d)", d->S, qblk);
  if (d->topk > hga::kMaxTopk) return fail(HGA_ERR_SHAPE, "topk %d > %d", d->topk, hga::kMaxTopk);
  const double tokens = (double)d->B * ((double)d->n_hist_blocks * d->block + d->S) * d->Hq * d->d;
  if (tokens > 4.0e12) return fail(HGA_ERR_SHAPE, "problem too large");
  out->B = d->B; out->Hq = d->Hq; out->Hkv = d->Hkv; out->d = d->d; out->blk = d->block; out->S = d->S;
  out->nblk = d->n_hist_blocks; out->topk = d->topk; out->bf16 = (d->dtype == HGA_BF16); out->qblk = qblk;
  return HGA_OK;
}

template <typename... P>
bool any_null(P... p) {
  return ((p == nullptr) || ...);
}

hga_status check_attn_ptrs(const hga::Shape& s, int n_kv_blocks, const void* q, const void* ks, const void* vs,
                           const void* kh, const void* vh, const int32_t* idx) {
  if (any_null(q, ks, vs, idx)) return fail(HGA_ERR_INVALID_ARG, "NULL input pointer");
  if (n_kv_blocks < 0) return fail(HGA_ERR_INVALID_ARG, "n_kv_blocks < 0");
  if (n_kv_blocks > 0 && any_null(kh, vh)) return fail(HGA_ERR_INVALID_ARG, "NULL history pointer");
  if (!aligned16(q) || !aligned16(ks) || !aligned16(vs) || (n_kv_blocks > 0 && (!aligned16(kh) || !aligned16(vh))))
    return fail(HGA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  (void)s;
  return HGA_OK;
}

// The tensor-core kernels take the shape, and with 64-token history blocks
// they pack two block indices of 15 bits into one tile entry.
bool use_tc(const hga::Shape& s, int n_kv_blocks) {
  return hga::tc_supported(s) && (s.blk != 64 || n_kv_blocks < 0x7FFF);
}

// Query heads per CTA of the tensor-core forward: hga_set_forward_heads_per_cta
// fixes it for the calling thread (like hga_last_error, per thread); by
// default a pair, unless the pairs' grid would leave SMs idle.
thread_local int g_fwd_heads = 0;

int fwd_heads_per_cta(const hga::Shape& s) {
  const int forced = g_fwd_heads;
  if (forced != 0) return forced;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  return (long long)s.B * s.Hkv * (s.G() / 2) * s.nqb() < n_sm ? 1 : 2;
}

hga_status build_maps(const hga::Shape& s, int nkv, const void* q, const void* d_o, const void* ks, const void* vs,
                      const void* kh, const void* vh, hga::TcMaps* m) {
  hga_status r;
  if ((r = encode_tokens(&m->q, q, s.B, s.S, s.Hq, s.d)) != HGA_OK) return r;
  if ((r = encode_tokens(&m->d_o, d_o ? d_o : q, s.B, s.S, s.Hq, s.d)) != HGA_OK) return r;
  if ((r = encode_tokens(&m->ks, ks, s.B, s.S, s.Hkv, s.d)) != HGA_OK) return r;
  if ((r = encode_tokens(&m->vs, vs, s.B, s.S, s.Hkv, s.d)) != HGA_OK) return r;
  // With no history the history maps are never read; point them at the segment.
  const int hr = nkv > 0 ? s.blk : 128;  // history box rows: one block
  if ((r = encode_tokens(&m->kh, nkv > 0 ? kh : ks, s.B, nkv > 0 ? nkv * s.blk : s.S, s.Hkv, s.d, hr)) != HGA_OK)
    return r;
  if ((r = encode_tokens(&m->vh, nkv > 0 ? vh : vs, s.B, nkv > 0 ? nkv * s.blk : s.S, s.Hkv, s.d, hr)) != HGA_OK)
    return r;
  return HGA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// A working copy of a caller's block cache.  The fetch and segment-insert
// calls plan on the copy and commit it only after every copy they depend on
// has been queued, so a call that fails part-way leaves the caller's cache
// as it was (no block is recorded as resident whose bytes were never sent).
struct CacheDraft {
  std::vector<int32_t> slot_of_block, block_of_slot;
  std::vector<int64_t> last_use;
  hga_block_cache view;
  hga_block_cache* target;

  explicit CacheDraft(hga_block_cache* c)
      : slot_of_block(c->slot_of_block, c->slot_of_block + std::max(0, c->host_capacity_blocks)),
        block_of_slot(c->block_of_slot, c->block_of_slot + std::max(0, c->pool_slots)),
        last_use(c->last_use, c->last_use + std::max(0, c->pool_slots)),
        target(c) {
    view = *c;
    view.slot_of_block = slot_of_block.data();
    view.block_of_slot = block_of_slot.data();
    view.last_use = last_use.data();
  }
  void commit() {
    std::copy(slot_of_block.begin(), slot_of_block.end(), target->slot_of_block);
    std::copy(block_of_slot.begin(), block_of_slot.end(), target->block_of_slot);
    std::copy(last_use.begin(), last_use.end(), target->last_use);
    target->tick = view.tick;
  }
};

bool cache_arrays_ok(const hga_block_cache* c) {
  return c->host_capacity_blocks >= 0 && c->pool_slots >= 0 &&
         (c->host_capacity_blocks == 0 || c->slot_of_block != nullptr) &&
         (c->pool_slots == 0 || (c->block_of_slot != nullptr && c->last_use != nullptr));
}

}  // namespace

extern "C" {

const char* hga_status_string(hga_status s) {
  switch (s) {
    case HGA_OK: return "HGA_OK";
    case HGA_ERR_INVALID_ARG: return "HGA_ERR_INVALID_ARG";
    case HGA_ERR_SHAPE: return "HGA_ERR_SHAPE";
    case HGA_ERR_UNSUPPORTED: return "HGA_ERR_UNSUPPORTED";
    case HGA_ERR_INDEX: return "HGA_ERR_INDEX";
    case HGA_ERR_TIMEOUT: return "HGA_ERR_TIMEOUT";
    case HGA_ERR_CUDA: return "HGA_ERR_CUDA";
  }
  return "HGA_ERR_UNKNOWN";
}

const char* hga_last_error(void) { return g_last_error; }

hga_status hga_device_status(hga_stream_t stream) {
  int* flag = nullptr;
  hga_status s = device_err_ptr(&flag);
  if (s != HGA_OK) return s;
  int host = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&host, flag, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error flag");
  if (host == 0) return HGA_OK;
  e = cudaMemsetAsync(flag, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error flag");
  if (host & hga::kDevErrIndex) return fail(HGA_ERR_INDEX, "a kernel met an idx entry outside [-1, n_kv_blocks)");
  return fail(HGA_ERR_TIMEOUT, "a kernel pipeline wait expired");
}

hga_status hga_block_summaries(const hga_dims* dims, const void* k_hist, int blk_begin, int blk_end, float* summ,
                               hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (blk_begin < 0 || blk_end > s.nblk || blk_begin > blk_end)
    return fail(HGA_ERR_INVALID_ARG, "block range [%d,%d) outside [0,%d)", blk_begin, blk_end, s.nblk);
  if (blk_end == blk_begin) return HGA_OK;
  if (any_null(k_hist, summ)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k_hist)) return fail(HGA_ERR_INVALID_ARG, "k_hist must be 16-byte aligned");
  cudaError_t e = hga::launch_block_summaries(s, k_hist, s.nblk * s.blk, blk_begin, blk_begin, blk_end - blk_begin,
                                              summ, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "block summaries launch");
}

hga_status hga_segment_summaries(const hga_dims* dims, const void* k_seg, int at_block, float* summ,
                                 hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (at_block < 0 || at_block + s.nsb() > s.nblk)
    return fail(HGA_ERR_INVALID_ARG, "blocks [%d,%d) outside the summary array's %d", at_block, at_block + s.nsb(),
                s.nblk);
  if (any_null(k_seg, summ)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k_seg)) return fail(HGA_ERR_INVALID_ARG, "k_seg must be 16-byte aligned");
  cudaError_t e = hga::launch_block_summaries(s, k_seg, s.S, 0, at_block, s.nsb(), summ,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "segment summaries launch");
}

hga_status hga_select_topk(const hga_dims* dims, const void* q_seg, const float* summ, int32_t* idx,
                           float* scores_or_null, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (s.nblk > hga::kMaxSelectBlocks)
    return fail(HGA_ERR_SHAPE, "n_hist_blocks %d > %d", s.nblk, hga::kMaxSelectBlocks);
  if (any_null(q_seg, idx) || (s.nblk > 0 && summ == nullptr)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q_seg)) return fail(HGA_ERR_INVALID_ARG, "q must be 16-byte aligned");
  cudaError_t e = hga::launch_select_topk(s, q_seg, summ, idx, scores_or_null, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "select launch");
}

hga_status hga_attn_fwd(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                        const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx, void* o,
                        float* lse, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if ((r = check_attn_ptrs(s, n_kv_blocks, q, k_seg, v_seg, k_hist, v_hist, idx)) != HGA_OK) return r;
  if (any_null(o, lse)) return fail(HGA_ERR_INVALID_ARG, "NULL output pointer");
  if (!aligned16(o)) return fail(HGA_ERR_INVALID_ARG, "o must be 16-byte aligned");
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (use_tc(s, n_kv_blocks)) {
    hga::TcMaps m;
    if ((r = build_maps(s, n_kv_blocks, q, nullptr, k_seg, v_seg, k_hist, v_hist, &m)) != HGA_OK) return r;
    e = hga::launch_attn_fwd_tc(s, m, n_kv_blocks, idx, o, lse, err, st, fwd_heads_per_cta(s));
  } else {
    e = hga::launch_attn_fwd_simt(s, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, o, lse, err, st);
  }
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "attention forward launch");
}

size_t hga_attn_bwd_workspace_size(const hga_dims* dims) {
  if (!dims) return 0;
  return round256((size_t)dims->B * dims->Hq * dims->S * sizeof(float));
}

}  // extern "C"

namespace {

// Shared checks and dispatch of the backward stages (parts: hga::kBwdDq |
// hga::kBwdDkdv; preprocess when `pre` is set).
// A library-owned side stream per device, with a fork and a join event: the
// dQ and dK/dV kernels of one backward run concurrently (each kernel's last
// partial wave is filled by the other's CTAs).  The mutex is held from the
// fork's record to the join's wait, so concurrent callers never see each
// other's events.  Stream capture follows the fork into the side stream and
// back, so the pair also records into a CUDA graph as two branches.
struct SideStream {
  std::mutex mu;
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool tried = false;
};
SideStream* side_stream(int dev) {
  static SideStream pool[64];
  if (dev < 0 || dev >= 64) return nullptr;
  SideStream* x = &pool[dev];
  return x;
}
bool side_ready(SideStream* x) {  // called with x->mu held
  if (!x->tried) {
    x->tried = true;
    if (cudaStreamCreateWithFlags(&x->side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&x->fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x->join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      x->side = nullptr;
    }
  }
  return x->side != nullptr;
}

hga_status run_bwd(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg, const void* k_hist,
                   const void* v_hist, int n_kv_blocks, const int32_t* idx, const void* o, const float* lse,
                   const void* d_o, float* dq, float* dk_seg, float* dv_seg, const void* ws, size_t ws_bytes,
                   bool pre, int parts, hga_stream_t stream, const uint8_t* qmask = nullptr, float gscale = 1.0f) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(ws)) return fail(HGA_ERR_INVALID_ARG, "NULL workspace");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(HGA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (ws_bytes < hga_attn_bwd_workspace_size(dims))
    return fail(HGA_ERR_INVALID_ARG, "workspace %zu bytes < %zu", ws_bytes, hga_attn_bwd_workspace_size(dims));
  if (pre && (any_null(o, d_o) || !aligned16(o) || !aligned16(d_o)))
    return fail(HGA_ERR_INVALID_ARG, "o and d_o must be non-NULL and 16-byte aligned");
  if (parts) {
    if ((r = check_attn_ptrs(s, (parts & hga::kBwdDq) ? n_kv_blocks : 0, q, k_seg, v_seg, k_hist, v_hist,
                             (parts & hga::kBwdDq) ? idx : reinterpret_cast<const int32_t*>(q))) != HGA_OK)
      return r;
    if (any_null(lse, d_o) || !aligned16(lse) || !aligned16(d_o))
      return fail(HGA_ERR_INVALID_ARG, "lse and d_o must be non-NULL and 16-byte aligned");
    if ((parts & hga::kBwdDq) && (any_null(dq) || !aligned16(dq)))
      return fail(HGA_ERR_INVALID_ARG, "dq must be non-NULL and 16-byte aligned");
    if ((parts & hga::kBwdDkdv) && (any_null(dk_seg, dv_seg) || !aligned16(dk_seg) || !aligned16(dv_seg)))
      return fail(HGA_ERR_INVALID_ARG, "dk_seg/dv_seg must be non-NULL and 16-byte aligned");
  }
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* Dr = static_cast<float*>(const_cast<void*>(ws));
  cudaError_t e;
  if (pre && (e = hga::launch_bwd_preprocess(s, o, d_o, Dr, st)) != cudaSuccess)
    return cuda_fail(e, "backward preprocess launch");
  if (!parts) return HGA_OK;
  if (use_tc(s, n_kv_blocks)) {
    hga::TcMaps m;
    if ((r = build_maps(s, n_kv_blocks, q, d_o, k_seg, v_seg, k_hist, v_hist, &m)) != HGA_OK) return r;
    int dev = 0;
    SideStream* x = (parts == (hga::kBwdDq | hga::kBwdDkdv) && cudaGetDevice(&dev) == cudaSuccess) ? side_stream(dev)
                                                                                                   : nullptr;
    if (x) {
      std::lock_guard<std::mutex> lock(x->mu);
      if (side_ready(x)) {
        // dQ (the longer kernel) first on the caller's stream, dK/dV on the side stream, joined back
        if ((e = cudaEventRecord(x->fork, st)) != cudaSuccess || (e = cudaStreamWaitEvent(x->side, x->fork, 0)) !=
                                                                       cudaSuccess)
          return cuda_fail(e, "backward fork");
        if ((e = hga::launch_attn_bwd_tc(s, m, n_kv_blocks, idx, lse, Dr, dq, dk_seg, dv_seg, hga::kBwdDq, err, st,
                                         qmask, gscale)) != cudaSuccess)
          return cuda_fail(e, "attention backward launch (dQ)");
        if ((e = hga::launch_attn_bwd_tc(s, m, n_kv_blocks, idx, lse, Dr, dq, dk_seg, dv_seg, hga::kBwdDkdv, err,
                                         x->side, qmask, gscale)) != cudaSuccess)
          return cuda_fail(e, "attention backward launch (dK/dV)");
        if ((e = cudaEventRecord(x->join, x->side)) != cudaSuccess || (e = cudaStreamWaitEvent(st, x->join, 0)) !=
                                                                          cudaSuccess)
          return cuda_fail(e, "backward join");
        return HGA_OK;
      }
    }
    e = hga::launch_attn_bwd_tc(s, m, n_kv_blocks, idx, lse, Dr, dq, dk_seg, dv_seg, parts, err, st, qmask, gscale);
  } else {
    e = hga::launch_attn_bwd_simt(s, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, lse, Dr, d_o, dq, dk_seg,
                                  dv_seg, parts, err, st, qmask, gscale);
  }
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "attention backward launch");
}

}  // namespace

extern "C" {

int hga_attn_uses_tensor_cores(const hga_dims* dims, int n_kv_blocks) {
  hga::Shape s{};
  if (check_dims(dims, &s) != HGA_OK || n_kv_blocks < 0) return -1;
  return use_tc(s, n_kv_blocks) ? 1 : 0;
}

hga_status hga_set_forward_heads_per_cta(int heads) {
  if (heads < 0 || heads > 2) return fail(HGA_ERR_INVALID_ARG, "heads per CTA must be 0 (automatic), 1 or 2");
  g_fwd_heads = heads;
  return HGA_OK;
}

hga_status hga_attn_bwd(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                        const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx, const void* o,
                        const float* lse, const void* d_o, float* dq, float* dk_seg, float* dv_seg, void* ws,
                        size_t ws_bytes, hga_stream_t stream) {
  return run_bwd(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, o, lse, d_o, dq, dk_seg, dv_seg, ws,
                 ws_bytes, true, hga::kBwdDq | hga::kBwdDkdv, stream);
}

hga_status hga_attn_bwd_sparse(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                               const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx,
                               const void* o, const float* lse, const void* d_o, const uint8_t* qblock_mask,
                               float scale, float* dq, float* dk_seg, float* dv_seg, void* ws, size_t ws_bytes,
                               hga_stream_t stream) {
  if (!qblock_mask) return fail(HGA_ERR_INVALID_ARG, "qblock_mask is NULL");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(HGA_ERR_INVALID_ARG, "scale must be finite");
  return run_bwd(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, o, lse, d_o, dq, dk_seg, dv_seg, ws,
                 ws_bytes, true, hga::kBwdDq | hga::kBwdDkdv, stream, qblock_mask, scale);
}

hga_status hga_attn_bwd_preprocess(const hga_dims* dims, const void* o, const void* d_o, void* ws, size_t ws_bytes,
                                   hga_stream_t stream) {
  return run_bwd(dims, nullptr, nullptr, nullptr, nullptr, nullptr, 0, nullptr, o, nullptr, d_o, nullptr, nullptr,
                 nullptr, ws, ws_bytes, true, 0, stream);
}

hga_status hga_attn_bwd_dkdv(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                             const float* lse, const void* d_o, const void* ws, size_t ws_bytes, float* dk_seg,
                             float* dv_seg, hga_stream_t stream) {
  return run_bwd(dims, q, k_seg, v_seg, nullptr, nullptr, 0, nullptr, nullptr, lse, d_o, nullptr, dk_seg, dv_seg,
                 ws, ws_bytes, false, hga::kBwdDkdv, stream);
}

hga_status hga_attn_bwd_dq(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                           const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx,
                           const float* lse, const void* d_o, const void* ws, size_t ws_bytes, float* dq,
                           hga_stream_t stream) {
  return run_bwd(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, nullptr, lse, d_o, dq, nullptr, nullptr,
                 ws, ws_bytes, false, hga::kBwdDq, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- backward without a caller workspace
// For callers that cannot allocate device memory (a framework-owned pool that
// forbids outside allocations, a fixed memory plan, a plugin that only sees
// its inputs and outputs): the backward's scratch lives in this fixed array.
// 1,048,576 floats = 4 MiB, the Dr row statistics of B*Hq*S <= 2^20 rows.
// Every GPU that loads the library holds it until the process exits.
namespace {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_bwd_scratch[kNoAllocScratchFloats];

// In host code g_bwd_scratch names a host-side stand-in, not device memory:
// the device address is looked up once per device, with that device current.
float* g_bwd_scratch_ptr[kMaxDevices] = {nullptr};

hga_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HGA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_bwd_scratch_ptr[dev]) {
    float* p = nullptr;
    e = cudaGetSymbolAddress((void**)&p, g_bwd_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(backward scratch)");
    g_bwd_scratch_ptr[dev] = p;
  }
  *out = g_bwd_scratch_ptr[dev];
  return HGA_OK;
}

}  // namespace

extern "C" {

hga_status hga_attn_bwd_noalloc(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                                const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx,
                                const void* o, const float* lse, const void* d_o, float* dq, float* dk_seg,
                                float* dv_seg, hga_stream_t stream) {
  if (!dims) return fail(HGA_ERR_INVALID_ARG, "dims is NULL");
  const size_t rows = (size_t)(dims->B > 0 ? dims->B : 0) * (size_t)(dims->Hq > 0 ? dims->Hq : 0) *
                      (size_t)(dims->S > 0 ? dims->S : 0);
  if (rows > kNoAllocScratchFloats)
    return fail(HGA_ERR_SHAPE,
                "B*Hq*S = %zu exceeds the %zu rows of the built-in backward scratch; call hga_attn_bwd with a "
                "caller-owned workspace instead",
                rows, kNoAllocScratchFloats);
  float* scratch = nullptr;
  hga_status r = noalloc_scratch(&scratch);
  if (r != HGA_OK) return r;
  // Dr is written in full by the preprocess stage before any stage reads it,
  // so the previous call's contents need no clearing.
  return run_bwd(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, o, lse, d_o, dq, dk_seg, dv_seg, scratch,
                 kNoAllocScratchFloats * sizeof(float), true, hga::kBwdDq | hga::kBwdDkdv, stream);
}

namespace {
// The selection's idx into the caller's host scratch, queued on `st`.  Pinned
// scratch mapped into the device is written by a small kernel (SM stores over
// the host link), so this transfer does not wait in the device-to-host copy
// queue behind large copies queued earlier on other streams (the offload of a
// finished segment to the host tier); other host memory takes a copy.
hga_status idx_to_host(const int32_t* idx_dev, int32_t* host_scratch, size_t n, cudaStream_t st) {
  cudaPointerAttributes at;
  cudaError_t e = cudaPointerGetAttributes(&at, host_scratch);
  if (e != cudaSuccess) cudaGetLastError();  // memory CUDA does not know: plain pageable host memory
  if (e == cudaSuccess && at.type == cudaMemoryTypeHost && at.devicePointer != nullptr) {
    e = hga::launch_store_mapped_i32(idx_dev, static_cast<int32_t*>(at.devicePointer), n, st);
    return e == cudaSuccess ? HGA_OK : cuda_fail(e, "idx store to host");
  }
  e = cudaMemcpyAsync(host_scratch, idx_dev, n * sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "idx copy to host");
}
}  // namespace

hga_status hga_fetch_blocks(const hga_dims* dims, const void* host_k, const void* host_v, int host_capacity_blocks,
                            const int32_t* idx_dev,
                            int32_t* host_idx_scratch, void* pool_k, void* pool_v, int pool_slots,
                            int32_t* idx_pool_dev, int* n_unique_out, hga_stream_t compute_stream,
                            hga_stream_t copy_stream, hga_event_t done, int timeout_ms) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(host_k, host_v, idx_dev, host_idx_scratch, pool_k, pool_v, idx_pool_dev, done))
    return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (pool_slots < 0) return fail(HGA_ERR_INVALID_ARG, "pool_slots < 0");
  if (host_capacity_blocks < dims->n_hist_blocks)
    return fail(HGA_ERR_INVALID_ARG, "host tier holds %d blocks < n_hist_blocks %d", host_capacity_blocks,
                dims->n_hist_blocks);
  cudaStream_t cst = reinterpret_cast<cudaStream_t>(compute_stream);
  cudaStream_t xst = reinterpret_cast<cudaStream_t>(copy_stream);
  const size_t n_idx = (size_t)s.B * s.Hkv * s.nqb() * s.topk;
  cudaEvent_t landed = nullptr;
  cudaError_t e = cudaEventCreateWithFlags(&landed, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(e, "event create");
  struct Guard {
    cudaEvent_t a;
    ~Guard() { cudaEventDestroy(a); }
  } guard{landed};
  // 1. idx -> host on the compute stream, after the selection queued there (so
  //    the wait does not queue behind earlier block copies on copy_stream);
  //    the copies below are ordered after it, hence after every kernel queued
  //    on the compute stream so far.
  if ((r = idx_to_host(idx_dev, host_idx_scratch, n_idx, cst)) != HGA_OK) return r;
  if ((e = cudaEventRecord(landed, cst)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = cudaStreamWaitEvent(xst, landed, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    e = cudaEventQuery(landed);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) return cuda_fail(e, "waiting for idx");
    if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms))
      return fail(HGA_ERR_TIMEOUT, "idx copy did not complete within %d ms", timeout_ms);
    std::this_thread::yield();
  }
  // 2. distinct selected blocks, ascending -> pool slots.
  std::vector<int32_t> slot_of(s.nblk > 0 ? s.nblk : 1, -1);
  for (size_t k = 0; k < n_idx; ++k) {
    const int n = host_idx_scratch[k];
    if (n == -1) continue;
    if (n < 0 || n >= s.nblk) return fail(HGA_ERR_INDEX, "idx entry %d outside [-1, %d)", n, s.nblk);
    slot_of[n] = 0;
  }
  int n_unique = 0;
  for (int n = 0; n < s.nblk; ++n)
    if (slot_of[n] == 0) slot_of[n] = n_unique++;
  if (n_unique > pool_slots)
    return fail(HGA_ERR_INVALID_ARG, "%d distinct blocks selected, pool holds %d", n_unique, pool_slots);
  // 3. host -> pool copies, one per run of consecutive blocks, per batch and tensor.
  const size_t es = s.bf16 ? 2 : 4;
  const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * es;
  for (int n = 0; n < s.nblk;) {
    if (slot_of[n] < 0) {
      ++n;
      continue;
    }
    int run = 1;
    while (n + run < s.nblk && slot_of[n + run] >= 0) ++run;
    for (int b = 0; b < s.B; ++b) {
      const size_t src = ((size_t)b * host_capacity_blocks + n) * blk_bytes;
      const size_t dst = ((size_t)b * pool_slots + slot_of[n]) * blk_bytes;
      if ((e = cudaMemcpyAsync(static_cast<char*>(pool_k) + dst, static_cast<const char*>(host_k) + src,
                               run * blk_bytes, cudaMemcpyHostToDevice, xst)) != cudaSuccess)
        return cuda_fail(e, "K block copy");
      if ((e = cudaMemcpyAsync(static_cast<char*>(pool_v) + dst, static_cast<const char*>(host_v) + src,
                               run * blk_bytes, cudaMemcpyHostToDevice, xst)) != cudaSuccess)
        return cuda_fail(e, "V block copy");
    }
    n += run;
  }
  // 4. idx rewritten to pool slots (in the pinned scratch), then uploaded.
  for (size_t k = 0; k < n_idx; ++k) {
    const int n = host_idx_scratch[k];
    host_idx_scratch[k] = n < 0 ? -1 : slot_of[n];
  }
  if ((e = cudaMemcpyAsync(idx_pool_dev, host_idx_scratch, n_idx * sizeof(int32_t), cudaMemcpyHostToDevice, xst)) !=
      cudaSuccess)
    return cuda_fail(e, "pool idx upload");
  if ((e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(done), xst)) != cudaSuccess)
    return cuda_fail(e, "event record");
  if (n_unique_out) *n_unique_out = n_unique;
  return HGA_OK;
}

hga_status hga_block_cache_reset(hga_block_cache* c) {
  if (any_null(c) || c->host_capacity_blocks < 0 || c->pool_slots < 0 ||
      (c->host_capacity_blocks > 0 && c->slot_of_block == nullptr) ||
      (c->pool_slots > 0 && (c->block_of_slot == nullptr || c->last_use == nullptr)))
    return fail(HGA_ERR_INVALID_ARG, "block cache: NULL arrays or negative sizes");
  for (int n = 0; n < c->host_capacity_blocks; ++n) c->slot_of_block[n] = -1;
  for (int k = 0; k < c->pool_slots; ++k) {
    c->block_of_slot[k] = -1;
    c->last_use[k] = -1;
  }
  c->tick = 0;
  return HGA_OK;
}

hga_status hga_block_cache_plan(hga_block_cache* c, const int32_t* need, int n_need, int32_t* slot_out,
                                int32_t* miss_out, int* n_miss) {
  if (any_null(c, n_miss) || n_need < 0 || (n_need > 0 && any_null(need, slot_out, miss_out)))
    return fail(HGA_ERR_INVALID_ARG, "block cache plan: NULL pointer or negative count");
  if (n_need > c->pool_slots)
    return fail(HGA_ERR_INVALID_ARG, "%d distinct blocks needed, pool holds %d", n_need, c->pool_slots);
  for (int k = 0; k < n_need; ++k) {
    if (need[k] < 0 || need[k] >= c->host_capacity_blocks)
      return fail(HGA_ERR_INVALID_ARG, "needed block %d outside [0, %d)", need[k], c->host_capacity_blocks);
    if (k > 0 && need[k] <= need[k - 1]) return fail(HGA_ERR_INVALID_ARG, "needed blocks not ascending");
  }
  const int64_t now = c->tick + 1;
  // hits first: they pin their slots for this call
  for (int k = 0; k < n_need; ++k) {
    const int slot = c->slot_of_block[need[k]];
    slot_out[k] = slot;
    if (slot >= 0) c->last_use[slot] = now;
  }
  // misses: an empty slot, else the least recently used slot not needed now
  int nm = 0;
  for (int k = 0; k < n_need; ++k) {
    if (slot_out[k] >= 0) continue;
    int best = -1;
    for (int x = 0; x < c->pool_slots; ++x) {
      if (c->last_use[x] == now) continue;  // needed by this call
      if (c->block_of_slot[x] < 0) {
        best = x;
        break;
      }
      if (best < 0 || c->last_use[x] < c->last_use[best]) best = x;
    }
    // n_need <= pool_slots guarantees a slot that this call has not claimed
    const int old = c->block_of_slot[best];
    if (old >= 0) c->slot_of_block[old] = -1;
    c->block_of_slot[best] = need[k];
    c->slot_of_block[need[k]] = best;
    c->last_use[best] = now;
    slot_out[k] = best;
    miss_out[nm++] = need[k];
  }
  c->tick = now;
  *n_miss = nm;
  return HGA_OK;
}

hga_status hga_fetch_blocks_cached(const hga_dims* dims, const void* host_k, const void* host_v,
                                   const int32_t* idx_dev, int32_t* host_idx_scratch, void* pool_k, void* pool_v,
                                   hga_block_cache* cache, int32_t* idx_pool_dev, int* n_unique_out,
                                   int* n_fetched_out, hga_stream_t compute_stream, hga_stream_t copy_stream,
                                   hga_event_t done, int timeout_ms) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(host_k, host_v, idx_dev, host_idx_scratch, pool_k, pool_v, cache, idx_pool_dev, done))
    return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!cache_arrays_ok(cache)) return fail(HGA_ERR_INVALID_ARG, "block cache: NULL arrays or negative sizes");
  const int cap = cache->host_capacity_blocks, pool_slots = cache->pool_slots;
  if (cap < dims->n_hist_blocks)
    return fail(HGA_ERR_INVALID_ARG, "host tier holds %d blocks < n_hist_blocks %d", cap, dims->n_hist_blocks);
  cudaStream_t cst = reinterpret_cast<cudaStream_t>(compute_stream);
  cudaStream_t xst = reinterpret_cast<cudaStream_t>(copy_stream);
  const size_t n_idx = (size_t)s.B * s.Hkv * s.nqb() * s.topk;
  cudaEvent_t landed = nullptr;
  cudaError_t e = cudaEventCreateWithFlags(&landed, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(e, "event create");
  struct Guard {
    cudaEvent_t a;
    ~Guard() { cudaEventDestroy(a); }
  } guard{landed};
  // 1. idx -> host on the compute stream, after the work queued there; the
  //    pool copies on copy_stream are ordered after it, hence after every
  //    kernel that may still read the pool slots they overwrite.
  if ((r = idx_to_host(idx_dev, host_idx_scratch, n_idx, cst)) != HGA_OK) return r;
  if ((e = cudaEventRecord(landed, cst)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = cudaStreamWaitEvent(xst, landed, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    e = cudaEventQuery(landed);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) return cuda_fail(e, "waiting for idx");
    if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms))
      return fail(HGA_ERR_TIMEOUT, "idx copy did not complete within %d ms", timeout_ms);
    std::this_thread::yield();
  }
  // 2. distinct selected blocks, ascending; cache plan.
  std::vector<char> used(s.nblk > 0 ? s.nblk : 1, 0);
  for (size_t k = 0; k < n_idx; ++k) {
    const int n = host_idx_scratch[k];
    if (n == -1) continue;
    if (n < 0 || n >= s.nblk) return fail(HGA_ERR_INDEX, "idx entry %d outside [-1, %d)", n, s.nblk);
    used[n] = 1;
  }
  std::vector<int32_t> need;
  for (int n = 0; n < s.nblk; ++n)
    if (used[n]) need.push_back(n);
  std::vector<int32_t> slot(need.size() + 1), miss(need.size() + 1);
  int n_miss = 0;
  CacheDraft draft(cache);
  if ((r = hga_block_cache_plan(&draft.view, need.data(), (int)need.size(), slot.data(), miss.data(), &n_miss)) !=
      HGA_OK)
    return r;
  const int32_t* slot_of_block = draft.slot_of_block.data();
  // 3. host -> pool copies of the misses, merged where blocks and slots are both consecutive.
  const size_t es = s.bf16 ? 2 : 4;
  const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * es;
  for (int k = 0; k < n_miss;) {
    const int n0 = miss[k], s0 = slot_of_block[n0];
    int run = 1;
    while (k + run < n_miss && miss[k + run] == n0 + run && slot_of_block[n0 + run] == s0 + run) ++run;
    for (int b = 0; b < s.B; ++b) {
      const size_t src = ((size_t)b * cap + n0) * blk_bytes;
      const size_t dst = ((size_t)b * pool_slots + s0) * blk_bytes;
      if ((e = cudaMemcpyAsync(static_cast<char*>(pool_k) + dst, static_cast<const char*>(host_k) + src,
                               run * blk_bytes, cudaMemcpyHostToDevice, xst)) != cudaSuccess)
        return cuda_fail(e, "K block copy");
      if ((e = cudaMemcpyAsync(static_cast<char*>(pool_v) + dst, static_cast<const char*>(host_v) + src,
                               run * blk_bytes, cudaMemcpyHostToDevice, xst)) != cudaSuccess)
        return cuda_fail(e, "V block copy");
    }
    k += run;
  }
  // 4. idx rewritten to slots (in the pinned scratch), then uploaded.
  for (size_t k = 0; k < n_idx; ++k) {
    const int n = host_idx_scratch[k];
    host_idx_scratch[k] = n < 0 ? -1 : slot_of_block[n];
  }
  if ((e = cudaMemcpyAsync(idx_pool_dev, host_idx_scratch, n_idx * sizeof(int32_t), cudaMemcpyHostToDevice, xst)) !=
      cudaSuccess)
    return cuda_fail(e, "pool idx upload");
  if ((e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(done), xst)) != cudaSuccess)
    return cuda_fail(e, "event record");
  draft.commit();  // every copy is queued: the plan becomes the cache's state
  if (n_unique_out) *n_unique_out = (int)need.size();
  if (n_fetched_out) *n_fetched_out = n_miss;
  return HGA_OK;
}

hga_status hga_cache_segment(const hga_dims* dims, const void* k_seg, const void* v_seg, void* pool_k, void* pool_v,
                             hga_block_cache* cache, int at_block, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(k_seg, v_seg, pool_k, pool_v, cache)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!cache_arrays_ok(cache)) return fail(HGA_ERR_INVALID_ARG, "block cache: NULL arrays or negative sizes");
  const int nseg = s.nsb();
  if (at_block < 0 || at_block + nseg > cache->host_capacity_blocks)
    return fail(HGA_ERR_INVALID_ARG, "blocks [%d,%d) outside the cache's %d", at_block, at_block + nseg,
                cache->host_capacity_blocks);
  std::vector<int32_t> need(nseg), slot(nseg), miss(nseg);
  for (int t = 0; t < nseg; ++t) need[t] = at_block + t;
  int n_miss = 0;
  CacheDraft draft(cache);
  if ((r = hga_block_cache_plan(&draft.view, need.data(), nseg, slot.data(), miss.data(), &n_miss)) != HGA_OK)
    return r;
  // every block is copied, resident or not: the caller states that these blocks now hold this segment
  const size_t es = s.bf16 ? 2 : 4;
  const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * es;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int t = 0; t < nseg;) {
    int run = 1;
    while (t + run < nseg && slot[t + run] == slot[t] + run) ++run;
    for (int b = 0; b < s.B; ++b) {
      const size_t src = ((size_t)b * nseg + t) * blk_bytes;
      const size_t dst = ((size_t)b * cache->pool_slots + slot[t]) * blk_bytes;
      cudaError_t e = cudaMemcpyAsync(static_cast<char*>(pool_k) + dst, static_cast<const char*>(k_seg) + src,
                                      run * blk_bytes, cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(static_cast<char*>(pool_v) + dst, static_cast<const char*>(v_seg) + src,
                            run * blk_bytes, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e, "segment cache copy");
    }
    t += run;
  }
  draft.commit();
  return HGA_OK;
}

namespace {

// Device address of pinned, mapped host memory covering [p, p + bytes).
hga_status mapped_device_ptr(const void* p, size_t bytes, const char* name, const void** out) {
  cudaPointerAttributes a0, a1;
  cudaError_t e = cudaPointerGetAttributes(&a0, p);
  if (e == cudaSuccess && bytes > 0) e = cudaPointerGetAttributes(&a1, static_cast<const char*>(p) + bytes - 1);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(HGA_ERR_INVALID_ARG, "%s: not pinned host memory (%s)", name, cudaGetErrorString(e));
  }
  if (a0.type != cudaMemoryTypeHost || (bytes > 0 && a1.type != cudaMemoryTypeHost) || a0.devicePointer == nullptr)
    return fail(HGA_ERR_INVALID_ARG, "%s: the whole tier must be pinned host memory mapped into the device", name);
  *out = a0.devicePointer;
  return HGA_OK;
}

}  // namespace

hga_status hga_gather_blocks_mapped(const hga_dims* dims, const void* host_k, const void* host_v,
                                    int host_capacity_blocks, const int32_t* idx_dev, void* pool_k, void* pool_v,
                                    int pool_slots, int32_t* idx_pool_dev, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(host_k, host_v, idx_dev, pool_k, pool_v, idx_pool_dev)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (pool_slots < 1) return fail(HGA_ERR_INVALID_ARG, "pool_slots < 1");
  if (host_capacity_blocks < s.nblk)
    return fail(HGA_ERR_INVALID_ARG, "host tier holds %d blocks < n_hist_blocks %d", host_capacity_blocks, s.nblk);
  if (s.nblk > hga::gather_max_blocks())
    return fail(HGA_ERR_SHAPE, "n_hist_blocks %d > %d", s.nblk, hga::gather_max_blocks());
  if (!aligned16(host_k) || !aligned16(host_v) || !aligned16(pool_k) || !aligned16(pool_v))
    return fail(HGA_ERR_INVALID_ARG, "tier and pool must be 16-byte aligned");
  const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * (s.bf16 ? 2 : 4);
  const size_t tier_bytes = (size_t)s.B * host_capacity_blocks * blk_bytes;
  const void *dk = nullptr, *dv = nullptr;
  if ((r = mapped_device_ptr(host_k, tier_bytes, "host_k", &dk)) != HGA_OK) return r;
  if ((r = mapped_device_ptr(host_v, tier_bytes, "host_v", &dv)) != HGA_OK) return r;
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device attributes");
  e = hga::launch_gather_mapped(s, idx_dev, dk, dv, host_capacity_blocks, pool_k, pool_v, pool_slots, idx_pool_dev,
                                err, n_sm, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "mapped gather launch");
}

hga_status hga_append_segment(const hga_dims* dims, const void* k_seg, const void* v_seg, int at_block, float* summ,
                              void* pool_k, void* pool_v, hga_block_cache* cache, void* host_k, void* host_v,
                              int tier_capacity_blocks, hga_stream_t stream, hga_stream_t copy_stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  const int nseg = s.nsb();
  if (nseg > hga::kMaxQueryBlocks) return fail(HGA_ERR_SHAPE, "segment of %d blocks > %d", nseg, hga::kMaxQueryBlocks);
  if (any_null(k_seg, v_seg, summ)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k_seg) || !aligned16(v_seg)) return fail(HGA_ERR_INVALID_ARG, "k_seg/v_seg must be 16-byte aligned");
  if (at_block < 0 || at_block + nseg > s.nblk)
    return fail(HGA_ERR_INVALID_ARG, "blocks [%d,%d) outside the summary array's %d", at_block, at_block + nseg,
                s.nblk);
  if (cache) {
    if (any_null(pool_k, pool_v)) return fail(HGA_ERR_INVALID_ARG, "NULL pool with a block cache");
    if (!aligned16(pool_k) || !aligned16(pool_v)) return fail(HGA_ERR_INVALID_ARG, "pool must be 16-byte aligned");
    if (!cache_arrays_ok(cache)) return fail(HGA_ERR_INVALID_ARG, "block cache: NULL arrays or negative sizes");
    if (at_block + nseg > cache->host_capacity_blocks)
      return fail(HGA_ERR_INVALID_ARG, "blocks [%d,%d) outside the cache's %d", at_block, at_block + nseg,
                  cache->host_capacity_blocks);
  }
  const bool offload = host_k != nullptr || host_v != nullptr;
  if (offload) {
    if (any_null(host_k, host_v)) return fail(HGA_ERR_INVALID_ARG, "host_k and host_v go together");
    if (at_block + nseg > tier_capacity_blocks)
      return fail(HGA_ERR_INVALID_ARG, "blocks [%d,%d) outside the tier's %d", at_block, at_block + nseg,
                  tier_capacity_blocks);
  }
  // 1. slots of the new blocks (planned on a draft of the cache)
  std::vector<int32_t> need(nseg), slot(nseg), miss(nseg);
  for (int t = 0; t < nseg; ++t) need[t] = at_block + t;
  int n_miss = 0;
  std::unique_ptr<CacheDraft> draft;
  if (cache) {
    draft.reset(new CacheDraft(cache));
    if ((r = hga_block_cache_plan(&draft->view, need.data(), nseg, slot.data(), miss.data(), &n_miss)) != HGA_OK)
      return r;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  // 2. the host-tier copy reads k_seg/v_seg on copy_stream, concurrently with the kernel
  if (offload) {
    cudaStream_t xst = copy_stream ? reinterpret_cast<cudaStream_t>(copy_stream) : st;
    if (xst != st) {
      cudaEvent_t ready = nullptr;
      if ((e = cudaEventCreateWithFlags(&ready, cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail(e, "event create");
      e = cudaEventRecord(ready, st);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(xst, ready, 0);
      cudaEventDestroy(ready);
      if (e != cudaSuccess) return cuda_fail(e, "ordering the offload after the segment's producers");
    }
    const size_t es = s.bf16 ? 2 : 4;
    const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * es;
    for (int b = 0; b < s.B; ++b) {
      const size_t dst = ((size_t)b * tier_capacity_blocks + at_block) * blk_bytes;
      const size_t src = (size_t)b * nseg * blk_bytes;
      e = cudaMemcpyAsync(static_cast<char*>(host_k) + dst, static_cast<const char*>(k_seg) + src, nseg * blk_bytes,
                          cudaMemcpyDeviceToHost, xst);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(static_cast<char*>(host_v) + dst, static_cast<const char*>(v_seg) + src,
                            nseg * blk_bytes, cudaMemcpyDeviceToHost, xst);
      if (e != cudaSuccess) return cuda_fail(e, "segment offload copy");
    }
  }
  // 3. one pass over K and V: summaries, and the pool copies when caching
  e = hga::launch_append_segment(s, k_seg, v_seg, at_block, summ, cache ? pool_k : nullptr,
                                 cache ? pool_v : nullptr, cache ? cache->pool_slots : 0, slot.data(), st);
  if (e != cudaSuccess) return cuda_fail(e, "segment append launch");
  if (draft) draft->commit();
  return HGA_OK;
}

hga_status hga_remap_idx(const hga_dims* dims, const int32_t* idx_dev, const int32_t* slot_of_block_dev,
                         int32_t* idx_pool_dev, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(idx_dev, idx_pool_dev) || (s.nblk > 0 && slot_of_block_dev == nullptr))
    return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  cudaError_t e =
      hga::launch_remap_idx(s, idx_dev, slot_of_block_dev, idx_pool_dev, err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "idx remap launch");
}

hga_status hga_offload_segment(const hga_dims* dims, const void* k_seg, const void* v_seg, void* host_k,
                               void* host_v, int capacity_blocks, int at_block, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (any_null(k_seg, v_seg, host_k, host_v)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  const int nseg = s.nsb();
  if (at_block < 0 || at_block + nseg > capacity_blocks)
    return fail(HGA_ERR_INVALID_ARG, "blocks [%d,%d) outside the tier's %d", at_block, at_block + nseg,
                capacity_blocks);
  const size_t es = s.bf16 ? 2 : 4;
  const size_t blk_bytes = (size_t)s.blk * s.Hkv * s.d * es;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int b = 0; b < s.B; ++b) {
    const size_t dst = ((size_t)b * capacity_blocks + at_block) * blk_bytes;
    const size_t src = (size_t)b * nseg * blk_bytes;
    cudaError_t e = cudaMemcpyAsync(static_cast<char*>(host_k) + dst, static_cast<const char*>(k_seg) + src,
                                    nseg * blk_bytes, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(host_v) + dst, static_cast<const char*>(v_seg) + src, nseg * blk_bytes,
                          cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "segment offload copy");
  }
  return HGA_OK;
}

hga_status hga_decode_select(const hga_dims* dims, int n_q, const void* q_new, const float* summ, int32_t* idx,
                             float* scores_or_null, void* ws, size_t ws_bytes, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (n_q < 1 || n_q > s.qblk) return fail(HGA_ERR_SHAPE, "n_q %d outside [1, query block = %d]", n_q, s.qblk);
  if (s.nblk > hga::kMaxSelectBlocks)
    return fail(HGA_ERR_SHAPE, "n_hist_blocks %d > %d", s.nblk, hga::kMaxSelectBlocks);
  if (any_null(q_new, idx, ws) || (s.nblk > 0 && summ == nullptr)) return fail(HGA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q_new) || !aligned16(ws)) return fail(HGA_ERR_INVALID_ARG, "q_new and ws must be 16-byte aligned");
  const size_t need = hga_decode_workspace_size(dims, n_q);
  if (ws_bytes < need) return fail(HGA_ERR_INVALID_ARG, "workspace %zu bytes < %zu", ws_bytes, need);
  cudaError_t e = hga::launch_decode_select(s, n_q, q_new, summ, idx, scores_or_null, ws,
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "decode select launch");
}

size_t hga_decode_workspace_size(const hga_dims* dims, int n_q) {
  hga::Shape s{};
  if (check_dims(dims, &s) != HGA_OK || n_q < 1 || n_q > s.qblk) return 0;
  const size_t attn = hga::decode_workspace_floats(s, n_q) * sizeof(float);
  const size_t select = (size_t)s.B * s.Hkv * (s.nblk > 0 ? s.nblk : 1) * sizeof(unsigned long long);
  return round256(attn > select ? attn : select);
}

hga_status hga_decode_attn(const hga_dims* dims, int n_q, int t0, const void* q_new, const void* k_seg,
                           const void* v_seg, const void* k_hist, const void* v_hist, int n_kv_blocks,
                           const int32_t* idx, void* o, float* lse, void* ws, size_t ws_bytes, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (n_q < 1 || n_q > s.qblk) return fail(HGA_ERR_SHAPE, "n_q %d outside [1, query block = %d]", n_q, s.qblk);
  if (t0 < 0 || t0 + n_q > s.S)
    return fail(HGA_ERR_SHAPE, "new tokens [%d, %d) outside the segment buffer of %d", t0, t0 + n_q, s.S);
  if (s.topk + (s.S + s.blk - 1) / s.blk > 512)
    return fail(HGA_ERR_SHAPE, "topk + S/block = %d key chunks > 512", s.topk + (s.S + s.blk - 1) / s.blk);
  if ((r = check_attn_ptrs(s, n_kv_blocks, q_new, k_seg, v_seg, k_hist, v_hist, idx)) != HGA_OK) return r;
  if (any_null(o, lse, ws)) return fail(HGA_ERR_INVALID_ARG, "NULL output or workspace pointer");
  if (!aligned16(ws)) return fail(HGA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  const size_t need = hga_decode_workspace_size(dims, n_q);
  if (ws_bytes < need) return fail(HGA_ERR_INVALID_ARG, "workspace %zu bytes < %zu", ws_bytes, need);
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  cudaError_t e = hga::launch_decode_attn(s, n_q, t0, q_new, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx, o, lse,
                                          static_cast<float*>(ws), err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "decode attention launch");
}

hga_status hga_selftest_attn_fwd_stalled(const hga_dims* dims, const void* q, const void* k_seg, const void* v_seg,
                                         const void* k_hist, const void* v_hist, int n_kv_blocks, const int32_t* idx,
                                         void* o, float* lse, hga_stream_t stream) {
  hga::Shape s{};
  hga_status r = check_dims(dims, &s);
  if (r != HGA_OK) return r;
  if (!hga::tc_supported(s)) return fail(HGA_ERR_UNSUPPORTED, "the stall self test runs the tensor-core forward only");
  if ((r = check_attn_ptrs(s, n_kv_blocks, q, k_seg, v_seg, k_hist, v_hist, idx)) != HGA_OK) return r;
  if (any_null(o, lse)) return fail(HGA_ERR_INVALID_ARG, "NULL output pointer");
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  hga::TcMaps m;
  if ((r = build_maps(s, n_kv_blocks, q, nullptr, k_seg, v_seg, k_hist, v_hist, &m)) != HGA_OK) return r;
  cudaError_t e =
      hga::launch_attn_fwd_tc(s, m, n_kv_blocks, idx, o, lse, err, reinterpret_cast<cudaStream_t>(stream),
                              fwd_heads_per_cta(s), true);
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "stalled forward launch");
}

hga_status hga_selftest_umma(int form, const void* a, const void* b, float* d, hga_stream_t stream) {
  if (form < 0 || form > 3) return fail(HGA_ERR_INVALID_ARG, "form %d not in 0..3", form);
  if (any_null(a, b, d) || !aligned16(a) || !aligned16(b)) return fail(HGA_ERR_INVALID_ARG, "bad pointer");
  CUtensorMap ma, mb;
  hga_status r;
  if ((r = encode_tokens(&ma, a, 1, 128, 1, 128)) != HGA_OK) return r;
  if ((r = encode_tokens(&mb, b, 1, 128, 1, 128)) != HGA_OK) return r;
  int* err = nullptr;
  if ((r = device_err_ptr(&err)) != HGA_OK) return r;
  cudaError_t e = hga::launch_selftest_umma(form, ma, mb, a, d, err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HGA_OK : cuda_fail(e, "selftest launch");
}

}  // extern "C"
