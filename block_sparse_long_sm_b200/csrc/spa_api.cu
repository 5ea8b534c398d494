// spa_api.cu -- the C ABI declared in include/spa.h except the attention
// entry point (spa_attn.cu): workspace size, selection (plan), statistics and
// the allocation-free selection.  The attention kernels live in their own
// translation unit, so that their code is laid out independently of the
// selection kernels'.  Nothing here allocates device memory.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "fp8_quant.cuh"
#include "host.cuh"
#include "ptx.cuh"
#include "sale.cuh"
#include "select.cuh"

namespace {

using namespace spa;

// FP8 quantisation: the scales array (documented in spa.h) and the scratch.
struct Fp8Layout {
  long long qs = 0, ks = 0, vs = 0, kmean = 0, floats = 0;   // float offsets
  size_t kpart = 0, kabs = 0, vabs = 0, scratch = 0;        // byte offsets
};

Fp8Layout fp8_layout(const spa_params* p) {
  Fp8Layout f;
  const long long nqb = (p->seq_len + 127) / 128;
  const long long bh = (long long)p->batch * p->heads_q, bkv = (long long)p->batch * p->heads_kv;
  f.qs = 0;
  f.ks = bh * nqb;
  f.vs = f.ks + bkv;
  f.kmean = f.vs + bkv * 128;
  f.floats = f.kmean + bkv * 128;
  f.kpart = kHeaderBytes;      // reserved bytes first: every valid call has a non-zero size
  f.kabs = align_up(f.kpart + (size_t)bkv * kKmeanChunks * 128 * 8);
  f.vabs = align_up(f.kabs + (size_t)bkv * 4);
  f.scratch = align_up(f.vabs + (size_t)bkv * 128 * 4);
  return f;
}

}  // namespace

extern "C" {

SPA_API size_t sparse_prefill_workspace_bytes(const spa_params* p) {
  if (validate(p) != SPA_OK) return 0;
  return layout_of(p).total;
}

SPA_API const char* sparse_prefill_status_string(spa_status s) {
  switch (s) {
    case SPA_OK: return "ok";
    case SPA_ERR_INVALID: return "invalid argument";
    case SPA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SPA_ERR_WORKSPACE: return "workspace too small";
    case SPA_ERR_CUDA: return "CUDA error";
    case SPA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

SPA_API spa_status sparse_prefill_plan(const spa_params* p, const void* q, const void* k,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  Layout lo;
  spa_status st = common_checks(p, workspace, workspace_bytes, &lo);
  if (st != SPA_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, stream) != cudaSuccess) return SPA_ERR_CUDA;
  const int B = p->batch, Hq = p->heads_q, Hkv = p->heads_kv, L = p->seq_len;
  if (B == 0 || L == 0 || p->mode == SPA_MODE_DENSE) return SPA_OK;
  if (!q || !k || !aligned16(q) || !aligned16(k)) return SPA_ERR_INVALID;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  const float scale = eff_scale(p);
  const long long BH = (long long)B * Hq, BKV = (long long)B * Hkv;

  if (p->mode == SPA_MODE_ANCHOR) {
    CUtensorMap tq, tk, tqbar;
    if (!map_2d(&tq, kBF16, 2, q, 128, BH * L, 64, 128, kSW128) ||
        !map_2d(&tk, kBF16, 2, k, 128, BKV * L, 64, 128, kSW128) ||
        !map_3d(&tqbar, kBF16, 2, ws + lo.qbar, 128, lo.nqb, 2 * BH, 64, 128, kSW128))
      return SPA_ERR_CUDA;
    PoolArgs pa{B, Hq, Hkv, L, lo.nqb, lo.group, p->sink, p->local, scale,
                reinterpret_cast<float*>(ws + lo.xbar),
                reinterpret_cast<__nv_bfloat16*>(ws + lo.qbar), err, wait_ns(p),
                (lo.nqb + kPoolQbs - 1) / kPoolQbs};
    if (set_smem(anchor_pool_kernel, kPoolSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    anchor_pool_kernel<<<(unsigned)(BH * pa.groups), kPoolThreads, kPoolSmemBytes, stream>>>(
        tq, tk, pa);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;

    if (lo.fused) {
      // scan + compaction in one pass; a head pair shares each CTA's M tile
      const int hpi = lo.paired ? 2 : 1;
      const int R = 128 / hpi;
      const int n_mt = (lo.nqb + R - 1) / R;
      CUtensorMap tqsel;
      if (!map_3d(&tqsel, kBF16, 2, ws + lo.qbar, 128, lo.nqb, 2 * BH, 64, (uint32_t)R, kSW128))
        return SPA_ERR_CUDA;
      SelectArgs sa{B, Hq, Hkv, L, lo.nqb, lo.group, p->sink, p->local, p->step, p->theta,
                    hpi, R, n_mt, (int)(BH / hpi),
                    reinterpret_cast<const float*>(ws + lo.xbar),
                    reinterpret_cast<int*>(ws + lo.lists), lo.list_per_head, lo.cap_a,
                    reinterpret_cast<int*>(ws + lo.counts),
                    reinterpret_cast<uint4*>(ws + lo.tmask), lo.tmask_per_head, lo.tc,
                    reinterpret_cast<uint32_t*>(ws + lo.tbits), lo.tbit_words, err, wait_ns(p)};
      if (set_smem(stripe_select_kernel, kSelSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
      stripe_select_kernel<<<(unsigned)(n_mt * (BH / hpi)), kSelThreads, kSelSmemBytes, stream>>>(
          tqsel, tk, sa);
      if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
      return SPA_OK;
    }
    const int nmt = (lo.nqb + 127) / 128;
    const int key_end = std::max(0, lo.nqb * 128 - p->local);
    const int kt0 = p->sink / 128;
    const int kt_end = (key_end + 127) / 128;
    const int nchunk = key_end > p->sink
                           ? (kt_end - kt0 + kScanTilesPerChunk - 1) / kScanTilesPerChunk
                           : 0;
    if (nchunk > 0) {
      ScanArgs sa{B, Hq, Hkv, L, lo.nqb, lo.group, p->sink, p->local, p->theta,
                  reinterpret_cast<const float*>(ws + lo.xbar),
                  reinterpret_cast<uint32_t*>(ws + lo.mask), lo.nwords, err, wait_ns(p)};
      if (set_smem(stripe_scan_kernel, kScanSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
      stripe_scan_kernel<<<dim3(nchunk, nmt, (unsigned)BH), kScanThreads, kScanSmemBytes,
                           stream>>>(tqbar, tk, sa);
      if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
    }
  } else {
    KmeanArgs ka{static_cast<const __nv_bfloat16*>(k), L, reinterpret_cast<double*>(ws + lo.kpart),
                 reinterpret_cast<float*>(ws + lo.kmean)};
    kmean_partial_kernel<<<dim3(kKmeanChunks, (unsigned)BKV), 128, 0, stream>>>(ka);
    kmean_final_kernel<<<(unsigned)BKV, 128, 0, stream>>>(ka);
    QuantArgs qk{static_cast<const __nv_bfloat16*>(k), reinterpret_cast<const float*>(ws + lo.kmean),
                 L, p->block_k, lo.nkb, reinterpret_cast<int8_t*>(ws + lo.k8),
                 reinterpret_cast<float*>(ws + lo.sk)};
    quant_kernel<<<dim3(lo.nkb, (unsigned)BKV), 128, 0, stream>>>(qk);
    QuantArgs qq{static_cast<const __nv_bfloat16*>(q), nullptr, L, 128, lo.nqb,
                 reinterpret_cast<int8_t*>(ws + lo.q8), reinterpret_cast<float*>(ws + lo.sq)};
    quant_kernel<<<dim3(lo.nqb, (unsigned)BH), 128, 0, stream>>>(qq);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
    CUtensorMap tq8, tk8;
    if (!map_2d(&tq8, kI8, 1, ws + lo.q8, 128, BH * L, 128, 128, kSW128) ||
        !map_2d(&tk8, kI8, 1, ws + lo.k8, 128, BKV * L, 128, kSaleKeys, kSW128))
      return SPA_ERR_CUDA;
    const int chunks = (lo.group + kSaleHeads - 1) / kSaleHeads;
    SaleArgs sa{B, Hq, Hkv, L, lo.nqb, lo.group, p->sink, p->local, p->block_k, lo.nkb,
                __builtin_ctz((unsigned)p->block_k), chunks, scale, p->tau, reinterpret_cast<const float*>(ws + lo.sq),
                reinterpret_cast<const float*>(ws + lo.sk),
                reinterpret_cast<uint32_t*>(ws + lo.mask), lo.nwords, err, wait_ns(p), {}};
    for (int h = 0; h < Hq && h < SPA_MAX_TAU_HEADS; ++h)
      sa.tau_h[h] = p->tau_per_head ? p->tau_per_head[h] : p->tau;
    if (set_smem(sale_scan_kernel, kSaleSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sale_scan_kernel<<<(unsigned)(BKV * lo.nqb * chunks), kSaleThreads, kSaleSmemBytes, stream>>>(
        tq8, tk8, sa);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  {
    CompactArgs ca{(int)lo.nb, lo.nqb, L, p->sink, p->local, lo.unit, p->step,
                   reinterpret_cast<const uint32_t*>(ws + lo.mask), lo.nwords,
                   reinterpret_cast<int*>(ws + lo.lists), lo.list_per_head, lo.cap_a,
                   reinterpret_cast<int*>(ws + lo.counts)};
    compact_kernel<<<(unsigned)lo.nb, kCompactThreads, 0, stream>>>(ca);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  if (lo.tmask_per_head > 0) {
    TileMaskArgs ta{lo.nqb, p->sink, p->local, lo.unit, p->step, lo.tc,
                    reinterpret_cast<const uint32_t*>(ws + lo.mask), lo.nwords,
                    reinterpret_cast<uint4*>(ws + lo.tmask), lo.tmask_per_head,
                    reinterpret_cast<uint32_t*>(ws + lo.tbits), lo.tbit_words};
    tile_mask_kernel<<<(unsigned)lo.nb, 128, 0, stream>>>(ta);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  return SPA_OK;
}

SPA_API spa_status sparse_prefill_stats(const spa_params* p, const void* workspace, size_t workspace_bytes,
                                spa_stats* out, cudaStream_t stream) {
  Layout lo;
  spa_status st = common_checks(p, workspace, workspace_bytes, &lo);
  if (st != SPA_OK) return st;
  if (!out) return SPA_ERR_INVALID;
  uint8_t* ws = const_cast<uint8_t*>(static_cast<const uint8_t*>(workspace));
  unsigned long long* acc = reinterpret_cast<unsigned long long*>(ws + 8);
  if (cudaMemsetAsync(acc, 0, 5 * sizeof(unsigned long long), stream) != cudaSuccess)
    return SPA_ERR_CUDA;
  if (lo.nb > 0) {
    StatsArgs sa{(int)lo.nb, lo.nqb, p->seq_len, p->sink, p->local,
                 p->mode == SPA_MODE_DENSE ? kModeDense : 0, lo.unit,
                 reinterpret_cast<const int*>(ws + lo.counts), acc};
    stats_kernel<<<(unsigned)((lo.nb + 255) / 256), 256, 0, stream>>>(sa);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  uint8_t host[48];
  if (cudaMemcpyAsync(host, ws, sizeof(host), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return SPA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SPA_ERR_CUDA;
  uint32_t errw;
  unsigned long long v[5];
  std::memcpy(&errw, host, 4);
  std::memcpy(v, host + 8, sizeof(v));
  out->error_bits = errw;
  out->reserved = 0;
  out->query_blocks = (int64_t)v[0];
  out->candidates = (int64_t)v[1];
  out->kept_candidates = (int64_t)v[2];
  out->kept_pairs = (int64_t)v[3];
  out->dense_pairs = (int64_t)v[4];
  if (errw & kErrTimeout) return SPA_ERR_TIMEOUT;
  if (errw & kErrBadIndex) return SPA_ERR_INVALID;
  return SPA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of the ANCHOR-mode plan.
//
// Some callers cannot hand this library a workspace: plugin hosts whose
// enqueue step may not allocate device memory, serving stacks that reserve
// their whole memory budget at start-up and own every byte afterwards, and
// hot paths that must not call cudaMalloc because it can synchronise the
// device.  For them the selection's scratch (workspace header, anchor means,
// pooled queries, key bitmask) lives in the fixed array below; the caller
// still provides the inputs (Q, K) and the outputs (counts, lists).
//
// The array is kStaticScratchBytes per GPU, held by every GPU that loads the
// library until the process exits.  All calls share it and it keeps the last
// call's contents, so two calls that overlap on the GPU (different streams,
// different threads) race; callers must serialise them.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = SPA_STATIC_SCRATCH_BYTES;
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void* g_static_ptr[kMaxDevices] = {};
void* g_static_ctx[kMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);

// The current context of the calling thread (driver API through the runtime's
// entry-point lookup, so the library needs no link against libcuda).
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  }
  void* ctx = nullptr;
  return fn(&ctx) == 0 ? ctx : nullptr;
}

// Device address of g_static_scratch on the current device (the host-side
// name is only a stand-in, not a device address).  Looked up with the device
// current on the first call of each device, and again whenever the device's
// context has changed since (after a cudaDeviceReset the old address is gone).
void* static_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  // makes the device's primary context current (no allocation)
  if (cudaSetDevice(dev) != cudaSuccess) return nullptr;
  void* ctx = current_context();
  if (!ctx) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev] || g_static_ctx[dev] != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
    g_static_ptr[dev] = ptr;
    g_static_ctx[dev] = ctx;
  }
  return g_static_ptr[dev];
}

struct StaticLayout {
  size_t xbar, qbar, mask, total;
};

StaticLayout static_layout(const spa_params* p, const Layout& lo) {
  StaticLayout s;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  s.xbar = take(lo.nb * 4);
  s.qbar = take((size_t)2 * lo.nb * 128 * 2);
  s.mask = take((size_t)lo.nb * lo.nwords * 4);
  s.total = off;
  (void)p;
  return s;
}

}  // namespace

extern "C" {

SPA_API spa_status sparse_prefill_plan_static(const spa_params* p, const void* q, const void* k,
                                              int32_t* counts, int32_t* lists,
                                              size_t lists_elems, uint32_t* error_word,
                                              cudaStream_t stream) {
  spa_status st = validate(p);
  if (st != SPA_OK) return st;
  if (p->mode != SPA_MODE_ANCHOR) return SPA_ERR_UNSUPPORTED;
  const Layout lo = layout_of(p);
  const StaticLayout sl = static_layout(p, lo);
  if (sl.total > kStaticScratchBytes) return SPA_ERR_UNSUPPORTED;
  const int B = p->batch, Hq = p->heads_q, Hkv = p->heads_kv, L = p->seq_len;
  if (B == 0 || L == 0) {
    // nothing to select; the caller's error word still reports this call
    if (error_word && cudaMemsetAsync(error_word, 0, sizeof(uint32_t), stream) != cudaSuccess)
      return SPA_ERR_CUDA;
    return SPA_OK;
  }
  if (!q || !k || !counts || !aligned16(q) || !aligned16(k) ||
      (reinterpret_cast<uintptr_t>(counts) & 3u))
    return SPA_ERR_INVALID;
  const long long list_elems = (long long)B * Hq * lo.list_per_head;
  if ((size_t)list_elems > lists_elems) return SPA_ERR_WORKSPACE;
  if (list_elems > 0 && (!lists || (reinterpret_cast<uintptr_t>(lists) & 3u)))
    return SPA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(static_scratch_ptr());
  if (!ws) return SPA_ERR_CUDA;
  // the header (error word) must start at zero; the rest is fully rewritten
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, stream) != cudaSuccess) return SPA_ERR_CUDA;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  const float scale = eff_scale(p);
  const long long BH = (long long)B * Hq, BKV = (long long)B * Hkv;
  CUtensorMap tq, tk, tqbar;
  if (!map_2d(&tq, kBF16, 2, q, 128, BH * L, 64, 128, kSW128) ||
      !map_2d(&tk, kBF16, 2, k, 128, BKV * L, 64, 128, kSW128) ||
      !map_3d(&tqbar, kBF16, 2, ws + sl.qbar, 128, lo.nqb, 2 * BH, 64, 128, kSW128))
    return SPA_ERR_CUDA;
  PoolArgs pa{B, Hq, Hkv, L, lo.nqb, lo.group, p->sink, p->local, scale,
              reinterpret_cast<float*>(ws + sl.xbar),
              reinterpret_cast<__nv_bfloat16*>(ws + sl.qbar), err, wait_ns(p),
              (lo.nqb + kPoolQbs - 1) / kPoolQbs};
  if (set_smem(anchor_pool_kernel, kPoolSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
  anchor_pool_kernel<<<(unsigned)(BH * pa.groups), kPoolThreads, kPoolSmemBytes, stream>>>(tq, tk,
                                                                                          pa);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  const int nmt = (lo.nqb + 127) / 128;
  const int key_end = std::max(0, lo.nqb * 128 - p->local);
  const int kt0 = p->sink / 128;
  const int kt_end = (key_end + 127) / 128;
  const int nchunk = key_end > p->sink
                         ? (kt_end - kt0 + kScanTilesPerChunk - 1) / kScanTilesPerChunk
                         : 0;
  if (nchunk > 0) {
    ScanArgs sa{B, Hq, Hkv, L, lo.nqb, lo.group, p->sink, p->local, p->theta,
                reinterpret_cast<const float*>(ws + sl.xbar),
                reinterpret_cast<uint32_t*>(ws + sl.mask), lo.nwords, err, wait_ns(p)};
    if (set_smem(stripe_scan_kernel, kScanSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    stripe_scan_kernel<<<dim3(nchunk, nmt, (unsigned)BH), kScanThreads, kScanSmemBytes,
                         stream>>>(tqbar, tk, sa);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  CompactArgs ca{(int)lo.nb, lo.nqb, L, p->sink, p->local, 1, p->step,
                 reinterpret_cast<const uint32_t*>(ws + sl.mask), lo.nwords, lists,
                 lo.list_per_head, lo.cap_a, counts};
  compact_kernel<<<(unsigned)lo.nb, kCompactThreads, 0, stream>>>(ca);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  if (error_word &&
      cudaMemcpyAsync(error_word, err, sizeof(uint32_t), cudaMemcpyDeviceToDevice, stream) !=
          cudaSuccess)
    return SPA_ERR_CUDA;
  return SPA_OK;
}

SPA_API size_t sparse_fp8_scales_floats(const spa_params* p) {
  if (validate(p) != SPA_OK) return 0;
  return (size_t)fp8_layout(p).floats;
}

SPA_API size_t sparse_fp8_scratch_bytes(const spa_params* p) {
  if (validate(p) != SPA_OK) return 0;
  return fp8_layout(p).scratch;
}

SPA_API spa_status sparse_fp8_quantize(const spa_params* p, const void* q, const void* k,
                                       const void* v, void* q8, void* k8, void* v8,
                                       float* scales, void* scratch, size_t scratch_bytes,
                                       cudaStream_t stream) {
  spa_status st = validate(p);
  if (st != SPA_OK) return st;
  const Fp8Layout f = fp8_layout(p);
  if (!scratch || !aligned16(scratch)) return SPA_ERR_INVALID;
  if (scratch_bytes < f.scratch) return SPA_ERR_WORKSPACE;
  const int B = p->batch, L = p->seq_len;
  if (B == 0 || L == 0) return SPA_OK;
  if (!q || !k || !v || !q8 || !k8 || !v8 || !scales || !aligned16(q) || !aligned16(k) ||
      !aligned16(v) || !aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(scales))
    return SPA_ERR_INVALID;
  const long long BH = (long long)B * p->heads_q, BKV = (long long)B * p->heads_kv;
  const int nqb = (L + 127) / 128;
  uint8_t* sc = static_cast<uint8_t*>(scratch);
  KmeanArgs ka{static_cast<const __nv_bfloat16*>(k), L, reinterpret_cast<double*>(sc + f.kpart),
               scales + f.kmean};
  kmean_partial_kernel<<<dim3(kKmeanChunks, (unsigned)BKV), 128, 0, stream>>>(ka);
  kmean_final_kernel<<<(unsigned)BKV, 128, 0, stream>>>(ka);
  if (cudaMemsetAsync(sc + f.kabs, 0, f.scratch - f.kabs, stream) != cudaSuccess)
    return SPA_ERR_CUDA;
  Fp8QuantArgs a{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                 static_cast<const __nv_bfloat16*>(v), scales + f.kmean, L, nqb,
                 static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), static_cast<uint8_t*>(v8),
                 scales + f.qs, scales + f.ks, scales + f.vs,
                 reinterpret_cast<uint32_t*>(sc + f.kabs), reinterpret_cast<uint32_t*>(sc + f.vabs)};
  fp8_quant_q_kernel<<<dim3(nqb, (unsigned)BH), 128, 0, stream>>>(a);
  fp8_kv_absmax_kernel<<<dim3(kFp8Chunks, (unsigned)BKV), 128, 0, stream>>>(a);
  fp8_kv_quant_kernel<<<dim3(kFp8Chunks, (unsigned)BKV), 128, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

}  // extern "C"
