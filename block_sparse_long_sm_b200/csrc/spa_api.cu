// spa_api.cu -- the C ABI declared in include/spa.h: argument validation,
// closed-form workspace layout, TMA descriptor encoding and kernel launches.
// Nothing here allocates device memory.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "attn.cuh"
#include "attn_pair.cuh"
#include "ptx.cuh"
#include "sale.cuh"
#include "select.cuh"

namespace {

using namespace spa;

constexpr size_t kHeaderBytes = 256;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  bool ok = false;
  int nqb = 0, nkb = 0, group = 1, unit = 1;
  long long nb = 0;                 // query blocks
  long long list_per_head = 0;      // list elements per (b, h)
  long long cap_a = 0;
  int nwords = 0;                   // bitmask words per block row
  size_t counts = 0, lists = 0, xbar = 0, qbar = 0, mask = 0;
  size_t kpart = 0, kmean = 0, q8 = 0, k8 = 0, sq = 0, sk = 0;
  bool paired = false;              // two q heads per attention CTA (Hq / Hkv even)
  bool fused = false;               // ANCHOR: scan and compaction in one kernel
  size_t pair_counts = 0, pair_lists = 0;
  size_t total = 0;
};

// The fused ANCHOR selection keeps each selection group inside one warp.
bool fused_step(int step) { return step >= 1 && step <= 32 && (step & (step - 1)) == 0; }

spa_status validate(const spa_params* p) {
  if (!p) return SPA_ERR_INVALID;
  if (p->batch < 0 || p->heads_q < 1 || p->heads_kv < 1 || p->seq_len < 0)
    return SPA_ERR_INVALID;
  if (p->heads_q % p->heads_kv != 0) return SPA_ERR_INVALID;
  if (p->head_dim != 128) return SPA_ERR_UNSUPPORTED;
  if (p->causal != 1) return SPA_ERR_UNSUPPORTED;
  if (p->block_q != 128) return SPA_ERR_UNSUPPORTED;
  if (p->step < 1) return SPA_ERR_INVALID;
  if (p->sink < 0) return SPA_ERR_INVALID;
  if (p->local < p->block_q || p->local % p->block_q != 0) return SPA_ERR_INVALID;
  if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale)) return SPA_ERR_INVALID;
  const long long rows = (long long)p->batch * (p->heads_q > p->heads_kv ? p->heads_q : p->heads_kv) *
                         (long long)p->seq_len;
  if (rows >= (1LL << 31)) return SPA_ERR_UNSUPPORTED;
  if ((long long)p->batch * p->heads_q > 65535) return SPA_ERR_UNSUPPORTED;
  switch (p->mode) {
    case SPA_MODE_ANCHOR:
      if (p->block_k != 1) return SPA_ERR_UNSUPPORTED;
      if (std::isnan(p->theta)) return SPA_ERR_INVALID;
      break;
    case SPA_MODE_SALE:
      if (p->block_k != 16 && p->block_k != 32 && p->block_k != 64 && p->block_k != 128)
        return SPA_ERR_UNSUPPORTED;
      if (p->sink % p->block_k != 0) return SPA_ERR_UNSUPPORTED;
      if (!(p->tau > 0.f && p->tau <= 1.f)) return SPA_ERR_INVALID;
      if (p->tau_per_head) {
        if (p->heads_q > SPA_MAX_TAU_HEADS) return SPA_ERR_UNSUPPORTED;
        for (int h = 0; h < p->heads_q; ++h)
          if (!(p->tau_per_head[h] > 0.f && p->tau_per_head[h] <= 1.f)) return SPA_ERR_INVALID;
      }
      if (p->seq_len > 262144) return SPA_ERR_UNSUPPORTED;
      break;
    case SPA_MODE_DENSE:
      break;
    default:
      return SPA_ERR_INVALID;
  }
  return SPA_OK;
}

Layout layout_of(const spa_params* p) {
  Layout lo;
  const int L = p->seq_len;
  lo.nqb = (L + 127) / 128;
  lo.group = p->heads_q / p->heads_kv;
  lo.nb = (long long)p->batch * p->heads_q * lo.nqb;
  lo.cap_a = (long long)p->local + p->sink;
  const long long bh = (long long)p->batch * p->heads_q;
  const long long bkv = (long long)p->batch * p->heads_kv;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  if (p->mode == SPA_MODE_ANCHOR) {
    lo.unit = 1;
    lo.list_per_head = cap_prefix(lo.nqb, 128, lo.cap_a);
    lo.nwords = ((L + 127) / 128) * 4;
    lo.counts = take(lo.nb * 4);
    lo.lists = take((size_t)bh * lo.list_per_head * 4);
    lo.xbar = take(lo.nb * 4);
    lo.qbar = take((size_t)2 * lo.nb * 128 * 2);
    lo.fused = fused_step(p->step);
    if (!lo.fused) lo.mask = take((size_t)lo.nb * lo.nwords * 4);
  } else if (p->mode == SPA_MODE_SALE) {
    lo.unit = p->block_k;
    lo.nkb = (L + p->block_k - 1) / p->block_k;
    lo.list_per_head = cap_prefix(lo.nqb, 128, lo.cap_a) / p->block_k;
    lo.nwords = (lo.nkb + 31) / 32;
    lo.counts = take(lo.nb * 4);
    lo.lists = take((size_t)bh * lo.list_per_head * 4);
    lo.kpart = take((size_t)bkv * kKmeanChunks * 128 * 8);
    lo.kmean = take((size_t)bkv * 128 * 4);
    lo.q8 = take((size_t)bh * L * 128);
    lo.k8 = take((size_t)bkv * L * 128);
    lo.sq = take(lo.nb * 4);
    lo.sk = take((size_t)bkv * lo.nkb * 4);
    lo.mask = take((size_t)lo.nb * lo.nwords * 4);
  } else {
    lo.unit = 1;
    lo.counts = take(lo.nb * 4);
  }
  lo.paired = (lo.group % 2) == 0;
  if (lo.paired && p->mode != SPA_MODE_DENSE) {
    // tagged union lists of head pairs and their sizes, for the paired
    // attention kernel (opaque scratch)
    lo.pair_counts = take((lo.nb / 2) * 4);
    lo.pair_lists = take((size_t)(bh / 2) * lo.list_per_head * 4);
  }
  lo.total = off;
  lo.ok = true;
  return lo;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// ---------------------------------------------------------------------------
// TMA descriptors
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D map over a row-major [rows x cols] matrix of `esize`-byte elements.
bool map_2d(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base,
            uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
            CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over [d2][d1][cols].
bool map_3d(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base,
            uint64_t cols, uint64_t d1, uint64_t d2, uint32_t box_cols, uint32_t box_d1,
            CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cols, d1, d2};
  const cuuint64_t strides[2] = {cols * esize, cols * esize * d1};
  const cuuint32_t box[3] = {box_cols, box_d1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapDataType kI8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
constexpr CUtensorMapSwizzle kSW128 = CU_TENSOR_MAP_SWIZZLE_128B;

float eff_scale(const spa_params* p) {
  return p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(128.0f);
}
uint64_t wait_ns(const spa_params* p) {
  return (uint64_t)(p->wait_limit_us ? p->wait_limit_us : 250000u) * 1000ull;
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

spa_status common_checks(const spa_params* p, const void* workspace, size_t ws_bytes,
                         Layout* lo) {
  spa_status st = validate(p);
  if (st != SPA_OK) return st;
  *lo = layout_of(p);
  if (!workspace || !aligned16(workspace)) return SPA_ERR_INVALID;
  if (ws_bytes < lo->total) return SPA_ERR_WORKSPACE;
  return SPA_OK;
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
                reinterpret_cast<__nv_bfloat16*>(ws + lo.qbar), err, wait_ns(p)};
    if (set_smem(anchor_pool_kernel, kPoolSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    anchor_pool_kernel<<<(unsigned)lo.nb, kPoolThreads, kPoolSmemBytes, stream>>>(tq, tk, pa);
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
                    lo.paired ? reinterpret_cast<int*>(ws + lo.pair_counts) : nullptr,
                    lo.paired ? reinterpret_cast<uint32_t*>(ws + lo.pair_lists) : nullptr, err,
                    wait_ns(p)};
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
    sale_scan_kernel<<<(unsigned)(BKV * lo.nqb * chunks), kSaleThreads, kSaleSmemBytes,
                       stream>>>(tq8, tk8, sa);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  if (lo.paired) {
    // one pass writes both heads' lists and their tagged union list
    PairCompactArgs pc{lo.nqb, Hq, p->sink, p->local, lo.unit, p->step,
                       reinterpret_cast<const uint32_t*>(ws + lo.mask), lo.nwords,
                       reinterpret_cast<int*>(ws + lo.lists), reinterpret_cast<int*>(ws + lo.counts),
                       reinterpret_cast<uint32_t*>(ws + lo.pair_lists), lo.list_per_head, lo.cap_a,
                       reinterpret_cast<int*>(ws + lo.pair_counts)};
    pair_compact_kernel<<<(unsigned)(lo.nb / 2), kCompactThreads, 0, stream>>>(pc);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  } else {
    CompactArgs ca{(int)lo.nb, lo.nqb, L, p->sink, p->local, lo.unit, p->step,
                   reinterpret_cast<const uint32_t*>(ws + lo.mask), lo.nwords,
                   reinterpret_cast<int*>(ws + lo.lists), lo.list_per_head, lo.cap_a,
                   reinterpret_cast<int*>(ws + lo.counts)};
    compact_kernel<<<(unsigned)lo.nb, kCompactThreads, 0, stream>>>(ca);
    if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  }
  return SPA_OK;
}

SPA_API spa_status sparse_prefill_attn(const spa_params* p, const void* q, const void* k, const void* v,
                               void* workspace, size_t workspace_bytes, void* o, float* lse,
                               cudaStream_t stream) {
  Layout lo;
  spa_status st = common_checks(p, workspace, workspace_bytes, &lo);
  if (st != SPA_OK) return st;
  const int B = p->batch, Hq = p->heads_q, Hkv = p->heads_kv, L = p->seq_len;
  if (B == 0 || L == 0) return SPA_OK;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SPA_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SPA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const long long BH = (long long)B * Hq, BKV = (long long)B * Hkv;
  CUtensorMap tq, tk, tkg, tv, tvg;
  if (!map_2d(&tq, kBF16, 2, q, 128, BH * L, 64, 128, kSW128) ||
      !map_2d(&tk, kBF16, 2, k, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tkg, kBF16, 2, k, 128, BKV * L, 64, 1, kSW128) ||
      !map_2d(&tv, kBF16, 2, v, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tvg, kBF16, 2, v, 128, BKV * L, 64, 1, kSW128))
    return SPA_ERR_CUDA;
  AttnArgs aa;
  aa.B = B; aa.Hq = Hq; aa.Hkv = Hkv; aa.L = L; aa.nqb = lo.nqb; aa.group = lo.group;
  aa.sink = p->sink; aa.local = p->local;
  aa.mode = p->mode == SPA_MODE_ANCHOR ? kModeAnchor : (p->mode == SPA_MODE_SALE ? kModeSale : kModeDense);
  aa.bk = p->block_k;
  aa.sl2 = eff_scale(p) * 1.4426950408889634f;
  aa.counts = reinterpret_cast<const int*>(ws + lo.counts);
  aa.lists = reinterpret_cast<const int*>(ws + lo.lists);
  aa.list_per_head = lo.list_per_head;
  aa.cap_a = lo.cap_a;
  aa.list_unit = lo.unit;
  aa.pair_counts = reinterpret_cast<const int*>(ws + lo.pair_counts);
  aa.pair_lists = reinterpret_cast<const uint32_t*>(ws + lo.pair_lists);
  aa.pair_per_head = lo.list_per_head;
  aa.o = static_cast<__nv_bfloat16*>(o);
  aa.lse = lse;
  aa.err = reinterpret_cast<uint32_t*>(ws);
  aa.wait_ns = wait_ns(p);
  aa.debug = p->debug_flags;
  if (lo.paired) {
    if (set_smem(sparse_attn_pair_kernel, kPairSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_pair_kernel<<<(unsigned)(lo.nb / 2), kPairThreads, kPairSmemBytes, stream>>>(
        tq, tk, tkg, tv, tvg, aa);
  } else {
    if (set_smem(sparse_attn_kernel, kAttnSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_kernel<<<(unsigned)lo.nb, kAttnThreads, kAttnSmemBytes, stream>>>(tq, tk, tkg,
                                                                                 tv, tvg, aa);
  }
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
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

// Device address of g_static_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in, not a device address).
void* static_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
    g_static_ptr[dev] = ptr;
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
  if (B == 0 || L == 0) return SPA_OK;
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
              reinterpret_cast<__nv_bfloat16*>(ws + sl.qbar), err, wait_ns(p)};
  if (set_smem(anchor_pool_kernel, kPoolSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
  anchor_pool_kernel<<<(unsigned)lo.nb, kPoolThreads, kPoolSmemBytes, stream>>>(tq, tk, pa);
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

}  // extern "C"
