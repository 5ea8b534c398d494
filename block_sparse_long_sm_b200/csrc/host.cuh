// host.cuh -- host-side helpers shared by the C-ABI translation units:
// argument validation, the closed-form workspace layout, TMA descriptor
// encoding.  Each translation unit gets its own (internal-linkage) copy.
#pragma once

#include <cmath>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "common.cuh"
#include "tiles.cuh"

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
  int tc = 0;                       // candidate-tile constant tmask_c(sink, local)
  long long tmask_per_head = 0;     // candidate-tile masks per (b, h)
  size_t tmask = 0;                 // uint4 [B*Hq][tmask_per_head]
  int tbit_words = 0;               // words of one tile bitmap
  size_t tbits = 0;                 // uint32 [B*Hq*nqb][3][tbit_words]
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
  if (p->mode != SPA_MODE_DENSE) {
    // one 128-bit mask per (b, h, query block, candidate key tile): the
    // selection the paired attention kernel reads its tiles from
    lo.tc = tmask_c(p->sink, p->local);
    lo.tmask_per_head = tmask_prefix(lo.nqb, lo.tc);
    lo.tmask = take((size_t)bh * lo.tmask_per_head * 16);
    lo.tbit_words = lo.nqb > 0 ? tmask_bit_words(lo.nqb, lo.tc) : 0;
    lo.tbits = take((size_t)lo.nb * 3 * lo.tbit_words * 4);
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

// The plan's geometry and lists as the tile-walking kernels read them.
TileGeom tile_geom(const spa_params* p, const Layout& lo, uint8_t* ws) {
  TileGeom g;
  g.Hq = p->heads_q;
  g.Hkv = p->heads_kv;
  g.L = p->seq_len;
  g.nqb = lo.nqb;
  g.group = lo.group;
  g.sink = p->sink;
  g.local = p->local;
  g.mode = p->mode == SPA_MODE_ANCHOR ? kModeAnchor
                                      : (p->mode == SPA_MODE_SALE ? kModeSale : kModeDense);
  g.counts = reinterpret_cast<const int*>(ws + lo.counts);
  g.lists = reinterpret_cast<const int*>(ws + lo.lists);
  g.list_per_head = lo.list_per_head;
  g.cap_a = lo.cap_a;
  g.list_unit = lo.unit;
  return g;
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

