// attn_pair.cuh -- sparse causal attention forward for two q heads of one GQA
// group at once, sharing every K/V tile (used when Hq / Hkv is even).
//
// Same computation as sparse_attn_kernel (AnchorAttention Sec. 3.4 /
// SALE Computation Pass, FlashAttention online softmax), organised so that
// the exponentials of one head overlap the tensor-core work of the other.
//
// One CTA = (b, kv head, query block, head pair (2p, 2p+1)).  Its key tiles:
//   sink tiles       keys [0, sink_end), contiguous;
//   dense tiles      candidate tiles (128 aligned keys) of which either
//                    head keeps at least tile_dense_min keys (64 of keys
//                    selected one by one, all 128 of key blocks): loaded
//                    contiguously, the keys a head did not keep masked out of
//                    its softmax;
//   gathered tiles   the kept keys of the sparser candidate tiles, 128 at a
//                    time (the last one padded), copied row by row, or 16
//                    consecutive keys at once;
//   local tiles      keys [ls, row0 + 128), contiguous; the last one is the
//                    causally masked diagonal.
// They are loaded in the order sink, dense, local before the diagonal,
// gathered, diagonal: the gathered tiles' keys are being collected while the
// first tiles load, and the diagonal is always the last tile.
// The candidate tiles come from the plan's tile masks (one 128-bit keep mask
// per head, query block and candidate tile), so the kernel reads 32 bytes of
// selection per 128 candidate keys and no index list.  Attention over a key
// set does not depend on the order of its tiles.
//
// Roles (384 threads, 3 warpgroups):
//   warp 8       producer: Q of both heads once; per tile it picks the keys
//                (sink, dense, gathered or local), publishes a descriptor and
//                the two heads' column masks through the tile's tag barrier,
//                and loads the tile with TMA into rings of 3 (K) and 2 (V)
//                stages: contiguous tiles as two 64-column boxes per operand.
//                Gathered tiles are copied row by row with TMA gather4 (four
//                rows per instruction, issued by the 32 lanes);
//   warps 10,11  collectors: each turns the masks of half of the sparse
//                candidate tiles (bitmap words of one parity) into gathered
//                tiles of 128 keys and their column masks, one buffer ahead
//                of the producer;//   warp 9       TMEM allocation and the single MMA-issuing thread, in the
//                order PV_A(t), QK_A(t+1), PV_B(t), QK_B(t+1), so the tensor
//                core works on one head while the other head's softmax runs.
//                P is written by the softmax into the first 64 columns of its
//                own S accumulator and read there by the PV GEMM; the next QK
//                GEMM into the same columns is issued after that PV GEMM
//                (tcgen05 MMAs of one thread execute in issue order);
//   warps 0-3 / 4-7  softmax of head A / B, thread = query row = TMEM lane.
//
// The number of tiles depends on the masks, so every tile carries a
// descriptor (valid columns, causal, masked, last, gathered); the MMA and
// softmax warps stop after the tile marked last (a local tile: there is
// always at least one, the diagonal).
//
// TMEM columns: S_A [0,128) (P_A in [0,64)), S_B [128,256) (P_B in
// [128,192)), O_A [256,384), O_B [384,512).
#pragma once

#include "attn.cuh"
#include "ptx.cuh"

namespace spa {

constexpr int kPairKStages = 3;
constexpr int kPairVStages = 2;
constexpr int kPairThreads = 384;   // 3 warpgroups: softmax A, softmax B, load + MMA
constexpr uint32_t kPairBarBytes = 2048u;   // barriers, masks, descriptors, collected keys
constexpr uint32_t kPairSmemBytes =
    1024u + 2u * kTileBytes + (kPairKStages + kPairVStages) * kTileBytes + kPairBarBytes;
static_assert(kPairSmemBytes <= 232448u, "more shared memory than a CTA may use");

// tile descriptor bits (bits 0-8: valid columns)
constexpr uint32_t kDescCausal = 1u << 9;
constexpr uint32_t kDescMasked = 1u << 10;
constexpr uint32_t kDescLast = 1u << 11;
constexpr uint32_t kDescGather = 1u << 12;

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// 32 columns from the first 16 registers of two arrays.
__device__ __forceinline__ void tmem_st32_halves(uint32_t taddr, const uint32_t* a,
                                                 const uint32_t* b) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
      "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]),
      "r"(a[15]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(b[4]), "r"(b[5]), "r"(b[6]),
      "r"(b[7]), "r"(b[8]), "r"(b[9]), "r"(b[10]), "r"(b[11]), "r"(b[12]), "r"(b[13]),
      "r"(b[14]), "r"(b[15])
      : "memory");
}

struct PairItem {
  AttnItem it;          // geometry; it.h is head A
  int n_ct;             // candidate tiles of the block
  const uint4* ma;      // head A's tile masks of this block
  const uint4* mb;      // head B's
  const uint32_t* ba;   // head A's tile bitmaps of this block (non-empty, dense, full)
  const uint32_t* bb;   // head B's
};

__device__ __forceinline__ PairItem pair_item(const AttnArgs& a, int x) {
  PairItem pi;
  AttnItem& it = pi.it;
  const int ppk = a.group / 2;                 // head pairs per kv head
  const int per_kv = a.nqb * ppk;
  const int bkv = x / per_kv;
  const int rem = x - bkv * per_kv;
  it.qb = a.nqb - 1 - rem / ppk;
  const int pp = rem % ppk;
  it.b = bkv / a.Hkv;
  it.kvh = bkv - it.b * a.Hkv;
  it.h = it.kvh * a.group + 2 * pp;
  it.row0 = it.qb * 128;
  it.le = min(it.row0 + 128, a.L);
  it.ls = max(0, it.row0 + 128 - a.local);
  it.sink_end = min(a.sink, it.ls);
  it.n_sel = 0;
  it.n_sel_t = 0;
  it.list_off = 0;
  pi.n_ct = 0;
  pi.ma = nullptr;
  pi.mb = nullptr;
  pi.ba = nullptr;
  pi.bb = nullptr;
  if (a.mode == kModeDense) {
    it.n_sink_t = 0;
    it.loc_start = 0;
  } else {
    it.n_sink_t = (it.sink_end + 127) / 128;
    it.loc_start = it.ls;
    pi.n_ct = tmask_tiles(it.qb, a.tc);
    const long long bhA = (long long)it.b * a.Hq + it.h;
    pi.ma = a.tmask + bhA * a.tmask_per_head + tmask_prefix(it.qb, a.tc);
    pi.mb = pi.ma + a.tmask_per_head;
    pi.ba = a.tbits + (bhA * a.nqb + it.qb) * 3 * a.tbit_words;
    pi.bb = pi.ba + (long long)a.nqb * 3 * a.tbit_words;
  }
  it.n_loc_t = (it.le - it.loc_start + 127) / 128;
  return pi;
}

__global__ void __launch_bounds__(kPairThreads, 1)
sparse_attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_kg,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_vg,
                        const __grid_constant__ CUtensorMap tm_k16,
                        const __grid_constant__ CUtensorMap tm_v16, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;                                      // Q_A, then Q_B
  auto s_k = [&](int st) { return s_base + kTileBytes * (2 + st); };
  auto s_v = [&](int st) { return s_base + kTileBytes * (2 + kPairKStages + st); };
  uint8_t* bar_area = smem + kTileBytes * (2 + kPairKStages + kPairVStages);
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_q = b0;
  auto bar_kfull = [&](int st) { return b0 + 8u * (1 + st); };
  auto bar_kempty = [&](int st) { return b0 + 8u * (1 + kPairKStages + st); };
  auto bar_vfull = [&](int st) { return b0 + 8u * (1 + 2 * kPairKStages + st); };
  auto bar_vempty = [&](int st) { return b0 + 8u * (1 + 2 * kPairKStages + kPairVStages + st); };
  const uint32_t bar_sfull0 = b0 + 8u * (1 + 2 * kPairKStages + 2 * kPairVStages);   // [2 heads]
  const uint32_t bar_pfull0 = bar_sfull0 + 16u;                                       // [2 heads]
  const uint32_t bar_odone = bar_sfull0 + 32u;
  const uint32_t bar_drain = bar_sfull0 + 40u;
  const uint32_t bar_stall = bar_sfull0 + 48u;
  const uint32_t bar_tag0 = bar_sfull0 + 56u;                                         // [vstages]
  uint32_t* tags = reinterpret_cast<uint32_t*>(bar_area + 256);   // [vstage][head][4 words]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 320);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  // per V slot, the descriptor of the tile in it: valid columns (bits 0-8)
  // and the kDesc* flags; written by the producer before it arrives on the
  // slot's tag barrier
  uint32_t* tdesc = reinterpret_cast<uint32_t*>(bar_area + 336);
  // Gathered tiles are collected by warps 10 and 11, one buffer each: the
  // keys row by row (index | head A kept it << 30 | head B kept it << 31;
  // padding rows repeat row 0's key with neither head's bit), the tile's
  // column masks (words 0-3 head A, 4-7 head B) and the number of keys (0:
  // that collector has no more).
  const uint32_t bar_cfull0 = bar_sfull0 + 72u;    // [2] collector -> producer
  const uint32_t bar_cempty0 = bar_sfull0 + 88u;   // [2] producer -> collector
  uint32_t* ccount = tdesc + 2;                                     // [2]
  uint32_t* cmask = reinterpret_cast<uint32_t*>(bar_area + 384);    // [2][8]
  uint32_t* cbuf = reinterpret_cast<uint32_t*>(bar_area + 512);     // [2][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int st = 0; st < kPairKStages; ++st) {
      mbar_init(bar_kfull(st), 1);
      mbar_init(bar_kempty(st), 1);
    }
    for (int st = 0; st < kPairVStages; ++st) {
      mbar_init(bar_vfull(st), 1);
      mbar_init(bar_vempty(st), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull0 + 8u * i, 1);
      mbar_init(bar_pfull0 + 8u * i, 128);
    }
    for (int st = 0; st < kPairVStages; ++st) mbar_init(bar_tag0 + 8u * st, 1);
    for (int c = 0; c < 2; ++c) {
      mbar_init(bar_cfull0 + 8u * c, 1);
      mbar_init(bar_cempty0 + 8u * c, 1);
    }
    mbar_init(bar_odone, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_kg);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_vg);
    prefetch_tensormap(&tm_k16);
    prefetch_tensormap(&tm_v16);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};

  const PairItem pi = pair_item(a, blockIdx.x);
  const AttnItem& it = pi.it;
  const int kv_row0 = (it.b * a.Hkv + it.kvh) * a.L;

  // Register split: the load/MMA warpgroup (warps 8-11, executing this one
  // instruction together) needs few registers, the softmax warpgroups hold a
  // full 128-column S row each.  Launched with 168 per thread (384 threads):
  // 128 x 88 + 256 x 208 = 384 x 168.
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
  if (warp == 8) {
    // ------------------------------------------------------------- producer
    int issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 2 * kTileBytes);
      const int qrow = (it.b * a.Hq + it.h) * a.L + it.row0;
      tma_load_2d(s_q, &tm_q, bar_q, 0, qrow);
      tma_load_2d(s_q + kHalfBytes, &tm_q, bar_q, 64, qrow);
      tma_load_2d(s_q + kTileBytes, &tm_q, bar_q, 0, qrow + a.L);
      tma_load_2d(s_q + kTileBytes + kHalfBytes, &tm_q, bar_q, 64, qrow + a.L);
    }
    const int kt0 = a.sink / 128;
    const int W = a.tbit_words;
    const int nw = (pi.n_ct + 31) / 32;            // bitmap words of this block
    // The bitmaps are read 32 words (1024 tiles) at a time, lane l holding
    // word l of the chunk.
    // Dense tiles: set in either head's dense bitmap; full when both heads
    // keep all 128 keys.
    int dchunk = 0, dwi = -1;
    uint32_t dword = 0u, fword = 0u;               // this lane's word of the chunk
    uint32_t dbits = 0u, fbits = 0u;               // the word in use: tiles left, full tiles
    auto load_dense_chunk = [&](int c) {
      const int wi = 32 * c + lane;
      dword = fword = 0u;
      if (wi < nw) {
        dword = pi.ba[W + wi] | pi.bb[W + wi];
        fword = pi.ba[2 * W + wi] & pi.bb[2 * W + wi];
      }
    };
    // next dense tile (candidate index) and whether it is full, or -1
    auto next_dense = [&](bool& full) -> int {
      while (dbits == 0u) {
        if (32 * dchunk >= nw) return -1;
        const uint32_t cand = __ballot_sync(0xffffffffu, dword != 0u) &
                              (dwi < 31 ? (0xffffffffu << (dwi + 1)) : 0u);
        if (cand) {
          dwi = __ffs(cand) - 1;
          dbits = __shfl_sync(0xffffffffu, dword, dwi);
          fbits = __shfl_sync(0xffffffffu, fword, dwi);
        } else {
          ++dchunk;
          dwi = -1;
          if (32 * dchunk < nw) load_dense_chunk(dchunk);
        }
      }
      const int b = __ffs(dbits) - 1;
      dbits &= dbits - 1u;
      full = ((fbits >> b) & 1u) != 0u;
      return 32 * (32 * dchunk + dwi) + b;
    };
    if (nw > 0) load_dense_chunk(0);
    // Tile order: sink, dense, the local tiles before the diagonal, gathered
    // (the collectors fill their first buffers meanwhile), the diagonal.
    int phase = 0;        // 0 sink, 1 dense, 2 early local, 3 gathered, 4 diagonal
    int n_sink = 0, n_loc = 0;
    int col = 0;                                   // collector to take the next gathered tile from
    int taken0 = 0, taken1 = 0;                    // buffers taken from each collector
    bool cdone0 = false, cdone1 = false;
    // The next tile, prepared while the previous tile's loads are in flight:
    // its descriptor, its first key (contiguous tiles), lane l's four rows
    // 4 l .. 4 l + 3 (gathered tiles) and, in lanes 0-7, word l of the two
    // heads' column masks (0-3 head A, 4-7 head B).
    uint32_t nx_desc = 0u;
    int nx_key0 = 0;
    int nx_row[4] = {0, 0, 0, 0};
    uint32_t nx_mask = 0u;
    auto prepare = [&]() -> bool {
      nx_desc = 0u;
      if (phase == 0) {
        if (n_sink < it.n_sink_t) {
          nx_key0 = 128 * n_sink++;
          nx_desc = static_cast<uint32_t>(min(128, it.sink_end - nx_key0));
          return true;
        }
        phase = 1;
      }
      if (phase == 1) {
        bool full = false;
        const int j = nw > 0 ? next_dense(full) : -1;
        if (j >= 0) {
          if (!full && lane < 8)
            nx_mask = reinterpret_cast<const uint32_t*>(lane < 4 ? pi.ma + j : pi.mb + j)[lane & 3];
          nx_key0 = 128 * (kt0 + j);
          nx_desc = 128u | (full ? 0u : kDescMasked);
          return true;
        }
        phase = 2;
      }
      if (phase == 2) {
        if (n_loc + 1 < it.n_loc_t) {
          nx_key0 = it.loc_start + 128 * n_loc++;
          nx_desc = static_cast<uint32_t>(min(128, it.le - nx_key0)) |
                    (nx_key0 == it.row0 ? kDescCausal : 0u);
          return true;
        }
        phase = 3;
      }
      if (phase == 3) {
        // the gathered tiles the two collector warps prepare, taken in turn
        while (!(cdone0 && cdone1)) {
          if (col == 0 ? cdone0 : cdone1) col ^= 1;
          const int c = col;
          const int tk = c == 0 ? taken0++ : taken1++;
          if (!warp_wait(bar_cfull0 + 8u * c, tk & 1, wc)) return false;
          const int n = static_cast<int>(ccount[c]);
          if (n == 0) {                            // that collector is done
            if (c == 0) cdone0 = true; else cdone1 = true;
            continue;
          }
          const uint32_t* buf = cbuf + 128 * c;
#pragma unroll
          for (int r = 0; r < 4; ++r)
            nx_row[r] = kv_row0 + static_cast<int>(buf[4 * lane + r] & 0x3FFFFFFFu);
          if (lane < 8) nx_mask = cmask[8 * c + lane];
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_cempty0 + 8u * c);
          col = c ^ 1;
          nx_desc = 128u | kDescMasked | kDescGather;
          return true;
        }
        phase = 4;
      }
      nx_key0 = it.loc_start + 128 * n_loc++;
      nx_desc = static_cast<uint32_t>(min(128, it.le - nx_key0)) |
                (nx_key0 == it.row0 ? kDescCausal : 0u) | (n_loc == it.n_loc_t ? kDescLast : 0u);
      return true;
    };
    for (int t = 0;; ++t) {
      if (!prepare()) break;
      const int ks = t % kPairKStages, vs = t % kPairVStages;
      if (t >= kPairKStages &&
          !warp_wait(bar_kempty(ks), ((t / kPairKStages) - 1) & 1, wc))
        break;
      if (t >= kPairVStages &&
          !warp_wait(bar_vempty(vs), ((t / kPairVStages) - 1) & 1, wc))
        break;
      const uint32_t desc = nx_desc;
      // publish the tile: its masks, then its descriptor
      if ((desc & kDescMasked) && lane < 8) tags[vs * 8 + lane] = nx_mask;
      __syncwarp();
      if (lane == 0) {
        tdesc[vs] = desc;
        mbar_arrive(bar_tag0 + 8u * vs);
      }
      const uint32_t kf = bar_kfull(ks), vf = bar_vfull(vs);
      if (lane == 0) {
        mbar_arrive_expect_tx(kf, kTileBytes);
        mbar_arrive_expect_tx(vf, kTileBytes);
      }
      __syncwarp();
      if (desc & kDescGather) {
        // rows 4 l .. 4 l + 3 of the tile from lane l: one gather4 per operand
        // half; a 16-row chunk (lanes 4 c .. 4 c + 3) of consecutive keys, as
        // every chunk of a selection in 16-key blocks is, is one tiled box
        // per operand half from its first lane instead
        const uint32_t roff = lane * 4u * 128u;
        const int prev_last = __shfl_up_sync(0xffffffffu, nx_row[3], 1);
        const bool seq = nx_row[1] == nx_row[0] + 1 && nx_row[2] == nx_row[0] + 2 &&
                         nx_row[3] == nx_row[0] + 3 && ((lane & 3) == 0 || prev_last + 1 == nx_row[0]);
        const uint32_t seq_bits = __ballot_sync(0xffffffffu, seq);
        if (((seq_bits >> (lane & ~3)) & 0xFu) != 0xFu) {
          tma_gather4(s_k(ks) + roff, &tm_kg, kf, 0, nx_row[0], nx_row[1], nx_row[2], nx_row[3]);
          tma_gather4(s_k(ks) + kHalfBytes + roff, &tm_kg, kf, 64, nx_row[0], nx_row[1], nx_row[2],
                      nx_row[3]);
          tma_gather4(s_v(vs) + roff, &tm_vg, vf, 0, nx_row[0], nx_row[1], nx_row[2], nx_row[3]);
          tma_gather4(s_v(vs) + kHalfBytes + roff, &tm_vg, vf, 64, nx_row[0], nx_row[1], nx_row[2],
                      nx_row[3]);
        } else if ((lane & 3) == 0) {
          tma_load_2d(s_k(ks) + roff, &tm_k16, kf, 0, nx_row[0]);
          tma_load_2d(s_k(ks) + kHalfBytes + roff, &tm_k16, kf, 64, nx_row[0]);
          tma_load_2d(s_v(vs) + roff, &tm_v16, vf, 0, nx_row[0]);
          tma_load_2d(s_v(vs) + kHalfBytes + roff, &tm_v16, vf, 64, nx_row[0]);
        }
      } else if (lane == 0) {
        tma_load_2d(s_k(ks), &tm_k, kf, 0, kv_row0 + nx_key0);
        tma_load_2d(s_k(ks) + kHalfBytes, &tm_k, kf, 64, kv_row0 + nx_key0);
        tma_load_2d(s_v(vs), &tm_v, vf, 0, kv_row0 + nx_key0);
        tma_load_2d(s_v(vs) + kHalfBytes, &tm_v, vf, 64, kv_row0 + nx_key0);
      }
      __syncwarp();
      issued = t + 1;
      if (desc & kDescLast) break;
    }
    if (lane == 0) {   // no copy may still be in flight when the CTA exits
      mbar_drain(bar_q, 0, a.wait_ns);
      for (int t = max(0, issued - kPairKStages); t < issued; ++t)
        mbar_drain(bar_kfull(t % kPairKStages), (t / kPairKStages) & 1, a.wait_ns);
      for (int t = max(0, issued - kPairVStages); t < issued; ++t)
        mbar_drain(bar_vfull(t % kPairVStages), (t / kPairVStages) & 1, a.wait_ns);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      if (a.debug & 1u) ok = mbar_wait(bar_stall, 0, wc);   // never signalled: test hook
      if (ok) ok = mbar_wait(bar_q, 0, wc);
      auto qk = [&](int t, int hd) {
        const int ks = t % kPairKStages;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
          mma_bf16_ss(tmem + 128u * hd, smem_desc_sw128(s_q + hd * kTileBytes + off, 16),
                      smem_desc_sw128(s_k(ks) + off, 16), kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull0 + 8u * hd);
      };
      auto pv = [&](int t, int hd) {
        const int vs = t % kPairVStages;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = smem_desc_sw128(s_v(vs) + kk * 2048u, kHalfBytes);
          mma_bf16_ts(tmem + 256u + 128u * hd, tmem + 128u * hd + 8u * kk, bd, kIdescPV,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
      };
      if (ok) {
        if ((ok = mbar_wait(bar_kfull(0), 0, wc))) {
          tc_fence_after();
          qk(0, 0);
          qk(0, 1);
          mma_commit(bar_kempty(0));
        }
      }
      for (int t = 0; ok; ++t) {
        const int vs = t % kPairVStages;
        // tile t's descriptor was written before its loads were armed, and
        // kfull of tile t has been observed (QK(t) is issued)
        const bool more = a.mode == kModeDense ? t + 1 < it.n_loc_t : (tdesc[vs] & kDescLast) == 0u;
        // head A: PV(t), then QK(t+1)
        if (!(ok = mbar_wait(bar_pfull0, t & 1, wc))) break;
        if (!(ok = mbar_wait(bar_vfull(vs), (t / kPairVStages) & 1, wc))) break;
        tc_fence_after();
        pv(t, 0);
        if (more) {
          const int ks = (t + 1) % kPairKStages;
          if (!(ok = mbar_wait(bar_kfull(ks), ((t + 1) / kPairKStages) & 1, wc))) break;
          tc_fence_after();
          qk(t + 1, 0);
        }
        // head B: PV(t), then QK(t+1)
        if (!(ok = mbar_wait(bar_pfull0 + 8u, t & 1, wc))) break;
        tc_fence_after();
        pv(t, 1);
        mma_commit(bar_vempty(vs));
        if (more) {
          qk(t + 1, 1);
          mma_commit(bar_kempty((t + 1) % kPairKStages));
        } else {
          mma_commit(bar_odone);
          break;
        }
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- collectors (warps 10, 11)
    // Collector c gathers the keys of the sparse tiles in the bitmap words
    // w with w % 2 == c into its buffer, 128 at a time, with the tile's
    // column masks, and hands each buffer to the producer (a count of 0
    // ends it).
    const int cpar = warp - 10;
    const int kt0 = a.sink / 128;
    const int W = a.tbit_words;
    const int nw = (pi.n_ct + 31) / 32;
    // The keys of the tiles that are non-empty and not dense, among the
    // bitmap words of this collector's parity, taken a window of 32 such
    // tiles at a time (lane j holding the j-th), the next window's masks
    // loaded ahead.  The bitmap is read 32 words (1024 tiles) at a time.
    int sc = 0;
    bool s_done = nw == 0;
    uint32_t sword = 0u;                           // this lane's sparse word of chunk sc
    int sbase = 0;                                 // rank of its first sparse tile in the chunk
    int stot = 0, srank = 0;                       // sparse tiles in the chunk, handed out
    auto load_sparse_chunk = [&](int c) {
      const int wi = 32 * c + lane;
      sword = 0u;
      if (wi < nw && (wi & 1) == cpar)
        sword = (pi.ba[wi] | pi.bb[wi]) & ~(pi.ba[W + wi] | pi.bb[W + wi]);
      const int cw = __popc(sword);
      int incl = cw;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      sbase = incl - cw;
      stot = __shfl_sync(0xffffffffu, incl, 31);
      srank = 0;
    };
    bool p_valid = false;                          // prefetched window
    int p_n = 0, p_tile = 0;
    uint4 p_a = make_uint4(0u, 0u, 0u, 0u), p_b = p_a;
    auto scan_next = [&]() {
      p_valid = false;
      while (!s_done) {
        if (srank < stot) {
          // lane j: the sparse tile of rank srank + j, in the last word whose
          // first rank is at most that
          const int R = srank + lane;
          int w = 0;
#pragma unroll
          for (int step = 16; step > 0; step >>= 1) {
            const int c = w + step;
            const int bc = __shfl_sync(0xffffffffu, sbase, c & 31);
            if (c < 32 && bc <= R) w = c;
          }
          const uint32_t word = __shfl_sync(0xffffffffu, sword, w);
          const int wb = __shfl_sync(0xffffffffu, sbase, w);
          p_n = min(32, stot - srank);
          if (lane < p_n) {
            p_tile = 32 * (32 * sc + w) + static_cast<int>(__fns(word, 0, R - wb + 1));
            p_a = pi.ma[p_tile];
            p_b = pi.mb[p_tile];
          }
          srank += p_n;
          p_valid = true;
          return;
        }
        ++sc;
        if (32 * sc >= nw) {
          s_done = true;
          return;
        }
        load_sparse_chunk(sc);
      }
    };
    bool g_valid = false;                          // window in use
    int g_tile = 0, g_cnt = 0;
    uint4 g_a = p_a, g_b = p_a;
    int j0 = 0, cons = 0;                          // first lane not used up, its keys taken
    auto take_window = [&]() {
      g_valid = p_valid;
      if (!g_valid) return;
      g_tile = p_tile;
      g_a = p_a;
      g_b = p_b;
      g_cnt = lane < p_n ? __popc(g_a.x | g_b.x) + __popc(g_a.y | g_b.y) +
                               __popc(g_a.z | g_b.z) + __popc(g_a.w | g_b.w)
                         : 0;
      j0 = 0;
      cons = 0;
      scan_next();
    };
    if (nw > 0) {
      load_sparse_chunk(0);
      scan_next();
      take_window();
    }
    uint32_t* buf = cbuf + 128 * cpar;
    for (int n = 0;; ++n) {
      if (n > 0 && !warp_wait(bar_cempty0 + 8u * cpar, (n - 1) & 1, wc)) break;
      // the next 128 keys of this collector's sparse tiles
      int filled = 0;
      while (filled < 128 && g_valid) {
        const int skip = lane == j0 ? cons : 0;
        const int cnt = lane >= j0 ? g_cnt - skip : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const int excl = incl - cnt;
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        const int take = min(tot, 128 - filled);
        const bool mine = cnt > 0 && excl < take;
        const uint32_t act = __ballot_sync(0xffffffffu, mine);
        if (__reduce_max_sync(0xffffffffu, mine ? g_cnt : 0) > 6 * __popc(act)) {
          // few tiles with many keys each (a bit loop per lane would be
          // long): the warp places one tile's keys at a time, a 32-key word
          // per step, lane l taking column l
          for (uint32_t rest = act; rest; rest &= rest - 1u) {
            const int j = __ffs(rest) - 1;
            const int ex = __shfl_sync(0xffffffffu, excl, j);
            const int sk = __shfl_sync(0xffffffffu, skip, j);
            const int base_key = 128 * (kt0 + __shfl_sync(0xffffffffu, g_tile, j));
            int rbase = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              // word w of lane j's two masks (each lane passes its own word w)
              const uint32_t ua = __shfl_sync(0xffffffffu, w == 0 ? g_a.x : w == 1 ? g_a.y : w == 2 ? g_a.z : g_a.w, j);
              const uint32_t ub = __shfl_sync(0xffffffffu, w == 0 ? g_b.x : w == 1 ? g_b.y : w == 2 ? g_b.z : g_b.w, j);
              const uint32_t m = ua | ub;
              const int rk = rbase + __popc(m & ((1u << lane) - 1u));
              const int pos = ex + rk - sk;
              if (((m >> lane) & 1u) && rk >= sk && pos < take)
                buf[filled + pos] = static_cast<uint32_t>(base_key + 32 * w + lane) |
                                    (((ua >> lane) & 1u) << 30) | (((ub >> lane) & 1u) << 31);
              rbase += __popc(m);
            }
          }
        } else if (mine) {
          // this lane's tile: its keys of rank skip, skip + 1, ... go to
          // slots filled + excl, ... while they are below filled + take
          const uint32_t ua[4] = {g_a.x, g_a.y, g_a.z, g_a.w};
          const uint32_t ub[4] = {g_b.x, g_b.y, g_b.z, g_b.w};
          const int base_key = 128 * (kt0 + g_tile);
          int r = 0;
          for (int w = 0; w < 4; ++w) {
            uint32_t rem = ua[w] | ub[w];
            while (rem) {
              const int bpos = __ffs(rem) - 1;
              rem &= rem - 1u;
              if (r >= skip) {
                const int pos = excl + r - skip;
                if (pos < take)
                  buf[filled + pos] = static_cast<uint32_t>(base_key + 32 * w + bpos) |
                                        (((ua[w] >> bpos) & 1u) << 30) |
                                        (((ub[w] >> bpos) & 1u) << 31);
              }
              ++r;
            }
          }
        }
        filled += take;
        if (take == tot) {
          take_window();
        } else {
          // the window continues at the lane holding the first key not taken
          const uint32_t cut = __ballot_sync(0xffffffffu, cnt > 0 && excl <= take && take < excl + cnt);
          const int J = __ffs(cut) - 1;
          const int eJ = __shfl_sync(0xffffffffu, excl, J);
          cons = (J == j0 ? cons : 0) + (take - eJ);
          j0 = J;
        }
      }
      __syncwarp();
      if (filled > 0) {
        const uint32_t first = buf[0] & 0x3FFFFFFFu;
        for (int r = filled + lane; r < 128; r += 32) buf[r] = first;
        __syncwarp();
        // column masks: row 32 w + l of the tile is bit l of word w
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t e = buf[32 * w + lane];
          const uint32_t ma = __ballot_sync(0xffffffffu, (e >> 30) & 1u);
          const uint32_t mb = __ballot_sync(0xffffffffu, (e >> 31) & 1u);
          if (lane == w) cmask[8 * cpar + w] = ma;
          if (lane == 4 + w) cmask[8 * cpar + 4 + w] = mb;
        }
      }
      if (lane == 0) ccount[cpar] = static_cast<uint32_t>(filled);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_cfull0 + 8u * cpar);
      if (filled == 0) break;
    }
  }
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    const int hd = warp >> 2;                  // 0: head A (warps 0-3), 1: head B (4-7)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = 128u * hd, o_col = 256u + 128u * hd;
    const float sl2 = a.sl2;
    float m_used = -INFINITY;
    float lsum = 0.f;
    bool ok = true;
    bool last = false;
    // When both heads keep every key of every candidate tile (the near-dense
    // case), the tiles are sink, n_ct full tiles and local, in the producer's
    // order, and their descriptors are known here without waiting for them.
    bool known = a.mode == kModeDense;
    if (!known && pi.n_ct > 0) {
      const int nwf = (pi.n_ct + 31) / 32;
      int missing = 0;
      for (int w0 = 0; w0 < nwf; w0 += 32) {
        const int wi = w0 + lane;
        if (wi < nwf) {
          const uint32_t f = pi.ba[2 * a.tbit_words + wi] & pi.bb[2 * a.tbit_words + wi];
          const int n = min(32, pi.n_ct - 32 * wi);
          const uint32_t need = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
          missing += (f & need) != need ? 1 : 0;
        }
      }
      known = __reduce_add_sync(0xffffffffu, missing) == 0;
    }
    const int n_full = a.mode == kModeDense ? 0 : pi.n_ct;
    for (int t = 0; !last; ++t) {
      if (!(ok = warp_wait(bar_sfull0 + 8u * hd, t & 1, wc))) break;
      tc_fence_after();
      const int vs = t % kPairVStages;
      uint32_t dw;
      if (known) {
        if (t < it.n_sink_t) {
          dw = static_cast<uint32_t>(min(128, it.sink_end - 128 * t));
        } else if (t < it.n_sink_t + n_full) {
          dw = 128u;
        } else {
          const int li = t - it.n_sink_t - n_full;
          const int k0 = it.loc_start + 128 * li;
          dw = static_cast<uint32_t>(min(128, it.le - k0)) | (k0 == it.row0 ? kDescCausal : 0u) |
               (li + 1 == it.n_loc_t ? kDescLast : 0u);
        }
      } else {
        // every tile arrives once on its V slot's tag barrier, before its loads
        if (!(ok = warp_wait(bar_tag0 + 8u * vs, (t / kPairVStages) & 1, wc))) break;
        dw = tdesc[vs];
      }
      last = (dw & kDescLast) != 0u;
      const int valid = static_cast<int>(dw & 0x1FFu);
      const int limit = (dw & kDescCausal) ? min(valid, r + 1) : valid;
      uint32_t tw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (dw & kDescMasked) {
#pragma unroll
        for (int w = 0; w < 4; ++w) tw[w] = tags[(vs * 2 + hd) * 4 + w];
      }
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + s_col + 32u * c, sr[c]);
      tmem_ld_wait();
      // the column bound folded into the membership words, so that a column
      // costs one bit test and one select
      const bool masked = (limit < 128) || ((tw[0] & tw[1] & tw[2] & tw[3]) != 0xffffffffu);
      if (masked) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n = limit - 32 * c;
          const uint32_t keep = tw[c] & (n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u)));
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            // all ones when column e is kept: bit e moved to the sign, then spread
            const uint32_t k = static_cast<uint32_t>(static_cast<int32_t>(keep << (31 - e)) >> 31);
            sr[c][e] = (sr[c][e] & k) | (0xff800000u & ~k);
          }
        }
      }
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(sr[c][e]));
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      const float mx2 = mx * sl2;
      const bool grow = mx2 > m_used + 8.0f;
      if (t == 0) {
        m_used = mx2;
      } else if (__any_sync(0xffffffffu, grow)) {
        // every PV of this head up to tile t-1 completed before S_t was ready
        const float f = grow ? fast_exp2(m_used - mx2) : 1.0f;
        if (grow) {
          lsum *= f;
          m_used = mx2;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + o_col + 32u * c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(tmem + lane_off + o_col + 32u * c, ov);
        }
        tmem_st_wait();
      }
      // p = 2^(s * scale * log2 e - m) -> P (bf16) into S's first 64 columns
      // (S is entirely in registers by now)
      const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
      float ps[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * h2 + cc;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sr[c][e]), sl2, neg_m));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sr[c][e + 1]), sl2, neg_m));
            ps[(e >> 1) & 7] += p0 + p1;
            sr[c][e >> 1] = pack_bf16x2(p0, p1);   // in place: index e/2 was consumed
          }
        }
        tmem_st32_halves(tmem + lane_off + s_col + 32u * h2, sr[2 * h2], sr[2 * h2 + 1]);
      }
      lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull0 + 8u * hd);
    }
    if (ok) {
      ok = warp_wait(bar_odone, 0, wc);
      if (ok) {
        tc_fence_after();
        const int h = it.h + hd;
        const int row = it.row0 + r;
        const float inv = 1.0f / lsum;
        __nv_bfloat16* orow = a.o + (((long long)(it.b * a.Hq + h) * a.L) + row) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + o_col + 32u * c, ov);
          tmem_ld_wait();
          if (row < a.L) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
              dst[v4] = w;
            }
          }
        }
        if (row < a.L && a.lse != nullptr) {
          a.lse[(long long)(it.b * a.Hq + h) * a.L + row] =
              m_used * 0.69314718055994531f + logf(lsum);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

}  // namespace spa
