// HCA prefill attention: a cluster of two CTA pairs per 256-row tile.
//
// What is computed ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1; xenospectrum
// analysis, section 活性140億パラメータと長文処理を支える仕組み): for each query
// position t and head h, one softmax over the compressed entries j < nc(t) and
// the raw keys max(0, t-127) .. t, then out = sigmoid(g) * (P . V).
//
// Layout of the work.  An item is 4 consecutive positions x 64 heads = 256
// rows; all of them share the one KV head, so every key tile serves all 256
// rows.  The cluster has four CTAs in two tcgen05 CTA pairs:
//   ranks 0, 1 (S pair): S = Q K^T as M = 256 MMAs issued by rank 0.  Each CTA
//     keeps its own 128 Q rows (positions t0 + 2c, t0 + 2c + 1) in shared
//     memory and loads half of every key tile (the pair splits B by columns),
//     so an SM streams half the key bytes per FLOP of a one-CTA MMA.  Each CTA
//     runs the online softmax of its 128 rows out of its own TMEM and writes
//     P (bf16) to a small L2-resident scratch, 128 keys at a time.
//   ranks 2, 3 (O pair): O += P V as M = 256 MMAs issued by rank 2.  CTA 2 + c
//     holds the P rows of its partner S-CTA c (loaded from the scratch) and
//     128 of the 256 value columns of each MMA, and accumulates O for its 128
//     rows x 512 value columns in its TMEM; it rescales those rows when a row
//     maximum grows and runs their gated epilogue out = sigmoid(g) O / l.
// Why pairs.  A 128 x 512 fp32 O fills all 512 TMEM columns of an SM, so no
// SM can hold O and the scores: computing S and O on different CTAs keeps Q K^T
// computed once.  Pairing the CTAs of each role halves what every SM loads per
// MMA and what its single issuing thread spends per FLOP, the two limits of a
// one-CTA M = 128 design at this head width.
//
// Barriers.  A pair's operands are counted on the even CTA's barriers: every
// CTA's loads of pair operands (Q, K, P, V) signal the even CTA's "full"
// barrier (.cta_group::2 copies), whose producer posts the bytes of both CTAs;
// the MMA completions arrive on the "empty" barriers of both CTAs
// (multicast commit).  Everything one CTA alone consumes (scores, O, gate
// stages, statistics) has local barriers.
//
// Tiles.  Key tiles: ceil(nc(t0+3) / 256) compressed tiles of up to 256
// entries and one raw tile of 144 keys [t0-127, t0+16] (the window of all four
// positions, padded to a multiple of 16); P and V move in 128-key sub-tiles.
//
// Virtual head attention (kVha; same pages, §2.1, VHA): after the gate, the
// 64 heads of each position are mixed, y = x + M' x with M' = up down^T
// (64 x 64, rank r).  It runs in the O pair's epilogue as one more pair MMA
// per 128-column gate stage, transposed so that the operands already sit
// where the epilogue leaves them: A = x^T (the gated bf16 stage in shared
// memory read MN-major: M = 128 value columns per CTA, K = the 64 heads of one
// position), B = I then M'^T (two K passes into one accumulator, so the
// identity term is exact; each CTA holds 32 of the 64 columns of each, 8 KB),
// D = the 128 TMEM columns of O that the stage has just read out (lane =
// value column, column = head): D is y itself, which the epilogue rounds and
// writes over x.  The V ring drops to 4 stages to make room for B.  The mix
// of value half 1 is issued after the next item's first P.V stages of value
// half 0, so that waiting for it never holds those back.
//
// Warp roles (544 threads): warps 0-1 TMA producers, warp 2 TMEM owner and (in
// even CTAs) MMA issuer, warps 3-10 compute: two warps per TMEM lane quadrant.
// On S-CTAs each owns one 128-key half of the score rows; on O-CTAs they
// rescale O and run the epilogue of value columns 0-255.  O-CTAs also run
// warp 11 (P copier), warp 12 (output stores) and warps 13-16 (epilogue of
// value columns 256-511).
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace prefill3 {

constexpr int kRows = 128;      // rows per CTA
constexpr int kPos = 4;         // positions per item (two per CTA of a pair)
constexpr int kHeads = 64;
constexpr int kKT = 256;        // compressed key tile
constexpr int kWinN = 144;      // raw key tile
constexpr int kWinHalf = kWinN / 2;
constexpr int kThreads = 544;
constexpr int kSlot = 32768;                       // one P sub-tile image
constexpr int kScratchPerCluster = 2 * 4 * kSlot;  // 2 S-CTAs x 2 parities x 2 sub-tiles
constexpr float kTau = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---- S-CTA shared memory
constexpr int S_Q = 0;             // 8 slabs x [128 rows][64]
constexpr int kQHalf = 65536;
constexpr int S_KRING = 131072;    // 3 stages x 2 slabs x [128 keys][64]
constexpr int kKStages = 3;
constexpr int kKStage = 32768;
constexpr int kKSlab = 16384;
// ---- O-CTA shared memory
constexpr int O_P = 0;             // 2 sub-tile buffers x [16 key chunks][128 rows][8 keys]
constexpr int kPBuf = 32768;
constexpr int O_VRING = 65536;     // 5 stages (4 with VHA) x 2 slabs x [128 keys][64 dv]
constexpr int kVStages = 5;
constexpr int kVStagesVha = 4;
constexpr int kVStage = 32768;
constexpr int O_VHAB = O_VRING + kVStagesVha * kVStage;   // VHA B: 2 x [32 heads][64 heads] bf16

// ---- barriers (every CTA, same offsets)
constexpr int BAR = 229376;
enum {
  QFULL = 0, QEMPTY = 2, KFULL = 4, KEMPTY = KFULL + kKStages, SFULL = KEMPTY + kKStages,
  SFREE = SFULL + 2, PFREE = SFREE + 2, STATSFREE = PFREE + 4,
  VFULL = STATSFREE + 1, GFULL = VFULL + kVStages, VEMPTY = GFULL + kVStages,
  PREADY = VEMPTY + kVStages, PFULL = PREADY + 4, PBUFFREE = PFULL + 2, CORR = PBUFFREE + 2,
  PVDONE = CORR + 2, OFULL = PVDONE + 2, OFREE = OFULL + 2, STATSFULL = OFREE + 2,
  STAGED = STATSFULL + 1, XSTAGED = STAGED + 4, VHADONE = XSTAGED + 4, DRAIN = VHADONE + 4,
  NBAR = DRAIN + 1
};
constexpr int kBarBytes = 640;
constexpr int kTmemSlot = BAR + 8 * NBAR;
constexpr int kAbortSlot = kTmemSlot + 4;
// S-CTA: per-row maxima exchanged by the two warps of a row ([2][2][128]
// float) and their ok flags ([2][2][4] int)
constexpr int S_XMAX = BAR + kBarBytes;
constexpr int S_XOK = S_XMAX + 2048;
// O-CTA: rescale factors [2 tile parities][128], flags [2][4], 1/l [128]
constexpr int O_ALPHA = BAR + kBarBytes;
constexpr int O_FLAGS = O_ALPHA + 1024;
constexpr int O_INVL = O_FLAGS + 64;
constexpr int kSmemBytes = S_XOK + 64;
constexpr int kSmemAlloc = kSmemBytes;
static_assert(kAbortSlot + 4 <= BAR + kBarBytes, "barrier region overflow");
static_assert(O_VRING + kVStages * kVStage <= BAR, "O-CTA ring overflow");
static_assert(O_VHAB + 8192 <= BAR, "O-CTA VHA operand overflow");
static_assert(O_INVL + 512 <= kSmemBytes, "O-CTA layout overflow");
static_assert(S_KRING + kKStages * kKStage <= BAR, "S-CTA layout overflow");
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr uint16_t kMaskS = 0x3;   // CTAs 0, 1
constexpr uint16_t kMaskO = 0xC;   // CTAs 2, 3

struct Params {
  int B, T;
  int row_tiles;     // ceil(T / 4)
  int items;         // B * row_tiles
  float scale_log2;  // softmax scale * log2(e)
  float* lse;        // [B, T, 64] or null
  uint8_t* pscratch; // [clusters][2][4][32 KB] P sub-tile images
  const uint16_t* vha_down;   // VHA factors [64][vha_rank] bf16 (kVha only)
  const uint16_t* vha_up;
  int vha_rank;
};

struct Maps {
  CUtensorMap q4;    // (64, T*64, 8, B)  box (64, 128, 4, 1): one Q half of one CTA
  CUtensorMap ck;    // [B][nb][512]      box (64, 64, 1)
  CUtensorMap kwin;  // [B][T][512]       box (64, 72, 1): half of the raw key tile
  CUtensorMap cv4;   // (64, nb, 8, B)    box (64, 128, 2, 1)
  CUtensorMap v4;    // (64, T, 8, B)     box (64, 128, 2, 1)
  CUtensorMap v4t;   // (64, T, 8, B)     box (64, 16, 1, 1): one slab of keys t0+1 .. t0+16
  CUtensorMap g4;    // (64, T*64, 8, B)  box (64, 128, 2, 1)
  CUtensorMap out4;  // same as g4
  CUtensorMap p128;  // P scratch as [rows of 256 B], box (256, 128): one 32 KB slot
  CUtensorMap p16;   // same, box (256, 16): the first 16 keys of a slot
};

__device__ __forceinline__ int nc_of(int t) { return t >= 127 ? (t - 127) / 128 : 0; }

struct Item {
  int b, t0, np;      // batch, first position, valid positions (1..4)
  int ncmax, n_ctiles, ntiles;
};

__device__ __forceinline__ Item decode_item(const Params& p, int it) {
  Item x;
  const int rank = it / p.B;
  x.b = it - rank * p.B;
  x.t0 = kPos * (p.row_tiles - 1 - rank);
  x.np = min(kPos, p.T - x.t0);
  x.ncmax = nc_of(x.t0 + x.np - 1);
  x.n_ctiles = (x.ncmax + kKT - 1) / kKT;
  x.ntiles = x.n_ctiles + 1;
  return x;
}

// MMA width of key tile j (multiple of 16)
__device__ __forceinline__ int tile_n(const Item& x, int j) {
  if (j < x.n_ctiles) return (min(kKT, x.ncmax - j * kKT) + 15) & ~15;
  return kWinN;
}
// keys of sub-tile h (0: columns 0..127, 1: columns 128..) of a tile of width n
__device__ __forceinline__ int sub_n(int n, int h) { return h == 0 ? min(n, 128) : max(0, n - 128); }

// P.V stage order of one tile (value half dh, sub-tile h), walked by the V
// producers and the MMA issuer.  An item's first and last tiles run value
// half major (the previous item's epilogue hands O back one half at a time,
// and this item's epilogue starts on half 0 while half 1 accumulates); the
// tiles between run sub-tile major (P buffer h is free once both halves used
// it).  A tile has 2 stages per non-empty sub-tile.
__device__ __forceinline__ void pv_stage(int s, bool two, bool half_major, int& dh, int& h) {
  if (!two) {
    dh = s;
    h = 0;
  } else if (half_major) {
    dh = s >> 1;
    h = s & 1;
  } else {
    h = s >> 1;
    dh = s & 1;
  }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int x, int y, int z, int w) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

template <bool kVha>
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kThreads, 1)
    prefill3_kernel(const __grid_constant__ Maps maps, const Params p) {
  constexpr int NV = kVha ? kVStagesVha : kVStages;   // V ring stages
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  if ((sb & 1023u) != 0) {  // uniform: every thread sees the same base
    if (threadIdx.x == 0) record_error(DEVERR_LAYOUT, 300);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sb + BAR + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortSlot);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool isO = rank >= 2;
  const int half = static_cast<int>(rank & 1);   // which 128 rows / which half of B
  const bool leader = half == 0;
  const uint32_t lead = rank & ~1u;              // the even CTA of this pair
  const int cluster = blockIdx.x >> 2;
  const int nclusters = gridDim.x >> 2;
  // a barrier of the even CTA of this pair, as a shared::cluster address
  auto lbar = [&](int i) -> uint32_t { return mapa_shared(bar(i), lead); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(SFREE + 0), 16);            // softmax warps of both S-CTAs
    mbar_init(bar(SFREE + 1), 16);
    mbar_init(bar(STATSFREE), 12);            // the partner O-CTA's epilogue warps
    for (int q = 0; q < 4; ++q) mbar_init(bar(PREADY + q), 4);
    mbar_init(bar(CORR + 0), 16);             // correction warps of both O-CTAs
    mbar_init(bar(CORR + 1), 16);
    mbar_init(bar(OFREE + 0), 16);            // epilogue warps of value half 0, both O-CTAs
    mbar_init(bar(OFREE + 1), 8);             // helper warps (value half 1), both O-CTAs
    mbar_init(bar(STATSFULL), 4);
    for (int e = 0; e < 4; ++e) mbar_init(bar(STAGED + e), 4);   // one arrive per epilogue warp
    for (int e = 0; e < 4; ++e) mbar_init(bar(XSTAGED + e), 8);  // epilogue warps, both O-CTAs
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (kVha && isO) {
    // this CTA's halves of B: rows n = 32 half + i of the identity and of
    // M' = up down^T, K-major (k = input head contiguous), 128B-swizzled; M'
    // as fp32 sums rounded to bf16
    for (int idx = threadIdx.x; idx < 32 * 64; idx += kThreads) {
      const int i = idx >> 6, k = idx & 63;
      const int n = 32 * half + i;
      float acc = 0.f;
      for (int r = 0; r < p.vha_rank; ++r)
        acc = fmaf(__uint_as_float(static_cast<uint32_t>(p.vha_up[n * p.vha_rank + r]) << 16),
                   __uint_as_float(static_cast<uint32_t>(p.vha_down[k * p.vha_rank + r]) << 16),
                   acc);
      const uint32_t off = sw128_offset(i, k >> 3) + 2 * (k & 7);
      *reinterpret_cast<uint16_t*>(smem + O_VHAB + off) = k == n ? 0x3F80u : 0u;   // 1.0, 0
      *reinterpret_cast<uint16_t*>(smem + O_VHAB + 4096 + off) =
          static_cast<uint16_t>(pack_bf16x2(acc, 0.f) & 0xFFFFu);
    }
    fence_proxy_async_smem();   // read by the VHA MMAs (async proxy)
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  cluster_sync_all();  // every CTA's barriers exist before any remote access
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (!isO) {
    // =====================================================================
    // S-CTA (rank 0 or 1)
    // =====================================================================
    if (warp <= 1) {
      // --------------------------------------------------------- producers
      if (lane == 0) {
        const int me = warp;
        uint32_t u = 0, nitem = 0;
        bool ok = true;
        for (int it = cluster; it < p.items && ok; it += nclusters, ++nitem) {
          const Item x = decode_item(p, it);
          if (me == 0 && it + nclusters < p.items) {  // warm L2 with the next item's Q rows
            const Item y = decode_item(p, it + nclusters);
            tma_prefetch_4d(&maps.q4, 0, (y.t0 + 2 * half) * kHeads, 0, y.b);
            tma_prefetch_4d(&maps.q4, 0, (y.t0 + 2 * half) * kHeads, 4, y.b);
          }
          // Q half `me` (4 slabs) of this CTA's 128 rows
          ok = mbar_wait(bar(QEMPTY + me), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs, 310);
          if (!ok) break;
          if (leader) mbar_expect_tx(bar(QFULL + me), 2 * kQHalf);
          tma_load_4d_pair(sb + S_Q + me * kQHalf, &maps.q4, lbar(QFULL + me), 0,
                           (x.t0 + 2 * half) * kHeads, 4 * me, x.b);
          for (int j = 0; j < x.ntiles && ok; ++j) {
            const bool comp = j < x.n_ctiles;
            const int n = tile_n(x, j);
            const int nhalf = n >> 1;                 // keys of this CTA
            const int n64 = (nhalf + 63) >> 6;        // 64-row boxes of a compressed half
#pragma unroll 1
            for (int d2 = 0; d2 < 4; ++d2, ++u) {     // stage = 2 slabs of 64 channels
              if ((u & 1) != static_cast<uint32_t>(me)) continue;
              const uint32_t st = u % kKStages;
              ok = mbar_wait(bar(KEMPTY + st), ((u / kKStages) & 1) ^ 1, abort_flag, kWaitLimitNs,
                             311);
              if (!ok) break;
              const uint32_t dst = sb + S_KRING + st * kKStage;
              const uint32_t fb = lbar(KFULL + st);
              if (comp) {
                if (leader) mbar_expect_tx(bar(KFULL + st), 2 * 2 * n64 * 8192);
#pragma unroll 1
                for (int s = 0; s < 2; ++s)
#pragma unroll 1
                  for (int r = 0; r < n64; ++r)
                    tma_load_3d_pair(dst + s * kKSlab + r * 8192, &maps.ck, fb, 64 * (2 * d2 + s),
                                     j * kKT + half * nhalf + 64 * r, x.b);
              } else {
                if (leader) mbar_expect_tx(bar(KFULL + st), 2 * 2 * kWinHalf * 128);
#pragma unroll 1
                for (int s = 0; s < 2; ++s)
                  tma_load_3d_pair(dst + s * kKSlab, &maps.kwin, fb, 64 * (2 * d2 + s),
                                   x.t0 - 127 + half * kWinHalf, x.b);
              }
            }
          }
        }
      }
    } else if (warp == 2) {
      // --------------------------------------------------------- MMA (S = Q K^T), even CTA
      if (leader && lane == 0) {
        uint32_t u = 0, sj = 0, nitem = 0;
        bool ok = true;
        for (int it = cluster; it < p.items && ok; it += nclusters, ++nitem) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            const uint32_t buf = sj & 1;
            ok &= mbar_wait_cluster(bar(SFREE + buf), ((sj >> 1) & 1) ^ 1, abort_flag,
                                    kWaitLimitNs, 320);
            const uint32_t idesc = idesc_bf16_f32(2 * kRows, tile_n(x, j), false, false);
            const uint32_t dS = tmem + 256 * buf;
            const bool first = j == 0, last = j + 1 == x.ntiles;
#pragma unroll 1
            for (int d2 = 0; d2 < 4; ++d2, ++u) {
              if (first && (d2 & 1) == 0)
                ok &= mbar_wait(bar(QFULL + (d2 >> 1)), nitem & 1, abort_flag, kWaitLimitNs, 321);
              const uint32_t st = u % kKStages;
              ok &= mbar_wait(bar(KFULL + st), (u / kKStages) & 1, abort_flag, kWaitLimitNs, 322);
              tc_fence_after();
              const uint32_t ka = sb + S_KRING + st * kKStage;
#pragma unroll
              for (int s = 0; s < 2; ++s) {
                const int d = 2 * d2 + s;
                const uint32_t qa = sb + S_Q + (d >> 2) * kQHalf + (d & 3) * 16384;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  umma_pair_if(dS, sdesc_sw128(qa + 32 * k, 16, 1024),
                               sdesc_sw128(ka + s * kKSlab + 32 * k, 16, 1024), idesc,
                               (d | k) != 0, true);
              }
              umma_pair_commit_mc(bar(KEMPTY + st), kMaskS);
              umma_pair_commit_mc_if(bar(QEMPTY + (d2 >> 1)), kMaskS, last && (d2 & 1) == 1);
            }
            umma_pair_commit_mc(bar(SFULL + buf), kMaskS);
          }
        }
        umma_pair_commit_mc(bar(DRAIN), 1u << rank);
        mbar_wait(bar(DRAIN), 0, abort_flag, kWaitLimitNs, 323);
      }
    } else if (warp >= 11) {
      // the P copier, store and helper roles exist on O-CTAs only
    } else {
      // --------------------------------------------------------- softmax
      const int wq = warp & 3;
      const int kh = (warp - 3) >> 2;         // key columns [128 kh, 128 kh + 128)
      const int row = wq * 32 + lane;
      const int pos = 2 * half + (row >> 6);  // position t0 + pos of this row
      const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      float* xmax = reinterpret_cast<float*>(smem + S_XMAX);
      volatile int* xok = reinterpret_cast<volatile int*>(smem + S_XOK);
      uint8_t* const pscr =
          p.pscratch + (static_cast<size_t>(cluster) * 2 + half) * (kScratchPerCluster / 2);
      const uint32_t partner = 2 + half;
      const uint32_t peerAlpha = mapa_shared(sb + O_ALPHA, partner);
      const uint32_t peerFlags = mapa_shared(sb + O_FLAGS, partner);
      const uint32_t peerInvl = mapa_shared(sb + O_INVL, partner);
      const uint32_t peerPReady = mapa_shared(bar(PREADY), partner);
      const uint32_t peerStatsFull = mapa_shared(bar(STATSFULL), partner);
      uint32_t sj = 0, nitem = 0, nx = 0;
      bool ok = true, both = true;
      // A row is shared by two warps (one per key half): both write, a
      // 64-thread named barrier, both read.  The ok flags travel with the
      // value, so the two warps leave their loops at the same exchange.
      auto exchange = [&](float v) -> float {
        const uint32_t xp = nx & 1;
        xmax[(xp * 2 + kh) * 128 + row] = v;
        if (lane == 0) xok[(xp * 2 + kh) * 4 + wq] = ok ? 1 : 0;
        named_bar_sync(1 + wq, 64);
        const float o = xmax[(xp * 2 + (kh ^ 1)) * 128 + row];
        both = ok && xok[(xp * 2 + (kh ^ 1)) * 4 + wq] != 0;
        ++nx;
        return o;
      };
      // P stores of a tile are published one step later (after the next
      // tile's row max), so the wait for them to drain overlaps that work.
      uint32_t pend = 0;   // scratch slot + 1 of the unpublished sub-tile
      auto publish = [&]() {
        fence_proxy_async_global();  // the scratch is read next by a TMA copy (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(peerPReady + 8 * (pend - 1));
        pend = 0;
      };
      for (int it = cluster; it < p.items; it += nclusters, ++nitem) {
        const Item x = decode_item(p, it);
        const int t = x.t0 + pos;
        const int ncp = nc_of(min(t, p.T - 1));
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < x.ntiles; ++j, ++sj) {
          const uint32_t buf = sj & 1;
          if (ok) ok = mbar_wait_warp(bar(SFULL + buf), (sj >> 1) & 1, abort_flag, kWaitLimitNs, 330);
          tc_fence_after();
          const int n = tile_n(x, j);
          const int nh = sub_n(n, kh);
          // visible columns of this tile for this row: [clo, chi)
          int clo = 0, chi;
          if (j < x.n_ctiles) {
            chi = min(n, max(0, ncp - j * kKT));
          } else {
            clo = max(127 - x.t0, pos);
            chi = 128 + pos;
          }
          const int c0 = 128 * kh;
          const uint32_t sbase = tl + 256 * buf + c0;
          // pass A: this half's row max of the raw scores
          float mraw = -INFINITY;
#pragma unroll 1
          for (int cc = 0; ok && cc < nh; cc += 32) {
            uint32_t r[32];
            tmem_ld32(sbase + cc, r);
            tmem_wait_ld_dep32(r);
            const int lo = clo - c0 - cc, hi = chi - c0 - cc;
            if (lo <= 0 && hi >= 32) {   // warp-uniform: the whole chunk visible
              float mx[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) mx[i] = __uint_as_float(r[i]);
#pragma unroll
              for (int c = 4; c < 32; ++c) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(r[c]));
              mraw = fmaxf(mraw, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                mraw = fmaxf(mraw, (c >= lo && c < hi) ? __uint_as_float(r[c]) : -INFINITY);
            }
          }
          mraw = fmaxf(mraw, exchange(mraw));
          if (!both) break;
          if (pend) publish();
          const float mt = mraw * p.scale_log2;  // scale > 0
          float alpha = 1.f;
          bool resc = false;
          if (mt > m + kTau) {
            resc = (m != -INFINITY);
            alpha = resc ? ex2_approx(m - mt) : 0.f;
            m = mt;
          }
          const float mu = (m == -INFINITY) ? 0.f : m;
          // scratch slot (tile parity, key half): free once the O pair has
          // finished P.V of the tile two back
          const uint32_t slot = (sj & 1) * 2 + kh;
          if (ok)
            ok = mbar_wait_cluster_warp(bar(PFREE + slot), ((sj >> 1) & 1) ^ 1, abort_flag,
                                        kWaitLimitNs, 331);
          uint8_t* const gdst = pscr + slot * kSlot;
          // pass B: probabilities into the scratch slot
          float rs = 0.f;
#pragma unroll 1
          for (int cc = 0; ok && cc < nh; cc += 32) {
            uint32_t r[32];
            tmem_ld32(sbase + cc, r);
            tmem_wait_ld_dep32(r);
            uint32_t pk[16];
            const int lo = clo - c0 - cc, hi = chi - c0 - cc;
            if (lo <= 0 && hi >= 32) {   // warp-uniform: the whole chunk visible
              float2 acc = make_float2(0.f, 0.f);
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                const float2 xx = fma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])),
                                       p.scale_log2, -mu);
                const float2 ee = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
                acc = add2(acc, ee);
                pk[c / 2] = pack_bf16x2(ee.x, ee.y);
              }
              rs += acc.x + acc.y;
            } else {
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                // masked scores enter ex2 as -inf and come out as 0
                const float x0 = (c >= lo && c < hi) ? fmaf(__uint_as_float(r[c]), p.scale_log2, -mu)
                                                     : -INFINITY;
                const float x1 = (c + 1 >= lo && c + 1 < hi)
                                     ? fmaf(__uint_as_float(r[c + 1]), p.scale_log2, -mu)
                                     : -INFINITY;
                const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
                rs += e0 + e1;
                pk[c / 2] = pack_bf16x2(e0, e1);
              }
            }
            // chunk-major image: 8-key chunk k8 of row `row` at k8 * 2048 + 16 * row
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              const int k8 = (cc >> 3) + c8;
              *reinterpret_cast<uint4*>(gdst + k8 * 2048 + 16 * row) =
                  make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
            }
          }
          if (ok && kh == 0) {
            st_cluster_b32(peerAlpha + 512 * (sj & 1) + 4 * row, __float_as_uint(alpha));
            const int any = __any_sync(0xffffffffu, resc) ? 1 : 0;
            if (lane == 0)
              st_cluster_b32(peerFlags + 16 * (sj & 1) + 4 * wq, static_cast<uint32_t>(any));
          }
          tc_fence_before();
          __syncwarp();
          // S buffer read out.  The arrive publishes no data (the TMEM loads
          // have completed at tcgen05.wait::ld), so it is relaxed: a release
          // arrive would also wait for this warp's P stores to drain.
          if (lane == 0) mbar_arrive_cluster_relaxed(lbar(SFREE + buf));
          pend = slot + 1;
          l = l * alpha + rs;
        }
        if (!both) break;
        // row sum = both halves (one more exchange); 1/l to the partner's
        // epilogue, lse to the caller
        l += exchange(l);
        if (!both) break;
        if (pend) publish();
        if (kh == 0) {
          if (!mbar_wait_cluster_warp(bar(STATSFREE), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs,
                                      332)) {
            ok = false;
            continue;  // the next exchange takes both warps out
          }
          st_cluster_b32(peerInvl + 4 * row, __float_as_uint(1.f / l));
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(peerStatsFull);
          if (p.lse != nullptr && t < p.T)
            p.lse[(static_cast<size_t>(x.b) * p.T + t) * kHeads + (row & 63)] =
                (m + __log2f(l)) * 0.6931471805599453f;
        }
      }
    }
  } else {
    // =====================================================================
    // O-CTA (rank 2 or 3)
    // =====================================================================
    // ring uses of one item: every P.V stage of every tile, then 4 gate stages
    auto v_uses = [&](const Item& x) -> uint32_t {
      uint32_t n_uses = 0;
      for (int j = 0; j < x.ntiles; ++j) n_uses += sub_n(tile_n(x, j), 1) > 0 ? 4 : 2;
      return n_uses;
    };
    const int orow0 = 2 * half;   // first position of this CTA's rows
    if (warp <= 1) {
      // --------------------------------------------------------- producers
      if (lane == 0) {
        const int me = warp;
        uint32_t u = 0;
        bool ok = true;
        for (int it = cluster; it < p.items && ok; it += nclusters) {
          const Item x = decode_item(p, it);
          if (me == 0) {  // warm L2 with this item's gate rows; they are staged after its V
#pragma unroll 1
            for (int e = 0; e < 4; ++e)
              tma_prefetch_4d(&maps.g4, 0, (x.t0 + orow0) * kHeads, 2 * e, x.b);
          }
          for (int j = 0; j < x.ntiles && ok; ++j) {
            const int n = tile_n(x, j);
            const bool comp = j < x.n_ctiles;
            const bool two = sub_n(n, 1) > 0;
            const int nst = two ? 4 : 2;
            for (int s = 0; s < nst && ok; ++s, ++u) {
              if ((u & 1) != static_cast<uint32_t>(me)) continue;
              int dh, h;
              pv_stage(s, two, j == 0 || j == x.ntiles - 1, dh, h);
              const uint32_t st = u % NV;
              ok = mbar_wait(bar(VEMPTY + st), ((u / NV) & 1) ^ 1, abort_flag, kWaitLimitNs,
                             340);
              if (!ok) break;
              // two 64-column slabs of 128 keys; raw sub-tile 1 is 16 keys: two
              // 16-row boxes placed where the slabs of a full stage start
              const bool tail = !comp && h == 1;
              const uint32_t bytes = tail ? 2 * 16 * 128 : 2 * 128 * 128;
              if (leader) mbar_expect_tx(bar(VFULL + st), 2 * bytes);
              const int key = 128 * h;
              const uint32_t dst = sb + O_VRING + st * kVStage;
              const int z = 4 * dh + 2 * half;
              if (tail) {
                tma_load_4d_pair(dst, &maps.v4t, lbar(VFULL + st), 0, x.t0 - 127 + key, z, x.b);
                tma_load_4d_pair(dst + 16384, &maps.v4t, lbar(VFULL + st), 0, x.t0 - 127 + key,
                                 z + 1, x.b);
              } else {
                tma_load_4d_pair(dst, comp ? &maps.cv4 : &maps.v4, lbar(VFULL + st), 0,
                                 comp ? j * kKT + key : x.t0 - 127 + key, z, x.b);
              }
            }
          }
#pragma unroll 1
          for (int e = 0; e < 4 && ok; ++e, ++u) {   // gate stages of this CTA's rows
            if ((u & 1) != static_cast<uint32_t>(me)) continue;
            const uint32_t st = u % NV;
            ok = mbar_wait(bar(VEMPTY + st), ((u / NV) & 1) ^ 1, abort_flag, kWaitLimitNs,
                           341);
            if (!ok) break;
            mbar_expect_tx(bar(GFULL + st), kVStage);
            tma_load_4d(sb + O_VRING + st * kVStage, &maps.g4, bar(GFULL + st), 0,
                        (x.t0 + orow0) * kHeads, 2 * e, x.b);
          }
        }
      }
    } else if (warp == 11) {
      // --------------------------------------------------------- P copier
      if (lane == 0) {
        const int prow0 = ((cluster * 2 + half) * 4) * (kSlot / 256);  // first 256-B row of my slots
        uint32_t sj = 0;
        bool ok = true;
        for (int it = cluster; it < p.items && ok; it += nclusters) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            const int n = tile_n(x, j);
#pragma unroll 1
            for (int h = 0; h < 2 && ok; ++h) {
              const int nh = sub_n(n, h);
              ok = mbar_wait_cluster(bar(PREADY + (sj & 1) * 2 + h), (sj >> 1) & 1, abort_flag,
                                     kWaitLimitNs, 345) &&
                   mbar_wait(bar(PBUFFREE + h), (sj & 1) ^ 1, abort_flag, kWaitLimitNs, 346);
              if (!ok) break;
              if (nh > 0) {
                fence_proxy_async_global();
                const bool small = nh <= 16;
                if (leader) mbar_expect_tx(bar(PFULL + h), small ? 2 * 4096 : 2 * kSlot);
                tma_load_2d_pair(sb + O_P + h * kPBuf, small ? &maps.p16 : &maps.p128,
                                 lbar(PFULL + h), 0,
                                 prow0 + ((sj & 1) * 2 + h) * (kSlot / 256));
              } else if (leader) {
                mbar_arrive(bar(PFULL + h));
              }
            }
          }
        }
      }
    } else if (warp == 12) {
      // --------------------------------------------------------- out stores
      if (lane == 0) {
        uint32_t ubase = 0, nitem = 0;
        bool ok = true;
        for (int it = cluster; it < p.items && ok; it += nclusters, ++nitem) {
          const Item x = decode_item(p, it);
          const uint32_t gbase = ubase + v_uses(x);
          ubase = gbase + 4;
#pragma unroll 1
          for (int e = 0; e < 4 && ok; ++e) {
            const uint32_t st = (gbase + e) % NV;
            ok = mbar_wait(bar(STAGED + e), nitem & 1, abort_flag, kWaitLimitNs, 370);
            if (!ok) break;
            tma_store_4d(&maps.out4, sb + O_VRING + st * kVStage, 0, (x.t0 + orow0) * kHeads,
                         2 * e, x.b);
            bulk_commit();
            if (e & 1) {
              // both stages of this value half are in flight: release them as
              // their reads complete
              bulk_wait_read_n<1>();
              mbar_arrive(bar(VEMPTY + (gbase + e - 1) % NV));
              bulk_wait_read_all();
              mbar_arrive(bar(VEMPTY + st));
            }
          }
        }
        bulk_wait_all();
      }
    } else if (warp == 2) {
      // --------------------------------------------------------- MMA (O += P V), even CTA
      if (leader && lane == 0) {
        uint32_t u = 0, sj = 0, nitem = 0, ncorr = 0, vpar = 0;
        bool ok = true;
        const uint32_t idesc = idesc_bf16_f32(2 * kRows, 256, false, true);
        // VHA of gate stages [e0, e1) of the item whose gate stages start at
        // ring use `gb` (parity `par`): D[c, n] = sum_k x[k, c] (I + M')[n, k]
        // per position, A = the staged x read MN-major (LBO: next 64 value
        // columns, SBO: next 8 heads), B = I then M'^T (K-major), 2 x 4 K
        // steps of 16 heads
        auto vha_issue = [&](int e0, int e1, uint32_t gb, uint32_t par) -> bool {
          if constexpr (kVha) {
            const uint32_t vdesc = idesc_bf16_f32(2 * kRows, 64, true, false);
            const uint64_t bi = sdesc_sw128(sb + O_VHAB, 16, 1024);
            const uint64_t bm = sdesc_sw128(sb + O_VHAB + 4096, 16, 1024);
#pragma unroll 1
            for (int e = e0; e < e1; ++e) {
              if (!mbar_wait_cluster(bar(XSTAGED + e), par, abort_flag, kWaitLimitNs, 355))
                return false;
              tc_fence_after();
              const uint32_t st = (gb + e) % NV;
#pragma unroll
              for (int pp = 0; pp < 2; ++pp) {
                const uint64_t ad =
                    sdesc_sw128(sb + O_VRING + st * kVStage + 8192 * pp, 16384, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  umma_pair_if(tmem + 128 * e + 64 * pp, ad + 128 * (k & 3),
                               (k < 4 ? bi : bm) + 2 * (k & 3), vdesc, k == 0 ? 0u : 1u, true);
              }
              umma_pair_commit_mc(bar(VHADONE + e), kMaskO);
            }
          }
          return true;
        };
        // value half 1 of the previous item is mixed as soon as its stages
        // are staged (polled between P.V stages), at the latest before the
        // first P.V stage of value half 1, whose O columns its D occupies
        int vha_next = 4;           // next gate stage still to mix (4: none)
        uint32_t vha_gb = 0, vha_par = 0;
        auto vha_poll = [&](bool block) -> bool {
          while (vha_next < 4) {
            if (!block && !mbar_try_wait_acq_cluster(bar(XSTAGED + vha_next), vha_par)) return true;
            if (!vha_issue(vha_next, vha_next + 1, vha_gb, vha_par)) return false;
            ++vha_next;
          }
          return true;
        };
        for (int it = cluster; it < p.items && ok; it += nclusters, ++nitem) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            const int n = tile_n(x, j);
            if (j > 0)  // an item's first tile never needs a rescale of O
              ok &= mbar_wait_cluster(bar(CORR + (ncorr & 1)), (ncorr >> 1) & 1, abort_flag,
                                      kWaitLimitNs, 351);
            ncorr += (j > 0);
            const bool first = j == 0, last = j == x.ntiles - 1;
            const int nh1 = sub_n(n, 1);
            const bool two = nh1 > 0;
            const int nst = two ? 4 : 2;
            const uint32_t pfree0 = bar(PFREE + (sj & 1) * 2);
#pragma unroll 1
            for (int s = 0; s < nst; ++s, ++u) {
              int dh, h;
              pv_stage(s, two, first || last, dh, h);
              if (kVha && vha_next < 4) ok &= vha_poll(first && dh == 1);
              if (first && h == 0)  // this value half of the last item's O is read out
                ok &= mbar_wait_cluster(bar(OFREE + dh), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs,
                                        352);
              if (dh == 0) ok &= mbar_wait(bar(PFULL + h), sj & 1, abort_flag, kWaitLimitNs, 350);
              const uint32_t st = u % NV;
              ok &= mbar_wait(bar(VFULL + st), (vpar >> st) & 1, abort_flag, kWaitLimitNs, 353);
              vpar ^= 1u << st;
              tc_fence_after();
              // eight K steps of 16 keys; descriptors move by their start address
              const int ksteps = sub_n(n, h) >> 4;
              const uint64_t ad = sdesc_noswz(sb + O_P + h * kPBuf, 2048, 128);
              const uint64_t bd = sdesc_sw128(sb + O_VRING + st * kVStage, 16384, 1024);
              const uint32_t dt = tmem + 256 * dh;
              const uint32_t acc0 = (first && h == 0) ? 0u : 1u;
#pragma unroll
              for (int k = 0; k < 8; ++k)
                umma_pair_if(dt, ad + 256 * k, bd + 128 * k, idesc, k == 0 ? acc0 : 1u, k < ksteps);
              umma_pair_commit_mc(bar(VEMPTY + st), kMaskO);
              // P buffer h done once value half 1 used it; O half 0 final after
              // the last tile's half-0 stages
              const bool pdone = dh == 1;
              const bool o0 = last && dh == 0 && h == (two ? 1 : 0);
              if (pdone || o0) {
                umma_pair_commit_mc_if(bar(PBUFFREE + h), kMaskO, pdone);  // smem P buffers
                umma_pair_commit_mc_if(pfree0 + 8 * h, kMaskS, pdone);     // scratch slots
                umma_pair_commit_mc_if(bar(OFULL + 0), kMaskO, o0);
              }
            }
            if (!two) {  // empty sub-tile 1: its buffer handshake still runs
              ok &= mbar_wait(bar(PFULL + 1), sj & 1, abort_flag, kWaitLimitNs, 350);
              tc_fence_after();
              umma_pair_commit_mc(bar(PBUFFREE + 1), kMaskO);
              umma_pair_commit_mc(pfree0 + 8, kMaskS);
            }
            umma_pair_commit_mc(bar(PVDONE + (sj & 1)), kMaskO);   // all of tile sj's P.V
          }
          if (!ok) break;
          umma_pair_commit_mc(bar(OFULL + 1), kMaskO);
          if constexpr (kVha) {
            ok = vha_issue(0, 2, u, nitem & 1);   // value half 0 now, half 1 polled
            if (!ok) break;
            vha_next = 2;
            vha_gb = u;
            vha_par = nitem & 1;
          }
          u += 4;  // gate stages, consumed by the epilogue
        }
        if (kVha && ok) ok = vha_poll(true);
        umma_pair_commit_mc(bar(DRAIN), 1u << rank);
        mbar_wait(bar(DRAIN), 0, abort_flag, kWaitLimitNs, 354);
      }
    } else if (warp >= 3) {
      // --------------------------------------------------------- correction + epilogue
      // warps 3-10: correction, and the epilogue of value half 0 (stage kv);
      // warps 13-16 (helpers): the epilogue of value half 1 (stages 2 and 3)
      const bool helper = warp >= 13;
      const int wq = warp & 3;
      const int kv = helper ? 0 : (warp - 3) >> 2;
      const int row = wq * 32 + lane;
      const uint32_t tq = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      const uint32_t tl = tq + 256 * kv;     // rescale: value columns [256 kv, +256)
      const volatile int* flags = reinterpret_cast<const volatile int*>(smem + O_FLAGS);
      const volatile float* alpha_s = reinterpret_cast<const volatile float*>(smem + O_ALPHA);
      const volatile float* invl_s = reinterpret_cast<const volatile float*>(smem + O_INVL);
      const uint32_t partnerStatsFree = mapa_shared(bar(STATSFREE), rank - 2);
      uint32_t sj = 0, nitem = 0, ubase = 0, ncorr = 0, gpar = 0;
      bool ok = true;
      for (int it = cluster; it < p.items && ok; it += nclusters, ++nitem) {
        const Item x = decode_item(p, it);
        ++sj;  // the first tile of an item needs no correction
        for (int j = 1; j < x.ntiles && !helper; ++j, ++sj, ++ncorr) {
          if (!mbar_wait_cluster_warp(bar(PREADY + (sj & 1) * 2), (sj >> 1) & 1, abort_flag,
                                      kWaitLimitNs, 360)) {
            ok = false;
            break;
          }
          // rarely: rescale O rows before the next P.V accumulates into them
          const volatile int* fl = flags + 4 * (sj & 1);
          const bool any = (fl[0] | fl[1] | fl[2] | fl[3]) != 0;
          if (any) {
            const uint32_t pj = sj - 1;   // wait for every P.V of the previous tile
            if (!mbar_wait_warp(bar(PVDONE + (pj & 1)), (pj >> 1) & 1, abort_flag, kWaitLimitNs,
                                361)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float a = alpha_s[128 * (sj & 1) + row];
            uint32_t r[32];
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
              tmem_ld32(tl + c, r);
              tmem_wait_ld_dep32(r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * a);
              tmem_st32(tl + c, r);
            }
            tmem_wait_st();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(lbar(CORR + (ncorr & 1)));  // TMEM only
        }
        if (!ok) break;
        if (helper) sj += x.ntiles - 1;
        // ---------------------------------------------------------- epilogue
        const int ee = helper ? 1 : 0;
        if (!mbar_wait_cluster_warp(bar(STATSFULL), nitem & 1, abort_flag, kWaitLimitNs, 363)) {
          ok = false;
          break;
        }
        const float il = invl_s[row];
        const float hil = 0.5f * il;
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(partnerStatsFree);
        if (!mbar_wait_warp(bar(OFULL + ee), nitem & 1, abort_flag, kWaitLimitNs, 362)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t gbase = ubase + v_uses(x);
        ubase = gbase + 4;
        // parity of each gate stage's use count so far (every epilogue warp
        // walks all four stages' uses, reading only its own)
        uint32_t gwait = 0;   // bit e: the wait parity of gate stage e
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t st = (gbase + e) % NV;
          gwait |= ((gpar >> st) & 1u) << e;
          gpar ^= 1u << st;
        }
#pragma unroll 1
        for (int e2 = 0; e2 < (helper ? 2 : 1); ++e2) {
          const int e = helper ? 2 + e2 : kv;   // g / out stage: value columns [128e, 128e + 128)
          const uint32_t st = (gbase + e) % NV;
          if (!mbar_wait_warp(bar(GFULL + st), (gwait >> e) & 1u, abort_flag, kWaitLimitNs, 364)) {
            ok = false;
            break;
          }
          uint8_t* stage = smem + O_VRING + st * kVStage;
#pragma unroll 1
          for (int q32 = 0; q32 < 4; ++q32) {
            const int sl = q32 >> 1;
            uint32_t o[32];
            tmem_ld32(tq + 128 * e + 32 * q32, o);
            tmem_wait_ld_dep32(o);
            if (!kVha && q32 == 3 && e2 == (helper ? 1 : 0)) {  // this warp's part of O read out
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster_relaxed(lbar(OFREE + ee));
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const int c = 4 * (q32 & 1) + c4;   // 16-byte chunk of the 128-byte slab row
              uint4* ptr = reinterpret_cast<uint4*>(stage + sl * 16384 + sw128_offset(row, c));
              const uint4 gv = *ptr;
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
              uint32_t ow[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int oc = 8 * c4 + 2 * q;
                ow[q] = gate_pair_bf16(__uint_as_float(o[oc]), __uint_as_float(o[oc + 1]), hil,
                                       gw[q]);
              }
              *ptr = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
          }
          fence_proxy_async_smem();   // this thread's writes, read next by the TMA store
          if constexpr (kVha) {       // ... or first by the VHA MMA, which also
            tc_fence_before();        // overwrites the O columns read above
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lbar(XSTAGED + e));
          } else {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(STAGED + e));
          }
        }
        if constexpr (kVha) {
          // y = D: lane = value column c of the stage, D columns = heads.
          // Lanes c (even) and c + 1 swap one D value per pair of heads
          // (j, j + 4) so that each writes one bf16 pair: the even lane head
          // j, the odd lane head j + 4 (rows 4 apart fall on disjoint banks).
          const int cw = row & ~1;                 // even column of the pair
          const bool odd = (lane & 1) != 0;
#pragma unroll 1
          for (int e2 = 0; e2 < (helper ? 2 : 1) && ok; ++e2) {
            const int e = helper ? 2 + e2 : kv;
            const uint32_t st = (gbase + e) % NV;
            if (!mbar_wait_warp(bar(VHADONE + e), nitem & 1, abort_flag, kWaitLimitNs, 365)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* stage = smem + O_VRING + st * kVStage + (cw >> 6) * 16384;
#pragma unroll 1
            for (int i = 0; i < 4; ++i) {          // position i >> 1, heads 32 (i & 1) + 0..31
              uint32_t d[32];
              tmem_ld32(tq + 128 * e + 32 * i, d);
              tmem_wait_ld_dep32(d);
              if (i == 3 && e2 == (helper ? 1 : 0)) {  // this warp's D read out: O is free
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(lbar(OFREE + ee));
              }
              const int r0 = 32 * i + (odd ? 4 : 0);  // stage row of head j (+4 if odd)
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (j & 4) continue;
                const uint32_t send = odd ? d[j] : d[j + 4];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 1);
                const float dl = __uint_as_float(odd ? recv : d[j]);
                const float dh = __uint_as_float(odd ? d[j + 4] : recv);
                *reinterpret_cast<uint32_t*>(stage + sw128_offset(r0 + j, (cw & 63) >> 3) +
                                             2 * (cw & 7)) = pack_bf16x2(dl, dh);
              }
            }
            fence_proxy_async_smem();   // read next by the TMA store
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(STAGED + e));
          }
        }
      }
    }
  }

  __syncwarp();
  if (threadIdx.x == 0) abort_drain(abort_flag);
  cluster_sync_all();  // no CTA leaves while a peer may still touch its shared memory or TMEM
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace prefill3
}  // namespace hca
