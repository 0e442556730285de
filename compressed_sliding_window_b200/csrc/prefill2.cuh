// HCA prefill attention, version 2: an asymmetric CTA pair per 128-row tile.
//
// What is computed ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1; xenospectrum
// analysis, section 活性140億パラメータと長文処理を支える仕組み): for each query
// position t and head h, one softmax over the compressed entries j < nc(t) and
// the raw keys max(0, t-127) .. t, then out = sigmoid(g) * (P . V).
//
// Why a pair.  A 128-row fp32 accumulator 512 wide fills all 512 TMEM columns
// of an SM, so no single SM can hold O and the scores.  The cluster's two CTAs
// split the work by operation instead of by value columns:
//   rank 0, the S-CTA: Q resident in shared memory, S = Q K^T on tcgen05 into
//     two 256-column TMEM buffers, the online softmax, and P (bf16) in 128-key
//     sub-tiles.  P does not go over DSMEM (its per-SM store rate is far below
//     what a tile needs): the S-CTA writes each sub-tile to a small
//     L2-resident scratch with plain global stores, already in the no-swizzle
//     core-matrix layout the MMA reads (8-key chunk major, so the 32 rows of a
//     warp store 512 contiguous bytes), and a warp of rank 1 pulls it with one
//     bulk copy.  Only the per-row rescale factors cross over DSMEM.
//   rank 1, the O-CTA: the full O (128 x 512 fp32) in TMEM, O += P V on
//     tcgen05, the rare O rescale, and the epilogue out = O / l * sigmoid(g)
//     (g staged by TMA, out written in place and TMA-stored).
// Each SM issues only N = 256 MMAs (M = 128, K = 16), the shape that reaches
// the tensor-core peak; QK^T is computed once.
//
// Tiles.  Rows = 2 consecutive positions x 64 heads (one shared KV head).  Key
// tiles: ceil(nc(t0+1) / 256) compressed tiles of up to 256 entries and one
// raw tile of 144 keys [t0-127, t0+16] (the window of both positions plus key
// t0+1 for the second one, padded to a multiple of 16).
//
// TMA.  Two producer warps per CTA alternate ring stages (one issuing warp
// cannot keep an SM's copy engine busy).  V and g use 3-D boxes over a
// (64-element slab, row, slab index) view of the [.., 512] rows, so one copy
// brings 4 (V) or 2 (g) 64-wide column slabs, already in the layout the MMA
// and the epilogue read.
//
// Warp roles (544 threads): warps 0-1 TMA producers, warp 2 MMA issuer and
// TMEM owner, warps 3-10 compute: two warps per TMEM lane quadrant, so a tile
// row is shared by two threads.  On rank 0 each of them owns one 128-key half
// of the score tile (= one P sub-tile; the row max is exchanged through shared
// memory under a 64-thread named barrier); on rank 1 they rescale O (each 256
// of the 512 value columns) and run the epilogue of O's value half 0 (128
// columns per warp).  Rank 1 also has warp 11, the P copier, warp 12, which
// stores the epilogue's output stages and hands them back to the producers,
// and warps 13-16, one per lane quadrant, which run the epilogue of value
// half 1 (both of its stages) in parallel with half 0 (the epilogue is bound
// by instruction latency, not issue slots).  Warps 11-16 of rank 0 have no
// role.
//
// Code size.  The kernel is bound by instruction fetch long before its loops
// are: every role's hot loop is kept small (32-column chunks, one code path
// for masked and unmasked chunks, bounded waits polled out of line).
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace prefill2 {

constexpr int kRows = 128;
constexpr int kHeads = 64;
constexpr int kKT = 256;     // compressed key tile
constexpr int kWinN = 144;   // raw key tile
constexpr int kThreads = 544;
constexpr int kScratchPerPair = 4 * 32768;   // 2 tile parities x 2 sub-tiles
constexpr float kTau = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---- S-CTA shared memory
constexpr int S_Q = 0;                       // 2 halves x [4 slabs][128 rows][64]
constexpr int kQHalf = 65536;
constexpr int S_KRING = 131072;              // 3 stages x [256 keys][64]
constexpr int kKStages = 3;
constexpr int kKStage = 32768;
// ---- O-CTA shared memory
constexpr int O_P = 0;                       // 2 sub-tile buffers x [16 key chunks][128 rows][8 keys]
constexpr int kPBuf = 32768;
constexpr int O_VRING = 65536;               // 5 stages x [4 slabs][64 keys][64 dv]
constexpr int kVStages = 5;
constexpr int kVStage = 32768;

// ---- barriers (both CTAs, same offsets)
constexpr int BAR = 229376;
enum {
  QFULL = 0, QEMPTY = 2, KFULL = 4, KEMPTY = KFULL + kKStages, SFULL = KEMPTY + kKStages,
  SFREE = SFULL + 2, PFREE = SFREE + 2, STATSFREE = PFREE + 4,
  VFULL = STATSFREE + 1, VEMPTY = VFULL + kVStages, PREADY = VEMPTY + kVStages,
  PFULL = PREADY + 4, PBUFFREE = PFULL + 2, CORR = PBUFFREE + 2,
  PVDONE = CORR + 2, OFULL = PVDONE + 2, OFREE = OFULL + 2, STATSFULL = OFREE + 2,
  STAGED = STATSFULL + 1, DRAIN = STAGED + 4, NBAR = DRAIN + 1
};
constexpr int kTmemSlot = BAR + 8 * NBAR;
constexpr int kAbortSlot = kTmemSlot + 4;
// S-CTA: per-row statistics exchanged between the two warps of a row
// ([2 parity][2 halves][128] float) and their ok flags ([2][2][4 quadrants] int)
constexpr int S_XMAX = BAR + 512;
constexpr int S_XOK = S_XMAX + 2048;
// O-CTA: rescale factors [2 tile parities][128] float, rescale flags
// [2 tile parities][4] int, 1/l [128] float
constexpr int O_ALPHA = BAR + 512;
constexpr int O_FLAGS = O_ALPHA + 1024;
constexpr int O_INVL = O_FLAGS + 64;
constexpr int kSmemBytes = S_XOK + 64;
// The dynamic shared memory base is 1024-aligned (checked at run time), so no
// alignment slack is allocated: the S-CTA needs every byte.
constexpr int kSmemAlloc = kSmemBytes;
static_assert(kAbortSlot + 4 <= kSmemBytes, "barrier region overflow");
static_assert(O_VRING + kVStages * kVStage <= BAR, "O-CTA ring overflow");
static_assert(O_INVL + 512 <= kSmemBytes, "O-CTA layout overflow");
static_assert(S_KRING + kKStages * kKStage <= BAR, "S-CTA layout overflow");
static_assert(kSmemAlloc <= 232448, "shared memory budget");

struct Params {
  int B, T;
  int row_tiles;    // ceil(T / 2)
  int items;        // B * row_tiles
  float scale_log2; // softmax scale * log2(e)
  float* lse;       // [B, T, 64] or null
  uint8_t* pscratch;  // [pairs][4][32 KB] P sub-tile images
};

struct Maps {
  CUtensorMap q4;    // (64, T*64, 8, B)  box (64, 128, 4, 1): one Q half
  CUtensorMap ck;    // [B][nb][512]      box (64, 64, 1): tiles load only the rows they use
  CUtensorMap kwin;  // [B][T][512]       box (64, 144, 1)
  CUtensorMap cv4;   // (64, nb, 8, B)    box (64, 64, 4, 1)
  CUtensorMap v4;    // (64, T, 8, B)     box (64, 64, 4, 1)
  CUtensorMap g4;    // (64, T*64, 8, B)  box (64, 128, 2, 1)
  CUtensorMap out4;  // same as g4
};

__device__ __forceinline__ int nc_of(int t) { return t >= 127 ? (t - 127) / 128 : 0; }

struct Item {
  int b, t0;
  bool has_p1;
  int nc0, nc1, n_ctiles, ntiles;
};

__device__ __forceinline__ Item decode_item(const Params& p, int it) {
  Item x;
  const int rank = it / p.B;
  x.b = it - rank * p.B;
  x.t0 = 2 * (p.row_tiles - 1 - rank);
  x.has_p1 = x.t0 + 1 < p.T;
  x.nc0 = nc_of(x.t0);
  x.nc1 = x.has_p1 ? nc_of(x.t0 + 1) : x.nc0;
  x.n_ctiles = (x.nc1 + kKT - 1) / kKT;
  x.ntiles = x.n_ctiles + 1;
  return x;
}

// MMA width of key tile j (multiple of 16)
__device__ __forceinline__ int tile_n(const Item& x, int j) {
  if (j < x.n_ctiles) return (min(kKT, x.nc1 - j * kKT) + 15) & ~15;
  return kWinN;
}
// keys of sub-tile h (0: columns 0..127, 1: columns 128..) of a tile of width n
__device__ __forceinline__ int sub_n(int n, int h) { return h == 0 ? min(n, 128) : max(0, n - 128); }

// P.V order of one tile, walked by both the V producer and the MMA issuer:
// step s of 2 * nkt (nkt = 64-key chunks of both sub-tiles, nk0 of them in
// sub-tile 0) -> value half dh, sub-tile h, chunk kc.  An item's first and
// last tiles run value half major (the previous item's epilogue hands O back
// one half at a time, and this item's epilogue starts on half 0 while half 1
// still accumulates); the tiles between run sub-tile major (P buffer h is
// free as soon as both value halves have used it).
struct PvStep {
  int dh, h, kc;
};
__device__ __forceinline__ PvStep pv_step(int s, int nk0, int nkt, bool half_major) {
  PvStep r;
  int q;
  if (half_major) {
    r.dh = s >= nkt ? 1 : 0;
    q = s - r.dh * nkt;
  } else {
    r.dh = s & 1;
    q = s >> 1;
  }
  r.h = q >= nk0 ? 1 : 0;
  r.kc = q - r.h * nk0;
  return r;
}

// 4-D tensor-map TMA copies
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    prefill2_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  if ((sb & 1023u) != 0) {  // uniform: every thread sees the same base
    if (threadIdx.x == 0) record_error(DEVERR_LAYOUT, 100);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sb + BAR + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortSlot);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(SFREE + 0), 8);
    mbar_init(bar(SFREE + 1), 8);
    mbar_init(bar(STATSFREE), 12);
    for (int q = 0; q < 4; ++q) mbar_init(bar(PREADY + q), 4);
    mbar_init(bar(CORR + 0), 8);
    mbar_init(bar(CORR + 1), 8);
    mbar_init(bar(OFREE + 0), 8);
    mbar_init(bar(OFREE + 1), 4);
    mbar_init(bar(STATSFULL), 4);
    for (int e = 0; e < 4; ++e) mbar_init(bar(STAGED + e), 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  cluster_sync_all();  // both CTAs' barriers exist before any remote access
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (rank == 0) {
    // =====================================================================
    // S-CTA
    // =====================================================================
    if (warp <= 1) {
      // --------------------------------------------------------- producers
      if (lane == 0) {
        const int me = warp;
        uint32_t u = 0, nitem = 0;
        bool ok = true;
        for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
          const Item x = decode_item(p, it);
          if (me == 0 && it + npairs < p.items) {  // warm L2 with the next item's Q
            const Item y = decode_item(p, it + npairs);
            tma_prefetch_4d(&maps.q4, 0, y.t0 * kHeads, 0, y.b);
            tma_prefetch_4d(&maps.q4, 0, y.t0 * kHeads, 4, y.b);
          }
          // Q half `me`
          ok = mbar_wait(bar(QEMPTY + me), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs, 110);
          if (!ok) break;
          mbar_expect_tx(bar(QFULL + me), kQHalf);
          tma_load_4d(sb + S_Q + me * kQHalf, &maps.q4, bar(QFULL + me), 0, x.t0 * kHeads, 4 * me,
                      x.b);
          for (int j = 0; j < x.ntiles && ok; ++j) {
            const bool comp = j < x.n_ctiles;
#pragma unroll 1
            for (int d = 0; d < 8; ++d, ++u) {
              if ((u & 1) != static_cast<uint32_t>(me)) continue;
              const uint32_t st = u % kKStages;
              ok = mbar_wait(bar(KEMPTY + st), ((u / kKStages) & 1) ^ 1, abort_flag, kWaitLimitNs,
                             111);
              if (!ok) break;
              const uint32_t dst = sb + S_KRING + st * kKStage;
              if (comp) {
                const int n64 = (tile_n(x, j) + 63) >> 6;   // 64-row boxes this tile uses
                mbar_expect_tx(bar(KFULL + st), n64 * 8192);
#pragma unroll 1
                for (int r = 0; r < n64; ++r)
                  tma_load_3d(dst + r * 8192, &maps.ck, bar(KFULL + st), 64 * d, j * kKT + 64 * r,
                              x.b);
              } else {
                mbar_expect_tx(bar(KFULL + st), kWinN * 128);
                tma_load_3d(dst, &maps.kwin, bar(KFULL + st), 64 * d, x.t0 - 127, x.b);
              }
            }
          }
        }
      }
    } else if (warp == 2) {
      // --------------------------------------------------------- MMA (S = Q K^T)
      if (lane == 0) {
        uint32_t u = 0, sj = 0, nitem = 0;
        bool ok = true;
        for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            // straight step loop, predicated commits (see the O-CTA issuer)
            const uint32_t buf = sj & 1;
            ok &= mbar_wait(bar(SFREE + buf), ((sj >> 1) & 1) ^ 1, abort_flag, kWaitLimitNs, 120);
            const uint32_t idesc = idesc_bf16_f32(kRows, tile_n(x, j), false, false);
            const uint32_t dS = tmem + 256 * buf;
            const bool first = j == 0, last = j + 1 == x.ntiles;
#pragma unroll 1
            for (int d = 0; d < 8; ++d, ++u) {
              if (first && (d & 3) == 0)
                ok &= mbar_wait(bar(QFULL + (d >> 2)), nitem & 1, abort_flag, kWaitLimitNs, 121);
              const uint32_t st = u % kKStages;
              ok &= mbar_wait(bar(KFULL + st), (u / kKStages) & 1, abort_flag, kWaitLimitNs, 122);
              tc_fence_after();
              const uint32_t qa = sb + S_Q + (d >> 2) * kQHalf + (d & 3) * 16384;
              const uint32_t ka = sb + S_KRING + st * kKStage;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_bf16(dS, sdesc_sw128(qa + 32 * k, 16, 1024), sdesc_sw128(ka + 32 * k, 16, 1024),
                          idesc, (d | k) != 0);
              umma_commit(bar(KEMPTY + st));
              umma_commit_if(bar(QEMPTY + (d >> 2)), last && (d & 3) == 3);
            }
            umma_commit(bar(SFULL + buf));
          }
        }
        umma_commit(bar(DRAIN));
        mbar_wait(bar(DRAIN), 0, abort_flag, kWaitLimitNs, 123);
      }
    } else if (warp >= 11) {
      // the P copier and out store roles exist on rank 1 only
    } else {
      // --------------------------------------------------------- softmax
      const int wq = warp & 3;
      const int half = (warp - 3) >> 2;       // key columns [128 half, 128 half + 128)
      const int row = wq * 32 + lane;
      const int pos = row >> 6;
      const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      float* xmax = reinterpret_cast<float*>(smem + S_XMAX);
      volatile int* xok = reinterpret_cast<volatile int*>(smem + S_XOK);
      uint8_t* const pscr = p.pscratch + static_cast<size_t>(pair) * kScratchPerPair;
      const uint32_t peerAlpha = mapa_shared(sb + O_ALPHA, 1);
      const uint32_t peerFlags = mapa_shared(sb + O_FLAGS, 1);
      const uint32_t peerInvl = mapa_shared(sb + O_INVL, 1);
      const uint32_t peerPReady = mapa_shared(bar(PREADY), 1);
      const uint32_t peerStatsFull = mapa_shared(bar(STATSFULL), 1);
      uint32_t sj = 0, nitem = 0, nx = 0;
      bool ok = true, both = true;
      // A row is shared with warp (warp ^ 4's partner): both write, a 64-thread
      // named barrier, both read.  The ok flags travel with the value, so the
      // two warps always leave their loops at the same exchange and never
      // wait at the named barrier for a warp that has gone.
      auto exchange = [&](float v) -> float {
        const uint32_t xp = nx & 1;
        xmax[(xp * 2 + half) * 128 + row] = v;
        if (lane == 0) xok[(xp * 2 + half) * 4 + wq] = ok ? 1 : 0;
        named_bar_sync(1 + wq, 64);
        const float o = xmax[(xp * 2 + (half ^ 1)) * 128 + row];
        both = ok && xok[(xp * 2 + (half ^ 1)) * 4 + wq] != 0;
        ++nx;
        return o;
      };
      // The P stores of a tile are published one step later (after the next
      // tile's row max), so the wait for them to drain overlaps that work.
      uint32_t pend = 0;   // scratch slot + 1 of the unpublished sub-tile
      auto publish = [&]() {
        fence_proxy_async_all();  // the scratch is read by the peer's bulk copy (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(peerPReady + 8 * (pend - 1));
        pend = 0;
      };
      for (int it = pair; it < p.items; it += npairs, ++nitem) {
        const Item x = decode_item(p, it);
        const int t = x.t0 + pos;
        const int ncp = pos ? x.nc1 : x.nc0;
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < x.ntiles; ++j, ++sj) {
          const uint32_t buf = sj & 1;
          if (ok) ok = mbar_wait_warp(bar(SFULL + buf), (sj >> 1) & 1, abort_flag, kWaitLimitNs, 130);
          tc_fence_after();
          const int n = tile_n(x, j);
          const int nh = sub_n(n, half);
          // visible columns of this tile for this row: [clo, chi)
          int clo = 0, chi;
          if (j < x.n_ctiles) {
            chi = min(n, max(0, ncp - j * kKT));
          } else {
            clo = max(127 - x.t0, pos);
            chi = 128 + pos;
          }
          const int c0 = 128 * half;
          const uint32_t sbase = tl + 256 * buf + c0;
          // One code path for full and partly masked chunks (the unrolled
          // loops are the hot code; a second copy of each costs more in
          // instruction fetch than the two compares per score save).
          // pass A: this half's row max of the raw scores
          float mraw = -INFINITY;
          // 32-column chunks keep the unrolled bodies small (instruction fetch)
#pragma unroll 1
          for (int cc = 0; ok && cc < nh; cc += 32) {
            uint32_t r[32];
            tmem_ld32(sbase + cc, r);
            tmem_wait_ld_dep32(r);
            const int lo = clo - c0 - cc, hi = chi - c0 - cc;   // visible range in this chunk
#pragma unroll
            for (int c = 0; c < 32; ++c)
              mraw = fmaxf(mraw, (c >= lo && c < hi) ? __uint_as_float(r[c]) : -INFINITY);
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
          // scratch slot of this (tile parity, half): free once the O-CTA has
          // finished P.V of the tile two back
          const uint32_t slot = (sj & 1) * 2 + half;
          if (ok)
            ok = mbar_wait_cluster_warp(bar(PFREE + slot), ((sj >> 1) & 1) ^ 1, abort_flag,
                                        kWaitLimitNs, 131);
          uint8_t* const gdst = pscr + slot * 32768;
          // pass B: probabilities into the scratch slot
          float rs = 0.f;
#pragma unroll 1
          for (int cc = 0; ok && cc < nh; cc += 32) {
            uint32_t r[32];
            tmem_ld32(sbase + cc, r);
            tmem_wait_ld_dep32(r);
            uint32_t pk[16];
            const int lo = clo - c0 - cc, hi = chi - c0 - cc;
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
            // chunk-major image: 8-key chunk k8 of row `row` at k8 * 2048 + 16 * row,
            // so the 32 lanes of a warp store 512 contiguous bytes
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              const int k8 = (cc >> 3) + c8;
              *reinterpret_cast<uint4*>(gdst + k8 * 2048 + 16 * row) =
                  make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
            }
          }
          if (ok && half == 0) {
            st_cluster_b32(peerAlpha + 512 * (sj & 1) + 4 * row, __float_as_uint(alpha));
            const int any = __any_sync(0xffffffffu, resc) ? 1 : 0;
            if (lane == 0)
              st_cluster_b32(peerFlags + 16 * (sj & 1) + 4 * wq, static_cast<uint32_t>(any));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(SFREE + buf));  // S buffer read out
          pend = slot + 1;
          l = l * alpha + rs;
        }
        if (!both) break;
        // row sum = both halves (one more exchange); 1/l to the O-CTA
        // epilogue, lse to the caller
        l += exchange(l);
        if (!both) break;
        if (pend) publish();
        if (half == 0) {
          if (!mbar_wait_cluster_warp(bar(STATSFREE), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs,
                                      132)) {
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
    // O-CTA
    // =====================================================================
    // V stage uses of one item: per tile, both value halves of every 64-key
    // chunk of both sub-tiles
    auto v_uses = [&](const Item& x) -> uint32_t {
      uint32_t n_uses = 0;
      for (int j = 0; j < x.ntiles; ++j) {
        const int n = tile_n(x, j);
        n_uses += 2 * ((sub_n(n, 0) + 63) / 64) + 2 * ((sub_n(n, 1) + 63) / 64);
      }
      return n_uses;
    };
    if (warp <= 1) {
      // --------------------------------------------------------- producers
      if (lane == 0) {
        const int me = warp;
        uint32_t u = 0;
        bool ok = true;
        auto stage_load = [&](const CUtensorMap* map, int y, int z, int w) -> bool {
          if ((u & 1) == static_cast<uint32_t>(me)) {
            const uint32_t st = u % kVStages;
            if (!mbar_wait(bar(VEMPTY + st), ((u / kVStages) & 1) ^ 1, abort_flag, kWaitLimitNs,
                           140))
              return false;
            mbar_expect_tx(bar(VFULL + st), kVStage);
            tma_load_4d(sb + O_VRING + st * kVStage, map, bar(VFULL + st), 0, y, z, w);
          }
          ++u;
          return true;
        };
        for (int it = pair; it < p.items && ok; it += npairs) {
          const Item x = decode_item(p, it);
          if (me == 0) {  // warm L2 with this item's gate rows; they are staged after its V
#pragma unroll 1
            for (int e = 0; e < 4; ++e) tma_prefetch_4d(&maps.g4, 0, x.t0 * kHeads, 2 * e, x.b);
          }
          for (int j = 0; j < x.ntiles && ok; ++j) {
            const int n = tile_n(x, j);
            const bool comp = j < x.n_ctiles;
            const int nk0 = (sub_n(n, 0) + 63) >> 6;
            const int nkt = nk0 + ((sub_n(n, 1) + 63) >> 6);
            for (int s = 0; s < 2 * nkt && ok; ++s) {
              const PvStep q = pv_step(s, nk0, nkt, j == 0 || j == x.ntiles - 1);
              const int key = 128 * q.h + 64 * q.kc;
              ok = stage_load(comp ? &maps.cv4 : &maps.v4, comp ? j * kKT + key : x.t0 - 127 + key,
                              4 * q.dh, x.b);
            }
          }
#pragma unroll 1
          for (int e = 0; e < 4 && ok; ++e) ok = stage_load(&maps.g4, x.t0 * kHeads, 2 * e, x.b);
        }
      }
    } else if (warp == 11) {
      // --------------------------------------------------------- P copier
      if (lane == 0) {
        const uint8_t* const pscr = p.pscratch + static_cast<size_t>(pair) * kScratchPerPair;
        uint32_t sj = 0;
        bool ok = true;
        for (int it = pair; it < p.items && ok; it += npairs) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            const int n = tile_n(x, j);
#pragma unroll 1
            for (int h = 0; h < 2 && ok; ++h) {
              const int nh = sub_n(n, h);
              ok = mbar_wait_cluster(bar(PREADY + (sj & 1) * 2 + h), (sj >> 1) & 1, abort_flag,
                                     kWaitLimitNs, 145) &&
                   mbar_wait(bar(PBUFFREE + h), (sj & 1) ^ 1, abort_flag, kWaitLimitNs, 146);
              if (!ok) break;
              if (nh > 0) {
                fence_proxy_async_all();
                const uint32_t bytes = nh > 64 ? 32768u : 16384u;
                mbar_expect_tx(bar(PFULL + h), bytes);
                asm volatile(
                    "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
                    " [%0], [%1], %2, [%3];" ::"r"(sb + O_P + h * kPBuf),
                    "l"(pscr + ((sj & 1) * 2 + h) * 32768), "r"(bytes), "r"(bar(PFULL + h))
                    : "memory");
              } else {
                mbar_arrive(bar(PFULL + h));
              }
            }
          }
        }
      }
    } else if (warp == 12) {
      // --------------------------------------------------------- out stores
      // The epilogue writes out over the g image of each 128-column stage;
      // this warp stores the stage and hands it back to the producers once
      // the copy engine has read it.
      if (lane == 0) {
        uint32_t ubase = 0, nitem = 0;
        bool ok = true;
        for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
          const Item x = decode_item(p, it);
          const uint32_t gbase = ubase + v_uses(x);
          ubase = gbase + 4;
#pragma unroll 1
          for (int e = 0; e < 4 && ok; ++e) {
            const uint32_t st = (gbase + e) % kVStages;
            ok = mbar_wait(bar(STAGED + e), nitem & 1, abort_flag, kWaitLimitNs, 170);
            if (!ok) break;
            tma_store_4d(&maps.out4, sb + O_VRING + st * kVStage, 0, x.t0 * kHeads, 2 * e, x.b);
            bulk_commit();
            if (e & 1) {
              // both stages of this value half are in flight: release them as
              // their reads complete
              bulk_wait_read_n<1>();
              mbar_arrive(bar(VEMPTY + (gbase + e - 1) % kVStages));
              bulk_wait_read_all();
              mbar_arrive(bar(VEMPTY + st));
            }
          }
        }
        bulk_wait_all();
      }
    } else if (warp == 2) {
      // --------------------------------------------------------- MMA (O += P V)
      if (lane == 0) {
        uint32_t u = 0, sj = 0, nitem = 0, ncorr = 0;
        bool ok = true;
        const uint32_t idesc = idesc_bf16_f32(kRows, 256, false, true);
        // The issuing thread's time goes to its own branches as much as to
        // waiting: the step loop is kept straight (commits and the short last
        // K steps predicated, the ok flag checked per tile; after a failed
        // bounded wait the abort flag makes every later wait return at once).
        for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            const int n = tile_n(x, j);
            if (j > 0)  // an item's first tile never needs a rescale of O
              ok &= mbar_wait(bar(CORR + (ncorr & 1)), (ncorr >> 1) & 1, abort_flag, kWaitLimitNs,
                              151);
            ncorr += (j > 0);
            const bool first = j == 0, last = j == x.ntiles - 1;
            const int nk0 = (sub_n(n, 0) + 63) >> 6, nk1 = (sub_n(n, 1) + 63) >> 6;
            const int nkt = nk0 + nk1;
            const uint32_t pfree0 = bar(PFREE + (sj & 1) * 2);
#pragma unroll 1
            for (int s = 0; s < 2 * nkt; ++s) {
              const PvStep q = pv_step(s, nk0, nkt, first || last);
              if (first && (s == 0 || s == nkt))  // this half of the last item's O is read out
                ok &= mbar_wait(bar(OFREE + q.dh), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs, 152);
              if (q.dh == 0 && q.kc == 0)
                ok &= mbar_wait(bar(PFULL + q.h), sj & 1, abort_flag, kWaitLimitNs, 150);
              // P.V of one 64-key chunk into one value half
              const int ksteps = min(4, (sub_n(n, q.h) - 64 * q.kc) >> 4);
              const uint32_t st = u % kVStages;
              ok &= mbar_wait(bar(VFULL + st), (u / kVStages) & 1, abort_flag, kWaitLimitNs, 153);
              ++u;
              tc_fence_after();
              // descriptors of the chunk's first K step; later steps only move
              // the start address (bits 0-13 hold address >> 4, no carry)
              const uint64_t ad = sdesc_noswz(sb + O_P + q.h * kPBuf + q.kc * 16384, 2048, 128);
              const uint64_t bd = sdesc_sw128(sb + O_VRING + st * kVStage, 8192, 1024);
              const uint32_t dt = tmem + 256 * q.dh;
              umma_bf16(dt, ad, bd, idesc, (first && q.h == 0 && q.kc == 0) ? 0u : 1u);
              umma_bf16_if(dt, ad + 256, bd + 128, idesc, 1u, ksteps > 1);
              umma_bf16_if(dt, ad + 512, bd + 256, idesc, 1u, ksteps > 2);
              umma_bf16_if(dt, ad + 768, bd + 384, idesc, 1u, ksteps > 3);
              umma_commit(bar(VEMPTY + st));
              // P buffer h done once value half 1 used its last chunk; O half 0
              // final after the last tile's half-0 pass
              const bool pdone = q.dh == 1 && q.kc == (q.h ? nk1 : nk0) - 1;
              const bool o0 = last && s == nkt - 1;
              if (pdone || o0) {  // rare: one branch instead of three predicated commits a step
                umma_commit_if(bar(PBUFFREE + q.h), pdone);           // smem P buffer reusable
                umma_commit_mc_if(pfree0 + 8 * q.h, 0x1, pdone);      // scratch slot (rank 0)
                umma_commit_if(bar(OFULL + 0), o0);
              }
            }
            if (nk1 == 0) {  // empty sub-tile 1: its buffer handshake still runs
              ok &= mbar_wait(bar(PFULL + 1), sj & 1, abort_flag, kWaitLimitNs, 150);
              tc_fence_after();
              umma_commit(bar(PBUFFREE + 1));
              umma_commit_mc(pfree0 + 8, 0x1);
            }
            umma_commit(bar(PVDONE + (sj & 1)));   // all of tile sj's P.V
          }
          if (!ok) break;
          umma_commit(bar(OFULL + 1));
          u += 4;  // g stages, consumed by the epilogue
        }
        umma_commit(bar(DRAIN));
        mbar_wait(bar(DRAIN), 0, abort_flag, kWaitLimitNs, 154);
      }
    } else {
      // --------------------------------------------------------- correction + epilogue
      // warps 3-10: correction, and the epilogue of value half 0 (stage half);
      // warps 13-16 (helpers): the epilogue of value half 1 (stages 2 and 3)
      const bool helper = warp >= 13;
      const int wq = warp & 3;
      const int half = helper ? 0 : (warp - 3) >> 2;
      const int row = wq * 32 + lane;
      const uint32_t tq = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      const uint32_t tl = tq + 256 * half;     // rescale: value columns [256 half, +256)
      const volatile int* flags = reinterpret_cast<const volatile int*>(smem + O_FLAGS);
      const volatile float* alpha_s = reinterpret_cast<const volatile float*>(smem + O_ALPHA);
      const volatile float* invl_s = reinterpret_cast<const volatile float*>(smem + O_INVL);
      const uint32_t peerStatsFree = mapa_shared(bar(STATSFREE), 0);
      uint32_t sj = 0, nitem = 0, ubase = 0, ncorr = 0;
      bool ok = true;
      for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
        const Item x = decode_item(p, it);
        ++sj;  // the first tile of an item needs no correction (its running max starts there)
        for (int j = 1; j < x.ntiles && !helper; ++j, ++sj, ++ncorr) {
          if (!mbar_wait_cluster_warp(bar(PREADY + (sj & 1) * 2), (sj >> 1) & 1, abort_flag,
                                      kWaitLimitNs, 160)) {
            ok = false;
            break;
          }
          // rarely: rescale O rows before the next P.V accumulates into them
          const volatile int* fl = flags + 4 * (sj & 1);
          const bool any = (fl[0] | fl[1] | fl[2] | fl[3]) != 0;
          if (any) {
            // wait for every P.V of the previous tile
            const uint32_t pj = sj - 1;
            if (!mbar_wait_warp(bar(PVDONE + (pj & 1)), (pj >> 1) & 1, abort_flag, kWaitLimitNs,
                                161)) {
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
          if (lane == 0) mbar_arrive(bar(CORR + (ncorr & 1)));
        }
        if (!ok) break;
        // ---------------------------------------------------------- epilogue
        // 1/l first (the S-CTA reuses its slot once all 12 warps took it),
        // then this warp's value half of O once its last P.V completed
        const int ee = helper ? 1 : 0;
        if (!mbar_wait_cluster_warp(bar(STATSFULL), nitem & 1, abort_flag, kWaitLimitNs, 163)) {
          ok = false;
          break;
        }
        const float il = invl_s[row];
        const float hil = 0.5f * il;
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(peerStatsFree);
        if (!mbar_wait_warp(bar(OFULL + ee), nitem & 1, abort_flag, kWaitLimitNs, 162)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t gbase = ubase + v_uses(x);
        ubase = gbase + 4;
#pragma unroll 1
        for (int e2 = 0; e2 < (helper ? 2 : 1); ++e2) {
          const int e = helper ? 2 + e2 : half;  // g / out stage: value columns [128e, 128e + 128)
          const uint32_t ug = gbase + e;
          const uint32_t st = ug % kVStages;
          if (!mbar_wait_warp(bar(VFULL + st), (ug / kVStages) & 1, abort_flag, kWaitLimitNs, 164)) {
            ok = false;
            break;
          }
          uint8_t* stage = smem + O_VRING + st * kVStage;
          // 32 value columns per step: a 64-column slab of the stage holds
          // steps 2 sl and 2 sl + 1
#pragma unroll 1
          for (int q32 = 0; q32 < 4; ++q32) {
            const int sl = q32 >> 1;
            uint32_t o[32];
            tmem_ld32(tq + 128 * e + 32 * q32, o);
            tmem_wait_ld_dep32(o);
            if (q32 == 3 && e2 == (helper ? 1 : 0)) {  // this warp's part of O read out
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(OFREE + ee));
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
          fence_proxy_async_smem();
          mbar_arrive(bar(STAGED + e));
        }
      }
    }
  }

  __syncwarp();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace prefill2
}  // namespace hca
