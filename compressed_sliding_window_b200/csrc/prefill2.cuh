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
//     two 256-column TMEM buffers, the online softmax (thread = row), and P
//     (bf16) shipped to rank 1's shared memory over DSMEM in 128-key sub-tiles
//     together with the per-row rescale factor.
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
// Warp roles (352 threads): warps 0-1 TMA producers, warp 2 MMA issuer and
// TMEM owner, warps 3-10 compute: two warps per TMEM lane quadrant, so a tile
// row is shared by two threads.  On rank 0 each of them owns one 128-key half
// of the score tile (= one P sub-tile; the row max is exchanged through shared
// memory); on rank 1 each owns 256 of the 512 value columns (rescale and
// epilogue).
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace prefill2 {

constexpr int kRows = 128;
constexpr int kHeads = 64;
constexpr int kKT = 256;     // compressed key tile
constexpr int kWinN = 144;   // raw key tile
constexpr int kThreads = 352;
constexpr float kTau = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---- S-CTA shared memory
constexpr int S_Q = 0;                       // 2 halves x [4 slabs][128 rows][64]
constexpr int kQHalf = 65536;
constexpr int S_KRING = 131072;              // 3 stages x [256 keys][64]
constexpr int kKStages = 3;
constexpr int kKStage = 32768;
// ---- O-CTA shared memory
constexpr int O_P = 0;                       // 2 sub-tile buffers x [2 slabs][128 rows][64 keys]
constexpr int kPBuf = 32768;
constexpr int O_VRING = 65536;               // 4 stages x [4 slabs][64 keys][64 dv]
constexpr int kVStages = 4;
constexpr int kVStage = 32768;
constexpr int O_ALPHA = O_VRING + kVStages * kVStage;  // [128] float
constexpr int O_FLAGS = O_ALPHA + 512;                  // [4] int
constexpr int O_INVL = O_FLAGS + 64;                    // [128] float

// ---- barriers (both CTAs, same offsets)
constexpr int BAR = 229376;
enum {
  QFULL = 0, QEMPTY = 2, KFULL = 4, KEMPTY = KFULL + kKStages, SFULL = KEMPTY + kKStages,
  SFREE = SFULL + 2, PFREE = SFREE + 2, STATSFREE = PFREE + 2,
  VFULL = STATSFREE + 1, VEMPTY = VFULL + kVStages, PFULL = VEMPTY + kVStages, CORR = PFULL + 2,
  PVDONE = CORR + 1, OFULL = PVDONE + 1, OFREE = OFULL + 1, STATSFULL = OFREE + 1,
  STAGED = STATSFULL + 1, DRAIN = STAGED + 2, XMAX = DRAIN + 1, NBAR = XMAX + 4
};
constexpr int kTmemSlot = BAR + 8 * NBAR;
constexpr int kAbortSlot = kTmemSlot + 4;
// S-CTA: per-row statistics exchanged between the two warps of a row
// ([2 parity][2 halves][128] float)
constexpr int S_XMAX = BAR + 512;
constexpr int kSmemBytes = S_XMAX + 2048;
// The dynamic shared memory base is 1024-aligned (checked at run time), so no
// alignment slack is allocated: the S-CTA needs every byte.
constexpr int kSmemAlloc = kSmemBytes;
static_assert(kAbortSlot + 4 <= kSmemBytes, "barrier region overflow");
static_assert(O_INVL + 512 <= BAR, "O-CTA layout overflow");
static_assert(S_KRING + kKStages * kKStage <= BAR, "S-CTA layout overflow");
static_assert(kSmemAlloc <= 232448, "shared memory budget");

struct Params {
  int B, T;
  int row_tiles;    // ceil(T / 2)
  int items;        // B * row_tiles
  float scale_log2; // softmax scale * log2(e)
  float* lse;       // [B, T, 64] or null
};

struct Maps {
  CUtensorMap q4;    // (64, T*64, 8, B)  box (64, 128, 4, 1): one Q half
  CUtensorMap ck;    // [B][nb][512]      box (64, 256, 1)
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
    mbar_init(bar(STATSFREE), 8);
    mbar_init(bar(PFULL + 0), 4);
    mbar_init(bar(PFULL + 1), 4);
    mbar_init(bar(CORR), 8);
    mbar_init(bar(OFREE), 8);
    mbar_init(bar(STATSFULL), 4);
    mbar_init(bar(STAGED + 0), 128);
    mbar_init(bar(STAGED + 1), 128);
    for (int q = 0; q < 4; ++q) mbar_init(bar(XMAX + q), 2);
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
            for (int d = 0; d < 8; ++d, ++u) {
              if ((u & 1) != static_cast<uint32_t>(me)) continue;
              const uint32_t st = u % kKStages;
              ok = mbar_wait(bar(KEMPTY + st), ((u / kKStages) & 1) ^ 1, abort_flag, kWaitLimitNs,
                             111);
              if (!ok) break;
              const uint32_t dst = sb + S_KRING + st * kKStage;
              if (comp) {
                mbar_expect_tx(bar(KFULL + st), kKT * 128);
                tma_load_3d(dst, &maps.ck, bar(KFULL + st), 64 * d, j * kKT, x.b);
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
            const uint32_t buf = sj & 1;
            ok = mbar_wait(bar(SFREE + buf), ((sj >> 1) & 1) ^ 1, abort_flag, kWaitLimitNs, 120);
            if (!ok) break;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(kRows, tile_n(x, j), false, false);
            const uint32_t dS = tmem + 256 * buf;
            for (int d = 0; d < 8 && ok; ++d, ++u) {
              if (j == 0 && (d & 3) == 0) {
                ok = mbar_wait(bar(QFULL + (d >> 2)), nitem & 1, abort_flag, kWaitLimitNs, 121);
                if (!ok) break;
              }
              const uint32_t st = u % kKStages;
              ok = mbar_wait(bar(KFULL + st), (u / kKStages) & 1, abort_flag, kWaitLimitNs, 122);
              if (!ok) break;
              tc_fence_after();
              const uint32_t qa = sb + S_Q + (d >> 2) * kQHalf + (d & 3) * 16384;
              const uint32_t ka = sb + S_KRING + st * kKStage;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_bf16(dS, sdesc_sw128(qa + 32 * k, 16, 1024), sdesc_sw128(ka + 32 * k, 16, 1024),
                          idesc, (d | k) != 0);
              umma_commit(bar(KEMPTY + st));
              if (j + 1 == x.ntiles && (d & 3) == 3) umma_commit(bar(QEMPTY + (d >> 2)));
            }
            if (!ok) break;
            umma_commit(bar(SFULL + buf));
          }
        }
        umma_commit(bar(DRAIN));
        mbar_wait(bar(DRAIN), 0, abort_flag, kWaitLimitNs, 123);
      }
    } else {
      // --------------------------------------------------------- softmax
      const int wq = warp & 3;
      const int half = (warp - 3) >> 2;       // key columns [128 half, 128 half + 128)
      const int row = wq * 32 + lane;
      const int pos = row >> 6;
      const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      float* xmax = reinterpret_cast<float*>(smem + S_XMAX);
      const uint32_t peerP = mapa_shared(sb + O_P + half * kPBuf, 1);
      const uint32_t peerAlpha = mapa_shared(sb + O_ALPHA, 1);
      const uint32_t peerFlags = mapa_shared(sb + O_FLAGS, 1);
      const uint32_t peerInvl = mapa_shared(sb + O_INVL, 1);
      const uint32_t peerPFull = mapa_shared(bar(PFULL + half), 1);
      const uint32_t peerStatsFull = mapa_shared(bar(STATSFULL), 1);
      uint32_t sj = 0, nitem = 0, nx = 0;
      bool ok = true;
      for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
        const Item x = decode_item(p, it);
        const int t = x.t0 + pos;
        const int ncp = pos ? x.nc1 : x.nc0;
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < x.ntiles; ++j, ++sj) {
          const uint32_t buf = sj & 1;
          if (!mbar_wait_warp(bar(SFULL + buf), (sj >> 1) & 1, abort_flag, kWaitLimitNs, 130)) {
            ok = false;
            break;
          }
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
          const bool full = (clo <= c0) && (chi >= c0 + 128);
          const uint32_t sbase = tl + 256 * buf + c0;
          // pass A: this half's row max of the raw scores
          float mraw = -INFINITY;
          for (int cc = 0; cc < nh; cc += 64) {
            uint32_t r[64];
            tmem_ld32(sbase + cc, r);
            tmem_ld32(sbase + cc + 32, r + 32);
            tmem_wait_ld_dep32(r);
            reg_dep32(r + 32);
            if (full) {
#pragma unroll
              for (int c = 0; c < 64; ++c) mraw = fmaxf(mraw, __uint_as_float(r[c]));
            } else {
#pragma unroll
              for (int c = 0; c < 64; ++c) {
                const int col = c0 + cc + c;
                if (col >= clo && col < chi) mraw = fmaxf(mraw, __uint_as_float(r[c]));
              }
            }
          }
          // exchange with the warp that holds the other half of the row
          const uint32_t xp = nx & 1;
          xmax[(xp * 2 + half) * 128 + row] = mraw;
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(XMAX + wq));
          if (!mbar_wait_warp(bar(XMAX + wq), nx & 1, abort_flag, kWaitLimitNs, 133)) {
            ok = false;
            break;
          }
          mraw = fmaxf(mraw, xmax[(xp * 2 + (half ^ 1)) * 128 + row]);
          ++nx;
          const float mt = mraw * p.scale_log2;  // scale > 0
          float alpha = 1.f;
          bool resc = false;
          if (mt > m + kTau) {
            resc = (m != -INFINITY);
            alpha = resc ? ex2_approx(m - mt) : 0.f;
            m = mt;
          }
          const float mu = (m == -INFINITY) ? 0.f : m;
          // the O-CTA has finished reading this half's P buffer (previous tile)
          if (!mbar_wait_cluster_warp(bar(PFREE + half), (sj & 1) ^ 1, abort_flag, kWaitLimitNs,
                                      131)) {
            ok = false;
            break;
          }
          // pass B: probabilities, written straight into the O-CTA's P buffer
          float rs = 0.f;
          for (int cc = 0; cc < nh; cc += 64) {
            uint32_t r[64];
            tmem_ld32(sbase + cc, r);
            tmem_ld32(sbase + cc + 32, r + 32);
            tmem_wait_ld_dep32(r);
            reg_dep32(r + 32);
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const int col = c0 + cc + c;
              float e0 = ex2_approx(fmaf(__uint_as_float(r[c]), p.scale_log2, -mu));
              float e1 = ex2_approx(fmaf(__uint_as_float(r[c + 1]), p.scale_log2, -mu));
              if (!full) {
                e0 = (col >= clo && col < chi) ? e0 : 0.f;
                e1 = (col + 1 >= clo && col + 1 < chi) ? e1 : 0.f;
              }
              rs += e0 + e1;
              pk[c / 2] = pack_bf16x2(e0, e1);
            }
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
              const int k8 = (cc >> 3) + c8;   // 8-key chunk index within the sub-tile
              const uint32_t off = (k8 >> 3) * 16384 + sw128_offset(row, k8 & 7);
              st_cluster_v4(peerP + off, pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2],
                            pk[4 * c8 + 3]);
            }
          }
          if (half == 0) {
            st_cluster_b32(peerAlpha + 4 * row, __float_as_uint(alpha));
            const int any = __any_sync(0xffffffffu, resc) ? 1 : 0;
            if (lane == 0) st_cluster_b32(peerFlags + 4 * wq, static_cast<uint32_t>(any));
          }
          fence_proxy_async_all();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster(peerPFull);
            mbar_arrive(bar(SFREE + buf));
          }
          l = l * alpha + rs;
        }
        if (!ok) break;
        // row sum = both halves (one more round of the same exchange); 1/l to
        // the O-CTA epilogue, lse to the caller
        {
          const uint32_t xp = nx & 1;
          xmax[(xp * 2 + half) * 128 + row] = l;
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(XMAX + wq));
          if (!mbar_wait_warp(bar(XMAX + wq), nx & 1, abort_flag, kWaitLimitNs, 134)) {
            ok = false;
            break;
          }
          l += xmax[(xp * 2 + (half ^ 1)) * 128 + row];
          ++nx;
        }
        if (half == 0) {
          if (!mbar_wait_cluster_warp(bar(STATSFREE), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs,
                                      132)) {
            ok = false;
            break;
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
          for (int j = 0; j < x.ntiles && ok; ++j) {
            const int n = tile_n(x, j);
            const bool comp = j < x.n_ctiles;
            for (int h = 0; h < 2 && ok; ++h) {
              const int nh = sub_n(n, h);
              for (int kc = 0; kc * 64 < nh && ok; ++kc) {
                for (int dh = 0; dh < 2 && ok; ++dh) {
                  if (comp) ok = stage_load(&maps.cv4, j * kKT + 128 * h + 64 * kc, 4 * dh, x.b);
                  else ok = stage_load(&maps.v4, x.t0 - 127 + 128 * h + 64 * kc, 4 * dh, x.b);
                }
              }
            }
          }
          for (int e = 0; e < 4 && ok; ++e) ok = stage_load(&maps.g4, x.t0 * kHeads, 2 * e, x.b);
        }
      }
    } else if (warp == 2) {
      // --------------------------------------------------------- MMA (O += P V)
      if (lane == 0) {
        uint32_t u = 0, sj = 0, nitem = 0;
        bool ok = true;
        const uint32_t idesc = idesc_bf16_f32(kRows, 256, false, true);
        for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
          const Item x = decode_item(p, it);
          for (int j = 0; j < x.ntiles && ok; ++j, ++sj) {
            const int n = tile_n(x, j);
            for (int h = 0; h < 2 && ok; ++h) {
              const int nh = sub_n(n, h);
              ok = mbar_wait_cluster(bar(PFULL + h), sj & 1, abort_flag, kWaitLimitNs, 150);
              if (!ok) break;
              if (h == 0) {
                ok = mbar_wait(bar(CORR), sj & 1, abort_flag, kWaitLimitNs, 151);
                if (!ok) break;
                if (j == 0) {
                  ok = mbar_wait(bar(OFREE), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs, 152);
                  if (!ok) break;
                }
              }
              tc_fence_after();
              const uint32_t pa = sb + O_P + h * kPBuf;
              for (int kc = 0; kc * 64 < nh && ok; ++kc) {
                const int ksteps = min(4, (nh - 64 * kc) >> 4);
                for (int dh = 0; dh < 2; ++dh, ++u) {
                  const uint32_t st = u % kVStages;
                  ok = mbar_wait(bar(VFULL + st), (u / kVStages) & 1, abort_flag, kWaitLimitNs, 153);
                  if (!ok) break;
                  tc_fence_after();
                  const uint32_t va = sb + O_VRING + st * kVStage;
                  for (int ks = 0; ks < ksteps; ++ks) {
                    const bool first = (j == 0 && h == 0 && kc == 0 && ks == 0);
                    umma_bf16(tmem + 256 * dh, sdesc_sw128(pa + kc * 16384 + 32 * ks, 16, 1024),
                              sdesc_sw128(va + 2048 * ks, 8192, 1024), idesc, first ? 0u : 1u);
                  }
                  umma_commit(bar(VEMPTY + st));
                }
              }
              if (!ok) break;
              umma_commit(bar(PVDONE));
              umma_commit_mc(bar(PFREE + h), 0x1);  // sub-tile buffer h is free again (rank 0)
            }
          }
          if (!ok) break;
          umma_commit(bar(OFULL));
          u += 4;  // g stages, consumed by the epilogue
        }
        umma_commit(bar(DRAIN));
        mbar_wait(bar(DRAIN), 0, abort_flag, kWaitLimitNs, 154);
      }
    } else {
      // --------------------------------------------------------- correction + epilogue
      const int wq = warp & 3;
      const int half = (warp - 3) >> 2;       // value columns [256 half, 256 half + 256)
      const int row = wq * 32 + lane;
      const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16) + 256 * half;
      const volatile int* flags = reinterpret_cast<const volatile int*>(smem + O_FLAGS);
      const volatile float* alpha_s = reinterpret_cast<const volatile float*>(smem + O_ALPHA);
      const volatile float* invl_s = reinterpret_cast<const volatile float*>(smem + O_INVL);
      const uint32_t peerStatsFree = mapa_shared(bar(STATSFREE), 0);
      uint32_t sj = 0, nitem = 0, pv = 0, ubase = 0;
      bool ok = true;
      for (int it = pair; it < p.items && ok; it += npairs, ++nitem) {
        const Item x = decode_item(p, it);
        uint32_t vstages = 0;
        for (int j = 0; j < x.ntiles; ++j, ++sj) {
          const int n = tile_n(x, j);
          vstages += 2 * ((sub_n(n, 0) + 63) / 64) + 2 * ((sub_n(n, 1) + 63) / 64);
          if (!mbar_wait_cluster_warp(bar(PFULL), sj & 1, abort_flag, kWaitLimitNs, 160)) {
            ok = false;
            break;
          }
          // rarely: rescale O rows before the next P.V accumulates into them
          const bool any = (flags[0] | flags[1] | flags[2] | flags[3]) != 0;
          if (any) {
            // wait for every P.V issued so far (the last one is sub-tile 1 of tile j-1)
            if (!mbar_wait_warp(bar(PVDONE), (pv + 1) & 1, abort_flag, kWaitLimitNs, 161)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float a = alpha_s[row];
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
          if (lane == 0) mbar_arrive(bar(CORR));
          pv += 2;  // P.V of both sub-tiles of this tile will be committed to PVDONE
        }
        if (!ok) break;
        // ---------------------------------------------------------- epilogue
        if (!mbar_wait_warp(bar(OFULL), nitem & 1, abort_flag, kWaitLimitNs, 162) ||
            !mbar_wait_cluster_warp(bar(STATSFULL), nitem & 1, abort_flag, kWaitLimitNs, 163)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float il = invl_s[row];
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(peerStatsFree);
        const uint32_t gbase = ubase + vstages;
        ubase = gbase + 4;
        for (int ee = 0; ee < 2; ++ee) {
          const int e = 2 * half + ee;          // g / out stage: value columns [128e, 128e + 128)
          const uint32_t ug = gbase + e;
          const uint32_t st = ug % kVStages;
          if (!mbar_wait_warp(bar(VFULL + st), (ug / kVStages) & 1, abort_flag, kWaitLimitNs, 164)) {
            ok = false;
            break;
          }
          uint8_t* stage = smem + O_VRING + st * kVStage;
#pragma unroll 1
          for (int sl = 0; sl < 2; ++sl) {
            uint32_t o[64];
            tmem_ld32(tl + 128 * ee + 64 * sl, o);
            tmem_ld32(tl + 128 * ee + 64 * sl + 32, o + 32);
            tmem_wait_ld_dep32(o);
            reg_dep32(o + 32);
            if (ee == 1 && sl == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(OFREE));
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4* ptr = reinterpret_cast<uint4*>(stage + sl * 16384 + sw128_offset(row, c));
              const uint4 gv = *ptr;
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
              uint32_t ow[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int oc = 8 * c + 2 * q;
                ow[q] = pack_bf16x2(__uint_as_float(o[oc]) * il * sigmoid_fast(bf16lo_to_f32(gw[q])),
                                    __uint_as_float(o[oc + 1]) * il *
                                        sigmoid_fast(bf16hi_to_f32(gw[q])));
              }
              *ptr = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(bar(STAGED + half));
          if (warp == 3 + 4 * half && lane == 0) {
            if (mbar_wait(bar(STAGED + half), (2u * nitem + ee) & 1, abort_flag, kWaitLimitNs,
                          165)) {
              tma_store_4d(&maps.out4, sb + O_VRING + st * kVStage, 0, x.t0 * kHeads, 2 * e, x.b);
              bulk_commit();
              bulk_wait_read_all();
              mbar_arrive(bar(VEMPTY + st));
            }
          }
        }
      }
      if (lane == 0 && (warp == 3 || warp == 7)) bulk_wait_all();
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
