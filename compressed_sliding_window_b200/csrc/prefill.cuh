// HCA prefill attention on tcgen05 / TMEM / TMA.
//
// What is computed ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1; xenospectrum
// analysis, section 活性140億パラメータと長文処理を支える仕組み): for each query
// position t and head h, one softmax over the compressed entries j < nc(t) and
// the raw keys max(0, t-127) .. t, then out = sigmoid(g) * (P . V).
//
// Tiling.  A work item is a 128-row tile = 2 consecutive positions x 64 heads
// (one shared KV head, so all 128 rows attend the same keys up to a 1-key
// difference) and one half of the 512-wide value dimension.  Rows are
// contiguous in q/g/out, so every tile is a plain 128 x 512 box.  The keys a
// tile visits come as key tiles of 128: ceil(nc(t0+1)/128) compressed tiles,
// one raw tile [t0-127, t0], and a 16-key tail holding key t0+1 (seen only by
// the second position).
//
// Why the value dimension is split.  A 128-row fp32 accumulator 512 wide fills
// all 512 TMEM columns, leaving none for the scores.  Each item therefore owns
// O[:, 256 half] (256 columns) plus two 128-column score buffers, and the two
// items of a row tile recompute S = Q K^T independently.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = MMA issuer and
// TMEM owner, warps 2-5 = softmax, O correction and epilogue (thread = row).
// The CTA is persistent over a static, longest-first item order.
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace prefill {

constexpr int kRows = 128;          // tile rows: 2 positions x 64 heads
constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kKeyTile = 128;
constexpr int kTail = 16;
constexpr int kStages = 4;
constexpr int kSlab = 16384;        // [128 rows x 64 bf16], 128B-swizzled
constexpr int kQBytes = 8 * kSlab;
constexpr int kPBytes = 2 * kSlab;  // P: 128 rows x 128 keys bf16
constexpr int kSmemQ = 0;
constexpr int kSmemRing = kSmemQ + kQBytes;
constexpr int kSmemP = kSmemRing + kStages * kSlab;
constexpr int kSmemBar = kSmemP + kPBytes;
constexpr int kSmemBytes = kSmemBar + 256;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024
constexpr int kThreads = 192;
constexpr float kTau = 8.0f;                   // lazy-rescale threshold (log2 units)
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// barrier slots (8 bytes each) inside the kSmemBar region
enum {
  B_QFULL = 0, B_QEMPTY = 1, B_FULL = 2, B_EMPTY = B_FULL + kStages,
  B_SFULL = B_EMPTY + kStages, B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2,
  B_PFREE = B_PFULL + 1, B_OFULL = B_PFREE + 1, B_OFREE = B_OFULL + 1, B_DRAIN = B_OFREE + 1,
  B_STAGED = B_DRAIN + 1, B_COUNT = B_STAGED + 1
};
constexpr int kTmemSlot = 8 * B_COUNT;       // byte offset of the TMEM base address
constexpr int kAbortSlot = kTmemSlot + 4;    // byte offset of the abort flag
static_assert(kAbortSlot + 4 <= 256, "barrier region overflow");
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256, kTmemCols = 512;

struct Params {
  int B, T;
  int row_tiles;    // ceil(T / 2) per batch
  int items;        // B * row_tiles * 2
  float scale_log2; // softmax scale * log2(e)
  float* lse;       // [B, T, 64] or null
};

// Number of compressed entries visible to query t: blocks lying wholly before
// its window [t-127, t].
__device__ __forceinline__ int nc_of(int t) { return t >= 127 ? (t - 127) / 128 : 0; }

struct Item {
  int b, t0, half;
  bool has_p1;      // position t0+1 exists
  int nc0, nc1;     // visible entries for positions t0 and t0+1
  int n_ctiles;     // compressed key tiles
  int ntiles;       // all key tiles
};

__device__ __forceinline__ Item decode_item(const Params& p, int it) {
  Item x;
  x.half = it & 1;
  const int r = it >> 1;
  const int rank = r / p.B;
  x.b = r - rank * p.B;
  x.t0 = 2 * (p.row_tiles - 1 - rank);
  x.has_p1 = x.t0 + 1 < p.T;
  x.nc0 = nc_of(x.t0);
  x.nc1 = x.has_p1 ? nc_of(x.t0 + 1) : x.nc0;
  x.n_ctiles = (x.nc1 + kKeyTile - 1) / kKeyTile;
  x.ntiles = x.n_ctiles + 1 + (x.has_p1 ? 1 : 0);
  return x;
}

// kind: 0 = compressed, 1 = raw window, 2 = tail
__device__ __forceinline__ int tile_kind(const Item& x, int j) {
  return j < x.n_ctiles ? 0 : (j == x.n_ctiles ? 1 : 2);
}
// MMA width (keys) of key tile j: a multiple of 16
__device__ __forceinline__ int tile_n(const Item& x, int j) {
  if (j < x.n_ctiles) {
    const int rem = min(kKeyTile, x.nc1 - j * kKeyTile);
    return (rem + 15) & ~15;
  }
  return j == x.n_ctiles ? kKeyTile : kTail;
}

struct Maps {
  CUtensorMap q;    // [B][T*64][512], box 64 x 128
  CUtensorMap g;    // same shape as q
  CUtensorMap out;  // same shape as q
  CUtensorMap k;    // [B][T][512],   box 64 x 128
  CUtensorMap v;
  CUtensorMap k16;  // [B][T][512],   box 64 x 16
  CUtensorMap v16;
  CUtensorMap ck;   // [B][nb][512],  box 64 x 128
  CUtensorMap cv;
};

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kSmemQ, sRing = sbase + kSmemRing, sP = sbase + kSmemP;
  const uint32_t sBar = sbase + kSmemBar;
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemBar + kAbortSlot);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemBar + kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_SFREE + s), 4);
    }
    mbar_init(bar(B_PFULL), 4);
    mbar_init(bar(B_PFREE), 1);
    mbar_init(bar(B_OFULL), 1);
    mbar_init(bar(B_OFREE), 4);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_STAGED), 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    tma_prefetch_desc(&maps.ck);
    tma_prefetch_desc(&maps.cv);
    tma_prefetch_desc(&maps.g);
    tma_prefetch_desc(&maps.out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t ring = 0, quse = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int x, int y, int z, uint32_t bytes) -> bool {
        const uint32_t st = ring % kStages;
        if (!mbar_wait(bar(B_EMPTY + st), ((ring / kStages) & 1) ^ 1, abort_flag, kWaitLimitNs, 10))
          return false;
        mbar_expect_tx(bar(B_FULL + st), bytes);
        tma_load_3d(sRing + st * kSlab, map, bar(B_FULL + st), x, y, z);
        ++ring;
        return true;
      };
      auto load_k = [&](const Item& x, int j) -> bool {
        const int kind = tile_kind(x, j);
        for (int d = 0; d < 8 && ok; ++d) {
          if (kind == 0) ok = load(&maps.ck, 64 * d, j * kKeyTile, x.b, kSlab);
          else if (kind == 1) ok = load(&maps.k, 64 * d, x.t0 - 127, x.b, kSlab);
          else ok = load(&maps.k16, 64 * d, x.t0 + 1, x.b, kTail * 128);
        }
        return ok;
      };
      auto load_v = [&](const Item& x, int j) -> bool {
        const int kind = tile_kind(x, j);
        for (int e = 0; e < 4 && ok; ++e) {
          const int xc = 256 * x.half + 64 * e;
          if (kind == 0) ok = load(&maps.cv, xc, j * kKeyTile, x.b, kSlab);
          else if (kind == 1) ok = load(&maps.v, xc, x.t0 - 127, x.b, kSlab);
          else ok = load(&maps.v16, xc, x.t0 + 1, x.b, kTail * 128);
        }
        return ok;
      };
      for (int it = blockIdx.x; it < p.items && ok; it += gridDim.x) {
        const Item x = decode_item(p, it);
        ok = mbar_wait(bar(B_QEMPTY), (quse & 1) ^ 1, abort_flag, kWaitLimitNs, 11);
        if (!ok) break;
        mbar_expect_tx(bar(B_QFULL), kQBytes);
        for (int d = 0; d < 8; ++d)
          tma_load_3d(sQ + d * kSlab, &maps.q, bar(B_QFULL), 64 * d, x.t0 * kHeads, x.b);
        ++quse;
        if (!load_k(x, 0)) break;
        for (int j = 0; j < x.ntiles && ok; ++j) {
          if (j + 1 < x.ntiles && !load_k(x, j + 1)) break;
          if (!load_v(x, j)) break;
        }
        for (int e = 0; e < 4 && ok; ++e)
          ok = load(&maps.g, 256 * x.half + 64 * e, x.t0 * kHeads, x.b, kSlab);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t ring = 0, quse = 0, sidx = 0, pvidx = 0, nitem = 0;
      bool ok = true;
      const uint32_t idesc_pv = idesc_bf16_f32(kRows, 128, false, true);
      auto issue_s = [&](const Item& x, int j) -> bool {
        const uint32_t buf = sidx & 1;
        if (!mbar_wait(bar(B_SFREE + buf), ((sidx >> 1) & 1) ^ 1, abort_flag, kWaitLimitNs, 20))
          return false;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(kRows, tile_n(x, j), false, false);
        const uint32_t dS = tmem + (buf ? kTmemS1 : kTmemS0);
        for (int d = 0; d < 8; ++d) {
          const uint32_t st = ring % kStages;
          if (!mbar_wait(bar(B_FULL + st), (ring / kStages) & 1, abort_flag, kWaitLimitNs, 21))
            return false;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_sw128(sQ + d * kSlab + 32 * k, 16, 1024);
            const uint64_t bd = sdesc_sw128(sRing + st * kSlab + 32 * k, 16, 1024);
            umma_bf16(dS, ad, bd, idesc, (d | k) != 0);
          }
          umma_commit(bar(B_EMPTY + st));
          ++ring;
        }
        umma_commit(bar(B_SFULL + buf));
        ++sidx;
        return true;
      };
      auto issue_pv = [&](const Item& x, int j) -> bool {
        if (!mbar_wait(bar(B_PFULL), pvidx & 1, abort_flag, kWaitLimitNs, 22)) return false;
        if (j == 0 &&
            !mbar_wait(bar(B_OFREE), (nitem & 1) ^ 1, abort_flag, kWaitLimitNs, 23))
          return false;
        tc_fence_after();
        const int ksteps = tile_n(x, j) / 16;
        for (int pair = 0; pair < 2; ++pair) {
          const uint32_t stA = ring % kStages;
          const uint32_t stB = (ring + 1) % kStages;
          if (!mbar_wait(bar(B_FULL + stA), (ring / kStages) & 1, abort_flag, kWaitLimitNs, 24))
            return false;
          if (!mbar_wait(bar(B_FULL + stB), ((ring + 1) / kStages) & 1, abort_flag, kWaitLimitNs,
                         25))
            return false;
          tc_fence_after();
          const uint32_t dO = tmem + kTmemO + 128 * pair;
          for (int k = 0; k < ksteps; ++k) {
            const uint64_t ad = sdesc_sw128(sP + (k >> 2) * kSlab + 32 * (k & 3), 16, 1024);
            const uint64_t bd = sdesc_sw128(sRing + stA * kSlab + 2048 * k, kSlab, 1024);
            umma_bf16(dO, ad, bd, idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(bar(B_EMPTY + stA));
          umma_commit(bar(B_EMPTY + stB));
          ring += 2;
        }
        umma_commit(bar(B_PFREE));
        ++pvidx;
        return true;
      };
      for (int it = blockIdx.x; it < p.items && ok; it += gridDim.x) {
        const Item x = decode_item(p, it);
        ok = mbar_wait(bar(B_QFULL), quse & 1, abort_flag, kWaitLimitNs, 26);
        if (!ok) break;
        ++quse;
        tc_fence_after();
        if (!issue_s(x, 0)) { ok = false; break; }
        if (x.ntiles == 1) umma_commit(bar(B_QEMPTY));
        for (int j = 0; j < x.ntiles && ok; ++j) {
          if (j + 1 < x.ntiles) {
            if (!issue_s(x, j + 1)) { ok = false; break; }
            if (j + 2 == x.ntiles) umma_commit(bar(B_QEMPTY));
          }
          if (!issue_pv(x, j)) { ok = false; break; }
        }
        if (!ok) break;
        umma_commit(bar(B_OFULL));
        ring += 4;  // the epilogue consumes the 4 g-slab stages of this item
        ++nitem;
      }
      // Make sure no MMA is still writing TMEM before the CTA tears down.
      umma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, abort_flag, kWaitLimitNs, 27);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int wq = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;          // tile row == TMEM lane
    const int pos = row >> 6;                // 0 or 1: which of the two positions
    const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint32_t sidx = 0, pvidx = 0, nitem = 0, ring_base = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < p.items && ok; it += gridDim.x) {
      const Item x = decode_item(p, it);
      const int t = x.t0 + pos;
      const int ncp = pos ? x.nc1 : x.nc0;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < x.ntiles; ++j) {
        const uint32_t buf = sidx & 1;
        if (!mbar_wait_warp(bar(B_SFULL + buf), (sidx >> 1) & 1, abort_flag, kWaitLimitNs, 30)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float sv[kKeyTile];
        {
          uint32_t r[kKeyTile];
#pragma unroll
          for (int c = 0; c < kKeyTile; c += 32) tmem_ld32(tl + (buf ? kTmemS1 : kTmemS0) + c, r + c);
          tmem_wait_ld_dep32(r);
#pragma unroll
          for (int c = 32; c < kKeyTile; c += 32) reg_dep32(r + c);
#pragma unroll
          for (int i = 0; i < kKeyTile; ++i) sv[i] = __uint_as_float(r[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_SFREE + buf));
        ++sidx;

        // visible columns of this key tile for this row: [clo, chi)
        const int kind = tile_kind(x, j);
        int clo = 0, chi = 0;
        if (kind == 0) {
          chi = min(kKeyTile, max(0, ncp - j * kKeyTile));
        } else if (kind == 1) {
          clo = max(127 - x.t0, pos);
          chi = kKeyTile;
        } else {
          chi = pos;  // only key t0+1, only for the second position
        }
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) {
          const float xv = (c >= clo && c < chi) ? sv[c] * p.scale_log2 : -INFINITY;
          sv[c] = xv;
          mt = fmaxf(mt, xv);
        }
        float alpha = 1.f;
        bool resc = false;
        if (mt > m + kTau) {
          resc = (m != -INFINITY);
          alpha = resc ? ex2_approx(m - mt) : 0.f;
          m = mt;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        float rs = 0.f;
        uint32_t pk[kKeyTile / 2];
#pragma unroll
        for (int c = 0; c < kKeyTile; c += 2) {
          const float e0 = ex2_approx(sv[c] - mu);
          const float e1 = ex2_approx(sv[c + 1] - mu);
          rs += e0 + e1;
          pk[c / 2] = pack_bf16x2(e0, e1);
        }
        l = l * alpha + rs;

        // P buffer and O are free once the previous P.V has completed.
        if (!mbar_wait_warp(bar(B_PFREE), (pvidx & 1) ^ 1, abort_flag, kWaitLimitNs, 31)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          uint32_t r[32];
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            tmem_ld32(tl + kTmemO + c, r);
            tmem_wait_ld_dep32(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tl + kTmemO + c, r);
          }
          tmem_wait_st();
        }
        // P row -> swizzled K-major smem (two 64-key slabs)
        uint8_t* prow = smem + kSmemP;
#pragma unroll
        for (int c8 = 0; c8 < kKeyTile / 8; ++c8) {
          const uint32_t off = (c8 >> 3) * kSlab + sw128_offset(row, c8 & 7);
          *reinterpret_cast<uint4*>(prow + off) =
              make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL));
        ++pvidx;
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!mbar_wait_warp(bar(B_OFULL), nitem & 1, abort_flag, kWaitLimitNs, 32)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = 1.f / l;
      const uint32_t g_use = ring_base + 12u * x.ntiles;
      ring_base = g_use + 4;
      for (int e = 0; e < 4; ++e) {
        const uint32_t u = g_use + e;
        const uint32_t st = u % kStages;
        if (!mbar_wait_warp(bar(B_FULL + st), (u / kStages) & 1, abort_flag, kWaitLimitNs, 33)) {
          ok = false;
          break;
        }
        uint32_t o[64];
        tmem_ld32(tl + kTmemO + 64 * e, o);
        tmem_ld32(tl + kTmemO + 64 * e + 32, o + 32);
        tmem_wait_ld_dep32(o);
        reg_dep32(o + 32);
        if (e == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_OFREE));
        }
        uint8_t* stage = smem + kSmemRing + st * kSlab;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(stage + sw128_offset(row, c));
          const uint4 gv = *ptr;
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
          uint32_t ow[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float g0 = bf16lo_to_f32(gw[q]), g1 = bf16hi_to_f32(gw[q]);
            const float s0 = 1.f / (1.f + ex2_approx(-1.4426950408889634f * g0));
            const float s1 = 1.f / (1.f + ex2_approx(-1.4426950408889634f * g1));
            const float o0 = __uint_as_float(o[8 * c + 2 * q]) * inv_l * s0;
            const float o1 = __uint_as_float(o[8 * c + 2 * q + 1]) * inv_l * s1;
            ow[q] = pack_bf16x2(o0, o1);
          }
          *ptr = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_STAGED));
        if (threadIdx.x == 64) {
          // all 128 rows of this slab are staged -> one TMA store, then free the stage
          if (mbar_wait(bar(B_STAGED), (4u * nitem + e) & 1, abort_flag, kWaitLimitNs, 34)) {
            tma_store_3d(&maps.out, sRing + st * kSlab, 256 * x.half + 64 * e, x.t0 * kHeads,
                         x.b);
            bulk_commit();
            bulk_wait_read_all();
            mbar_arrive(bar(B_EMPTY + st));
          }
        }
      }
      if (!ok) break;
      if (p.lse != nullptr && x.half == 0 && t < p.T) {
        const float lse2 = m + __log2f(l);
        p.lse[(static_cast<size_t>(x.b) * p.T + t) * kHeads + (row & 63)] =
            lse2 * 0.6931471805599453f;
      }
      ++nitem;
    }
    if (threadIdx.x == 64) bulk_wait_all();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill
}  // namespace hca
