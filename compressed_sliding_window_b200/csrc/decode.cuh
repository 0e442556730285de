// HCA decode: one new query token per sequence, split-KV over all SMs, then a
// log-sum-exp combine.
//
// What is computed ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1; xenospectrum
// analysis, section 活性140億パラメータと長文処理を支える仕組み): for sequence
// i with context length L (new token included, query at t = L-1) and head h,
// one softmax over the compressed entries j < nc(L-1) = max(0, floor((L-128)/128))
// and the min(L, 128) newest raw tokens, then out = sigmoid(g) * (P . V).
//
// Work split.  Every sequence is cut into key tiles of 128 (ceil(nc/128)
// compressed tiles + one window tile).  The tiles of all sequences are laid
// end to end and CTA c takes the contiguous range [floor(cN/G), floor((c+1)N/G)),
// so every SM streams the same number of cache bytes whatever the length mix.
// A CTA writes one partial (unnormalised O, running max m, running sum l) per
// sequence it touches, into slot c + i of the workspace (slots never collide:
// a CTA's sequences are consecutive and later CTAs start at later sequences).
//
// Tensor-core mapping (swap-AB).  With 64 heads a plain S = Q K^T would use
// M = 64; instead keys go on the 128-lane M axis:
//   S^T[key, head] = K_tile[key, :] . Q[head, :]        (M=128, N=64, K=512)
//   O^T[dv, head] += V_tile[:, dv]^T . P^T[:, head]      (4 x M=128 dv, N=64, K=128)
// TMEM holds O^T (4 x 64 columns) and two 64-column S^T buffers.  The softmax
// runs across lanes: each thread owns one key and its 64 head scores, and the
// per-head max / sum over the 128 keys come from a shuffle transpose-reduce
// (62 shuffles per warp) plus one small shared-memory step.
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace decode {

constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kKeyTile = 128;
constexpr int kWin = 128;
constexpr int kStages = 4;
constexpr int kSlab = 16384;        // [128 keys x 64 bf16] swizzled
constexpr int kStage = 2 * kSlab;   // one copy: two 64-wide slabs of a 128-key tile
constexpr int kQSlab = 8192;        // [64 heads x 64 bf16] swizzled
constexpr int kSmemQ = 0;           // 8 x 8 KB
constexpr int kSmemRing = 65536;    // 4 x 32 KB
constexpr int kSmemPT = kSmemRing + kStages * kStage;  // P^T [128 keys x 64 heads] bf16, 16 KB
constexpr int kSmemRed = kSmemPT + 16384;             // reductions, 4 KB
constexpr int kSmemBar = kSmemRed + 4096;
constexpr int kSmemBytes = kSmemBar + 256;
constexpr int kSmemAlloc = kSmemBytes + 1024;
constexpr int kThreads = 224;
constexpr float kTau = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kMaxSeqs = 8192;      // prefix sums kept in shared memory? no: global scan, see below
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// reduction area layout (floats)
constexpr int R_MAX = 0;            // [4][64]
constexpr int R_SUM = 256;          // [4][64]
constexpr int R_MUSE = 512;         // [64]  m used for this tile
constexpr int R_ALPHA = 576;        // [64]
constexpr int R_MRUN = 640;         // [64]
constexpr int R_LRUN = 704;         // [64]
constexpr int R_FLAG = 768;         // ints: [0] ok, [1] any-rescale

enum {
  B_QFULL = 0, B_QEMPTY = 1, B_FULL = 2, B_EMPTY = B_FULL + kStages, B_SFULL = B_EMPTY + kStages,
  B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2, B_PFREE = B_PFULL + 1, B_OFULL = B_PFREE + 1,
  B_OFREE = B_OFULL + 1, B_DRAIN = B_OFREE + 1, B_COUNT = B_DRAIN + 1
};
constexpr int kTmemSlot = 8 * B_COUNT;
constexpr int kAbortSlot = kTmemSlot + 4;
static_assert(kAbortSlot + 4 <= 256, "barrier region overflow");

constexpr uint32_t kTmemO = 0, kTmemS0 = 256, kTmemS1 = 320, kTmemCols = 512;

// Workspace layout (bytes): [slots][64][512] fp32 partial O, then [slots][2][64] fp32 (m, l)
// in log2 units.  slots = grid + S.
__host__ __device__ inline size_t ws_o_bytes(int slots) {
  return static_cast<size_t>(slots) * kHeads * kDim * 4;
}
__host__ __device__ inline size_t ws_bytes(int slots) {
  return ws_o_bytes(slots) + static_cast<size_t>(slots) * 2 * kHeads * 4;
}

struct Params {
  const int* ctx_len;  // [S] device
  int S;
  int max_nc;
  float scale_log2;
  float* ws_o;         // [slots][64][512]
  float* ws_ml;        // [slots][2][64]
  long long* seq_tile; // [S + 1] exclusive prefix of tile counts (computed by plan kernel)
};

__device__ __forceinline__ int nc_of_len(int L) { return L >= 128 ? (L - 128) / 128 : 0; }

// ---------------------------------------------------------------------------
// Plan: tile counts per sequence and their exclusive prefix (one CTA).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(const int* __restrict__ ctx_len, int S,
                                                    int max_nc, long long* __restrict__ seq_tile) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ long long carry;
  __shared__ long long wsum[32];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < S; base += blockDim.x) {
    const int i = base + threadIdx.x;
    long long n = 0;
    if (i < S) {
      int L = ctx_len[i];
      int nc = nc_of_len(L);
      if (L < 1 || nc > max_nc) record_error(DEVERR_BAD_INPUT, 100);
      nc = min(max(nc, 0), max_nc);
      n = (nc + kKeyTile - 1) / kKeyTile + 1;
    }
    // block-wide inclusive scan
    long long x = n;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {
      long long s = (lane < static_cast<int>(blockDim.x >> 5)) ? wsum[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;
    }
    __syncthreads();
    const long long incl = x + (w > 0 ? wsum[w - 1] : 0) + carry;
    if (i < S) seq_tile[i] = incl - n;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) seq_tile[S] = carry;
}

struct SeqInfo {
  int L, nc, nct;   // context length, visible entries, compressed tiles
};

__device__ __forceinline__ SeqInfo seq_info(const Params& p, int s) {
  SeqInfo r;
  r.L = max(1, p.ctx_len[s]);
  r.nc = min(max(nc_of_len(r.L), 0), p.max_nc);
  r.nct = (r.nc + kKeyTile - 1) / kKeyTile;
  return r;
}

// first sequence whose tile range contains global tile x (binary search)
__device__ __forceinline__ int find_seq(const long long* seq_tile, int S, long long x) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_tile[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// 4-D views (64, rows, 8 slabs, S) of [S][rows][512] tensors: a box
// (64, rows, n, 1) lands as n 64-wide slabs of [rows][64], 128B-swizzled.
struct Maps {
  CUtensorMap q;    // (64, S*64, 8, 1),  box (64, 64, 8, 1): the whole q of one sequence
  CUtensorMap ck;   // (64, max_nc, 8, S), box (64, 128, 2, 1)
  CUtensorMap cv;
  CUtensorMap wk;   // (64, 128, 8, S),   box (64, 128, 2, 1)
  CUtensorMap wv;
};

__device__ __forceinline__ void tma_load_4d_dec(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}

// Transpose-reduce of 64 per-lane values across the 32 lanes of a warp: on
// return a[0], a[1] hold the reduction over all lanes for heads 2*lane and
// 2*lane+1.
template <bool kMax>
__device__ __forceinline__ void warp_transpose_reduce64(float* a) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16, n = 64; o >= 1; o >>= 1, n >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = up ? a[i] : a[i + n / 2];
      const float keep = up ? a[i + n / 2] : a[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, o);
      a[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kSmemQ, sRing = sbase + kSmemRing, sPT = sbase + kSmemPT;
  const uint32_t sBar = sbase + kSmemBar;
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemBar + kAbortSlot);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemBar + kTmemSlot);
  float* red = reinterpret_cast<float*>(smem + kSmemRed);
  volatile int* flags = reinterpret_cast<volatile int*>(red + R_FLAG);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The plan kernel may still be running (programmatic dependent launch):
  // wait for its results, then let the combine kernel launch early.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long N = p.seq_tile[p.S];
  const long long A0 = N * blockIdx.x / gridDim.x;
  const long long A1 = N * (blockIdx.x + 1) / gridDim.x;
  if (A0 >= A1) return;  // uniform across the CTA: nothing allocated yet

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_SFREE + s), 1);
    }
    mbar_init(bar(B_PFULL), 1);
    mbar_init(bar(B_PFREE), 1);
    mbar_init(bar(B_OFULL), 1);
    mbar_init(bar(B_OFREE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.ck);
    tma_prefetch_desc(&maps.cv);
    tma_prefetch_desc(&maps.wk);
    tma_prefetch_desc(&maps.wv);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Segments: maximal runs of this CTA's tiles inside one sequence.
  const int s_first = find_seq(p.seq_tile, p.S, A0);

  if (warp <= 1) {
    // ------------------------------------------------------------ producers
    // Two warps alternate ring stages: one issuing thread cannot keep enough
    // copies in flight to cover HBM latency.
    if (lane == 0) {
      const int me = warp;
      uint32_t u = 0, quse = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int y, int z, int w) -> bool {
        if ((u & 1) == static_cast<uint32_t>(me)) {
          const uint32_t st = u % kStages;
          if (!mbar_wait(bar(B_EMPTY + st), ((u / kStages) & 1) ^ 1, abort_flag, kWaitLimitNs, 40))
            return false;
          mbar_expect_tx(bar(B_FULL + st), kStage);
          tma_load_4d_dec(sRing + st * kStage, map, bar(B_FULL + st), 0, y, z, w);
        }
        ++u;
        return true;
      };
      long long x = A0;
      for (int s = s_first; x < A1 && ok; ++s) {
        const SeqInfo si = seq_info(p, s);
        const long long seg_end = min(A1, p.seq_tile[s + 1]);
        const int j0 = static_cast<int>(x - p.seq_tile[s]);
        const int j1 = static_cast<int>(seg_end - p.seq_tile[s]);
        if (me == 0) {
          ok = mbar_wait(bar(B_QEMPTY), (quse & 1) ^ 1, abort_flag, kWaitLimitNs, 41);
          if (!ok) break;
          mbar_expect_tx(bar(B_QFULL), 8 * kQSlab);
          tma_load_4d_dec(sQ, &maps.q, bar(B_QFULL), 0, s * kHeads, 0, 0);
        }
        ++quse;
        auto load_k = [&](int j) -> bool {
          for (int d = 0; d < 4 && ok; ++d)
            ok = (j < si.nct) ? load(&maps.ck, j * kKeyTile, 2 * d, s) : load(&maps.wk, 0, 2 * d, s);
          return ok;
        };
        auto load_v = [&](int j) -> bool {
          for (int e = 0; e < 4 && ok; ++e)
            ok = (j < si.nct) ? load(&maps.cv, j * kKeyTile, 2 * e, s) : load(&maps.wv, 0, 2 * e, s);
          return ok;
        };
        if (!load_k(j0)) break;
        for (int j = j0; j < j1 && ok; ++j) {
          if (j + 1 < j1 && !load_k(j + 1)) break;
          if (!load_v(j)) break;
        }
        x = seg_end;
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t ring = 0, quse = 0, sidx = 0, pvidx = 0, nseg = 0;
      bool ok = true;
      const uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64, true, true);
      auto issue_s = [&]() -> bool {
        const uint32_t buf = sidx & 1;
        if (!mbar_wait(bar(B_SFREE + buf), ((sidx >> 1) & 1) ^ 1, abort_flag, kWaitLimitNs, 50))
          return false;
        tc_fence_after();
        const uint32_t dS = tmem + (buf ? kTmemS1 : kTmemS0);
        for (int d2 = 0; d2 < 4; ++d2) {
          const uint32_t st = ring % kStages;
          if (!mbar_wait(bar(B_FULL + st), (ring / kStages) & 1, abort_flag, kWaitLimitNs, 51))
            return false;
          tc_fence_after();
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            const int d = 2 * d2 + sl;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = sdesc_sw128(sRing + st * kStage + sl * kSlab + 32 * k, 16, 1024);
              const uint64_t bd = sdesc_sw128(sQ + d * kQSlab + 32 * k, 16, 1024);
              umma_bf16(dS, ad, bd, idesc_s, (d | k) != 0);
            }
          }
          umma_commit(bar(B_EMPTY + st));
          ++ring;
        }
        umma_commit(bar(B_SFULL + buf));
        ++sidx;
        return true;
      };
      auto issue_pv = [&](bool first) -> bool {
        if (!mbar_wait(bar(B_PFULL), pvidx & 1, abort_flag, kWaitLimitNs, 52)) return false;
        if (first && !mbar_wait(bar(B_OFREE), (nseg & 1) ^ 1, abort_flag, kWaitLimitNs, 53))
          return false;
        tc_fence_after();
        for (int c = 0; c < 4; ++c) {
          const uint32_t st = ring % kStages;
          if (!mbar_wait(bar(B_FULL + st), (ring / kStages) & 1, abort_flag, kWaitLimitNs, 54))
            return false;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t ad = sdesc_sw128(sRing + st * kStage + 2048 * k, kSlab, 1024);
            const uint64_t bd = sdesc_sw128(sPT + 2048 * k, kSlab, 1024);
            umma_bf16(tmem + kTmemO + 64 * c, ad, bd, idesc_o, (!first || k > 0) ? 1u : 0u);
          }
          umma_commit(bar(B_EMPTY + st));
          ++ring;
        }
        umma_commit(bar(B_PFREE));
        ++pvidx;
        return true;
      };
      long long x = A0;
      for (int s = s_first; x < A1 && ok; ++s) {
        const long long seg_end = min(A1, p.seq_tile[s + 1]);
        const int ntl = static_cast<int>(seg_end - x);
        ok = mbar_wait(bar(B_QFULL), quse & 1, abort_flag, kWaitLimitNs, 56);
        if (!ok) break;
        ++quse;
        tc_fence_after();
        if (!issue_s()) { ok = false; break; }
        if (ntl == 1) umma_commit(bar(B_QEMPTY));
        for (int j = 0; j < ntl && ok; ++j) {
          if (j + 1 < ntl) {
            if (!issue_s()) { ok = false; break; }
            if (j + 2 == ntl) umma_commit(bar(B_QEMPTY));
          }
          if (!issue_pv(j == 0)) { ok = false; break; }
        }
        if (!ok) break;
        umma_commit(bar(B_OFULL));
        ++nseg;
        x = seg_end;
      }
      umma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, abort_flag, kWaitLimitNs, 57);
    }
  } else {
    // ------------------------------------------------------------ softmax / partial epilogue
    const int tid = threadIdx.x - 96;        // 0..127
    const int wq = warp & 3;
    const int gw = warp - 3;                 // 0..3 within the group
    const int key = wq * 32 + lane;          // TMEM lane == key row of S^T / dv row of O^T
    const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint32_t sidx = 0, pvidx = 0, nseg = 0;
    // leader-waits-then-broadcasts keeps the 128 threads in lockstep
    auto group_wait = [&](uint32_t b, uint32_t parity, unsigned where) -> bool {
      if (tid == 0) flags[0] = mbar_wait(b, parity, abort_flag, kWaitLimitNs, where) ? 1 : 0;
      named_bar_sync(1, 128);
      const bool ok = flags[0] != 0;
      named_bar_sync(1, 128);
      return ok;
    };
    bool ok = true;
    long long x = A0;
    for (int s = s_first; x < A1 && ok; ++s) {
      const SeqInfo si = seq_info(p, s);
      const long long seg_end = min(A1, p.seq_tile[s + 1]);
      const int j0 = static_cast<int>(x - p.seq_tile[s]);
      const int j1 = static_cast<int>(seg_end - p.seq_tile[s]);
      if (tid < 64) {
        red[R_MRUN + tid] = -INFINITY;
        red[R_LRUN + tid] = 0.f;
      }
      for (int j = j0; j < j1; ++j) {
        const uint32_t buf = sidx & 1;
        if (!group_wait(bar(B_SFULL + buf), (sidx >> 1) & 1, 60)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[64];
        tmem_ld32(tl + (buf ? kTmemS1 : kTmemS0), r);
        tmem_ld32(tl + (buf ? kTmemS1 : kTmemS0) + 32, r + 32);
        tmem_wait_ld_dep32(r);
        reg_dep32(r + 32);
        tc_fence_before();
        named_bar_sync(1, 128);
        if (tid == 0) mbar_arrive(bar(B_SFREE + buf));
        ++sidx;

        // validity of this thread's key
        bool valid;
        if (j < si.nct) valid = j * kKeyTile + key < si.nc;
        else valid = (si.L >= kWin) || (key < si.L);
        float a[64];
#pragma unroll
        for (int h = 0; h < 64; ++h) a[h] = valid ? __uint_as_float(r[h]) * p.scale_log2 : -INFINITY;
        float xv[64];
#pragma unroll
        for (int h = 0; h < 64; ++h) xv[h] = a[h];
        warp_transpose_reduce64<true>(a);
        red[R_MAX + gw * 64 + 2 * lane] = a[0];
        red[R_MAX + gw * 64 + 2 * lane + 1] = a[1];
        named_bar_sync(1, 128);
        if (tid < 64) {
          const float tm = fmaxf(fmaxf(red[R_MAX + tid], red[R_MAX + 64 + tid]),
                                 fmaxf(red[R_MAX + 128 + tid], red[R_MAX + 192 + tid]));
          const float m = red[R_MRUN + tid];
          float alpha = 1.f;
          int resc = 0;
          float mnew = m;
          if (tm > m + kTau) {
            resc = (m != -INFINITY);
            alpha = resc ? ex2_approx(m - tm) : 0.f;
            mnew = tm;
          }
          red[R_MRUN + tid] = mnew;
          red[R_MUSE + tid] = (mnew == -INFINITY) ? 0.f : mnew;
          red[R_ALPHA + tid] = alpha;
          const int any = __any_sync(0xffffffffu, resc);
          if (lane == 0) flags[2 + (tid >> 5)] = any;
        }
        named_bar_sync(1, 128);
        const bool any_resc = (flags[2] | flags[3]) != 0;
        // probabilities for this key, all heads
        uint32_t pk[32];
        float ps[64];
#pragma unroll
        for (int h = 0; h < 64; h += 2) {
          const float e0 = ex2_approx(xv[h] - red[R_MUSE + h]);
          const float e1 = ex2_approx(xv[h + 1] - red[R_MUSE + h + 1]);
          ps[h] = e0;
          ps[h + 1] = e1;
          pk[h / 2] = pack_bf16x2(e0, e1);
        }
        warp_transpose_reduce64<false>(ps);
        red[R_SUM + gw * 64 + 2 * lane] = ps[0];
        red[R_SUM + gw * 64 + 2 * lane + 1] = ps[1];

        // P^T buffer and O^T are free once the previous O^T MMA completed.
        if (!group_wait(bar(B_PFREE), (pvidx & 1) ^ 1, 61)) { ok = false; break; }
        tc_fence_after();
        if (tid < 64) {
          const float ssum = red[R_SUM + tid] + red[R_SUM + 64 + tid] + red[R_SUM + 128 + tid] +
                             red[R_SUM + 192 + tid];
          red[R_LRUN + tid] = red[R_LRUN + tid] * red[R_ALPHA + tid] + ssum;
        }
        if (any_resc) {
          // O^T[dv, h] *= alpha[h] for the 4 dv chunks this lane holds
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int hh = 0; hh < 64; hh += 32) {
              uint32_t o[32];
              tmem_ld32(tl + kTmemO + 64 * c + hh, o);
              tmem_wait_ld_dep32(o);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                o[i] = __float_as_uint(__uint_as_float(o[i]) * red[R_ALPHA + hh + i]);
              tmem_st32(tl + kTmemO + 64 * c + hh, o);
            }
          }
          tmem_wait_st();
        }
        uint8_t* ptrow = smem + kSmemPT;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(ptrow + sw128_offset(key, c)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(1, 128);
        if (tid == 0) mbar_arrive(bar(B_PFULL));
        ++pvidx;
      }
      if (!ok) break;
      // ---------------------------------------------------------- partial out
      if (!group_wait(bar(B_OFULL), nseg & 1, 62)) { ok = false; break; }
      tc_fence_after();
      const int slot = blockIdx.x + s;
      float* wo = p.ws_o + static_cast<size_t>(slot) * kHeads * kDim;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int hh = 0; hh < 64; hh += 32) {
          uint32_t o[32];
          tmem_ld32(tl + kTmemO + 64 * c + hh, o);
          tmem_wait_ld_dep32(o);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            wo[static_cast<size_t>(hh + i) * kDim + 128 * c + key] = __uint_as_float(o[i]);
        }
      }
      tc_fence_before();
      named_bar_sync(1, 128);
      if (tid == 0) mbar_arrive(bar(B_OFREE));
      if (tid < 64) {
        p.ws_ml[static_cast<size_t>(slot) * 128 + tid] = red[R_MRUN + tid];
        p.ws_ml[static_cast<size_t>(slot) * 128 + 64 + tid] = red[R_LRUN + tid];
      }
      named_bar_sync(1, 128);
      ++nseg;
      x = seg_end;
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Combine: CTA (sequence s, 8 heads), one warp per head, 16 value columns per
// lane.  The partials are merged online (running max, rescaled accumulator),
// two per round, so the loads of a round's (m, l) and its partial rows go out
// together and the kernel needs few enough registers to run in one wave.
// Empty splits are recognised arithmetically; a split whose keys were all
// masked has m = -inf, weight 0 and a zero row.
// ---------------------------------------------------------------------------
constexpr int kCombineHeads = 8;

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__global__ void __launch_bounds__(32 * kCombineHeads)
    combine_kernel(const Params p, int grid, const uint16_t* __restrict__ g,
                   uint16_t* __restrict__ out) {
  const int s = blockIdx.x;
  const int h = blockIdx.y * kCombineHeads + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  // the gate row does not depend on the split pass: load it before waiting
  const size_t obase = (static_cast<size_t>(s) * kHeads + h) * kDim + 16 * lane;
  const uint4* gp = reinterpret_cast<const uint4*>(g + obase);
  const uint4 gv0 = __ldg(gp), gv1 = __ldg(gp + 1);
  pdl_wait();  // the split pass (a prerequisite grid) has finished and its writes are visible
  const long long N = p.seq_tile[p.S];
  const long long P0 = p.seq_tile[s], P1 = p.seq_tile[s + 1];
  // CTA that owns global tile x: ceil((x + 1) * grid / N) - 1
  auto owner = [&](long long x) -> int {
    return static_cast<int>(((x + 1) * grid + N - 1) / N) - 1;
  };
  const int c0 = owner(P0), c1 = owner(P1 - 1);
  const int np = c1 - c0 + 1;
  auto nonempty = [&](int c) { return N * c / grid < N * (c + 1) / grid; };
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float M = -INFINITY, L = 0.f;
#pragma unroll 1
  for (int i0 = 0; i0 < np; i0 += 2) {
    float m2[2], l2[2];
    float4 o[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = c0 + i0 + u;
      if (i0 + u < np && nonempty(c)) {
        const size_t slot = static_cast<size_t>(c + s);
        m2[u] = __ldg(p.ws_ml + slot * 128 + h);
        l2[u] = __ldg(p.ws_ml + slot * 128 + 64 + h);
        const float4* src =
            reinterpret_cast<const float4*>(p.ws_o + (slot * kHeads + h) * kDim) + lane * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) o[u][q] = __ldg(src + q);
      } else {
        m2[u] = -INFINITY;
        l2[u] = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) o[u][q] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const float Mn = fmaxf(M, fmaxf(m2[0], m2[1]));
    const float Mu = (Mn == -INFINITY) ? 0.f : Mn;
    const float sc = (M == -INFINITY) ? 0.f : ex2_approx(M - Mu);
    const float w0 = (m2[0] == -INFINITY) ? 0.f : ex2_approx(m2[0] - Mu);
    const float w1 = (m2[1] == -INFINITY) ? 0.f : ex2_approx(m2[1] - Mu);
    L = L * sc + w0 * l2[0] + w1 * l2[1];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[4 * q + 0] = fmaf(w1, o[1][q].x, fmaf(w0, o[0][q].x, acc[4 * q + 0] * sc));
      acc[4 * q + 1] = fmaf(w1, o[1][q].y, fmaf(w0, o[0][q].y, acc[4 * q + 1] * sc));
      acc[4 * q + 2] = fmaf(w1, o[1][q].z, fmaf(w0, o[0][q].z, acc[4 * q + 2] * sc));
      acc[4 * q + 3] = fmaf(w1, o[1][q].w, fmaf(w0, o[0][q].w, acc[4 * q + 3] * sc));
    }
    M = Mn;
  }
  const float inv = 1.f / L;
  uint4* op = reinterpret_cast<uint4*>(out + obase);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint4 gv = q ? gv1 : gv0;
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t ow[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a0 = acc[8 * q + 2 * k] * inv * sigmoid_fast(bf16lo_to_f32(gw[k]));
      const float a1 = acc[8 * q + 2 * k + 1] * inv * sigmoid_fast(bf16hi_to_f32(gw[k]));
      ow[k] = pack_bf16x2(a0, a1);
    }
    op[q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

}  // namespace decode
}  // namespace hca
