// HCA backward: the gradients of L = sum(dout * out) with respect to q, k, v,
// the block scores s and the gate g ('BaiduがERNIE 5.5 Flash Baseを公開' §3:
// the model is trained at 128K context; the forward is the attention of §2.1
// and the xenospectrum analysis, section 活性140億パラメータと長文処理を支える仕組み).
//
// With o the ungated output, out = sigmoid(g) o and P the softmax over each
// query's visible keys (compressed entries and raw window):
//   dg = dout out (1 - sigmoid(g)),  dO = dout sigmoid(g),  D = sum_d dout out
//   dP = dO . value,  dS = P (dP - D)
//   dq = scale sum dS key,  dkey = scale sum dS q,  dvalue = sum P dO
// and the entry gradients flow through each block's compressor (softmax
// weights w of its scores): dK_i += w_i dcK, dV_i += w_i dcV,
// ds_i = w_i (a_i - sum_m w_m a_m) with a_i = dcK . K_i + dcV . V_i.
//
// Five kernels, each streaming what the next needs through HBM:
//   prep      one warp per (position, head) row: dO (bf16), dg, D.
//   score     per 128-row tile (two positions x 64 heads) and key tile: S =
//             Q K^T and dP = dO V^T as two tcgen05 accumulators (double-
//             buffered in TMEM, so one tile's epilogue overlaps the next
//             tile's MMAs); the epilogue recomputes P from the forward's
//             log-sum-exp and writes P and dS (bf16, masked keys as 0) to a
//             scratch in the layout the GEMMs below load with TMA.
//   dq        per row tile: dq = scale dS [cK ; K_window], M = 128 rows,
//             N = 512 (two N = 256 accumulators fill TMEM).
//   dkv       per key tile of 128 keys: dV = P^T dO and dK = scale dS^T Q,
//             both operands read MN-major straight from the row-major
//             scratch and activations, K = 64 rows (one position) per stage;
//             a compressed tile is seen by most of the sequence, so its
//             positions are split into ranges whose fp32 partials are added
//             with vector reductions; raw tiles see at most 255 positions.
//   compress  per block: ds and the entry gradients into dK, dV.
// The GEMM kernels share one shape: warp 0 issues TMA copies into a ring,
// warp 1 owns TMEM and issues the MMAs, warps 2-5 run the epilogue (one TMEM
// lane quadrant each).
#pragma once

#include "hca_ptx.cuh"

namespace hca {
namespace bwd {

constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kThreads = 192;
constexpr int kRawW = 144;          // raw window columns of a row tile's scratch rows
constexpr int kRaw0 = 80;           // raw key tiles of the score pass: 80 + 64 keys
constexpr int kPosChunk = 512;      // positions per partial of a compressed dK/dV tile
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ int nc_of(int t) { return t >= 127 ? (t - 127) / 128 : 0; }
// first key of the raw scratch columns of the row tile starting at position
// t0: 8-aligned so that TMA boxes over the scratch start on 16-byte bounds
__device__ __forceinline__ int raw_base(int t0) { return ((t0 - 127) >> 3) << 3; }

struct Params {
  int B, T, nb;       // nb = T / 128 compressed entries per sequence
  int ncpad;          // row length of the compressed scratch (multiple of 128)
  int ut;             // row tiles per sequence, ceil(T / 2)
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
  const uint16_t* dout;   // [B, T, 64, 512]
  const uint16_t* out;
  const uint16_t* g;
  const float* lse;       // [B, T, 64] natural log (forward)
  uint16_t* dO;           // [B, T, 64, 512] scratch
  float* delta;           // [B, T, 64] scratch
  uint16_t* dg;           // [B, T, 64, 512]
  uint16_t* pc;           // [B][T * 64][ncpad] P over compressed entries
  uint16_t* dsc;          // same, dS
  uint16_t* pr;           // [B][T * 64][144] P over the raw window
  uint16_t* dsr;
  uint16_t* dq;           // [B, T, 64, 512]
  float* dk;              // [B, T, 512] accumulated
  float* dv;
  float* dck;             // [B, nb, 512] accumulated (scratch)
  float* dcv;
  const uint16_t* k;      // [B, T, 512]
  const uint16_t* v;
  const uint16_t* s;      // [B, T]
  float* ds;              // [B, T]
};

struct Maps {
  CUtensorMap q;      // (512, T*64, B) box (64, 128, 1)
  CUtensorMap dO;     // same, over the dO scratch
  CUtensorMap ck;     // (512, nb, B) box (64, 128, 1)
  CUtensorMap cv;
  CUtensorMap k;      // (512, T, B) box (64, 128, 1)
  CUtensorMap v;
  CUtensorMap dsc_a;  // (ncpad, T*64, B) box (64, 128, 1): [128 rows][64 entries]
  CUtensorMap dsr_a;  // (144, T*64, B) box (64, 128, 1)
  CUtensorMap ck4;    // (64, nb, 8, B) box (64, 64, 8, 1): [64 entries][512] as 8 slabs
  CUtensorMap k4;     // (64, T, 8, B) box (64, 64, 8, 1)
  CUtensorMap pc_t;   // (ncpad, T*64, B) box (64, 64, 1): [64 rows][64 entries]
  CUtensorMap dsc_t;
  CUtensorMap pr_t;   // (144, T*64, B) box (64, 64, 1)
  CUtensorMap dsr_t;
  CUtensorMap q4;     // (64, T*64, 8, B) box (64, 64, 8, 1): [64 rows][512] as 8 slabs
  CUtensorMap dO4;
};

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// ---------------------------------------------------------------------------
// prep: one warp per row; lane l holds elements 16 l .. 16 l + 15
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) prep_kernel(const Params p, long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const size_t off = static_cast<size_t>(row) * kDim + 16 * lane;
  const uint4* pd = reinterpret_cast<const uint4*>(p.dout + off);
  const uint4* po = reinterpret_cast<const uint4*>(p.out + off);
  const uint4* pg = reinterpret_cast<const uint4*>(p.g + off);
  uint4 wd[2] = {ld_nc_v4(pd), ld_nc_v4(pd + 1)};
  uint4 wo[2] = {ld_nc_v4(po), ld_nc_v4(po + 1)};
  uint4 wg[2] = {ld_nc_v4(pg), ld_nc_v4(pg + 1)};
  uint32_t rdo[8], rdg[8];
  float dsum = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = (&wd[i >> 2].x)[i & 3], o = (&wo[i >> 2].x)[i & 3],
                   gg = (&wg[i >> 2].x)[i & 3];
    float d2[2] = {bf16lo_to_f32(a), bf16hi_to_f32(a)};
    float o2[2] = {bf16lo_to_f32(o), bf16hi_to_f32(o)};
    float g2[2] = {bf16lo_to_f32(gg), bf16hi_to_f32(gg)};
    float x[2], y[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float sg = 1.f / (1.f + __expf(-g2[j]));
      x[j] = d2[j] * sg;
      y[j] = d2[j] * o2[j] * (1.f - sg);
      dsum = fmaf(d2[j], o2[j], dsum);
    }
    rdo[i] = pack_bf16x2(x[0], x[1]);
    rdg[i] = pack_bf16x2(y[0], y[1]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  uint4* qo = reinterpret_cast<uint4*>(p.dO + off);
  uint4* qg = reinterpret_cast<uint4*>(p.dg + off);
  qo[0] = make_uint4(rdo[0], rdo[1], rdo[2], rdo[3]);
  qo[1] = make_uint4(rdo[4], rdo[5], rdo[6], rdo[7]);
  qg[0] = make_uint4(rdg[0], rdg[1], rdg[2], rdg[3]);
  qg[1] = make_uint4(rdg[4], rdg[5], rdg[6], rdg[7]);
  if (lane == 0) p.delta[row] = dsum;
}

// ---------------------------------------------------------------------------
// Shared pieces of the GEMM kernels
// ---------------------------------------------------------------------------
enum { FULL = 0, EMPTY = 3, TFULL = 6, TFREE = 8, NBAR = 10 };
constexpr int kBarOff = 0;                  // barriers, TMEM slot, abort flag: 256 B
constexpr int kRingOff = 1024;
constexpr int kStages3 = 3;                 // score: 3 x 64 KB
constexpr int kStageScore = 65536;
constexpr int kStages2 = 2;                 // dq, dkv: 2 x 80 KB
constexpr int kStageGemm = 81920;
constexpr int kSmemScore = kRingOff + kStages3 * kStageScore;
constexpr int kSmemGemm = kRingOff + kStages2 * kStageGemm;
constexpr int kSmemAllocScore = kSmemScore + 1024;
constexpr int kSmemAllocGemm = kSmemGemm + 1024;
static_assert(kSmemAllocScore <= 232448 && kSmemAllocGemm <= 232448, "shared memory budget");

struct Ctx {
  uint8_t* smem;
  uint32_t sb;
  volatile int* abort_flag;
  uint32_t* tmem_slot;
  __device__ uint32_t bar(int i) const { return sb + kBarOff + 8u * static_cast<uint32_t>(i); }
};

__device__ __forceinline__ Ctx gemm_setup(uint8_t* smem_raw, int nstages) {
  Ctx c;
  c.smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  c.sb = smem_u32(c.smem);
  c.abort_flag = reinterpret_cast<volatile int*>(c.smem + kBarOff + 8 * NBAR);
  c.tmem_slot = reinterpret_cast<uint32_t*>(c.smem + kBarOff + 8 * NBAR + 4);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) {
      mbar_init(c.bar(FULL + s), 1);
      mbar_init(c.bar(EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(c.bar(TFULL + i), 1);
      mbar_init(c.bar(TFREE + i), 4);
    }
    *c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(c.tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  return c;
}

__device__ __forceinline__ void gemm_teardown(const Ctx& c, uint32_t tmem) {
  __syncwarp();
  if (threadIdx.x == 0) abort_drain(c.abort_flag);
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// score: S = Q K^T and dP = dO V^T per (row tile, key tile); writes P and dS
// ---------------------------------------------------------------------------
struct ScoreTile {
  int b, t0, nct, ntiles, kb;
};
__device__ __forceinline__ ScoreTile score_tile(const Params& p, int id) {
  ScoreTile x;
  x.b = id / p.ut;
  x.t0 = 2 * (id - x.b * p.ut);
  const int nc = nc_of(min(x.t0 + 1, p.T - 1));
  x.nct = (nc + 127) >> 7;
  x.ntiles = x.nct + 2;
  x.kb = raw_base(x.t0);
  return x;
}
// keys of key tile j and its first key (compressed: entry index)
__device__ __forceinline__ int score_n(const ScoreTile& x, int j) {
  return j < x.nct ? 128 : (j == x.nct ? kRaw0 : kRawW - kRaw0);
}

__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Ctx c = gemm_setup(smem_raw, kStages3);
  const uint32_t tmem = *c.tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = p.B * p.ut;
  if (warp == 0) {
    if (lane == 0) {
      uint32_t u = 0;
      bool ok = true;
      for (int id = blockIdx.x; id < ntile && ok; id += gridDim.x) {
        const ScoreTile x = score_tile(p, id);
        for (int j = 0; j < x.ntiles && ok; ++j) {
          const bool comp = j < x.nct;
          const int key0 = comp ? 128 * j : x.kb + (j == x.nct ? 0 : kRaw0);
#pragma unroll 1
          for (int d = 0; d < 8; ++d, ++u) {
            const uint32_t st = u % kStages3;
            ok = mbar_wait(c.bar(EMPTY + st), ((u / kStages3) & 1) ^ 1, c.abort_flag,
                           kWaitLimitNs, 400);
            if (!ok) break;
            const uint32_t dst = c.sb + kRingOff + st * kStageScore;
            const uint32_t fb = c.bar(FULL + st);
            mbar_expect_tx(fb, kStageScore);
            tma_load_3d(dst, &maps.q, fb, 64 * d, x.t0 * kHeads, x.b);
            tma_load_3d(dst + 16384, &maps.dO, fb, 64 * d, x.t0 * kHeads, x.b);
            tma_load_3d(dst + 32768, comp ? &maps.ck : &maps.k, fb, 64 * d, key0, x.b);
            tma_load_3d(dst + 49152, comp ? &maps.cv : &maps.v, fb, 64 * d, key0, x.b);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t u = 0, kt = 0;
      bool ok = true;
      for (int id = blockIdx.x; id < ntile && ok; id += gridDim.x) {
        const ScoreTile x = score_tile(p, id);
        for (int j = 0; j < x.ntiles && ok; ++j, ++kt) {
          const uint32_t bb = kt & 1;
          ok = mbar_wait(c.bar(TFREE + bb), ((kt >> 1) & 1) ^ 1, c.abort_flag, kWaitLimitNs, 401);
          if (!ok) break;
          tc_fence_after();
          const uint32_t idesc = idesc_bf16_f32(128, score_n(x, j), false, false);
          const uint32_t dS = tmem + 256 * bb, dP = dS + 128;
#pragma unroll 1
          for (int d = 0; d < 8; ++d, ++u) {
            const uint32_t st = u % kStages3;
            ok = mbar_wait(c.bar(FULL + st), (u / kStages3) & 1, c.abort_flag, kWaitLimitNs, 402);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a = c.sb + kRingOff + st * kStageScore;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t acc = (d | k) != 0;
              umma_bf16(dS, sdesc_sw128(a + 32 * k, 16, 1024),
                        sdesc_sw128(a + 32768 + 32 * k, 16, 1024), idesc, acc);
              umma_bf16(dP, sdesc_sw128(a + 16384 + 32 * k, 16, 1024),
                        sdesc_sw128(a + 49152 + 32 * k, 16, 1024), idesc, acc);
            }
            umma_commit(c.bar(EMPTY + st));
          }
          if (!ok) break;
          umma_commit(c.bar(TFULL + bb));
        }
      }
    }
  } else {
    // epilogue: thread = row of the tile (TMEM lane)
    const int row = 32 * (warp & 3) + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    uint32_t kt = 0;
    bool ok = true;
    for (int id = blockIdx.x; id < ntile && ok; id += gridDim.x) {
      const ScoreTile x = score_tile(p, id);
      const int t = x.t0 + (row >> 6);
      const bool valid = t < p.T;
      const size_t grow = (static_cast<size_t>(x.b) * p.T + (valid ? t : 0)) * kHeads + (row & 63);
      const float lse2 = valid ? p.lse[grow] * 1.4426950408889634f : 0.f;
      const float dl = valid ? p.delta[grow] : 0.f;
      const int ncv = nc_of(t);
      const int wlo = max(0, t - 127);
      for (int j = 0; j < x.ntiles && ok; ++j, ++kt) {
        const uint32_t bb = kt & 1;
        if (!mbar_wait_warp(c.bar(TFULL + bb), (kt >> 1) & 1, c.abort_flag, kWaitLimitNs, 403)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool comp = j < x.nct;
        const int n = score_n(x, j);
        const int key0 = comp ? 128 * j : x.kb + (j == x.nct ? 0 : kRaw0);
        uint16_t* prow = comp ? p.pc + grow * p.ncpad + 128 * j
                              : p.pr + grow * kRawW + (j == x.nct ? 0 : kRaw0);
        uint16_t* drow = comp ? p.dsc + grow * p.ncpad + 128 * j
                              : p.dsr + grow * kRawW + (j == x.nct ? 0 : kRaw0);
#pragma unroll 1
        for (int c0 = 0; c0 < n; c0 += 32) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tq + 256 * bb + c0, sr);
          tmem_ld32(tq + 256 * bb + 128 + c0, dr);
          tmem_wait_ld_dep32(sr);
          reg_dep32(dr);
          uint32_t pw[16], dw[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float pv[2], dv2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int key = key0 + c0 + i + e;
              const bool vis = comp ? key < ncv : (key >= wlo && key <= t);
              const float pr = vis ? ex2_approx(fmaf(__uint_as_float(sr[i + e]), p.scale_log2,
                                                     -lse2))
                                   : 0.f;
              pv[e] = pr;
              dv2[e] = pr * (__uint_as_float(dr[i + e]) - dl);
            }
            pw[i >> 1] = pack_bf16x2(pv[0], pv[1]);
            dw[i >> 1] = pack_bf16x2(dv2[0], dv2[1]);
          }
          if (valid) {
            const int nv = min(32, n - c0);   // 32 or 16
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              if (8 * q4 < nv) {
                st_v4(reinterpret_cast<uint4*>(prow + c0 + 8 * q4),
                      make_uint4(pw[4 * q4], pw[4 * q4 + 1], pw[4 * q4 + 2], pw[4 * q4 + 3]));
                st_v4(reinterpret_cast<uint4*>(drow + c0 + 8 * q4),
                      make_uint4(dw[4 * q4], dw[4 * q4 + 1], dw[4 * q4 + 2], dw[4 * q4 + 3]));
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(TFREE + bb));
      }
    }
  }
  gemm_teardown(c, tmem);
}

// ---------------------------------------------------------------------------
// dq: per row tile, dq = scale dS [cK ; K_window]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Ctx c = gemm_setup(smem_raw, kStages2);
  const uint32_t tmem = *c.tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = p.B * p.ut;
  // chunks of 64 keys: 2 nct compressed, then 3 raw (64 + 64 + 16 keys; the
  // scratch columns past 144 read as zeros)
  if (warp == 0) {
    if (lane == 0) {
      uint32_t u = 0;
      bool ok = true;
      for (int id = blockIdx.x; id < ntile && ok; id += gridDim.x) {
        const ScoreTile x = score_tile(p, id);
        const int nch = 2 * x.nct + 3;
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch, ++u) {
          const uint32_t st = u % kStages2;
          ok = mbar_wait(c.bar(EMPTY + st), ((u / kStages2) & 1) ^ 1, c.abort_flag, kWaitLimitNs,
                         410);
          if (!ok) break;
          const uint32_t dst = c.sb + kRingOff + st * kStageGemm;
          const uint32_t fb = c.bar(FULL + st);
          mbar_expect_tx(fb, kStageGemm);
          const bool comp = ch < 2 * x.nct;
          const int rc = ch - 2 * x.nct;
          tma_load_3d(dst, comp ? &maps.dsc_a : &maps.dsr_a, fb, comp ? 64 * ch : 64 * rc,
                      x.t0 * kHeads, x.b);
          tma_load_4d(dst + 16384, comp ? &maps.ck4 : &maps.k4, fb, 0,
                      comp ? 64 * ch : x.kb + 64 * rc, 0, x.b);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t u = 0, it = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32(128, 256, false, true);
      for (int id = blockIdx.x; id < ntile && ok; id += gridDim.x, ++it) {
        const ScoreTile x = score_tile(p, id);
        const int nch = 2 * x.nct + 3;
        ok = mbar_wait(c.bar(TFREE), (it & 1) ^ 1, c.abort_flag, kWaitLimitNs, 411);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch, ++u) {
          const uint32_t st = u % kStages2;
          ok = mbar_wait(c.bar(FULL + st), (u / kStages2) & 1, c.abort_flag, kWaitLimitNs, 412);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = c.sb + kRingOff + st * kStageGemm;
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
              umma_bf16(tmem + 256 * nh, sdesc_sw128(a + 32 * k, 16, 1024),
                        sdesc_sw128(a + 16384 + 2048 * k + 32768 * nh, 8192, 1024), idesc,
                        (ch | k) != 0);
          umma_commit(c.bar(EMPTY + st));
        }
        if (!ok) break;
        umma_commit(c.bar(TFULL));
      }
    }
  } else {
    const int row = 32 * (warp & 3) + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    uint32_t it = 0;
    for (int id = blockIdx.x; id < ntile; id += gridDim.x, ++it) {
      const ScoreTile x = score_tile(p, id);
      if (!mbar_wait_warp(c.bar(TFULL), it & 1, c.abort_flag, kWaitLimitNs, 413)) break;
      tc_fence_after();
      const int t = x.t0 + (row >> 6);
      const bool valid = t < p.T;
      uint4* dst = reinterpret_cast<uint4*>(
          p.dq + ((static_cast<size_t>(x.b) * p.T + (valid ? t : 0)) * kHeads + (row & 63)) *
                     kDim);
#pragma unroll 1
      for (int c0 = 0; c0 < kDim; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tq + c0, r);
        tmem_wait_ld_dep32(r);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * p.scale,
                             __uint_as_float(r[2 * i + 1]) * p.scale);
        if (valid) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            st_v4(dst + (c0 >> 3) + q4,
                  make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(TFREE));
    }
  }
  gemm_teardown(c, tmem);
}

// ---------------------------------------------------------------------------
// dkv: per key tile (128 keys) and gradient (V: P^T dO, K: scale dS^T Q)
// ---------------------------------------------------------------------------
struct KvItem {
  int b, which;       // which: 0 = dV, 1 = dK
  bool comp;
  int m;              // key tile
  int p0, p1;         // positions [p0, p1)
};

// compressed tile m is seen by positions t >= 128 (128 m + 1) + 127
__device__ __forceinline__ int comp_first_pos(int m) { return 128 * (128 * m + 1) + 127; }
__device__ __forceinline__ int comp_splits(const Params& p, int m) {
  const int n = p.T - comp_first_pos(m);
  return n > 0 ? (n + kPosChunk - 1) / kPosChunk : 0;
}
__device__ __forceinline__ int kv_items_per_bw(const Params& p) {
  int n = (p.T + 127) >> 7;   // raw tiles
  for (int m = 0; m < (p.nb + 127) >> 7; ++m) n += comp_splits(p, m);
  return n;
}
__device__ __forceinline__ KvItem kv_item(const Params& p, int per_bw, int id) {
  KvItem x;
  const int bw = id / per_bw;
  int r = id - bw * per_bw;
  x.b = bw >> 1;
  x.which = bw & 1;
  const int nct = (p.nb + 127) >> 7;
  for (int m = 0; m < nct; ++m) {
    const int sp = comp_splits(p, m);
    if (r < sp) {
      x.comp = true;
      x.m = m;
      x.p0 = comp_first_pos(m) + r * kPosChunk;
      x.p1 = min(p.T, x.p0 + kPosChunk);
      return x;
    }
    r -= sp;
  }
  x.comp = false;
  x.m = r;
  x.p0 = 128 * r;
  x.p1 = min(p.T, 128 * r + 255);
  return x;
}

__global__ void __launch_bounds__(kThreads, 1)
    dkv_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Ctx c = gemm_setup(smem_raw, kStages2);
  const uint32_t tmem = *c.tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_bw = kv_items_per_bw(p);
  const int nitems = p.B * 2 * per_bw;
  if (warp == 0) {
    if (lane == 0) {
      uint32_t u = 0;
      bool ok = true;
      for (int id = blockIdx.x; id < nitems && ok; id += gridDim.x) {
        const KvItem x = kv_item(p, per_bw, id);
        const CUtensorMap* am = x.comp ? (x.which ? &maps.dsc_t : &maps.pc_t)
                                       : (x.which ? &maps.dsr_t : &maps.pr_t);
        const CUtensorMap* bm = x.which ? &maps.q4 : &maps.dO4;
#pragma unroll 1
        for (int t = x.p0; t < x.p1; ++t, ++u) {
          const uint32_t st = u % kStages2;
          ok = mbar_wait(c.bar(EMPTY + st), ((u / kStages2) & 1) ^ 1, c.abort_flag, kWaitLimitNs,
                         420);
          if (!ok) break;
          const uint32_t dst = c.sb + kRingOff + st * kStageGemm;
          const uint32_t fb = c.bar(FULL + st);
          mbar_expect_tx(fb, kStageGemm);
          const int x0 = x.comp ? 128 * x.m : 128 * x.m - raw_base(t & ~1);
          tma_load_3d(dst, am, fb, x0, t * kHeads, x.b);
          tma_load_3d(dst + 8192, am, fb, x0 + 64, t * kHeads, x.b);
          tma_load_4d(dst + 16384, bm, fb, 0, t * kHeads, 0, x.b);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t u = 0, it = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32(128, 256, true, true);
      for (int id = blockIdx.x; id < nitems && ok; id += gridDim.x, ++it) {
        const KvItem x = kv_item(p, per_bw, id);
        ok = mbar_wait(c.bar(TFREE), (it & 1) ^ 1, c.abort_flag, kWaitLimitNs, 421);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int t = x.p0; t < x.p1; ++t, ++u) {
          const uint32_t st = u % kStages2;
          ok = mbar_wait(c.bar(FULL + st), (u / kStages2) & 1, c.abort_flag, kWaitLimitNs, 422);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = c.sb + kRingOff + st * kStageGemm;
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
              umma_bf16(tmem + 256 * nh, sdesc_sw128(a + 2048 * k, 8192, 1024),
                        sdesc_sw128(a + 16384 + 2048 * k + 32768 * nh, 8192, 1024), idesc,
                        (t != x.p0 || k != 0) ? 1u : 0u);
          umma_commit(c.bar(EMPTY + st));
        }
        if (!ok) break;
        umma_commit(c.bar(TFULL));
      }
    }
  } else {
    const int row = 32 * (warp & 3) + lane;   // key of the tile
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    uint32_t it = 0;
    for (int id = blockIdx.x; id < nitems; id += gridDim.x, ++it) {
      const KvItem x = kv_item(p, per_bw, id);
      if (!mbar_wait_warp(c.bar(TFULL), it & 1, c.abort_flag, kWaitLimitNs, 423)) break;
      tc_fence_after();
      const int key = 128 * x.m + row;
      const bool valid = x.comp ? key < p.nb : key < p.T;
      const float mul = x.which ? p.scale : 1.f;
      float* dst = x.comp ? (x.which ? p.dck : p.dcv) + (static_cast<size_t>(x.b) * p.nb + key) * kDim
                          : (x.which ? p.dk : p.dv) + (static_cast<size_t>(x.b) * p.T + key) * kDim;
#pragma unroll 1
      for (int c0 = 0; c0 < kDim; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tq + c0, r);
        tmem_wait_ld_dep32(r);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            red_add_v4(dst + c0 + i, __uint_as_float(r[i]) * mul, __uint_as_float(r[i + 1]) * mul,
                       __uint_as_float(r[i + 2]) * mul, __uint_as_float(r[i + 3]) * mul);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(TFREE));
    }
  }
  gemm_teardown(c, tmem);
}

// ---------------------------------------------------------------------------
// compress: per block j, ds and the entry gradients into dK, dV.  Warp w
// takes tokens w, w + 4, ..; lane l elements 16 l .. 16 l + 15.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) compress_bwd_kernel(const Params p) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float w_s[128], a_s[128], red[4];
  const size_t tok0 = static_cast<size_t>(b) * p.T + 128 * j;
  // softmax weights of the block's scores
  const float sv = __uint_as_float(static_cast<uint32_t>(p.s[tok0 + threadIdx.x]) << 16);
  float m = sv;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float e = __expf(sv - m);
  float sum = e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  __syncthreads();
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = red[0] + red[1] + red[2] + red[3];
  w_s[threadIdx.x] = e / sum;
  __syncthreads();
  const float4* gk = reinterpret_cast<const float4*>(p.dck + (static_cast<size_t>(b) * p.nb + j) * kDim + 16 * lane);
  const float4* gv = reinterpret_cast<const float4*>(p.dcv + (static_cast<size_t>(b) * p.nb + j) * kDim + 16 * lane);
  float ck[16], cv[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = gk[i], y = gv[i];
    ck[4 * i] = x.x; ck[4 * i + 1] = x.y; ck[4 * i + 2] = x.z; ck[4 * i + 3] = x.w;
    cv[4 * i] = y.x; cv[4 * i + 1] = y.y; cv[4 * i + 2] = y.z; cv[4 * i + 3] = y.w;
  }
#pragma unroll 1
  for (int i = warp; i < 128; i += 4) {
    const size_t tok = tok0 + i;
    const float wi = w_s[i];
    const uint4* kr = reinterpret_cast<const uint4*>(p.k + tok * kDim + 16 * lane);
    const uint4* vr = reinterpret_cast<const uint4*>(p.v + tok * kDim + 16 * lane);
    const uint4 k0 = ld_nc_v4(kr), k1 = ld_nc_v4(kr + 1), v0 = ld_nc_v4(vr), v1 = ld_nc_v4(vr + 1);
    const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
    const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float a = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a = fmaf(ck[2 * q], bf16lo_to_f32(kw[q]), a);
      a = fmaf(ck[2 * q + 1], bf16hi_to_f32(kw[q]), a);
      a = fmaf(cv[2 * q], bf16lo_to_f32(vw[q]), a);
      a = fmaf(cv[2 * q + 1], bf16hi_to_f32(vw[q]), a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) a_s[i] = a;
    float4* dkr = reinterpret_cast<float4*>(p.dk + tok * kDim + 16 * lane);
    float4* dvr = reinterpret_cast<float4*>(p.dv + tok * kDim + 16 * lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4 x = dkr[q], y = dvr[q];
      x.x = fmaf(wi, ck[4 * q], x.x); x.y = fmaf(wi, ck[4 * q + 1], x.y);
      x.z = fmaf(wi, ck[4 * q + 2], x.z); x.w = fmaf(wi, ck[4 * q + 3], x.w);
      y.x = fmaf(wi, cv[4 * q], y.x); y.y = fmaf(wi, cv[4 * q + 1], y.y);
      y.z = fmaf(wi, cv[4 * q + 2], y.z); y.w = fmaf(wi, cv[4 * q + 3], y.w);
      dkr[q] = x;
      dvr[q] = y;
    }
  }
  __syncthreads();
  float wa = w_s[threadIdx.x] * a_s[threadIdx.x];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wa += __shfl_xor_sync(0xffffffffu, wa, o);
  if (lane == 0) red[warp] = wa;
  __syncthreads();
  const float tot = red[0] + red[1] + red[2] + red[3];
  p.ds[tok0 + threadIdx.x] = w_s[threadIdx.x] * (a_s[threadIdx.x] - tot);
}

}  // namespace bwd
}  // namespace hca
