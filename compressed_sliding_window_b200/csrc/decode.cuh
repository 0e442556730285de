// HCA decode: one new query token per sequence, split-KV over all SMs, then,
// in the same kernel behind a grid barrier, a log-sum-exp combine.
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
// A CTA writes one partial (O / l in bf16, running max m, running sum l) per
// sequence it touches, into slot c + i of the workspace (slots never collide:
// a CTA's sequences are consecutive and later CTAs start at later sequences).
// Up to kInlineSeqs sequences every CTA computes the tile prefix itself in
// shared memory; beyond that a one-CTA plan kernel does.
// The launch is cooperative; after every CTA has written its partials (an
// atomic counter, bounded spin) every CTA merges a share of the (sequence,
// head) rows, its partial rows staged in shared memory by bulk copies.
//
// Tensor-core mapping (swap-AB).  With 64 heads a plain S = Q K^T would use
// M = 64; instead keys go on the 128-lane M axis:
//   S^T[key, head] = K_tile[key, :] . Q[head, :]        (M=128, N=64, K=512)
//   O^T[dv, head] += V_tile[:, dv]^T . P^T[:, head]      (4 x M=128 dv, N=64, K=128)
// TMEM holds O^T (4 x 64 columns) and two 64-column S^T buffers.
//
// FP8 cache (decode_kernel<true>).  The cache rows are e4m3 codes with one
// fp32 scale per row (half the bytes to stream).  Each producer warp loads
// 16 KB code tiles (128 keys x 128 channels) into its own staging slots and,
// with all 32 lanes, turns a landed tile into its f16 ring stage (a few
// integer operations and one f16x2 multiply per two values: every e4m3 value
// is exact in f16); Q is turned from bf16 into f16 in place by the softmax
// warps at each segment start (exact for |q| < 65504), and the MMAs run in
// f16.  Each softmax thread owns one key: it multiplies its scores by the
// key's K scale and its probabilities by the key's V scale before they feed
// P.V (the row sums use the unscaled probabilities), so no scaling touches
// the operand tiles.
//
// The softmax runs across lanes: each thread owns one key and its 64 head scores, and the
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
constexpr int kSmemRing = 65536;    // 4 x 32 KB (FP8 cache: 2 x 32 KB, then 4 x 16 KB staging)
constexpr int kStagesF8 = 2;
constexpr int kStgBytes = 16384;    // one FP8 code tile: [128 keys][128 bytes]
constexpr int kSmemStg = kSmemRing + kStagesF8 * 2 * kSlab;
constexpr int kSmemPT = kSmemRing + kStages * kStage;  // P^T [128 keys x 64 heads] bf16, 16 KB
constexpr int kSmemRed = kSmemPT + 16384;             // reductions, 4 KB
constexpr int kSmemBar = kSmemRed + 4096;
constexpr int kInlineSeqs = 1024;   // up to this many sequences each CTA plans for itself
constexpr int kSmemTiles = kSmemBar + 256;                  // [kInlineSeqs + 1] int64 prefix
constexpr int kSmemCtx = kSmemTiles + 8 * (kInlineSeqs + 1) + 8;  // [kInlineSeqs] int32
constexpr int kSmemBytes = kSmemCtx + 4 * kInlineSeqs;
constexpr int kSmemAlloc = kSmemBytes + 1024;
constexpr int kThreads = 224;
constexpr float kTau = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
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
  B_OFREE = B_OFULL + 1, B_DRAIN = B_OFREE + 1, B_COMB = B_DRAIN + 1, B_STG = B_COMB + 1,
  B_QCONV = B_STG + 4, B_COUNT = B_QCONV + 1
};
constexpr int kTmemSlot = 8 * B_COUNT;
constexpr int kAbortSlot = kTmemSlot + 4;
static_assert(kAbortSlot + 4 <= 256, "barrier region overflow");
static_assert(kSmemStg + 4 * kStgBytes == kSmemRing + kStages * 2 * 16384, "FP8 layout");

constexpr uint32_t kTmemO = 0, kTmemS0 = 256, kTmemS1 = 320, kTmemCols = 512;

// Workspace layout (bytes): [slots][64 heads][128][4] bf16 partial O, normalised by its
// l and stored with value column 128c + r at [r][c] (one 8-byte store per head
// and TMEM lane); then [slots][2][64] fp32 (m, l)
// in log2 units.  slots = grid + S.
__host__ __device__ inline size_t ws_o_bytes(int slots) {
  return static_cast<size_t>(slots) * kHeads * kDim * 2;
}
__host__ __device__ inline size_t ws_bytes(int slots) {
  return ws_o_bytes(slots) + static_cast<size_t>(slots) * 2 * kHeads * 4;
}

struct Params {
  const int* ctx_len;  // [S] device
  int S;
  int max_nc;
  float scale_log2;
  uint16_t* ws_o;      // [slots][64][128][4] bf16
  float* ws_ml;        // [slots][2][64]
  long long* seq_tile; // [S + 1] exclusive prefix of tile counts (plan kernel, S > kInlineSeqs)
  unsigned long long* gsync;  // grid barrier arrivals (zero before first use, see below)
  const uint16_t* g;   // [S, 64, 512] bf16 gate
  uint16_t* out;       // [S, 64, 512] bf16
  // FP8 cache only: per-row scales of ck, cv [S, max_nc] and wk, wv [S, 128]
  const float* sck;
  const float* scv;
  const float* swk;
  const float* swv;
  // virtual head attention factors [64][vha_rank] bf16 (vha_rank = 0: none)
  const uint16_t* vha_down;
  const uint16_t* vha_up;
  int vha_rank;
};

__device__ __forceinline__ int nc_of_len(int L) { return L >= 128 ? (L - 128) / 128 : 0; }

// floor(a / b) for a >= 0, b > 0, in 32-bit arithmetic whenever both fit
// (the 64-bit division is a long instruction sequence on the GPU).
__device__ __forceinline__ long long div_nn(long long a, long long b) {
  if (((static_cast<unsigned long long>(a) | static_cast<unsigned long long>(b)) >> 32) == 0)
    return static_cast<long long>(static_cast<uint32_t>(a) / static_cast<uint32_t>(b));
  return a / b;
}

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

__device__ __forceinline__ SeqInfo seq_info(const int* lens, int max_nc, int s) {
  SeqInfo r;
  r.L = max(1, lens[s]);
  r.nc = min(max(nc_of_len(r.L), 0), max_nc);
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

// Inline plan (S <= kInlineSeqs): every CTA reads the context lengths into
// shared memory and computes the tile prefix itself, which saves the plan
// kernel's launch.  Thread t takes a run of ceil(S / kThreads) sequences; the
// runs' sums are scanned across the block.  Only CTA 0 reports bad lengths.
__device__ __forceinline__ void inline_plan(const Params& p, long long* sT, int* sL) {
  __shared__ long long wsum[kThreads / 32];
  constexpr int kPer = (kInlineSeqs + kThreads - 1) / kThreads;
  const int per = (p.S + kThreads - 1) / kThreads;
  const int i0 = threadIdx.x * per;
  int n[kPer];
  long long run = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    n[u] = 0;
    const int i = i0 + u;
    if (u < per && i < p.S) {
      const int L = p.ctx_len[i];
      int nc = nc_of_len(L);
      if ((L < 1 || nc > p.max_nc) && blockIdx.x == 0) record_error(DEVERR_BAD_INPUT, 101);
      nc = min(max(nc, 0), p.max_nc);
      n[u] = (nc + kKeyTile - 1) / kKeyTile + 1;
      sL[i] = L;
      run += n[u];
    }
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  long long x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  long long before = x - run;
  for (int v = 0; v < w; ++v) before += wsum[v];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = i0 + u;
    if (u < per && i < p.S) {
      sT[i] = before;
      before += n[u];
    }
  }
  if (threadIdx.x == kThreads - 1) {
    long long tot = 0;
    for (int v = 0; v < kThreads / 32; ++v) tot += wsum[v];
    sT[p.S] = tot;
  }
  __syncthreads();
}

// 4-D views (64, rows, 8 slabs, S) of [S][rows][512] tensors: a box
// (64, rows, n, 1) lands as n 64-wide slabs of [rows][64], 128B-swizzled.
// (FP8 cache: ck, cv, wk, wv are [S][rows][512 bytes] code maps, box
// (128 bytes, 128 rows, 1), no swizzle.)
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

// ---------------------------------------------------------------------------
// Combine phase.  CTA c merges rows [cR/G, (c+1)R/G) of the R = 64 S
// (sequence, head) rows, kCombRows at a time.  The partial rows a group needs
// are, for each of its (at most two) sequences, the same head range of every
// split that touched the sequence: contiguous runs of 2 KB per head in the
// workspace.  They are brought into shared memory by bulk copies, together
// with the splits' (m, l) vectors, up to kCombItems runs and the 192 KB of the
// Q and ring buffers per batch, so a whole batch of reads is in flight at
// once.  Everything that does not read a partial -- the group's split ranges,
// the gate loads and sigmoid(g) -- is done before the grid barrier, while
// the slowest CTAs are still streaming.  Warp w merges rows
// w, w+7, w+14, w+21 of the group, the four rows interleaved: per batch the
// largest m of its splits first, one rescale of the running sum, then one
// weight per split; lane l covers value columns 128q + 4l .. 128q + 4l + 3
// (q = 0..3), which keeps the shared memory reads conflict-free and the gate
// loads and output stores 8 bytes per lane.  Empty splits (a CTA that got no
// tile) are skipped; a split whose keys were all masked has m = -inf and
// weight 0.
// ---------------------------------------------------------------------------
constexpr int kCombRows = 28;              // 7 warps x 4 rows
constexpr int kCombItems = 32;             // runs per batch (bounded by the (m, l) area)
constexpr int kCombData = kSmemPT;         // [Q | ring]: 192 KB of partial rows
constexpr int kCombMl = kSmemPT;           // P^T area: 32 x 512 B of (m, l)
static_assert(kCombItems * 512 <= 16384, "(m, l) staging area");
static_assert(2 * kHeads * kHeads * 4 + kThreads / 32 * kHeads * 8 * 2 <= kSmemPT - kSmemQ,
              "head-mix factors and tiles");

// sigmoid(g) is held as f16 pairs until the store (its relative rounding,
// 2^-11, is below that of the bf16 output)
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float f16lo_to_f32(uint32_t v) {
  float r;
  asm("{.reg .f16 a, b;\n mov.b32 {a, b}, %1;\n cvt.f32.f16 %0, a;}" : "=f"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ float f16hi_to_f32(uint32_t v) {
  float r;
  asm("{.reg .f16 a, b;\n mov.b32 {a, b}, %1;\n cvt.f32.f16 %0, b;}" : "=f"(r) : "r"(v));
  return r;
}

struct CombSeq {
  int s;       // sequence
  int h0, nh;  // head range [h0, h0 + nh) of the group inside the sequence
  int c0, n;   // split CTAs c0 .. c0 + n - 1
};

// Merge of one batch's runs into a warp's first NK rows, NU runs per step
// (NK x NU <= 4 row-runs in flight per step).  Runs are taken in order;
// `run_of(f)` gives run f's byte offset in the staged buffer and whether it
// holds data (an empty split's run was never copied), `seq_a(f)` whether run
// f belongs to the group's first sequence.  A row of the other sequence reads
// some in-bounds words and replaces them by zeros with weight 0.
template <int NK, int NU, typename RunOf, typename SeqA>
__device__ __forceinline__ void merge_runs(const uint8_t* smem, int fs, int fe,
                                           const bool (&rowA)[4], const int (&hrow)[4],
                                           const uint32_t (&roff)[4], const float (&Mu)[4],
                                           float (&L)[4], float (&acc)[4][16], RunOf&& run_of,
                                           SeqA&& seq_a) {
#pragma unroll 1
  for (int f = fs; f < fe; f += NU) {
    uint4 x[NU][NK][2];
    float w[NU][NK];
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      const int fu = min(f + u, fe - 1);
      bool live;
      const uint32_t base = run_of(fu, live);
      live = live && f + u < fe;
      const bool inA = seq_a(fu);
      const float* ml = reinterpret_cast<const float*>(smem + kCombMl + 512 * (fu - fs));
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        const uint4* row = reinterpret_cast<const uint4*>(smem + kSmemQ + base + roff[k]);
        x[u][k][0] = row[0];
        x[u][k][1] = row[1];
        const float mi = ml[hrow[k]], li = ml[64 + hrow[k]];
        // the partial row is normalised: its weight carries its sum l
        const bool mine = live && rowA[k] == inA;
        w[u][k] = (mine && mi != -INFINITY) ? li * ex2_approx(mi - Mu[k]) : 0.f;
        if (!mine) {  // not this row's data (or never copied): may hold anything
          x[u][k][0] = make_uint4(0u, 0u, 0u, 0u);
          x[u][k][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    // lane l: rows 4l + t (t = 0..3) of the [128][4] layout, i.e. value
    // columns 128c + 4l + t, in words (t, c = 0|1) and (t, c = 2|3)
#pragma unroll
    for (int k = 0; k < NK; ++k) {
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        L[k] += w[u][k];
        const uint32_t wd[8] = {x[u][k][0].x, x[u][k][0].y, x[u][k][0].z, x[u][k][0].w,
                                x[u][k][1].x, x[u][k][1].y, x[u][k][1].z, x[u][k][1].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc[k][t] = fmaf(w[u][k], bf16lo_to_f32(wd[2 * t]), acc[k][t]);
          acc[k][4 + t] = fmaf(w[u][k], bf16hi_to_f32(wd[2 * t]), acc[k][4 + t]);
          acc[k][8 + t] = fmaf(w[u][k], bf16lo_to_f32(wd[2 * t + 1]), acc[k][8 + t]);
          acc[k][12 + t] = fmaf(w[u][k], bf16hi_to_f32(wd[2 * t + 1]), acc[k][12 + t]);
        }
      }
    }
  }
}

template <typename GridArrive, typename GridWait>
__device__ __forceinline__ void combine_cta(const Params& p, const long long* tiles, int grid,
                                            uint8_t* smem, uint32_t sbase, uint32_t bar_comb,
                                            volatile int* abort_flag, int warp, int lane,
                                            GridArrive&& grid_arrive, GridWait&& grid_wait) {
  const long long N = tiles[p.S];
  // CTA that owns global tile x: ceil((x + 1) * grid / N) - 1
  auto owner = [&](long long x) -> int {
    return static_cast<int>(div_nn((x + 1) * grid + N - 1, N)) - 1;
  };
  // With at least one tile per CTA every split is non-empty: the 64-bit
  // divisions of the general test are kept off the common path.
  const bool dense = N >= grid;
  auto nonempty = [&](int c) { return dense || div_nn(N * c, grid) < div_nn(N * (c + 1), grid); };
  auto seq = [&](int s, int h0, int nh) -> CombSeq {
    CombSeq q;
    q.s = s;
    q.h0 = h0;
    q.nh = nh;
    q.c0 = owner(tiles[s]);
    q.n = owner(tiles[s + 1] - 1) - q.c0 + 1;
    return q;
  };
  const long long R = static_cast<long long>(p.S) * kHeads;
  const long long r0 = div_nn(R * blockIdx.x, grid), r1 = div_nn(R * (blockIdx.x + 1), grid);
  grid_arrive();  // every CTA, exactly once
  bool waited = false;
  uint32_t nbatch = 0;
#pragma unroll 1
  for (long long g0 = r0; g0 < r1; g0 += kCombRows) {
    const int ng = static_cast<int>(min(r1 - g0, static_cast<long long>(kCombRows)));
    const int sA = static_cast<int>(g0 / kHeads);
    const int hA = static_cast<int>(g0 - static_cast<long long>(sA) * kHeads);
    const int nA = min(ng, kHeads - hA);
    const CombSeq A = seq(sA, hA, nA);
    const CombSeq B = (ng > nA) ? seq(sA + 1, 0, ng - nA) : CombSeq{sA + 1, 0, 0, 0, 0};
    const int nItems = A.n + B.n;
    const uint32_t szA = static_cast<uint32_t>(A.nh) * kDim * 2;
    const uint32_t szB = static_cast<uint32_t>(B.nh) * kDim * 2;

    // this warp's rows: merge state and sigmoid(g)
    float M[4], L[4], acc[4][16];
    uint32_t sg[4][8];
    {
      // all gate loads first (rows past the group re-read its last row)
      uint2 gv[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = min(warp + 7 * k, ng - 1);
        const uint2* gp = reinterpret_cast<const uint2*>(
            p.g + static_cast<size_t>(g0 + i) * kDim + 4 * lane);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) gv[k][q4] = __ldg(gp + 32 * q4);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        M[k] = -INFINITY;
        L[k] = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          acc[k][4 * q4 + 0] = acc[k][4 * q4 + 1] = acc[k][4 * q4 + 2] = acc[k][4 * q4 + 3] = 0.f;
          sg[k][2 * q4] = pack_f16x2(sigmoid_fast(bf16lo_to_f32(gv[k][q4].x)),
                                     sigmoid_fast(bf16hi_to_f32(gv[k][q4].x)));
          sg[k][2 * q4 + 1] = pack_f16x2(sigmoid_fast(bf16lo_to_f32(gv[k][q4].y)),
                                         sigmoid_fast(bf16hi_to_f32(gv[k][q4].y)));
        }
      }
    }

#pragma unroll 1
    for (int fs = 0; fs < nItems;) {
      // batch [fs, fe): at most kCombItems runs and kCombData bytes
      int fe = fs;
      uint32_t bytes = 0;
      while (fe < nItems && fe - fs < kCombItems) {
        const uint32_t sz = fe < A.n ? szA : szB;
        if (bytes + sz > static_cast<uint32_t>(kCombData)) break;
        bytes += sz;
        ++fe;
      }
      if (!waited) {
        grid_wait();  // every CTA's partials are written
        waited = true;
      }
      if (threadIdx.x == 0) {
        fence_proxy_async_smem();  // earlier generic reads of these buffers come first
        uint32_t tx = 0;
        for (int f = fs; f < fe; ++f) {
          const bool inA = f < A.n;
          if (nonempty(inA ? A.c0 + f : B.c0 + f - A.n)) tx += (inA ? szA : szB) + 512;
        }
        mbar_expect_tx(bar_comb, tx);
        uint32_t off = 0;
        for (int f = fs; f < fe; ++f) {
          const bool inA = f < A.n;
          const CombSeq& q = inA ? A : B;
          const int c = inA ? A.c0 + f : B.c0 + f - A.n;
          const uint32_t sz = inA ? szA : szB;
          if (nonempty(c)) {
            const size_t slot = static_cast<size_t>(c + q.s);
            const uint16_t* src = p.ws_o + (slot * kHeads + q.h0) * kDim;
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
                " [%0], [%1], %2, [%3];" ::"r"(sbase + kSmemQ + off),
                "l"(src), "r"(sz), "r"(bar_comb)
                : "memory");
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
                " [%0], [%1], %2, [%3];" ::"r"(sbase + kCombMl + 512u * (f - fs)),
                "l"(p.ws_ml + slot * 128), "r"(512u), "r"(bar_comb)
                : "memory");
          }
          off += sz;
        }
      }
      if (!mbar_wait_warp(bar_comb, nbatch & 1, abort_flag, kWaitLimitNs, 71)) {
        if (lane == 0) abort_drain(abort_flag);   // this batch's copies may still land
        return;
      }
      ++nbatch;
      const int nAb = max(0, min(fe, A.n) - fs);  // runs of sequence A in this batch
      // Per row: the batch's largest m first (lane u reads split fs + u, then a
      // warp max), one rescale of the running sum, then one weight per split.
      float Mb[4];
      {
        const int f = fs + lane;
        const bool inA = f < A.n;
        const bool have = f < fe && nonempty(inA ? A.c0 + f : B.c0 + f - A.n);
        const float* ml = reinterpret_cast<const float*>(smem + kCombMl + 512 * lane);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = warp + 7 * k;
          const bool rowA = i < A.nh;
          const int h = (rowA ? A.h0 + i : i - A.nh) & 63;
          float m = (have && rowA == inA) ? ml[h] : -INFINITY;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          Mb[k] = fmaxf(M[k], m);
        }
      }
      float Mu[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        Mu[k] = (Mb[k] == -INFINITY) ? 0.f : Mb[k];
        const float sc = (M[k] == -INFINITY) ? 0.f : ex2_approx(M[k] - Mu[k]);
        L[k] *= sc;
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[k][t] *= sc;
        M[k] = Mb[k];
      }
      // The warp's rows (k < nk) with a loop specialised to their count, so
      // that no read is spent on a row past the group and a single row still
      // has several runs in flight.
      bool rowA[4];
      int hrow[4];
      uint32_t roff[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = min(warp + 7 * k, ng - 1);
        rowA[k] = i < A.nh;
        const int r = rowA[k] ? i : i - A.nh;
        hrow[k] = (rowA[k] ? A.h0 : B.h0) + r;
        roff[k] = static_cast<uint32_t>(r) * kDim * 2 + 32u * lane;
      }
      auto run_of = [&](int f, bool& live) -> uint32_t {
        const bool inA = f < A.n;
        live = nonempty(inA ? A.c0 + f : B.c0 + f - A.n);
        return inA ? static_cast<uint32_t>(f - fs) * szA
                   : static_cast<uint32_t>(nAb) * szA +
                         static_cast<uint32_t>(f - max(fs, A.n)) * szB;
      };
      auto seq_a = [&](int f) { return f < A.n; };
      const int nk = ng > warp ? min(4, (ng - warp + 6) / 7) : 0;
      if (nk == 4)
        merge_runs<4, 1>(smem, fs, fe, rowA, hrow, roff, Mu, L, acc, run_of, seq_a);
      else if (nk == 3)
        merge_runs<3, 1>(smem, fs, fe, rowA, hrow, roff, Mu, L, acc, run_of, seq_a);
      else if (nk == 2)
        merge_runs<2, 2>(smem, fs, fe, rowA, hrow, roff, Mu, L, acc, run_of, seq_a);
      else if (nk == 1)
        merge_runs<1, 4>(smem, fs, fe, rowA, hrow, roff, Mu, L, acc, run_of, seq_a);
      __syncthreads();  // the next batch overwrites the buffers
      fs = fe;
    }

    // normalise, gate, store
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = warp + 7 * k;
      if (i >= ng) continue;
      const float inv = 1.f / L[k];
      uint2* op = reinterpret_cast<uint2*>(p.out + static_cast<size_t>(g0 + i) * kDim + 4 * lane);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float* a = &acc[k][4 * q4];
        const uint32_t e01 = sg[k][2 * q4], e23 = sg[k][2 * q4 + 1];
        op[32 * q4] = make_uint2(
            pack_bf16x2(a[0] * inv * f16lo_to_f32(e01), a[1] * inv * f16hi_to_f32(e01)),
            pack_bf16x2(a[2] * inv * f16lo_to_f32(e23), a[3] * inv * f16hi_to_f32(e23)));
      }
    }
  }
}

// Four e4m3 codes (one word, lowest address in the low byte) -> four f16
// values, exactly, with integer operations.  Each code moves into its own
// 16-bit lane shifted left by 7: its exponent and mantissa bits then sit where
// f16 keeps them (the f16 value is 2^-8 times the code's value; e4m3
// subnormals land on f16 subnormals); its sign bit, now at bit 14, moves to
// bit 15 by adding bit 14 to itself (no carry leaves the lane); one f16x2
// multiply by 2^8 restores the value.
__device__ __forceinline__ uint32_t mul_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t a = __byte_perm(w, 0u, 0x4140) << 7;   // codes 0, 1
  const uint32_t b = __byte_perm(w, 0u, 0x4342) << 7;   // codes 2, 3
  lo = mul_f16x2(a + (a & 0x40004000u), 0x5C005C00u);   // x 256 (f16 0x5C00)
  hi = mul_f16x2(b + (b & 0x40004000u), 0x5C005C00u);
}
// a bf16 pair -> an f16 pair (exact for |x| < 65504 with at most 11 significant bits)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return pack_f16x2(bf16lo_to_f32(w), bf16hi_to_f32(w));
}

// ---------------------------------------------------------------------------
// Virtual head attention ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1, VHA):
// after every CTA's combined rows are in `out` (a second grid barrier), the
// warps mix the 64 heads of each sequence in place, y = x + up (down^T x).
// A warp takes 8 value columns of one sequence: the [64 heads][8] tile comes
// into its own 1 KB of shared memory with two 16-byte loads per lane; lane
// (c, q) then holds column c of heads q, q + 4, .., q + 60, forms its part of
// the rank sums z = down^T x 8 ranks at a time, completes them with two
// shuffles across the four lanes of its column, and adds up z to its 16
// accumulators; the tile leaves with 16-byte stores.  Short dependency chains
// and a small loop body: this code runs once per launch on every warp.  The
// factors sit in shared memory as fp32, padded with zeros to a multiple of 8
// ranks.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int vha_rank8(const Params& p) { return (p.vha_rank + 7) & ~7; }

__device__ __forceinline__ void vha_load_factors(const Params& p, float* fd, float* fu) {
  const int r = p.vha_rank, r8 = vha_rank8(p);
  for (int i = threadIdx.x; i < kHeads * r8; i += kThreads) {
    const int h = i / r8, rr = i - h * r8;
    const bool in = rr < r;
    fd[i] = in ? __uint_as_float(static_cast<uint32_t>(p.vha_down[h * r + rr]) << 16) : 0.f;
    fu[i] = in ? __uint_as_float(static_cast<uint32_t>(p.vha_up[h * r + rr]) << 16) : 0.f;
  }
}

__device__ __forceinline__ void vha_mix_columns(const Params& p, const float* fd, const float* fu,
                                                uint16_t* tile, int warp, int lane) {
  const int r8 = vha_rank8(p);
  const int wpc = kThreads / 32;
  const int units = p.S * (kDim / 8);
  const int c = lane & 7, q = lane >> 3;   // this lane: column c, heads q + 4 i (i < 16)
#pragma unroll 1
  for (int un = blockIdx.x * wpc + warp; un < units; un += gridDim.x * wpc) {
    // written by other CTAs in this launch: plain loads (the barrier acquired them)
    uint16_t* src = p.out + static_cast<size_t>(un >> 6) * kHeads * kDim + 8 * (un & 63);
    const uint4 a = *reinterpret_cast<const uint4*>(src + lane * kDim);
    const uint4 b = *reinterpret_cast<const uint4*>(src + (lane + 32) * kDim);
    *reinterpret_cast<uint4*>(tile + 8 * lane) = a;
    *reinterpret_cast<uint4*>(tile + 8 * (lane + 32)) = b;
    __syncwarp();
    float x[16], y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      x[i] = __uint_as_float(static_cast<uint32_t>(tile[(q + 4 * i) * 8 + c]) << 16);
      y[i] = x[i];
    }
#pragma unroll 1
    for (int r0 = 0; r0 < r8; r0 += 8) {
      float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 16; ++i) {     // this lane's 16 heads of z = down^T x
        const float* f = fd + (q + 4 * i) * r8 + r0;
        const float4 fa = *reinterpret_cast<const float4*>(f);
        const float4 fb = *reinterpret_cast<const float4*>(f + 4);
        z[0] = fmaf(fa.x, x[i], z[0]);
        z[1] = fmaf(fa.y, x[i], z[1]);
        z[2] = fmaf(fa.z, x[i], z[2]);
        z[3] = fmaf(fa.w, x[i], z[3]);
        z[4] = fmaf(fb.x, x[i], z[4]);
        z[5] = fmaf(fb.y, x[i], z[5]);
        z[6] = fmaf(fb.z, x[i], z[6]);
        z[7] = fmaf(fb.w, x[i], z[7]);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {      // all 64 heads: the four lanes of column c
        z[j] += __shfl_xor_sync(0xffffffffu, z[j], 8);
        z[j] += __shfl_xor_sync(0xffffffffu, z[j], 16);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {     // y += up z
        const float* f = fu + (q + 4 * i) * r8 + r0;
        const float4 fa = *reinterpret_cast<const float4*>(f);
        const float4 fb = *reinterpret_cast<const float4*>(f + 4);
        float t = y[i];
        t = fmaf(fa.x, z[0], t);
        t = fmaf(fa.y, z[1], t);
        t = fmaf(fa.z, z[2], t);
        t = fmaf(fa.w, z[3], t);
        t = fmaf(fb.x, z[4], t);
        t = fmaf(fb.y, z[5], t);
        t = fmaf(fb.z, z[6], t);
        y[i] = fmaf(fb.w, z[7], t);
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 16; ++i)
      tile[(q + 4 * i) * 8 + c] = static_cast<uint16_t>(pack_bf16x2(y[i], 0.f) & 0xFFFFu);
    __syncwarp();
    *reinterpret_cast<uint4*>(src + lane * kDim) = *reinterpret_cast<const uint4*>(tile + 8 * lane);
    *reinterpret_cast<uint4*>(src + (lane + 32) * kDim) =
        *reinterpret_cast<const uint4*>(tile + 8 * (lane + 32));
    __syncwarp();   // the next unit overwrites the tile
  }
}

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ Maps maps, const Params p) {
  constexpr int NS = kF8 ? kStagesF8 : kStages;   // ring stages
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, derived from smem_raw itself so that the compiler
  // keeps accesses through it in the shared state space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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
  // Set-up that needs no plan first, so that it overlaps the plan's loads:
  // barriers, tensor-map prefetch, TMEM.
  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    if (kF8) {
      for (int s = 0; s < 4; ++s) mbar_init(bar(B_STG + s), 1);
      mbar_init(bar(B_QCONV), 4);   // one arrive per softmax warp
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
    mbar_init(bar(B_COMB), 1);
    *abort_flag = 0;
    fence_mbar_init();
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
  // Tile prefix and context lengths: planned here for up to kInlineSeqs
  // sequences, else by the plan kernel, which may still be running
  // (programmatic dependent launch): wait for it.  Either way a CTA barrier
  // follows, which also publishes the set-up above.
  const bool inl = p.S <= kInlineSeqs;
  long long* sT = reinterpret_cast<long long*>(smem + kSmemTiles);
  int* sL = reinterpret_cast<int*>(smem + kSmemCtx);
  if (inl) {
    inline_plan(p, sT, sL);
  } else {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long* tiles = inl ? sT : p.seq_tile;
  const int* lens = inl ? sL : p.ctx_len;
  const long long N = tiles[p.S];
  const long long A0 = div_nn(N * blockIdx.x, gridDim.x);
  const long long A1 = div_nn(N * (blockIdx.x + 1), gridDim.x);
  if (A0 < A1) {  // uniform across the CTA; a CTA without tiles only helps combine

  // Segments: maximal runs of this CTA's tiles inside one sequence.
  const int s_first = find_seq(tiles, p.S, A0);

  if (warp <= 1 && kF8) {
    // ------------------------------------------------------------ producers, FP8 cache
    // Each warp loads the code tiles of its ring uses (alternate uses, as
    // below) into its two staging slots, keeping up to two in flight, and
    // converts each landed tile into its ring stage with all 32 lanes.
    const int me = warp;
    const uint32_t sStg = sbase + kSmemStg;
    uint32_t u = 0, quse = 0, nown = 0, first = 0, npend = 0;
    bool ok = true;
    // convert this warp's oldest pending use (own use index `first`)
    auto convert_oldest = [&]() -> bool {
      const uint32_t slot = first & 1;
      const uint32_t uu = 2 * first + static_cast<uint32_t>(me);
      const uint32_t st = uu % NS;
      bool w_ok = true;
      if (lane == 0)
        w_ok = mbar_wait(bar(B_STG + 2 * me + slot), (first >> 1) & 1, abort_flag, kWaitLimitNs,
                         42) &&
               mbar_wait(bar(B_EMPTY + st), ((uu / NS) & 1) ^ 1, abort_flag, kWaitLimitNs, 40);
      w_ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0;
      if (!w_ok) return false;
      mbar_try_wait(bar(B_STG + 2 * me + slot), (first >> 1) & 1);   // this lane's acquire
      const uint8_t* src = smem + kSmemStg + (2 * me + slot) * kStgBytes;
      uint8_t* dst = smem + kSmemRing + st * kStage;
      // 16-byte source chunk ci (16 codes): key row ci / 8, bytes 16 (ci % 8) of
      // the 128-channel row, i.e. slab (ci % 8) / 4 and 16-byte output chunks
      // 2 (ci % 4) and 2 (ci % 4) + 1 of that slab's row
#pragma unroll 2
      for (int it = 0; it < 32; ++it) {
        const int ci = it * 32 + lane;
        const int row = ci >> 3, sl = (ci >> 2) & 1, c = (ci & 3) * 2;
        const uint4 x = *reinterpret_cast<const uint4*>(src + ci * 16);
        uint32_t f[8];
        e4m3x4_to_f16x4(x.x, f[0], f[1]);
        e4m3x4_to_f16x4(x.y, f[2], f[3]);
        e4m3x4_to_f16x4(x.z, f[4], f[5]);
        e4m3x4_to_f16x4(x.w, f[6], f[7]);
        uint8_t* drow = dst + sl * kSlab;
        *reinterpret_cast<uint4*>(drow + sw128_offset(row, c)) = make_uint4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<uint4*>(drow + sw128_offset(row, c + 1)) =
            make_uint4(f[4], f[5], f[6], f[7]);
      }
      fence_proxy_async_smem();   // read next by the tensor core (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_FULL + st));
      ++first;
      --npend;
      return true;
    };
    // code tile (channels [64 z, 64 z + 128), rows y..y+127) of use u
    auto load = [&](const CUtensorMap* map, int y, int z, int w) -> bool {
      if ((u & 1) == static_cast<uint32_t>(me)) {
        if (npend == 2 && !convert_oldest()) return false;
        const uint32_t slot = nown & 1;
        if (lane == 0) {
          mbar_expect_tx(bar(B_STG + 2 * me + slot), kStgBytes);
          tma_load_3d(sStg + (2 * me + slot) * kStgBytes, map, bar(B_STG + 2 * me + slot), 64 * z,
                      y, w);
        }
        ++nown;
        ++npend;
      }
      ++u;
      return true;
    };
    long long x = A0;
    for (int s = s_first; x < A1 && ok; ++s) {
      const SeqInfo si = seq_info(lens, p.max_nc, s);
      const long long seg_end = min(A1, tiles[s + 1]);
      const int j0 = static_cast<int>(x - tiles[s]);
      const int j1 = static_cast<int>(seg_end - tiles[s]);
      if (me == 0) {
        if (lane == 0) {
          ok = mbar_wait(bar(B_QEMPTY), (quse & 1) ^ 1, abort_flag, kWaitLimitNs, 41);
          if (ok) {
            mbar_expect_tx(bar(B_QFULL), 8 * kQSlab);
            tma_load_4d_dec(sQ, &maps.q, bar(B_QFULL), 0, s * kHeads, 0, 0);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
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
    while (ok && npend > 0) ok = convert_oldest();
    if (me == 0 && lane == 0) {
      const long long R = static_cast<long long>(p.S) * kHeads;
      const long long r0 = div_nn(R * blockIdx.x, gridDim.x);
      const long long r1 = div_nn(R * (blockIdx.x + 1), gridDim.x);
      if (r1 > r0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.g + r0 * kDim),
                     "r"(static_cast<uint32_t>(r1 - r0) * kDim * 2)
                     : "memory");
    }
  } else if (warp <= 1) {
    // ------------------------------------------------------------ producers
    // Two warps alternate ring stages: one issuing thread cannot keep enough
    // copies in flight to cover HBM latency.
    if (lane == 0) {
      const int me = warp;
      uint32_t u = 0, quse = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int y, int z, int w) -> bool {
        if ((u & 1) == static_cast<uint32_t>(me)) {
          const uint32_t st = u % NS;
          if (!mbar_wait(bar(B_EMPTY + st), ((u / NS) & 1) ^ 1, abort_flag, kWaitLimitNs, 40))
            return false;
          mbar_expect_tx(bar(B_FULL + st), kStage);
          tma_load_4d_dec(sRing + st * kStage, map, bar(B_FULL + st), 0, y, z, w);
        }
        ++u;
        return true;
      };
      long long x = A0;
      for (int s = s_first; x < A1 && ok; ++s) {
        const SeqInfo si = seq_info(lens, p.max_nc, s);
        const long long seg_end = min(A1, tiles[s + 1]);
        const int j0 = static_cast<int>(x - tiles[s]);
        const int j1 = static_cast<int>(seg_end - tiles[s]);
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
      // The last copies are out: bring the gate rows this CTA combines into
      // L2 while its final tiles are processed.
      if (me == 0) {
        const long long R = static_cast<long long>(p.S) * kHeads;
        const long long r0 = div_nn(R * blockIdx.x, gridDim.x);
        const long long r1 = div_nn(R * (blockIdx.x + 1), gridDim.x);
        if (r1 > r0)
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.g + r0 * kDim),
                       "r"(static_cast<uint32_t>(r1 - r0) * kDim * 2)
                       : "memory");
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t ring = 0, quse = 0, sidx = 0, pvidx = 0, nseg = 0;
      bool ok = true;
      const uint32_t idesc_s = kF8 ? idesc_f16_f32(128, 64, false, false)
                                   : idesc_bf16_f32(128, 64, false, false);
      const uint32_t idesc_o = kF8 ? idesc_f16_f32(128, 64, true, true)
                                   : idesc_bf16_f32(128, 64, true, true);
      auto issue_s = [&]() -> bool {
        const uint32_t buf = sidx & 1;
        if (!mbar_wait(bar(B_SFREE + buf), ((sidx >> 1) & 1) ^ 1, abort_flag, kWaitLimitNs, 50))
          return false;
        tc_fence_after();
        const uint32_t dS = tmem + (buf ? kTmemS1 : kTmemS0);
        for (int d2 = 0; d2 < 4; ++d2) {
          const uint32_t st = ring % NS;
          if (!mbar_wait(bar(B_FULL + st), (ring / NS) & 1, abort_flag, kWaitLimitNs, 51))
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
          const uint32_t st = ring % NS;
          if (!mbar_wait(bar(B_FULL + st), (ring / NS) & 1, abort_flag, kWaitLimitNs, 54))
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
        const long long seg_end = min(A1, tiles[s + 1]);
        const int ntl = static_cast<int>(seg_end - x);
        // FP8 cache: Q once the softmax warps turned it into f16
        ok = mbar_wait(bar(kF8 ? B_QCONV : B_QFULL), quse & 1, abort_flag, kWaitLimitNs, 56);
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
      const SeqInfo si = seq_info(lens, p.max_nc, s);
      const long long seg_end = min(A1, tiles[s + 1]);
      const int j0 = static_cast<int>(x - tiles[s]);
      const int j1 = static_cast<int>(seg_end - tiles[s]);
      if (tid < 64) {
        red[R_MRUN + tid] = -INFINITY;
        red[R_LRUN + tid] = 0.f;
      }
      if constexpr (kF8) {
        // this segment's Q, bf16 -> f16 in place (same byte positions), for the MMA
        if (!group_wait(bar(B_QFULL), nseg & 1, 63)) { ok = false; break; }
        uint4* qa = reinterpret_cast<uint4*>(smem + kSmemQ);
#pragma unroll 4
        for (int i = 0; i < 8 * kQSlab / 16 / 128; ++i) {
          uint4 w = qa[i * 128 + tid];
          w = make_uint4(bf16x2_to_f16x2(w.x), bf16x2_to_f16x2(w.y), bf16x2_to_f16x2(w.z),
                         bf16x2_to_f16x2(w.w));
          qa[i * 128 + tid] = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_QCONV));
      }
      for (int j = j0; j < j1; ++j) {
        const uint32_t buf = sidx & 1;
        // FP8 cache: this key's row scales (loaded before the wait)
        float sk = 1.f, sv = 1.f;
        if constexpr (kF8) {
          const bool comp = j < si.nct;
          const int e = j * kKeyTile + key;
          if (comp ? e < si.nc : ((si.L >= kWin) || (key < si.L))) {
            const size_t ix = comp ? static_cast<size_t>(s) * p.max_nc + e
                                   : static_cast<size_t>(s) * kWin + key;
            sk = __ldg((comp ? p.sck : p.swk) + ix);
            sv = __ldg((comp ? p.scv : p.swv) + ix);
          }
        }
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
        const float sc = p.scale_log2 * sk;
#pragma unroll
        for (int h = 0; h < 64; ++h) a[h] = valid ? __uint_as_float(r[h]) * sc : -INFINITY;
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
          // FP8 cache: the key's V scale rides on its probabilities (f16 P)
          pk[h / 2] = kF8 ? pack_f16x2(e0 * sv, e1 * sv) : pack_bf16x2(e0, e1);
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
      // O^T / l in bf16: this thread holds value columns 128c + key (c = 0..3)
      // and writes them as one 8-byte word per head.
      if (!group_wait(bar(B_OFULL), nseg & 1, 62)) { ok = false; break; }
      tc_fence_after();
      if (tid < 64) {
        const float l = red[R_LRUN + tid];
        red[R_ALPHA + tid] = l > 0.f ? 1.f / l : 0.f;
      }
      named_bar_sync(1, 128);
      const int slot = blockIdx.x + s;
      uint2* wo = reinterpret_cast<uint2*>(p.ws_o + static_cast<size_t>(slot) * kHeads * kDim) + key;
#pragma unroll 1
      for (int hh = 0; hh < 64; hh += 16) {
        uint32_t o[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(tl + kTmemO + 64 * c + hh, o + 16 * c);
        tmem_wait_ld_dep32(o);
        reg_dep32(o + 32);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float inv = red[R_ALPHA + hh + i];
          wo[(hh + i) * kKeyTile] =
              make_uint2(pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[16 + i]) * inv),
                         pack_bf16x2(__uint_as_float(o[32 + i]) * inv,
                                     __uint_as_float(o[48 + i]) * inv));
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

  }  // A0 < A1
  if (threadIdx.x == 0) abort_drain(abort_flag);
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  // ---------------------------------------------------------------- combine
  // Grid barrier (the launch is cooperative: every CTA is resident), then the
  // CTAs merge the partials of their share of the (sequence, head) rows.
  // The partials are read back by bulk copies (the async proxy): every writer
  // orders its generic stores before them.
  // The arrival counter is never reset: every barrier adds exactly gridDim.x
  // (each CTA arrives once, on every path; a launch with the head mix holds
  // two barriers, and every CTA waits for the first to complete before it
  // arrives at the second -- also a CTA that had no rows to combine and so
  // never needed the first), so a barrier's arrivals fill the window
  // [k G, (k + 1) G) that the counter's value at its first arrival falls in,
  // and the barrier is complete when the counter reaches (k + 1) G.
  // It starts at zero (the workspace is zero-filled before first use) and is
  // 64-bit, so it does not wrap.
  __shared__ unsigned long long bar_target;
  __shared__ int bar_done;
  auto grid_arrive = [&]() {
    fence_proxy_async_all();
    __syncthreads();
    if (threadIdx.x == 0) {
      // acq_rel: releases this CTA's partials (ordered before it by the CTA
      // barrier above); the last arrival also acquires everybody else's and
      // so needs no polling
      const unsigned long long G = gridDim.x;
      unsigned long long old;
      asm volatile("atom.add.acq_rel.gpu.global.u64 %0, [%1], 1;"
                   : "=l"(old)
                   : "l"(p.gsync)
                   : "memory");
      bar_target = (old / G + 1) * G;
      bar_done = (old + 1 == bar_target) ? 1 : 0;
    }
  };
  auto grid_wait = [&]() {
    if (threadIdx.x == 0 && !bar_done) {
      const uint64_t t0 = globaltimer_ns();
      for (uint32_t i = 1;; ++i) {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p.gsync) : "memory");
        if (v >= bar_target) break;
        if ((i & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
          record_error(DEVERR_TIMEOUT, 70);
          break;
        }
      }
    }
    if (threadIdx.x == 0) fence_proxy_async_all();
    __syncthreads();
  };
  combine_cta(p, tiles, gridDim.x, smem, sbase, bar(B_COMB), abort_flag, warp, lane,
              grid_arrive, grid_wait);
  if (!kF8 && p.vha_rank > 0) {
    // the combine's buffers are free once every warp is here
    float* fd = reinterpret_cast<float*>(smem + kSmemQ);   // [64][r8]
    float* fu = fd + kHeads * kHeads;                       // [64][r8]
    uint16_t* tiles = reinterpret_cast<uint16_t*>(fu + kHeads * kHeads);   // 1 KB per warp
    __syncthreads();
    grid_wait();    // the first barrier is complete (a no-op if combining waited for it)
    vha_load_factors(p, fd, fu);
    grid_arrive();  // this CTA's rows of out are written (second barrier of the launch)
    grid_wait();
    vha_mix_columns(p, fd, fu, tiles + warp * kHeads * 8, warp, lane);
  }
}

// ---------------------------------------------------------------------------
}  // namespace decode
}  // namespace hca
