// libhca.so: the C ABI declared in include/hca.h.
//
// Host-side work only: argument validation, TMA tensor-map encoding, grid
// sizing and launches.  Every step of the computation runs in the kernels
// included below.  One translation unit, so the device-side error word is a
// single symbol shared by all kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "../../include/hca.h"
#include "hca_ptx.cuh"
#include "compress.cuh"
#include "prefill3.cuh"
#include "decode.cuh"
#include "append.cuh"
#include "backward.cuh"
#include "quant.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D bf16 tensor [Z][Y][X] (X contiguous, X = 512), box (64, box_y, 1),
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t X, uint64_t Y, uint64_t Z,
              uint32_t box_y) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {X, Y, Z};
  const cuuint64_t strides[2] = {X * 2, X * Y * 2};
  const cuuint32_t box[3] = {64, box_y, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view (64, Y, 8, W) of a [W][Y][512] bf16 tensor: x = element inside a
// 64-wide column slab, y = row, z = slab index, w = batch.  A box
// (64, box_y, box_z, 1) lands in shared memory as box_z slabs of
// [box_y rows][64], each 128B-swizzled.
bool make_map4(CUtensorMap* m, const void* base, uint64_t Y, uint64_t W, uint32_t box_y,
               uint32_t box_z) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {64, Y, 8, W};
  const cuuint64_t strides[3] = {1024, 128, Y * 1024};
  const cuuint32_t box[4] = {64, box_y, box_z, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

// 2-D byte view [rows][256] of a buffer, box (256, box_rows), no swizzle:
// moves contiguous 256-byte rows.
bool make_map_bytes(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {256, rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D byte view [Z][Y][512] of e4m3 code rows, box (128 bytes, 128 rows, 1),
// no swizzle: one 128-channel, 128-key code tile.
bool make_map_codes(CUtensorMap* m, const void* base, uint64_t Y, uint64_t Z) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {512, Y, Z};
  const cuuint64_t strides[2] = {512, 512 * Y};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// How many 4-CTA clusters of the prefill kernel fit on the current device at
// once (the smaller answer of its two variants, which share their launch
// shape).  The shared-memory attribute is a per-device property of each
// kernel, so it is set, and the occupancy asked, once for every device the
// process uses (with that device current).
int prefill_max_clusters() {
  static int cached[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] > 0) return cached[dev];
  namespace P = hca::prefill3;
  if (cudaFuncSetAttribute(P::prefill3_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           P::kSmemAlloc) != cudaSuccess ||
      cudaFuncSetAttribute(P::prefill3_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           P::kSmemAlloc) != cudaSuccess)
    return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4, 1, 1);
  cfg.blockDim = dim3(P::kThreads, 1, 1);
  cfg.dynamicSmemBytes = P::kSmemAlloc;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 4;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0, nv = 0;
  if (cudaOccupancyMaxActiveClusters(&n, P::prefill3_kernel<false>, &cfg) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&nv, P::prefill3_kernel<true>, &cfg) != cudaSuccess)
    return -1;
  n = n < nv ? n : nv;
  if (n <= 0) return -1;
  cached[dev] = n;
  return n;
}

// The decode pass: for more than kInlineSeqs sequences the plan kernel first
// (the decode kernel then starts early and waits for it inside), else the
// decode kernel alone, which plans for itself.  Cooperative either way: the
// kernel holds a grid barrier.
template <bool kF8>
cudaError_t launch_decode(const hca::decode::Maps& maps, const hca::decode::Params& prm, int grid,
                          cudaStream_t stream) {
  namespace D = hca::decode;
  cudaError_t err = cudaFuncSetAttribute(D::decode_kernel<kF8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, D::kSmemAlloc);
  if (err != cudaSuccess) return err;
  const bool inl = prm.S <= D::kInlineSeqs;
  if (!inl) {
    D::plan_kernel<<<1, 1024, 0, stream>>>(prm.ctx_len, prm.S, prm.max_nc, prm.seq_tile);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(D::kThreads);
  cfg.dynamicSmemBytes = D::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = inl ? 1 : 2;
  return cudaLaunchKernelEx(&cfg, D::decode_kernel<kF8>, maps, prm);
}

hca_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? HCA_OK : HCA_ERR_CUDA;
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return sms;
}

bool scale_ok(float scale) { return std::isfinite(scale) && scale > 0.f; }

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar_storage;
  __shared__ int abort_flag;
  const uint32_t b = hca::smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    hca::mbar_init(b, 1);
    abort_flag = 0;
    hca::fence_mbar_init();
  }
  __syncthreads();
  // Nobody arrives: the wait must give up after limit_ns and record a timeout.
  hca::mbar_wait(b, 0, &abort_flag, limit_ns, 900);
}

}  // namespace

extern "C" {

hca_status_t hca_compress(const hca_bf16* k, const hca_bf16* v, const hca_bf16* s, int B, int T,
                          hca_bf16* ck, hca_bf16* cv, hca_stream_t stream) {
  if (B < 1 || T < 1 || k == nullptr || v == nullptr || s == nullptr) return HCA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return HCA_ERR_INVALID_ARG;
  const int nb = T / HCA_BLOCK;
  if (nb == 0) return HCA_OK;
  if (ck == nullptr || cv == nullptr) return HCA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * nb > 0x7fffffffLL) return HCA_ERR_UNSUPPORTED;
  dim3 grid(B * nb, 8);
  hca::compress_kernel<<<grid, hca::kCompressThreads, 0, stream>>>(k, v, s, T, nb, ck, cv);
  return launch_status();
}

size_t hca_prefill_workspace_size(int B, int T) {
  if (B < 1 || T < 1) return 0;
  const long long items = static_cast<long long>(B) * ((T + 3) / 4);
  const int max_clusters = prefill_max_clusters();
  if (max_clusters <= 0) return 0;
  const long long clusters = items < max_clusters ? items : max_clusters;
  return static_cast<size_t>(clusters) * hca::prefill3::kScratchPerCluster + 256;
}

namespace {
// hca_prefill_fwd and hca_prefill_fwd_vha (vha_rank = 0: no head mix)
hca_status_t prefill_impl(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                          const hca_bf16* ck, const hca_bf16* cv, const hca_bf16* g, int B, int T,
                          int H, float scale, const hca_bf16* vha_down, const hca_bf16* vha_up,
                          int vha_rank, hca_bf16* out, float* lse, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  namespace P = hca::prefill3;
  if (H != HCA_NUM_HEADS) return HCA_ERR_UNSUPPORTED;
  if (B < 1 || T < 1 || !scale_ok(scale)) return HCA_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || g == nullptr || out == nullptr ||
      ws == nullptr)
    return HCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return HCA_ERR_INVALID_ARG;
  const int nb = T / HCA_BLOCK;
  if (nb > 0 && (ck == nullptr || cv == nullptr)) return HCA_ERR_INVALID_ARG;
  const void* ptrs[7] = {q, k, v, g, out, ck, cv};
  for (const void* ptr : ptrs)
    if (ptr != nullptr && !aligned16(ptr)) return HCA_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * HCA_NUM_HEADS > 0x7fffffffLL) return HCA_ERR_UNSUPPORTED;
  const long long row_tiles = (T + 3) / 4;
  const long long items = static_cast<long long>(B) * row_tiles;
  if (items > 0x7fffffffLL) return HCA_ERR_UNSUPPORTED;

  const int max_clusters = prefill_max_clusters();
  if (max_clusters <= 0) return HCA_ERR_CUDA;
  const int clusters = static_cast<int>(items < max_clusters ? items : max_clusters);
  if (ws_bytes < static_cast<size_t>(clusters) * P::kScratchPerCluster) return HCA_ERR_INVALID_ARG;

  P::Maps maps;
  const uint64_t rows = static_cast<uint64_t>(T) * HCA_NUM_HEADS;
  const uint64_t prows = static_cast<uint64_t>(clusters) * P::kScratchPerCluster / 256;
  bool ok = make_map4(&maps.q4, q, rows, B, 128, 4) && make_map4(&maps.g4, g, rows, B, 128, 2) &&
            make_map4(&maps.out4, out, rows, B, 128, 2) &&
            make_map(&maps.kwin, k, HCA_HEAD_DIM, T, B, P::kWinHalf) &&
            make_map4(&maps.v4, v, T, B, 128, 2) && make_map4(&maps.v4t, v, T, B, 16, 1) &&
            make_map_bytes(&maps.p128, ws, prows, 128) && make_map_bytes(&maps.p16, ws, prows, 16);
  if (ok && nb > 0) {
    ok = make_map(&maps.ck, ck, HCA_HEAD_DIM, nb, B, 64) && make_map4(&maps.cv4, cv, nb, B, 128, 2);
  } else if (ok) {  // no compressed entry exists; these maps are never used
    ok = make_map(&maps.ck, k, HCA_HEAD_DIM, T, B, 64) && make_map4(&maps.cv4, v, T, B, 128, 2);
  }
  if (!ok) return HCA_ERR_CUDA;

  P::Params prm = {};
  prm.B = B;
  prm.T = T;
  prm.row_tiles = static_cast<int>(row_tiles);
  prm.items = static_cast<int>(items);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.lse = lse;
  prm.pscratch = static_cast<uint8_t*>(ws);
  prm.vha_down = vha_down;
  prm.vha_up = vha_up;
  prm.vha_rank = vha_rank;
  if (vha_rank > 0)
    P::prefill3_kernel<true><<<4 * clusters, P::kThreads, P::kSmemAlloc, stream>>>(maps, prm);
  else
    P::prefill3_kernel<false><<<4 * clusters, P::kThreads, P::kSmemAlloc, stream>>>(maps, prm);
  return launch_status();
}
}  // namespace

hca_status_t hca_prefill_fwd(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                             const hca_bf16* ck, const hca_bf16* cv, const hca_bf16* g, int B,
                             int T, int H, float scale, hca_bf16* out, float* lse, void* ws,
                             size_t ws_bytes, hca_stream_t stream) {
  return prefill_impl(q, k, v, ck, cv, g, B, T, H, scale, nullptr, nullptr, 0, out, lse, ws,
                      ws_bytes, static_cast<cudaStream_t>(stream));
}

hca_status_t hca_prefill_fwd_vha(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                                 const hca_bf16* ck, const hca_bf16* cv, const hca_bf16* g,
                                 int B, int T, int H, float scale, const hca_bf16* vha_down,
                                 const hca_bf16* vha_up, int vha_rank, hca_bf16* out, float* lse,
                                 void* ws, size_t ws_bytes, hca_stream_t stream) {
  if (vha_rank < 1 || vha_rank > HCA_NUM_HEADS) return HCA_ERR_INVALID_ARG;
  if (vha_down == nullptr || vha_up == nullptr) return HCA_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, ck, cv, g, B, T, H, scale, vha_down, vha_up, vha_rank, out, lse,
                      ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t hca_decode_workspace_size(int S) {
  if (S < 1) return 0;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  const int slots = sms + S;
  // the grid barrier counter (256-byte block at offset 0), partial O and
  // (m, l) per slot, then the tile prefix [S + 1] int64
  return 256 + hca::decode::ws_bytes(slots) + 256 + static_cast<size_t>(S + 1) * 8;
}

}  // extern "C"

namespace {
// hca_decode and hca_decode_vha (vha_rank = 0: no head mix)
hca_status_t decode_impl(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv, int max_nc,
                         const hca_bf16* wk, const hca_bf16* wv, const int32_t* ctx_len,
                         const hca_bf16* g, int S, int H, float scale, const hca_bf16* vha_down,
                         const hca_bf16* vha_up, int vha_rank, void* ws, size_t ws_bytes,
                         hca_bf16* out, cudaStream_t stream) {
  namespace D = hca::decode;
  if (H != HCA_NUM_HEADS) return HCA_ERR_UNSUPPORTED;
  if (S < 1 || max_nc < 0 || !scale_ok(scale)) return HCA_ERR_INVALID_ARG;
  if (q == nullptr || wk == nullptr || wv == nullptr || ctx_len == nullptr || g == nullptr ||
      out == nullptr || ws == nullptr)
    return HCA_ERR_INVALID_ARG;
  if (max_nc > 0 && (ck == nullptr || cv == nullptr)) return HCA_ERR_INVALID_ARG;
  const void* ptrs[7] = {q, wk, wv, g, out, ck, cv};
  for (const void* ptr : ptrs)
    if (ptr != nullptr && !aligned16(ptr)) return HCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return HCA_ERR_INVALID_ARG;
  if (ws_bytes < hca_decode_workspace_size(S)) return HCA_ERR_INVALID_ARG;
  if (static_cast<long long>(S) * HCA_NUM_HEADS > 0x7fffffffLL || S > 65535)
    return HCA_ERR_UNSUPPORTED;

  const int sms = device_sms();
  if (sms <= 0) return HCA_ERR_CUDA;
  const int slots = sms + S;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  D::Params prm = {};
  prm.ctx_len = ctx_len;
  prm.S = S;
  prm.max_nc = max_nc;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.gsync = reinterpret_cast<unsigned long long*>(wsb);
  prm.ws_o = reinterpret_cast<uint16_t*>(wsb + 256);
  prm.ws_ml = reinterpret_cast<float*>(wsb + 256 + D::ws_o_bytes(slots));
  prm.seq_tile =
      reinterpret_cast<long long*>(wsb + 256 + ((D::ws_bytes(slots) + 255) & ~size_t(255)));
  prm.g = g;
  prm.out = out;
  prm.vha_down = vha_down;
  prm.vha_up = vha_up;
  prm.vha_rank = vha_rank;

  D::Maps maps;
  bool ok = make_map4(&maps.q, q, static_cast<uint64_t>(S) * HCA_NUM_HEADS, 1, 64, 8) &&
            make_map4(&maps.wk, wk, HCA_WINDOW, S, 128, 2) &&
            make_map4(&maps.wv, wv, HCA_WINDOW, S, 128, 2);
  if (ok && max_nc > 0) {
    ok = make_map4(&maps.ck, ck, max_nc, S, 128, 2) && make_map4(&maps.cv, cv, max_nc, S, 128, 2);
  } else if (ok) {
    maps.ck = maps.wk;
    maps.cv = maps.wv;
  }
  if (!ok) return HCA_ERR_CUDA;

  if (launch_decode<false>(maps, prm, sms, stream) != cudaSuccess) return HCA_ERR_CUDA;
  return launch_status();
}
}  // namespace

extern "C" {

hca_status_t hca_decode(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv, int max_nc,
                        const hca_bf16* wk, const hca_bf16* wv, const int32_t* ctx_len,
                        const hca_bf16* g, int S, int H, float scale, void* ws, size_t ws_bytes,
                        hca_bf16* out, hca_stream_t stream) {
  return decode_impl(q, ck, cv, max_nc, wk, wv, ctx_len, g, S, H, scale, nullptr, nullptr, 0, ws,
                     ws_bytes, out, stream);
}

hca_status_t hca_decode_vha(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv,
                            int max_nc, const hca_bf16* wk, const hca_bf16* wv,
                            const int32_t* ctx_len, const hca_bf16* g, int S, int H, float scale,
                            const hca_bf16* vha_down, const hca_bf16* vha_up, int vha_rank,
                            void* ws, size_t ws_bytes, hca_bf16* out, hca_stream_t stream) {
  if (vha_rank < 1 || vha_rank > HCA_NUM_HEADS) return HCA_ERR_INVALID_ARG;
  if (vha_down == nullptr || vha_up == nullptr) return HCA_ERR_INVALID_ARG;
  return decode_impl(q, ck, cv, max_nc, wk, wv, ctx_len, g, S, H, scale, vha_down, vha_up,
                     vha_rank, ws, ws_bytes, out, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation decode: the same kernels as hca_decode, with their scratch in
// a fixed device array owned by the library.
// ---------------------------------------------------------------------------
namespace {

constexpr int kNoAllocSlots = HCA_NOALLOC_MAX_CTAS + HCA_NOALLOC_MAX_SEQS;
// per slot: partial O [64][512] bf16 + (m, l) [2][64] fp32
constexpr size_t kNoAllocSlotBytes = static_cast<size_t>(64) * 512 * 2 + 2 * 64 * 4;
constexpr size_t kNoAllocPrefixOffset =
    256 + ((kNoAllocSlots * kNoAllocSlotBytes + 255) & ~static_cast<size_t>(255));
constexpr size_t kNoAllocScratchBytes =
    kNoAllocPrefixOffset + static_cast<size_t>(HCA_NOALLOC_MAX_SEQS + 1) * 8;

// The grid barrier counter (zero at load), partial O / (m, l) of up to
// kNoAllocSlots split slots, then the tile prefix.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the current device's context.  The
// array's name is only a host-side handle, so the address is asked of the
// runtime, with the device current.  It is asked on every call rather than
// cached: a cached address would outlive a cudaDeviceReset (which unloads the
// module and places the array anew in the next context).  The first call on a
// device loads the module there.  Null on failure.
void* noalloc_scratch_address() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return ptr;
}

}  // namespace

extern "C" {

hca_status_t hca_decode_noalloc(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv,
                                int max_nc, const hca_bf16* wk, const hca_bf16* wv,
                                const int32_t* ctx_len, const hca_bf16* g, int S, int H,
                                float scale, hca_bf16* out, hca_stream_t stream) {
  namespace D = hca::decode;
  if (H != HCA_NUM_HEADS) return HCA_ERR_UNSUPPORTED;
  if (S < 1 || max_nc < 0 || !scale_ok(scale)) return HCA_ERR_INVALID_ARG;
  if (S > HCA_NOALLOC_MAX_SEQS) return HCA_ERR_UNSUPPORTED;
  if (q == nullptr || wk == nullptr || wv == nullptr || ctx_len == nullptr || g == nullptr ||
      out == nullptr)
    return HCA_ERR_INVALID_ARG;
  if (max_nc > 0 && (ck == nullptr || cv == nullptr)) return HCA_ERR_INVALID_ARG;
  const void* ptrs[7] = {q, wk, wv, g, out, ck, cv};
  for (const void* ptr : ptrs)
    if (ptr != nullptr && !aligned16(ptr)) return HCA_ERR_INVALID_ARG;

  const int sms = device_sms();
  if (sms <= 0) return HCA_ERR_CUDA;
  const int grid = sms < HCA_NOALLOC_MAX_CTAS ? sms : HCA_NOALLOC_MAX_CTAS;
  const int slots = grid + S;
  uint8_t* wsb = static_cast<uint8_t*>(noalloc_scratch_address());
  if (wsb == nullptr) return HCA_ERR_CUDA;

  D::Params prm = {};
  prm.ctx_len = ctx_len;
  prm.S = S;
  prm.max_nc = max_nc;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.gsync = reinterpret_cast<unsigned long long*>(wsb);
  prm.ws_o = reinterpret_cast<uint16_t*>(wsb + 256);
  prm.ws_ml = reinterpret_cast<float*>(wsb + 256 + D::ws_o_bytes(slots));
  prm.seq_tile = reinterpret_cast<long long*>(wsb + kNoAllocPrefixOffset);
  prm.g = g;
  prm.out = out;

  D::Maps maps;
  bool ok = make_map4(&maps.q, q, static_cast<uint64_t>(S) * HCA_NUM_HEADS, 1, 64, 8) &&
            make_map4(&maps.wk, wk, HCA_WINDOW, S, 128, 2) &&
            make_map4(&maps.wv, wv, HCA_WINDOW, S, 128, 2);
  if (ok && max_nc > 0) {
    ok = make_map4(&maps.ck, ck, max_nc, S, 128, 2) && make_map4(&maps.cv, cv, max_nc, S, 128, 2);
  } else if (ok) {
    maps.ck = maps.wk;
    maps.cv = maps.wv;
  }
  if (!ok) return HCA_ERR_CUDA;

  if (launch_decode<false>(maps, prm, grid, stream) != cudaSuccess) return HCA_ERR_CUDA;
  return launch_status();
}

hca_status_t hca_cache_append(const hca_bf16* k_new, const hca_bf16* v_new,
                              const hca_bf16* s_new, const int32_t* ctx_len, int S, hca_bf16* wk,
                              hca_bf16* wv, hca_bf16* ws, hca_bf16* ck, hca_bf16* cv, int max_nc,
                              hca_stream_t stream) {
  if (S < 1 || max_nc < 0) return HCA_ERR_INVALID_ARG;
  if (k_new == nullptr || v_new == nullptr || s_new == nullptr || ctx_len == nullptr ||
      wk == nullptr || wv == nullptr || ws == nullptr)
    return HCA_ERR_INVALID_ARG;
  if (max_nc > 0 && (ck == nullptr || cv == nullptr)) return HCA_ERR_INVALID_ARG;
  const void* ptrs[6] = {k_new, v_new, wk, wv, ck, cv};
  for (const void* ptr : ptrs)
    if (ptr != nullptr && !aligned16(ptr)) return HCA_ERR_INVALID_ARG;
  if (S > 0x7fffffff / HCA_WINDOW) return HCA_ERR_UNSUPPORTED;
  hca::append::append_kernel<<<S, hca::append::kThreads, 0, stream>>>(
      k_new, v_new, s_new, ctx_len, wk, wv, ws, ck, cv, max_nc);
  return launch_status();
}

hca_status_t hca_decode_step(const hca_bf16* q, const hca_bf16* g, const hca_bf16* k_new,
                             const hca_bf16* v_new, const hca_bf16* s_new,
                             const int32_t* ctx_len, int S, int H, float scale, hca_bf16* wk,
                             hca_bf16* wv, hca_bf16* ws, hca_bf16* ck, hca_bf16* cv, int max_nc,
                             void* workspace, size_t ws_bytes, hca_bf16* out,
                             hca_stream_t stream) {
  // validate both halves before launching either
  if (H != HCA_NUM_HEADS) return HCA_ERR_UNSUPPORTED;
  if (S < 1 || max_nc < 0 || !scale_ok(scale)) return HCA_ERR_INVALID_ARG;
  if (S > 65535) return HCA_ERR_UNSUPPORTED;
  if (q == nullptr || g == nullptr || out == nullptr || workspace == nullptr)
    return HCA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(g) || !aligned16(out)) return HCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return HCA_ERR_INVALID_ARG;
  if (ws_bytes < hca_decode_workspace_size(S)) return HCA_ERR_INVALID_ARG;
  hca_status_t st =
      hca_cache_append(k_new, v_new, s_new, ctx_len, S, wk, wv, ws, ck, cv, max_nc, stream);
  if (st != HCA_OK) return st;
  return hca_decode(q, ck, cv, max_nc, wk, wv, ctx_len, g, S, H, scale, workspace, ws_bytes, out,
                    stream);
}

hca_status_t hca_quantize_e4m3(const hca_bf16* x, long long rows, uint8_t* codes, float* scale,
                               hca_stream_t stream) {
  if (rows < 0 || (rows > 0 && (x == nullptr || codes == nullptr || scale == nullptr)))
    return HCA_ERR_INVALID_ARG;
  if (rows == 0) return HCA_OK;
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
    return HCA_ERR_INVALID_ARG;
  namespace Q = hca::quant;
  const long long ctas = (rows + Q::kRowsPerCta - 1) / Q::kRowsPerCta;
  if (ctas > 0x7fffffffLL) return HCA_ERR_UNSUPPORTED;
  Q::quantize_e4m3_kernel<<<static_cast<unsigned>(ctas), Q::kThreads, 0, stream>>>(x, rows, codes,
                                                                                   scale);
  return launch_status();
}

hca_status_t hca_decode_e4m3(const hca_bf16* q, const uint8_t* ck, const float* ck_scale,
                             const uint8_t* cv, const float* cv_scale, int max_nc,
                             const uint8_t* wk, const float* wk_scale, const uint8_t* wv,
                             const float* wv_scale, const int32_t* ctx_len, const hca_bf16* g,
                             int S, int H, float scale, void* ws, size_t ws_bytes, hca_bf16* out,
                             hca_stream_t stream) {
  namespace D = hca::decode;
  if (H != HCA_NUM_HEADS) return HCA_ERR_UNSUPPORTED;
  if (S < 1 || max_nc < 0 || !scale_ok(scale)) return HCA_ERR_INVALID_ARG;
  if (q == nullptr || wk == nullptr || wv == nullptr || wk_scale == nullptr ||
      wv_scale == nullptr || ctx_len == nullptr || g == nullptr || out == nullptr || ws == nullptr)
    return HCA_ERR_INVALID_ARG;
  if (max_nc > 0 && (ck == nullptr || cv == nullptr || ck_scale == nullptr || cv_scale == nullptr))
    return HCA_ERR_INVALID_ARG;
  const void* ptrs[7] = {q, wk, wv, g, out, ck, cv};
  for (const void* ptr : ptrs)
    if (ptr != nullptr && !aligned16(ptr)) return HCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return HCA_ERR_INVALID_ARG;
  if (ws_bytes < hca_decode_workspace_size(S)) return HCA_ERR_INVALID_ARG;
  if (static_cast<long long>(S) * HCA_NUM_HEADS > 0x7fffffffLL || S > 65535)
    return HCA_ERR_UNSUPPORTED;

  const int sms = device_sms();
  if (sms <= 0) return HCA_ERR_CUDA;
  const int slots = sms + S;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  D::Params prm = {};
  prm.ctx_len = ctx_len;
  prm.S = S;
  prm.max_nc = max_nc;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.gsync = reinterpret_cast<unsigned long long*>(wsb);
  prm.ws_o = reinterpret_cast<uint16_t*>(wsb + 256);
  prm.ws_ml = reinterpret_cast<float*>(wsb + 256 + D::ws_o_bytes(slots));
  prm.seq_tile =
      reinterpret_cast<long long*>(wsb + 256 + ((D::ws_bytes(slots) + 255) & ~size_t(255)));
  prm.g = g;
  prm.out = out;
  prm.sck = ck_scale;
  prm.scv = cv_scale;
  prm.swk = wk_scale;
  prm.swv = wv_scale;

  D::Maps maps;
  bool ok = make_map4(&maps.q, q, static_cast<uint64_t>(S) * HCA_NUM_HEADS, 1, 64, 8) &&
            make_map_codes(&maps.wk, wk, HCA_WINDOW, S) &&
            make_map_codes(&maps.wv, wv, HCA_WINDOW, S);
  if (ok && max_nc > 0) {
    ok = make_map_codes(&maps.ck, ck, max_nc, S) && make_map_codes(&maps.cv, cv, max_nc, S);
  } else if (ok) {
    maps.ck = maps.wk;
    maps.cv = maps.wv;
  }
  if (!ok) return HCA_ERR_CUDA;
  if (launch_decode<true>(maps, prm, sms, stream) != cudaSuccess) return HCA_ERR_CUDA;
  return launch_status();
}

hca_status_t hca_get_device_error(hca_stream_t stream, unsigned int* where) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HCA_ERR_CUDA;
  unsigned int word = 0, w = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, hca::g_error_word, sizeof(word)) != cudaSuccess)
    return HCA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&w, hca::g_error_where, sizeof(w)) != cudaSuccess) return HCA_ERR_CUDA;
  if (cudaMemcpyToSymbol(hca::g_error_word, &zero, sizeof(zero)) != cudaSuccess ||
      cudaMemcpyToSymbol(hca::g_error_where, &zero, sizeof(zero)) != cudaSuccess)
    return HCA_ERR_CUDA;
  if (where != nullptr) *where = w;
  if (word & hca::DEVERR_TIMEOUT) return HCA_ERR_TIMEOUT;
  if (word & hca::DEVERR_BAD_INPUT) return HCA_ERR_DEVICE_INPUT;
  return HCA_OK;
}

hca_status_t hca_selftest_bounded_wait(int limit_us, hca_stream_t stream) {
  if (limit_us < 1 || limit_us > 10000000) return HCA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000ull);
  return launch_status();
}

const char* hca_status_string(hca_status_t status) {
  switch (status) {
    case HCA_OK: return "HCA_OK";
    case HCA_ERR_INVALID_ARG: return "HCA_ERR_INVALID_ARG";
    case HCA_ERR_UNSUPPORTED: return "HCA_ERR_UNSUPPORTED";
    case HCA_ERR_CUDA: return "HCA_ERR_CUDA";
    case HCA_ERR_TIMEOUT: return "HCA_ERR_TIMEOUT";
    case HCA_ERR_DEVICE_INPUT: return "HCA_ERR_DEVICE_INPUT";
  }
  return "HCA_ERR_UNKNOWN";
}

int hca_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------
namespace {

struct BwdLayout {
  size_t dO, delta, pc, dsc, pr, dsr, dck, dcv, total;
  int ncpad;
};

BwdLayout bwd_layout(int B, int T) {
  BwdLayout L = {};
  const size_t rows = static_cast<size_t>(B) * T * HCA_NUM_HEADS;
  const int nb = T / HCA_BLOCK;
  L.ncpad = ((nb + 127) / 128) * 128;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  size_t off = 0;
  L.dO = off;    off = up(off + rows * HCA_HEAD_DIM * 2);
  L.delta = off; off = up(off + rows * 4);
  L.pc = off;    off = up(off + rows * L.ncpad * 2);
  L.dsc = off;   off = up(off + rows * L.ncpad * 2);
  L.pr = off;    off = up(off + rows * hca::bwd::kRawW * 2);
  L.dsr = off;   off = up(off + rows * hca::bwd::kRawW * 2);
  L.dck = off;   off = up(off + static_cast<size_t>(B) * nb * HCA_HEAD_DIM * 4);
  L.dcv = off;   off = up(off + static_cast<size_t>(B) * nb * HCA_HEAD_DIM * 4);
  L.total = off;
  return L;
}

// the shared-memory attributes of the backward kernels, once per device
bool bwd_configured() {
  static bool done[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return true;
  namespace W = hca::bwd;
  if (cudaFuncSetAttribute(W::score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           W::kSmemAllocScore) != cudaSuccess ||
      cudaFuncSetAttribute(W::dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           W::kSmemAllocGemm) != cudaSuccess ||
      cudaFuncSetAttribute(W::dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           W::kSmemAllocGemm) != cudaSuccess)
    return false;
  done[dev] = true;
  return true;
}

}  // namespace

extern "C" {

size_t hca_prefill_bwd_workspace_size(int B, int T) {
  if (B < 1 || T < 1) return 0;
  return bwd_layout(B, T).total;
}

hca_status_t hca_prefill_bwd(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                             const hca_bf16* s, const hca_bf16* ck, const hca_bf16* cv,
                             const hca_bf16* g, const hca_bf16* out, const float* lse,
                             const hca_bf16* dout, int B, int T, int H, float scale, hca_bf16* dq,
                             float* dk, float* dv, float* ds, hca_bf16* dg, void* ws,
                             size_t ws_bytes, hca_stream_t stream) {
  namespace W = hca::bwd;
  if (H != HCA_NUM_HEADS) return HCA_ERR_UNSUPPORTED;
  if (B < 1 || T < 1 || !scale_ok(scale)) return HCA_ERR_INVALID_ARG;
  const void* need[14] = {q, k, v, s, g, out, lse, dout, dq, dk, dv, ds, dg, ws};
  for (const void* ptr : need)
    if (ptr == nullptr || !aligned16(ptr)) return HCA_ERR_INVALID_ARG;
  const int nb = T / HCA_BLOCK;
  if (nb > 0 && (ck == nullptr || cv == nullptr || !aligned16(ck) || !aligned16(cv)))
    return HCA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return HCA_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * HCA_NUM_HEADS > 0x7fffffffLL) return HCA_ERR_UNSUPPORTED;
  const BwdLayout L = bwd_layout(B, T);
  if (ws_bytes < L.total) return HCA_ERR_INVALID_ARG;
  const int sms = device_sms();
  if (sms <= 0 || !bwd_configured()) return HCA_ERR_CUDA;
  cudaStream_t st = stream;
  uint8_t* w = static_cast<uint8_t*>(ws);

  W::Params prm = {};
  prm.B = B;
  prm.T = T;
  prm.nb = nb;
  prm.ncpad = L.ncpad;
  prm.ut = (T + 1) / 2;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.dout = dout;
  prm.out = out;
  prm.g = g;
  prm.lse = lse;
  prm.dO = reinterpret_cast<uint16_t*>(w + L.dO);
  prm.delta = reinterpret_cast<float*>(w + L.delta);
  prm.dg = dg;
  prm.pc = reinterpret_cast<uint16_t*>(w + L.pc);
  prm.dsc = reinterpret_cast<uint16_t*>(w + L.dsc);
  prm.pr = reinterpret_cast<uint16_t*>(w + L.pr);
  prm.dsr = reinterpret_cast<uint16_t*>(w + L.dsr);
  prm.dq = dq;
  prm.dk = dk;
  prm.dv = dv;
  prm.dck = reinterpret_cast<float*>(w + L.dck);
  prm.dcv = reinterpret_cast<float*>(w + L.dcv);
  prm.k = k;
  prm.v = v;
  prm.s = s;
  prm.ds = ds;

  W::Maps maps;
  const uint64_t rows = static_cast<uint64_t>(T) * HCA_NUM_HEADS;
  const void* ckb = nb > 0 ? static_cast<const void*>(ck) : static_cast<const void*>(k);
  const void* cvb = nb > 0 ? static_cast<const void*>(cv) : static_cast<const void*>(v);
  const uint64_t ny = nb > 0 ? nb : T;
  const uint64_t ncx = L.ncpad > 0 ? L.ncpad : W::kRawW;
  const void* pcb = L.ncpad > 0 ? static_cast<const void*>(prm.pc) : prm.pr;
  const void* dscb = L.ncpad > 0 ? static_cast<const void*>(prm.dsc) : prm.dsr;
  bool ok = make_map(&maps.q, q, HCA_HEAD_DIM, rows, B, 128) &&
            make_map(&maps.dO, prm.dO, HCA_HEAD_DIM, rows, B, 128) &&
            make_map(&maps.ck, ckb, HCA_HEAD_DIM, ny, B, 128) &&
            make_map(&maps.cv, cvb, HCA_HEAD_DIM, ny, B, 128) &&
            make_map(&maps.k, k, HCA_HEAD_DIM, T, B, 128) &&
            make_map(&maps.v, v, HCA_HEAD_DIM, T, B, 128) &&
            make_map(&maps.dsc_a, dscb, ncx, rows, B, 128) &&
            make_map(&maps.dsr_a, prm.dsr, W::kRawW, rows, B, 128) &&
            make_map4(&maps.ck4, ckb, ny, B, 64, 8) && make_map4(&maps.k4, k, T, B, 64, 8) &&
            make_map(&maps.pc_t, pcb, ncx, rows, B, 64) &&
            make_map(&maps.dsc_t, dscb, ncx, rows, B, 64) &&
            make_map(&maps.pr_t, prm.pr, W::kRawW, rows, B, 64) &&
            make_map(&maps.dsr_t, prm.dsr, W::kRawW, rows, B, 64) &&
            make_map4(&maps.q4, q, rows, B, 64, 8) && make_map4(&maps.dO4, prm.dO, rows, B, 64, 8);
  if (!ok) return HCA_ERR_CUDA;

  const size_t nkv = static_cast<size_t>(B) * T * HCA_HEAD_DIM * 4;
  if (cudaMemsetAsync(dk, 0, nkv, st) != cudaSuccess ||
      cudaMemsetAsync(dv, 0, nkv, st) != cudaSuccess ||
      cudaMemsetAsync(ds, 0, static_cast<size_t>(B) * T * 4, st) != cudaSuccess ||
      (nb > 0 && cudaMemsetAsync(w + L.dck, 0, L.total - L.dck, st) != cudaSuccess))
    return HCA_ERR_CUDA;
  const long long nrows = static_cast<long long>(B) * rows;
  W::prep_kernel<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, st>>>(prm, nrows);
  W::score_kernel<<<sms, W::kThreads, W::kSmemAllocScore, st>>>(maps, prm);
  W::dq_kernel<<<sms, W::kThreads, W::kSmemAllocGemm, st>>>(maps, prm);
  W::dkv_kernel<<<sms, W::kThreads, W::kSmemAllocGemm, st>>>(maps, prm);
  if (nb > 0) W::compress_bwd_kernel<<<dim3(nb, B), 128, 0, st>>>(prm);
  return launch_status();
}

}  // extern "C"
