/*
 * hca.h — C ABI of libhca.so, a B200 (sm_100a) implementation of the forward
 * hot path of Heavily Compressed Attention (HCA).
 *
 * The method.  'BaiduがERNIE 5.5 Flash Baseを公開' §2.1 (Latent-Gated Sparse
 * Attention) and its Chinese twin 'ERNIE 5.5 Flash Base 正式发布' §2.1 describe
 * HCA layers that turn every 128 tokens into one cache entry and run one dense
 * softmax over all of those entries plus a short window of recent raw tokens,
 * with 64 query heads of width 512; every layer multiplies its attention
 * output by a learned gate.  The xenospectrum analysis of the same release
 * (section 活性140億パラメータと長文処理を支える仕組み) gives the window: the
 * newest 128 tokens, kept uncompressed.  Where the pages are silent this
 * library fixes: one shared KV head; entry j = softmax(s over block j)-weighted
 * sum of the block's K rows (and, with the same weights, of its V rows), with s
 * a per-token score; query t sees entry j only when block j lies wholly before
 * its window, i.e. j < nc(t) = max(0, floor((t - 127) / 128)), and the raw keys
 * max(0, t - 127) .. t; out = sigmoid(g) * o elementwise.
 *
 * Conventions shared by every call:
 *  - bf16 values are passed as raw 16-bit patterns (hca_bf16).  Every tensor is
 *    dense, row-major, on the current CUDA device, and 16-byte aligned.
 *  - The caller owns every buffer and the stream; the library allocates no
 *    memory and keeps no per-call state.  Calls are asynchronous on `stream`
 *    (NULL = legacy default stream).
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call returns HCA_ERR_INVALID_ARG or HCA_ERR_UNSUPPORTED and
 *    launches nothing.  HCA_ERR_CUDA reports a launch failure.
 *  - Kernels never trap.  Every wait inside them is bounded; a wait that runs
 *    out, or a device-resident argument found out of range (decode context
 *    lengths), is recorded in a device-side error word that
 *    hca_get_device_error() reads back.
 *  - No C++ exception crosses this interface.
 */
#ifndef HCA_H
#define HCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HCA_OK = 0,
  HCA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or scale       */
  HCA_ERR_UNSUPPORTED = 2, /* a shape outside what the kernels implement       */
  HCA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed                */
  HCA_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out               */
  HCA_ERR_DEVICE_INPUT = 5 /* a device-resident argument was out of range      */
} hca_status_t;

typedef uint16_t hca_bf16;              /* raw bfloat16 bits                   */
typedef struct CUstream_st* hca_stream_t; /* same type as cudaStream_t         */

#define HCA_HEAD_DIM 512 /* width of q, k, v and o rows                        */
#define HCA_NUM_HEADS 64 /* query heads sharing the single KV head             */
#define HCA_BLOCK 128    /* tokens per compressed entry                        */
#define HCA_WINDOW 128   /* raw tokens each query attends (itself included)    */

/*
 * hca_compress — block compressor.
 *   'BaiduがERNIE 5.5 Flash Baseを公開' §2.1: 128 tokens -> one cache entry.
 *   For every complete block j < nb = floor(T / 128) of every batch b:
 *     w = softmax(s[b, 128j : 128j + 128])            (fp32)
 *     ck[b, j, :] = sum_i w_i * k[b, 128j + i, :]      (fp32 accumulate, bf16 RNE)
 *     cv[b, j, :] = sum_i w_i * v[b, 128j + i, :]
 *   Tokens of a trailing partial block are not compressed.
 * Layout:  k, v  [B, T, 512] bf16;  s [B, T] bf16;  ck, cv [B, nb, 512] bf16.
 * Errors:  B < 1 or T < 1 -> HCA_ERR_INVALID_ARG.  nb == 0 launches nothing.
 */
hca_status_t hca_compress(const hca_bf16* k, const hca_bf16* v, const hca_bf16* s, int B, int T,
                          hca_bf16* ck, hca_bf16* cv, hca_stream_t stream);

/*
 * hca_prefill_workspace_size — bytes of device scratch hca_prefill_fwd needs
 * on the current device (probability tiles in flight between the CTAs of
 * each cluster; under 10 MB on a B200).  The answer depends on how many
 * clusters fit on the device, which is queried once per device.  Returns 0
 * for B < 1 or T < 1 or when the query fails.
 */
size_t hca_prefill_workspace_size(int B, int T);

/*
 * hca_prefill_fwd — HCA attention for every position of B sequences.
 *   For query t of batch b and head h (page sources as above):
 *     keys   = [ck[b, 0 : nc(t)] ; k[b, max(0, t-127) : t+1]]
 *     values = [cv[b, 0 : nc(t)] ; v[b, max(0, t-127) : t+1]]
 *     p      = softmax(scale * keys . q[b, t, h])      (one softmax over both sets)
 *     out[b, t, h, :] = sigmoid(g[b, t, h, :]) * (p . values)
 *   lse (optional) receives ln(sum exp(scale * keys . q)) per (b, t, h).
 * Layout:  q, g, out [B, T, H, 512] bf16 (H = 64);  k, v [B, T, 512] bf16;
 *          ck, cv [B, floor(T/128), 512] bf16 as written by hca_compress;
 *          lse [B, T, H] fp32 or NULL;  ws: caller-owned device scratch of at
 *          least hca_prefill_workspace_size(B, T) bytes, 256-byte aligned (its
 *          contents need no initialisation and are meaningless afterwards;
 *          two calls in flight at once need two workspaces).
 * Errors:  H != 64 -> HCA_ERR_UNSUPPORTED; B < 1, T < 1, a null pointer (other
 *          than lse), a pointer not 16-byte aligned, a workspace too small or
 *          misaligned, or a non-finite or non-positive scale ->
 *          HCA_ERR_INVALID_ARG.
 */
hca_status_t hca_prefill_fwd(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                             const hca_bf16* ck, const hca_bf16* cv, const hca_bf16* g, int B,
                             int T, int H, float scale, hca_bf16* out, float* lse, void* ws,
                             size_t ws_bytes, hca_stream_t stream);

/*
 * hca_prefill_fwd_vha — hca_prefill_fwd followed, inside the same kernel, by
 *   virtual head attention ('BaiduがERNIE 5.5 Flash Baseを公開' §2.1 and
 *   'ERNIE 5.5 Flash Base 正式发布' §2.1, VHA: after attention, a light
 *   low-rank mix across heads with an identity skip, fused into the attention
 *   kernel at inference).  With x[b, t] the [H, 512] gated output above:
 *     out[b, t, h, :] = x[h, :] + sum_r up[h, r] * sum_k down[k, r] * x[k, :]
 *   (the pages give no rank and do not say where the gate sits; this reads
 *   the mix as acting on the gated output of each position).
 * Layout:  as hca_prefill_fwd;  vha_down, vha_up [64, vha_rank] bf16
 *          row-major, device memory, 1 <= vha_rank <= 64.  The mix runs in
 *          fp32 on bf16 operands: x rounded to bf16 and the 64 x 64 product
 *          up down^T formed in fp32 and rounded to bf16 once per launch.
 * Errors:  those of hca_prefill_fwd; HCA_ERR_INVALID_ARG for a rank outside
 *          [1, 64] or a NULL factor.
 */
hca_status_t hca_prefill_fwd_vha(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                                 const hca_bf16* ck, const hca_bf16* cv, const hca_bf16* g,
                                 int B, int T, int H, float scale, const hca_bf16* vha_down,
                                 const hca_bf16* vha_up, int vha_rank, hca_bf16* out, float* lse,
                                 void* ws, size_t ws_bytes, hca_stream_t stream);

/*
 * hca_prefill_bwd_workspace_size — bytes of device scratch hca_prefill_bwd
 * needs: dO, the probabilities and their gradients over every visited
 * (row, key) pair in bf16, and the fp32 entry gradients (about 2 KB per
 * (position, head) row per 512 compressed entries, plus 1.6 KB per row).
 * Returns 0 for B < 1 or T < 1.
 */
size_t hca_prefill_bwd_workspace_size(int B, int T);

/*
 * hca_prefill_bwd — gradients of L = sum(dout * out) for out =
 *   hca_prefill_fwd(q, k, v, hca_compress(k, v, s), g) (the model trains at
 *   128K context, 'BaiduがERNIE 5.5 Flash Baseを公開' §3).  With o the
 *   ungated output and P the softmax of each query:
 *     dg = dout * out * (1 - sigmoid(g)),  dO = dout * sigmoid(g)
 *     dS = P (dO . value - sum_d dout * out),  dq = scale sum dS key,
 *     dkey = scale sum dS q,  dvalue = sum P dO  (raw keys and entries),
 *   and the entry gradients through each block's compressor into dk, dv and
 *   ds (ds_i = w_i (a_i - sum w a), a_i = dcK . k_i + dcV . v_i).
 * Layout:  q, g, out, dout, dq, dg [B, T, 64, 512] bf16;  k, v [B, T, 512]
 *          bf16;  s [B, T] bf16;  ck, cv the forward's [B, T/128, 512];
 *          lse [B, T, 64] fp32 as written by hca_prefill_fwd;  dk, dv
 *          [B, T, 512] fp32;  ds [B, T] fp32 (0 for tokens of a partial
 *          block).  All device memory, 16-byte aligned; ws 256-byte aligned,
 *          at least hca_prefill_bwd_workspace_size(B, T) bytes, contents
 *          meaningless before and after.  Five launches on `stream`.
 * Errors:  HCA_ERR_UNSUPPORTED for H != 64 or T * 64 >= 2^31;
 *          HCA_ERR_INVALID_ARG for a NULL or misaligned pointer, B, T < 1, a
 *          non-finite or non-positive scale, or a short workspace;
 *          HCA_ERR_CUDA for a launch failure.
 */
hca_status_t hca_prefill_bwd(const hca_bf16* q, const hca_bf16* k, const hca_bf16* v,
                             const hca_bf16* s, const hca_bf16* ck, const hca_bf16* cv,
                             const hca_bf16* g, const hca_bf16* out, const float* lse,
                             const hca_bf16* dout, int B, int T, int H, float scale, hca_bf16* dq,
                             float* dk, float* dv, float* ds, hca_bf16* dg, void* ws,
                             size_t ws_bytes, hca_stream_t stream);

/*
 * hca_decode_workspace_size — bytes of scratch hca_decode needs for S
 * sequences on the current device (partial results of the split-KV pass and
 * a grid-barrier counter).  A workspace must be zero-filled once before its
 * first hca_decode call (e.g. cudaMemsetAsync); every call leaves it valid for
 * the next one, whatever S, on the same device.
 */
size_t hca_decode_workspace_size(int S);

/*
 * hca_decode — one new token per sequence (split-KV over all SMs, then a
 * log-sum-exp combine, in one cooperative launch of one CTA per SM; above
 * 1024 sequences a one-CTA plan kernel runs first).
 *   For sequence i with context length L = ctx_len[i] (which counts the new
 *   token, so the query sits at t = L - 1):
 *     keys   = [ck[i, 0 : nc(L-1)] ; the min(L, 128) newest raw keys]
 *     out[i, h, :] = sigmoid(g[i, h, :]) * softmax(scale * keys . q[i, h]) . values
 *   The raw window is a ring: the token at position p lives in slot p mod 128
 *   of wk/wv; when L < 128 only slots 0 .. L-1 are read.  Slot order does not
 *   change the result (no positional term).
 * Layout:  q, g, out [S, H, 512] bf16 (H = 64);  ck, cv [S, max_nc, 512] bf16;
 *          wk, wv [S, 128, 512] bf16;  ctx_len [S] int32 on the device;
 *          ws: caller-owned device scratch of at least
 *          hca_decode_workspace_size(S) bytes, 256-byte aligned, zero-filled
 *          before its first use; one call at a time per workspace.
 * Errors:  host-checked as for prefill (and ws_bytes too small ->
 *          HCA_ERR_INVALID_ARG).  A device-side ctx_len < 1 or one needing more
 *          than max_nc entries is clamped and reported later by
 *          hca_get_device_error() as HCA_ERR_DEVICE_INPUT.
 */
hca_status_t hca_decode(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv, int max_nc,
                        const hca_bf16* wk, const hca_bf16* wv, const int32_t* ctx_len,
                        const hca_bf16* g, int S, int H, float scale, void* ws, size_t ws_bytes,
                        hca_bf16* out, hca_stream_t stream);

/*
 * hca_decode_vha — hca_decode followed, inside the same kernel, by virtual
 *   head attention on each sequence's gated output (same passage and reading
 *   as hca_prefill_fwd_vha):
 *     out[s, h, :] = x[h, :] + sum_r up[h, r] * sum_k down[k, r] * x[k, :]
 *   with x[s] the [64, 512] output hca_decode would write.  The mix runs in
 *   fp32 on x rounded to bf16 (a second grid barrier of the launch separates
 *   the two phases).
 * Layout:  as hca_decode;  vha_down, vha_up [64, vha_rank] bf16 row-major,
 *          device memory, 1 <= vha_rank <= 64.
 * Errors:  those of hca_decode; HCA_ERR_INVALID_ARG for a rank outside
 *          [1, 64] or a NULL factor.
 */
hca_status_t hca_decode_vha(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv,
                            int max_nc, const hca_bf16* wk, const hca_bf16* wv,
                            const int32_t* ctx_len, const hca_bf16* g, int S, int H, float scale,
                            const hca_bf16* vha_down, const hca_bf16* vha_up, int vha_rank,
                            void* ws, size_t ws_bytes, hca_bf16* out, hca_stream_t stream);

/*
 * hca_decode_noalloc — hca_decode for callers that cannot allocate device
 * memory.  The paper has no counterpart: this is a deployment variant.
 *   Some callers have no way to provide scratch: a plugin loaded into a host
 *   program that owns all device memory and exposes no allocator, or a
 *   latency-critical serving loop where a cudaMalloc (which can synchronise
 *   the whole device) is not allowed.  This entry point takes the same
 *   inputs and output as hca_decode but no workspace; its scratch lives in
 *   one fixed device array inside the library (224 split slots of 66,048
 *   bytes plus a small index and the grid-barrier counter: about 14.8 MB),
 *   which every GPU that loads the library keeps until the process exits.
 *   Limits: S <= HCA_NOALLOC_MAX_SEQS (64); larger S returns
 *   HCA_ERR_UNSUPPORTED without launching.  The split uses at most
 *   HCA_NOALLOC_MAX_CTAS (160) CTAs.
 *   Set-up: every call looks up the array's device address in the current
 *   device's context (cudaGetSymbolAddress, with that device current; the
 *   array's name in host code is only a handle).  The first call on a device
 *   also loads the library's module there, so make that first call outside
 *   any stream capture.  Nothing is allocated, ever.
 *   Sharing: every call uses the same array.  Its grid-barrier counter starts
 *   at zero when the library loads and every call leaves it valid (each call
 *   writes every other scratch value it later reads), but two calls that
 *   overlap on the GPU (other streams, other threads) race on it: serialise
 *   them.
 */
#define HCA_NOALLOC_MAX_SEQS 64
#define HCA_NOALLOC_MAX_CTAS 160
hca_status_t hca_decode_noalloc(const hca_bf16* q, const hca_bf16* ck, const hca_bf16* cv,
                                int max_nc, const hca_bf16* wk, const hca_bf16* wv,
                                const int32_t* ctx_len, const hca_bf16* g, int S, int H,
                                float scale, hca_bf16* out, hca_stream_t stream);

/*
 * hca_cache_append — incremental update of a decode cache by one new token per
 * sequence (the step on either side of hca_decode in serving).
 *   'BaiduがERNIE 5.5 Flash Baseを公開' §2.1: every 128 tokens become one
 *   cache entry; the xenospectrum analysis (section 活性140億パラメータと
 *   長文処理を支える仕組み): the newest 128 tokens stay raw.
 *   For sequence i with L = ctx_len[i] (which counts the new token, at
 *   position p = L - 1):
 *     wk[i, p mod 128] = k_new[i];  wv[i, p mod 128] = v_new[i];
 *     ws[i, p mod 128] = s_new[i]                       (the ring of raw tokens)
 *   and when L is a multiple of 128, block j = L/128 - 1 (now exactly the ring)
 *   is compressed into entry j:
 *     w = softmax(ws[i, 0:128]) (fp32);  ck[i, j] = sum_r w_r wk[i, r];
 *     cv[i, j] = sum_r w_r wv[i, r]           (fp32 accumulate, bf16 RNE)
 *   -- the value hca_compress gives for that block of the raw sequence.
 * Layout:  k_new, v_new [S, 512] bf16;  s_new [S] bf16;  ctx_len [S] int32 on
 *          the device;  wk, wv [S, 128, 512] bf16 and ws [S, 128] bf16 rings,
 *          updated in place;  ck, cv [S, max_nc, 512] bf16, entry j written in
 *          place (may be NULL when max_nc = 0).
 * Errors:  host-checked: S < 1, max_nc < 0, a null or (for the 512-wide
 *          tensors) misaligned pointer -> HCA_ERR_INVALID_ARG.  A device-side
 *          ctx_len < 1, or a completed block j >= max_nc, writes nothing for
 *          that sequence (ctx_len < 1) or skips the entry, and is reported by
 *          hca_get_device_error() as HCA_ERR_DEVICE_INPUT.
 */
hca_status_t hca_cache_append(const hca_bf16* k_new, const hca_bf16* v_new,
                              const hca_bf16* s_new, const int32_t* ctx_len, int S, hca_bf16* wk,
                              hca_bf16* wv, hca_bf16* ws, hca_bf16* ck, hca_bf16* cv, int max_nc,
                              hca_stream_t stream);

/*
 * hca_decode_step — one serving step: hca_cache_append of the new tokens,
 * then hca_decode of their queries against the updated cache, in stream
 * order on `stream` (two launches).  Arguments as in those two calls;
 * everything is validated before either kernel is launched.
 */
hca_status_t hca_decode_step(const hca_bf16* q, const hca_bf16* g, const hca_bf16* k_new,
                             const hca_bf16* v_new, const hca_bf16* s_new,
                             const int32_t* ctx_len, int S, int H, float scale, hca_bf16* wk,
                             hca_bf16* wv, hca_bf16* ws, hca_bf16* ck, hca_bf16* cv, int max_nc,
                             void* workspace, size_t ws_bytes, hca_bf16* out,
                             hca_stream_t stream);

/*
 * hca_quantize_e4m3 — FP8 storage of 512-wide bf16 rows (e.g. cache entries
 * and window rows for hca_decode_e4m3).
 *   The pages train with FP8 mixed precision and ship FP8 weights
 *   ('BaiduがERNIE 5.5 Flash Baseを公開' §3 and §5); the library stores a
 *   decode cache the same way.  Per row r:
 *     scale[r] = amax(|x[r, :]|) / 448            (fp32; 1 for an all-zero row)
 *     codes[r, c] = e4m3(x[r, c] / scale[r])      (fp32 division, round to
 *                                                   nearest even, saturating at
 *                                                   +-448)
 *   so the stored value is e4m3_value(codes) * scale.
 * Layout:  x [rows, 512] bf16 (16-byte aligned);  codes [rows, 512] bytes
 *          (16-byte aligned);  scale [rows] fp32.  Rows must be finite.
 * Errors:  rows < 0 or a null / misaligned pointer -> HCA_ERR_INVALID_ARG.
 */
hca_status_t hca_quantize_e4m3(const hca_bf16* x, long long rows, uint8_t* codes, float* scale,
                               hca_stream_t stream);

/*
 * hca_decode_e4m3 — hca_decode over an FP8 cache: the compressed entries and
 * the raw window rows stored by hca_quantize_e4m3 (half the bytes a decode
 * step streams).  The result is the HCA decode of the stored values
 * (code * row scale), as defined for hca_decode; q and g stay bf16, and q must
 * satisfy |q| < 65504 (the kernel runs its MMAs in f16: every e4m3 value and
 * every such bf16 value is exact in f16).
 * Layout:  q, g, out [S, 64, 512] bf16;  ck, cv [S, max_nc, 512] codes with
 *          ck_scale, cv_scale [S, max_nc] fp32;  wk, wv [S, 128, 512] codes (ring,
 *          slot = position mod 128) with wk_scale, wv_scale [S, 128] fp32;
 *          ctx_len [S] int32 on the device;  ws as for hca_decode (the same
 *          workspace serves both calls).
 * Errors:  as hca_decode; every scale pointer is required (ck / cv scales only
 *          when max_nc > 0).
 */
hca_status_t hca_decode_e4m3(const hca_bf16* q, const uint8_t* ck, const float* ck_scale,
                             const uint8_t* cv, const float* cv_scale, int max_nc,
                             const uint8_t* wk, const float* wk_scale, const uint8_t* wv,
                             const float* wv_scale, const int32_t* ctx_len, const hca_bf16* g,
                             int S, int H, float scale, void* ws, size_t ws_bytes, hca_bf16* out,
                             hca_stream_t stream);

/*
 * hca_get_device_error — synchronises `stream`, then reads and clears the
 * device-side error word of the current device.  Returns HCA_OK,
 * HCA_ERR_TIMEOUT, HCA_ERR_DEVICE_INPUT or HCA_ERR_CUDA.  `where`, if not
 * NULL, receives an internal code naming the wait that gave up.
 * The error word is one per device for the whole process: every stream and
 * every host thread that launches this library's kernels on that device
 * records into it, and this call reads and clears it for all of them.  A
 * caller that drives one device from several threads or streams therefore
 * sees (and clears) errors of the others' launches too; serialise the checks
 * or attribute errors per device, not per stream.
 */
hca_status_t hca_get_device_error(hca_stream_t stream, unsigned int* where);

/*
 * hca_selftest_bounded_wait — launches one CTA that waits on an mbarrier
 * nobody arrives on, with a limit of `limit_us` microseconds (1 .. 10^7).
 * The kernel gives up, records HCA_ERR_TIMEOUT and exits normally; the
 * context stays usable.  Exists to test the failure path without faulting.
 */
hca_status_t hca_selftest_bounded_wait(int limit_us, hca_stream_t stream);

/* hca_status_string — static, human-readable name of a status code. */
const char* hca_status_string(hca_status_t status);

/* hca_version — library version as major*10000 + minor*100 + patch. */
int hca_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HCA_H */
