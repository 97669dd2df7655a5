/*
 * sagesla.h -- C ABI of the SageSLA attention library for NVIDIA B200 (sm_100a).
 *
 * SageSLA attention, as the TurboDiffusion pages describe it
 *   ("揭秘TurboDiffusion：如何让视频生成实现百倍加速？", 支柱一 SageAttention and
 *    支柱二 SLA; "TurboDiffusion跨模态：图文音视频多模态融合探索", 2.1-2.2;
 *    量子位 news, 技术解密 1-2):
 *   - SageAttention: QK^T in INT8 after a smoothing step that removes channel
 *     outliers (here: the per-head mean of K is subtracted), P.V in FP8;
 *   - SLA: per query block, only the top-k fraction of key blocks (sla_topk,
 *     default 0.1) is computed exactly; every other key block contributes
 *     through a linear-attention branch phi(Q)(phi(K)^T V), phi = elu + 1,
 *     followed by a d x d projection, added to the sparse output.
 *
 * Readings taken where the pages are silent (all stated here once):
 *   - INT8 Q and K codes per 64-token block with one fp32 scale each
 *     (amax/127, symmetric, round half to even); FP8 E4M3 V codes with one
 *     fp32 scale per channel (amax/448); K is smoothed by its per-channel mean
 *     over the N tokens before quantisation.
 *   - Block scores: mean-pooled Q_i . mean-pooled (K-mu)_j / sqrt(d) in fp32;
 *     k = clamp(ceil(topk * Nb), 1, Nb) blocks per query block, ties to the
 *     lower block index, walked in ascending order.
 *   - Online softmax: P = exp(S - running max); P~ = e4m3(448 P); the row sum
 *     is taken over the same P~ that weight V.
 *   - Linear branch from the raw bf16 Q, K, V: for row r of query block i,
 *     O_l = phi(q_r) H_i / phi(q_r) Z_i with H_i = sum over unselected key
 *     blocks j of phi(K_j)^T V_j and Z_i = sum of phi(K_j) rows; y = O_l W^T
 *     (W = proj_w, [d_out][d_in] row-major, shared by all heads, no bias).
 *     Empty complement (topk = 1) -> the branch contributes 0.
 *   - out = bf16(O_s + y), rounded once.
 *
 * Conventions for every entry point:
 *   - Tensors are DEVICE pointers owned by the caller, bf16, contiguous
 *     [B][H][N][d], 16-byte aligned.  Inputs are never written; rows n >= N
 *     are never read or written.
 *   - The call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  It performs no host synchronisation, except that the
 *     first call needing a larger workspace on a (device, stream) allocates it
 *     stream-ordered.
 *   - Supported: d == 128, block in {64, 128}, 0 < topk <= 1, B, H, N >= 1,
 *     B*H <= 65535, ceil(N / block) <= 12288 (N <= 786432 at block 64,
 *     1572864 at block 128), B*H*N*d < 2^40.  Anything else returns
 *     SAGESLA_ERR_INVALID without launching.  There is no CPU fallback and no
 *     alternative backend.
 *   - The library owns a workspace cache keyed by (device, stream);
 *     sagesla_release() frees it.
 */
#ifndef SAGESLA_H_
#define SAGESLA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sagesla_stream_t; /* same type as cudaStream_t */

enum {
  SAGESLA_OK = 0,
  SAGESLA_ERR_INVALID = -1,        /* bad argument (null, size, d, block, topk, NaN) */
  SAGESLA_ERR_MISALIGNED = -2,     /* a pointer is not 16-byte aligned */
  SAGESLA_ERR_OOM = -3,            /* workspace allocation failed */
  SAGESLA_ERR_LAUNCH = -4,         /* a CUDA launch or runtime call failed */
  SAGESLA_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait gave up */
  SAGESLA_ERR_NO_DEVICE = -6       /* current device is not sm_100 */
};

/*
 * sagesla_attn: the whole SageSLA path (smoothing + quantisation, pooled
 * top-k block mask, linear branch, block-sparse INT8/FP8 flash attention with
 * the linear output and projection added in its epilogue).
 *   q, k, v  bf16 [B][H][N][d] device.
 *   proj_w   bf16 [d][d] device, row-major, y = x W^T; NULL turns the linear
 *            branch off (out = O_s).
 *   out      bf16 [B][H][N][d] device (written).
 *   block    64 or 128 (query and key block size of the mask).
 *   topk     fraction of key blocks computed exactly per query block.
 * Returns SAGESLA_OK or a negative SAGESLA_ERR_* code (nothing written on an
 * argument error).
 */
int sagesla_attn(const void* q, const void* k, const void* v, const void* proj_w, void* out, int B,
                 int H, int N, int d, int block, float topk, sagesla_stream_t stream);

/*
 * dense_int8_attn: the dense reference point of the same kernels, identical
 * to sagesla_attn(q, k, v, NULL, out, B, H, N, d, 64, 1.0f, stream): every
 * key block selected, linear branch off.
 */
int dense_int8_attn(const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                    int d, sagesla_stream_t stream);

/*
 * sagesla_attn_host: sagesla_attn on HOST buffers (pinned memory gives
 * asynchronous copies).  Copies q, k, v (and proj_w) to the device, runs the
 * path, copies out back and synchronises before returning.  The B*H heads are
 * independent problems, so the call runs in up to 20 chunks of heads as a
 * pipeline: host->device copies of the next chunk and device->host copies of
 * the previous one (on two copy streams the library creates once per device)
 * overlap the path on the current chunk (on `stream`).  The result is
 * bit-identical to sagesla_attn.  Same shapes and codes as sagesla_attn;
 * proj_w may be NULL.  The device staging (4 x B*H*N*d bf16 + d*d) is cached
 * per (device, stream) until sagesla_release.
 */
int sagesla_attn_host(const void* q, const void* k, const void* v, const void* proj_w, void* out,
                      int B, int H, int N, int d, int block, float topk, sagesla_stream_t stream);

/*
 * sagesla_attn_opts: sagesla_attn with the SageAttention2++ quantisation
 * options (量子位 news, 技术解密 1: codes of 8 and, further, 4 bits, and a
 * quantisation calibrated per thread):
 *   qk_bits      8: Q and K codes in +-127 (the default path); 4: codes in
 *                +-7 with scale amax/7.  tcgen05 has no 4-bit integer MMA, so
 *                the 4-bit codes run through the same INT8 tensor-core path:
 *                an accuracy option, not a faster one.
 *   q_per_token  0: one Q scale per 64-token block (the default path); 1: one
 *                Q scale per token (the row a softmax thread owns), K keeps
 *                one scale per 64-token block.
 * Other arguments and behaviour as sagesla_attn; SAGESLA_ERR_INVALID for
 * other option values.  sagesla_attn is sagesla_attn_opts(..., 8, 0, ...).
 */
int sagesla_attn_opts(const void* q, const void* k, const void* v, const void* proj_w, void* out, int B, int H,
                      int N, int d, int block, float topk, int qk_bits, int q_per_token, sagesla_stream_t stream);

/*
 * sagesla_attn_qknorm: sagesla_attn on RMS-normalised q and k, the norm
 * fused into the kernels that load them (the DiT normalises q and k right
 * before attention: "thu-ml/TurboDiffusion" radar page §二 step 5, 量子位 news
 * 技术解密 4).  Reading: per token, over all H heads x d channels,
 *   x_n = bf16( fl32( fl32(x * inv) * gamma[h*d + c] ) ),
 *   inv = fl32( 1 / sqrt(sum of x^2 / (H*d) + eps) )  (the sum in fp64),
 * for q with gamma_q and for k with gamma_k (bf16 [H*d] device, 16-byte
 * aligned; eps in [0, 1]).  The result equals sagesla_attn on the
 * normalised tensors, without writing them: one extra read of q and k for
 * the per-token sums instead of a write and a read of both.
 */
int sagesla_attn_qknorm(const void* q, const void* k, const void* v, const void* gamma_q, const void* gamma_k,
                        float eps, const void* proj_w, void* out, int B, int H, int N, int d, int block, float topk,
                        sagesla_stream_t stream);

/*
 * sagesla_attn_bnhd: the attention on q, k, v in the token-major layout a
 * DiT's projections emit, bf16 [B][N][H][d] (the row of token n, head h at
 * ((b*N + n)*H + h)*d), read in place by the kernels that load them; out in
 * the same layout.  gamma_q and gamma_k both NULL: no norm (then eps is
 * ignored); both set: the QK RMSNorm of sagesla_attn_qknorm (the per-token
 * sums run over the H*d contiguous channels of each token).  The result equals
 * sagesla_attn / sagesla_attn_qknorm on the tensors permuted to [B][H][N][d],
 * bit for bit.  Note the argument order B, N, H.  Codes as sagesla_attn;
 * SAGESLA_ERR_INVALID when only one gamma is given.
 */
int sagesla_attn_bnhd(const void* q, const void* k, const void* v, const void* gamma_q, const void* gamma_k,
                      float eps, const void* proj_w, void* out, int B, int N, int H, int d, int block, float topk,
                      sagesla_stream_t stream);

/*
 * sagesla_get_quant: the smoothing + quantisation step alone (for parity).
 *   q8, k8   int8 [B][H][N][d] device: INT8 codes, row-major.
 *   v8       uint8 [B][H][N][d] device: FP8 E4M3 codes, row-major.
 *   sq, sk   float [B][H][ceil(N/64)] device: per-64-token-block scales.
 *   sv, mu   float [B][H][d] device: per-channel V scale, K mean.
 */
int sagesla_get_quant(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                      int8_t* q8, int8_t* k8, uint8_t* v8, float* sq, float* sk, float* sv, float* mu,
                      sagesla_stream_t stream);

/*
 * sagesla_get_mask: the block mask alone (for parity).
 *   idx_out  int32 [B][H][Nb][k] device, Nb = ceil(N/block), k as above;
 *            each row sorted ascending.
 *   qbar, kbar  float [B][H][Nb][d] device, or NULL: the pooled means.
 *   k_out    host int*: receives k (may be NULL).
 */
int sagesla_get_mask(const void* q, const void* k, int B, int H, int N, int d, int block,
                     float topk, int32_t* idx_out, float* qbar, float* kbar, int* k_out,
                     sagesla_stream_t stream);

/*
 * sagesla_smooth_stats_noalloc: the smoothing statistics of the path -- the
 * per-channel mean of K (mu, as in sagesla_get_quant) and the per-channel FP8
 * scale of V (sv) -- computed WITHOUT allocating any device memory.  The
 * pages have no counterpart: this is an interface for callers that cannot
 * allocate once running (a process that fixes its device-memory budget at
 * start-up, or code running where an allocation would stall or fail).  The
 * regular entry points allocate a workspace on first use; this one uses a
 * fixed 4 MiB scratch array that is part of the library image on every GPU
 * that loads the library, until the process exits.
 *   k, v     bf16 [B][H][N][d] device, 16-byte aligned.
 *   mu, sv   float [B][H][d] device (written).
 * The first call on a device looks up the scratch array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls share the scratch: calls that
 * overlap on the GPU (other streams or host threads on the same device) race
 * and must be serialised by the caller.  The rows are split as in the
 * regular path, so mu and sv have the same bits as sagesla_get_quant's; when
 * the partial sums of all heads do not fit the scratch the heads run in
 * chunks, one after another on `stream`.  A length whose partial sums for a
 * single head exceed the scratch (N above 2 795 520 tokens) returns
 * SAGESLA_ERR_INVALID without launching; other argument errors as for
 * sagesla_attn.
 */
int sagesla_smooth_stats_noalloc(const void* k, const void* v, int B, int H, int N, int d, float* mu,
                                 float* sv, sagesla_stream_t stream);

/* Number of key blocks kept per query block: clamp(ceil(topk*nb*(1-1e-6)), 1, nb). */
int sagesla_topk_count(int nb, float topk);

/*
 * sagesla_sync_status: synchronises `stream` and returns SAGESLA_OK, or
 * SAGESLA_ERR_DEVICE_TIMEOUT if a bounded device-side wait of an earlier
 * call gave up (the flag is then cleared), or SAGESLA_ERR_LAUNCH.  The flag
 * is one word per DEVICE, shared by all streams: a timeout on any stream of
 * the current device is reported by the next sagesla_sync_status() on any
 * stream (after that stream's work, not necessarily the other stream's).
 * Callers that use several streams synchronise them all, then call this once.
 */
int sagesla_sync_status(sagesla_stream_t stream);

/*
 * sagesla_watchdog_selftest: exercises the failure-detection path on the GPU
 * without faulting it.  Launches (on `stream`) one thread that waits on an
 * mbarrier nothing ever arrives on, `probes` times (1 .. 1048576; each probe
 * may suspend the thread briefly), and then records the expiry in the
 * device's watchdog word the way every bounded wait of the library does.
 * The next sagesla_sync_status() on the stream returns
 * SAGESLA_ERR_DEVICE_TIMEOUT and clears the word; the context stays usable.
 * Returns SAGESLA_ERR_INVALID for `probes` out of range (no launch),
 * SAGESLA_ERR_NO_DEVICE / SAGESLA_ERR_LAUNCH as the other entry points.
 */
int sagesla_watchdog_selftest(int probes, sagesla_stream_t stream);

/*
 * sagesla_debug_flash_stall: the failure-detection path of the real sparse
 * flash kernel, made to run on purpose without faulting the GPU.  Runs
 * sagesla_attn(q, k, v, NULL, out, B, H, N, d, 64, topk) with three changes
 * to its block-64 flash launch:
 *   - `grid` CTAs (>= 1; capped at the normal persistent grid), so that one
 *     CTA can be made to serve many query blocks;
 *   - every bounded wait of the flash kernel gives up after `spin_limit`
 *     probes (1024 .. 16777216, the default being 16777216);
 *   - for stall_step >= 0, CTA 0's first pipeline omits the key-tile copies
 *     of its step `stall_step` (counted over all its query blocks), so the
 *     wait of the MMA issuer on that stage never completes; it gives up,
 *     raises the CTA's abort flag (every role stops at its next wait), waits
 *     for the copies and MMAs already in flight, frees its tensor memory and
 *     returns, and the device's watchdog word is set.  stall_step == -1
 *     stalls nothing (the output is then that of sagesla_attn).
 * The next sagesla_sync_status() returns SAGESLA_ERR_DEVICE_TIMEOUT once;
 * the context stays usable.  `out` is partly unwritten after a stall.
 * Returns SAGESLA_ERR_INVALID for arguments out of range (no launch), else
 * as sagesla_attn.
 */
int sagesla_debug_flash_stall(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                              float topk, int grid, int stall_step, long long spin_limit, sagesla_stream_t stream);

/*
 * W8A8 linear layer: y = x W^T with weights and activations both INT8,
 * quantised in blocks of 128 x 128 ("揭秘TurboDiffusion：如何让视频生成实现
 * 百倍加速？", 支柱三 W8A8线性层量化; 量子位 news, 技术解密 4).
 * Reading (the pages give only the block size): one fp32 scale per 128 x 128
 * block of x [M][K] and of W [N][K] (the nn.Linear convention), the same
 * symmetric quantiser as Q and K above (s = amax/127, code = RNE(x*127/amax)
 * clamped to +-127, amax = 0 -> s = 1, codes 0; a last block of rows shorter
 * than 128 is quantised over its valid rows), and
 *   y[m][n] = sum over 128-wide K blocks kb of
 *             s_x[m/128][kb] * s_w[n/128][kb] * (integer dot on kb),
 * accumulated in fp32 in kb order, rounded once to bf16.
 *
 * Code layout ("tile images"): for a [rows][cols] matrix, ceil(rows/128) x
 * (cols/128) blocks of 16384 bytes in [row block][column block] order; in a
 * block, code (r, c) sits at byte (r/8)*1024 + (c/16)*128 + (r%8)*16 + c%16
 * (the tcgen05 K-major no-swizzle operand image); rows past `rows` hold 0.
 * Scales: fp32 [ceil(rows/128)][cols/128].
 *
 * sagesla_w8a8_quant: codes and scales of a bf16 [rows][cols] device matrix
 *   (cols a multiple of 128; rows <= 8388480).  Used once for W, and by
 *   sagesla_w8a8_linear for x.  a, codes 16-byte aligned; scales 4-byte.
 * sagesla_w8a8_gemm: y (bf16 [M][N] device, 16-byte aligned) from the codes
 *   and scales of x ([M][K]) and W ([N][K]); N, K multiples of 128.
 * sagesla_w8a8_linear: quantises x (bf16 [M][K] device) into the library's
 *   workspace of the stream, then the GEMM.
 * All three are asynchronous on `stream` and return SAGESLA_ERR_INVALID /
 * SAGESLA_ERR_MISALIGNED without launching on a bad argument.
 */
int sagesla_w8a8_quant(const void* a, int rows, int cols, void* codes, float* scales, sagesla_stream_t stream);
int sagesla_w8a8_gemm(const void* xq, const float* sx, const void* wq, const float* sw, void* y, int M, int N, int K,
                      sagesla_stream_t stream);
int sagesla_w8a8_linear(const void* x, const void* wq, const float* sw, void* y, int M, int N, int K,
                        sagesla_stream_t stream);

/* Human-readable text for a return code (static storage). */
const char* sagesla_strerror(int code);

/*
 * Measurement hooks.  sagesla_profile(1) brackets every kernel the library
 * launches with CUDA events recorded on the launching stream;
 * sagesla_profile_read() waits for them and returns, per kernel id, the
 * summed milliseconds and the number of launches since the last read, then
 * forgets them.  Kernel ids: 0 stats, 1 stats finalise, 2 quantise,
 * 3 pooled top-k, 4 linear per-block phi(K)^T V, 5 linear complement sum,
 * 6 sparse flash, 7 projection-weight tiling, 8 linear output (phi(Q) H,
 * normalisation, projection), 9 W8A8 block quantiser, 10 W8A8 GEMM,
 * 11 QK RMSNorm per-token sums.
 * ms / launches are arrays of nkernels entries (either may be NULL).
 * Profiling is off by default.
 */
#define SAGESLA_NUM_KERNELS 12
void sagesla_profile(int enable);
int sagesla_profile_read(double* ms, int* launches, int nkernels);

/* Frees every cached workspace (synchronises the device first). */
void sagesla_release(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGESLA_H_ */
