// kernels.h -- host-side launchers of the SageSLA kernels (internal; the
// public C ABI is include/sagesla.h).  All launchers are asynchronous on
// `st` and return the cudaGetLastError() of their launch.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace sagesla {

// Geometry shared by the launchers.
struct Geom {
  int BH;      // B*H
  int N;       // tokens
  int block;   // 64 or 128 (mask block)
  int nb;      // ceil(N/block)
  int nq;      // 64-token quantisation tiles per head, padded: 2*ceil(N/128)
  int kc;      // key blocks kept per query block
  int split;   // row splits of the statistics pass
  int H = 1;   // heads (B = BH / H)
  int tok = 0; // q, k, v, out layout: 0 = [B][H][N][d], 1 = [B][N][H][d] (token-major, as a DiT emits it)
};

// QK RMSNorm applied where a kernel loads q or k (inv == nullptr: off):
// x * inv[b][n] * gamma[h*d + c], rounded to bf16.
struct QKNorm {
  const float* inv = nullptr;  // [B][N] per-token 1 / rms over the H*d channels
  const uint4* gamma = nullptr;  // bf16 [H*d] as 16-byte units (8 channels each)
  int H = 1, N = 1;
};
// Per-token 1 / rms of q and k (QK RMSNorm), [B][N] each.
cudaError_t launch_rms_inv(const void* q, const void* k, int B, int H, int N, double eps, float* inv_q, float* inv_k,
                           cudaStream_t st, int tok = 0);
// K1: per-split fp64 sums of K and fp32 max|V| per channel.
cudaError_t launch_stats_partial(const void* k, const void* v, const Geom& g, double* psum, float* pmax,
                                 cudaStream_t st, QKNorm nk = QKNorm());
// K1b: mu = fl32(sum/N); V scale amax/448 and multiplier 448/amax per channel.
cudaError_t launch_stats_final(const double* psum, const float* pmax, const Geom& g, float* mu, float* sv,
                               float* mv, cudaStream_t st);
// K2: smoothing + INT8 Q/K tiles + FP8 V^T tiles + per-64-row pooled sums.
cudaError_t launch_quant(const void* q, const void* k, const void* v, const float* mu, const float* mv,
                         const Geom& g, uint8_t* q8t, uint8_t* k8t, uint8_t* v8t, float* sq, float* sk,
                         float* qsum, float* ksum, int* wd, cudaStream_t st, int qmax = 127, int q_tok = 0,
                         QKNorm nq = QKNorm(), QKNorm nk = QKNorm());
// Untile the quantised tiles back to row-major codes (parity entry only).
cudaError_t launch_untile(const uint8_t* q8t, const uint8_t* k8t, const uint8_t* v8t, const Geom& g, int8_t* q8,
                          int8_t* k8, uint8_t* v8, cudaStream_t st);
// K3: pooled block means (written to qbar/kbar, [BH][nb][128], required),
// then block scores and the per-query-block top-k list (ascending).
// With zin != NULL also writes the selection bitmask (2*ceil(nb/64) words
// per query block) and Z_i = sum of z_j over the unselected key blocks.
cudaError_t launch_pool_topk(const float* qsum, const float* ksum, const Geom& g, int32_t* idx, float* qbar,
                             float* kbar, const float* zin, float* ztot, uint32_t* selbits, float* zout,
                             cudaStream_t st);
// K4a: per key block h_j = phi(K_j)^T V_j (bf16 mask-GEMM tiles) and z_j.
cudaError_t launch_linear_kv(const void* k, const void* v, const Geom& g, uint8_t* hs, float* z, int* wd,
                             cudaStream_t st, QKNorm nk = QKNorm());
// K4b: H_i = sum over unselected j of h_j, as bf16 operand images [nb][128*128].
cudaError_t launch_linear_sum(const uint8_t* hs, const uint32_t* selbits, const Geom& g, uint16_t* hout, int* wd,
                              cudaStream_t st);
// K4c: y = (phi(Q_i) H_i / phi(Q_i) Z_i) W^T per row, written (bf16) to out.
cudaError_t launch_linear_apply(const void* q, const uint16_t* himg, const float* zl, const uint16_t* wimg,
                                const Geom& g, void* out, int* wd, cudaStream_t st, QKNorm nq = QKNorm());
// proj_w [d][d] -> the bf16 B-operand image read by the flash epilogue.
cudaError_t launch_w_tile(const void* w, uint16_t* wt, cudaStream_t st);
// K5: block-sparse INT8/FP8 flash attention over the index lists.
struct FlashArgs {
  const uint8_t* q8t;
  const uint8_t* k8t;
  const uint8_t* v8t;
  const float* sq;
  const float* sk;
  const float* sv;
  const int32_t* idx;  // [BH][nb][kc]; NULL = dense (every block, ascending)
  void* out;           // bf16 rows of 128 in the Geom's layout
  int add_out;          // 1: out already holds the linear branch y (bf16); add O_s to it
  int q_tok;            // 1: sq holds one Q scale per token ([BH][nq*64]) instead of per 64-token tile
  // Watchdog test of the block-64 kernel (all 0 in a normal call): a grid of
  // dbg_grid CTAs instead of the persistent grid, dbg_spin probes per
  // bounded wait instead of the default, and, for dbg_stall > 0, slot 0's K
  // producer of CTA 0 omits the copies of its step dbg_stall - 1.
  int dbg_grid;
  int dbg_stall;
  long dbg_spin;
};
cudaError_t launch_flash(const FlashArgs& a, const Geom& g, cudaStream_t st, int* wd);
// W8A8 linear layer (k_w8a8.cu).
size_t w8a8_codes_bytes(int rows, int cols);
size_t w8a8_scales_count(int rows, int cols);
cudaError_t launch_w8a8_quant(const void* a, int rows, int cols, uint8_t* codes, float* scales, cudaStream_t st);
cudaError_t launch_w8a8_gemm(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw, void* y, int M,
                             int N, int K, int* wd, cudaStream_t st);
// Waits `probes` times on an mbarrier that never completes, then sets *wd.
cudaError_t launch_watchdog_selftest(int probes, int* wd, cudaStream_t st);

}  // namespace sagesla
