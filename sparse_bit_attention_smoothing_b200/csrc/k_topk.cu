// k_topk.cu -- K3: pooled block scores and the SLA block mask.
//
// "揭秘TurboDiffusion：如何让视频生成实现百倍加速？", 支柱二 SLA: per query block
// only the most important key blocks (the top sla_topk fraction) are computed
// exactly.  Importance is read as the mean-pooled block score
//   sbar_ij = fl32( dot(qbar_i, kbar_j) ) * fl32(1/sqrt(d)),
// qbar_i / kbar_j the means of Q / (K - mu) over the valid rows of block i / j,
// everything in fp32.  The k largest per row are kept, ties going to the
// lower block index, and listed in ascending order.
//
// One CTA: TQ query blocks of one head.  Phase 1 scores all key blocks
// (chunks of kbar staged in shared memory, fp32 FMA); phase 2 selects the
// k-th largest orderable key per row by a 32-step bitwise search with warp
// counts, then compacts the selection in index order.
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

constexpr int kTQ = 8;       // query blocks per CTA (one warp each in phase 2)
constexpr int kKC = 64;      // key blocks per staged chunk
constexpr int kPad = 132;    // padded row length of the kbar chunk (floats)

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Mean over the valid rows of attention block `blk` from the per-64-row sums.
__device__ __forceinline__ float pooled(const float* __restrict__ sums, int blk, int block, int N, int c) {
  const int sub = block / kQB;
  float a = 0.f;
  for (int s = 0; s < sub; ++s) a += sums[(size_t)(blk * sub + s) * kD + c];
  const int n0 = blk * block;
  const int cnt = min(block, N - n0);
  return __fdiv_rn(a, (float)cnt);
}

// Pooled means of every attention block, once: grid (nb, BH), 128 threads.
__global__ void pool_means_kernel(const float* __restrict__ qsum, const float* __restrict__ ksum, int N, int block,
                                  int nb, int nq, float* __restrict__ qbar, float* __restrict__ kbar) {
  const int i = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  qbar[((size_t)bh * nb + i) * kD + c] = pooled(qsum + (size_t)bh * nq * kD, i, block, N, c);
  kbar[((size_t)bh * nb + i) * kD + c] = pooled(ksum + (size_t)bh * nq * kD, i, block, N, c);
}

// Linear-branch outputs (when zin != NULL): selbits [nb][nbw] words with
// bit j set when key block j is selected; zout [nb][128] the fp32 sums
// Z_i = sum_{j not in S_i} z_j, formed as (sum over all j) - (sum over S_i).
__global__ void __launch_bounds__(256) pool_topk_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                        int nb, int kc, int32_t* __restrict__ idx,
                                                        const float* __restrict__ zin,
                                                        uint32_t* __restrict__ selbits, int nbw,
                                                        float* __restrict__ zout) {
  extern __shared__ __align__(16) float sm[];
  float* qb = sm;                            // [kTQ][128]
  float* kb = qb + kTQ * kD;                 // [kKC][kPad]
  float* sc = kb + kKC * kPad;               // [kTQ][nb]
  const int bh = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int i0 = blockIdx.x * kTQ;
  const float* qh = qbar + (size_t)bh * nb * kD;
  const float* kh = kbar + (size_t)bh * nb * kD;
  const float rs = 1.0f / sqrtf((float)kD);

  for (int e = t; e < kTQ * kD; e += 256) {
    const int r = e / kD;
    qb[e] = i0 + r < nb ? qh[(size_t)i0 * kD + e] : 0.f;
  }
  // Phase 1: scores.  Thread -> key block jj = t % 64 of the chunk, query
  // rows 2*(t/64) and 2*(t/64)+1.
  const int jj = t & 63, qg = t >> 6;
  for (int j0 = 0; j0 < nb; j0 += kKC) {
    __syncthreads();
    for (int e = t; e < kKC * kD / 4; e += 256) {
      const int r = e / (kD / 4), c4 = e % (kD / 4);
      const int j = j0 + r;
      const float4 val = j < nb ? *reinterpret_cast<const float4*>(kh + (size_t)j * kD + 4 * c4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(kb + r * kPad + 4 * c4) = val;
    }
    __syncthreads();
    const int j = j0 + jj;
    if (j < nb) {
      float a0 = 0.f, a1 = 0.f;
      const float* kr = kb + jj * kPad;
      const float* q0 = qb + (2 * qg) * kD;
      const float* q1 = q0 + kD;
#pragma unroll 8
      for (int c = 0; c < kD; c += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kr + c);
        const float4 x0 = *reinterpret_cast<const float4*>(q0 + c);
        const float4 x1 = *reinterpret_cast<const float4*>(q1 + c);
        a0 = fmaf(x0.x, k4.x, a0);
        a0 = fmaf(x0.y, k4.y, a0);
        a0 = fmaf(x0.z, k4.z, a0);
        a0 = fmaf(x0.w, k4.w, a0);
        a1 = fmaf(x1.x, k4.x, a1);
        a1 = fmaf(x1.y, k4.y, a1);
        a1 = fmaf(x1.z, k4.z, a1);
        a1 = fmaf(x1.w, k4.w, a1);
      }
      sc[(2 * qg) * nb + j] = a0 * rs;
      sc[(2 * qg + 1) * nb + j] = a1 * rs;
    }
  }
  // Total of z over all key blocks of the head (fixed order), for Z_i.
  __shared__ float ztot[kD];
  if (zin && t < kD) {
    float a = 0.f;
    for (int j = 0; j < nb; ++j) a += zin[((size_t)bh * nb + j) * kD + t];
    ztot[t] = a;
  }
  __syncthreads();
  // Phase 2: one warp per query row.
  const int i = i0 + warp;
  if (i >= nb) return;
  const float* row = sc + warp * nb;
  // Largest T with #{key >= T} >= kc: built bit by bit from the top.
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    int cnt = 0;
    for (int j = lane; j < nb; j += 32) cnt += order_key(row[j]) >= cand ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= kc) T = cand;
  }
  int gt = 0;
  for (int j = lane; j < nb; j += 32) gt += order_key(row[j]) > T ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  const int need_eq = kc - gt;  // >= 1 by construction of T
  int32_t* out = idx + ((size_t)bh * nb + i) * kc;
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < nb ? order_key(row[j]) : 0u;
    const bool is_eq = j < nb && key == T;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eqm & ((1u << lane) - 1u));
    const bool sel = j < nb && (key > T || (is_eq && eq_rank < need_eq));
    const unsigned sm_ = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(sm_ & ((1u << lane) - 1u))] = j;
    if (selbits && lane == 0) selbits[((size_t)bh * nb + i) * nbw + (j0 >> 5)] = sm_;
    pos += __popc(sm_);
    eq_seen += __popc(eqm);
  }
  if (selbits)
    for (int w = ((nb + 31) >> 5) + lane; w < nbw; w += 32) selbits[((size_t)bh * nb + i) * nbw + w] = 0u;
  if (zin) {
    __syncwarp();
    float zs[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) zs[m] = 0.f;
    for (int tt = 0; tt < kc; ++tt) {
      const int j = out[tt];
#pragma unroll
      for (int m = 0; m < 4; ++m) zs[m] += zin[((size_t)bh * nb + j) * kD + lane + 32 * m];
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) zout[((size_t)bh * nb + i) * kD + lane + 32 * m] = ztot[lane + 32 * m] - zs[m];
  }
}

size_t pool_topk_smem(int nb) { return sizeof(float) * ((size_t)kTQ * kD + (size_t)kKC * kPad + (size_t)kTQ * nb); }

cudaError_t launch_pool_topk(const float* qsum, const float* ksum, const Geom& g, int32_t* idx, float* qbar,
                             float* kbar, const float* zin, uint32_t* selbits, float* zout, cudaStream_t st) {
  pool_means_kernel<<<dim3(g.nb, g.BH), kD, 0, st>>>(qsum, ksum, g.N, g.block, g.nb, g.nq, qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = pool_topk_smem(g.nb);
  e = cudaFuncSetAttribute(pool_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  pool_topk_kernel<<<dim3((g.nb + kTQ - 1) / kTQ, g.BH), 256, smem, st>>>(qbar, kbar, g.nb, g.kc, idx, zin, selbits,
                                                                           2 * ((g.nb + 63) / 64), zout);
  return cudaGetLastError();
}

}  // namespace sagesla
