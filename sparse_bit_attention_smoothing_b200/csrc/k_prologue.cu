// k_prologue.cu -- the HBM-bound front of the SageSLA path.
//
// K1  stats:  per (b,h,channel) the mean of K over the N tokens (fp64 sums,
//             rounded once to fp32) and max |V| (for the per-channel FP8
//             scale).  "异常值平滑" / smoothing: 量子位 news 技术解密 1 and
//             揭秘TurboDiffusion 支柱一 SageAttention.
// K2  quant:  Q -> INT8 per 64-token block, K - mu -> INT8 per 64-token
//             block, V -> FP8 E4M3 per channel, written as tensor-core tiles;
//             plus per-64-token column sums of Q and K - mu for the pooled
//             block scores of the SLA mask (揭秘TurboDiffusion 支柱二 SLA).
// Arithmetic that decides a code is done exactly as specified in fp32:
//   ks = fl32(k - mu); mult = fl32(127/amax); code = rne(fl32(x*mult)),
//   clamped to +-127; V: code = e4m3_rne_sat(fl32(v * fl32(448/amax_c))).
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

// ---------------------------------------------------------------- K1 ----
// grid (split, BH), 128 threads.  Thread t covers channels 8*(t%16)..+7 of
// rows t/16, t/16+8, ... of its split.
__global__ void __launch_bounds__(128) stats_partial_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                            int N, int rows_per_split, double* __restrict__ psum,
                                                            float* __restrict__ pmax) {
  const int bh = blockIdx.y, sp = blockIdx.x, t = threadIdx.x;
  const int cg = t & 15, r0 = t >> 4;
  const int n_begin = sp * rows_per_split;
  const int n_end = min(N, n_begin + rows_per_split);
  double s[8];
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s[i] = 0.0;
    m[i] = 0.f;
  }
  const size_t base = (size_t)bh * N * 16;  // in uint4 (8 bf16) units
#pragma unroll 4
  for (int n = n_begin + r0; n < n_end; n += 8) {  // unrolled: four row pairs of loads in flight
    uint4 kk = __ldg(k + base + (size_t)n * 16 + cg);
    uint4 vv = __ldg(v + base + (size_t)n * 16 + cg);
    uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w};
    uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s[2 * i] += (double)bf16_lo(kw[i]);
      s[2 * i + 1] += (double)bf16_hi(kw[i]);
      m[2 * i] = fmaxf(m[2 * i], fabsf(bf16_lo(vw[i])));
      m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16_hi(vw[i])));
    }
  }
  __shared__ double ss[8][128];
  __shared__ float sm[8][128];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ss[r0][cg * 8 + i] = s[i];
    sm[r0][cg * 8 + i] = m[i];
  }
  __syncthreads();
  double a = 0.0;
  float b = 0.f;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    a += ss[r][t];
    b = fmaxf(b, sm[r][t]);
  }
  const size_t o = ((size_t)bh * gridDim.x + sp) * kD + t;
  psum[o] = a;
  pmax[o] = b;
}

// grid BH, 128 threads (one per channel); fixed summation order over splits.
__global__ void stats_final_kernel(const double* __restrict__ psum, const float* __restrict__ pmax, int split, int N,
                                   float* __restrict__ mu, float* __restrict__ sv, float* __restrict__ mv) {
  const int bh = blockIdx.x, c = threadIdx.x;
  double a = 0.0;
  float b = 0.f;
  for (int s = 0; s < split; ++s) {
    a += psum[((size_t)bh * split + s) * kD + c];
    b = fmaxf(b, pmax[((size_t)bh * split + s) * kD + c]);
  }
  mu[(size_t)bh * kD + c] = (float)(a / (double)N);
  sv[(size_t)bh * kD + c] = b > 0.f ? __fdiv_rn(b, 448.f) : 1.f;
  mv[(size_t)bh * kD + c] = b > 0.f ? __fdiv_rn(448.f, b) : 0.f;
}

// ---------------------------------------------------------------- K2 ----
// grid (nq, BH), 128 threads: one 64-token tile of Q, K and V.
// Thread t handles channel group cg = t/8 (8 channels) of rows t%8 + 8*i:
// the lanes of a warp span 8 rows and 4 channel groups, which keeps the
// stores into the tile images (whose channel groups lie 512 or 1024 bytes
// apart, one bank) at most 4-way conflicted.
__device__ __forceinline__ float block_max128(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  float r = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return r;
}

// rne(fl32(x * mult)) as a byte.  |x| <= amax and mult = fl32(127/amax), so
// the product lies within 127 * (1 + 2^-23) and no clamp is needed; adding
// 1.5 * 2^23 rounds it to the nearest integer (ties to even) in the low
// mantissa bits, on the FMA pipe rather than the conversion unit.
__device__ __forceinline__ uint32_t i8code(float x, float mult) {
  return (uint32_t)__float_as_int(__fadd_rn(__fmul_rn(x, mult), 12582912.0f)) & 0xFFu;
}

__global__ void __launch_bounds__(128) quant_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                    const uint4* __restrict__ v, const float* __restrict__ mu,
                                                    const float* __restrict__ mv, int N, int nq,
                                                    uint8_t* __restrict__ q8t, uint8_t* __restrict__ k8t,
                                                    uint8_t* __restrict__ v8t, float* __restrict__ sq,
                                                    float* __restrict__ sk, float* __restrict__ qsum,
                                                    float* __restrict__ ksum) {
  const int bh = blockIdx.y, tile = blockIdx.x, t = threadIdx.x;
  const int cg = t >> 3, rr = t & 7;
  const int n0 = tile * kQB;
  __shared__ __align__(16) uint8_t sq8[kTile];
  __shared__ __align__(16) uint8_t sk8[kTile];
  __shared__ __align__(16) uint8_t sv8[kTile];
  __shared__ float red[4];
  __shared__ float psq[8][kD];
  __shared__ float psk[8][kD];

  float muc[8], mvc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    muc[i] = mu[(size_t)bh * kD + cg * 8 + i];
    mvc[i] = mv[(size_t)bh * kD + cg * 8 + i];
  }
  // Load this thread's 8 rows x 8 channels of Q, K, V (zeros past N).
  float xq[8][8], xk[8][8];
  uint32_t vw[8][4];
  const size_t base = (size_t)bh * N * 16;
  float aq = 0.f, ak = 0.f;
  float sumq[8], sumk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sumq[i] = 0.f;
    sumk[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = rr + 8 * i;
    const int n = n0 + r;
    uint4 qq = make_uint4(0, 0, 0, 0), kk = qq, vv = qq;
    const bool valid = n < N;
    if (valid) {
      qq = __ldg(q + base + (size_t)n * 16 + cg);
      kk = __ldg(k + base + (size_t)n * 16 + cg);
      vv = __ldg(v + base + (size_t)n * 16 + cg);
    }
    uint32_t qw[4] = {qq.x, qq.y, qq.z, qq.w};
    uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w};
    vw[i][0] = vv.x;
    vw[i][1] = vv.y;
    vw[i][2] = vv.z;
    vw[i][3] = vv.w;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xq[i][2 * j] = bf16_lo(qw[j]);
      xq[i][2 * j + 1] = bf16_hi(qw[j]);
      xk[i][2 * j] = valid ? __fsub_rn(bf16_lo(kw[j]), muc[2 * j]) : 0.f;
      xk[i][2 * j + 1] = valid ? __fsub_rn(bf16_hi(kw[j]), muc[2 * j + 1]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      aq = fmaxf(aq, fabsf(xq[i][j]));
      ak = fmaxf(ak, fabsf(xk[i][j]));
      sumq[j] += xq[i][j];
      sumk[j] += xk[i][j];
    }
  }
  aq = block_max128(aq, red);
  ak = block_max128(ak, red);
  const float mq = aq > 0.f ? __fdiv_rn(127.f, aq) : 0.f;
  const float mk = ak > 0.f ? __fdiv_rn(127.f, ak) : 0.f;
  if (t == 0) {
    sq[(size_t)bh * nq + tile] = aq > 0.f ? __fdiv_rn(aq, 127.f) : 1.f;
    sk[(size_t)bh * nq + tile] = ak > 0.f ? __fdiv_rn(ak, 127.f) : 1.f;
  }
  // Codes into the smem tile images.
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = rr + 8 * i;
    uint32_t qa = 0, qb = 0, ka = 0, kb = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      qa |= i8code(xq[i][j], mq) << (8 * j);
      qb |= i8code(xq[i][j + 4], mq) << (8 * j);
      ka |= i8code(xk[i][j], mk) << (8 * j);
      kb |= i8code(xk[i][j + 4], mk) << (8 * j);
    }
    const uint32_t off = kmajor_off(r, cg * 8, kQK_LBO, kQK_SBO);
    *reinterpret_cast<uint2*>(sq8 + off) = make_uint2(qa, qb);
    *reinterpret_cast<uint2*>(sk8 + off) = make_uint2(ka, kb);
    // V^T tile: element (channel c, key r).
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c0 = cg * 8 + 2 * j;
      const float v0 = __fmul_rn(bf16_lo(vw[i][j]), mvc[2 * j]);
      const float v1 = __fmul_rn(bf16_hi(vw[i][j]), mvc[2 * j + 1]);
      const uint32_t pr = e4m3x2(v0, v1);
      sv8[kmajor_off(c0, r, kV_LBO, kV_SBO)] = (uint8_t)(pr & 0xFF);
      sv8[kmajor_off(c0 + 1, r, kV_LBO, kV_SBO)] = (uint8_t)(pr >> 8);
    }
  }
  // Pooled column sums over this tile's valid rows.
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    psq[rr][cg * 8 + j] = sumq[j];
    psk[rr][cg * 8 + j] = sumk[j];
  }
  __syncthreads();
  {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      a += psq[r][t];
      b += psk[r][t];
    }
    qsum[((size_t)bh * nq + tile) * kD + t] = a;
    ksum[((size_t)bh * nq + tile) * kD + t] = b;
  }
  // Coalesced 16-byte copies of the three 8 KB tiles.
  const size_t tb = ((size_t)bh * nq + tile) * kTile;
#pragma unroll
  for (int i = 0; i < kTile / 16 / 128; ++i) {
    const int o = (t + i * 128) * 16;
    *reinterpret_cast<uint4*>(q8t + tb + o) = *reinterpret_cast<const uint4*>(sq8 + o);
    *reinterpret_cast<uint4*>(k8t + tb + o) = *reinterpret_cast<const uint4*>(sk8 + o);
    *reinterpret_cast<uint4*>(v8t + tb + o) = *reinterpret_cast<const uint4*>(sv8 + o);
  }
}

// Row-major codes from the tiles (parity entry point only).
__global__ void untile_kernel(const uint8_t* __restrict__ q8t, const uint8_t* __restrict__ k8t,
                              const uint8_t* __restrict__ v8t, int N, int nq, int8_t* __restrict__ q8,
                              int8_t* __restrict__ k8, uint8_t* __restrict__ v8) {
  const int bh = blockIdx.y;
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;  // element within head
  if (e >= (size_t)N * kD) return;
  const int n = (int)(e / kD), c = (int)(e % kD);
  const int tile = n / kQB, r = n % kQB;
  const size_t tb = ((size_t)bh * nq + tile) * kTile;
  const size_t o = (size_t)bh * N * kD + e;
  q8[o] = (int8_t)q8t[tb + kmajor_off(r, c, kQK_LBO, kQK_SBO)];
  k8[o] = (int8_t)k8t[tb + kmajor_off(r, c, kQK_LBO, kQK_SBO)];
  v8[o] = v8t[tb + kmajor_off(c, r, kV_LBO, kV_SBO)];
}

cudaError_t launch_stats_partial(const void* k, const void* v, const Geom& g, double* psum, float* pmax,
                                 cudaStream_t st) {
  const int rows = (g.N + g.split - 1) / g.split;
  stats_partial_kernel<<<dim3(g.split, g.BH), 128, 0, st>>>((const uint4*)k, (const uint4*)v, g.N, rows, psum, pmax);
  return cudaGetLastError();
}

cudaError_t launch_stats_final(const double* psum, const float* pmax, const Geom& g, float* mu, float* sv, float* mv,
                               cudaStream_t st) {
  stats_final_kernel<<<g.BH, kD, 0, st>>>(psum, pmax, g.split, g.N, mu, sv, mv);
  return cudaGetLastError();
}

cudaError_t launch_quant(const void* q, const void* k, const void* v, const float* mu, const float* mv, const Geom& g,
                         uint8_t* q8t, uint8_t* k8t, uint8_t* v8t, float* sq, float* sk, float* qsum, float* ksum,
                         cudaStream_t st) {
  quant_kernel<<<dim3(g.nq, g.BH), 128, 0, st>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, mu, mv, g.N, g.nq,
                                                 q8t, k8t, v8t, sq, sk, qsum, ksum);
  return cudaGetLastError();
}

cudaError_t launch_untile(const uint8_t* q8t, const uint8_t* k8t, const uint8_t* v8t, const Geom& g, int8_t* q8,
                          int8_t* k8, uint8_t* v8, cudaStream_t st) {
  const size_t per = (size_t)g.N * kD;
  untile_kernel<<<dim3((unsigned)((per + 255) / 256), g.BH), 256, 0, st>>>(q8t, k8t, v8t, g.N, g.nq, q8, k8, v8);
  return cudaGetLastError();
}

}  // namespace sagesla
