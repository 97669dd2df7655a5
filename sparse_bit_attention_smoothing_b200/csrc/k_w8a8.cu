// k_w8a8.cu -- the W8A8 linear layer: y = x W^T with both operands INT8 in
// 128 x 128 blocks ("揭秘TurboDiffusion：如何让视频生成实现百倍加速？", 支柱三
// W8A8线性层量化; 量子位 news, 技术解密 4: INT8 weights and activations, block
// granularity 128 x 128, run on the INT8 tensor cores).
//
// Quantiser: one fp32 scale per 128 x 128 block, s = fl32(amax/127), code =
// RNE(fl32(x * fl32(127/amax))) clamped to +-127 (amax = 0 -> s = 1, codes
// 0); a short last block of rows is quantised over its valid rows and its
// missing rows are zero codes.  Codes are written as 16 KB tcgen05 operand
// images, one per block: [128 rows][128 K] INT8, K-major, no swizzle (8 x 16 B
// core matrices; LBO 128 B along K, SBO 1024 B along rows), blocks ordered
// [row block][K block].
//
// GEMM: y[m][n] = sum over K blocks kb of s_x[m/128][kb] s_w[n/128][kb]
// (integer dot over the block), fp32 in kb order, bf16 output.  The scale
// changes with every K block, so each block's INT32 product is read out of
// TMEM and folded into fp32 running sums (the promotion) while the tensor
// core computes the next blocks.
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kWB = 128;                 // block edge
constexpr int kWTile = kWB * kWB;        // 16 KB INT8 operand image
constexpr int kStages = 6;               // A + B per stage: 32 KB
constexpr int kAccBufs = 4;              // INT32 accumulators of 128 TMEM columns each
constexpr int kEpiWarps = 8;             // two per TMEM lane quadrant, 64 columns each
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);
constexpr int kGemmSmem = kStages * 2 * kWTile + 1024 + 1024;

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

// ------------------------------------------------------------- quantiser --
// One CTA per 128 x 128 block (grid: cols/128 x ceil(rows/128)), 256
// threads; thread t holds row t/2, columns 64 (t%2) .. +63 of the block.
__global__ void __launch_bounds__(256) w8a8_quant_kernel(const uint16_t* __restrict__ a, int rows, int cols,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scales) {
  __shared__ float red[8];
  const int cb = blockIdx.x, rb = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int r = t >> 1, h = t & 1;
  const int row = rb * kWB + r;
  const bool valid = row < rows;
  const uint4* src = reinterpret_cast<const uint4*>(a + (size_t)(valid ? row : 0) * cols + cb * kWB + 64 * h);
  uint4 v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = valid ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float mult = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
  const int ncb = cols / kWB;
  if (t == 0) scales[(size_t)rb * ncb + cb] = amax > 0.f ? __fdiv_rn(amax, 127.f) : 1.f;
  uint8_t* tile = codes + ((size_t)rb * ncb + cb) * kWTile;
#pragma unroll
  for (int j = 0; j < 8; j += 2) {  // 16 codes = one core-matrix row per store
    const uint32_t w[8] = {v[j].x, v[j].y, v[j].z, v[j].w, v[j + 1].x, v[j + 1].y, v[j + 1].z, v[j + 1].w};
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float f[4] = {bf16_lo(w[2 * e]), bf16_hi(w[2 * e]), bf16_lo(w[2 * e + 1]), bf16_hi(w[2 * e + 1])};
      uint32_t b = 0;
#pragma unroll
      for (int z = 0; z < 4; ++z) {
        int c = __float2int_rn(__fmul_rn(f[z], mult));
        c = max(-127, min(127, c));
        b |= ((uint32_t)c & 0xFFu) << (8 * z);
      }
      pk[e] = b;
    }
    const int c0 = 64 * h + 8 * j;  // first column of these 16 codes
    *reinterpret_cast<uint4*>(tile + kmajor_off(r, c0, 128, 1024)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// ------------------------------------------------------------------ GEMM --
// Persistent: CTA b takes output tiles b, b + gridDim.x, ... (tile t = row
// block t / nN, column block t % nN: the CTAs in flight share a few row
// blocks of x and all of W in L2).  Warp 0: bulk copies of the A (x) and B
// (W) tiles of each K block into a 6-stage ring; warp 1: TMEM allocation and
// the MMAs, four M=128 N=128 K=32 INT8 MMAs per K block into one of four
// 128-column INT32 accumulators; warps 2-9: the promotion, two warps per
// TMEM lane quadrant (64 columns each), and the bf16 store.  Every wait is
// bounded (watchdog).
__global__ void __launch_bounds__(kGemmThreads, 1) w8a8_gemm_kernel(const uint8_t* __restrict__ xq,
                                                                    const float* __restrict__ sx,
                                                                    const uint8_t* __restrict__ wq,
                                                                    const float* __restrict__ sw,
                                                                    __nv_bfloat16* __restrict__ y, int M, int N,
                                                                    int K, int* wd) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  struct Bars {
    uint64_t full[kStages], empty[kStages];
    uint64_t acc_full[kAccBufs], acc_empty[kAccBufs];
    uint64_t fin;
    uint32_t tmem;
    int abort;
  };
  Bars* bars = reinterpret_cast<Bars*>(smem + kStages * 2 * kWTile);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nM = (M + kWB - 1) / kWB, nN = N / kWB, nK = K / kWB;
  const int ntiles = nM * nN;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], kEpiWarps);
    }
    mbar_init(&bars->fin, 1);
    bars->abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        const int mb = t / nN, nb = t - mb * nN;
        for (int kb = 0; kb < nK; ++kb, ++it) {
          const int st = it % kStages;
          if (it >= kStages && !(ok = mbar_wait(&bars->empty[st], ((it / kStages) - 1) & 1, abort, wd))) break;
          uint8_t* dst = smem + st * 2 * kWTile;
          mbar_expect_tx(&bars->full[st], 2 * kWTile);
          bulk_g2s(dst, xq + ((size_t)mb * nK + kb) * kWTile, kWTile, &bars->full[st]);
          bulk_g2s(dst + kWTile, wq + ((size_t)nb * nK + kb) * kWTile, kWTile, &bars->full[st]);
        }
      }
      // Drain: only the stages issued after the last proven-consumed one can
      // still be in flight.
      for (int g = max(0, it - kStages); g < it; ++g) mbar_wait_drain(&bars->full[g % kStages], (g / kStages) & 1, wd);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      const uint64_t d0 = smem_desc(smem, kQK_LBO, kQK_SBO);
      const uint32_t id = idesc_i8(128, 128);
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        for (int kb = 0; kb < nK; ++kb, ++it) {
          const int st = it % kStages, buf = it % kAccBufs;
          if (!(ok = mbar_wait(&bars->full[st], (it / kStages) & 1, abort, wd))) break;
          if (it >= kAccBufs && !(ok = mbar_wait(&bars->acc_empty[buf], ((it / kAccBufs) - 1) & 1, abort, wd))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(tmem + buf * 128, desc_at(d0, st * 2 * kWTile + kk * 256),
                   desc_at(d0, st * 2 * kWTile + kWTile + kk * 256), id, kk > 0);
          mma_commit(&bars->empty[st]);
          mma_commit(&bars->acc_full[buf]);
        }
      }
      mma_commit(&bars->fin);
    }
  } else {
    // ------------------------------ promotion -----------------------------
    const int q = warp & 3;              // TMEM lane quadrant: rows 32q .. 32q+31
    const int hc = (warp - 2) >> 2;      // column half: 64 hc .. 64 hc + 63
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + 64 * hc;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      const int mb = t / nN, nb = t - mb * nN;
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      const float* sxr = sx + (size_t)mb * nK;
      const float* swr = sw + (size_t)nb * nK;
      float c_next = __fmul_rn(__ldg(sxr), __ldg(swr));
      for (int kb = 0; kb < nK; ++kb, ++it) {
        const int buf = it % kAccBufs;
        const float c = c_next;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_full[buf], (it / kAccBufs) & 1, abort, wd));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[64];
        SAGESLA_TMEM_LD32(tl + buf * 128, v);
        SAGESLA_TMEM_LD32(tl + buf * 128 + 32, v + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
        if (kb + 1 < nK) c_next = __fmul_rn(__ldg(sxr + kb + 1), __ldg(swr + kb + 1));
        // |dot| <= 128 * 127 * 127 < 2^22: the float of an INT32 code is its
        // bits added to those of 1.5 * 2^23, minus 1.5 * 2^23 (both exact).
        const uint64_t cc = f32x2_pack(c, c);
        const uint64_t off = f32x2_pack(-12582912.f, -12582912.f);
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const uint64_t f = f32x2_add(
              f32x2_pack(__int_as_float((int)v[j] + 0x4B400000), __int_as_float((int)v[j + 1] + 0x4B400000)), off);
          const uint64_t s = f32x2_fma(f, cc, f32x2_pack(acc[j], acc[j + 1]));
          f32x2_unpack(s, acc[j], acc[j + 1]);
        }
      }
      if (!ok) break;
      const int m = mb * kWB + 32 * q + lane;
      if (m < M) {
        uint4* dst = reinterpret_cast<uint4*>(y + (size_t)m * N + nb * kWB + 64 * hc);
#pragma unroll
        for (int j = 0; j < 64; j += 8)
          dst[j / 8] = make_uint4(pack_bf16x2(acc[j], acc[j + 1]), pack_bf16x2(acc[j + 2], acc[j + 3]),
                                  pack_bf16x2(acc[j + 4], acc[j + 5]), pack_bf16x2(acc[j + 6], acc[j + 7]));
      }
    }
  }
  if (warp == 1) {
    if (lane == 0) mbar_wait_drain(&bars->fin, 0, wd);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t w8a8_codes_bytes(int rows, int cols) { return (size_t)((rows + kWB - 1) / kWB) * (cols / kWB) * kWTile; }
size_t w8a8_scales_count(int rows, int cols) { return (size_t)((rows + kWB - 1) / kWB) * (cols / kWB); }

cudaError_t launch_w8a8_quant(const void* a, int rows, int cols, uint8_t* codes, float* scales, cudaStream_t st) {
  w8a8_quant_kernel<<<dim3(cols / kWB, (rows + kWB - 1) / kWB), 256, 0, st>>>(static_cast<const uint16_t*>(a), rows,
                                                                              cols, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_w8a8_gemm(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw, void* y, int M,
                             int N, int K, int* wd, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = ((M + kWB - 1) / kWB) * (N / kWB);
  const int grid = ntiles < sms ? ntiles : sms;
  cudaError_t e = cudaFuncSetAttribute(w8a8_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  w8a8_gemm_kernel<<<grid, kGemmThreads, kGemmSmem, st>>>(xq, sx, wq, sw, static_cast<__nv_bfloat16*>(y), M, N, K,
                                                          wd);
  return cudaGetLastError();
}

}  // namespace sagesla
