// k_linear.cu -- the SLA linear-attention branch.
//
// "揭秘TurboDiffusion：如何让视频生成实现百倍加速？" 支柱二 SLA and
// "TurboDiffusion跨模态" 2.2: besides the exactly computed blocks, a light
// global linear-attention component (kernel-function approximation) covers
// the rest.  Read as phi(Q)(phi(K)^T V) over the key blocks NOT selected for
// query block i, phi = elu + 1, from the raw bf16 Q, K, V:
//   h_j = phi(K_j)^T V_j  (d x d),  z_j = sum of the rows of phi(K_j)
//   H_i = sum_{j not in S_i} h_j   (a 0/1 complement-mask GEMM per head)
//
// K4a linear_kv:  per key block, h_j on tcgen05 (kind::f16, both operands
//   MN-major, staged from the token-major rows), fp32 accumulate, stored in
//   bf16 as the B tiles of the mask GEMM; z_j in fp32.
// K4b linear_sum: per head, H = (1 - M) . Hstack with tcgen05 (M=128 query
//   blocks x N=256 columns of the d*d matrices, K = key blocks); the 0/1 A
//   tiles are expanded in shared memory from the selection bitmask.  Each
//   output row is the bf16 image of H_i^T in the operand layout the
//   linear_apply kernel's MMA reads (one bulk copy there).
// K4c linear_apply: y = (phi(Q) H_i / phi(Q) Z_i) W^T into `out`, to which
//   the flash kernel adds the sparse output.
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

// Layout of H_i^T as a K-major bf16 B operand [N = cv][K = ck]:
// element (cv, ck) at (cv/8)*2048 + (ck/8)*128 + (cv%8)*16 + (ck%8)*2 bytes.
__device__ __forceinline__ uint32_t himg_off(uint32_t cv, uint32_t ck) {
  return (cv >> 3) * 2048u + (ck >> 3) * 128u + (cv & 7u) * 16u + (ck & 7u) * 2u;
}

// Mask-GEMM B tiles (64 key blocks x 256 image columns), MN-major: element
// (j, n) at (n%256/8)*1024 + (j%64/8)*128 + (j%8)*16 + (n%8)*2 within the
// 32 KB tile of (j/64, n/256).  Tiles ordered [n/256][j/64].
constexpr int kHsTile = 64 * 256 * 2;  // 32 KB
constexpr uint32_t kHs_LBO = 128, kHs_SBO = 1024;

__device__ __forceinline__ size_t hs_chunk(int nbt, int j, int chunk) {
  // chunk = n / 8 (16-byte group of 8 bf16)
  const int nt = chunk >> 5, c = chunk & 31;
  return ((size_t)nt * nbt + (j >> 6)) * kHsTile + (size_t)c * kHs_SBO + ((j & 63) >> 3) * kHs_LBO + (j & 7) * 16;
}

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

// ---------------------------------------------------------------- K4a ----
// grid (nbt*64, BH): CTA x handles key block j = x (zeros past nb, so the
// mask-GEMM tiles hold no garbage).  256 threads; thread t owns channels
// 8*(t%16).. and token rows t/16 + 16r of 64-row rounds: all its K and V
// loads of a round are issued before any is used.  Small CTAs (128 TMEM
// columns, ~40 KB of shared memory) so that four share an SM and their load
// phases overlap each other's compute.  Thread 0 issues the MMAs.  Dynamic
// smem: A (phi(K) rows) and B (V rows) MN-major, BLK x 128 bf16 each; after
// the MMAs the h image goes from TMEM straight to the mask-GEMM tiles.
template <int BLK>
__global__ void __launch_bounds__(256, 4) linear_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                           int N, int nb, int nbt, uint8_t* __restrict__ hs,
                                                           float* __restrict__ z, int* wd, const QKNorm nk) {
  constexpr int kOpBytes = BLK * 128 * 2;  // one operand tile
  constexpr uint32_t kSBO = (BLK / 8) * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  __shared__ float zred[16][kD];
  const int bh = blockIdx.y, t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int j = blockIdx.x;
  const size_t base = (size_t)bh * N * 16;
  if (t == 0) {
    mbar_init(&bar, 1);
    abort_s = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&tmem_s, 128);
  const int cg = t & 15, r0 = t >> 4;
  float zacc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) zacc[c] = 0.f;
#pragma unroll
  for (int rd = 0; rd < BLK / 64; ++rd) {
    uint4 kk[4], vv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = 64 * rd + r0 + 16 * r, n = j * BLK + row;
      const bool valid = j < nb && n < N;
      kk[r] = valid ? __ldg(k + base + (size_t)n * 16 + cg) : make_uint4(0, 0, 0, 0);
      vv[r] = valid ? __ldg(v + base + (size_t)n * 16 + cg) : make_uint4(0, 0, 0, 0);
    }
    if (nk.inv) {  // QK RMSNorm of the key rows
      const uint4 gk = __ldg(nk.gamma + (bh % nk.H) * 16 + cg);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int n = j * BLK + 64 * rd + r0 + 16 * r;
        if (j < nb && n < N) kk[r] = rms_row8(kk[r], __ldg(nk.inv + (size_t)(bh / nk.H) * N + n), gk);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = 64 * rd + r0 + 16 * r, n = j * BLK + row;
      const bool valid = j < nb && n < N;
      const uint32_t kw[4] = {kk[r].x, kk[r].y, kk[r].z, kk[r].w};
      uint32_t pw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float f0 = valid ? phi(bf16_lo(kw[e])) : 0.f;
        const float f1 = valid ? phi(bf16_hi(kw[e])) : 0.f;
        zacc[2 * e] += f0;
        zacc[2 * e + 1] += f1;
        pw[e] = pack_bf16(f0, f1);
      }
      // MN-major core matrix: (m/8)*SBO + (tok/8)*128 + (tok%8)*16 + (m%8)*2
      const uint32_t off = cg * kSBO + (row >> 3) * 128 + (row & 7) * 16;
      *reinterpret_cast<uint4*>(smem + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      *reinterpret_cast<uint4*>(smem + kOpBytes + off) = vv[r];
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  // h_j^T = V_j^T phi(K_j): A = the V rows (M = value channel cv), B = the
  // phi(K) rows (N = key channel ck), so TMEM lane cv, column ck holds
  // h_j[ck][cv] and each thread later owns 8 consecutive ck of one cv: one
  // 16-byte chunk of the image.
  if (t == 0) {
    const uint32_t id = idesc_bf16(128, 128, 1) | (1u << 15);  // A and B MN-major
#pragma unroll
    for (int ks = 0; ks < BLK / 16; ++ks)
      mma_bf16(tmem, smem_desc(smem + kOpBytes + ks * 256, 128, kSBO), smem_desc(smem + ks * 256, 128, kSBO), id,
               ks > 0);
    mma_commit(&bar);
  }
  // z_j: the 16 row slots' channel sums, added in slot order.
#pragma unroll
  for (int c = 0; c < 8; ++c) zred[r0][cg * 8 + c] = zacc[c];
  __syncthreads();
  if (t < kD) {
    float a = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) a += zred[r][t];
    if (j < nb) z[((size_t)bh * nb + j) * kD + t] = a;
  }
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0, &abort_s, wd));
  tc_fence_after();
  // Warp w holds cv = 32(w%4) + lane, columns ck in [64(w/4), +64); every
  // 8 columns are one 16-byte chunk of the bf16 image of H^T (element (cv,
  // ck) at himg_off), stored straight into its place in the mask-GEMM tile.
  {
    const int cv = 32 * (warp & 3) + lane, cb = 64 * (warp >> 2);
    uint8_t* hsb = hs + (size_t)bh * nbt * 64 * 16384 * 2;
#pragma unroll 1
    for (int c0 = cb; c0 < cb + 64; c0 += 16) {
      uint32_t r[16];
      SAGESLA_TMEM_LD16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w4[e] = ok ? pack_bf16(__uint_as_float(r[8 * h + 2 * e]), __uint_as_float(r[8 * h + 2 * e + 1])) : 0u;
        const int chunk = (int)(himg_off(cv, c0 + 8 * h) >> 4);
        *reinterpret_cast<uint4*>(hsb + hs_chunk(nbt, j, chunk)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------- K4b ----
// grid (ceil(nb/256), 64 n-tiles, BH): the CTAs that read the same B tiles
// are neighbours in launch order.  A CTA covers two M=128 tiles of query
// blocks, so each B tile it loads feeds two MMA chains.  320 threads: warp 0
// bulk-loads the B tiles, warp 1 issues MMAs, warps 2-9 expand the 0/1 A
// tiles from the selection bitmask and run the epilogue.  K tiles of 64 key
// blocks, 3-stage ring; D = 2 x (128 x 256) fp32 in TMEM.
namespace {
constexpr int kLStages = 3;
constexpr int kSumTiles = 2;          // M=128 query-block tiles per CTA
constexpr int kATile = 128 * 64 * 2;  // 16 KB per M tile
constexpr int kAThreads = 128 * kSumTiles;
struct LBars {
  uint64_t b_full[kLStages], a_full[kLStages], empty[kLStages], done;
  uint32_t tmem;
  int abort;
};
}  // namespace

__global__ void __launch_bounds__(64 + kAThreads, 1) linear_sum_kernel(const uint8_t* __restrict__ hs,
                                                             const uint32_t* __restrict__ selbits, int nb, int nbt,
                                                             int nbw, uint16_t* __restrict__ hout, int* wd) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;                               // kLStages x 32 KB
  uint8_t* sA = smem + kLStages * kHsTile;          // kLStages x kSumTiles x 16 KB
  LBars* bars = reinterpret_cast<LBars*>(sA + kLStages * kSumTiles * kATile);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int it = blockIdx.x, nt = blockIdx.y, bh = blockIdx.z;
  const int i0 = it * 128 * kSumTiles;
  const uint8_t* hs_head = hs + (size_t)bh * nbt * 64 * 16384 * 2;
  if (tid == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&bars->b_full[s], 1);
      mbar_init(&bars->a_full[s], kAThreads);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < nbt && !*abort; ++kt) {
        const int st = kt % kLStages;
        if (kt >= kLStages && !mbar_wait(&bars->empty[st], ((kt / kLStages) - 1) & 1, abort, wd)) break;
        mbar_expect_tx(&bars->b_full[st], kHsTile);
        bulk_g2s(sB + st * kHsTile, hs_head + ((size_t)nt * nbt + kt) * kHsTile, kHsTile, &bars->b_full[st]);
        issued = kt + 1;
      }
      for (int kt = (issued > kLStages ? issued - kLStages : 0); kt < issued; ++kt)
        mbar_wait_drain(&bars->b_full[kt % kLStages], (kt / kLStages) & 1, wd);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(128, 256, 1);  // B MN-major
      bool ok = true;
      for (int kt = 0; kt < nbt && ok; ++kt) {
        const int st = kt % kLStages;
        ok = mbar_wait(&bars->a_full[st], (kt / kLStages) & 1, abort, wd) &&
             mbar_wait(&bars->b_full[st], (kt / kLStages) & 1, abort, wd);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int u = 0; u < kSumTiles; ++u)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tmem + u * 256, smem_desc(sA + (st * kSumTiles + u) * kATile + ks * 256, kQK_LBO, kQK_SBO),
                     smem_desc(sB + st * kHsTile + ks * 2 * kHs_LBO, kHs_LBO, kHs_SBO), id, (kt > 0 || ks > 0));
        mma_commit(&bars->empty[st]);
      }
      mma_commit(&bars->done);
      mbar_wait_drain(&bars->done, 0, wd);
    }
  } else {
    // A producer: thread -> query block row i = i0 + (tid - 64); 64 key
    // blocks per K tile from two bitmask words; 1 = NOT selected, j < nb.
    const int u = (tid - 64) >> 7, r = (tid - 64) & 127;
    const int i = i0 + 128 * u + r;
    bool ok = true;
    for (int kt = 0; kt < nbt; ++kt) {
      const int st = kt % kLStages;
      if (kt >= kLStages) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->empty[st], ((kt / kLStages) - 1) & 1, abort, wd));
        if (!ok) break;
      }
      // ones = NOT selected and j < nb (and i < nb), as 64 bits
      uint64_t ones = 0;
      if (i < nb) {
        const uint64_t w = (uint64_t)selbits[((size_t)bh * nb + i) * nbw + 2 * kt] |
                           ((uint64_t)selbits[((size_t)bh * nb + i) * nbw + 2 * kt + 1] << 32);
        const int left = nb - kt * 64;  // key blocks of this tile that exist
        ones = ~w & (left >= 64 ? ~0ull : ((1ull << left) - 1ull));
      }
      uint8_t* A = sA + (st * kSumTiles + u) * kATile;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {  // 8 keys per 16-byte chunk
        const uint32_t b8 = (uint32_t)(ones >> (8 * ch)) & 0xFFu;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)  // bf16 1.0 = 0x3F80 in each half whose bit is set
          pk[e] = (((b8 >> (2 * e)) & 1u) * 0x3F80u) | (((b8 >> (2 * e + 1)) & 1u) * 0x3F800000u);
        *reinterpret_cast<uint4*>(A + kmajor_off(r, ch * 16, kQK_LBO, kQK_SBO)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->a_full[st]);
    }
    // Epilogue: row i of D (256 fp32 columns) -> bf16 image columns.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, abort, wd));
    if (ok) {
      tc_fence_after();
      const int q = warp & 3, ue = (warp - 2) >> 2;  // TMEM quadrant, M tile
      const int row = 32 * q + lane;  // TMEM lane == row of the M=128 tile
      const int ir = i0 + 128 * ue + row;
      uint16_t* dst = hout + ((size_t)bh * nb + (ir < nb ? ir : 0)) * 16384 + (size_t)nt * 256;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 16) {
        uint32_t v16[16];
        SAGESLA_TMEM_LD16(tmem + ((uint32_t)(32 * q) << 16) + ue * 256 + c0, v16);
        tmem_ld_wait();
        if (ir < nb) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(__uint_as_float(v16[2 * e]), __uint_as_float(v16[2 * e + 1]));
          *reinterpret_cast<uint4*>(dst + c0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(dst + c0 + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- K4c ----
// linear_apply: y_r = (phi(q_r) H_i / phi(q_r) Z_i) W^T for every row r of
// query block i, written (bf16) into `out`; the flash kernel adds O_s to it.
// Block 64: two query blocks per CTA whose M=64 accumulators share TMEM at
// lane offsets 0 / 16 (all 128 threads hold a row); block 128: M = 128.
// 128 threads; thread 0 issues the copies and MMAs.  TMEM: num (128 cols) and
// y (128 cols).  Shared: H images (the W image replaces them once num is
// done, so two CTAs fit on an SM), phi(Q) (reused for O_l).
template <int MODE>
__global__ void __launch_bounds__(128) linear_apply_kernel(const uint16_t* __restrict__ q,
                                                           const uint8_t* __restrict__ himg,
                                                           const float* __restrict__ zl,
                                                           const uint8_t* __restrict__ wimg, int N, int nb,
                                                           __nv_bfloat16* __restrict__ out, int* wd,
                                                           const QKNorm nq) {
  constexpr int kImg = 32768;
  constexpr int nH = MODE == 0 ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sH = smem;                       // nH x 32 KB: H images, then the W image
  uint8_t* sW = smem;                       // (W lands where H was once num is done)
  uint8_t* sA = smem + nH * kImg;           // 32 KB: phi(Q), then O_l
  __shared__ uint64_t bar_in, bar_n, bar_y, bar_w;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int bh = blockIdx.y;
  const int iA = MODE == 0 ? 2 * (int)blockIdx.x : (int)blockIdx.x;
  const int iB = MODE == 0 ? iA + 1 : -1;
  const bool hasB = MODE == 0 && iB < nb;
  if (t == 0) {
    mbar_init(&bar_in, 1);
    mbar_init(&bar_n, 1);
    mbar_init(&bar_y, 1);
    mbar_init(&bar_w, 1);
    abort_s = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&tmem_s, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  if (t == 0) {
    mbar_expect_tx(&bar_in, nH * kImg);
    for (int x = 0; x < nH; ++x) {
      const int i = (x == 0 || !hasB) ? iA : iB;
      bulk_g2s(sH + x * kImg, himg + ((size_t)bh * nb + i) * kImg, kImg, &bar_in);
    }
  }
  // Row of this thread (same TMEM lane mapping as the flash kernel).
  int row, i;
  bool active;
  if (MODE == 0) {
    row = 16 * warp + (lane & 15);
    i = lane >= 16 ? iB : iA;
    active = lane >= 16 ? hasB : true;
  } else {
    row = 32 * warp + lane;
    i = iA;
    active = true;
  }
  const int blk = MODE == 0 ? 64 : 128;
  const int n = i * blk + row;
  const bool store = active && n < N;
  const int xo = (MODE == 0 && lane >= 16) ? 1 : 0;
  uint8_t* arow = sA + xo * (kImg / 2);
  const uint4* qrow = reinterpret_cast<const uint4*>(q + ((size_t)bh * N + (store ? n : 0)) * kD);
  const float4* zrow = reinterpret_cast<const float4*>(zl + ((size_t)bh * nb + (active ? i : 0)) * kD);
  float den = 0.f;
  uint4 qq[16];
#pragma unroll
  for (int ch = 0; ch < 16; ++ch) qq[ch] = store ? __ldg(qrow + ch) : make_uint4(0, 0, 0, 0);
  if (nq.inv && store) {  // QK RMSNorm of the query row
    const float inv = __ldg(nq.inv + (size_t)(bh / nq.H) * N + n);
    const uint4* gq = nq.gamma + (bh % nq.H) * 16;
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) qq[ch] = rms_row8(qq[ch], inv, __ldg(gq + ch));
  }
#pragma unroll
  for (int ch = 0; ch < 16; ++ch) {
    const uint32_t w4[4] = {qq[ch].x, qq[ch].y, qq[ch].z, qq[ch].w};
    const float4 z0 = __ldg(zrow + 2 * ch), z1 = __ldg(zrow + 2 * ch + 1);
    const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = phi(bf16_lo(w4[e])), b = phi(bf16_hi(w4[e]));
      den = fmaf(a, zz[2 * e], den);
      den = fmaf(b, zz[2 * e + 1], den);
      pk[e] = pack_bf16(a, b);
    }
    *reinterpret_cast<uint4*>(arow + kmajor_off(row, ch * 16, 128, 2048)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  fence_proxy_async_smem();
  __syncthreads();
  const int M = MODE == 0 ? 64 : 128;
  const uint32_t id = idesc_bf16(M, 128);
  const int nx = MODE == 0 ? (hasB ? 2 : 1) : 1;
  if (t == 0) {
    if (mbar_wait(&bar_in, 0, &abort_s, wd)) {
      tc_fence_after();
      for (int x = 0; x < nx; ++x) {
        const uint32_t d = tmem + ((uint32_t)(x * 16) << 16);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16(d, smem_desc(sA + x * (kImg / 2) + ks * 256, 128, 2048), smem_desc(sH + x * kImg + ks * 256, 128, 2048),
                   id, ks > 0);
      }
    }
    mma_commit(&bar_n);
  }
  bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_n, 0, &abort_s, wd));
  tc_fence_after();
  // The MMAs are done reading H: bring the W image (L2-resident) into its
  // place while num becomes O_l.
  if (t == 0) {
    mbar_expect_tx(&bar_w, kImg);
    bulk_g2s(sW, wimg, kImg, &bar_w);
  }
  const uint32_t lb = (uint32_t)(32 * warp) << 16;
  {
    const float inv_den = (store && den > 0.f) ? 1.f / den : 0.f;
#pragma unroll 1
    for (int c = 0; c < kD; c += 16) {
      uint32_t v16[16];
      SAGESLA_TMEM_LD16(tmem + lb + c, v16);
      tmem_ld_wait();
      uint32_t pk[8];
#pragma unroll
      for (int z2 = 0; z2 < 8; ++z2)
        pk[z2] = pack_bf16(ok ? __uint_as_float(v16[2 * z2]) * inv_den : 0.f,
                           ok ? __uint_as_float(v16[2 * z2 + 1]) * inv_den : 0.f);
      *reinterpret_cast<uint4*>(arow + kmajor_off(row, c * 2, 128, 2048)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(arow + kmajor_off(row, c * 2 + 16, 128, 2048)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (t == 0) {
    tc_fence_after();
    if (ok && mbar_wait(&bar_w, 0, &abort_s, wd)) {
      for (int x = 0; x < nx; ++x) {
        const uint32_t d = tmem + 128 + ((uint32_t)(x * 16) << 16);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16(d, smem_desc(sA + x * (kImg / 2) + ks * 256, 128, 2048), smem_desc(sW + ks * 256, 128, 2048), id,
                   ks > 0);
      }
    }
    mma_commit(&bar_y);
  }
  ok = __all_sync(0xffffffffu, mbar_wait(&bar_y, 0, &abort_s, wd)) && ok;
  tc_fence_after();
  __nv_bfloat16* orow = out + ((size_t)bh * N + (store ? n : 0)) * kD;
#pragma unroll 1
  for (int c = 0; c < kD; c += 16) {
    uint32_t v16[16];
    SAGESLA_TMEM_LD16(tmem + lb + 128 + c, v16);
    tmem_ld_wait();
    if (store) {
      uint32_t pk[8];
#pragma unroll
      for (int z2 = 0; z2 < 8; ++z2)
        pk[z2] = pack_bf16(ok ? __uint_as_float(v16[2 * z2]) : 0.f, ok ? __uint_as_float(v16[2 * z2 + 1]) : 0.f);
      *reinterpret_cast<uint4*>(orow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(orow + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
  }
  // The inputs' bulk copies must have landed before the CTA exits.
  if (t == 0) {
    mbar_wait_drain(&bar_in, 0, wd);
    mbar_wait_drain(&bar_w, 0, wd);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

int linear_apply_smem(int block) { return (block == 64 ? 3 : 2) * 32768 + 1024; }

cudaError_t launch_linear_apply(const void* q, const uint16_t* himg, const float* zl, const uint16_t* wimg,
                                const Geom& g, void* out, int* wd, cudaStream_t st, QKNorm nq) {
  const int smem = linear_apply_smem(g.block);
  cudaError_t e;
  if (g.block == 64) {
    e = cudaFuncSetAttribute(linear_apply_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<0><<<dim3((g.nb + 1) / 2, g.BH), 128, smem, st>>>(
        (const uint16_t*)q, (const uint8_t*)himg, zl, (const uint8_t*)wimg, g.N, g.nb, (__nv_bfloat16*)out, wd, nq);
  } else {
    e = cudaFuncSetAttribute(linear_apply_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<1><<<dim3(g.nb, g.BH), 128, smem, st>>>(
        (const uint16_t*)q, (const uint8_t*)himg, zl, (const uint8_t*)wimg, g.N, g.nb, (__nv_bfloat16*)out, wd, nq);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------- W image ---
// proj_w [c_out][c_in] row-major -> K-major B operand image [N=c_out][K=c_in].
__global__ void w_tile_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ wt) {
  const int co = blockIdx.x, ci = threadIdx.x;
  wt[himg_off(co, ci) / 2] = w[co * kD + ci];
}

int linear_kv_smem(int block) { return 2 * block * 128 * 2 + 1024; }
int linear_sum_smem() { return kLStages * (kHsTile + kSumTiles * kATile) + (int)sizeof(LBars) + 1024; }

cudaError_t launch_linear_kv(const void* k, const void* v, const Geom& g, uint8_t* hs, float* z, int* wd,
                             cudaStream_t st, QKNorm nk) {
  const int nbt = (g.nb + 63) / 64;
  const int smem = linear_kv_smem(g.block);
  cudaError_t e;
  if (g.block == 64) {
    e = cudaFuncSetAttribute(linear_kv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    linear_kv_kernel<64><<<dim3(nbt * 64, g.BH), 256, smem, st>>>((const uint4*)k, (const uint4*)v, g.N, g.nb, nbt, hs,
                                                                  z, wd, nk);
  } else {
    e = cudaFuncSetAttribute(linear_kv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    linear_kv_kernel<128><<<dim3(nbt * 64, g.BH), 256, smem, st>>>((const uint4*)k, (const uint4*)v, g.N, g.nb, nbt,
                                                                   hs, z, wd, nk);
  }
  return cudaGetLastError();
}

cudaError_t launch_linear_sum(const uint8_t* hs, const uint32_t* selbits, const Geom& g, uint16_t* hout, int* wd,
                              cudaStream_t st) {
  const int nbt = (g.nb + 63) / 64;
  const int smem = linear_sum_smem();
  cudaError_t e = cudaFuncSetAttribute(linear_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  linear_sum_kernel<<<dim3((g.nb + 128 * kSumTiles - 1) / (128 * kSumTiles), 64, g.BH), 64 + kAThreads, smem, st>>>(
      hs, selbits, g.nb, nbt, 2 * nbt, hout, wd);
  return cudaGetLastError();
}

cudaError_t launch_w_tile(const void* w, uint16_t* wt, cudaStream_t st) {
  w_tile_kernel<<<kD, kD, 0, st>>>((const uint16_t*)w, wt);
  return cudaGetLastError();
}

}  // namespace sagesla
