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
//   MN-major, staged from the 128-channel rows of K and V), fp32 accumulate, stored in
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

// Shared-memory load kept in program order (not hoisted by the compiler, so
// a loop over chunks does not hold every chunk's operands in registers).
__device__ __forceinline__ float4 lds_f4(const float4* p) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "r"(smem_u32(p)));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

// ---------------------------------------------------------------- K4a ----
// Persistent, one CTA per SM.  An item is kKvJ consecutive key blocks
// j0..j0+kKvJ-1 of one head (j < nbt*64; zeros past nb, so the mask-GEMM
// tiles hold no garbage); items are dealt round-robin.  In the mask-GEMM
// tiles the 16-byte pieces of consecutive j are adjacent, so the blocks of an
// item are stored as 16*kKvJ-byte runs.  TMEM holds 4/kKvJ sets of kKvJ
// accumulators, so the MMAs of the next item can run while the epilogue
// drains the last one when kKvJ = 2.  A key block is consumed as BLK/64 chunks
// of 64 tokens:
//   warp 0      bulk-copies a chunk's K and V rows (16 KB each, contiguous
//               in [BH][N][128]) into a 3-stage ring;
//   warps 2-9   (converters) apply the QK norm and phi to K, add phi(K) into
//               z, and write phi(K) and V as MN-major bf16 MMA operands into
//               one of two operand buffers;
//   warp 1      issues h_j^T += V^T phi(K) (M = 128 value channels, N = 128
//               key channels, K = 64 tokens) into TMEM accumulator j - j0
//               of the item's set;
//   warps 10-17 (epilogue) read the item's accumulators 16 columns at a
//               time, regroup the bf16 pieces through shared memory so that
//               kKvJ consecutive lanes hold the kKvJ blocks of one piece, and
//               store them.
// Converter slot (r0, cg) owns channels 8*cg.. and rows r0 + 16r of each
// chunk; z_j adds a slot's rows in token order, then the 16 row slots in
// slot order.  Every wait is bounded.
namespace {
constexpr int kKvJ = 4;                           // key blocks per item (2 or 4)
constexpr int kKvAcc = 4 / kKvJ;                  // item accumulator sets in TMEM (512 columns)
constexpr int kKvP = 2 * kKvJ;                    // regrouped pieces per lane per round
constexpr int kKvFs = kKvP == 8 ? 0 : 1;          // lane shift of the regrouping swizzle
constexpr int kKvStages = 3;                      // raw chunk ring
constexpr int kKvHalf = 64 * kD * 2;              // 16 KB: 64 bf16 rows
constexpr int kKvRaw = 2 * kKvHalf;               // K rows, then V rows
constexpr int kKvOps = 2;                         // operand buffers
constexpr int kKvConv = 8, kKvEpi = 8;            // warps
constexpr int kKvThreads = 32 * (2 + kKvConv + kKvEpi);
constexpr uint32_t kKvSBO = 8 * 128;              // MN-major operand of 64 tokens
constexpr int kKvOffOp = kKvStages * kKvRaw;      // phi(K) (B), then V (A)
constexpr int kKvOffZ = kKvOffOp + kKvOps * kKvRaw;
constexpr int kKvStage = 32 * kKvP * 16;          // regrouping space per epilogue warp
constexpr int kKvOffSt = kKvOffZ + 2 * 16 * kD * 4;
constexpr int kKvOffBars = kKvOffSt + kKvEpi * kKvStage;
struct KvBars {
  uint64_t raw_full[kKvStages], raw_empty[kKvStages], op_full[kKvOps], op_empty[kKvOps];
  uint64_t acc_full[kKvAcc], acc_empty[kKvAcc], z_ready[2], fin;
  uint32_t tmem;
  int abort;
};
constexpr int kKvSmem = kKvOffBars + (int)sizeof(KvBars) + 1024;
}  // namespace

template <int BLK>
__global__ void __launch_bounds__(kKvThreads, 1) linear_kv_kernel(const uint4* __restrict__ k,
                                                                 const uint4* __restrict__ v, int N, int nb, int nbt,
                                                                 int nitems, uint8_t* __restrict__ hs,
                                                                 float* __restrict__ z, int* wd, const QKNorm nk,
                                                                 int H, int tok) {
  constexpr int kChunks = BLK / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  KvBars* bars = reinterpret_cast<KvBars*>(smem + kKvOffBars);
  float* zred = reinterpret_cast<float*>(smem + kKvOffZ);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nit = nbt * (64 / kKvJ);  // items per head
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&bars->raw_full[s], 1);
      mbar_init(&bars->raw_empty[s], kKvConv);
    }
    for (int b = 0; b < kKvOps; ++b) {
      mbar_init(&bars->op_full[b], kKvConv);
      mbar_init(&bars->op_empty[b], 1);
    }
    for (int a = 0; a < kKvAcc; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kKvEpi);
    }
    mbar_init(&bars->z_ready[0], kKvConv);
    mbar_init(&bars->z_ready[1], kKvConv);
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
      int u = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x) {
        const int bh = item / nit, j0 = (item - bh * nit) * kKvJ;
        for (int jj = 0; ok && jj < kKvJ; ++jj) {
          const int j = j0 + jj;
          for (int c = 0; c < kChunks; ++c, ++u) {
            const int s = u % kKvStages;
            if (u >= kKvStages && !(ok = mbar_wait(&bars->raw_empty[s], ((u / kKvStages) - 1) & 1, abort, wd)))
              break;
            const int n0 = j * BLK + 64 * c;
            const int rows = j < nb ? max(0, min(64, N - n0)) : 0;
            const uint32_t bytes = (uint32_t)rows * (kD * 2);
            mbar_expect_tx(&bars->raw_full[s], 2 * bytes);
            if (rows && !tok) {  // the chunk's rows are contiguous
              const size_t off = ((size_t)bh * N + n0) * 16;
              bulk_g2s(smem + s * kKvRaw, k + off, bytes, &bars->raw_full[s]);
              bulk_g2s(smem + s * kKvRaw + kKvHalf, v + off, bytes, &bars->raw_full[s]);
            } else {  // token-major: one 256-byte row per copy
              for (int r = 0; r < rows; ++r) {
                const size_t off = row_elems(1, H, N, bh, n0 + r) / 8;
                bulk_g2s(smem + s * kKvRaw + r * (kD * 2), k + off, kD * 2, &bars->raw_full[s]);
                bulk_g2s(smem + s * kKvRaw + kKvHalf + r * (kD * 2), v + off, kD * 2, &bars->raw_full[s]);
              }
            }
          }
        }
      }
      // Drain: only the uses issued after the last proven-consumed one can
      // still have copies in flight.
      for (int g = max(0, u - kKvStages); g < u; ++g)
        mbar_wait_drain(&bars->raw_full[g % kKvStages], (g / kKvStages) & 1, wd);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      const uint32_t id = idesc_bf16(128, 128, 1) | (1u << 15);  // A and B MN-major
      int u = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x, ++it) {
        const int a = it % kKvAcc;
        if (it >= kKvAcc && !(ok = mbar_wait(&bars->acc_empty[a], ((it / kKvAcc) - 1) & 1, abort, wd))) break;
        for (int jj = 0; ok && jj < kKvJ; ++jj) {
          for (int c = 0; c < kChunks; ++c, ++u) {
            const int b = u % kKvOps;
            if (!(ok = mbar_wait(&bars->op_full[b], (u / kKvOps) & 1, abort, wd))) break;
            tc_fence_after();
            // h_j^T = V_j^T phi(K_j): A = the V rows (M = value channel cv), B
            // = the phi(K) rows (N = key channel ck): TMEM lane cv, column ck.
            const uint8_t* op = smem + kKvOffOp + b * kKvRaw;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(tmem + (a * kKvJ + jj) * 128, smem_desc(op + kKvHalf + ks * 256, 128, kKvSBO),
                       smem_desc(op + ks * 256, 128, kKvSBO), id, (c > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&bars->op_empty[b]);
          }
        }
        if (!ok) break;
        mma_commit(&bars->acc_full[a]);
      }
      mma_commit(&bars->fin);
    }
  } else if (warp < 2 + kKvConv) {
    // ------------------------------ converters ----------------------------
    // Slot of this thread: row%8 differs across each group of eight lanes
    // (conflict-free operand stores) and so does cg%8 (conflict-free row
    // reads); over the 256 threads every (r0, cg) occurs once.
    const int cw = warp - 2, qd = lane & 7, hi = lane >> 3;
    const int r0 = qd + 8 * (cw & 1), cg = (qd + hi + 4 * (cw >> 1)) & 15;
    const int ct = threadIdx.x - 64;
    int u = 0, zi = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x) {
      const int bh = item / nit, j0 = (item - bh * nit) * kKvJ;
      uint4 gk = make_uint4(0, 0, 0, 0);
      if (nk.inv) gk = __ldg(nk.gamma + (bh % nk.H) * 16 + cg);
      for (int jj = 0; ok && jj < kKvJ; ++jj, ++zi) {
        const int j = j0 + jj;
        float zacc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
        for (int c = 0; c < kChunks; ++c, ++u) {
          const int s = u % kKvStages, b = u % kKvOps;
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->raw_full[s], (u / kKvStages) & 1, abort, wd));
          if (ok && u >= kKvOps)
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->op_empty[b], ((u / kKvOps) - 1) & 1, abort, wd));
          if (!ok) break;
          const uint8_t* raw = smem + s * kKvRaw;
          uint8_t* op = smem + kKvOffOp + b * kKvRaw;
          uint4 kk[4], vv[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int row = r0 + 16 * r;
            kk[r] = *reinterpret_cast<const uint4*>(raw + row * (kD * 2) + cg * 16);
            vv[r] = *reinterpret_cast<const uint4*>(raw + kKvHalf + row * (kD * 2) + cg * 16);
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int row = r0 + 16 * r, n = j * BLK + 64 * c + row;
            const bool valid = j < nb && n < N;
            if (valid && nk.inv) kk[r] = rms_row8(kk[r], __ldg(nk.inv + (size_t)(bh / nk.H) * N + n), gk);
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
            const uint32_t off = cg * kKvSBO + (row >> 3) * 128 + (row & 7) * 16;
            *reinterpret_cast<uint4*>(op + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            *reinterpret_cast<uint4*>(op + kKvHalf + off) = valid ? vv[r] : make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bars->op_full[b]);
            mbar_arrive(&bars->raw_empty[s]);
          }
        }
        if (!ok) break;
        // z_j: the 16 row slots' channel sums, added in slot order.
        float* zr = zred + (zi & 1) * 16 * kD;
        *reinterpret_cast<float4*>(zr + r0 * kD + cg * 8) = make_float4(zacc[0], zacc[1], zacc[2], zacc[3]);
        *reinterpret_cast<float4*>(zr + r0 * kD + cg * 8 + 4) = make_float4(zacc[4], zacc[5], zacc[6], zacc[7]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->z_ready[zi & 1]);
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->z_ready[zi & 1], (zi >> 1) & 1, abort, wd));
        if (!ok) break;
        if (ct < kD) {
          float a = 0.f;
#pragma unroll
          for (int r = 0; r < 16; ++r) a += zr[r * kD + ct];
          if (j < nb) z[((size_t)bh * nb + j) * kD + ct] = a;
        }
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    // Warp w reads TMEM lanes 32(w%4).. (cv = 32(w%4) + lane) and columns ck
    // in [64 hc, +64) of the item's accumulators, 16 columns per round.  A
    // round's pieces (cv, 8-column chunk ch, block jj) go to shared memory at
    // piece index (cv%32, ch, jj), the index within the lane's kKvP pieces
    // XOR-ed with a function of cv that spreads eight lanes over the banks;
    // read back 32 consecutive pieces per instruction, kKvJ consecutive lanes
    // hold the blocks of one (cv, ch), which are contiguous in a mask-GEMM
    // tile (element (cv, ck) of h_j at himg_off).
    const int q = warp & 3, hc = (warp - 2 - kKvConv) >> 2;
    const int cb = 64 * hc;
    uint8_t* stg = smem + kKvOffSt + (warp - 2 - kKvConv) * kKvStage;
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x, ++it) {
      const int bh = item / nit, j0 = (item - bh * nit) * kKvJ;
      const int a = it % kKvAcc;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_full[a], (it / kKvAcc) & 1, abort, wd));
      if (!ok) break;
      tc_fence_after();
      uint8_t* hsb = hs + (size_t)bh * nbt * 64 * 16384 * 2;
#pragma unroll 1
      for (int rd = 0; rd < 4; ++rd) {
        const int c0 = cb + 16 * rd;
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + a * kKvJ * 128 + c0;
#pragma unroll
        for (int jp = 0; jp < kKvJ; jp += 2) {  // two accumulators at a time
          uint32_t r[2][16];
          SAGESLA_TMEM_LD16(tl + jp * 128, r[0]);
          SAGESLA_TMEM_LD16(tl + (jp + 1) * 128, r[1]);
          tmem_ld_wait();
          if (rd == 3 && jp + 2 == kKvJ) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[a]);
          }
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w4[e] = pack_bf16(__uint_as_float(r[x][8 * ch + 2 * e]), __uint_as_float(r[x][8 * ch + 2 * e + 1]));
              const int pidx = lane * kKvP + ((ch * kKvJ + jp + x) ^ ((lane >> kKvFs) & (kKvP - 1)));
              *reinterpret_cast<uint4*>(stg + pidx * 16) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
        __syncwarp();
#pragma unroll
        for (int x = 0; x < kKvP; ++x) {
          const int p = 32 * x + lane;  // piece (cv%32 = p/kKvP, ch, jj = p%kKvJ)
          const int cvl = p / kKvP, li = p % kKvP, ch = li / kKvJ, jj = li % kKvJ;
          const uint4 w =
              *reinterpret_cast<const uint4*>(stg + (cvl * kKvP + (li ^ ((cvl >> kKvFs) & (kKvP - 1)))) * 16);
          const int chunk = (int)(himg_off(32 * q + cvl, c0 + 8 * ch) >> 4);
          *reinterpret_cast<uint4*>(hsb + hs_chunk(nbt, j0 + jj, chunk)) = w;
        }
        __syncwarp();
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

// ---------------------------------------------------------------- K4b ----
// Persistent, one CTA per SM.  Tiles (query-block group it, n-tile nt, head
// bh) are numbered it fastest, then nt, then bh, and dealt round-robin, so the
// CTAs that read the same B tiles work on them at the same time.  A tile is
// two M=128 tiles of query blocks, so each B tile loaded feeds two MMA
// chains.  320 threads: warp 0 bulk-loads the B tiles, warp 1 issues MMAs,
// warps 2-9 expand the 0/1 A tiles from the selection bitmask and run the
// epilogue.  K tiles of 64 key blocks through a 3-stage ring whose stages
// continue across tiles, so the next tile's first stages fill while this
// tile's epilogue drains TMEM; D = 2 x (128 x 256) fp32 in TMEM.
namespace {
constexpr int kLStages = 3;
constexpr int kSumTiles = 2;          // M=128 query-block tiles per CTA tile
constexpr int kATile = 128 * 64 * 2;  // 16 KB per M tile
constexpr int kAThreads = 128 * kSumTiles;
constexpr int kAWarps = kAThreads / 32;
constexpr int kSumStg = 32 * 64 * 2;  // per epilogue warp: 32 rows x 64 bf16 columns
struct LBars {
  uint64_t b_full[kLStages], a_full[kLStages], empty[kLStages], acc_full, acc_empty, fin;
  uint32_t tmem;
  int abort;
};
constexpr int kSumOffStg = kLStages * (kHsTile + kSumTiles * kATile);
constexpr int kSumOffBars = kSumOffStg + kAWarps * kSumStg;
}  // namespace

__global__ void __launch_bounds__(64 + kAThreads, 1) linear_sum_kernel(const uint8_t* __restrict__ hs,
                                                             const uint32_t* __restrict__ selbits, int nb, int nbt,
                                                             int nbw, int ngrp, int ntiles,
                                                             uint16_t* __restrict__ hout, int* wd) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;                               // kLStages x 32 KB
  uint8_t* sA = smem + kLStages * kHsTile;          // kLStages x kSumTiles x 16 KB
  LBars* bars = reinterpret_cast<LBars*>(smem + kSumOffBars);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&bars->b_full[s], 1);
      mbar_init(&bars->a_full[s], kAWarps);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kAWarps);
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
    // ------------------------------ B producer ----------------------------
    if (lane == 0) {
      int g = 0;  // K stages issued, over all tiles
      bool ok = true;
      for (int T = blockIdx.x; ok && T < ntiles; T += gridDim.x) {
        const int nt = (T / ngrp) % 64, bh = T / (ngrp * 64);
        const uint8_t* hs_head = hs + (size_t)bh * nbt * 64 * 16384 * 2;
        for (int kt = 0; kt < nbt; ++kt, ++g) {
          const int st = g % kLStages;
          if (g >= kLStages && !(ok = mbar_wait(&bars->empty[st], ((g / kLStages) - 1) & 1, abort, wd))) break;
          mbar_expect_tx(&bars->b_full[st], kHsTile);
          bulk_g2s(sB + st * kHsTile, hs_head + ((size_t)nt * nbt + kt) * kHsTile, kHsTile, &bars->b_full[st]);
        }
      }
      for (int x = max(0, g - kLStages); x < g; ++x) mbar_wait_drain(&bars->b_full[x % kLStages], (x / kLStages) & 1, wd);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      const uint32_t id = idesc_bf16(128, 256, 1);  // B MN-major
      int g = 0, lt = 0;
      bool ok = true;
      for (int T = blockIdx.x; ok && T < ntiles; T += gridDim.x, ++lt) {
        if (lt > 0 && !(ok = mbar_wait(&bars->acc_empty, (lt - 1) & 1, abort, wd))) break;
        for (int kt = 0; kt < nbt; ++kt, ++g) {
          const int st = g % kLStages;
          ok = mbar_wait(&bars->a_full[st], (g / kLStages) & 1, abort, wd) &&
               mbar_wait(&bars->b_full[st], (g / kLStages) & 1, abort, wd);
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
        if (!ok) break;
        mma_commit(&bars->acc_full);
      }
      mma_commit(&bars->fin);
      mbar_wait_drain(&bars->fin, 0, wd);
    }
  } else {
    // A producer: thread -> query block row i = i0 + (tid - 64); 64 key
    // blocks per K tile from two bitmask words (loaded two K tiles ahead);
    // 1 = NOT selected, j < nb.
    const int u = (tid - 64) >> 7, r = (tid - 64) & 127;
    const int q = warp & 3, ue = (warp - 2) >> 2;  // epilogue: TMEM quadrant, M tile
    uint4* stg = reinterpret_cast<uint4*>(smem + kSumOffStg + (warp - 2) * kSumStg);
    int g = 0, lt = 0;
    bool ok = true;
    for (int T = blockIdx.x; ok && T < ntiles; T += gridDim.x, ++lt) {
      const int it = T % ngrp, nt = (T / ngrp) % 64, bh = T / (ngrp * 64);
      const int i0 = it * 128 * kSumTiles;
      const int i = i0 + 128 * u + r;
      const uint32_t* sb = selbits + ((size_t)bh * nb + (i < nb ? i : 0)) * nbw;
      auto sel_word = [&](int kt) -> uint64_t {
        return (i < nb && kt < nbt) ? ((uint64_t)__ldg(sb + 2 * kt) | ((uint64_t)__ldg(sb + 2 * kt + 1) << 32)) : 0ull;
      };
      uint64_t wa = sel_word(0), wb = sel_word(1);
      for (int kt = 0; kt < nbt; ++kt, ++g) {
        const int st = g % kLStages;
        const uint64_t w = wa;
        wa = wb;
        wb = sel_word(kt + 2);
        if (g >= kLStages) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->empty[st], ((g / kLStages) - 1) & 1, abort, wd));
          if (!ok) break;
        }
        // ones = NOT selected and j < nb (and i < nb), as 64 bits
        uint64_t ones = 0;
        if (i < nb) {
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
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->a_full[st]);
      }
      if (!ok) break;
      // Epilogue: rows of D (256 fp32 columns) -> bf16 image columns, 64 at a
      // time through this warp's staging area (16-byte piece p of row l at
      // slot 8 l + (p ^ (l % 8)): eight lanes, eight bank groups); read back,
      // eight lanes write one row's 128 contiguous bytes.
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_full, lt & 1, abort, wd));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 64) {
        uint32_t v[64];
        const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + ue * 256 + c0;
        SAGESLA_TMEM_LD16(ta, v);
        SAGESLA_TMEM_LD16(ta + 16, v + 16);
        SAGESLA_TMEM_LD16(ta + 32, v + 32);
        SAGESLA_TMEM_LD16(ta + 48, v + 48);
        tmem_ld_wait();
        if (c0 == 192) {  // every TMEM read of this tile done
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->acc_empty);
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) pk[e] = pack_bf16(__uint_as_float(v[8 * p + 2 * e]), __uint_as_float(v[8 * p + 2 * e + 1]));
          stg[8 * lane + (p ^ (lane & 7))] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rl = 4 * k + (lane >> 3), p = lane & 7;      // row of this warp, piece
          const int ir = i0 + 128 * ue + 32 * q + rl;             // TMEM lane 32q + rl == row of the M tile
          const uint4 w4 = stg[8 * rl + (p ^ (rl & 7))];
          if (ir < nb)
            *reinterpret_cast<uint4*>(hout + ((size_t)bh * nb + ir) * 16384 + (size_t)nt * 256 + c0 + 8 * p) = w4;
        }
        __syncwarp();
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
// Persistent, one CTA per SM.  An item is 128 query rows: two query blocks at
// block 64 (M=64 accumulators at TMEM lane offsets 0 / 16), one at block 128
// (M=128).  The CTA's items alternate between two groups of four row warps
// (one row per thread), each with its own shared-memory stage and 256 TMEM
// columns (num, then y), so one group's copies, MMAs and stores overlap the
// other group's work:
//   warp 0      bulk-copies an item's H_i images and Z_i rows into the
//               group's stage once the first MMA of the group's previous
//               item has read them; the W image once;
//   warp 11     bulk-copies the item's q rows (up to 32 KB) once the group's
//               previous item is stored;
//   warp 1      issues num = phi(Q) H_i for every item;
//   warp 10     issues y = O_l W^T for every item;
//   warps 2-9   (row groups) read their q rows (chunk c ^ (lane%8) at step c,
//               so eight lanes hit eight banks, then put back in channel
//               order), write the phi(Q) operand over them, scale num by
//               1/(phi(q) . Z_i) into the O_l operand, and store y through a
//               swizzled staging area so that each instruction writes two
//               whole rows.
// Per row, the arithmetic and its order are those of one thread per row
// reading its q row from global memory.  Every wait is bounded.
namespace {
constexpr int kApImg = 32768;
constexpr int kApOffZ = 3 * kApImg;   // in a stage: q rows -> phi(Q) -> O_l -> y staging; two H images; two Z rows
constexpr int kApStage = kApOffZ + 2 * kD * 4;
constexpr int kApOffW = 2 * kApStage;
constexpr int kApOffBars = kApOffW + kApImg;
constexpr int kApThreads = 32 * 12;
struct ApBars {
  uint64_t full[2], empty[2], h_empty[2], qread[2], a_full[2], num_full[2], o_full[2], y_full[2], w_full, fin[2];
  uint32_t tmem;
  int abort;
};
constexpr int kApSmem = kApOffBars + (int)sizeof(ApBars) + 16;
}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kApThreads, 1) linear_apply_kernel(const uint16_t* __restrict__ q,
                                                                    const uint8_t* __restrict__ himg,
                                                                    const float* __restrict__ zl,
                                                                    const uint8_t* __restrict__ wimg, int N, int nb,
                                                                    int nitems, __nv_bfloat16* __restrict__ out,
                                                                    int* wd, const QKNorm nq, int H, int tok) {
  constexpr int M = MODE == 0 ? 64 : 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
  ApBars* bars = reinterpret_cast<ApBars*>(smem + kApOffBars);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbi = MODE == 0 ? (nb + 1) / 2 : nb;  // items per head
  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bars->full[g], 2);
      mbar_init(&bars->empty[g], 4);
      mbar_init(&bars->h_empty[g], 1);
      mbar_init(&bars->qread[g], 4);
      mbar_init(&bars->a_full[g], 4);
      mbar_init(&bars->num_full[g], 1);
      mbar_init(&bars->o_full[g], 4);
      mbar_init(&bars->y_full[g], 1);
      mbar_init(&bars->fin[g], 1);
    }
    mbar_init(&bars->w_full, 1);
    bars->abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const uint32_t id = idesc_bf16(M, 128);

  if (warp == 0 || warp == 11) {
    // ------------------------------ producers -----------------------------
    const bool hq = warp == 0;  // H images and Z rows (and W), or q rows
    if (lane == 0) {
      if (hq) {
        mbar_expect_tx(&bars->w_full, kApImg);
        bulk_g2s(smem + kApOffW, wimg, kApImg, &bars->w_full);
      }
      int it = 0;
      for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
        const int g = it & 1, bh = item / nbi, t = item - bh * nbi;
        if (it >= 2 && !mbar_wait(hq ? &bars->h_empty[g] : &bars->empty[g], ((it >> 1) - 1) & 1, abort, wd)) break;
        uint8_t* st = smem + g * kApStage;
        if (hq) {
          const int i0 = MODE == 0 ? 2 * t : t;
          const int nimg = (MODE == 0 && i0 + 1 < nb) ? 2 : 1;
          mbar_expect_tx(&bars->full[g], nimg * (kApImg + kD * 4));
          for (int x = 0; x < nimg; ++x) {
            bulk_g2s(st + kApImg + x * kApImg, himg + ((size_t)bh * nb + i0 + x) * kApImg, kApImg, &bars->full[g]);
            bulk_g2s(st + kApOffZ + x * kD * 4, zl + ((size_t)bh * nb + i0 + x) * kD, kD * 4, &bars->full[g]);
          }
        } else {
          const int n0 = 128 * t, rows = min(128, N - n0);
          mbar_expect_tx(&bars->full[g], (uint32_t)rows * (kD * 2));
          if (!tok)  // the item's rows are contiguous
            bulk_g2s(st, q + ((size_t)bh * N + n0) * kD, (uint32_t)rows * (kD * 2), &bars->full[g]);
          else  // token-major: one 256-byte row per copy
            for (int r = 0; r < rows; ++r)
              bulk_g2s(st + r * (kD * 2), q + row_elems(1, H, N, bh, n0 + r), kD * 2, &bars->full[g]);
        }
      }
      // Drain: the last two items' copies (earlier ones were consumed) and W.
      for (int g2 = max(0, it - 2); g2 < it; ++g2) mbar_wait_drain(&bars->full[g2 & 1], (g2 >> 1) & 1, wd);
      if (hq) mbar_wait_drain(&bars->w_full, 0, wd);
    }
  } else if (warp == 1 || warp == 10) {
    // ------------------------------ MMA issuers ---------------------------
    const int second = warp == 10;  // 0: num = phi(Q) H_i; 1: y = O_l W^T
    if (lane == 0) {
      bool ok = !second || mbar_wait(&bars->w_full, 0, abort, wd);
      int it = 0;
      for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x, ++it) {
        const int g = it & 1, t = item - (item / nbi) * nbi;
        const int nx = (MODE == 0 && 2 * t + 1 < nb) ? 2 : 1;
        uint64_t* wait_bar = second ? &bars->o_full[g] : &bars->a_full[g];
        if (!(ok = mbar_wait(wait_bar, (it >> 1) & 1, abort, wd))) break;
        tc_fence_after();
        const uint8_t* st = smem + g * kApStage;
        for (int x = 0; x < (MODE == 0 ? nx : 1); ++x) {
          const uint32_t d = tmem + g * 256 + (second ? 128 : 0) + ((uint32_t)(x * 16) << 16);
          const uint8_t* bsrc = second ? smem + kApOffW : st + kApImg + x * kApImg;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16(d, smem_desc(st + x * (kApImg / 2) + ks * 256, 128, 2048), smem_desc(bsrc + ks * 256, 128, 2048),
                     id, ks > 0);
        }
        if (second) {
          mma_commit(&bars->y_full[g]);
        } else {
          mma_commit(&bars->num_full[g]);
          mma_commit(&bars->h_empty[g]);  // H images and Z rows read
        }
      }
      mma_commit(&bars->fin[second]);
      mbar_wait_drain(&bars->fin[second], 0, wd);
    }
  } else {
    // ------------------------------ row groups ----------------------------
    const int grp = (warp - 2) >> 2, wq = warp & 3;  // TMEM lane quadrant wq
    const int x = MODE == 0 ? lane >> 4 : 0;
    const int row = MODE == 0 ? 16 * wq + (lane & 15) : 32 * wq + lane;  // row of the M tile (TMEM lane)
    const int R = 64 * x + row;                                         // row of the item
    const uint32_t lb = (uint32_t)(32 * wq) << 16;
    const int sw = lane & 7;
    bool ok = true;
    // This group's items: the CTA's items k = grp, grp + 2, ...; use u = k / 2.
    for (int k = grp, item = blockIdx.x + grp * gridDim.x; item < nitems; k += 2, item += 2 * gridDim.x) {
      const int g = grp, u = k >> 1;
      const int bh = item / nbi, t = item - bh * nbi;
      const int n = 128 * t + R;
      const bool store = n < N;  // (a block past nb has no rows below N)
      uint8_t* st = smem + g * kApStage;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->full[g], u & 1, abort, wd));
      if (!ok) break;
      // Own q row, chunk (c ^ sw) at step c: eight lanes, eight bank groups.
      uint4 qq[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        qq[c] = store ? *reinterpret_cast<const uint4*>(st + R * (kD * 2) + ((c ^ sw) * 16)) : make_uint4(0, 0, 0, 0);
      // Back to channel order: qq[c] <- chunk c (an XOR permutation, one
      // conditional exchange per bit of sw).
#pragma unroll
      for (int b = 0; b < 3; ++b) {
        const bool sb = (sw >> b) & 1;
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (!(c & (1 << b))) {
            const uint4 lo = qq[c], hi = qq[c | (1 << b)];
            qq[c] = sb ? hi : lo;
            qq[c | (1 << b)] = sb ? lo : hi;
          }
      }
      // Every row of the group read before the operand overwrites them.
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->qread[g]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->qread[g], u & 1, abort, wd));
      if (!ok) break;
      if (nq.inv && store) {  // QK RMSNorm of the query row
        const float inv = __ldg(nq.inv + (size_t)(bh / nq.H) * N + n);
        const uint4* gq = nq.gamma + (bh % nq.H) * 16;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) qq[ch] = rms_row8(qq[ch], inv, __ldg(gq + ch));
      }
      // Z_i of this row's block, staged (rows of a block past nb are never stored).
      const float4* zrow = reinterpret_cast<const float4*>(st + kApOffZ + x * kD * 4);
      float den = 0.f;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint32_t w4[4] = {qq[ch].x, qq[ch].y, qq[ch].z, qq[ch].w};
        const float4 z0 = lds_f4(zrow + 2 * ch), z1 = lds_f4(zrow + 2 * ch + 1);
        const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = phi(bf16_lo(w4[e])), b = phi(bf16_hi(w4[e]));
          den = fmaf(a, zz[2 * e], den);
          den = fmaf(b, zz[2 * e + 1], den);
          pk[e] = pack_bf16(a, b);
        }
        *reinterpret_cast<uint4*>(st + kmajor_off(R, ch * 16, 128, 2048)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->a_full[g]);
      // num -> O_l = num / den (bf16), the A operand of the second MMA.
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->num_full[g], u & 1, abort, wd));
      if (!ok) break;
      tc_fence_after();
      {
        const float inv_den = (store && den > 0.f) ? 1.f / den : 0.f;
#pragma unroll 1
        for (int c = 0; c < kD; c += 16) {
          uint32_t v16[16];
          SAGESLA_TMEM_LD16(tmem + lb + g * 256 + c, v16);
          tmem_ld_wait();
          uint32_t pk[8];
#pragma unroll
          for (int z2 = 0; z2 < 8; ++z2)
            pk[z2] = pack_bf16(__uint_as_float(v16[2 * z2]) * inv_den, __uint_as_float(v16[2 * z2 + 1]) * inv_den);
          *reinterpret_cast<uint4*>(st + kmajor_off(R, c * 2, 128, 2048)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(st + kmajor_off(R, c * 2 + 16, 128, 2048)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_full[g]);
      // y -> bf16 rows.  Staging (this warp's 8 KB of the stage): piece
      // (chunk C, lane l) at slot 32 C + (l ^ (C % 8)).
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->y_full[g], u & 1, abort, wd));
      if (!ok) break;
      tc_fence_after();
      uint8_t* stg = st + ((warp - 2) & 3) * 8192;
#pragma unroll 1
      for (int c = 0; c < kD; c += 16) {
        uint32_t v16[16];
        SAGESLA_TMEM_LD16(tmem + lb + g * 256 + 128 + c, v16);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[4];
#pragma unroll
          for (int z2 = 0; z2 < 4; ++z2)
            pk[z2] = pack_bf16(__uint_as_float(v16[8 * h + 2 * z2]), __uint_as_float(v16[8 * h + 2 * z2 + 1]));
          const int C = c / 8 + h;
          *reinterpret_cast<uint4*>(stg + (32 * C + (lane ^ (C & 7))) * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      // Rows of this warp: lane l wrote row R(l) = 64 (l/16) + 16 wq + l%16
      // (block 64) or 32 wq + l (block 128); lanes 2k and 2k+1 are adjacent
      // tokens.  Instruction k: lanes 0-15 write row 2k + 0, lanes 16-31 row
      // 2k + 1, chunk lane % 16.
#pragma unroll 4
      for (int k = 0; k < 16; ++k) {
        const int lr = 2 * k + (lane >> 4), C = lane & 15;
        const int Rr = MODE == 0 ? 64 * (lr >> 4) + 16 * wq + (lr & 15) : 32 * wq + lr;
        const int nr = 128 * t + Rr;
        const uint4 w = *reinterpret_cast<const uint4*>(stg + (32 * C + (lr ^ (C & 7))) * 16);
        if (nr < N) *reinterpret_cast<uint4*>(out + row_elems(tok, H, N, bh, nr) + C * 8) = w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[g]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

int linear_apply_smem(int) { return kApSmem; }

cudaError_t launch_linear_apply(const void* q, const uint16_t* himg, const float* zl, const uint16_t* wimg,
                                const Geom& g, void* out, int* wd, cudaStream_t st, QKNorm nq) {
  const int nbi = g.block == 64 ? (g.nb + 1) / 2 : g.nb;
  const int nitems = g.BH * nbi;
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = min(nitems, sms);
  if (g.block == 64) {
    e = cudaFuncSetAttribute(linear_apply_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kApSmem);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<0><<<grid, kApThreads, kApSmem, st>>>((const uint16_t*)q, (const uint8_t*)himg, zl,
                                                              (const uint8_t*)wimg, g.N, g.nb, nitems,
                                                              (__nv_bfloat16*)out, wd, nq, g.H, g.tok);
  } else {
    e = cudaFuncSetAttribute(linear_apply_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kApSmem);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<1><<<grid, kApThreads, kApSmem, st>>>((const uint16_t*)q, (const uint8_t*)himg, zl,
                                                              (const uint8_t*)wimg, g.N, g.nb, nitems,
                                                              (__nv_bfloat16*)out, wd, nq, g.H, g.tok);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------- W image ---
// proj_w [c_out][c_in] row-major -> K-major B operand image [N=c_out][K=c_in].
__global__ void w_tile_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ wt) {
  const int co = blockIdx.x, ci = threadIdx.x;
  wt[himg_off(co, ci) / 2] = w[co * kD + ci];
}

int linear_kv_smem(int) { return kKvSmem; }
int linear_sum_smem() { return kSumOffBars + (int)sizeof(LBars) + 1024; }

cudaError_t launch_linear_kv(const void* k, const void* v, const Geom& g, uint8_t* hs, float* z, int* wd,
                             cudaStream_t st, QKNorm nk) {
  const int nbt = (g.nb + 63) / 64;
  const int nitems = g.BH * nbt * (64 / kKvJ);
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = min(nitems, sms);
  if (g.block == 64) {
    e = cudaFuncSetAttribute(linear_kv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
    if (e != cudaSuccess) return e;
    linear_kv_kernel<64><<<grid, kKvThreads, kKvSmem, st>>>((const uint4*)k, (const uint4*)v, g.N, g.nb, nbt, nitems,
                                                            hs, z, wd, nk, g.H, g.tok);
  } else {
    e = cudaFuncSetAttribute(linear_kv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
    if (e != cudaSuccess) return e;
    linear_kv_kernel<128><<<grid, kKvThreads, kKvSmem, st>>>((const uint4*)k, (const uint4*)v, g.N, g.nb, nbt,
                                                             nitems, hs, z, wd, nk, g.H, g.tok);
  }
  return cudaGetLastError();
}

cudaError_t launch_linear_sum(const uint8_t* hs, const uint32_t* selbits, const Geom& g, uint16_t* hout, int* wd,
                              cudaStream_t st) {
  const int nbt = (g.nb + 63) / 64;
  const int ngrp = (g.nb + 128 * kSumTiles - 1) / (128 * kSumTiles);
  const int ntiles = ngrp * 64 * g.BH;
  const int smem = linear_sum_smem();
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(linear_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  linear_sum_kernel<<<min(ntiles, sms), 64 + kAThreads, smem, st>>>(hs, selbits, g.nb, nbt, 2 * nbt, ngrp, ntiles, hout,
                                                                    wd);
  return cudaGetLastError();
}

cudaError_t launch_w_tile(const void* w, uint16_t* wt, cudaStream_t st) {
  w_tile_kernel<<<kD, kD, 0, st>>>((const uint16_t*)w, wt);
  return cudaGetLastError();
}

}  // namespace sagesla
