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

constexpr int kKC = 64;      // key blocks per staged chunk
constexpr int kPad = 132;    // padded row length of the kbar chunk (floats)

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

// Sum of z_j over all key blocks of each head, once: grid (BH), 1024
// threads.  Eight slices of 128 channels add every eighth block, then the
// slices are added in a fixed order (deterministic).
__global__ void __launch_bounds__(1024) z_total_kernel(const float* __restrict__ zin, int nb,
                                                       float* __restrict__ ztot) {
  __shared__ float part[8][kD];
  const int bh = blockIdx.x, c = threadIdx.x & (kD - 1), sl = threadIdx.x >> 7;
  const float* zh = zin + (size_t)bh * nb * kD + c;
  float a0 = 0.f, a1 = 0.f;
  int j = sl;
  for (; j + 8 < nb; j += 16) {
    a0 += zh[(size_t)j * kD];
    a1 += zh[(size_t)(j + 8) * kD];
  }
  if (j < nb) a0 += zh[(size_t)j * kD];
  part[sl][c] = a0 + a1;
  __syncthreads();
  if (sl == 0)
    ztot[(size_t)bh * kD + c] =
        ((part[0][c] + part[1][c]) + (part[2][c] + part[3][c])) + ((part[4][c] + part[5][c]) + (part[6][c] + part[7][c]));
}

// Linear-branch outputs (when zin != NULL): selbits [nb][nbw] words with
// bit j set when key block j is selected; zout [nb][128] the fp32 sums
// Z_i = sum_{j not in S_i} z_j, formed as (sum over all j, ztot) - (sum over
// S_i).
//
// TQ query blocks per CTA, 32*TQ threads.  Phase 1: thread -> key block
// t % 64 of each staged chunk and query rows 2*(t/64), 2*(t/64)+1.  Phase 2:
// one warp per query row; with PER > 0 each lane keeps the order keys of
// blocks lane, lane+32, ... (PER of them, nb <= 32*PER) in registers for the
// 32-step threshold search, else it rereads them from shared memory.
template <int TQ, int PER>
__global__ void __launch_bounds__(32 * TQ) pool_topk_kernel(const float* __restrict__ qbar,
                                                           const float* __restrict__ kbar, int nb, int kc,
                                                           int32_t* __restrict__ idx, const float* __restrict__ zin,
                                                           const float* __restrict__ ztot,
                                                           uint32_t* __restrict__ selbits, int nbw,
                                                           float* __restrict__ zout) {
  constexpr int kThr = 32 * TQ;
  extern __shared__ __align__(16) float sm[];
  float* qb = sm;                            // [TQ][128]
  float* kb = qb + TQ * kD;                  // [kKC][kPad]
  float* sc = kb + kKC * kPad;               // [TQ][nb]
  const int bh = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int i0 = blockIdx.x * TQ;
  const float* qh = qbar + (size_t)bh * nb * kD;
  const float* kh = kbar + (size_t)bh * nb * kD;
  const float rs = 1.0f / sqrtf((float)kD);

  for (int e = t; e < TQ * kD; e += kThr) {
    const int r = e / kD;
    qb[e] = i0 + r < nb ? qh[(size_t)i0 * kD + e] : 0.f;
  }
  // Phase 1: scores, fp32 FMA.  With TQ = 8, thread t takes key t % 64 of the
  // chunk and channel quarter t / 64 for all eight rows (a warp shares its
  // quarter, so the query reads are broadcasts and each key value feeds
  // eight FMAs); the four quarter sums are added in quarter order.  Other
  // TQ: key t % 64, rows 2*(t/64) and 2*(t/64)+1, channels in order.
  float* psc = sc + TQ * nb;  // [4][TQ][kKC] quarter sums (TQ == 8 only)
  const int jj = t & 63, qg = t >> 6;
  for (int j0 = 0; j0 < nb; j0 += kKC) {
    __syncthreads();
    for (int e = t; e < kKC * kD / 4; e += kThr) {
      const int r = e / (kD / 4), c4 = e % (kD / 4);
      const int j = j0 + r;
      const float4 val = j < nb ? *reinterpret_cast<const float4*>(kh + (size_t)j * kD + 4 * c4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(kb + r * kPad + 4 * c4) = val;
    }
    __syncthreads();
    const int j = j0 + jj;
    if (TQ == 8) {
      float a[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] = 0.f;
      const float* kr = kb + jj * kPad + 32 * qg;
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kr + c);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float4 x = *reinterpret_cast<const float4*>(qb + r * kD + 32 * qg + c);
          a[r] = fmaf(x.x, k4.x, a[r]);
          a[r] = fmaf(x.y, k4.y, a[r]);
          a[r] = fmaf(x.z, k4.z, a[r]);
          a[r] = fmaf(x.w, k4.w, a[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) psc[(qg * 8 + r) * kKC + jj] = a[r];
      __syncthreads();
      for (int e = t; e < 8 * kKC; e += kThr) {
        const int r = e / kKC, k = e % kKC, jk = j0 + k;
        if (jk < nb)
          sc[r * nb + jk] = ((psc[(0 * 8 + r) * kKC + k] + psc[(1 * 8 + r) * kKC + k]) +
                             (psc[(2 * 8 + r) * kKC + k] + psc[(3 * 8 + r) * kKC + k])) * rs;
      }
    } else if (j < nb) {
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
  __syncthreads();
  // Phase 2: one warp per query row.
  const int i = i0 + warp;
  if (i >= nb) return;
  const float* row = sc + warp * nb;
  // The selected indices are also kept in this row's score slots: entry
  // pos <= j is written only after every lane has read score j.
  int* lst = reinterpret_cast<int*>(sc + warp * nb);
  uint32_t keys[PER > 0 ? PER : 1];
  if (PER > 0) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int j = 32 * u + lane;
      keys[u] = j < nb ? order_key(row[j]) : 0u;  // 0 is never counted: every candidate is >= 1
    }
  }
  // Largest T with #{key >= T} >= kc: built bit by bit from the top.
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    int cnt = 0;
    if (PER > 0) {
      int c4[4] = {0, 0, 0, 0};  // four independent counters: short dependency chains
#pragma unroll
      for (int u = 0; u < PER; ++u) c4[u & 3] += keys[u] >= cand ? 1 : 0;
      cnt = (c4[0] + c4[1]) + (c4[2] + c4[3]);
    } else {
      for (int j = lane; j < nb; j += 32) cnt += order_key(row[j]) >= cand ? 1 : 0;
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= kc) T = cand;
  }
  int gt = 0;
  if (PER > 0) {
#pragma unroll
    for (int u = 0; u < PER; ++u) gt += (32 * u + lane < nb && keys[u] > T) ? 1 : 0;
  } else {
    for (int j = lane; j < nb; j += 32) gt += order_key(row[j]) > T ? 1 : 0;
  }
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = kc - gt;  // >= 1 by construction of T
  int32_t* out = idx + ((size_t)bh * nb + i) * kc;
  int pos = 0, eq_seen = 0;
  const int nch = (nb + 31) >> 5;
#pragma unroll
  for (int u = 0; u < (PER > 0 ? PER : 1); ++u) {
    for (int uu = u; uu < (PER > 0 ? u + 1 : nch); ++uu) {
      if (uu >= nch) break;
      const int j = 32 * uu + lane;
      const uint32_t key = j < nb ? (PER > 0 ? keys[u] : order_key(row[j])) : 0u;
      const bool is_eq = j < nb && key == T;
      const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
      const int eq_rank = eq_seen + __popc(eqm & ((1u << lane) - 1u));
      const bool sel = j < nb && (key > T || (is_eq && eq_rank < need_eq));
      const unsigned sm_ = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int at = pos + __popc(sm_ & ((1u << lane) - 1u));
        out[at] = j;
        lst[at] = j;
      }
      if (selbits && lane == 0) selbits[((size_t)bh * nb + i) * nbw + uu] = sm_;
      pos += __popc(sm_);
      eq_seen += __popc(eqm);
    }
  }
  if (selbits)
    for (int w = nch + lane; w < nbw; w += 32) selbits[((size_t)bh * nb + i) * nbw + w] = 0u;
  if (zin) {
    __syncwarp();
    float zs[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) zs[m] = 0.f;
    const float* zh = zin + (size_t)bh * nb * kD + lane;
    // Eight rows of z in flight per lane; added in list order.
    for (int t0 = 0; t0 < kc; t0 += 8) {
      float v[8][4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = t0 + u < kc ? lst[t0 + u] : -1;
#pragma unroll
        for (int m = 0; m < 4; ++m) v[u][m] = j >= 0 ? __ldg(zh + (size_t)j * kD + 32 * m) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int m = 0; m < 4; ++m) zs[m] += v[u][m];
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
      zout[((size_t)bh * nb + i) * kD + lane + 32 * m] = ztot[(size_t)bh * kD + lane + 32 * m] - zs[m];
  }
}

// Sixteen query blocks per CTA, 512 threads (one CTA per SM), for nb <=
// 1280.  Phase 1: the kbar chunks stream through a 3-buffer ring with
// cp.async, two chunks ahead of the one being scored; thread t takes keys
// t % 32 and t % 32 + 32 of the chunk, channel eighth (t / 32) % 8 and query
// rows 8 * (t / 256) .. + 7 (40 shared loads per 256 FMAs); the eight
// partial dot products of a score are added pairwise.
// Phase 2 as above, one warp per query row; Z_i gathers 16 rows of z at a
// time.
constexpr int kTQ16 = 16, kPER16 = 40, kKB16 = 3;
__global__ void __launch_bounds__(512, 1) pool_topk16_kernel(const float* __restrict__ qbar,
                                                            const float* __restrict__ kbar, int nb, int kc,
                                                            int32_t* __restrict__ idx, const float* __restrict__ zin,
                                                            const float* __restrict__ ztot,
                                                            uint32_t* __restrict__ selbits, int nbw,
                                                            float* __restrict__ zout) {
  constexpr int kThr = 512;
  extern __shared__ __align__(16) float sm[];
  float* qb = sm;                            // [16][128]
  float* kb = qb + kTQ16 * kD;               // [3][kKC][kPad]
  float* psc = kb + kKB16 * kKC * kPad;      // [8][16][kKC] eighth sums
  float* sc = psc + 8 * kTQ16 * kKC;         // [16][nb]
  const int bh = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int i0 = blockIdx.x * kTQ16;
  const float* qh = qbar + (size_t)bh * nb * kD;
  const float* kh = kbar + (size_t)bh * nb * kD;
  const float rs = 1.0f / sqrtf((float)kD);
  const int nchunk = (nb + kKC - 1) / kKC;
  // Chunk c of kbar into buffer c % 3 (rows past nb read as zeros).
  auto stage = [&](int c) {
    float* dst = kb + (c % kKB16) * kKC * kPad;
#pragma unroll
    for (int m = 0; m < kKC * kD / 4 / kThr; ++m) {
      const int e = t + m * kThr;
      const int r = e / (kD / 4), c4 = e % (kD / 4);
      const int j = c * kKC + r;
      cp_async16(dst + r * kPad + 4 * c4, kh + (size_t)(j < nb ? j : 0) * kD + 4 * c4, j < nb ? 16u : 0u);
    }
    cp_async_commit();
  };
  stage(0);
  if (nchunk > 1) stage(1);
  for (int e = t; e < kTQ16 * kD; e += kThr) {
    const int r = e / kD;
    qb[e] = i0 + r < nb ? qh[(size_t)i0 * kD + e] : 0.f;
  }
  const int jj = t & 31, cs = (t >> 5) & 7, rg = t >> 8;
  for (int c = 0; c < nchunk; ++c) {
    // Buffer (c + 2) % 3 was last read in chunk c - 1, before its second barrier.
    if (c + 2 < nchunk) {
      stage(c + 2);
      cp_async_wait<2>();
    } else if (c + 1 < nchunk) {
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // chunk c is in buffer c % 3 for every thread
    const float* kr = kb + (c % kKB16) * kKC * kPad + jj * kPad + 16 * cs;
    float a[8][2];
#pragma unroll
    for (int r = 0; r < 8; ++r) a[r][0] = a[r][1] = 0.f;
#pragma unroll
    for (int cc = 0; cc < 16; cc += 4) {
      const float4 ka = *reinterpret_cast<const float4*>(kr + cc);
      const float4 kb4 = *reinterpret_cast<const float4*>(kr + 32 * kPad + cc);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float4 x = *reinterpret_cast<const float4*>(qb + (8 * rg + r) * kD + 16 * cs + cc);
        a[r][0] = fmaf(x.x, ka.x, a[r][0]);
        a[r][0] = fmaf(x.y, ka.y, a[r][0]);
        a[r][0] = fmaf(x.z, ka.z, a[r][0]);
        a[r][0] = fmaf(x.w, ka.w, a[r][0]);
        a[r][1] = fmaf(x.x, kb4.x, a[r][1]);
        a[r][1] = fmaf(x.y, kb4.y, a[r][1]);
        a[r][1] = fmaf(x.z, kb4.z, a[r][1]);
        a[r][1] = fmaf(x.w, kb4.w, a[r][1]);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      psc[(cs * kTQ16 + 8 * rg + r) * kKC + jj] = a[r][0];
      psc[(cs * kTQ16 + 8 * rg + r) * kKC + jj + 32] = a[r][1];
    }
    __syncthreads();  // eighth sums complete; buffer c % 3 may be refilled
    for (int e = t; e < kTQ16 * kKC; e += kThr) {
      const int r = e / kKC, k = e % kKC, jk = c * kKC + k;
      const float* p = psc + r * kKC + k;
      constexpr int kS = kTQ16 * kKC;  // stride between eighths
      if (jk < nb)
        sc[r * nb + jk] = (((p[0] + p[kS]) + (p[2 * kS] + p[3 * kS])) +
                           ((p[4 * kS] + p[5 * kS]) + (p[6 * kS] + p[7 * kS]))) * rs;
    }
  }
  __syncthreads();
  // Phase 2: one warp per query row.
  const int i = i0 + warp;
  if (i >= nb) return;
  const float* row = sc + warp * nb;
  int* lst = reinterpret_cast<int*>(sc + warp * nb);
  uint32_t keys[kPER16];
#pragma unroll
  for (int u = 0; u < kPER16; ++u) {
    const int j = 32 * u + lane;
    keys[u] = j < nb ? order_key(row[j]) : 0u;  // 0 is never counted: every candidate is >= 1
  }
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    int c4[4] = {0, 0, 0, 0};
#pragma unroll
    for (int u = 0; u < kPER16; ++u) c4[u & 3] += keys[u] >= cand ? 1 : 0;
    const int cnt = __reduce_add_sync(0xffffffffu, (c4[0] + c4[1]) + (c4[2] + c4[3]));
    if (cnt >= kc) T = cand;
  }
  int gt = 0;
#pragma unroll
  for (int u = 0; u < kPER16; ++u) gt += (32 * u + lane < nb && keys[u] > T) ? 1 : 0;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = kc - gt;
  int32_t* out = idx + ((size_t)bh * nb + i) * kc;
  int pos = 0, eq_seen = 0;
  const int nch = (nb + 31) >> 5;
#pragma unroll
  for (int u = 0; u < kPER16; ++u) {
    if (u >= nch) break;
    const int j = 32 * u + lane;
    const uint32_t key = j < nb ? keys[u] : 0u;
    const bool is_eq = j < nb && key == T;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eqm & ((1u << lane) - 1u));
    const bool sel = j < nb && (key > T || (is_eq && eq_rank < need_eq));
    const unsigned sm_ = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int at = pos + __popc(sm_ & ((1u << lane) - 1u));
      out[at] = j;
      lst[at] = j;
    }
    if (selbits && lane == 0) selbits[((size_t)bh * nb + i) * nbw + u] = sm_;
    pos += __popc(sm_);
    eq_seen += __popc(eqm);
  }
  if (selbits)
    for (int w = nch + lane; w < nbw; w += 32) selbits[((size_t)bh * nb + i) * nbw + w] = 0u;
  if (zin) {
    __syncwarp();
    float zs[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) zs[m] = 0.f;
    const float* zh = zin + (size_t)bh * nb * kD + lane;
    // Sixteen rows of z in flight per lane; added in list order.
    for (int t0 = 0; t0 < kc; t0 += 16) {
      float v[16][4];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = t0 + u < kc ? lst[t0 + u] : -1;
#pragma unroll
        for (int m = 0; m < 4; ++m) v[u][m] = j >= 0 ? __ldg(zh + (size_t)j * kD + 32 * m) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u)
#pragma unroll
        for (int m = 0; m < 4; ++m) zs[m] += v[u][m];
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
      zout[((size_t)bh * nb + i) * kD + lane + 32 * m] = ztot[(size_t)bh * kD + lane + 32 * m] - zs[m];
  }
}

namespace {

size_t topk_smem(int tq, int nb) {
  return sizeof(float) * ((size_t)tq * kD + (size_t)kKC * kPad + (size_t)tq * nb + (tq == 8 ? 4 * 8 * kKC : 0));
}

template <int TQ, int PER>
cudaError_t launch_topk_cfg(const float* qbar, const float* kbar, const Geom& g, int32_t* idx, const float* zin,
                            const float* ztot, uint32_t* selbits, float* zout, cudaStream_t st) {
  const size_t smem = topk_smem(TQ, g.nb);
  cudaError_t e = cudaFuncSetAttribute(pool_topk_kernel<TQ, PER>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  pool_topk_kernel<TQ, PER><<<dim3((g.nb + TQ - 1) / TQ, g.BH), 32 * TQ, smem, st>>>(
      qbar, kbar, g.nb, g.kc, idx, zin, ztot, selbits, 2 * ((g.nb + 63) / 64), zout);
  return cudaGetLastError();
}

}  // namespace

size_t pool_topk_smem(int nb) { return topk_smem(4, nb); }

cudaError_t launch_pool_topk(const float* qsum, const float* ksum, const Geom& g, int32_t* idx, float* qbar,
                             float* kbar, const float* zin, float* ztot, uint32_t* selbits, float* zout,
                             cudaStream_t st) {
  pool_means_kernel<<<dim3(g.nb, g.BH), kD, 0, st>>>(qsum, ksum, g.N, g.block, g.nb, g.nq, qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (zin) {
    z_total_kernel<<<g.BH, 1024, 0, st>>>(zin, g.nb, ztot);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // Sixteen query blocks per CTA (512 threads, a 3-buffer ring of kbar chunks,
  // one CTA per SM) up to nb = 1280, where the order keys fit in registers;
  // else eight query blocks per CTA where the scores fit in shared memory;
  // else four.
  constexpr size_t kSmemMax = 227 * 1024;
  if (g.nb <= 32 * kPER16) {
    const size_t smem = sizeof(float) * ((size_t)kTQ16 * kD + kKB16 * (size_t)kKC * kPad + 8 * (size_t)kTQ16 * kKC +
                                         (size_t)kTQ16 * g.nb);
    e = cudaFuncSetAttribute(pool_topk16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    pool_topk16_kernel<<<dim3((g.nb + kTQ16 - 1) / kTQ16, g.BH), 512, smem, st>>>(
        qbar, kbar, g.nb, g.kc, idx, zin, ztot, selbits, 2 * ((g.nb + 63) / 64), zout);
    return cudaGetLastError();
  }
  if (topk_smem(8, g.nb) <= kSmemMax)
    return g.nb <= 32 * 40 ? launch_topk_cfg<8, 40>(qbar, kbar, g, idx, zin, ztot, selbits, zout, st)
                           : launch_topk_cfg<8, 0>(qbar, kbar, g, idx, zin, ztot, selbits, zout, st);
  return launch_topk_cfg<4, 0>(qbar, kbar, g, idx, zin, ztot, selbits, zout, st);
}

}  // namespace sagesla
