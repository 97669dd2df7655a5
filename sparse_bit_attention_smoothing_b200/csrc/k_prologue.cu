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
// rows t/16, t/16+8, ... of its split.  NORM: the QK RMSNorm is applied to
// the key rows; TOK: token-major input rows (H of them per token).  Each is a
// separate instance, so the plain loop stays branch-free.
template <bool NORM, bool TOK>
__global__ void __launch_bounds__(128) stats_partial_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                            int N, int H, int rows_per_split,
                                                            double* __restrict__ psum, float* __restrict__ pmax,
                                                            const QKNorm nk) {
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
  // row n of this head at base + n * pitch, in uint4 (8 bf16) units
  const size_t base = TOK ? ((size_t)(bh / H) * N * H + bh % H) * 16 : (size_t)bh * N * 16;
  const size_t pitch = TOK ? (size_t)H * 16 : 16;
  const uint4 gk = NORM ? __ldg(nk.gamma + (bh % nk.H) * 16 + cg) : make_uint4(0, 0, 0, 0);
  const float* invk = NORM ? nk.inv + (size_t)(bh / max(1, nk.H)) * N : nullptr;
#pragma unroll 4
  for (int n = n_begin + r0; n < n_end; n += 8) {  // unrolled: four row pairs of loads in flight
    uint4 kk = __ldg(k + base + (size_t)n * pitch + cg);
    uint4 vv = __ldg(v + base + (size_t)n * pitch + cg);
    if (NORM) kk = rms_row8(kk, __ldg(invk + n), gk);
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
// Persistent: one CTA per SM walks the list of (head, 64-token tile) pairs
// with a stride of gridDim.x.  Thread 0 stages the Q, K and V rows of the
// next kQStages tiles in shared memory with bulk copies (one per tensor,
// nvalid x 256 bytes, completing on the stage's mbarrier), so that the HBM
// reads of later tiles overlap the quantisation of this one.
//   Q/K: thread t holds channels 8*cg..+7 (cg = (t/8 + t%8) % 16) of the
//        rows t%8 + 32*(t/128) + 8*i, i < 4.  The eight lanes of a quarter
//        warp read eight rows at eight different cg%8, i.e. eight bank
//        groups, and a warp's 8-byte stores into the K-major tile images
//        cover all 32 banks twice (no conflict either way).
//   V:   warp w converts keys 16*(w/2)..+15 of channels 64*(w%2)..+63; lane
//        l the channel pair c0 = 64*(w%2) + 2l, c0 + 1.  Each channel gives
//        one 16-byte chunk (16 consecutive keys) of the V^T image; lanes
//        whose bit 2 is set store the odd channel first, which spreads the
//        chunks of a quarter warp over all 32 banks.
constexpr int kQStages = 3;
constexpr int kQThreads = 256;
constexpr int kRowBytes = kD * 2;  // one bf16 row of Q, K or V
constexpr int kSumPitch = kD + 1;  // pooled partial sums: padded rows (bank spread)
struct QuantSmem {
  uint8_t stage[kQStages][3][kQB * kRowBytes];  // Q, K, V rows of a tile (48 KB per stage)
  uint8_t img[3][kTile];                        // Q^, K^ and V^T tile images
  float psum[2][16][kSumPitch];                 // per-thread column sums of Q and K - mu
  float red[2][8];
  float rowmax[4][kQB];  // per-token Q absmax: the four channel-quarter warps' partial maxima
  uint64_t full[kQStages];
  int abort;
};

// rne(fl32(x * mult)) as a byte.  |x| <= amax and mult = fl32(qmax/amax)
// (qmax = 127, or 7 for the 4-bit option), so the product lies within
// qmax * (1 + 2^-23) and no clamp is needed; adding
// 1.5 * 2^23 rounds it to the nearest integer (ties to even) in the low
// mantissa bits, on the FMA pipe rather than the conversion unit.
__device__ __forceinline__ uint32_t i8code(float x, float mult) {
  return (uint32_t)__float_as_int(__fadd_rn(__fmul_rn(x, mult), 12582912.0f)) & 0xFFu;
}

__global__ void __launch_bounds__(kQThreads, 1)
    quant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ k, const uint8_t* __restrict__ v,
                 const float* __restrict__ mu, const float* __restrict__ mv, int N, int nq, int ntiles,
                 uint8_t* __restrict__ q8t, uint8_t* __restrict__ k8t, uint8_t* __restrict__ v8t,
                 float* __restrict__ sq, float* __restrict__ sk, float* __restrict__ qsum, float* __restrict__ ksum,
                 int* wd, int qmax, int q_tok, const QKNorm nrq, const QKNorm nrk, int H, int tok) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  QuantSmem& S = *reinterpret_cast<QuantSmem*>(smem_raw);
  volatile int* abort = &S.abort;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int cg = ((t >> 3) + (t & 7)) & 15, rr = t & 7, h = t >> 7;
  const int nmine = (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  if (t == 0) {
    for (int s = 0; s < kQStages; ++s) mbar_init(&S.full[s], 1);
    S.abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  // Thread 0: stage the rows of this CTA's j-th tile.
  auto issue = [&](int j) {
    const int gt = (int)blockIdx.x + j * (int)gridDim.x;
    const int bh = gt / nq, n0 = (gt - bh * nq) * kQB;
    uint64_t* bar = &S.full[j % kQStages];
    if (n0 >= N) {  // the padding tile of an odd tile count: nothing to load
      mbar_arrive(bar);
      return;
    }
    const int rows = min(kQB, N - n0);
    const uint32_t bytes = (uint32_t)rows * kRowBytes;
    mbar_expect_tx(bar, 3 * bytes);
    if (!tok) {  // the tile's rows are contiguous
      const size_t off = ((size_t)bh * N + n0) * kRowBytes;
      bulk_g2s(S.stage[j % kQStages][0], q + off, bytes, bar);
      bulk_g2s(S.stage[j % kQStages][1], k + off, bytes, bar);
      bulk_g2s(S.stage[j % kQStages][2], v + off, bytes, bar);
    } else {  // token-major: one 256-byte row per copy
      for (int r = 0; r < rows; ++r) {
        const size_t off = row_elems(1, H, N, bh, n0 + r) * 2;
        bulk_g2s(S.stage[j % kQStages][0] + r * kRowBytes, q + off, kRowBytes, bar);
        bulk_g2s(S.stage[j % kQStages][1] + r * kRowBytes, k + off, kRowBytes, bar);
        bulk_g2s(S.stage[j % kQStages][2] + r * kRowBytes, v + off, kRowBytes, bar);
      }
    }
  };
  int issued = 0;
  if (t == 0)
    for (; issued < min(kQStages, nmine); ++issued) issue(issued);

  int j = 0;
  for (; j < nmine; ++j) {
    const int st = j % kQStages;
    const bool ok = mbar_wait(&S.full[st], (uint32_t)(j / kQStages) & 1u, abort, wd);
    // Uniform exit; also orders the previous tile's reads of img/psum/red
    // before this tile's writes.
    if (__syncthreads_or(!ok)) break;
    const int gt = (int)blockIdx.x + j * (int)gridDim.x;
    const int bh = gt / nq, n0 = (gt - bh * nq) * kQB;
    const int nvalid = max(0, min(kQB, N - n0));  // rows past N read as 0
    const uint8_t* sQ = S.stage[st][0];
    const uint8_t* sK = S.stage[st][1];
    const uint8_t* sV = S.stage[st][2];

    // ---- Q, K rows: absmax and column sums (rows past N read as 0) ----
    // QK RMSNorm (option): this thread's eight channels of gamma for the head
    const uint4 gq = nrq.inv ? __ldg(nrq.gamma + (bh % nrq.H) * 16 + cg) : make_uint4(0, 0, 0, 0);
    const uint4 gk = nrk.inv ? __ldg(nrk.gamma + (bh % nrk.H) * 16 + cg) : make_uint4(0, 0, 0, 0);
    const size_t tok0 = (size_t)(bh / max(1, nrq.inv ? nrq.H : nrk.H)) * N + n0;
    const float4 mu0 = *reinterpret_cast<const float4*>(mu + (size_t)bh * kD + cg * 8);
    const float4 mu1 = *reinterpret_cast<const float4*>(mu + (size_t)bh * kD + cg * 8 + 4);
    const float muc[8] = {mu0.x, mu0.y, mu0.z, mu0.w, mu1.x, mu1.y, mu1.z, mu1.w};
    uint32_t rq[4][4], rk[4][4];
    float aq = 0.f, ak = 0.f, sumq[8], sumk[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      sumq[c] = 0.f;
      sumk[c] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = rr + 32 * h + 8 * i;
      uint4 qq = make_uint4(0, 0, 0, 0), kk = qq;
      if (r < nvalid) {
        qq = *reinterpret_cast<const uint4*>(sQ + r * kRowBytes + cg * 16);
        kk = *reinterpret_cast<const uint4*>(sK + r * kRowBytes + cg * 16);
        if (nrq.inv) qq = rms_row8(qq, __ldg(nrq.inv + tok0 + r), gq);
        if (nrk.inv) kk = rms_row8(kk, __ldg(nrk.inv + tok0 + r), gk);
      }
      rq[i][0] = qq.x; rq[i][1] = qq.y; rq[i][2] = qq.z; rq[i][3] = qq.w;
      rk[i][0] = kk.x; rk[i][1] = kk.y; rk[i][2] = kk.z; rk[i][3] = kk.w;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float xq = (c & 1) ? bf16_hi(rq[i][c >> 1]) : bf16_lo(rq[i][c >> 1]);
        const float xk =
            r < nvalid ? __fsub_rn((c & 1) ? bf16_hi(rk[i][c >> 1]) : bf16_lo(rk[i][c >> 1]), muc[c]) : 0.f;
        aq = fmaxf(aq, fabsf(xq));
        ak = fmaxf(ak, fabsf(xk));
        sumq[c] += xq;
        sumk[c] += xk;
      }
    }

    // ---- V -> FP8 codes, two 16-key chunks of the V^T image ----
    {
      const int c0 = 64 * (warp & 1) + 2 * lane, r0 = 16 * (warp >> 1);
      const float m0 = mv[(size_t)bh * kD + c0], m1 = mv[(size_t)bh * kD + c0 + 1];
      uint32_t e0[4] = {0u, 0u, 0u, 0u}, e1[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int m = 0; m < 16; m += 2) {
        const int r = r0 + m;
        const uint32_t w0 = r < nvalid ? *reinterpret_cast<const uint32_t*>(sV + r * kRowBytes + c0 * 2) : 0u;
        const uint32_t w1 = r + 1 < nvalid ? *reinterpret_cast<const uint32_t*>(sV + (r + 1) * kRowBytes + c0 * 2) : 0u;
        const uint32_t p0 = e4m3x2(__fmul_rn(bf16_lo(w0), m0), __fmul_rn(bf16_lo(w1), m0));
        const uint32_t p1 = e4m3x2(__fmul_rn(bf16_hi(w0), m1), __fmul_rn(bf16_hi(w1), m1));
        e0[m >> 2] |= p0 << (8 * (m & 2));
        e1[m >> 2] |= p1 << (8 * (m & 2));
      }
      const bool odd_first = (lane >> 2) & 1;
      const uint4 ev = make_uint4(e0[0], e0[1], e0[2], e0[3]), od = make_uint4(e1[0], e1[1], e1[2], e1[3]);
      *reinterpret_cast<uint4*>(S.img[2] + kmajor_off(odd_first ? c0 + 1 : c0, r0, kV_LBO, kV_SBO)) =
          odd_first ? od : ev;
      *reinterpret_cast<uint4*>(S.img[2] + kmajor_off(odd_first ? c0 : c0 + 1, r0, kV_LBO, kV_SBO)) =
          odd_first ? ev : od;
    }

    // ---- tile absmax of Q and K - mu ----
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      aq = fmaxf(aq, __shfl_xor_sync(0xffffffffu, aq, o));
      ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, o));
    }
    if (lane == 0) {
      S.red[0][warp] = aq;
      S.red[1][warp] = ak;
    }
    __syncthreads();  // every read of this stage is done: refill it
    if (t == 0 && issued < nmine) {
      fence_proxy_async_smem();
      issue(issued++);
    }
    aq = S.red[0][0];
    ak = S.red[1][0];
#pragma unroll
    for (int w = 1; w < kQThreads / 32; ++w) {
      aq = fmaxf(aq, S.red[0][w]);
      ak = fmaxf(ak, S.red[1][w]);
    }
    const float fq = (float)qmax;
    const float mq = aq > 0.f ? __fdiv_rn(fq, aq) : 0.f;
    const float mk = ak > 0.f ? __fdiv_rn(fq, ak) : 0.f;
    if (t == 0) {
      if (!q_tok) sq[gt] = aq > 0.f ? __fdiv_rn(aq, fq) : 1.f;
      sk[gt] = ak > 0.f ? __fdiv_rn(ak, fq) : 1.f;
    }
    // Per-token Q scales (option): the absmax of each row over its 128
    // channels.  A row's channels are held by lanes rr, rr+8, rr+16, rr+24 of
    // the four warps 4h .. 4h+3: shuffles, then the warps' partial maxima
    // through shared memory (S.rowmax[warp % 4][row]).
    float mqr[4] = {mq, mq, mq, mq};
    if (q_tok) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) a = fmaxf(a, fabsf((c & 1) ? bf16_hi(rq[i][c >> 1]) : bf16_lo(rq[i][c >> 1])));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 16));
        if (lane < 8) S.rowmax[warp & 3][rr + 32 * h + 8 * i] = a;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rr + 32 * h + 8 * i;
        const float a = fmaxf(fmaxf(S.rowmax[0][r], S.rowmax[1][r]), fmaxf(S.rowmax[2][r], S.rowmax[3][r]));
        mqr[i] = a > 0.f ? __fdiv_rn(fq, a) : 0.f;
        if ((t & 0x78) == 0) sq[(size_t)gt * kQB + r] = a > 0.f ? __fdiv_rn(a, fq) : 1.f;  // one writer per row
      }
    }

    // ---- Q, K codes into the tile images; partial column sums ----
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = rr + 32 * h + 8 * i;
      uint32_t qa = 0, qb = 0, ka = 0, kb = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float xq0 = (c & 1) ? bf16_hi(rq[i][c >> 1]) : bf16_lo(rq[i][c >> 1]);
        const float xq1 = (c & 1) ? bf16_hi(rq[i][2 + (c >> 1)]) : bf16_lo(rq[i][2 + (c >> 1)]);
        const float xk0 =
            r < nvalid ? __fsub_rn((c & 1) ? bf16_hi(rk[i][c >> 1]) : bf16_lo(rk[i][c >> 1]), muc[c]) : 0.f;
        const float xk1 =
            r < nvalid ? __fsub_rn((c & 1) ? bf16_hi(rk[i][2 + (c >> 1)]) : bf16_lo(rk[i][2 + (c >> 1)]), muc[c + 4])
                       : 0.f;
        qa |= i8code(xq0, mqr[i]) << (8 * c);
        qb |= i8code(xq1, mqr[i]) << (8 * c);
        ka |= i8code(xk0, mk) << (8 * c);
        kb |= i8code(xk1, mk) << (8 * c);
      }
      const uint32_t off = kmajor_off(r, cg * 8, kQK_LBO, kQK_SBO);
      *reinterpret_cast<uint2*>(S.img[0] + off) = make_uint2(qa, qb);
      *reinterpret_cast<uint2*>(S.img[1] + off) = make_uint2(ka, kb);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      S.psum[0][8 * h + rr][cg * 8 + c] = sumq[c];
      S.psum[1][8 * h + rr][cg * 8 + c] = sumk[c];
    }
    __syncthreads();

    // ---- pooled column sums (fixed order) and the tile images to HBM ----
    {
      const int which = t >> 7, col = t & 127;
      float a = 0.f;
#pragma unroll
      for (int p = 0; p < 16; ++p) a += S.psum[which][p][col];
      (which ? ksum : qsum)[(size_t)gt * kD + col] = a;
    }
    const size_t tb = (size_t)gt * kTile;
#pragma unroll
    for (int m = 0; m < 3 * kTile / 16 / kQThreads; ++m) {
      const int idx = t + m * kQThreads;  // 16-byte unit over the three images
      const int which = idx / (kTile / 16), o = (idx % (kTile / 16)) * 16;
      uint8_t* dst = which == 0 ? q8t : (which == 1 ? k8t : v8t);
      *reinterpret_cast<uint4*>(dst + tb + o) = *reinterpret_cast<const uint4*>(S.img[which] + o);
    }
  }
  // After an abort, wait for the copies still in flight before exiting.
  if (t == 0)
    for (int jj = j; jj < issued; ++jj) mbar_wait_drain(&S.full[jj % kQStages], (uint32_t)(jj / kQStages) & 1u, wd);
}

// Per-token 1 / rms of q and k over all H heads x d channels (QK RMSNorm):
// grid (ceil(N / 8), B), 256 threads, one warp per token; lane l reads
// channels 4l .. 4l+3 of every head's row (in either input layout; in the
// token-major one the H rows of a token are contiguous).  The squares of bf16 values are
// exact in fp64 and their sum is rounded far below the fp32 rounding of the
// result, so the order of the sum does not change inv = fl32(1 / sqrt(sum /
// (H d) + eps)), computed in fp64.
__global__ void __launch_bounds__(256) rms_inv_kernel(const uint2* __restrict__ q, const uint2* __restrict__ k, int H,
                                                      int N, double eps, float* __restrict__ inv_q,
                                                      float* __restrict__ inv_k, int tok) {
  const int b = blockIdx.y, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (n >= N) return;
  double sq = 0.0, sk = 0.0;
  for (int h = 0; h < H; ++h) {
    const size_t row = row_elems(tok, H, N, b * H + h, n) / 4 + lane;  // uint2 = 4 bf16
    const uint2 a = __ldg(q + row), c = __ldg(k + row);
    const uint32_t wa[2] = {a.x, a.y}, wc[2] = {c.x, c.y};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const double a0 = bf16_lo(wa[e]), a1 = bf16_hi(wa[e]), c0 = bf16_lo(wc[e]), c1 = bf16_hi(wc[e]);
      sq += a0 * a0 + a1 * a1;
      sk += c0 * c0 + c1 * c1;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    sk += __shfl_xor_sync(0xffffffffu, sk, o);
  }
  if (lane == 0) {
    const double hd = (double)H * kD;
    inv_q[(size_t)b * N + n] = (float)(1.0 / sqrt(sq / hd + eps));
    inv_k[(size_t)b * N + n] = (float)(1.0 / sqrt(sk / hd + eps));
  }
}

cudaError_t launch_rms_inv(const void* q, const void* k, int B, int H, int N, double eps, float* inv_q, float* inv_k,
                           cudaStream_t st, int tok) {
  rms_inv_kernel<<<dim3((N + 7) / 8, B), 256, 0, st>>>(static_cast<const uint2*>(q), static_cast<const uint2*>(k), H, N,
                                                        eps, inv_q, inv_k, tok);
  return cudaGetLastError();
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
                                 cudaStream_t st, QKNorm nk) {
  const int rows = (g.N + g.split - 1) / g.split;
  const dim3 grid(g.split, g.BH);
  const uint4 *k4 = (const uint4*)k, *v4 = (const uint4*)v;
  if (nk.inv && g.tok)
    stats_partial_kernel<true, true><<<grid, 128, 0, st>>>(k4, v4, g.N, g.H, rows, psum, pmax, nk);
  else if (nk.inv)
    stats_partial_kernel<true, false><<<grid, 128, 0, st>>>(k4, v4, g.N, g.H, rows, psum, pmax, nk);
  else if (g.tok)
    stats_partial_kernel<false, true><<<grid, 128, 0, st>>>(k4, v4, g.N, g.H, rows, psum, pmax, nk);
  else
    stats_partial_kernel<false, false><<<grid, 128, 0, st>>>(k4, v4, g.N, g.H, rows, psum, pmax, nk);
  return cudaGetLastError();
}

cudaError_t launch_stats_final(const double* psum, const float* pmax, const Geom& g, float* mu, float* sv, float* mv,
                               cudaStream_t st) {
  stats_final_kernel<<<g.BH, kD, 0, st>>>(psum, pmax, g.split, g.N, mu, sv, mv);
  return cudaGetLastError();
}

cudaError_t launch_quant(const void* q, const void* k, const void* v, const float* mu, const float* mv, const Geom& g,
                         uint8_t* q8t, uint8_t* k8t, uint8_t* v8t, float* sq, float* sk, float* qsum, float* ksum,
                         int* wd, cudaStream_t st, int qmax, int q_tok, QKNorm nq, QKNorm nk) {
  const int smem = (int)sizeof(QuantSmem);
  cudaError_t e = cudaFuncSetAttribute(quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int ntiles = g.BH * g.nq;
  quant_kernel<<<min(ntiles, sms), kQThreads, smem, st>>>((const uint8_t*)q, (const uint8_t*)k, (const uint8_t*)v, mu,
                                                          mv, g.N, g.nq, ntiles, q8t, k8t, v8t, sq, sk, qsum, ksum, wd,
                                                          qmax, q_tok, nq, nk, g.H, g.tok);
  return cudaGetLastError();
}

cudaError_t launch_untile(const uint8_t* q8t, const uint8_t* k8t, const uint8_t* v8t, const Geom& g, int8_t* q8,
                          int8_t* k8, uint8_t* v8, cudaStream_t st) {
  const size_t per = (size_t)g.N * kD;
  untile_kernel<<<dim3((unsigned)((per + 255) / 256), g.BH), 256, 0, st>>>(q8t, k8t, v8t, g.N, g.nq, q8, k8, v8);
  return cudaGetLastError();
}

}  // namespace sagesla
