// k_flash.cu -- K5: block-sparse SageAttention-style flash kernel on tcgen05.
//
// For each query block i and each key block j of its top-k list (ascending),
//   S = (q^ . k^) * s_q,i * s_k,j / sqrt(d)     INT8 x INT8 -> INT32 in TMEM
//   online softmax, P~ = e4m3(448 * exp(S - running max))
//   O += P~ . v^                                 FP8 x FP8 -> FP32 in TMEM
// and finally O_s = (O / rowsum(P~)) * s_v (per channel).  Sources:
// "揭秘TurboDiffusion：如何让视频生成实现百倍加速？" 支柱一 (INT8 attention with
// smoothing on integer tensor cores) and 支柱二 (only the selected blocks are
// computed exactly); 量子位 news 技术解密 1 (SageAttention2++).
//
// Layout on the SM (192 threads, 1 CTA/SM):
//   warp 0  producer: bulk copies of Q^, K^ and V^T tiles (pre-tiled in HBM
//           by the quantiser, so one cp.async.bulk moves a whole 8 KB tile);
//   warp 1  MMA issuer (one thread) + TMEM owner;
//   warps 2-5  softmax / rescale / epilogue, one query row per thread.
// Mode 64 (block 64): a CTA owns two query blocks A and B.  Their M=64
//   accumulators share TMEM columns at lane offsets 0 and 16, so all 128
//   softmax threads hold a row.  Each step takes two key blocks per query
//   block (S tile N = 128), PV is M=64, N=144 (128 V channels + 16 rows of
//   ones whose product is the row sum of P~).
// Mode 128 (block 128): one query block of 128 rows per CTA, M = 128.
// TMEM: S double buffer (2 x 128 cols) + O (144 cols) of 512 allocated.
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kStages = 2;
constexpr int kSoftThreads = 256;  // two warps per TMEM lane quadrant
constexpr int kThreads = 64 + kSoftThreads;
constexpr int kVSlot = kTile + 1024;  // 8 KB V^T tile + 16 rows of ones (1 KB)
constexpr uint32_t kOnesE4M3 = 0x38383838u;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;
constexpr uint32_t kTmemCols = 512, kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kNO = 144;  // PV N: 128 channels + 16 ones

struct Params {
  const uint8_t* q8t;
  const uint8_t* k8t;
  const uint8_t* v8t;
  const float* sq;
  const float* sk;
  const float* sv;
  const int32_t* idx;
  __nv_bfloat16* out;
  int* wd;
  int N, nb, nq, kc, nsteps;
  int add_out;  // 1: out already holds the linear branch (bf16); add O_s to it
};

template <int MODE>
struct Cfg {
  // MODE 0: two query blocks (A,B) x two 64-key sub-tiles per step.
  // MODE 1: one 128-row query block x one 128-key block per step.
  static constexpr int kQBytes = 2 * kTile;
  static constexpr int kKStage = (MODE == 0 ? 4 : 2) * kTile;
  static constexpr int kVStage = (MODE == 0 ? 4 : 2) * kVSlot;
  static constexpr int kPBuf = 2 * kTile;  // 128 rows x 128 keys (two 64-row halves in mode 0)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKStage;
  static constexpr int kOffP = kOffV + kStages * kVStage;
  static constexpr int kOffBar = kOffP + 2 * kPBuf;
  static constexpr int kSmem = kOffBar + 256 + 2048 + 1024;  // barriers, max exchange, alignment slack
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done;
  uint64_t fin;
  uint64_t xbar[4][2];  // row-max exchange between the two warps of a quadrant
  uint32_t tmem;
  int abort;
};

// key block (mask block index) of list entry t for query block i
__device__ __forceinline__ int list_at(const Params& p, int bh, int i, int t) {
  return p.idx ? __ldg(p.idx + ((size_t)bh * p.nb + i) * p.kc + t) : t;
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) flash_kernel(const Params p) {
  using C = Cfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  // Query blocks of this CTA (mask-block indices).
  const int iA = MODE == 0 ? 2 * (int)blockIdx.x : (int)blockIdx.x;
  const int iB = MODE == 0 ? 2 * (int)blockIdx.x + 1 : -1;
  const bool hasB = MODE == 0 && iB < p.nb;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], kSoftThreads);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->fin, 1);
    for (int qq = 0; qq < 4; ++qq)
      for (int b = 0; b < 2; ++b) mbar_init(&bars->xbar[qq][b], 64);
    bars->abort = 0;
    mbar_fence_init();
  }
  // Rows of ones under every V slot (PV's extra 16 output columns = row sum).
  for (int e = tid; e < kStages * (C::kVStage / kVSlot) * 64; e += kThreads) {
    const int slot = e / 64, w = e % 64;
    reinterpret_cast<uint32_t*>(smem + C::kOffV + slot * kVSlot + kTile)[w * 4 + 0] = kOnesE4M3;
    reinterpret_cast<uint32_t*>(smem + C::kOffV + slot * kVSlot + kTile)[w * 4 + 1] = kOnesE4M3;
    reinterpret_cast<uint32_t*>(smem + C::kOffV + slot * kVSlot + kTile)[w * 4 + 2] = kOnesE4M3;
    reinterpret_cast<uint32_t*>(smem + C::kOffV + slot * kVSlot + kTile)[w * 4 + 3] = kOnesE4M3;
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  const int nsteps = p.nsteps;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const size_t head_tiles = (size_t)bh * p.nq;
      mbar_expect_tx(&bars->q_full, C::kQBytes);
      if (MODE == 0) {
        bulk_g2s(smem + C::kOffQ, p.q8t + (head_tiles + iA) * kTile, kTile, &bars->q_full);
        const int ib = hasB ? iB : iA;  // keep the transaction count fixed
        bulk_g2s(smem + C::kOffQ + kTile, p.q8t + (head_tiles + ib) * kTile, kTile, &bars->q_full);
      } else {
        bulk_g2s(smem + C::kOffQ, p.q8t + (head_tiles + 2 * iA) * kTile, 2 * kTile, &bars->q_full);
      }
      int k_issued = 0, v_issued = 0;  // steps whose copies were issued
      for (int s = 0; s < nsteps && !*abort; ++s) {
        const int st = s % kStages;
        if (s >= kStages && !mbar_wait(&bars->k_empty[st], ((s / kStages) - 1) & 1, abort, p.wd)) break;
        uint8_t* kd = smem + C::kOffK + st * C::kKStage;
        uint8_t* vd = smem + C::kOffV + st * C::kVStage;
        if (MODE == 0) {
          const int nsub = min(2, p.kc - 2 * s);
          mbar_expect_tx(&bars->k_full[st], 2 * nsub * kTile);
          for (int x = 0; x < 2; ++x) {
            const int i = (x == 0 || !hasB) ? iA : iB;
            for (int u = 0; u < nsub; ++u) {
              const int j = list_at(p, bh, i, 2 * s + u);
              bulk_g2s(kd + (2 * x + u) * kTile, p.k8t + (head_tiles + j) * kTile, kTile, &bars->k_full[st]);
            }
          }
          k_issued = s + 1;
          if (s >= kStages && !mbar_wait(&bars->v_empty[st], ((s / kStages) - 1) & 1, abort, p.wd)) break;
          mbar_expect_tx(&bars->v_full[st], 2 * nsub * kTile);
          for (int x = 0; x < 2; ++x) {
            const int i = (x == 0 || !hasB) ? iA : iB;
            for (int u = 0; u < nsub; ++u) {
              const int j = list_at(p, bh, i, 2 * s + u);
              bulk_g2s(vd + (2 * x + u) * kVSlot, p.v8t + (head_tiles + j) * kTile, kTile, &bars->v_full[st]);
            }
          }
          v_issued = s + 1;
        } else {
          const int j = list_at(p, bh, iA, s);
          mbar_expect_tx(&bars->k_full[st], 2 * kTile);
          bulk_g2s(kd, p.k8t + (head_tiles + 2 * j) * kTile, 2 * kTile, &bars->k_full[st]);
          k_issued = s + 1;
          if (s >= kStages && !mbar_wait(&bars->v_empty[st], ((s / kStages) - 1) & 1, abort, p.wd)) break;
          mbar_expect_tx(&bars->v_full[st], 2 * kTile);
          bulk_g2s(vd, p.v8t + (head_tiles + 2 * j) * kTile, kTile, &bars->v_full[st]);
          bulk_g2s(vd + kVSlot, p.v8t + (head_tiles + 2 * j + 1) * kTile, kTile, &bars->v_full[st]);
          v_issued = s + 1;
        }
      }
      // Drain: every copy issued must land before the CTA may exit.
      mbar_wait_drain(&bars->q_full, 0, p.wd);
      for (int s = max(0, k_issued - kStages); s < k_issued; ++s)
        mbar_wait_drain(&bars->k_full[s % kStages], (s / kStages) & 1, p.wd);
      for (int s = max(0, v_issued - kStages); s < v_issued; ++s)
        mbar_wait_drain(&bars->v_full[s % kStages], (s / kStages) & 1, p.wd);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      const uint32_t id_s = MODE == 0 ? 0u : idesc_i8(128, 128);
      const uint32_t id_pv = idesc_e4m3(MODE == 0 ? 64 : 128, kNO);
      bool ok = mbar_wait(&bars->q_full, 0, abort, p.wd);
      auto issue_s = [&](int s) {
        const int st = s % kStages;
        const uint32_t dS = tmem + ((s & 1) ? kColS1 : kColS0);
        const uint8_t* kd = smem + C::kOffK + st * C::kKStage;
        if (MODE == 0) {
          const int nsub = min(2, p.kc - 2 * s);
          const uint32_t id = idesc_i8(64, 64 * nsub);
          for (int x = 0; x < (hasB ? 2 : 1); ++x) {
            const uint8_t* qa = smem + C::kOffQ + x * kTile;
            const uint8_t* kb = kd + 2 * x * kTile;
            const uint32_t d = dS + ((uint32_t)(x * 16) << 16);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(d, smem_desc(qa + kk * 256, kQK_LBO, kQK_SBO), smem_desc(kb + kk * 256, kQK_LBO, kQK_SBO), id,
                     kk > 0);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(dS, smem_desc(smem + C::kOffQ + kk * 256, kQK_LBO, kQK_SBO),
                   smem_desc(kd + kk * 256, kQK_LBO, kQK_SBO), id_s, kk > 0);
        }
        mma_commit(&bars->s_full[s & 1]);
        mma_commit(&bars->k_empty[st]);
      };
      if (ok && nsteps > 0) {
        ok = mbar_wait(&bars->k_full[0], 0, abort, p.wd);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
      }
      for (int s = 0; ok && s < nsteps; ++s) {
        if (s + 1 < nsteps) {
          const int st1 = (s + 1) % kStages;
          if (!(ok = mbar_wait(&bars->k_full[st1], ((s + 1) / kStages) & 1, abort, p.wd))) break;
          tc_fence_after();
          issue_s(s + 1);
        }
        const int st = s % kStages;
        if (!(ok = mbar_wait(&bars->p_full[s & 1], (s >> 1) & 1, abort, p.wd))) break;
        if (!(ok = mbar_wait(&bars->v_full[st], (s / kStages) & 1, abort, p.wd))) break;
        tc_fence_after();
        const uint8_t* vd = smem + C::kOffV + st * C::kVStage;
        const uint8_t* pb = smem + C::kOffP + (s & 1) * C::kPBuf;
        if (MODE == 0) {
          const int nsub = min(2, p.kc - 2 * s);
          for (int x = 0; x < (hasB ? 2 : 1); ++x) {
            const uint32_t d = tmem + kColO + ((uint32_t)(x * 16) << 16);
            for (int kk = 0; kk < 2 * nsub; ++kk) {
              const uint8_t* a = pb + x * kTile + kk * 256;
              const uint8_t* b = vd + (2 * x + (kk >> 1)) * kVSlot + (kk & 1) * 256;
              mma_e4m3(d, smem_desc(a, kQK_LBO, kQK_SBO), smem_desc(b, kV_LBO, kV_SBO), id_pv, (s > 0 || kk > 0));
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint8_t* a = pb + kk * 256;
            const uint8_t* b = vd + (kk >> 1) * kVSlot + (kk & 1) * 256;
            mma_e4m3(tmem + kColO, smem_desc(a, kQK_LBO, kQK_SBO), smem_desc(b, kV_LBO, kV_SBO), id_pv,
                     (s > 0 || kk > 0));
          }
        }
        mma_commit(&bars->o_done);
        mma_commit(&bars->v_empty[st]);
      }
      // Every MMA issued must be complete before TMEM is released.
      mma_commit(&bars->fin);
      mbar_wait_drain(&bars->fin, 0, p.wd);
    }
  } else {
    // ------------------------------ softmax -------------------------------
    // Two warps per TMEM lane quadrant: group g = 0 (warps 2-5) owns the
    // first 64-key sub-tile of each step, group 1 (warps 6-9) the second.
    // The two threads of a row trade their sub-tile maxima through a
    // double-buffered shared slot and a 64-thread named barrier.
    const int g = (warp - 2) >> 2;
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int row, i, qtile;
    bool active;
    if (MODE == 0) {
      const bool isB = lane >= 16;
      row = 16 * q + (lane & 15);
      i = isB ? iB : iA;
      active = isB ? hasB : true;
      qtile = i;
    } else {
      row = 32 * q + lane;
      i = iA;
      active = true;
      qtile = 2 * iA + (row >> 6);
    }
    const int block = MODE == 0 ? 64 : 128;
    const int n = i * block + row;
    const size_t tb = (size_t)bh * p.nq;
    const float c0 = active ? __ldg(p.sq + tb + qtile) * (kLog2e * 0.08838834764831845f) : 0.f;
    float* xch = reinterpret_cast<float*>(smem + C::kOffBar + sizeof(Bars));  // [2][2][128]
    const int xrow = 32 * q + lane;
    uint8_t* prow_base = smem + C::kOffP + (MODE == 0 && lane >= 16 ? kTile : 0);
    // Metadata of this thread's sub-tile, one step ahead of use.
    auto tile_of = [&](int s) -> int {
      if (MODE == 0) {
        const int t = 2 * s + g;
        return (active && t < p.kc) ? list_at(p, bh, i, t) : -1;
      }
      return 2 * list_at(p, bh, i, s) + g;
    };
    int kt_cur = tile_of(0);
    float sk_cur = kt_cur >= 0 ? __ldg(p.sk + tb + kt_cur) : 0.f;
    int kt_next = nsteps > 1 ? tile_of(1) : -1;
    float m_run = -INFINITY;
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[s & 1], (s >> 1) & 1, abort, p.wd));
      if (!ok) break;
      tc_fence_after();
      const int nsub = MODE == 0 ? min(2, p.kc - 2 * s) : 2;
      const bool have = g < nsub && active && kt_cur >= 0;
      const int nvalid = have ? max(0, min(64, p.N - kt_cur * 64)) : 0;
      const float cu = c0 * sk_cur;
      uint32_t acc[64];
      if (g < nsub) {
        const uint32_t sbase = tmem + lane_base + ((s & 1) ? kColS1 : kColS0) + 64 * g;
        SAGESLA_TMEM_LD16(sbase + 0, acc + 0);
        SAGESLA_TMEM_LD16(sbase + 16, acc + 16);
        SAGESLA_TMEM_LD16(sbase + 32, acc + 32);
        SAGESLA_TMEM_LD16(sbase + 48, acc + 48);
        tmem_ld_wait();
      }
      // Prefetch the key scale of the next step (its list entry arrived).
      const float sk_next = kt_next >= 0 ? __ldg(p.sk + tb + kt_next) : 0.f;
      const int kt_after = (s + 2 < nsteps) ? tile_of(s + 2) : -1;
      int mx = INT_MIN;
      if (nvalid == 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx = max(mx, (int)acc[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < nvalid) mx = max(mx, (int)acc[c]);
      }
      const float mu = nvalid > 0 ? __int2float_rn(mx) * cu : -INFINITY;
      xch[((s & 1) * 2 + g) * 128 + xrow] = mu;
      mbar_arrive(&bars->xbar[q][s & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->xbar[q][s & 1], (s >> 1) & 1, abort, p.wd));
      if (!ok) break;
      const float mo = xch[((s & 1) * 2 + (g ^ 1)) * 128 + xrow];
      const float m_new = fmaxf(m_run, fmaxf(mu, mo));
      const float alpha = (m_run == -INFINITY) ? 1.f : ex2(m_run - m_new);
      // exponent of 448*P: (acc - max_u) * c_u + (m_u - m_new) + log2(448);
      // the integer difference is exact, so values near the running max keep
      // full precision however large the scores are.
      const float off = nvalid > 0 ? (mu - m_new) + kLog2_448 : 0.f;
      uint8_t* pbuf = prow_base + (s & 1) * C::kPBuf;
      if (g < nsub) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 16-key chunks
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 16 * ch + 4 * e;
            float x[4];
#pragma unroll
            for (int z = 0; z < 4; ++z)
              x[z] = (nvalid == 64 || c + z < nvalid)
                         ? ex2(fmaf(__int2float_rn((int)acc[c + z] - mx), cu, off))
                         : 0.f;
            w[e] = e4m3x2(x[0], x[1]) | (e4m3x2(x[2], x[3]) << 16);
          }
          *reinterpret_cast<uint4*>(pbuf + kmajor_off(row, 64 * g + 16 * ch, kQK_LBO, kQK_SBO)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // Rescale O (and its row-sum columns) when the running max moved.  The
      // two groups split the 144 columns: 0-79 and 80-143.
      if (s > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (s - 1) & 1, abort, p.wd));
        if (!ok) break;
        tc_fence_after();
        const uint32_t obase = tmem + lane_base + kColO;
        const int cbeg = g == 0 ? 0 : 80, cend = g == 0 ? 80 : kNO;
#pragma unroll 1
        for (int c = cbeg; c < cend; c += 16) {
          uint32_t o[16];
          SAGESLA_TMEM_LD16(obase + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int z = 0; z < 16; ++z) o[z] = __float_as_uint(__uint_as_float(o[z]) * alpha);
          SAGESLA_TMEM_ST16(obase + c, o);
        }
        tmem_st_wait();
      }
      m_run = m_new;
      kt_cur = kt_next;
      sk_cur = sk_next;
      kt_next = kt_after;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full[s & 1]);
    }
    // Epilogue: O_s = O / l * s_v (+ the linear branch already in out) -> bf16.
    // The last PV steps may still be in flight here, and o_done may be more
    // than one phase behind (a step that skips its rescale never waits on
    // it), which a parity wait cannot tell apart; `fin` has a single phase,
    // committed after the MMA thread's last instruction.
    const bool store = active && n < p.N;
    __nv_bfloat16* orow = p.out + ((size_t)bh * p.N + (store ? n : 0)) * kD + 64 * g;
    uint4 yrow[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      yrow[c] = (p.add_out && store) ? *reinterpret_cast<const uint4*>(orow + 8 * c) : make_uint4(0, 0, 0, 0);
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->fin, 0, abort, p.wd));
    if (ok && nsteps > 0) {
      tc_fence_after();
      const uint32_t obase = tmem + lane_base + kColO;
      uint32_t lw[16];
      SAGESLA_TMEM_LD16(obase + 128, lw);
      tmem_ld_wait();
      const float inv_l = 1.f / __uint_as_float(lw[0]);
#pragma unroll
      for (int c = 0; c < 64; c += 16) {
        uint32_t o[16];
        SAGESLA_TMEM_LD16(obase + 64 * g + c, o);
        tmem_ld_wait();
        if (store) {
          uint32_t pk[8];
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            const uint32_t yw = z < 4 ? (&yrow[c / 8].x)[z] : (&yrow[c / 8 + 1].x)[z - 4];
            const int ch = 64 * g + c + 2 * z;
            const float a = __uint_as_float(o[2 * z]) * inv_l * __ldg(p.sv + (size_t)bh * kD + ch) + bf16_lo(yw);
            const float b = __uint_as_float(o[2 * z + 1]) * inv_l * __ldg(p.sv + (size_t)bh * kD + ch + 1) + bf16_hi(yw);
            const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
            pk[z] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(orow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(orow + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

cudaError_t launch_flash(const FlashArgs& a, const Geom& g, cudaStream_t st, int* wd) {
  Params p;
  p.q8t = a.q8t;
  p.k8t = a.k8t;
  p.v8t = a.v8t;
  p.sq = a.sq;
  p.sk = a.sk;
  p.sv = a.sv;
  p.idx = a.idx;
  p.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  p.wd = wd;
  p.N = g.N;
  p.nb = g.nb;
  p.nq = g.nq;
  p.kc = g.kc;
  p.add_out = a.add_out;
  if (g.block == 64) {
    p.nsteps = (g.kc + 1) / 2;
    const int smem = Cfg<0>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(flash_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    flash_kernel<0><<<dim3((g.nb + 1) / 2, g.BH), kThreads, smem, st>>>(p);
  } else {
    p.nsteps = g.kc;
    const int smem = Cfg<1>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(flash_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    flash_kernel<1><<<dim3(g.nb, g.BH), kThreads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sagesla
