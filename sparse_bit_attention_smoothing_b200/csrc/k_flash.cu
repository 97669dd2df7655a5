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
// Roles on the SM (16 warps, 1 CTA/SM):
//   warp 0     K producer: bulk copies of the Q^ and K^ tiles (pre-tiled in
//              HBM by the quantiser, so one cp.async.bulk moves a whole tile);
//   warp 1     QK^T issuer (one thread) and TMEM owner;
//   warp 2     PV issuer (one thread) -- two issuers keep the tensor pipe fed
//              while either of them waits;
//   warp 3     V producer: bulk copies of the V^T tiles.  K and V have their
//              own producers so a K copy never queues behind a V stage that
//              the later PV step still holds;
//   warps 4-11 softmax: two warps per TMEM lane quadrant, each owning one
//              64-key sub-tile of the 128-key step of every row;
//   warps 12-15 correction: one warp per quadrant; rescales O by
//              exp(m_old - m_new) between PV steps, off the softmax path, and
//              runs the epilogue.
// Mode 64 (block 64): a CTA owns two query blocks A and B.  Their M=64
//   accumulators share TMEM columns at lane offsets 0 and 16, so all 128
//   lanes hold a row.  Each step takes two key blocks per query block (S tile
//   N = 128); PV is M=64, N=144 (128 V channels + 16 rows of ones whose
//   product is the row sum of P~).
// Mode 128 (block 128): one query block of 128 rows per CTA, M = 128.
// TMEM: S double buffer (2 x 128 cols) + O (144 cols) of 512 allocated.
//
// Step hand-offs (s = step): S(s) -> s_full -> softmax(s) -> p_full(s) ->
// correction(s) [waits PV(s-1)] -> s_free(s), o_ready(s) -> PV(s) -> o_done.
// QK^T for step s+2 waits s_free(s) (its S buffer and alpha slot are then
// free); P is triple-buffered, so the buffer softmax(s+3) writes was read by
// PV(s), which correction(s+1) saw complete before s_free(s+1) released
// QK^T(s+3).  Every parity wait below is at most one phase behind its
// barrier (o_ready has the PV issuer as its only waiter).
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kStages = 2;
constexpr int kPBufs = 3;
constexpr int kSoftThreads = 256;
constexpr int kCorrThreads = 128;
constexpr int kWarpSoft0 = 4, kWarpCorr0 = 12;
constexpr int kThreads = 32 * 4 + kSoftThreads + kCorrThreads;  // 512
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
  static constexpr int kOffBar = kOffP + kPBufs * kPBuf;
  static constexpr int kBarBytes = 512;
  static constexpr int kOffX = kOffBar + kBarBytes;      // row-max exchange [2][2][128] f32
  static constexpr int kOffA = kOffX + 2 * 2 * 128 * 4;  // alpha [2][128] f32
  static constexpr int kSmem = kOffA + 2 * 128 * 4 + 1024;  // + alignment slack
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_ready, o_done;
  uint64_t s_free[2];
  uint64_t fin;
  uint64_t xbar[4][2];  // row-max exchange between the two softmax warps of a quadrant
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

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
  float* xch = reinterpret_cast<float*>(smem + C::kOffX);
  float* alpha_s = reinterpret_cast<float*>(smem + C::kOffA);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  // Query blocks of this CTA (mask-block indices).
  const int iA = MODE == 0 ? 2 * (int)blockIdx.x : (int)blockIdx.x;
  const int iB = MODE == 0 ? 2 * (int)blockIdx.x + 1 : -1;
  const bool hasB = MODE == 0 && iB < p.nb;
  const int nsteps = p.nsteps;

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
    mbar_init(&bars->o_ready, kCorrThreads);
    mbar_init(&bars->s_free[0], kCorrThreads);
    mbar_init(&bars->s_free[1], kCorrThreads);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->fin, 2);
    for (int qq = 0; qq < 4; ++qq)
      for (int b = 0; b < 2; ++b) mbar_init(&bars->xbar[qq][b], 64);
    bars->abort = 0;
    mbar_fence_init();
  }
  // Rows of ones under every V slot (PV's extra 16 output columns = row sum).
  for (int e = tid; e < kStages * (C::kVStage / kVSlot) * 64; e += kThreads) {
    const int slot = e / 64, w = e % 64;
    *reinterpret_cast<uint4*>(smem + C::kOffV + slot * kVSlot + kTile + w * 16) =
        make_uint4(kOnesE4M3, kOnesE4M3, kOnesE4M3, kOnesE4M3);
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp == 0 || warp == 3) {
    // ------------------------- K and V producers --------------------------
    // warp 0 copies Q^ and the K^ tiles of each step, warp 3 the V^T tiles.
    // The list entries of step s+1 are read before the wait for stage s, so
    // their latency hides behind it.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const size_t head_tiles = (size_t)bh * p.nq;
      if (is_k) {
        mbar_expect_tx(&bars->q_full, C::kQBytes);
        if (MODE == 0) {
          bulk_g2s(smem + C::kOffQ, p.q8t + (head_tiles + iA) * kTile, kTile, &bars->q_full);
          const int ib = hasB ? iB : iA;  // keep the transaction count fixed
          bulk_g2s(smem + C::kOffQ + kTile, p.q8t + (head_tiles + ib) * kTile, kTile, &bars->q_full);
        } else {
          bulk_g2s(smem + C::kOffQ, p.q8t + (head_tiles + 2 * iA) * kTile, 2 * kTile, &bars->q_full);
        }
      }
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const uint8_t* src = is_k ? p.k8t : p.v8t;
      auto entries = [&](int s, int (&jj)[2][2]) {
        jj[0][0] = jj[0][1] = jj[1][0] = jj[1][1] = -1;
        if (s >= nsteps) return;
        if (MODE == 0) {
          const int nsub = min(2, p.kc - 2 * s);
          for (int x = 0; x < 2; ++x) {
            const int i = (x == 0 || !hasB) ? iA : iB;
            for (int u = 0; u < nsub; ++u) jj[x][u] = list_at(p, bh, i, 2 * s + u);
          }
        } else {
          jj[0][0] = list_at(p, bh, iA, s);
        }
      };
      int jn[2][2];
      entries(0, jn);
      int issued = 0;  // steps whose copies were issued
      for (int s = 0; s < nsteps && !*abort; ++s) {
        const int st = s % kStages;
        int jj[2][2];
        for (int x = 0; x < 2; ++x)
          for (int u = 0; u < 2; ++u) jj[x][u] = jn[x][u];
        entries(s + 1, jn);
        if (s >= kStages && !mbar_wait(&empty[st], ((s / kStages) - 1) & 1, abort, p.wd)) break;
        if (MODE == 0) {
          const int nsub = min(2, p.kc - 2 * s);
          mbar_expect_tx(&full[st], 2 * nsub * kTile);
          for (int x = 0; x < 2; ++x)
            for (int u = 0; u < nsub; ++u) {
              uint8_t* dst = is_k ? smem + C::kOffK + st * C::kKStage + (2 * x + u) * kTile
                                  : smem + C::kOffV + st * C::kVStage + (2 * x + u) * kVSlot;
              bulk_g2s(dst, src + (head_tiles + jj[x][u]) * kTile, kTile, &full[st]);
            }
        } else {
          const int j = jj[0][0];
          mbar_expect_tx(&full[st], 2 * kTile);
          if (is_k) {
            bulk_g2s(smem + C::kOffK + st * C::kKStage, src + (head_tiles + 2 * j) * kTile, 2 * kTile, &full[st]);
          } else {
            uint8_t* vd = smem + C::kOffV + st * C::kVStage;
            bulk_g2s(vd, src + (head_tiles + 2 * j) * kTile, kTile, &full[st]);
            bulk_g2s(vd + kVSlot, src + (head_tiles + 2 * j + 1) * kTile, kTile, &full[st]);
          }
        }
        issued = s + 1;
      }
      // Drain: every copy issued must land before the CTA may exit.
      if (is_k) mbar_wait_drain(&bars->q_full, 0, p.wd);
      for (int s = max(0, issued - kStages); s < issued; ++s)
        mbar_wait_drain(&full[s % kStages], (s / kStages) & 1, p.wd);
    }
  } else if (warp == 1) {
    // ------------------------------ QK^T issuer ---------------------------
    if (lane == 0) {
      const uint64_t dqk = smem_desc(smem, kQK_LBO, kQK_SBO);
      bool ok = mbar_wait(&bars->q_full, 0, abort, p.wd);
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s % kStages;
        if (!(ok = mbar_wait(&bars->k_full[st], (s / kStages) & 1, abort, p.wd))) break;
        // S buffer s&1 and alpha slot s&1 are free once step s-2 is corrected.
        if (s >= 2) {
          if (!(ok = mbar_wait(&bars->s_free[s & 1], ((s - 2) >> 1) & 1, abort, p.wd))) break;
          tc_fence_after();
        }
        const uint32_t dS = tmem + ((s & 1) ? kColS1 : kColS0);
        const uint32_t koff = C::kOffK + st * C::kKStage;
        if (MODE == 0) {
          const uint32_t id = p.kc - 2 * s >= 2 ? idesc_i8(64, 128) : idesc_i8(64, 64);
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (x == 1 && !hasB) break;
            const uint32_t d = dS + ((uint32_t)(x * 16) << 16);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(d, desc_at(dqk, C::kOffQ + x * kTile + kk * 256), desc_at(dqk, koff + 2 * x * kTile + kk * 256), id,
                     kk > 0);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(dS, desc_at(dqk, C::kOffQ + kk * 256), desc_at(dqk, koff + kk * 256), idesc_i8(128, 128), kk > 0);
        }
        mma_commit(&bars->s_full[s & 1]);
        mma_commit(&bars->k_empty[st]);
      }
      mma_commit(&bars->fin);
    }
  } else if (warp == 2) {
    // ------------------------------ PV issuer -----------------------------
    if (lane == 0) {
      const uint64_t dqk = smem_desc(smem, kQK_LBO, kQK_SBO);
      const uint64_t dv = smem_desc(smem, kV_LBO, kV_SBO);
      const uint32_t id_pv = idesc_e4m3(MODE == 0 ? 64 : 128, kNO);
      bool ok = true;
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s % kStages;
        if (!(ok = mbar_wait(&bars->v_full[st], (s / kStages) & 1, abort, p.wd))) break;
        if (!(ok = mbar_wait(&bars->o_ready, s & 1, abort, p.wd))) break;
        tc_fence_after();
        const uint32_t voff = C::kOffV + st * C::kVStage;
        const uint32_t poff = C::kOffP + (s % kPBufs) * C::kPBuf;
        if (MODE == 0) {
          const int nk = p.kc - 2 * s >= 2 ? 4 : 2;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (x == 1 && !hasB) break;
            const uint32_t d = tmem + kColO + ((uint32_t)(x * 16) << 16);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk >= nk) break;
              mma_e4m3(d, desc_at(dqk, poff + x * kTile + kk * 256),
                       desc_at(dv, voff + (2 * x + (kk >> 1)) * kVSlot + (kk & 1) * 256), id_pv, (s > 0 || kk > 0));
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_e4m3(tmem + kColO, desc_at(dqk, poff + kk * 256), desc_at(dv, voff + (kk >> 1) * kVSlot + (kk & 1) * 256),
                     id_pv, (s > 0 || kk > 0));
        }
        mma_commit(&bars->o_done);
        mma_commit(&bars->v_empty[st]);
      }
      mma_commit(&bars->fin);
    }
  } else if (warp < kWarpCorr0) {
    // ------------------------------ softmax -------------------------------
    // Two warps per TMEM lane quadrant: group g = 0 owns the first 64-key
    // sub-tile of each step, group 1 the second.  The two threads of a row
    // trade their sub-tile maxima through a double-buffered shared slot and a
    // per-quadrant mbarrier (bounded wait).
    const int g = (warp - kWarpSoft0) >> 2;
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
    const size_t tb = (size_t)bh * p.nq;
    const float c0 = active ? __ldg(p.sq + tb + qtile) * (kLog2e * 0.08838834764831845f) : 0.f;
    const int xrow = 32 * q + lane;  // TMEM lane of this row
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
    for (int s = 0; s < nsteps; ++s) {
      bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[s & 1], (s >> 1) & 1, abort, p.wd));
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
      int mx = INT_MIN;
      if (nvalid == 64) {
        int m2[2] = {INT_MIN, INT_MIN};  // two chains of three-input maxima
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          m2[0] = __vimax3_s32(m2[0], (int)acc[c], (int)acc[c + 1]);
          m2[1] = __vimax3_s32(m2[1], (int)acc[c + 2], (int)acc[c + 3]);
        }
        mx = max(m2[0], m2[1]);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < nvalid) mx = max(mx, (int)acc[c]);
      }
      const float mu = nvalid > 0 ? __int2float_rn(mx) * cu : -INFINITY;
      xch[((s & 1) * 2 + g) * 128 + xrow] = mu;
      mbar_arrive(&bars->xbar[q][s & 1]);
      // Prefetch the key scale of the next step (its list entry arrived) only
      // now: an mbarrier arrive has release semantics and would wait for
      // these global loads to complete.
      const float sk_next = kt_next >= 0 ? __ldg(p.sk + tb + kt_next) : 0.f;
      const int kt_after = (s + 2 < nsteps) ? tile_of(s + 2) : -1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->xbar[q][s & 1], (s >> 1) & 1, abort, p.wd));
      if (!ok) break;
      const float mo = xch[((s & 1) * 2 + (g ^ 1)) * 128 + xrow];
      const float m_new = fmaxf(m_run, fmaxf(mu, mo));
      if (g == 0) alpha_s[(s & 1) * 128 + xrow] = (m_run == -INFINITY) ? 1.f : ex2(m_run - m_new);
      // exponent of 448*P: (acc - max_u) * c_u + (m_u - m_new) + log2(448); the
      // integer difference is exact, so values near the running max keep full
      // precision however large the scores are.
      // Exponent of 448*P~: S*log2(e) - m_new + log2(448), one fused
      // multiply-add per key on the integer score (exact in fp32: |acc| <
      // 2^24), two keys per f32x2 instruction; keys past the sequence end
      // (last key block) get P~ = 0.
      uint8_t* pbuf = prow_base + (s % kPBufs) * C::kPBuf;
      const float kk = kLog2_448 - m_new;
      const uint64_t cc = f32x2_pack(cu, cu), ko = f32x2_pack(kk, kk);
      // (two copies of the loop: the masked one only for a ragged last block)
      if (g < nsub && nvalid == 64) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 16-key chunks
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float x[4];
#pragma unroll
            for (int z = 0; z < 4; z += 2) {
              const int c = 16 * ch + 4 * e + z;
              const uint64_t d =
                  f32x2_fma(f32x2_pack(__int2float_rn((int)acc[c]), __int2float_rn((int)acc[c + 1])), cc, ko);
              float a, b;
              f32x2_unpack(d, a, b);
              x[z] = ex2(a);
              x[z + 1] = ex2(b);
            }
            w[e] = __byte_perm(e4m3x2(x[0], x[1]), e4m3x2(x[2], x[3]), 0x5410);
          }
          *reinterpret_cast<uint4*>(pbuf + kmajor_off(row, 64 * g + 16 * ch, kQK_LBO, kQK_SBO)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else if (g < nsub) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 16-key chunks
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float x[4];
#pragma unroll
            for (int z = 0; z < 4; z += 2) {
              const int c = 16 * ch + 4 * e + z;
              const uint64_t d =
                  f32x2_fma(f32x2_pack(__int2float_rn((int)acc[c]), __int2float_rn((int)acc[c + 1])), cc, ko);
              float a, b;
              f32x2_unpack(d, a, b);
              x[z] = ex2(a);
              x[z + 1] = ex2(b);
            }
#pragma unroll
            for (int z = 0; z < 4; ++z)
              if (16 * ch + 4 * e + z >= nvalid) x[z] = 0.f;
            w[e] = __byte_perm(e4m3x2(x[0], x[1]), e4m3x2(x[2], x[3]), 0x5410);
          }
          *reinterpret_cast<uint4*>(pbuf + kmajor_off(row, 64 * g + 16 * ch, kQK_LBO, kQK_SBO)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      m_run = m_new;
      kt_cur = kt_next;
      sk_cur = sk_next;
      kt_next = kt_after;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full[s & 1]);
    }
  } else {
    // ------------------------------ correction ----------------------------
    // One warp per quadrant; thread = TMEM lane (one row of A/B or of the
    // 128-row block).  Between PV(s-1) and PV(s) it multiplies the row's O
    // and row-sum columns by alpha(s) when the running max moved.
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const uint32_t obase = tmem + lane_base + kColO;
    const int xrow = 32 * q + lane;
    int row, i;
    bool active;
    if (MODE == 0) {
      row = 16 * q + (lane & 15);
      i = lane >= 16 ? iB : iA;
      active = lane >= 16 ? hasB : true;
    } else {
      row = 32 * q + lane;
      i = iA;
      active = true;
    }
    const int block = MODE == 0 ? 64 : 128;
    const int n = i * block + row;
    const bool store = active && n < p.N;
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_full[s & 1], (s >> 1) & 1, abort, p.wd));
      if (!ok) break;
      tc_fence_after();
      const float alpha = alpha_s[(s & 1) * 128 + xrow];
      // PV(s-1) must be complete before O is touched, before PV(s) may start
      // and before QK^T(s+2) may release the P buffer softmax(s+3) writes.
      if (s > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (s - 1) & 1, abort, p.wd));
        if (!ok) break;
        tc_fence_after();
      }
      tc_fence_before();
      mbar_arrive(&bars->s_free[s & 1]);
      if (s > 0) {
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < kNO; c += 16) {
            uint32_t o[16];
            SAGESLA_TMEM_LD16(obase + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int z = 0; z < 16; ++z) o[z] = __float_as_uint(__uint_as_float(o[z]) * alpha);
            SAGESLA_TMEM_ST16(obase + c, o);
          }
          tmem_st_wait();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_ready);
    }
    // Epilogue: O_s = O / l * s_v (+ the linear branch already in out) -> bf16.
    __nv_bfloat16* orow = p.out + ((size_t)bh * p.N + (store ? n : 0)) * kD;
    uint4 yrow[16];
#pragma unroll
    for (int c = 0; c < 16; ++c)
      yrow[c] = (p.add_out && store) ? *reinterpret_cast<const uint4*>(orow + 8 * c) : make_uint4(0, 0, 0, 0);
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->fin, 0, abort, p.wd));
    if (ok && nsteps > 0) {
      tc_fence_after();
      uint32_t lw[16];
      SAGESLA_TMEM_LD16(obase + 128, lw);
      tmem_ld_wait();
      const float inv_l = 1.f / __uint_as_float(lw[0]);
#pragma unroll
      for (int c = 0; c < kD; c += 16) {
        uint32_t o[16];
        SAGESLA_TMEM_LD16(obase + c, o);
        tmem_ld_wait();
        if (store) {
          uint32_t pk[8];
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            const uint32_t yw = z < 4 ? (&yrow[c / 8].x)[z] : (&yrow[c / 8 + 1].x)[z - 4];
            const int ch = c + 2 * z;
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
  // Every MMA has completed once `fin` has both issuers' arrivals.
  if (warp == 1) {
    if (lane == 0) mbar_wait_drain(&bars->fin, 0, p.wd);
    __syncwarp();
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
