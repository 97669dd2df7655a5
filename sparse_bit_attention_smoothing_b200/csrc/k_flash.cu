// k_flash.cu -- K5: block-sparse SageAttention-style flash kernel on tcgen05.
//
// For each query block i, the key blocks of its top-k list are walked in
// ascending order, one key block at a time:
//   S = (q^ . k^) * s_q,i * s_k,j / sqrt(d)       INT8 x INT8 -> INT32 in TMEM
//   running max m updated after the block; P~ = e4m3(448 * exp(S - m))
//   O = O * exp(m_old - m) + P~ . v^               FP8 x FP8 -> FP32 in TMEM
// and finally O_s = (O / rowsum(P~)) * s_v per channel.  Sources:
// "揭秘TurboDiffusion：如何让视频生成实现百倍加速？" 支柱一 (INT8 attention with
// smoothing on integer tensor cores) and 支柱二 (only the selected blocks are
// computed exactly); 量子位 news 技术解密 1 (SageAttention2++).
//
// Work unit: block 64 -- a pair of query blocks A, B (their M=64 accumulators
// sit at TMEM lane offsets 0 and 16, so every lane holds a row); block 128 --
// one 128-row query block (M=128).  The grid is persistent: one CTA per SM
// walks units u = blockIdx.x, blockIdx.x + gridDim.x, ... (head-major, so the
// SMs share the K^/V^ tiles of one or two heads in L2).
//
// Step: two 64-key halves g = 0, 1 -- at block 64 the list entries 2s and
// 2s+1 (two walk blocks), at block 128 the two halves of list entry s (one
// walk block).  QK^T of a step is one N=128 MMA chain per query block.
// Softmax warpgroup g exponentiates half g; each thread owns one row and
// reads the other half of its row too, so it knows both maxima without any
// exchange.  Because the walk updates the running max after every walk
// block, half g accumulates in its own TMEM accumulator O_g whose frame is
// the running max after that half's block (at block 128 both frames are the
// block's max): O_g is rescaled by exp(frame_old - frame_new) before its PV,
// and the epilogue combines O_0 and O_1 in the final max.  PV is M=64/128,
// N=136/144: 128 V channels plus rows of ones, so the row sum of P~ comes
// out of the tensor core in column 128.
//
// Roles (16 warps, 1 CTA/SM):
//   warp 0      K producer: Q^ tiles of each unit (double-buffered) and the
//               K^ tiles of each step (2-stage ring), one bulk copy per tile;
//   warp 1      QK^T issuer (one thread) and TMEM owner;
//   warp 2      PV issuer (one thread);
//   warp 3      V producer: V^T tiles (2-stage ring);
//   warps 4-11  softmax: warpgroup g = 0 (warps 4-7), g = 1 (warps 8-11);
//   warps 12-15 correction: rescales O_g between its PV steps, epilogue.
// TMEM: S (128 columns, single buffer: QK^T of step s+1 waits until both
// warpgroups have loaded S(s)), O_0 at column 128, O_1 at column 272.
//
// Barrier protocol (gs = global step of this CTA, b = gs & 1): every
// per-step barrier a role can run ahead on is double-buffered by b, and each
// chain of a step passes through p_empty (PV_g(gs-2) complete) before the
// softmax publishes anything for step gs, so no parity wait is ever more
// than one phase behind its barrier.  Every wait is bounded (watchdog).
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

constexpr int kThreads = 512;
constexpr int kWarpLoadK = 0, kWarpQK = 1, kWarpPV = 2, kWarpLoadV = 3, kWarpSoft0 = 4, kWarpCorr0 = 12;
constexpr uint32_t kOnesE4M3 = 0x38383838u;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;
constexpr float kRsqrtD = 0.08838834764831845f;  // 1/sqrt(128)
constexpr uint32_t kTmemCols = 512, kColS = 0, kColO0 = 128, kColO1 = 272;
constexpr uint32_t kP_LBO = 128, kP_SBO = 512;  // P~ tiles [rows][64 keys], K-major

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
  int N, nb, nq, kc;
  int upb;     // units per head
  int units;   // BH * upb
  int nsteps;  // steps per unit
  int add_out; // 1: out already holds the linear branch (bf16); add O_s to it
  int q_tok;   // 1: one Q scale per token (sq [BH][nq*64])
  int H, tok;   // heads; out layout: 0 = [B][H][N][d], 1 = [B][N][H][d]
};

template <int MODE>
struct Cfg {
  static constexpr int kNO = MODE == 0 ? 136 : 144;  // PV N: 128 channels + ones (M=128 needs N % 16 == 0)
  static constexpr int kOnes = (kNO - 128) * 64;     // bytes of ones rows under a V^T tile
  static constexpr int kVSlot = kTile + kOnes;
  static constexpr int kSlots = MODE == 0 ? 4 : 2;   // K^ / V^T tiles per step
  static constexpr int kQBytes = 2 * kTile;
  static constexpr int kKStage = kSlots * kTile;
  static constexpr int kVStage = kSlots * kVSlot;
  static constexpr int kPTile = 8192;                // 128 rows x 64 keys
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKStage;
  static constexpr int kOffP = kOffV + 2 * kVStage;  // [parity b][half g]
  static constexpr int kOffA = kOffP + 4 * kPTile;   // alpha [g][b][128] f32
  static constexpr int kOffF = kOffA + 2 * 2 * 128 * 4;  // final frames [unit parity][g][128] f32
  static constexpr int kOffM = kOffF + 2 * 2 * 128 * 4;  // StepMeta ring [4]
  static constexpr int kOffBar = kOffM + 4 * 32;
  static constexpr int kSmem = kOffBar + 512 + 1024;  // + alignment slack
};

struct Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full, s_free;
  uint64_t a_ready[2][4][2];  // [g][quadrant][b]: alpha of the quadrant's rows published
  uint64_t p_full[2][2];      // [g][b]: P~ stored
  uint64_t p_empty[2][2];     // [g][b]: PV that read the P~ buffer complete
  uint64_t o_ready[2][2];     // [g][b]: O_g rescaled, PV_g may accumulate
  uint64_t o_done[2];         // [g]: PV_g of the step complete
  uint64_t m_full[4], m_empty[4];  // step metadata ring (producer -> softmax)
  uint64_t fin;               // every MMA of both issuers complete
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

// Per-step metadata the K producer hands to the softmax warps: the 64-key
// tiles of the step (block 64: slot 2X+g = list entry 2s+g of query block X,
// -1 when absent; block 128: slots 0, 1 = the two halves of list entry s)
// and their INT8 key scales.
struct StepMeta {
  int tile[4];
  float sk[4];
};

struct Unit {
  int bh, iA, iB;
  bool hasB;
};

template <int MODE>
__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
  Unit x;
  x.bh = u / p.upb;
  const int pi = u - x.bh * p.upb;
  if (MODE == 0) {
    x.iA = 2 * pi;
    x.iB = 2 * pi + 1;
    x.hasB = x.iB < p.nb;
  } else {
    x.iA = pi;
    x.iB = -1;
    x.hasB = false;
  }
  return x;
}

// key block (mask block index) of list entry t for query block i
__device__ __forceinline__ int list_at(const Params& p, int bh, int i, int t) {
  return p.idx ? __ldg(p.idx + ((size_t)bh * p.nb + i) * p.kc + t) : t;
}

// Max of the first `nv` of `n` integer scores (n a multiple of 8): four
// independent chains of three-input maxima when all are valid.
template <int n>
__device__ __forceinline__ int max_valid(const uint32_t* t, int nv, int m) {
  if (nv >= n) {
    int c4[4] = {m, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
    for (int c = 0; c < n; c += 8) {
      c4[0] = __vimax3_s32(c4[0], (int)t[c], (int)t[c + 1]);
      c4[1] = __vimax3_s32(c4[1], (int)t[c + 2], (int)t[c + 3]);
      c4[2] = __vimax3_s32(c4[2], (int)t[c + 4], (int)t[c + 5]);
      c4[3] = __vimax3_s32(c4[3], (int)t[c + 6], (int)t[c + 7]);
    }
    return max(max(c4[0], c4[1]), max(c4[2], c4[3]));
  }
#pragma unroll
  for (int c = 0; c < n; ++c)
    if (c < nv) m = max(m, (int)t[c]);
  return m;
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) flash_kernel(const Params p) {
  using C = Cfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  float* alpha_s = reinterpret_cast<float*>(smem + C::kOffA);
  float* frame_s = reinterpret_cast<float*>(smem + C::kOffF);
  StepMeta* meta = reinterpret_cast<StepMeta*>(smem + C::kOffM);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nsteps = p.nsteps;

  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->q_full[x], 1);
      mbar_init(&bars->q_empty[x], 1);
      mbar_init(&bars->k_full[x], 1);
      mbar_init(&bars->k_empty[x], 1);
      mbar_init(&bars->v_full[x], 1);
      mbar_init(&bars->v_empty[x], 1);
      mbar_init(&bars->o_done[x], 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bars->p_full[x][b], 4);
        mbar_init(&bars->p_empty[x][b], 1);
        mbar_init(&bars->o_ready[x][b], 4);
        for (int w = 0; w < 4; ++w) mbar_init(&bars->a_ready[x][w][b], 1);
      }
    }
    for (int x = 0; x < 4; ++x) {
      mbar_init(&bars->m_full[x], 1);
      mbar_init(&bars->m_empty[x], 8);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 8);
    mbar_init(&bars->fin, 2);
    bars->abort = 0;
    mbar_fence_init();
  }
  // Rows of ones under every V^T slot (PV's extra output columns = row sum of P~).
  constexpr int kOnesWords = C::kOnes / 16;
  for (int e = tid; e < 2 * C::kSlots * kOnesWords; e += kThreads) {
    const int slot = e / kOnesWords, w = e % kOnesWords;
    *reinterpret_cast<uint4*>(smem + C::kOffV + slot * C::kVSlot + kTile + w * 16) =
        make_uint4(kOnesE4M3, kOnesE4M3, kOnesE4M3, kOnesE4M3);
  }
  fence_proxy_async_smem();
  if (warp == kWarpQK) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp == kWarpLoadK || warp == kWarpLoadV) {
    // ---------------------------- producers -------------------------------
    if (lane == 0) {
      const bool is_k = warp == kWarpLoadK;
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const uint8_t* src = is_k ? p.k8t : p.v8t;
      const int stage_bytes = is_k ? C::kKStage : C::kVStage;
      const int slot_bytes = is_k ? kTile : C::kVSlot;
      uint8_t* ring = smem + (is_k ? C::kOffK : C::kOffV);
      int gs = 0, ui = 0, issued = 0;  // issued: steps whose copies are out
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
        const Unit un = unit_of<MODE>(p, u);
        const size_t head_tiles = (size_t)un.bh * p.nq;
        if (is_k) {
          const int qb = ui & 1;
          if (ui >= 2 && !(ok = mbar_wait(&bars->q_empty[qb], ((ui >> 1) - 1) & 1, abort, p.wd))) break;
          uint8_t* qd = smem + C::kOffQ + qb * C::kQBytes;
          mbar_expect_tx(&bars->q_full[qb], C::kQBytes);
          if (MODE == 0) {
            bulk_g2s(qd, p.q8t + (head_tiles + un.iA) * kTile, kTile, &bars->q_full[qb]);
            bulk_g2s(qd + kTile, p.q8t + (head_tiles + (un.hasB ? un.iB : un.iA)) * kTile, kTile, &bars->q_full[qb]);
          } else {
            bulk_g2s(qd, p.q8t + (head_tiles + 2 * un.iA) * kTile, 2 * kTile, &bars->q_full[qb]);
          }
        }
        for (int s = 0; s < nsteps; ++s, ++gs) {
          // Tiles of this step: slot (2X + g) = list entry 2s+g of query block X (block 64);
          // slots 0, 1 = the two 64-key tiles of list entry s (block 128).
          int tiles[4];
          int nt = 0;
          if (MODE == 0) {
            for (int x = 0; x < 2; ++x)
              for (int g = 0; g < 2; ++g) {
                const int t = 2 * s + g;
                tiles[2 * x + g] = (t < p.kc && (x == 0 || un.hasB)) ? list_at(p, un.bh, x ? un.iB : un.iA, t) : -1;
                nt += tiles[2 * x + g] >= 0;
              }
          } else {
            const int j = list_at(p, un.bh, un.iA, s);
            tiles[0] = 2 * j;
            tiles[1] = 2 * j + 1;
            nt = 2;
          }
          const int st = gs & 1;
          if (gs >= 2 && !(ok = mbar_wait(&empty[st], ((gs >> 1) - 1) & 1, abort, p.wd))) break;
          mbar_expect_tx(&full[st], nt * kTile);
          for (int x = 0; x < C::kSlots; ++x)
            if (tiles[x] >= 0)
              bulk_g2s(ring + st * stage_bytes + x * slot_bytes, src + (head_tiles + tiles[x]) * kTile, kTile,
                       &full[st]);
          issued = gs + 1;
          if (is_k) {
            // the step's metadata for the softmax warps (a 4-deep ring)
            const int ms = gs & 3;
            float skv[4];
            for (int x = 0; x < 4; ++x) skv[x] = (x < C::kSlots && tiles[x] >= 0) ? __ldg(p.sk + head_tiles + tiles[x]) : 0.f;
            if (gs >= 4 && !(ok = mbar_wait(&bars->m_empty[ms], ((gs >> 2) - 1) & 1, abort, p.wd))) break;
            for (int x = 0; x < 4; ++x) {
              meta[ms].tile[x] = x < C::kSlots ? tiles[x] : -1;
              meta[ms].sk[x] = skv[x];
            }
            mbar_arrive(&bars->m_full[ms]);
          }
        }
      }
      // Drain: every copy issued must land before the CTA may exit.  The
      // empty-wait of step g proved the copies of step g-2 consumed, so only
      // the last two steps issued can still be in flight (also when a wait
      // gave up after the copies of its step were issued).
      for (int g2 = max(0, issued - 2); g2 < issued; ++g2) mbar_wait_drain(&full[g2 & 1], (g2 >> 1) & 1, p.wd);
      if (is_k)
        for (int u2 = max(0, ui - 2); u2 < ui; ++u2) mbar_wait_drain(&bars->q_full[u2 & 1], (u2 >> 1) & 1, p.wd);
    }
  } else if (warp == kWarpQK) {
    // ------------------------------ QK^T issuer ---------------------------
    if (lane == 0) {
      const uint64_t dq = smem_desc(smem, kQK_LBO, kQK_SBO);
      int gs = 0, ui = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
        const Unit un = unit_of<MODE>(p, u);
        const int qb = ui & 1;
        if (!(ok = mbar_wait(&bars->q_full[qb], (ui >> 1) & 1, abort, p.wd))) break;
        const uint32_t qoff = C::kOffQ + qb * C::kQBytes;
        for (int s = 0; s < nsteps; ++s, ++gs) {
          const int st = gs & 1;
          if (!(ok = mbar_wait(&bars->k_full[st], (gs >> 1) & 1, abort, p.wd))) break;
          if (gs > 0 && !(ok = mbar_wait(&bars->s_free, (gs - 1) & 1, abort, p.wd))) break;
          tc_fence_after();
          const uint32_t koff = C::kOffK + st * C::kKStage;
          if (MODE == 0) {
            const uint32_t id = 2 * s + 1 < p.kc ? idesc_i8(64, 128) : idesc_i8(64, 64);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (x == 1 && !un.hasB) break;
              const uint32_t d = tmem + kColS + ((uint32_t)(x * 16) << 16);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8(d, desc_at(dq, qoff + x * kTile + kk * 256), desc_at(dq, koff + 2 * x * kTile + kk * 256), id,
                       kk > 0);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(tmem + kColS, desc_at(dq, qoff + kk * 256), desc_at(dq, koff + kk * 256), idesc_i8(128, 128),
                     kk > 0);
          }
          mma_commit(&bars->s_full);
          mma_commit(&bars->k_empty[st]);
        }
        if (ok) mma_commit(&bars->q_empty[qb]);
      }
      mma_commit(&bars->fin);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------ PV issuer -----------------------------
    if (lane == 0) {
      const uint64_t dp = smem_desc(smem, kP_LBO, kP_SBO);
      const uint64_t dv = smem_desc(smem, kV_LBO, kV_SBO);
      const uint32_t id = idesc_e4m3(MODE == 0 ? 64 : 128, C::kNO);
      int gs = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const Unit un = unit_of<MODE>(p, u);
        for (int s = 0; s < nsteps; ++s, ++gs) {
          const int st = gs & 1, b = gs & 1, ph = (gs >> 1) & 1;
          if (!(ok = mbar_wait(&bars->v_full[st], ph, abort, p.wd))) break;
          for (int g = 0; g < 2; ++g) {
            if (!(ok = mbar_wait(&bars->p_full[g][b], ph, abort, p.wd))) break;
            if (!(ok = mbar_wait(&bars->o_ready[g][b], ph, abort, p.wd))) break;
            tc_fence_after();
            const bool has = MODE == 0 ? 2 * s + g < p.kc : true;
            if (has) {
              const uint32_t o = tmem + (g ? kColO1 : kColO0);
              const uint32_t poff = C::kOffP + (2 * b + g) * C::kPTile;
              const uint32_t voff = C::kOffV + st * C::kVStage;
#pragma unroll
              for (int x = 0; x < (MODE == 0 ? 2 : 1); ++x) {
                if (x == 1 && !un.hasB) break;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                  mma_e4m3(o + ((uint32_t)(x * 16) << 16), desc_at(dp, poff + x * 4096 + kk * 256),
                           desc_at(dv, voff + (MODE == 0 ? 2 * x + g : g) * C::kVSlot + kk * 256), id,
                           (s > 0 || kk > 0));
              }
            }
            mma_commit(&bars->o_done[g]);
            mma_commit(&bars->p_empty[g][b]);
          }
          if (!ok) break;
          mma_commit(&bars->v_empty[st]);
        }
      }
      mma_commit(&bars->fin);
    }
  } else if (warp < kWarpCorr0) {
    // ------------------------------ softmax -------------------------------
    const int g = (warp - kWarpSoft0) >> 2;
    const int w = warp & 3;  // TMEM lane quadrant
    const uint32_t lane_base = (uint32_t)(32 * w) << 16;
    const int L = 32 * w + lane;  // TMEM lane of this row
    int gs = 0, ui = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
      const Unit un = unit_of<MODE>(p, u);
      int r, qtile, xs;
      bool active;
      if (MODE == 0) {
        const bool isB = lane >= 16;
        r = 16 * w + (lane & 15);
        active = isB ? un.hasB : true;
        qtile = isB ? un.iB : un.iA;
        xs = isB ? 2 : 0;  // metadata slots of this row's query block
      } else {
        r = L;
        active = true;
        qtile = 2 * un.iA + (r >> 6);
        xs = 0;
      }
      const size_t sqi = (size_t)un.bh * p.nq + qtile;
      const float c0 = active ? __ldg(p.sq + (p.q_tok ? sqi * kQB + (r & 63) : sqi)) * (kLog2e * kRsqrtD) : 0.f;
      uint8_t* prow = smem + C::kOffP + g * C::kPTile + (MODE == 0 && lane >= 16 ? 4096 : 0);
      float m_all = -INFINITY, frame = -INFINITY;
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const int b = gs & 1;
        // Key tiles of this row's own half and of the other half, and their
        // scales, from the producer's metadata ring (no global loads here).
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->m_full[gs & 3], (gs >> 2) & 1, abort, p.wd));
        if (!ok) break;
        const StepMeta& mt = meta[gs & 3];
        const int t_own = active ? mt.tile[xs + g] : -1;
        const int t_oth = active ? mt.tile[xs + 1 - g] : -1;
        const int nv_own = t_own >= 0 ? max(0, min(64, p.N - 64 * t_own)) : 0;
        const int nv_oth = t_oth >= 0 ? max(0, min(64, p.N - 64 * t_oth)) : 0;
        const float cu_own = c0 * mt.sk[xs + g], cu_oth = c0 * mt.sk[xs + 1 - g];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->m_empty[gs & 3]);
        // The P~ buffer b was read by PV_g(gs-2); waiting for it first keeps
        // every barrier this warp publishes on at most one phase ahead.
        if (gs >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_empty[g][b], ((gs >> 1) - 1) & 1, abort, p.wd));
          if (!ok) break;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, gs & 1, abort, p.wd));
        if (!ok) break;
        tc_fence_after();
        uint32_t acc[64];
        int mx_oth = INT_MIN;
        {
          const uint32_t so = tmem + lane_base + kColS + 64 * g;
          const uint32_t sx = tmem + lane_base + kColS + 64 * (1 - g);
          uint32_t t[32];
          SAGESLA_TMEM_LD16(so + 0, acc + 0);
          SAGESLA_TMEM_LD16(so + 16, acc + 16);
          SAGESLA_TMEM_LD16(so + 32, acc + 32);
          SAGESLA_TMEM_LD16(so + 48, acc + 48);
          SAGESLA_TMEM_LD16(sx + 0, t + 0);
          SAGESLA_TMEM_LD16(sx + 16, t + 16);
          tmem_ld_wait();
          mx_oth = max_valid<32>(t, nv_oth, mx_oth);
          SAGESLA_TMEM_LD16(sx + 32, t + 0);
          SAGESLA_TMEM_LD16(sx + 48, t + 16);
          tmem_ld_wait();
          mx_oth = max_valid<32>(t, nv_oth - 32, mx_oth);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        const int mx_own = max_valid<64>(acc, nv_own, INT_MIN);
        const float mf_own = nv_own > 0 ? __int2float_rn(mx_own) * cu_own : -INFINITY;
        const float mf_oth = nv_oth > 0 ? __int2float_rn(mx_oth) * cu_oth : -INFINITY;
        // Frame of O_g after this step: at block 64 half 0 is walk block 2s
        // (max over the blocks so far and this one), half 1 is block 2s+1
        // (which has also seen block 2s); at block 128 both are the block's max.
        float fnew = (MODE == 0 && g == 0) ? fmaxf(m_all, mf_own) : fmaxf(m_all, fmaxf(mf_own, mf_oth));
        m_all = fmaxf(m_all, fmaxf(mf_own, mf_oth));
        if (nv_own == 0) fnew = frame;  // no block for this half: O_g keeps its frame
        const float alpha = (frame == -INFINITY || fnew == -INFINITY) ? 1.f : ex2(frame - fnew);
        frame = fnew;
        alpha_s[(g * 2 + b) * 128 + L] = alpha;
        if (s == nsteps - 1) frame_s[((ui & 1) * 2 + g) * 128 + L] = frame;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->a_ready[g][w][b]);
        // P~ of the own half: exponent of 448*P = S*c - frame + log2(448), one
        // fused multiply-add per key on the converted integer score, two keys
        // per f32x2 instruction; keys past the sequence end get P~ = 0.  Each
        // phase runs over all 64 keys so that the conversions, the
        // exponentials and the FP8 packing of different keys overlap.
        uint8_t* pbuf = prow + 2 * b * C::kPTile;
        // (block 128: a half past the sequence end still feeds the PV, with P~ = 0)
        if (nv_own > 0 || (MODE == 1 && active)) {
          const float kk = kLog2_448 - frame;
          const uint64_t cc = f32x2_pack(cu_own, cu_own), ko = f32x2_pack(kk, kk);
          // Software-pipelined over 16-key chunks: the conversions and FMAs of
          // chunk ch+1 (I2F and FMA pipes) are issued next to the exponentials
          // of chunk ch (ex2 unit), so the two pipes overlap.
          float xc[16], xn[16];
          auto conv = [&](int ch, float (&x)[16]) {
#pragma unroll
            for (int z = 0; z < 16; z += 2) {
              const int c = 16 * ch + z;
              const uint64_t dd =
                  f32x2_fma(f32x2_pack(__int2float_rn((int)acc[c]), __int2float_rn((int)acc[c + 1])), cc, ko);
              f32x2_unpack(dd, x[z], x[z + 1]);
            }
          };
          conv(0, xc);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            if (ch < 3) conv(ch + 1, xn);
#pragma unroll
            for (int z = 0; z < 16; ++z) xc[z] = ex2(xc[z]);
            if (nv_own < 64) {
#pragma unroll
              for (int z = 0; z < 16; ++z)
                if (16 * ch + z >= nv_own) xc[z] = 0.f;
            }
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              wv[e] = __byte_perm(e4m3x2(xc[4 * e], xc[4 * e + 1]), e4m3x2(xc[4 * e + 2], xc[4 * e + 3]), 0x5410);
            *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, 16 * ch, kP_LBO, kP_SBO)) =
                make_uint4(wv[0], wv[1], wv[2], wv[3]);
            if (ch < 3) {
#pragma unroll
              for (int z = 0; z < 16; ++z) xc[z] = xn[z];
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[g][b]);
      }
    }
  } else {
    // ------------------------------ correction ----------------------------
    // One warp per TMEM lane quadrant; thread = row.  Between PV_g(gs-1) and
    // PV_g(gs) it multiplies the row's O_g (channels and row sum) by alpha
    // when the frame moved; after a unit's last step it writes the output.
    const int w = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * w) << 16;
    const int L = 32 * w + lane;
    int gs = 0, ui = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
      const Unit un = unit_of<MODE>(p, u);
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const int b = gs & 1, ph = (gs >> 1) & 1;
        for (int g = 0; g < 2; ++g) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->a_ready[g][w][b], ph, abort, p.wd));
          if (!ok) break;
          const float alpha = alpha_s[(g * 2 + b) * 128 + L];
          const bool has = MODE == 0 ? 2 * s + g < p.kc : true;
          // PV_g(gs-1) must be complete before O_g is touched; the wait is
          // taken at every step (not only when rescaling) so that each parity
          // wait on o_done, the epilogue's included, is one phase ahead at most.
          if (s > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[g], (gs - 1) & 1, abort, p.wd));
            if (!ok) break;
          }
          if (s > 0 && has && __any_sync(0xffffffffu, alpha != 1.f)) {
            tc_fence_after();
            const uint32_t ob = tmem + lane_base + (g ? kColO1 : kColO0);
            const uint64_t a2 = f32x2_pack(alpha, alpha);
            // 144 columns (128 channels + the row-sum columns) in chunks of 32
            // (the last 16): the load of chunk c+1 is in flight while chunk c
            // is multiplied and stored.
            uint32_t o[2][32];
            SAGESLA_TMEM_LD16(ob + 0, o[0]);
            SAGESLA_TMEM_LD16(ob + 16, o[0] + 16);
            tmem_ld_wait();
#pragma unroll
            for (int ch = 0; ch < 5; ++ch) {
              uint32_t* cur = o[ch & 1];
              uint32_t* nxt = o[(ch + 1) & 1];
              if (ch < 3) {
                SAGESLA_TMEM_LD16(ob + 32 * (ch + 1), nxt);
                SAGESLA_TMEM_LD16(ob + 32 * (ch + 1) + 16, nxt + 16);
              } else if (ch == 3) {
                SAGESLA_TMEM_LD16(ob + 128, nxt);
              }
              const int n = ch < 4 ? 32 : 16;
#pragma unroll
              for (int z = 0; z < 32; z += 2) {
                if (z >= n) break;
                float a0, a1;
                f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(cur[z]), __uint_as_float(cur[z + 1])), a2), a0, a1);
                cur[z] = __float_as_uint(a0);
                cur[z + 1] = __float_as_uint(a1);
              }
              SAGESLA_TMEM_ST16(ob + 32 * ch, cur);
              if (n == 32) SAGESLA_TMEM_ST16(ob + 32 * ch + 16, cur + 16);
              if (ch < 4) tmem_ld_wait();
            }
            tmem_st_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->o_ready[g][b]);
        }
        if (!ok) break;
      }
      if (!ok) break;
      // ------------------------------ epilogue ----------------------------
      // out = (O_0 f_0 + O_1 f_1) / (l_0 f_0 + l_1 f_1) * s_v (+ the linear
      // branch already in out), f_g = exp(frame_g - max of both frames).
      int r, i;
      bool active;
      if (MODE == 0) {
        r = 16 * w + (lane & 15);
        i = lane >= 16 ? un.iB : un.iA;
        active = lane >= 16 ? un.hasB : true;
      } else {
        r = L;
        i = un.iA;
        active = true;
      }
      const int n = i * (MODE == 0 ? 64 : 128) + r;
      const bool store = active && n < p.N;
      const bool has1 = MODE == 1 || p.kc >= 2;
      __nv_bfloat16* orow = p.out + row_elems(p.tok, p.H, p.N, un.bh, store ? n : 0);
      const bool add = p.add_out && store;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[0], (gs - 1) & 1, abort, p.wd));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[1], (gs - 1) & 1, abort, p.wd));
      if (!ok) break;
      tc_fence_after();
      const float fr0 = frame_s[((ui & 1) * 2 + 0) * 128 + L];
      const float fr1 = has1 ? frame_s[((ui & 1) * 2 + 1) * 128 + L] : -INFINITY;
      const float fm = fmaxf(fr0, fr1);
      const float f0 = fr0 == -INFINITY ? 0.f : ex2(fr0 - fm);
      const float f1 = fr1 == -INFINITY ? 0.f : ex2(fr1 - fm);
      const uint32_t ob0 = tmem + lane_base + kColO0, ob1 = tmem + lane_base + kColO1;
      float l0, l1 = 0.f;
      {
        uint32_t t0[16], t1[16];
        SAGESLA_TMEM_LD16(ob0 + 128, t0);
        if (has1) SAGESLA_TMEM_LD16(ob1 + 128, t1);
        tmem_ld_wait();
        l0 = __uint_as_float(t0[0]);
        if (has1) l1 = __uint_as_float(t1[0]);
      }
      const float inv = 1.f / (l0 * f0 + l1 * f1);
      const float g0 = f0 * inv, g1 = f1 * inv;
      const float* svh = p.sv + (size_t)un.bh * kD;
#pragma unroll 1
      for (int c = 0; c < kD; c += 16) {
        uint32_t o0[16], o1[16];
        const uint4 y0 = add ? *reinterpret_cast<const uint4*>(orow + c) : make_uint4(0, 0, 0, 0);
        const uint4 y1 = add ? *reinterpret_cast<const uint4*>(orow + c + 8) : make_uint4(0, 0, 0, 0);
        SAGESLA_TMEM_LD16(ob0 + c, o0);
        if (has1) SAGESLA_TMEM_LD16(ob1 + c, o1);
        tmem_ld_wait();
        if (store) {
          const uint32_t yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
          uint32_t pk[8];
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            const uint32_t yw = yv[z];
            const int ch = c + 2 * z;
            float a = __uint_as_float(o0[2 * z]) * g0, bq = __uint_as_float(o0[2 * z + 1]) * g0;
            if (has1) {
              a = fmaf(__uint_as_float(o1[2 * z]), g1, a);
              bq = fmaf(__uint_as_float(o1[2 * z + 1]), g1, bq);
            }
            a = fmaf(a, __ldg(svh + ch), bf16_lo(yw));
            bq = fmaf(bq, __ldg(svh + ch + 1), bf16_hi(yw));
            const __nv_bfloat162 h = __floats2bfloat162_rn(a, bq);
            pk[z] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(orow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(orow + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      tc_fence_before();
    }
  }
  // Every MMA has completed once `fin` has both issuers' arrivals.
  if (warp == kWarpQK) {
    if (lane == 0) mbar_wait_drain(&bars->fin, 0, p.wd);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpQK) tmem_dealloc(tmem, kTmemCols);
}

// Block 128 (one 128-row query block per unit, M = 128); block 64 runs the
// two-slot kernel of k_flash64.cu.
cudaError_t launch_flash128(const FlashArgs& a, const Geom& g, cudaStream_t st, int* wd) {
  Params p;
  p.q8t = a.q8t;
  p.k8t = a.k8t;
  p.v8t = a.v8t;
  p.sq = a.sq;
  p.q_tok = a.q_tok;
  p.H = g.H;
  p.tok = g.tok;
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
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  p.upb = g.nb;
  p.nsteps = g.kc;
  p.units = g.BH * p.upb;
  const int grid = p.units < sms ? p.units : sms;
  const int smem = Cfg<1>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(flash_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  flash_kernel<1><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sagesla
