// k_flash64.cu -- K5 at block 64: block-sparse SageAttention-style flash
// kernel on tcgen05, two independent query-block pipelines per SM.
//
// For each query block i (64 rows) the key blocks of its top-k list are
// walked in ascending order, one selected block at a time:
//   S = (q^ . k^) * s_q,i * s_k,j / sqrt(d)       INT8 x INT8 -> INT32 in TMEM
//   running max m updated after the block; P~ = e4m3(448 * exp(S - m))
//   O = O * exp(m_old - m) + P~ . v^               FP8 x FP8 -> FP32 in TMEM
// and O_s = (O / rowsum(P~)) * s_v per channel.  Sources:
// "揭秘TurboDiffusion：如何让视频生成实现百倍加速？" 支柱一 (INT8 attention with
// smoothing on integer tensor cores) and 支柱二 (only the selected blocks are
// computed exactly); 量子位 news 技术解密 1 (SageAttention2++).
//
// Two slots per CTA.  An M=64 tcgen05 accumulator occupies TMEM lanes
// (r % 16) + 32 (r / 16) + 16 X, so slot X = 0 and slot X = 1 share every
// TMEM column but own disjoint lanes.  Each slot walks its own sequence of
// query blocks (items q = 2 blockIdx.x + X, + 2 gridDim.x, ...) with its own
// producers, MMA issuer, softmax warpgroup and barriers, so the two slots
// drift apart: one slot's TMEM loads and maxima overlap the other's
// exponentials and MMAs.
//
// Step: list entries 2s (half g = 0) and 2s+1 (half g = 1) of the slot's
// query block.  QK^T is one M=64, N=128 chain.  Softmax thread (row r, half
// g) of warp w reads its row's 64 scores of half g with a 16-lane TMEM load
// (threads 0-15 the first half, 16-31 the second), trades block maxima with
// its partner by one shuffle, and owns TMEM accumulator O_g of its row: the
// frame of O_g is the running max after walk block 2s+g, so O_g is rescaled
// by exp(frame_old - frame_new) before PV_g.  PV is M=64, N=136: 128 V
// channels plus 8 rows of ones whose product is the row sum of P~.
//
// Warps (448 threads, 1 CTA/SM):
//   0, 1   K producers of slot 0 / 1: Q^ tile of each item (double-buffered),
//          K^ tiles of each step (2-stage ring), step metadata (tiles, key
//          scales) for the softmax (4-deep ring);
//   2, 3   V producers of slot 0 / 1 (V^T tiles, 2-stage ring);
//   4-7    softmax warpgroup of slot 0; 8-11 of slot 1 (TMEM lane quadrant
//          = warp % 4);
//   12, 13 MMA issuer of slot 0 / 1 (one thread: QK^T(s) then PV(s-1)).
// TMEM: S columns 0-127, O_0 128-263, O_1 272-407 (512 allocated).
// Every per-step barrier a role can run ahead on is double-buffered by step
// parity, and the softmax publishes nothing for step gs before the P~ buffer
// it writes is free (PV(gs-2) complete), so no parity wait is ever more than
// one phase behind its barrier.  Every wait is bounded (watchdog).
#include "common.cuh"
#include "kernels.h"

namespace sagesla {

namespace {

// Warp roles.  The softmax warps of a slot must cover TMEM lane quadrants
// 0-3 (warp % 4); the other roles are single threads.
enum Role { kIdle, kProdK, kProdV, kSoft, kMma };
constexpr int kWarps = 14;
constexpr int kThreads = 32 * kWarps;
__host__ __device__ constexpr int role_of(int w) {
  return w < 2 ? kProdK : w < 4 ? kProdV : w < 12 ? kSoft : w < 14 ? kMma : kIdle;
}
__host__ __device__ constexpr int slot_of(int w) {
  return w < 4 ? (w & 1) : w < 12 ? (w - 4) >> 2 : w < 14 ? w - 12 : 0;
}
constexpr int kWarpTmem = 12;  // allocates and frees TMEM (an MMA warp)
static_assert(role_of(kWarpTmem) == kMma, "TMEM owner");
constexpr uint32_t kOnesE4M3 = 0x38383838u;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;
constexpr float kRsqrtD = 0.08838834764831845f;  // 1/sqrt(128)
constexpr uint32_t kTmemCols = 512, kColS = 0, kColO0 = 128, kColO1 = 272;
constexpr uint32_t kP_LBO = 128, kP_SBO = 512;  // P~ tiles [64 rows][64 keys], K-major
constexpr int kNO = 136;                        // PV N: 128 channels + 8 ones
constexpr int kVSlot = kTile + (kNO - 128) * 64;  // V^T tile + 8 rows of ones

// Shared memory of one slot.
constexpr int kOffQ = 0;                      // 2 x 8 KB
constexpr int kOffK = kOffQ + 2 * kTile;      // 2 stages x 2 tiles
constexpr int kOffV = kOffK + 2 * 2 * kTile;  // 2 stages x 2 slots
constexpr int kOffP = kOffV + 2 * 2 * kVSlot; // [b][g] 4 KB each
constexpr int kOffM = kOffP + 4 * 4096;       // StepMeta[4]
constexpr int kSlotBytes = (kOffM + 4 * 16 + 1023) / 1024 * 1024;
constexpr int kOffBars = 2 * kSlotBytes;
constexpr int kSmem = kOffBars + 1024 + 1024;  // barriers + alignment slack

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
  int items;   // BH * nb query blocks
  int nsteps;  // steps per query block: ceil(kc / 2)
  int add_out; // 1: out already holds the linear branch (bf16); add O_s to it
  int q_tok;    // 1: one Q scale per token (sq [BH][nq*64])
  int H, tok;   // heads; out layout: 0 = [B][H][N][d], 1 = [B][N][H][d]
  long spin;    // probe limit of every bounded wait that may give up
  int stall_gs; // >= 0: slot 0's K producer omits the copy of this step (watchdog test)
};

// The K producer's hand-off to the softmax warps: the two key tiles of a
// step (list entries 2s and 2s+1; -1 when absent) and their INT8 key scales.
struct StepMeta {
  int tile[2];
  float sk[2];
};

struct SlotBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t m_full[4], m_empty[4];
  uint64_t s_full, s_free;
  uint64_t p_full[2], p_empty[2];
  uint64_t o_done;
  uint64_t fin;
};

struct Bars {
  SlotBars sl[2];
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

__device__ __forceinline__ int list_at(const Params& p, int bh, int i, int t) {
  return p.idx ? __ldg(p.idx + ((size_t)bh * p.nb + i) * p.kc + t) : t;
}

// Max of the first `nv` of 64 integer scores (four chains of 3-input maxima
// when all are valid).
__device__ __forceinline__ int max_valid64(const uint32_t* t, int nv) {
  if (nv >= 64) {
    int c4[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
    for (int c = 0; c < 64; c += 8) {
      c4[0] = __vimax3_s32(c4[0], (int)t[c], (int)t[c + 1]);
      c4[1] = __vimax3_s32(c4[1], (int)t[c + 2], (int)t[c + 3]);
      c4[2] = __vimax3_s32(c4[2], (int)t[c + 4], (int)t[c + 5]);
      c4[3] = __vimax3_s32(c4[3], (int)t[c + 6], (int)t[c + 7]);
    }
    return max(max(c4[0], c4[1]), max(c4[2], c4[3]));
  }
  int m = INT_MIN;
#pragma unroll
  for (int c = 0; c < 64; ++c)
    if (c < nv) m = max(m, (int)t[c]);
  return m;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) flash64_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBars);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nsteps = p.nsteps;
  const int stride = 2 * (int)gridDim.x;

  if (tid == 0) {
    for (int X = 0; X < 2; ++X) {
      SlotBars& B = bars->sl[X];
      for (int x = 0; x < 2; ++x) {
        mbar_init(&B.q_full[x], 1);
        mbar_init(&B.q_empty[x], 1);
        mbar_init(&B.k_full[x], 1);
        mbar_init(&B.k_empty[x], 1);
        mbar_init(&B.v_full[x], 1);
        mbar_init(&B.v_empty[x], 1);
        mbar_init(&B.p_full[x], 4);
        mbar_init(&B.p_empty[x], 1);
      }
      for (int x = 0; x < 4; ++x) {
        mbar_init(&B.m_full[x], 1);
        mbar_init(&B.m_empty[x], 4);
      }
      mbar_init(&B.s_full, 1);
      mbar_init(&B.s_free, 4);
      mbar_init(&B.o_done, 1);
      mbar_init(&B.fin, 1);
    }
    bars->abort = 0;
    mbar_fence_init();
  }
  // Rows of ones under every V^T slot of both slots' rings.
  constexpr int kOnesWords = (kVSlot - kTile) / 16;
  for (int e = tid; e < 2 * 4 * kOnesWords; e += kThreads) {
    const int X = e / (4 * kOnesWords), v = (e / kOnesWords) % 4, wv = e % kOnesWords;
    *reinterpret_cast<uint4*>(smem + X * kSlotBytes + kOffV + v * kVSlot + kTile + wv * 16) =
        make_uint4(kOnesE4M3, kOnesE4M3, kOnesE4M3, kOnesE4M3);
  }
  fence_proxy_async_smem();
  if (warp == kWarpTmem) tmem_alloc(&bars->tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  const int role = role_of(warp);
  if (role == kProdK || role == kProdV) {
    // ---------------------------- producers -------------------------------
    if (lane == 0) {
      const bool is_k = role == kProdK;
      const int X = slot_of(warp);
      SlotBars& B = bars->sl[X];
      uint8_t* sb = smem + X * kSlotBytes;
      StepMeta* meta = reinterpret_cast<StepMeta*>(sb + kOffM);
      uint64_t* full = is_k ? B.k_full : B.v_full;
      uint64_t* empty = is_k ? B.k_empty : B.v_empty;
      const uint8_t* src = is_k ? p.k8t : p.v8t;
      uint8_t* ring = sb + (is_k ? kOffK : kOffV);
      const int stage_bytes = is_k ? 2 * kTile : 2 * kVSlot;
      const int slot_bytes = is_k ? kTile : kVSlot;
      int gs = 0, ui = 0, skipped = -1, issued = 0;  // issued: steps whose copies are out
      bool ok = true;
      for (int q = 2 * (int)blockIdx.x + X; ok && q < p.items; q += stride, ++ui) {
        const int bh = q / p.nb, i = q - bh * p.nb;
        const size_t head_tiles = (size_t)bh * p.nq;
        if (is_k) {
          const int qb = ui & 1;
          if (ui >= 2 && !(ok = mbar_wait(&B.q_empty[qb], ((ui >> 1) - 1) & 1, abort, p.wd, p.spin))) break;
          mbar_expect_tx(&B.q_full[qb], kTile);
          bulk_g2s(sb + kOffQ + qb * kTile, p.q8t + (head_tiles + i) * kTile, kTile, &B.q_full[qb]);
        }
        for (int s = 0; s < nsteps; ++s, ++gs) {
          const int t0 = list_at(p, bh, i, 2 * s);
          const int t1 = 2 * s + 1 < p.kc ? list_at(p, bh, i, 2 * s + 1) : -1;
          const int st = gs & 1;
          if (gs >= 2 && !(ok = mbar_wait(&empty[st], ((gs >> 1) - 1) & 1, abort, p.wd, p.spin))) break;
          if (is_k && X == 0 && blockIdx.x == 0 && gs == p.stall_gs) {
            skipped = gs;  // this stage's barrier never completes: its waiter gives up
          } else {
            mbar_expect_tx(&full[st], (t1 >= 0 ? 2 : 1) * kTile);
            bulk_g2s(ring + st * stage_bytes, src + (head_tiles + t0) * kTile, kTile, &full[st]);
            if (t1 >= 0)
              bulk_g2s(ring + st * stage_bytes + slot_bytes, src + (head_tiles + t1) * kTile, kTile, &full[st]);
          }
          issued = gs + 1;
          if (is_k) {
            const float sk0 = __ldg(p.sk + head_tiles + t0);
            const float sk1 = t1 >= 0 ? __ldg(p.sk + head_tiles + t1) : 0.f;
            const int ms = gs & 3;
            if (gs >= 4 && !(ok = mbar_wait(&B.m_empty[ms], ((gs >> 2) - 1) & 1, abort, p.wd, p.spin))) break;
            meta[ms].tile[0] = t0;
            meta[ms].tile[1] = t1;
            meta[ms].sk[0] = sk0;
            meta[ms].sk[1] = sk1;
            mbar_arrive(&B.m_full[ms]);
          }
        }
      }
      // Drain: every copy issued must land before the CTA may exit.  The
      // empty-wait of step g proved the copies of step g-2 consumed, so only
      // the last two steps issued can still be in flight (also when a wait
      // gave up after the copies of its step were issued).
      for (int g2 = max(0, issued - 2); g2 < issued; ++g2)
        if (g2 != skipped) mbar_wait_drain(&full[g2 & 1], (g2 >> 1) & 1, p.wd);
      if (is_k)
        for (int u2 = max(0, ui - 2); u2 < ui; ++u2) mbar_wait_drain(&B.q_full[u2 & 1], (u2 >> 1) & 1, p.wd);
    }
  } else if (role == kMma) {
    // ------------------------------ MMA issuer ----------------------------
    // Per slot, in this order: QK^T(gs), then PV(gs-1).
    if (lane == 0) {
      const int X = slot_of(warp);
      SlotBars& B = bars->sl[X];
      uint8_t* sb = smem + X * kSlotBytes;
      const uint64_t dq = smem_desc(sb, kQK_LBO, kQK_SBO);
      const uint64_t dp = smem_desc(sb, kP_LBO, kP_SBO);
      const uint64_t dv = smem_desc(sb, kV_LBO, kV_SBO);
      const uint32_t lane_off = (uint32_t)(16 * X) << 16;
      const uint32_t id_pv = idesc_e4m3(64, kNO);
      int items_mine = 0;
      for (int q = 2 * (int)blockIdx.x + X; q < p.items; q += stride) ++items_mine;
      const int total = items_mine * nsteps;
      bool ok = true;
      for (int gs = 0; ok && gs <= total; ++gs) {
        if (gs < total) {
          const int ui = gs / nsteps, s = gs - ui * nsteps, qb = ui & 1, st = gs & 1;
          if (s == 0 && !(ok = mbar_wait(&B.q_full[qb], (ui >> 1) & 1, abort, p.wd, p.spin))) break;
          if (!(ok = mbar_wait(&B.k_full[st], (gs >> 1) & 1, abort, p.wd, p.spin))) break;
          if (gs > 0 && !(ok = mbar_wait(&B.s_free, (gs - 1) & 1, abort, p.wd, p.spin))) break;
          tc_fence_after();
          const uint32_t id = 2 * s + 1 < p.kc ? idesc_i8(64, 128) : idesc_i8(64, 64);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(tmem + kColS + lane_off, desc_at(dq, kOffQ + qb * kTile + kk * 256),
                   desc_at(dq, kOffK + st * 2 * kTile + kk * 256), id, kk > 0);
          mma_commit(&B.s_full);
          mma_commit(&B.k_empty[st]);
          if (s == nsteps - 1) mma_commit(&B.q_empty[qb]);
        }
        if (gs > 0) {
          const int gp = gs - 1, s = gp % nsteps, b = gp & 1, st = gp & 1;
          if (!(ok = mbar_wait(&B.v_full[st], (gp >> 1) & 1, abort, p.wd, p.spin))) break;
          if (!(ok = mbar_wait(&B.p_full[b], (gp >> 1) & 1, abort, p.wd, p.spin))) break;
          tc_fence_after();
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            if (g == 1 && 2 * s + 1 >= p.kc) break;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_e4m3(tmem + (g ? kColO1 : kColO0) + lane_off, desc_at(dp, kOffP + (2 * b + g) * 4096 + kk * 256),
                       desc_at(dv, kOffV + st * 2 * kVSlot + g * kVSlot + kk * 256), id_pv, (s > 0 || kk > 0));
          }
          mma_commit(&B.o_done);
          mma_commit(&B.p_empty[b]);
          mma_commit(&B.v_empty[st]);
        }
      }
      mma_commit(&B.fin);
    }
  } else if (role == kSoft) {
    // ------------------------------ softmax -------------------------------
    const int X = slot_of(warp);
    const int w = warp & 3;  // TMEM lane quadrant
    SlotBars& B = bars->sl[X];
    uint8_t* sb = smem + X * kSlotBytes;
    const StepMeta* meta = reinterpret_cast<const StepMeta*>(sb + kOffM);
    const int g = lane >> 4;                 // half: 0 = list entry 2s, 1 = 2s+1
    const int r = 16 * w + (lane & 15);      // row of the query block
    // 16-lane TMEM address of this thread's rows (lanes 32w + 16X + 0..15)
    const uint32_t tl = tmem + ((uint32_t)(32 * w + 16 * X) << 16);
    const bool has1 = p.kc >= 2;  // O_1 receives at least one block
    int gs = 0;
    bool ok = true;
    for (int q = 2 * (int)blockIdx.x + X; ok && q < p.items; q += stride) {
      const int bh = q / p.nb, i = q - bh * p.nb;
      const size_t sqi = (size_t)bh * p.nq + i;
      const float c0 = __ldg(p.sq + (p.q_tok ? sqi * kQB + r : sqi)) * (kLog2e * kRsqrtD);
      float m_all = -INFINITY, frame = -INFINITY;
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const int b = gs & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&B.m_full[gs & 3], (gs >> 2) & 1, abort, p.wd, p.spin));
        if (!ok) break;
        const StepMeta& mt = meta[gs & 3];
        const int t_own = mt.tile[g], t_oth = mt.tile[1 - g];
        const int nv_own = t_own >= 0 ? max(0, min(64, p.N - 64 * t_own)) : 0;
        const int nv_oth = t_oth >= 0 ? max(0, min(64, p.N - 64 * t_oth)) : 0;
        const float cu_own = c0 * mt.sk[g], cu_oth = c0 * mt.sk[1 - g];
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.m_empty[gs & 3]);
        // The P~ buffer b was read by PV(gs-2): wait for it before anything of
        // this step is published.
        if (gs >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(&B.p_empty[b], ((gs >> 1) - 1) & 1, abort, p.wd, p.spin));
          if (!ok) break;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&B.s_full, gs & 1, abort, p.wd, p.spin));
        if (!ok) break;
        tc_fence_after();
        uint32_t acc[64];
        SAGESLA_TMEM_LD2H_X64(tl + kColS, 64, acc);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.s_free);
        const int mx_own = max_valid64(acc, nv_own);
        const int mx_oth = __shfl_xor_sync(0xffffffffu, mx_own, 16);
        const float mf_own = nv_own > 0 ? __int2float_rn(mx_own) * cu_own : -INFINITY;
        const float mf_oth = nv_oth > 0 ? __int2float_rn(mx_oth) * cu_oth : -INFINITY;
        // Frame of O_g after this step: half 0 is walk block 2s (max over the
        // blocks so far and this one), half 1 is block 2s+1 (which has also
        // seen block 2s).
        float fnew = g == 0 ? fmaxf(m_all, mf_own) : fmaxf(m_all, fmaxf(mf_own, mf_oth));
        m_all = fmaxf(m_all, fmaxf(mf_own, mf_oth));
        if (nv_own == 0) fnew = frame;  // no block for this half: O_g keeps its frame
        const float alpha = (frame == -INFINITY || fnew == -INFINITY) ? 1.f : ex2(frame - fnew);
        frame = fnew;
        // P~ of the own half: exponent of 448*P = S*c - frame + log2(448), one
        // fused multiply-add per key on the converted integer score, two keys
        // per f32x2 instruction; keys past the sequence end get P~ = 0.
        if (nv_own > 0) {
          uint8_t* pbuf = sb + kOffP + (2 * b + g) * 4096;
          const float kk = kLog2_448 - frame;
          const uint64_t cc = f32x2_pack(cu_own, cu_own), ko = f32x2_pack(kk, kk);
          // 8-key chunks, software-pipelined: the conversions and FMAs of chunk
          // c+1 (I2F and FMA pipes) sit next to the exponentials of chunk c.
          float xc[8], xn[8];
          auto conv = [&](int ch, float (&x)[8]) {
#pragma unroll
            for (int z = 0; z < 8; z += 2) {
              const int c = 8 * ch + z;
              const uint64_t dd =
                  f32x2_fma(f32x2_pack(__int2float_rn((int)acc[c]), __int2float_rn((int)acc[c + 1])), cc, ko);
              f32x2_unpack(dd, x[z], x[z + 1]);
            }
          };
          conv(0, xc);
          uint32_t wv[4];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            if (ch < 7) conv(ch + 1, xn);
#pragma unroll
            for (int z = 0; z < 8; ++z) xc[z] = ex2(xc[z]);
            if (nv_own < 64) {
#pragma unroll
              for (int z = 0; z < 8; ++z)
                if (8 * ch + z >= nv_own) xc[z] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e)
              wv[2 * (ch & 1) + e] =
                  __byte_perm(e4m3x2(xc[4 * e], xc[4 * e + 1]), e4m3x2(xc[4 * e + 2], xc[4 * e + 3]), 0x5410);
            if (ch & 1)
              *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, 16 * (ch >> 1), kP_LBO, kP_SBO)) =
                  make_uint4(wv[0], wv[1], wv[2], wv[3]);
            if (ch < 7) {
#pragma unroll
              for (int z = 0; z < 8; ++z) xc[z] = xn[z];
            }
          }
        }
        // Rescale O_g of this row (channels and row-sum columns) once PV(gs-1)
        // is complete (s_full(gs) implied PV(gs-2) complete: all MMAs of the
        // issuing thread before QK(gs), so this wait is one phase ahead at most).  Threads 0-15 hold O_0 rows, 16-31 O_1 rows (column
        // split 144 = kColO1 - kColO0); alpha is 1 where nothing moved.
        if (s > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&B.o_done, (gs - 1) & 1, abort, p.wd, p.spin));
          if (!ok) break;
          tc_fence_after();
          const uint64_t a2 = f32x2_pack(alpha, alpha);
          // 144 columns in 16-column chunks; the load of chunk c+1 is in
          // flight while chunk c is multiplied and stored.
          uint32_t o[2][16];
          SAGESLA_TMEM_LD2H_X16(tl + kColO0, 144, o[0]);
          tmem_ld_wait();
#pragma unroll
          for (int ch = 0; ch < 9; ++ch) {
            uint32_t* cur = o[ch & 1];
            if (ch < 8) SAGESLA_TMEM_LD2H_X16(tl + kColO0 + 16 * (ch + 1), 144, o[(ch + 1) & 1]);
#pragma unroll
            for (int z = 0; z < 16; z += 2) {
              float a0, a1;
              f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(cur[z]), __uint_as_float(cur[z + 1])), a2), a0, a1);
              cur[z] = __float_as_uint(a0);
              cur[z + 1] = __float_as_uint(a1);
            }
            SAGESLA_TMEM_ST2H_X16(tl + kColO0 + 16 * ch, 144, cur);
            if (ch < 8) tmem_ld_wait();
          }
          tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.p_full[b]);
      }
      if (!ok) break;
      // ------------------------------ epilogue ----------------------------
      // out = (O_0 f_0 + O_1 f_1) / (l_0 f_0 + l_1 f_1) * s_v (+ the linear
      // branch already in out), f_g = exp(frame_g - max of both frames);
      // threads 0-15 write channels 0-63 of their row, 16-31 channels 64-127.
      // The last PV(gs-1) must be complete.  Here o_done may have completed
      // PV(gs-2), PV(gs-1), both or neither, which no single parity wait on it
      // can tell apart; p_empty of the step's parity completes only for
      // PV(gs-1) and PV(gs-3) (this warp waited for the latter in its last
      // step, and PV(gs+1) needs this warp's next P~), so its wait is exact.
      ok = __all_sync(0xffffffffu, mbar_wait(&B.p_empty[(gs - 1) & 1], ((gs - 1) >> 1) & 1, abort, p.wd, p.spin));
      if (!ok) break;
      tc_fence_after();
      const float fr_oth = __shfl_xor_sync(0xffffffffu, frame, 16);
      const float fr0 = g == 0 ? frame : fr_oth;
      const float fr1 = has1 ? (g == 1 ? frame : fr_oth) : -INFINITY;
      const float fm = fmaxf(fr0, fr1);
      const float f0 = fr0 == -INFINITY ? 0.f : ex2(fr0 - fm);
      const float f1 = fr1 == -INFINITY ? 0.f : ex2(fr1 - fm);
      uint32_t lt[1];
      SAGESLA_TMEM_LD2H_X1(tl + kColO0 + 128, 144, lt);
      tmem_ld_wait();
      const float l_own = __uint_as_float(lt[0]);
      const float l_oth = __shfl_xor_sync(0xffffffffu, l_own, 16);
      const float l0 = g == 0 ? l_own : l_oth;
      const float l1 = has1 ? (g == 1 ? l_own : l_oth) : 0.f;
      const float inv = 1.f / (l0 * f0 + l1 * f1);
      const float g0 = f0 * inv, g1 = f1 * inv;
      const int n = i * 64 + r;
      const bool store = n < p.N;
      __nv_bfloat16* orow = p.out + row_elems(p.tok, p.H, p.N, bh, store ? n : 0) + 64 * g;
      const float* svh = p.sv + (size_t)bh * kD + 64 * g;
#pragma unroll 1
      for (int c = 0; c < 64; c += 16) {
        uint32_t o0[16], o1[16];
        SAGESLA_TMEM_LD2H_X16(tl + kColO0 + c, 64, o0);
        if (has1) SAGESLA_TMEM_LD2H_X16(tl + kColO1 + c, 64, o1);
        uint4 y[2];
#pragma unroll
        for (int z = 0; z < 2; ++z)
          y[z] = (p.add_out && store) ? *reinterpret_cast<const uint4*>(orow + c + 8 * z) : make_uint4(0, 0, 0, 0);
        tmem_ld_wait();
        if (store) {
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const uint32_t yv[4] = {y[z].x, y[z].y, y[z].z, y[z].w};
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int cc = 8 * z + 2 * e;
              float a = __uint_as_float(o0[cc]) * g0, bb = __uint_as_float(o0[cc + 1]) * g0;
              if (has1) {
                a = fmaf(__uint_as_float(o1[cc]), g1, a);
                bb = fmaf(__uint_as_float(o1[cc + 1]), g1, bb);
              }
              a = fmaf(a, __ldg(svh + c + cc), bf16_lo(yv[e]));
              bb = fmaf(bb, __ldg(svh + c + cc + 1), bf16_hi(yv[e]));
              const __nv_bfloat162 h = __floats2bfloat162_rn(a, bb);
              pk[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(orow + c + 8 * z) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      tc_fence_before();
    }
  }
  // Every MMA of both slots has completed once both `fin` barriers have fired.
  if (warp == kWarpTmem) {
    if (lane == 0) {
      mbar_wait_drain(&bars->sl[0].fin, 0, p.wd);
      mbar_wait_drain(&bars->sl[1].fin, 0, p.wd);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpTmem) tmem_dealloc(tmem, kTmemCols);
}

cudaError_t launch_flash128(const FlashArgs& a, const Geom& g, cudaStream_t st, int* wd);

cudaError_t launch_flash(const FlashArgs& a, const Geom& g, cudaStream_t st, int* wd) {
  if (g.block != 64) return launch_flash128(a, g, st, wd);
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
  p.q_tok = a.q_tok;
  p.H = g.H;
  p.tok = g.tok;
  p.items = g.BH * g.nb;
  p.nsteps = (g.kc + 1) / 2;
  p.spin = a.dbg_spin > 0 ? a.dbg_spin : kSpinLimit;
  p.stall_gs = a.dbg_stall - 1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int want = (p.items + 1) / 2;
  int grid = want < sms ? want : sms;
  if (a.dbg_grid > 0 && a.dbg_grid < grid) grid = a.dbg_grid;
  cudaError_t e = cudaFuncSetAttribute(flash64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  flash64_kernel<<<grid, kThreads, kSmem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sagesla
