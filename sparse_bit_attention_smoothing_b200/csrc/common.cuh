// common.cuh -- small PTX wrappers for sm_100a (mbarrier, bulk copy, tcgen05)
// and layout helpers shared by the SageSLA kernels.
//
// Operand tiles in shared memory use the canonical "no swizzle" K-major
// layout of the 5th-generation tensor cores: 8-row x 16-byte core matrices
// stored as 128 contiguous bytes; LBO = byte distance between core matrices
// adjacent along K, SBO = byte distance between core matrices adjacent along
// M/N.  The global copies of Q^, K^ and V^T are written in exactly this
// layout, so one bulk copy moves a whole tile.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace sagesla {

constexpr int kD = 128;        // head dimension supported
constexpr int kQB = 64;        // quantisation block of Q and K (tokens)
constexpr int kTile = kQB * kD;  // bytes of one 8-bit 64 x 128 tile (8192)
// Q^ / K^ tile [64 rows][128 bytes]: LBO 128 (K chunks adjacent), SBO 1024.
constexpr uint32_t kQK_LBO = 128, kQK_SBO = 1024;
// V^T tile [128 channels][64 keys]: LBO 128, SBO 512 (4 K chunks per row group).
constexpr uint32_t kV_LBO = 128, kV_SBO = 512;

// Byte offset of element (row r, byte column c) in a K-major no-swizzle tile.
__host__ __device__ __forceinline__ uint32_t kmajor_off(uint32_t r, uint32_t c, uint32_t lbo, uint32_t sbo) {
  return (r >> 3) * sbo + (c >> 4) * lbo + (r & 7) * 16 + (c & 15);
}

// Watchdog: every device-side wait is bounded; on expiry the kernel records
// the failure in a device word of the workspace (`wd`) and returns.  The
// host reads and clears it in sagesla_sync_status().
constexpr long kSpinLimit = 1L << 24;  // try_wait probes (each may suspend briefly)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------ mbarrier ---------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of a phase (cheap when it has already completed).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait of at most `limit` probes.  Returns false if it gave up: then
// it raises `abort` (a CTA-shared flag, so that every role of the CTA stops)
// and the global watchdog word `wd`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* wd,
                                          long limit = kSpinLimit) {
  if (mbar_test(bar, parity)) return true;
  for (long i = 0; i < limit; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 255) == 255 && *abort) return false;
  }
  *abort = 1;
  atomicExch(wd, 1);
  return false;
}

// Bounded wait that ignores the abort flag: used to drain work that always
// completes on its own (issued copies, issued MMAs) before the CTA exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, int* wd) {
  if (mbar_test(bar, parity)) return true;
  for (long i = 0; i < kSpinLimit; ++i)
    if (mbar_try(bar, parity)) return true;
  atomicExch(wd, 1);
  return false;
}

// --------------------------- input layouts --------------------------------
// Element offset of row (head bh = b*H + h, token n) of a bf16 tensor in the
// [B][H][N][128] layout (tok = 0) or the token-major [B][N][H][128] layout
// (tok = 1) in which a DiT's attention projections emit q, k and v.
__host__ __device__ __forceinline__ size_t row_elems(int tok, int H, int N, int bh, int n) {
  return tok ? (((size_t)(bh / H) * N + n) * H + bh % H) * kD : ((size_t)bh * N + n) * kD;
}

// ------------------------------ QK RMSNorm --------------------------------
// The DiT's RMSNorm of q and k, applied where the path loads them: per token,
// x / sqrt(mean over its H*d channels of x^2 + eps) * gamma, rounded to bf16
// (the per-token factor inv comes from rms_inv_kernel; see QKNorm).
__device__ __forceinline__ uint32_t rms_bf16x2(uint32_t w, float inv, uint32_t gw) {
  const float a = __fmul_rn(__fmul_rn(__uint_as_float(w << 16), inv), __uint_as_float(gw << 16));
  const float b = __fmul_rn(__fmul_rn(__uint_as_float(w & 0xFFFF0000u), inv), __uint_as_float(gw & 0xFFFF0000u));
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// Eight bf16 channels of one row: x * inv * gamma.
__device__ __forceinline__ uint4 rms_row8(uint4 x, float inv, uint4 g) {
  return make_uint4(rms_bf16x2(x.x, inv, g.x), rms_bf16x2(x.y, inv, g.y), rms_bf16x2(x.z, inv, g.z),
                    rms_bf16x2(x.w, inv, g.w));
}

// --------------------------- bulk async copy -----------------------------
// Global -> shared, completion counted in bytes on `bar`.  Both addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------- tcgen05 ---------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor, no swizzle (layout type 0), version 1.
__device__ __forceinline__ uint64_t smem_desc(const void* p, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((smem_u32(p) >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}
// Descriptor of smem offset `off` from a base descriptor (the start-address
// field holds address >> 4 in 14 bits; shared memory is < 256 KB, so adding
// off >> 4 to the low word never carries out of the field).
__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t off) { return base + (uint64_t)(off >> 4); }
// Instruction descriptors.  kind::i8 s8 x s8 -> s32; kind::f8f6f4 e4m3 x e4m3
// -> f32; kind::f16 bf16 x bf16 -> f32.  Both operands K-major unless b_mn.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn = 0) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_e4m3(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// TMEM -> registers: 32 lanes x 32-bit, N consecutive columns per thread.
#define SAGESLA_TMEM_LD16(taddr, r)                                                                               \
  asm volatile(                                                                                                   \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"    \
      : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]),         \
        "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]),     \
        "=r"((r)[14]), "=r"((r)[15])                                                                              \
      : "r"(taddr))
#define SAGESLA_TMEM_ST16(taddr, r)                                                                               \
  asm volatile(                                                                                                   \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"    \
      ::"r"(taddr), "r"((r)[0]), "r"((r)[1]), "r"((r)[2]), "r"((r)[3]), "r"((r)[4]), "r"((r)[5]), "r"((r)[6]),   \
      "r"((r)[7]), "r"((r)[8]), "r"((r)[9]), "r"((r)[10]), "r"((r)[11]), "r"((r)[12]), "r"((r)[13]),             \
      "r"((r)[14]), "r"((r)[15]))

// 32 lanes x 32 consecutive columns (one register per column per thread).
#define SAGESLA_TMEM_LD32(taddr, r) \
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];" \
               : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7]), \
                 "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]), "=r"((r)[14]), "=r"((r)[15]), \
                 "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]), "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), \
                 "=r"((r)[24]), "=r"((r)[25]), "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31]) \
               : "r"(taddr))

// 16-lane TMEM access, two halves of a warp: threads 0-15 read/write lanes
// (taddr.lane + t) at columns [taddr.col, taddr.col + n), threads 16-31 the
// same lanes at columns [taddr.col + split, taddr.col + split + n).
#define SAGESLA_TMEM_LD2H_X1(taddr, split, r)                                   \
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x1.b32 {%0}, [%1], " #split ";" \
               : "=r"((r)[0])                                                        \
               : "r"(taddr))
#define SAGESLA_TMEM_LD2H_X8(taddr, split, r)                                   \
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], " #split ";" \
               : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7])                                                        \
               : "r"(taddr))
#define SAGESLA_TMEM_ST2H_X8(taddr, split, r)                                   \
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], " #split ", {%1,%2,%3,%4,%5,%6,%7,%8};" \
               ::"r"(taddr), "r"((r)[0]), "r"((r)[1]), "r"((r)[2]), "r"((r)[3]), "r"((r)[4]), "r"((r)[5]), "r"((r)[6]), "r"((r)[7]))
#define SAGESLA_TMEM_LD2H_X16(taddr, split, r)                                   \
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], " #split ";" \
               : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]), "=r"((r)[14]), "=r"((r)[15])                                                        \
               : "r"(taddr))
#define SAGESLA_TMEM_LD2H_X32(taddr, split, r)                                   \
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], " #split ";" \
               : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]), "=r"((r)[14]), "=r"((r)[15]), "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]), "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), "=r"((r)[24]), "=r"((r)[25]), "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31])                                                        \
               : "r"(taddr))
#define SAGESLA_TMEM_LD2H_X64(taddr, split, r)                                   \
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64], " #split ";" \
               : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]), "=r"((r)[14]), "=r"((r)[15]), "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]), "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), "=r"((r)[24]), "=r"((r)[25]), "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31]), "=r"((r)[32]), "=r"((r)[33]), "=r"((r)[34]), "=r"((r)[35]), "=r"((r)[36]), "=r"((r)[37]), "=r"((r)[38]), "=r"((r)[39]), "=r"((r)[40]), "=r"((r)[41]), "=r"((r)[42]), "=r"((r)[43]), "=r"((r)[44]), "=r"((r)[45]), "=r"((r)[46]), "=r"((r)[47]), "=r"((r)[48]), "=r"((r)[49]), "=r"((r)[50]), "=r"((r)[51]), "=r"((r)[52]), "=r"((r)[53]), "=r"((r)[54]), "=r"((r)[55]), "=r"((r)[56]), "=r"((r)[57]), "=r"((r)[58]), "=r"((r)[59]), "=r"((r)[60]), "=r"((r)[61]), "=r"((r)[62]), "=r"((r)[63])                                                        \
               : "r"(taddr))
#define SAGESLA_TMEM_ST2H_X16(taddr, split, r)                                   \
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], " #split ", {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
               ::"r"(taddr), "r"((r)[0]), "r"((r)[1]), "r"((r)[2]), "r"((r)[3]), "r"((r)[4]), "r"((r)[5]), "r"((r)[6]), "r"((r)[7]), "r"((r)[8]), "r"((r)[9]), "r"((r)[10]), "r"((r)[11]), "r"((r)[12]), "r"((r)[13]), "r"((r)[14]), "r"((r)[15]))
#define SAGESLA_TMEM_ST2H_X32(taddr, split, r)                                   \
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], " #split ", {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" \
               ::"r"(taddr), "r"((r)[0]), "r"((r)[1]), "r"((r)[2]), "r"((r)[3]), "r"((r)[4]), "r"((r)[5]), "r"((r)[6]), "r"((r)[7]), "r"((r)[8]), "r"((r)[9]), "r"((r)[10]), "r"((r)[11]), "r"((r)[12]), "r"((r)[13]), "r"((r)[14]), "r"((r)[15]), "r"((r)[16]), "r"((r)[17]), "r"((r)[18]), "r"((r)[19]), "r"((r)[20]), "r"((r)[21]), "r"((r)[22]), "r"((r)[23]), "r"((r)[24]), "r"((r)[25]), "r"((r)[26]), "r"((r)[27]), "r"((r)[28]), "r"((r)[29]), "r"((r)[30]), "r"((r)[31]))
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// --------------------------- small numerics ------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// Two floats -> packed e4m3 pair (round to nearest even, saturate to +-448);
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction, two lanes
// of work, each rounded to nearest like its scalar form).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

}  // namespace sagesla
