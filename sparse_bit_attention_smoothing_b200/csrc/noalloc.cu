// noalloc.cu -- the smoothing statistics of the path through an entry point
// that allocates no device memory.
//
// Who needs it: callers that must not allocate device memory once they are
// running -- a serving process that reserves its whole memory budget at
// start-up and refuses later growth, or code that runs where an allocation
// would stall or fail (inside a custom allocator's hooks, under a pool that
// is already at its limit).  The regular entry points allocate their
// workspace on first use; this one keeps its scratch in a fixed array of
// device memory that is part of the library image instead.
//
// Scratch: one file-scope array of kNoAllocScratchBytes (4 MiB).  Every GPU
// that loads the library holds it until the process exits.  All calls share
// it, so calls whose work overlaps on the GPU (different streams, or
// different host threads on the same device) race on it; the caller must
// serialise them.  Each call writes every scratch word it later reads, so
// nothing has to start at zero.
//
// The rows of each head are split exactly as in the regular path (one split
// per 1024 tokens), so the fp64 partial sums of the K mean are added in the
// same order and mu comes out with the same bits.  When the partial sums of
// all heads do not fit the scratch, the heads are processed in chunks, one
// after another on the stream; only a single head whose partial sums exceed
// the scratch (N above about 2.8 million tokens) is refused.
#include <algorithm>
#include <cstdint>
#include <map>
#include <mutex>

#include "../../include/sagesla.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
// Per (b,h): split x 128 fp64 partial sums, split x 128 fp32 partial maxima,
// plus 128 fp32 multipliers (448/amax) that the statistics pass also writes.
constexpr size_t kPerSplitBytes = sagesla::kD * (sizeof(double) + sizeof(float));
constexpr size_t kPerHeadBytes = sagesla::kD * sizeof(float);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
std::map<int, unsigned char*> g_scratch_addr;  // device -> device address of the array

// The array's name in host code is only a stand-in; its device address is
// looked up once per device, with that device current.
int scratch_address(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_scratch_addr.find(dev);
  if (it == g_scratch_addr.end()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SAGESLA_ERR_LAUNCH;
    }
    it = g_scratch_addr.emplace(dev, static_cast<unsigned char*>(p)).first;
  }
  *out = it->second;
  return SAGESLA_OK;
}

}  // namespace

extern "C" int sagesla_smooth_stats_noalloc(const void* k, const void* v, int B, int H, int N, int d, float* mu,
                                            float* sv, sagesla_stream_t stream) {
  if (!k || !v || !mu || !sv) return SAGESLA_ERR_INVALID;
  if (B < 1 || H < 1 || N < 1 || d != sagesla::kD) return SAGESLA_ERR_INVALID;
  const long long BH = (long long)B * H;
  if (BH > 65535 || (double)BH * N * d >= 1099511627776.0) return SAGESLA_ERR_INVALID;
  const int split = (N + 1023) / 1024;
  const size_t per_head = (size_t)split * kPerSplitBytes + kPerHeadBytes;
  if (per_head > kNoAllocScratchBytes) return SAGESLA_ERR_INVALID;
  const int chunk = (int)std::min<long long>(BH, (long long)(kNoAllocScratchBytes / per_head));
  if ((reinterpret_cast<uintptr_t>(k) & 15u) || (reinterpret_cast<uintptr_t>(v) & 15u) ||
      (reinterpret_cast<uintptr_t>(mu) & 3u) || (reinterpret_cast<uintptr_t>(sv) & 3u))
    return SAGESLA_ERR_MISALIGNED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGESLA_ERR_NO_DEVICE;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return SAGESLA_ERR_NO_DEVICE;
  unsigned char* scratch = nullptr;
  const int rc = scratch_address(dev, &scratch);
  if (rc != SAGESLA_OK) return rc;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t head_elems = (size_t)N * d;
  for (long long h0 = 0; h0 < BH; h0 += chunk) {
    const int nh = (int)std::min<long long>(chunk, BH - h0);
    sagesla::Geom g{};
    g.BH = nh;
    g.N = N;
    g.block = 64;
    g.nb = (N + 63) / 64;
    g.nq = 2 * ((N + 127) / 128);
    g.kc = g.nb;
    g.split = split;
    double* psum = reinterpret_cast<double*>(scratch);
    float* pmax = reinterpret_cast<float*>(scratch + (size_t)nh * split * sagesla::kD * sizeof(double));
    float* mv = reinterpret_cast<float*>(scratch + (size_t)nh * split * kPerSplitBytes);
    const uint16_t* kh = static_cast<const uint16_t*>(k) + h0 * head_elems;
    const uint16_t* vh = static_cast<const uint16_t*>(v) + h0 * head_elems;
    if (sagesla::launch_stats_partial(kh, vh, g, psum, pmax, st) != cudaSuccess) return SAGESLA_ERR_LAUNCH;
    if (sagesla::launch_stats_final(psum, pmax, g, mu + h0 * sagesla::kD, sv + h0 * sagesla::kD, mv, st) !=
        cudaSuccess)
      return SAGESLA_ERR_LAUNCH;
  }
  return SAGESLA_OK;
}
