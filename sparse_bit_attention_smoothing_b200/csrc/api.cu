// api.cu -- the C ABI of include/sagesla.h: argument checks, the workspace
// cache and the launch sequence of the SageSLA path.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/sagesla.h"
#include "common.cuh"
#include "kernels.h"

namespace sagesla {
size_t pool_topk_smem(int nb);
}

using namespace sagesla;

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_mu;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;     // path workspace
std::map<std::pair<int, cudaStream_t>, Workspace> g_stage;  // host entry point's device staging
std::map<int, int*> g_wd;        // per-device watchdog word
std::map<int, int> g_dev_ok;     // per-device: 1 = sm_100, 0 = not

int check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGESLA_ERR_NO_DEVICE;
  *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_dev_ok.find(dev);
  if (it == g_dev_ok.end()) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : 0;
    it = g_dev_ok.find(dev);
  }
  if (!it->second) return SAGESLA_ERR_NO_DEVICE;
  if (!g_wd.count(dev)) {
    int* wd = nullptr;
    if (cudaMalloc(&wd, sizeof(int)) != cudaSuccess) return SAGESLA_ERR_OOM;
    if (cudaMemset(wd, 0, sizeof(int)) != cudaSuccess) return SAGESLA_ERR_LAUNCH;
    g_wd[dev] = wd;
  }
  return SAGESLA_OK;
}

int* watchdog(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_wd[dev];
}

// Stream-ordered workspace of at least `bytes`, cached per (device, stream).
int get_workspace(int dev, cudaStream_t st, size_t bytes, uint8_t** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[std::make_pair(dev, st)];
  if (w.bytes < bytes) {
    if (w.ptr) cudaFreeAsync(w.ptr, st);
    w.ptr = nullptr;
    w.bytes = 0;
    if (cudaMallocAsync(&w.ptr, bytes, st) != cudaSuccess) {
      cudaGetLastError();
      return SAGESLA_ERR_OOM;
    }
    w.bytes = bytes;
  }
  *out = static_cast<uint8_t*>(w.ptr);
  return SAGESLA_OK;
}

// ------------------------------------------------------------------ profiler
// When enabled, every kernel launch is bracketed by two CUDA events recorded
// on the launching stream; sagesla_profile_read() sums the durations per
// kernel.  Events come from a pool and are reused.
struct ProfRec {
  int kernel;
  cudaEvent_t a, b;
};
std::mutex g_pmu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_evpool;

cudaEvent_t ev_get() {
  if (!g_evpool.empty()) {
    cudaEvent_t e = g_evpool.back();
    g_evpool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct ProfScope {
  int kernel;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  ProfScope(int k, cudaStream_t s) : kernel(k), st(s) {
    std::lock_guard<std::mutex> lk(g_pmu);
    if (g_prof_on) {
      a = ev_get();
      cudaEventRecord(a, st);
    }
  }
  ~ProfScope() {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_pmu);
    cudaEvent_t b = ev_get();
    cudaEventRecord(b, st);
    g_prof.push_back({kernel, a, b});
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate(const void* q, const void* k, const void* v, const void* out, int B, int H, int N, int d, int block,
             float topk) {
  if (!q || !k || !v || !out) return SAGESLA_ERR_INVALID;
  if (B < 1 || H < 1 || N < 1 || d != kD) return SAGESLA_ERR_INVALID;
  if (block != 64 && block != 128) return SAGESLA_ERR_INVALID;
  if (!(topk > 0.f) || !(topk <= 1.f)) return SAGESLA_ERR_INVALID;  // rejects NaN
  const long long BH = (long long)B * H;
  if (BH > 65535) return SAGESLA_ERR_INVALID;
  if ((double)BH * N * d >= 1099511627776.0) return SAGESLA_ERR_INVALID;
  const int nb = (N + block - 1) / block;
  if (sagesla::pool_topk_smem(nb) > 227 * 1024) return SAGESLA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SAGESLA_ERR_MISALIGNED;
  return SAGESLA_OK;
}

Geom make_geom(int B, int H, int N, int block, float topk) {
  Geom g;
  g.BH = B * H;
  g.N = N;
  g.block = block;
  g.nb = (N + block - 1) / block;
  g.nq = 2 * ((N + 127) / 128);
  g.kc = sagesla_topk_count(g.nb, topk);
  // Row splits of the statistics pass: one per 1024 tokens.  The split
  // depends on N alone, so the fp64 partial sums of the K mean are added in
  // the same order whatever B*H a call covers (the host entry point's chunks
  // of heads give the same bits as one call over all heads).
  g.split = (N + 1023) / 1024;
  g.H = H;
  g.tok = 0;
  return g;
}

// Carve the workspace.  Every region 256-byte aligned.
struct Buffers {
  double* psum;
  float *pmax, *mu, *sv, *mv;
  uint8_t *q8t, *k8t, *v8t;
  float *sq, *sk, *qsum, *ksum;
  int32_t* idx;
  float *qbar, *kbar;  // pooled means [BH][nb][128]
  float *inv_q, *inv_k;  // QK RMSNorm: per-token 1 / rms [B][N]
  // linear branch
  uint8_t* hs;        // mask-GEMM B tiles of h_j (bf16)
  float* z;           // z_j [BH][nb][128]
  uint32_t* selbits;  // [BH][nb][2*nbt]
  float* zl;          // Z_i [BH][nb][128]
  float* ztot;        // sum of z_j over all j [BH][128]
  uint16_t* himg;     // H_i^T images [BH][nb][128*128]
  uint16_t* wimg;     // proj_w image
  size_t total;
};

Buffers carve(uint8_t* base, const Geom& g, bool linear = false, bool q_tok = false, int norm_B = 0) {
  Buffers b;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + o : nullptr;
    o += up(bytes);
    return p;
  };
  const size_t BH = (size_t)g.BH;
  b.psum = reinterpret_cast<double*>(take(BH * g.split * kD * sizeof(double)));
  b.pmax = reinterpret_cast<float*>(take(BH * g.split * kD * sizeof(float)));
  b.mu = reinterpret_cast<float*>(take(BH * kD * sizeof(float)));
  b.sv = reinterpret_cast<float*>(take(BH * kD * sizeof(float)));
  b.mv = reinterpret_cast<float*>(take(BH * kD * sizeof(float)));
  b.q8t = take(BH * g.nq * kTile);
  b.k8t = take(BH * g.nq * kTile);
  b.v8t = take(BH * g.nq * kTile);
  b.sq = reinterpret_cast<float*>(take(BH * g.nq * (q_tok ? kQB : 1) * sizeof(float)));
  b.sk = reinterpret_cast<float*>(take(BH * g.nq * sizeof(float)));
  b.qsum = reinterpret_cast<float*>(take(BH * g.nq * kD * sizeof(float)));
  b.ksum = reinterpret_cast<float*>(take(BH * g.nq * kD * sizeof(float)));
  b.idx = reinterpret_cast<int32_t*>(take(BH * g.nb * (size_t)g.kc * sizeof(int32_t)));
  b.qbar = reinterpret_cast<float*>(take(BH * g.nb * kD * sizeof(float)));
  b.kbar = reinterpret_cast<float*>(take(BH * g.nb * kD * sizeof(float)));
  b.inv_q = norm_B ? reinterpret_cast<float*>(take((size_t)norm_B * g.N * sizeof(float))) : nullptr;
  b.inv_k = norm_B ? reinterpret_cast<float*>(take((size_t)norm_B * g.N * sizeof(float))) : nullptr;
  if (linear) {
    const size_t nbt = (size_t)(g.nb + 63) / 64;
    b.hs = take(BH * nbt * 64 * 16384 * 2);
    b.z = reinterpret_cast<float*>(take(BH * g.nb * kD * sizeof(float)));
    b.selbits = reinterpret_cast<uint32_t*>(take(BH * g.nb * 2 * nbt * sizeof(uint32_t)));
    b.zl = reinterpret_cast<float*>(take(BH * g.nb * kD * sizeof(float)));
    b.ztot = reinterpret_cast<float*>(take(BH * kD * sizeof(float)));
    b.himg = reinterpret_cast<uint16_t*>(take(BH * g.nb * 16384 * sizeof(uint16_t)));
    b.wimg = reinterpret_cast<uint16_t*>(take(16384 * sizeof(uint16_t)));
  } else {
    b.hs = nullptr;
    b.z = b.zl = b.ztot = nullptr;
    b.selbits = nullptr;
    b.himg = b.wimg = nullptr;
  }
  b.total = o;
  return b;
}

inline int launch_rc(cudaError_t e) { return e == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_LAUNCH; }

#define SAGESLA_TRY(x)          \
  do {                          \
    int rc_ = (x);              \
    if (rc_ != SAGESLA_OK) return rc_; \
  } while (0)

// Stats + quantisation (the front shared by every entry point).
// QK RMSNorm inputs of the path (gq == nullptr: off).
struct NormIn {
  const void* gq = nullptr;
  const void* gk = nullptr;
  double eps = 0.0;
  int B = 0, H = 0;
};

QKNorm qk_norm(const float* inv, const void* gamma, const NormIn* n, const Geom& g) {
  QKNorm r;
  if (n && n->gq) {
    r.inv = inv;
    r.gamma = static_cast<const uint4*>(gamma);
    r.H = n->H;
    r.N = g.N;
  }
  return r;
}

int run_front(const void* q, const void* k, const void* v, const Geom& g, const Buffers& b, int dev,
              cudaStream_t st, int qmax = 127, int q_tok = 0, const NormIn* nrm = nullptr) {
  if (nrm && nrm->gq) {
    ProfScope ps(11, st);
    SAGESLA_TRY(launch_rc(launch_rms_inv(q, k, nrm->B, nrm->H, g.N, nrm->eps, b.inv_q, b.inv_k, st, g.tok)));
  }
  const QKNorm nq = qk_norm(b.inv_q, nrm ? nrm->gq : nullptr, nrm, g);
  const QKNorm nk = qk_norm(b.inv_k, nrm ? nrm->gk : nullptr, nrm, g);
  {
    ProfScope ps(0, st);
    SAGESLA_TRY(launch_rc(launch_stats_partial(k, v, g, b.psum, b.pmax, st, nk)));
  }
  {
    ProfScope ps(1, st);
    SAGESLA_TRY(launch_rc(launch_stats_final(b.psum, b.pmax, g, b.mu, b.sv, b.mv, st)));
  }
  {
    ProfScope ps(2, st);
    SAGESLA_TRY(launch_rc(
        launch_quant(q, k, v, b.mu, b.mv, g, b.q8t, b.k8t, b.v8t, b.sq, b.sk, b.qsum, b.ksum, watchdog(dev), st,
                     qmax, q_tok, nq, nk)));
  }
  return SAGESLA_OK;
}

int run_attn(const void* q, const void* k, const void* v, const void* proj_w, void* out, int B, int H, int N, int d,
             int block, float topk, cudaStream_t st, int dbg_grid = 0, int dbg_stall = 0, long dbg_spin = 0,
             int qmax = 127, int q_tok = 0, const NormIn* nrm = nullptr, int tok = 0) {
  SAGESLA_TRY(validate(q, k, v, out, B, H, N, d, block, topk));
  if (proj_w && !aligned16(proj_w)) return SAGESLA_ERR_MISALIGNED;
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  Geom g = make_geom(B, H, N, block, topk);
  g.tok = tok;
  const bool dense = g.kc == g.nb;
  // An empty complement (every key block selected) makes the linear branch 0.
  const bool linear = proj_w != nullptr && !dense;
  const int norm_B = (nrm && nrm->gq) ? B : 0;
  const Buffers sizes = carve(nullptr, g, linear, q_tok != 0, norm_B);
  uint8_t* base = nullptr;
  SAGESLA_TRY(get_workspace(dev, st, sizes.total, &base));
  const Buffers b = carve(base, g, linear, q_tok != 0, norm_B);
  SAGESLA_TRY(run_front(q, k, v, g, b, dev, st, qmax, q_tok, nrm));
  const QKNorm nq = qk_norm(b.inv_q, nrm ? nrm->gq : nullptr, nrm, g);
  const QKNorm nk = qk_norm(b.inv_k, nrm ? nrm->gk : nullptr, nrm, g);
  int* wd = watchdog(dev);
  if (linear) {
    {
      ProfScope ps(7, st);
      SAGESLA_TRY(launch_rc(launch_w_tile(proj_w, b.wimg, st)));
    }
    ProfScope ps(4, st);
    SAGESLA_TRY(launch_rc(launch_linear_kv(k, v, g, b.hs, b.z, wd, st, nk)));
  }
  if (!dense) {
    ProfScope ps(3, st);
    SAGESLA_TRY(launch_rc(launch_pool_topk(b.qsum, b.ksum, g, b.idx, b.qbar, b.kbar, linear ? b.z : nullptr,
                                           b.ztot, b.selbits, b.zl, st)));
  }
  if (linear) {
    {
      ProfScope ps(5, st);
      SAGESLA_TRY(launch_rc(launch_linear_sum(b.hs, b.selbits, g, b.himg, wd, st)));
    }
    ProfScope ps(8, st);
    SAGESLA_TRY(launch_rc(launch_linear_apply(q, b.himg, b.zl, b.wimg, g, out, wd, st, nq)));
  }
  FlashArgs fa;
  std::memset(&fa, 0, sizeof(fa));
  fa.q8t = b.q8t;
  fa.k8t = b.k8t;
  fa.v8t = b.v8t;
  fa.sq = b.sq;
  fa.sk = b.sk;
  fa.sv = b.sv;
  fa.idx = dense ? nullptr : b.idx;
  fa.out = out;
  fa.add_out = linear ? 1 : 0;
  fa.q_tok = q_tok;
  fa.dbg_grid = dbg_grid;
  fa.dbg_stall = dbg_stall;
  fa.dbg_spin = dbg_spin;
  {
    ProfScope ps(6, st);
    SAGESLA_TRY(launch_rc(launch_flash(fa, g, st, wd)));
  }
  return SAGESLA_OK;
}

int check_gemm(const void* xq, const float* sx, const void* wq, const float* sw, const void* y, int M, int N, int K) {
  if (!xq || !sx || !wq || !sw || !y || M < 1 || N < 128 || K < 128 || N % 128 != 0 || K % 128 != 0 ||
      M > 8388480 || (double)M * N >= 1099511627776.0 || (double)M * K >= 1099511627776.0)
    return SAGESLA_ERR_INVALID;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(y) || (reinterpret_cast<uintptr_t>(sx) & 3u) ||
      (reinterpret_cast<uintptr_t>(sw) & 3u))
    return SAGESLA_ERR_MISALIGNED;
  return SAGESLA_OK;
}

}  // namespace

extern "C" {

int sagesla_topk_count(int nb, float topk) {
  double t = (double)topk * (double)nb;
  t -= t * 1e-6;
  int k = (int)std::ceil(t);
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return k;
}

int sagesla_attn(const void* q, const void* k, const void* v, const void* proj_w, void* out, int B, int H, int N,
                 int d, int block, float topk, sagesla_stream_t stream) {
  return run_attn(q, k, v, proj_w, out, B, H, N, d, block, topk, reinterpret_cast<cudaStream_t>(stream));
}

int sagesla_attn_opts(const void* q, const void* k, const void* v, const void* proj_w, void* out, int B, int H,
                      int N, int d, int block, float topk, int qk_bits, int q_per_token, sagesla_stream_t stream) {
  if ((qk_bits != 8 && qk_bits != 4) || (q_per_token != 0 && q_per_token != 1)) return SAGESLA_ERR_INVALID;
  return run_attn(q, k, v, proj_w, out, B, H, N, d, block, topk, reinterpret_cast<cudaStream_t>(stream), 0, 0, 0,
                  qk_bits == 8 ? 127 : 7, q_per_token);
}

int sagesla_attn_qknorm(const void* q, const void* k, const void* v, const void* gamma_q, const void* gamma_k,
                        float eps, const void* proj_w, void* out, int B, int H, int N, int d, int block, float topk,
                        sagesla_stream_t stream) {
  if (!gamma_q || !gamma_k || !(eps >= 0.f) || eps > 1.f) return SAGESLA_ERR_INVALID;
  if (!aligned16(gamma_q) || !aligned16(gamma_k)) return SAGESLA_ERR_MISALIGNED;
  NormIn n;
  n.gq = gamma_q;
  n.gk = gamma_k;
  n.eps = (double)eps;
  n.B = B;
  n.H = H;
  return run_attn(q, k, v, proj_w, out, B, H, N, d, block, topk, reinterpret_cast<cudaStream_t>(stream), 0, 0, 0, 127,
                  0, &n);
}

int sagesla_attn_bnhd(const void* q, const void* k, const void* v, const void* gamma_q, const void* gamma_k,
                      float eps, const void* proj_w, void* out, int B, int N, int H, int d, int block, float topk,
                      sagesla_stream_t stream) {
  if ((gamma_q == nullptr) != (gamma_k == nullptr)) return SAGESLA_ERR_INVALID;
  NormIn n;
  if (gamma_q) {
    if (!(eps >= 0.f) || eps > 1.f) return SAGESLA_ERR_INVALID;
    if (!aligned16(gamma_q) || !aligned16(gamma_k)) return SAGESLA_ERR_MISALIGNED;
    n.gq = gamma_q;
    n.gk = gamma_k;
    n.eps = (double)eps;
    n.B = B;
    n.H = H;
  }
  return run_attn(q, k, v, proj_w, out, B, H, N, d, block, topk, reinterpret_cast<cudaStream_t>(stream), 0, 0, 0, 127,
                  0, gamma_q ? &n : nullptr, 1);
}

int dense_int8_attn(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                    sagesla_stream_t stream) {
  return run_attn(q, k, v, nullptr, out, B, H, N, d, 64, 1.0f, reinterpret_cast<cudaStream_t>(stream));
}

// Copy streams of the host-buffer entry point, one pair per device (created
// once, never destroyed: they live as long as the process).
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
};

int copy_streams(int dev, CopyStreams* out) {
  static std::mutex cmu;
  static std::map<int, CopyStreams> cs;
  std::lock_guard<std::mutex> lk(cmu);
  CopyStreams& c = cs[dev];
  if (!c.h2d) {
    if (cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      return SAGESLA_ERR_LAUNCH;
    }
  }
  *out = c;
  return SAGESLA_OK;
}

// The heads are independent problems, so the host-buffer call runs in chunks
// of heads as a three-stage pipeline: host->device copies of chunk c+1 (copy
// stream), the path on chunk c (the caller's stream) and device->host copies
// of chunk c-1 (a second copy stream) overlap.
int sagesla_attn_host(const void* q, const void* k, const void* v, const void* proj_w, void* out, int B, int H,
                      int N, int d, int block, float topk, sagesla_stream_t stream) {
  SAGESLA_TRY(validate(q, k, v, out, B, H, N, d, block, topk));
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CopyStreams cs;
  SAGESLA_TRY(copy_streams(dev, &cs));
  const size_t E = (size_t)B * H * N * d * 2;  // bytes of one bf16 tensor
  const size_t W = (size_t)d * d * 2;
  // Device staging lives in its own cached region per (device, stream).
  uint8_t* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_stage[std::make_pair(dev, st)];
    const size_t need = 4 * up(E) + up(W);
    if (w.bytes < need) {
      if (w.ptr) cudaFreeAsync(w.ptr, st);
      w.ptr = nullptr;
      w.bytes = 0;
      if (cudaMallocAsync(&w.ptr, need, st) != cudaSuccess) {
        cudaGetLastError();
        return SAGESLA_ERR_OOM;
      }
      w.bytes = need;
    }
    base = static_cast<uint8_t*>(w.ptr);
  }
  uint8_t* dq = base;
  uint8_t* dk = dq + up(E);
  uint8_t* dv = dk + up(E);
  uint8_t* dout = dv + up(E);
  uint8_t* dw = dout + up(E);
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  const uint8_t* hv = static_cast<const uint8_t*>(v);
  uint8_t* hout = static_cast<uint8_t*>(out);
  const int BH = B * H;
  const int nchunk = BH < 20 ? BH : 20;
  const int per = (BH + nchunk - 1) / nchunk;  // heads per chunk (the last may have fewer)
  const size_t head_bytes = (size_t)N * d * 2;
  std::vector<cudaEvent_t> ev(2 * nchunk + 1, nullptr);
  auto cleanup = [&]() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
  };
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      cleanup();
      return SAGESLA_ERR_LAUNCH;
    }
  int rc = SAGESLA_OK;
  // The staging buffers may still be read by work queued earlier on `st`.
  if (cudaEventRecord(ev[2 * nchunk], st) != cudaSuccess || cudaStreamWaitEvent(cs.h2d, ev[2 * nchunk], 0) != cudaSuccess)
    rc = SAGESLA_ERR_LAUNCH;
  if (rc == SAGESLA_OK && proj_w && cudaMemcpyAsync(dw, proj_w, W, cudaMemcpyHostToDevice, cs.h2d) != cudaSuccess)
    rc = SAGESLA_ERR_LAUNCH;
  for (int c = 0; rc == SAGESLA_OK && c < nchunk; ++c) {
    const int h0 = c * per, hn = (h0 + per <= BH ? per : BH - h0);
    if (hn <= 0) break;
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)hn * head_bytes;
    if (cudaMemcpyAsync(dq + off, hq + off, bytes, cudaMemcpyHostToDevice, cs.h2d) != cudaSuccess ||
        cudaMemcpyAsync(dk + off, hk + off, bytes, cudaMemcpyHostToDevice, cs.h2d) != cudaSuccess ||
        cudaMemcpyAsync(dv + off, hv + off, bytes, cudaMemcpyHostToDevice, cs.h2d) != cudaSuccess ||
        cudaEventRecord(ev[c], cs.h2d) != cudaSuccess || cudaStreamWaitEvent(st, ev[c], 0) != cudaSuccess) {
      rc = SAGESLA_ERR_LAUNCH;
      break;
    }
    rc = run_attn(dq + off, dk + off, dv + off, proj_w ? dw : nullptr, dout + off, 1, hn, N, d, block, topk, st);
    if (rc != SAGESLA_OK) break;
    if (cudaEventRecord(ev[nchunk + c], st) != cudaSuccess || cudaStreamWaitEvent(cs.d2h, ev[nchunk + c], 0) != cudaSuccess ||
        cudaMemcpyAsync(hout + off, dout + off, bytes, cudaMemcpyDeviceToHost, cs.d2h) != cudaSuccess) {
      rc = SAGESLA_ERR_LAUNCH;
      break;
    }
  }
  // Every queued copy and kernel must be finished before the caller's host
  // buffers are released (also on an error path).
  if (cudaStreamSynchronize(cs.h2d) != cudaSuccess) rc = SAGESLA_ERR_LAUNCH;
  if (cudaStreamSynchronize(st) != cudaSuccess) rc = SAGESLA_ERR_LAUNCH;
  if (cudaStreamSynchronize(cs.d2h) != cudaSuccess) rc = SAGESLA_ERR_LAUNCH;
  cleanup();
  return rc;
}

int sagesla_get_quant(const void* q, const void* k, const void* v, int B, int H, int N, int d, int8_t* q8,
                      int8_t* k8, uint8_t* v8, float* sq, float* sk, float* sv, float* mu, sagesla_stream_t stream) {
  SAGESLA_TRY(validate(q, k, v, q8, B, H, N, d, 64, 1.0f));
  if (!k8 || !v8 || !sq || !sk || !sv || !mu) return SAGESLA_ERR_INVALID;
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Geom g = make_geom(B, H, N, 64, 1.0f);
  const Buffers sizes = carve(nullptr, g);
  uint8_t* base = nullptr;
  SAGESLA_TRY(get_workspace(dev, st, sizes.total, &base));
  const Buffers b = carve(base, g);
  SAGESLA_TRY(run_front(q, k, v, g, b, dev, st));
  SAGESLA_TRY(launch_rc(launch_untile(b.q8t, b.k8t, b.v8t, g, q8, k8, v8, st)));
  const int nq64 = (N + 63) / 64;
  const size_t pitch = (size_t)g.nq * sizeof(float);
  if (cudaMemcpy2DAsync(sq, nq64 * sizeof(float), b.sq, pitch, nq64 * sizeof(float), g.BH, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
    return SAGESLA_ERR_LAUNCH;
  if (cudaMemcpy2DAsync(sk, nq64 * sizeof(float), b.sk, pitch, nq64 * sizeof(float), g.BH, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
    return SAGESLA_ERR_LAUNCH;
  if (cudaMemcpyAsync(sv, b.sv, (size_t)g.BH * kD * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SAGESLA_ERR_LAUNCH;
  if (cudaMemcpyAsync(mu, b.mu, (size_t)g.BH * kD * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SAGESLA_ERR_LAUNCH;
  return SAGESLA_OK;
}

int sagesla_get_mask(const void* q, const void* k, int B, int H, int N, int d, int block, float topk,
                     int32_t* idx_out, float* qbar, float* kbar, int* k_out, sagesla_stream_t stream) {
  SAGESLA_TRY(validate(q, k, k, idx_out, B, H, N, d, block, topk));
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Geom g = make_geom(B, H, N, block, topk);
  const Buffers sizes = carve(nullptr, g);
  uint8_t* base = nullptr;
  SAGESLA_TRY(get_workspace(dev, st, sizes.total, &base));
  const Buffers b = carve(base, g);
  // The mask needs only K's mean and the pooled sums; V is read as K here
  // (its quantised codes are discarded).
  SAGESLA_TRY(run_front(q, k, k, g, b, dev, st));
  SAGESLA_TRY(launch_rc(launch_pool_topk(b.qsum, b.ksum, g, idx_out, qbar ? qbar : b.qbar, kbar ? kbar : b.kbar,
                                         nullptr, nullptr, nullptr, nullptr, st)));
  if (k_out) *k_out = g.kc;
  return SAGESLA_OK;
}

int sagesla_watchdog_selftest(int probes, sagesla_stream_t stream) {
  if (probes < 1 || probes > (1 << 20)) return SAGESLA_ERR_INVALID;
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  return launch_rc(launch_watchdog_selftest(probes, watchdog(dev), reinterpret_cast<cudaStream_t>(stream)));
}

int sagesla_debug_flash_stall(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                              float topk, int grid, int stall_step, long long spin_limit, sagesla_stream_t stream) {
  if (grid < 1 || stall_step < -1 || spin_limit < 1024 || spin_limit > kSpinLimit) return SAGESLA_ERR_INVALID;
  return run_attn(q, k, v, nullptr, out, B, H, N, d, 64, topk, reinterpret_cast<cudaStream_t>(stream), grid,
                  stall_step + 1, (long)spin_limit);
}

// ------------------------------------------------------------- W8A8 linear
int sagesla_w8a8_quant(const void* a, int rows, int cols, void* codes, float* scales, sagesla_stream_t stream) {
  if (!a || !codes || !scales || rows < 1 || cols < 128 || cols % 128 != 0 || rows > 8388480 ||
      (double)rows * cols >= 1099511627776.0)
    return SAGESLA_ERR_INVALID;
  if (!aligned16(a) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return SAGESLA_ERR_MISALIGNED;
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope ps(9, st);
  return launch_rc(launch_w8a8_quant(a, rows, cols, static_cast<uint8_t*>(codes), scales, st));
}


int sagesla_w8a8_gemm(const void* xq, const float* sx, const void* wq, const float* sw, void* y, int M, int N, int K,
                      sagesla_stream_t stream) {
  SAGESLA_TRY(check_gemm(xq, sx, wq, sw, y, M, N, K));
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope ps(10, st);
  return launch_rc(launch_w8a8_gemm(static_cast<const uint8_t*>(xq), sx, static_cast<const uint8_t*>(wq), sw, y, M, N,
                                    K, watchdog(dev), st));
}

int sagesla_w8a8_linear(const void* x, const void* wq, const float* sw, void* y, int M, int N, int K,
                        sagesla_stream_t stream) {
  if (!x) return SAGESLA_ERR_INVALID;
  const float one = 1.f;
  SAGESLA_TRY(check_gemm(x, &one, wq, sw, y, M, N, K));  // x stands in for its codes in the checks
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t cb = up(w8a8_codes_bytes(M, K));
  uint8_t* base = nullptr;
  SAGESLA_TRY(get_workspace(dev, st, cb + w8a8_scales_count(M, K) * sizeof(float), &base));
  float* sx = reinterpret_cast<float*>(base + cb);
  {
    ProfScope ps(9, st);
    SAGESLA_TRY(launch_rc(launch_w8a8_quant(x, M, K, base, sx, st)));
  }
  ProfScope ps(10, st);
  return launch_rc(launch_w8a8_gemm(base, sx, static_cast<const uint8_t*>(wq), sw, y, M, N, K, watchdog(dev), st));
}

int sagesla_sync_status(sagesla_stream_t stream) {
  int dev = 0;
  SAGESLA_TRY(check_device(&dev));
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SAGESLA_ERR_LAUNCH;
  int* wd = watchdog(dev);
  int h = 0;
  if (cudaMemcpy(&h, wd, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SAGESLA_ERR_LAUNCH;
  if (h) {
    cudaMemset(wd, 0, sizeof(int));
    return SAGESLA_ERR_DEVICE_TIMEOUT;
  }
  return SAGESLA_OK;
}

const char* sagesla_strerror(int code) {
  switch (code) {
    case SAGESLA_OK: return "ok";
    case SAGESLA_ERR_INVALID: return "invalid argument";
    case SAGESLA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SAGESLA_ERR_OOM: return "workspace allocation failed";
    case SAGESLA_ERR_LAUNCH: return "CUDA launch or runtime error";
    case SAGESLA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case SAGESLA_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    default: return "unknown error";
  }
}

void sagesla_profile(int enable) {
  std::lock_guard<std::mutex> lk(g_pmu);
  g_prof_on = enable != 0;
}

int sagesla_profile_read(double* ms, int* launches, int nkernels) {
  std::lock_guard<std::mutex> lk(g_pmu);
  for (int i = 0; i < nkernels; ++i) {
    if (ms) ms[i] = 0.0;
    if (launches) launches[i] = 0;
  }
  int rc = SAGESLA_OK;
  for (auto& r : g_prof) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) rc = SAGESLA_ERR_LAUNCH;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) rc = SAGESLA_ERR_LAUNCH;
    if (r.kernel >= 0 && r.kernel < nkernels) {
      if (ms) ms[r.kernel] += t;
      if (launches) launches[r.kernel] += 1;
    }
    g_evpool.push_back(r.a);
    g_evpool.push_back(r.b);
  }
  g_prof.clear();
  return rc;
}

void sagesla_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  cudaDeviceSynchronize();
  for (auto& kv : g_ws)
    if (kv.second.ptr) cudaFree(kv.second.ptr);
  g_ws.clear();
  for (auto& kv : g_stage)
    if (kv.second.ptr) cudaFree(kv.second.ptr);
  g_stage.clear();
}

}  // extern "C"
