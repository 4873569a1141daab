// libslim C ABI: argument validation, workspace carving, stage sequencing on
// the caller's stream, device status mapping and per-stage timing.
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "../../include/slim.h"

namespace slim {
// stage launchers (defined in the kernel files)
cudaError_t launch_hessian(const void* X, int xdtype, int64_t N, int64_t n, double* H, void* part, DevStatus* st,
                           int num_sms, cudaStream_t s, cudaEvent_t* kev);
size_t hessian_ws_bytes(int64_t N, int64_t n, int xdtype);
size_t hinv_workspace_doubles(int64_t n);
cudaError_t launch_hessian_slices(const void* X, int64_t N, int64_t n, void* part, DevStatus* st, int num_sms,
                                  cudaStream_t s, int slice0, int nsl);
cudaError_t launch_hessian_reduce(int64_t N, int64_t n, const void* part, double* H, cudaStream_t s);
int hessian_slice_tokens();
cudaError_t launch_hinv(const double* H, int64_t n, double alpha, double* h, double* ws, DevStatus* st,
                        cudaStream_t s);
int salience_row_blocks(int64_t m);
cudaError_t launch_salience(const float* W, int64_t m, int64_t n, const double* h, int group, double* S,
                            int32_t* order, double* part, cudaStream_t st);
size_t sba_ws_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group);
size_t sba_prep_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group);
size_t sba_search_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group);
cudaError_t launch_sba_prep_w(const float* W, int64_t m, int64_t n, int64_t N, int xdtype, int group, int avg_bits,
                              uint8_t* pw, DevStatus* st, int num_sms, int bps, cudaStream_t s);
cudaError_t launch_sba_prep_x(const void* X, int64_t m, int64_t n, int64_t N, int xdtype, int group, int64_t t0,
                              int64_t t1, uint8_t* pw, DevStatus* st, int num_sms, int bps, cudaStream_t s);
size_t sba_yd_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group);
size_t sba_split_offset(int64_t m, int64_t n, int64_t N, int xdtype, int group, int* nbox);
cudaError_t launch_sba_phase_a(int64_t m, int64_t n, int xdtype, int64_t N, int group, int objective, int tp0,
                               int tp1, const uint8_t* pw, uint8_t* sw, float* yd, DevStatus* st, int num_sms,
                               cudaStream_t s);
cudaError_t launch_sba_steps(int64_t m, int64_t n, int xdtype, int64_t N, int group, int avg_bits,
                             const int32_t* order, int objective, double* kl, int32_t* p_star, uint8_t* bits,
                             const uint8_t* pw, uint8_t* sw, float* yd, DevStatus* st, int num_sms, cudaStream_t s);
cudaError_t launch_sba_search(int64_t m, int64_t n, int xdtype, int64_t N, int group, int avg_bits,
                              const int32_t* order, int objective, double* kl, int32_t* p_star, uint8_t* bits,
                              const uint8_t* pw, uint8_t* sw, DevStatus* st, int num_sms, cudaStream_t s,
                              cudaEvent_t* kev);
cudaError_t launch_sba(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                       int avg_bits, const int32_t* order, int objective, int precision, double* kl, int32_t* p_star,
                       uint8_t* bits, uint8_t* ws, DevStatus* st, int num_sms, cudaStream_t s, cudaEvent_t* kev);
cudaError_t launch_sba_select(const float* W, const void* X, int64_t m, int64_t n, int64_t N, int xdtype, int group,
                              int precision, uint8_t* pw, uint8_t* sw, cudaStream_t s);
cudaError_t launch_order_check(const int32_t* order, int k, int32_t* out, DevStatus* st, cudaStream_t s);
size_t gptq_workspace_doubles(int64_t m, int64_t n);
size_t dg_workspace_bytes(int64_t m, int64_t n, int group, int avg_bits, int64_t B);
cudaError_t launch_dequant_gemv(const uint32_t* codes, const uint8_t* bits, const float* scale, const float* zero,
                                int64_t m, int64_t n, int group, int avg_bits, const void* x, int xdtype, int B,
                                float* y, uint8_t* ws, cudaStream_t s);
cudaError_t launch_gptq(const float* W, int64_t m, int64_t n, const double* H, double alpha, const uint8_t* bits,
                        int group, int avg_bits, double lam, int n_tau, uint32_t* codes, float* scale, float* zero,
                        uint8_t* tau_idx, double* h, double* ws, DevStatus* st, int num_sms, cudaStream_t s);
cudaError_t launch_sqc(const float* W, int64_t m, int64_t n, const double* h, const uint8_t* bits, int group,
                       int avg_bits, double lam, int n_tau, uint32_t* codes, float* scale, float* zero,
                       uint8_t* tau_idx, int num_sms, cudaStream_t st);
static std::atomic<long long> g_launches{0};
void count_launches(int k) { g_launches.fetch_add(k, std::memory_order_relaxed); }
}  // namespace slim

using namespace slim;

namespace {

thread_local std::string g_last_cuda_error;
thread_local int g_last_detail = 0;
constexpr double kDampAlpha = 0.01;
constexpr size_t kStatusBytes = sizeof(DevStatus);
constexpr int kMaxGroups = 1024;

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = cudaGetErrorString(e);
  return SLIM_ECUDA;
}

#define SLIM_CUDA(call)                              \
  do {                                               \
    cudaError_t e__ = (call);                        \
    if (e__ != cudaSuccess) return cuda_fail(e__);   \
  } while (0)

// Current device must be an sm_100 part; returns its SM count.
int device_sms(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) { g_last_cuda_error = cudaGetErrorString(e); return SLIM_ENODEV; }
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return SLIM_ENODEV;
  cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  return SLIM_OK;
}

bool injected(const char* stage) {
  const char* f = std::getenv("SLIM_FAULT");
  return f && (std::strcmp(f, stage) == 0 || std::strcmp(f, "all") == 0);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_shape(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  if (m < 1 || n < 1 || N < 1) return SLIM_EINVAL;
  if (group != 32 && group != 64 && group != 128) return SLIM_EINVAL;
  if (n % group != 0) return SLIM_EINVAL;
  if (n / group > kMaxGroups) return SLIM_EINVAL;
  if (n > 65535 || m > (int64_t)1 << 30 || N > (int64_t)1 << 31) return SLIM_EINVAL;
  if (xdtype != SLIM_X_F32 && xdtype != SLIM_X_BF16) return SLIM_EINVAL;
  return SLIM_OK;
}

int check_bits(int avg_bits) { return (avg_bits >= 2 && avg_bits + 1 <= 8) ? SLIM_OK : SLIM_EINVAL; }

// Sync the stream, then map CUDA errors and the device status word.
int finish(cudaStream_t s, const DevStatus* dst) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  DevStatus hs;
  e = cudaMemcpy(&hs, dst, sizeof(hs), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  g_last_detail = hs.code ? hs.where : 0;
  if (hs.code == kStatusTimeout) return SLIM_ETIMEOUT;
  if (hs.code == kStatusNotPD) return SLIM_ENOTPD;
  if (hs.code == kStatusRangeCode) return SLIM_ERANGE;
  if (hs.code == kStatusInvalid) return SLIM_EINVAL;
  if (hs.code != 0) return SLIM_ECUDA;
  return SLIM_OK;
}

constexpr int kMaxDevices = 64;

// The library's own stream-ordered memory pool on the current device (created
// on first use, kept until the process exits). It keeps freed blocks instead of
// returning them to the driver at every synchronization, so repeated calls that
// let the library allocate do not re-map gigabytes each time; being the
// library's own, it leaves the device's default pool and its settings alone.
cudaError_t library_pool(cudaMemPool_t* out) {
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) { cudaMemPoolDestroy(pool); return e; }
    pools[dev] = pool;
  }
  *out = pools[dev];
  return cudaSuccess;
}

// Workspace holder: caller memory or a cudaMallocAsync'd block freed on scope exit.
struct Workspace {
  uint8_t* p = nullptr;
  bool owned = false;
  bool sync_on_release = true;  // false: the stream-ordered free is enough (asynchronous calls)
  cudaStream_t s = nullptr;
  int acquire(void* ws, size_t ws_bytes, size_t need, cudaStream_t st) {
    s = st;
    if (ws) {
      if (ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return SLIM_EINVAL;
      p = static_cast<uint8_t*>(ws);
      return SLIM_OK;
    }
    if (need == 0) {  // nothing to allocate
      p = nullptr;
      return SLIM_OK;
    }
    cudaMemPool_t pool;
    cudaError_t e = library_pool(&pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&p), need, pool, st);
    if (e != cudaSuccess) { g_last_cuda_error = cudaGetErrorString(e); cudaGetLastError(); return SLIM_ENOMEM; }
    owned = true;
    return SLIM_OK;
  }
  ~Workspace() {
    if (owned && p) {
      cudaFreeAsync(p, s);
      if (sync_on_release) cudaStreamSynchronize(s);
    }
  }
};

size_t hinv_bytes(int64_t n) { return hinv_workspace_doubles(n) * sizeof(double); }
size_t sal_bytes(int64_t m, int64_t n) { return (size_t)salience_row_blocks(m) * n * sizeof(double); }

// Per host thread and device: the side streams of the whole-layer paths.
// cs carries the host-buffer path's chunked host-to-device copy of X (it
// overlaps the Hessian; ev are its events); ps, at the lowest priority,
// prepares the SBA operands beside other stages (pe[0] forks it, pe[1] joins
// it): beside the chunked Hessian in the host-buffer path, beside the
// latency-bound inverse-Hessian stage in the device path.
struct HostCopy {
  int dev = -1;
  bool ok = false;
  cudaStream_t cs = nullptr, ps = nullptr;
  cudaEvent_t pe[2] = {};
  std::vector<cudaEvent_t> ev;
};
// Returns nullptr when the current device cannot be determined or its ordinal
// is beyond the table.
HostCopy* host_copy(int events) {
  thread_local HostCopy hc[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  HostCopy& x = hc[dev];
  if (x.dev != dev) {
    int least = 0, greatest = 0;
    cudaDeviceGetStreamPriorityRange(&least, &greatest);
    x.ok = cudaStreamCreateWithFlags(&x.cs, cudaStreamNonBlocking) == cudaSuccess &&
           cudaStreamCreateWithPriority(&x.ps, cudaStreamNonBlocking, least) == cudaSuccess &&
           cudaEventCreateWithFlags(&x.pe[0], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&x.pe[1], cudaEventDisableTiming) == cudaSuccess;
    x.dev = dev;
  }
  while (x.ok && (int)x.ev.size() < events) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      x.ok = false;
      break;
    }
    x.ev.push_back(e);
  }
  return &x;
}

// Layout of the full-path workspace. The scratch region holds the SBA
// operands, prepared beside the Hessian (at off_scratch), and behind them
// (off_rest) the scratch that the Hessian's partial sums, hinv, salience and
// the SBA search use in turn.
struct LayerWs {
  size_t off_H, off_h, off_S, off_order, off_kl, off_pstar, off_scratch, off_rest, total;
};
LayerWs layer_ws(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  LayerWs w{};
  const int64_t k = n / group;
  const int64_t P = k / 2 + 1;
  size_t off = kStatusBytes;
  w.off_H = off; off = al256(off + (size_t)n * n * 8);
  w.off_h = off; off = al256(off + (size_t)n * 8);
  w.off_S = off; off = al256(off + (size_t)k * 8);
  w.off_order = off; off = al256(off + (size_t)k * 4);
  w.off_kl = off; off = al256(off + (size_t)P * 8);
  w.off_pstar = off; off = al256(off + 8);
  size_t rest = hinv_bytes(n);
  size_t t = sal_bytes(m, n); if (t > rest) rest = t;
  t = sba_search_bytes(m, n, N, xdtype, group); if (t > rest) rest = t;
  t = hessian_ws_bytes(N, n, xdtype); if (t > rest) rest = t;
  t = gptq_workspace_doubles(m, n) * sizeof(double) + (size_t)n * sizeof(double) + 256; if (t > rest) rest = t;
  const size_t prep = al256(sba_prep_bytes(m, n, N, xdtype, group));
  w.off_scratch = off;
  w.off_rest = off + prep;
  off = al256(off + prep + rest);
  w.total = off;
  return w;
}

// On every return, s first waits for all work queued so far on the side
// stream `from` (through event e), so a workspace released or reused in s's
// order is never touched by work still running there.
struct JoinOnExit {
  cudaStream_t s, from;
  cudaEvent_t e;
  ~JoinOnExit() {
    if (cudaEventRecord(e, from) == cudaSuccess) cudaStreamWaitEvent(s, e, 0);
  }
};

// Forks onto the side stream, once everything queued on s so far is done,
// the preparation of the SBA weight operands and (X non-null) of all of X,
// at bps_w and bps_x blocks per SM. Join with join_prepare.
cudaError_t fork_prepare(HostCopy& side, const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N,
                         int group, int avg_bits, uint8_t* pw, DevStatus* st, int sms, int bps_w, int bps_x,
                         cudaStream_t s) {
  cudaError_t e = cudaEventRecord(side.pe[0], s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side.ps, side.pe[0], 0);
  if (e == cudaSuccess) e = launch_sba_prep_w(W, m, n, N, xdtype, group, avg_bits, pw, st, sms, bps_w, side.ps);
  if (e == cudaSuccess && X) e = launch_sba_prep_x(X, m, n, N, xdtype, group, 0, N, pw, st, sms, bps_x, side.ps);
  return e;
}
cudaError_t join_prepare(HostCopy& side, cudaStream_t s) {
  cudaError_t e = cudaEventRecord(side.pe[1], side.ps);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, side.pe[1], 0);
  return e;
}

}  // namespace

extern "C" {

const char* slim_status_string(int status) {
  switch (status) {
    case SLIM_OK: return "ok";
    case SLIM_EINVAL: return "invalid argument";
    case SLIM_ENOMEM: return "out of device memory";
    case SLIM_ECUDA: return "CUDA error";
    case SLIM_ETIMEOUT: return "device wait timed out";
    case SLIM_ENOTPD: return "damped Hessian is not positive definite";
    case SLIM_ENODEV: return "no sm_100 device";
    case SLIM_EINJECTED: return "injected failure";
    case SLIM_ERANGE: return "a value is out of the fp16 operand range";
    default: return "unknown status";
  }
}

const char* slim_last_cuda_error(void) { return g_last_cuda_error.c_str(); }
int slim_last_status_detail(void) { return g_last_detail; }
const char* slim_version(void) { return "libslim 0.1 (sm_100a)"; }

int slim_num_candidates(int64_t n, int group) {
  if (group <= 0 || n % group) return -1;
  return (int)(n / group / 2 + 1);
}
int64_t slim_row_words(int64_t n, int avg_bits) { return n * avg_bits / 32; }
int64_t slim_launch_count(void) { return g_launches.load(); }

// ------------------------------------------------------------------ hessian
size_t slim_hessian_workspace_bytes(int64_t N, int64_t n, int xdtype) {
  return kStatusBytes + al256(hessian_ws_bytes(N, n, xdtype));
}

int slim_hessian(const void* X, int xdtype, int64_t N, int64_t n, double* H, void* ws, size_t ws_bytes,
                 void* stream) {
  if (!X || !H || N < 1 || n < 32 || n % 32 || n > 65535 || (xdtype != 0 && xdtype != 1) || !aligned16(X))
    return SLIM_EINVAL;
  int sms = 0;
  int rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("hessian")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, slim_hessian_workspace_bytes(N, n, xdtype), s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
  SLIM_CUDA(launch_hessian(X, xdtype, N, n, H, w.p + kStatusBytes, st, sms, s, nullptr));
  return finish(s, st);
}

// ------------------------------------------------------------------ hinv_diag
size_t slim_hinv_diag_workspace_bytes(int64_t n) { return kStatusBytes + al256(hinv_bytes(n)); }

int slim_hinv_diag(const double* H, int64_t n, double alpha, double* h, void* ws, size_t ws_bytes, void* stream) {
  if (!H || !h || n < 1 || n > 65535 || !(alpha >= 0.0)) return SLIM_EINVAL;
  int sms = 0;
  int rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("hinv_diag")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, slim_hinv_diag_workspace_bytes(n), s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
  SLIM_CUDA(launch_hinv(H, n, alpha, h, reinterpret_cast<double*>(w.p + kStatusBytes), st, s));
  return finish(s, st);
}

// ------------------------------------------------------------------ salience
size_t slim_salience_workspace_bytes(int64_t m, int64_t n, int group) {
  (void)group;
  return kStatusBytes + al256(sal_bytes(m, n));
}

int slim_salience(const float* W, int64_t m, int64_t n, const double* h, int group, double* S, int32_t* order,
                  void* ws, size_t ws_bytes, void* stream) {
  if (!W || !h || !S || !order || !aligned16(W)) return SLIM_EINVAL;
  int rc = check_shape(m, n, 1, SLIM_X_BF16, group);
  if (rc) return rc;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("salience")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, slim_salience_workspace_bytes(m, n, group), s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
  SLIM_CUDA(launch_salience(W, m, n, h, group, S, order, reinterpret_cast<double*>(w.p + kStatusBytes), s));
  return finish(s, st);
}

// ------------------------------------------------------------------ sba_search
// Workspace of the search entries: [status][checked copy of the order][search].
size_t slim_sba_workspace_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  if (check_shape(m, n, N, xdtype, group)) return 0;
  return kStatusBytes + al256((size_t)(n / group) * 4) + al256(sba_ws_bytes(m, n, N, xdtype, group));
}

int slim_sba_search_ex(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                       int avg_bits, const int32_t* order, int objective, int precision, double* kl, int32_t* p_star,
                       uint8_t* bits, void* ws, size_t ws_bytes, void* stream) {
  if (!W || !X || !order || !bits || !aligned16(W) || !aligned16(X)) return SLIM_EINVAL;
  if (objective != SLIM_OBJ_KL && objective != SLIM_OBJ_MSE) return SLIM_EINVAL;
  if (precision != SLIM_SBA_ADAPTIVE && precision != SLIM_SBA_FULL) return SLIM_EINVAL;
  int rc = check_shape(m, n, N, xdtype, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("sba_search")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, slim_sba_workspace_bytes(m, n, N, xdtype, group), s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  int32_t* ord = reinterpret_cast<int32_t*>(w.p + kStatusBytes);
  uint8_t* sw = w.p + kStatusBytes + al256((size_t)(n / group) * 4);
  SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
  SLIM_CUDA(launch_order_check(order, (int)(n / group), ord, st, s));
  SLIM_CUDA(launch_sba(W, m, n, X, xdtype, N, group, avg_bits, ord, objective, precision, kl, p_star, bits, sw, st,
                       sms, s, nullptr));
  return finish(s, st);
}

int slim_sba_search(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                    int avg_bits, const int32_t* order, double* kl, int32_t* p_star, uint8_t* bits, void* ws,
                    size_t ws_bytes, void* stream) {
  return slim_sba_search_ex(W, m, n, X, xdtype, N, group, avg_bits, order, SLIM_OBJ_KL, SLIM_SBA_ADAPTIVE, kl,
                            p_star, bits, ws, ws_bytes, stream);
}

size_t slim_sba_split_workspace_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  if (check_shape(m, n, N, xdtype, group)) return 0;
  return kStatusBytes + al256((size_t)(n / group) * 4) + al256(sba_ws_bytes(m, n, N, xdtype, group)) +
         al256(sba_yd_bytes(m, n, N, xdtype, group));
}

int slim_sba_search_split(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                          int avg_bits, const int32_t* order, double* kl, int32_t* p_star, uint8_t* bits,
                          int64_t chunk_tokens, void* ws, size_t ws_bytes, void* stream) {
  if (!W || !X || !order || !bits || !aligned16(W) || !aligned16(X)) return SLIM_EINVAL;
  if (chunk_tokens <= 0 || chunk_tokens % 256) return SLIM_EINVAL;
  int rc = check_shape(m, n, N, xdtype, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("sba_search")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, slim_sba_split_workspace_bytes(m, n, N, xdtype, group), s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  int32_t* ord = reinterpret_cast<int32_t*>(w.p + kStatusBytes);
  uint8_t* pw = w.p + kStatusBytes + al256((size_t)(n / group) * 4);
  const size_t prep = sba_prep_bytes(m, n, N, xdtype, group);
  uint8_t* sw = pw + prep;
  float* yd = reinterpret_cast<float*>(pw + al256(sba_ws_bytes(m, n, N, xdtype, group)));
  SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
  SLIM_CUDA(launch_order_check(order, (int)(n / group), ord, st, s));
  SLIM_CUDA(launch_sba_prep_w(W, m, n, N, xdtype, group, avg_bits, pw, st, sms, 8, s));
  SLIM_CUDA(launch_sba_select(W, X, m, n, N, xdtype, group, SLIM_SBA_ADAPTIVE, pw, sw, s));
  for (int64_t t0 = 0; t0 < N; t0 += chunk_tokens) {
    const int64_t t1 = (t0 + chunk_tokens < N) ? t0 + chunk_tokens : N;
    SLIM_CUDA(launch_sba_prep_x(X, m, n, N, xdtype, group, t0, t1, pw, st, sms, 8, s));
    SLIM_CUDA(launch_sba_phase_a(m, n, xdtype, N, group, SLIM_OBJ_KL, (int)(t0 / 256), (int)((t1 + 255) / 256), pw,
                                 sw, yd, st, sms, s));
  }
  SLIM_CUDA(launch_sba_steps(m, n, xdtype, N, group, avg_bits, ord, SLIM_OBJ_KL, kl, p_star, bits, pw, sw, yd, st,
                             sms, s));
  return finish(s, st);
}

// ------------------------------------------------------------------ sqc
int slim_sqc(const float* W, int64_t m, int64_t n, const double* h, const uint8_t* bits, int group, int avg_bits,
             double lambda, int n_tau, uint32_t* codes, float* scale, float* zero, uint8_t* tau_idx,
             void* stream) {
  if (!W || !h || !bits || !codes || !scale || !zero) return SLIM_EINVAL;
  int rc = check_shape(m, n, 1, SLIM_X_BF16, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  if (!(lambda >= 0.0 && lambda < 1.0) || n_tau < 1 || n_tau > 256) return SLIM_EINVAL;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("sqc")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SLIM_CUDA(launch_sqc(W, m, n, h, bits, group, avg_bits, lambda, n_tau, codes, scale, zero, tau_idx, sms, s));
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

// ------------------------------------------------------------------ gptq
size_t slim_gptq_workspace_bytes(int64_t m, int64_t n) {
  if (m < 1 || n < 1) return 0;
  return kStatusBytes + al256(gptq_workspace_doubles(m, n) * sizeof(double) + (size_t)n * sizeof(double));
}

int slim_gptq(const float* W, int64_t m, int64_t n, const double* H, const uint8_t* bits, int group, int avg_bits,
              double lambda, int n_tau, uint32_t* codes, float* scale, float* zero, uint8_t* tau_idx, void* ws,
              size_t ws_bytes, void* stream) {
  if (!W || !H || !bits || !codes || !scale || !zero) return SLIM_EINVAL;
  int rc = check_shape(m, n, 1, SLIM_X_BF16, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  if (!(lambda >= 0.0 && lambda < 1.0) || n_tau < 1 || n_tau > 256) return SLIM_EINVAL;
  if (m > (int64_t)65535 * 64) return SLIM_EINVAL;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("gptq")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, slim_gptq_workspace_bytes(m, n), s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  double* gws = reinterpret_cast<double*>(w.p + kStatusBytes);
  double* gh = gws + gptq_workspace_doubles(m, n);
  SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
  SLIM_CUDA(launch_gptq(W, m, n, H, kDampAlpha, bits, group, avg_bits, lambda, n_tau, codes, scale, zero, tau_idx, gh,
                        gws, st, sms, s));
  return finish(s, st);
}

// ------------------------------------------------------------------ dequant gemv
size_t slim_dequant_gemv_workspace_bytes(int64_t m, int64_t n, int group, int avg_bits, int64_t batch) {
  if (m < 1 || n < 1 || group < 32 || n % group || batch < 1 || batch > 8 || avg_bits < 1 || avg_bits > 8) return 0;
  return al256(dg_workspace_bytes(m, n, group, avg_bits, batch));
}

int slim_dequant_gemv(const uint32_t* codes, const uint8_t* bits, const float* scale, const float* zero, int64_t m,
                      int64_t n, int group, int avg_bits, const void* x, int xdtype, int64_t batch, float* y,
                      void* ws, size_t ws_bytes, void* stream) {
  if (!codes || !bits || !scale || !zero || !x || !y || !aligned16(codes) || !aligned16(x)) return SLIM_EINVAL;
  int rc = check_shape(m, n, 1, xdtype, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  if (batch < 1 || batch > 8 || (n * avg_bits) % 32) return SLIM_EINVAL;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  if (injected("dequant_gemv")) return SLIM_EINJECTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w;
  w.sync_on_release = false;
  rc = w.acquire(ws, ws_bytes, slim_dequant_gemv_workspace_bytes(m, n, group, avg_bits, batch), s);
  if (rc) return rc;
  SLIM_CUDA(launch_dequant_gemv(codes, bits, scale, zero, m, n, group, avg_bits, x, xdtype, (int)batch, y, w.p, s));
  return SLIM_OK;
}

// ------------------------------------------------------------------ whole layer
size_t slim_workspace_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group, int avg_bits) {
  (void)avg_bits;
  if (check_shape(m, n, N, xdtype, group)) return 0;
  return layer_ws(m, n, N, xdtype, group).total;
}

int slim_quantize_layer_opts(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                             int avg_bits, double lambda, int n_tau, uint32_t* codes, float* scale, float* zero,
                             uint8_t* bits, void* ws, size_t ws_bytes, void* stream, const slim_options* opt,
                             slim_diag* diag) {
  if (!W || !X || !codes || !scale || !zero || !bits || !aligned16(W) || !aligned16(X)) return SLIM_EINVAL;
  int rc = check_shape(m, n, N, xdtype, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  if (!(lambda >= 0.0 && lambda < 1.0) || n_tau < 1 || n_tau > 256) return SLIM_EINVAL;
  const int objective = opt ? opt->objective : SLIM_OBJ_KL;
  const int precision = opt ? opt->sba_precision : SLIM_SBA_ADAPTIVE;
  const int32_t* given_order = opt ? opt->order : nullptr;
  if (objective != SLIM_OBJ_KL && objective != SLIM_OBJ_MSE) return SLIM_EINVAL;
  if (precision != SLIM_SBA_ADAPTIVE && precision != SLIM_SBA_FULL) return SLIM_EINVAL;
  const bool gptq = opt && opt->gptq != 0;
  if (opt && opt->gptq != 0 && opt->gptq != 1) return SLIM_EINVAL;
  if (gptq && m > (int64_t)65535 * 64) return SLIM_EINVAL;
  int sms = 0;
  rc = device_sms(&sms);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const LayerWs L = layer_ws(m, n, N, xdtype, group);
  Workspace w;
  rc = w.acquire(ws, ws_bytes, L.total, s);
  if (rc) return rc;
  DevStatus* st = reinterpret_cast<DevStatus*>(w.p);
  double* H = (diag && diag->H) ? diag->H : reinterpret_cast<double*>(w.p + L.off_H);
  double* h = (diag && diag->h) ? diag->h : reinterpret_cast<double*>(w.p + L.off_h);
  double* S = (diag && diag->S) ? diag->S : reinterpret_cast<double*>(w.p + L.off_S);
  int32_t* order = (diag && diag->order) ? diag->order : reinterpret_cast<int32_t*>(w.p + L.off_order);
  double* kl = (diag && diag->kl) ? diag->kl : reinterpret_cast<double*>(w.p + L.off_kl);
  int32_t* pstar = reinterpret_cast<int32_t*>(w.p + L.off_pstar);
  uint8_t* tau = diag ? diag->tau_idx : nullptr;
  uint8_t* scratch = w.p + L.off_scratch;
  uint8_t* rest = w.p + L.off_rest;
  HostCopy* side = host_copy(0);
  if (!side || !side->ok) return SLIM_ECUDA;
  JoinOnExit join{s, side->ps, side->pe[1]};

  cudaEvent_t ev[10] = {};
  const bool timed = diag != nullptr;
  if (timed)
    for (auto& e : ev) SLIM_CUDA(cudaEventCreate(&e));
  cudaEvent_t* kev_h = timed ? ev + 6 : nullptr;
  cudaEvent_t* kev_s = timed ? ev + 8 : nullptr;
  auto rec = [&](int i) { if (timed) cudaEventRecord(ev[i], s); };
  auto run = [&]() -> int {
    SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
    rec(0);
    if (injected("hessian")) return SLIM_EINJECTED;
    SLIM_CUDA(launch_hessian(X, xdtype, N, n, H, rest, st, sms, s, kev_h));
    rec(1);
    // beside the latency-bound inverse, at most 16K registers per SM (one
    // weight-operand block or two conversion blocks), so that a factorization
    // CTA (about 47K) still fits on every SM
    SLIM_CUDA(fork_prepare(*side, W, m, n, X, xdtype, N, group, avg_bits, scratch, st, sms, 1, 2, s));
    if (injected("hinv_diag")) return SLIM_EINJECTED;
    SLIM_CUDA(launch_hinv(H, n, kDampAlpha, h, reinterpret_cast<double*>(rest), st, s));
    rec(2);
    if (injected("salience")) return SLIM_EINJECTED;
    SLIM_CUDA(launch_salience(W, m, n, h, group, S, order, reinterpret_cast<double*>(rest), s));
    // a caller's group order replaces the salience order (checked: a
    // permutation of 0..k-1, else SLIM_EINVAL and the identity is used)
    if (given_order) SLIM_CUDA(launch_order_check(given_order, (int)(n / group), order, st, s));
    rec(3);
    if (injected("sba_search")) return SLIM_EINJECTED;
    SLIM_CUDA(join_prepare(*side, s));
    SLIM_CUDA(launch_sba_select(W, X, m, n, N, xdtype, group, precision, scratch, rest, s));
    SLIM_CUDA(launch_sba_search(m, n, xdtype, N, group, avg_bits, order, objective, kl, pstar, bits, scratch, rest,
                                st, sms, s, kev_s));
    if (diag && diag->sba_split) {
      int nbox = 0;
      const size_t off = sba_split_offset(m, n, N, xdtype, group, &nbox);
      SLIM_CUDA(cudaMemcpyAsync(diag->sba_split, scratch + off, (size_t)nbox, cudaMemcpyDeviceToDevice, s));
    }
    rec(4);
    if (injected("sqc")) return SLIM_EINJECTED;
    if (gptq) {
      // the GPTQ column loop with SBA's bits and SQC's quantizer, in place of SQC
      // on the unchanged weights (the diagonal it derives, behind its scratch)
      double* gws = reinterpret_cast<double*>(rest);
      double* gh = gws + gptq_workspace_doubles(m, n);
      SLIM_CUDA(launch_gptq(W, m, n, H, kDampAlpha, bits, group, avg_bits, lambda, n_tau, codes, scale, zero, tau, gh,
                            gws, st, sms, s));
    } else {
      SLIM_CUDA(launch_sqc(W, m, n, h, bits, group, avg_bits, lambda, n_tau, codes, scale, zero, tau, sms, s));
    }
    rec(5);
    return finish(s, st);
  };
  rc = run();
  if (timed) {
    cudaStreamSynchronize(s);
    if (rc == SLIM_OK) {
      for (int i = 0; i < 5; ++i) cudaEventElapsedTime(&diag->stage_ms[i], ev[i], ev[i + 1]);
      cudaEventElapsedTime(&diag->stage_ms[5], ev[0], ev[5]);
      diag->stage_ms[6] = diag->stage_ms[7] = 0.f;
      if (xdtype == SLIM_X_BF16) cudaEventElapsedTime(&diag->stage_ms[6], ev[6], ev[7]);
      cudaEventElapsedTime(&diag->stage_ms[7], ev[8], ev[9]);
      int32_t ps = -1;
      cudaMemcpy(&ps, pstar, sizeof(ps), cudaMemcpyDeviceToHost);
      diag->p_star = ps;
    }
    for (auto& e : ev) cudaEventDestroy(e);
  }
  return rc;
}

int slim_quantize_layer_ex(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                           int avg_bits, double lambda, int n_tau, uint32_t* codes, float* scale, float* zero,
                           uint8_t* bits, void* ws, size_t ws_bytes, void* stream, slim_diag* diag) {
  return slim_quantize_layer_opts(W, m, n, X, xdtype, N, group, avg_bits, lambda, n_tau, codes, scale, zero, bits, ws,
                                  ws_bytes, stream, nullptr, diag);
}

int slim_quantize_layer(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                        int avg_bits, double lambda, int n_tau, uint32_t* codes, float* scale, float* zero,
                        uint8_t* bits, void* ws, size_t ws_bytes, void* stream) {
  return slim_quantize_layer_ex(W, m, n, X, xdtype, N, group, avg_bits, lambda, n_tau, codes, scale, zero, bits,
                                ws, ws_bytes, stream, nullptr);
}

int slim_quantize_layer_host(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N,
                             int group, int avg_bits, double lambda, int n_tau, uint32_t* codes, float* scale,
                             float* zero, uint8_t* bits, void* stream) {
  if (!W || !X || !codes || !scale || !zero || !bits) return SLIM_EINVAL;
  int rc = check_shape(m, n, N, xdtype, group);
  if (rc) return rc;
  rc = check_bits(avg_bits);
  if (rc) return rc;
  if (!(lambda >= 0.0 && lambda < 1.0) || n_tau < 1 || n_tau > 256) return SLIM_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t k = n / group;
  const size_t wb = (size_t)m * n * 4, xb = (size_t)N * n * (xdtype == SLIM_X_BF16 ? 2 : 4);
  const size_t cb = (size_t)m * slim_row_words(n, avg_bits) * 4, sb = (size_t)m * k * 4;
  const LayerWs L = layer_ws(m, n, N, xdtype, group);
  size_t off = 0;
  const size_t o_w = off; off = al256(off + wb);
  const size_t o_x = off; off = al256(off + xb);
  const size_t o_c = off; off = al256(off + cb);
  const size_t o_s = off; off = al256(off + sb);
  const size_t o_z = off; off = al256(off + sb);
  const size_t o_b = off; off = al256(off + (size_t)k);
  const size_t o_ws = off; off = al256(off + L.total);
  // bf16 X: the SBA search runs split (below), with its partials and the
  // phase-A TMEM state in regions of their own
  const bool split = xdtype == SLIM_X_BF16;
  const size_t o_sw = off; off = split ? al256(off + sba_search_bytes(m, n, N, xdtype, group)) : off;
  const size_t o_yd = off; off = split ? al256(off + sba_yd_bytes(m, n, N, xdtype, group)) : off;
  Workspace w;
  rc = w.acquire(nullptr, 0, off, s);
  if (rc) return rc;
  const float* dW = reinterpret_cast<const float*>(w.p + o_w);
  uint8_t* dX = w.p + o_x;
  uint32_t* dcodes = reinterpret_cast<uint32_t*>(w.p + o_c);
  float* dscale = reinterpret_cast<float*>(w.p + o_s);
  float* dzero = reinterpret_cast<float*>(w.p + o_z);
  uint8_t* dbits = w.p + o_b;
  SLIM_CUDA(cudaMemcpyAsync(w.p + o_w, W, wb, cudaMemcpyHostToDevice, s));
  if (xdtype != SLIM_X_BF16) {
    SLIM_CUDA(cudaMemcpyAsync(dX, X, xb, cudaMemcpyHostToDevice, s));
    rc = slim_quantize_layer(dW, m, n, dX, xdtype, N, group, avg_bits, lambda, n_tau, dcodes, dscale, dzero, dbits,
                             w.p + o_ws, L.total, stream);
    if (rc) return rc;
  } else {
    // bf16 X: copied in chunks of whole Hessian token slices on a copy stream;
    // each chunk's slices of H = 2 X^T X are accumulated as soon as it lands,
    // so the tensor-core SYRK runs under the transfer. So does, on the side
    // stream, the part of the SBA search that does not depend on the salience
    // order: each chunk's fp16 copy and its phase A (y = X W^T and the
    // base-allocation d over the whole input width). After the inverse
    // Hessian and the salience order, the candidate steps continue from the
    // stored phase-A state.
    int sms = 0;
    rc = device_sms(&sms);
    if (rc) return rc;
    uint8_t* lw = w.p + o_ws;
    DevStatus* st = reinterpret_cast<DevStatus*>(lw);
    double* H = reinterpret_cast<double*>(lw + L.off_H);
    double* h = reinterpret_cast<double*>(lw + L.off_h);
    double* S = reinterpret_cast<double*>(lw + L.off_S);
    int32_t* order = reinterpret_cast<int32_t*>(lw + L.off_order);
    double* kl = reinterpret_cast<double*>(lw + L.off_kl);
    int32_t* pstar = reinterpret_cast<int32_t*>(lw + L.off_pstar);
    uint8_t* scratch = lw + L.off_scratch;
    uint8_t* rest = lw + L.off_rest;
    uint8_t* sw = w.p + o_sw;
    float* yd = reinterpret_cast<float*>(w.p + o_yd);
    const int64_t stok = hessian_slice_tokens();
    const int nsl = (int)((N + stok - 1) / stok);
    const int per = (nsl + 63) / 64;               // slices per chunk: at most 64 chunks
    const int nch = (nsl + per - 1) / per;
    HostCopy* hcp = host_copy(nch + 1);
    if (!hcp || !hcp->ok) return SLIM_ECUDA;
    HostCopy& hc = *hcp;
    SLIM_CUDA(cudaMemsetAsync(st, 0, kStatusBytes, s));
    SLIM_CUDA(cudaEventRecord(hc.ev[nch], s));          // the workspace exists before the copies start
    SLIM_CUDA(cudaStreamWaitEvent(hc.cs, hc.ev[nch], 0));
    const size_t row_bytes = (size_t)n * 2;
    // on every return from here, the caller's stream first waits for the
    // copies and the operand preparation, so the workspace is never released
    // under work still in flight
    JoinOnExit join{s, hc.cs, hc.ev[nch]}, join_prep{s, hc.ps, hc.pe[1]};
    for (int c = 0; c < nch; ++c) {
      const int64_t r0 = (int64_t)c * per * stok;
      const int64_t r1 = (r0 + (int64_t)per * stok < N) ? r0 + (int64_t)per * stok : N;
      SLIM_CUDA(cudaMemcpyAsync(dX + r0 * row_bytes, static_cast<const uint8_t*>(X) + r0 * row_bytes,
                                (size_t)(r1 - r0) * row_bytes, cudaMemcpyHostToDevice, hc.cs));
      SLIM_CUDA(cudaEventRecord(hc.ev[c], hc.cs));
    }
    // W (copied on s above) is resident: its operands are prepared on the
    // side stream, then each chunk of X is converted there as it lands
    SLIM_CUDA(fork_prepare(hc, dW, m, n, nullptr, xdtype, N, group, avg_bits, scratch, st, sms, 2, 2, s));
    if (injected("hessian")) return SLIM_EINJECTED;
    for (int c = 0; c < nch; ++c) {
      const int64_t r0 = (int64_t)c * per * stok;
      const int64_t r1 = (r0 + (int64_t)per * stok < N) ? r0 + (int64_t)per * stok : N;
      SLIM_CUDA(cudaStreamWaitEvent(s, hc.ev[c], 0));
      const int s0 = c * per, cnt = (s0 + per < nsl) ? per : nsl - s0;
      SLIM_CUDA(launch_hessian_slices(dX, N, n, rest, st, sms, s, s0, cnt));
      SLIM_CUDA(cudaStreamWaitEvent(hc.ps, hc.ev[c], 0));
      // the first chunk holds the token sample of the split selection (a chunk
      // is at least one 16384-token slice)
      if (c == 0) SLIM_CUDA(launch_sba_select(dW, dX, m, n, N, xdtype, group, SLIM_SBA_ADAPTIVE, scratch, sw, hc.ps));
      SLIM_CUDA(launch_sba_prep_x(dX, m, n, N, xdtype, group, r0, r1, scratch, st, sms, 2, hc.ps));
      // chunk boundaries are multiples of the slice length, so of 256 tokens:
      // no pair of 128-token tiles straddles two chunks
      SLIM_CUDA(launch_sba_phase_a(m, n, xdtype, N, group, SLIM_OBJ_KL, (int)(r0 / 256), (int)((r1 + 255) / 256),
                                   scratch, sw, yd, st, sms, hc.ps));
    }
    SLIM_CUDA(launch_hessian_reduce(N, n, rest, H, s));
    if (injected("hinv_diag")) return SLIM_EINJECTED;
    SLIM_CUDA(launch_hinv(H, n, kDampAlpha, h, reinterpret_cast<double*>(rest), st, s));
    if (injected("salience")) return SLIM_EINJECTED;
    SLIM_CUDA(launch_salience(dW, m, n, h, group, S, order, reinterpret_cast<double*>(rest), s));
    if (injected("sba_search")) return SLIM_EINJECTED;
    SLIM_CUDA(join_prepare(hc, s));
    SLIM_CUDA(launch_sba_steps(m, n, xdtype, N, group, avg_bits, order, SLIM_OBJ_KL, kl, pstar, dbits, scratch, sw, yd,
                               st, sms, s));
    if (injected("sqc")) return SLIM_EINJECTED;
    SLIM_CUDA(launch_sqc(dW, m, n, h, dbits, group, avg_bits, lambda, n_tau, dcodes, dscale, dzero, nullptr, sms, s));
    rc = finish(s, st);
    if (rc) return rc;
  }
  SLIM_CUDA(cudaMemcpyAsync(codes, dcodes, cb, cudaMemcpyDeviceToHost, s));
  SLIM_CUDA(cudaMemcpyAsync(scale, dscale, sb, cudaMemcpyDeviceToHost, s));
  SLIM_CUDA(cudaMemcpyAsync(zero, dzero, sb, cudaMemcpyDeviceToHost, s));
  SLIM_CUDA(cudaMemcpyAsync(bits, dbits, (size_t)k, cudaMemcpyDeviceToHost, s));
  SLIM_CUDA(cudaStreamSynchronize(s));
  return SLIM_OK;
}

}  // extern "C"
