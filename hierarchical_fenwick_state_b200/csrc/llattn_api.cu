// Host side of the C ABI declared in include/llattn.h: argument validation,
// workspace management, path dispatch and the device status word.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/llattn.h"
#include "llattn_bwd.h"
#include "llattn_decode.h"
#include "llattn_gdn.h"
#include "llattn_internal.h"

// Per-device status word: kernels OR LLATTN_DEV_* bits into it.
__device__ unsigned int g_llattn_status;

namespace {

thread_local int t_last_cuda = 0;

constexpr int kMaxDevices = 64;

struct DeviceState {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  unsigned int* status = nullptr;
  void* stage = nullptr;  // llattn_fwd_host staging (inputs, output, cu_seqlens)
  size_t stage_bytes = 0;
  cudaStream_t s_in = nullptr, s_out = nullptr;   // llattn_fwd_host copy streams
  std::vector<cudaEvent_t> ev;                    // llattn_fwd_host ordering events
};

std::mutex g_mu;
std::mutex g_host_mu;
std::mutex g_status_mu;   // lazy per-device lookup of the status word's address
DeviceState g_dev[kMaxDevices];

llattn_status cuda_fail(cudaError_t e) {
  t_last_cuda = static_cast<int>(e);
  return LLATTN_ERR_CUDA;
}

size_t round_up_host(size_t x) { return (x + 255) / 256 * 256; }

bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int default_chunk(int path, int T) {
  if (path == LLATTN_PATH_TCGEN05 || path == LLATTN_PATH_TCGEN05_SERIAL) return 128;
  return T <= 256 ? 16 : 64;
}

// Resolve AUTO, the chunk length, and check that the chosen path takes the shape.
llattn_status resolve(int in_dtype, int* path, int* chunk, int T, int dk, int dv) {
  if (in_dtype != LLATTN_F32 && in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
  if (*path < LLATTN_PATH_AUTO || *path > LLATTN_PATH_TCGEN05_SERIAL) return LLATTN_ERR_ARG;
  if (*path == LLATTN_PATH_AUTO) {
    const int c = *chunk ? *chunk : default_chunk(LLATTN_PATH_TCGEN05, T);
    *path = (in_dtype == LLATTN_BF16 && llattn::tc_supports(in_dtype, dk, dv, c, T))
                ? LLATTN_PATH_TCGEN05 : LLATTN_PATH_SIMT;
  }
  if (*chunk == 0) *chunk = default_chunk(*path, T);
  if (!pow2(*chunk)) return LLATTN_ERR_ARG;
  if (*path == LLATTN_PATH_SIMT) {
    if (*chunk < 8 || *chunk > 64) return LLATTN_ERR_ARG;
  } else {
    if (in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
    const bool ok = *path == LLATTN_PATH_TCGEN05_SERIAL
                        ? llattn::tc_serial_supports(in_dtype, dk, dv, *chunk, T)
                        : llattn::tc_supports(in_dtype, dk, dv, *chunk, T);
    if (!ok) return LLATTN_ERR_UNSUPPORTED;
  }
  return LLATTN_OK;
}

size_t workspace_for(int path, int chunk, int nseq, int H, int T, int dk, int dv, bool varlen) {
  if (path == LLATTN_PATH_SIMT) return llattn::simt_workspace_bytes(nseq, H, T, dk, dv, chunk);
  return llattn::tc_workspace_bytes(nseq, H, T, dk, dv, chunk, varlen);
}

llattn_status device_state(DeviceState** out, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return LLATTN_ERR_ARG;
  DeviceState& d = g_dev[dev];
  {
    // first calls from several host threads look the address up once, under a lock
    std::lock_guard<std::mutex> hold(g_status_mu);
    if (d.status == nullptr) {
      unsigned int* addr = nullptr;
      e = cudaGetSymbolAddress(reinterpret_cast<void**>(&addr), g_llattn_status);
      if (e != cudaSuccess) return cuda_fail(e);
      d.status = addr;
    }
  }
  *out = &d;
  *dev_out = dev;
  return LLATTN_OK;
}

// The scratch of one call: the caller's workspace (checked for size and alignment), or the
// library's per-device buffer, grown on demand under `lock`, which stays held for the launch.
llattn_status pick_workspace(DeviceState* ds, size_t need, void* workspace, size_t workspace_bytes,
                             std::unique_lock<std::mutex>& lock, void** ws) {
  *ws = workspace;
  if (workspace != nullptr) {
    if (workspace_bytes < need || !aligned(workspace, 256)) return LLATTN_ERR_WORKSPACE;
  } else if (need > 0) {
    lock.lock();
    if (ds->ws_bytes < need) {
      cudaError_t e;
      if (ds->ws) {
        if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e);
        cudaFree(ds->ws);
        ds->ws = nullptr;
        ds->ws_bytes = 0;
      }
      if ((e = cudaMalloc(&ds->ws, need)) != cudaSuccess) {
        ds->ws = nullptr;
        return cuda_fail(e);
      }
      ds->ws_bytes = need;
    }
    *ws = ds->ws;
  }
  return LLATTN_OK;
}

llattn_status forward(int in_dtype, int path, int chunk, const void* q, const void* k,
                      const void* v, const float* log_a, const float* lam, float* out, int B,
                      int H, int T, int dk, int dv, const int* cu_seqlens, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (B < 0 || H < 0 || T < 0) return LLATTN_ERR_SHAPE;
  if (!head_dim_ok(dk) || !head_dim_ok(dv)) return LLATTN_ERR_SHAPE;
  if (T > (1 << 24) || H > 65535 || B > 65535) return LLATTN_ERR_SHAPE;
  // the automatic choice with the default chunk takes the one-launch CUDA-core kernel for short
  // sequences where the tensor cores do not apply (a path or chunk the caller names is kept)
  const bool auto_default = path == LLATTN_PATH_AUTO && chunk == 0;
  llattn_status s = resolve(in_dtype, &path, &chunk, T, dk, dv);
  if (s != LLATTN_OK) return s;
  const bool short_path = auto_default && path == LLATTN_PATH_SIMT &&
                          llattn::simt_short_supports(T, llattn_num_levels(T));
  if (B == 0 || H == 0 || T == 0) return LLATTN_OK;  // nothing to compute
  if (!q || !k || !v || !log_a || !lam || !out) return LLATTN_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(log_a, 4) || !aligned(lam, 4) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return LLATTN_ERR_ALIGN;
  const void* ins[5] = {q, k, v, log_a, lam};
  for (const void* p : ins)
    if (p == static_cast<const void*>(out)) return LLATTN_ERR_ARG;
  const int L = llattn_num_levels(T);
  if (cu_seqlens == nullptr) {
    // dense: the whole output range must not overlap any input range
    const unsigned long long ntok = (unsigned long long)B * T;
    if (ntok * H * (unsigned long long)(dk > dv ? dk : dv) > (1ull << 40)) return LLATTN_ERR_SHAPE;
    const size_t esz = in_dtype == LLATTN_BF16 ? 2 : 4;
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out);
    const uintptr_t o1 = o0 + ntok * H * dv * sizeof(float);
    const struct { const void* p; size_t n; } rng[5] = {
        {q, ntok * H * dk * esz}, {k, ntok * H * dk * esz}, {v, ntok * H * dv * esz},
        {log_a, ntok * H * sizeof(float)}, {lam, ntok * H * L * sizeof(float)}};
    for (const auto& r : rng) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(r.p), a1 = a0 + r.n;
      if (a0 < o1 && o0 < a1) return LLATTN_ERR_ARG;
    }
  }
  DeviceState* ds = nullptr;
  int dev = 0;
  if ((s = device_state(&ds, &dev)) != LLATTN_OK) return s;
  const size_t need =
      short_path ? 0 : workspace_for(path, chunk, B, H, T, dk, dv, cu_seqlens != nullptr);
  void* ws = workspace;
  std::unique_lock<std::mutex> lock(g_mu, std::defer_lock);
  if ((s = pick_workspace(ds, need, workspace, workspace_bytes, lock, &ws)) != LLATTN_OK) return s;
  llattn::Problem p{in_dtype, q, k, v, log_a, lam, out, B, H, T, dk, dv, L, cu_seqlens,
                    ds->status};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = short_path ? llattn::simt_short_forward(p, st)
                  : path == LLATTN_PATH_SIMT
                      ? llattn::simt_forward(p, chunk, ws, st)
                      : llattn::tc_forward(p, chunk, ws, st, path == LLATTN_PATH_TCGEN05_SERIAL);
  if (e != cudaSuccess) return cuda_fail(e);
  return LLATTN_OK;
}

// ---- launch accounting ----
std::atomic<long long> g_total_launches{0};
std::atomic<bool> g_profiling{false};
std::mutex g_prof_mu;
struct EvPair { cudaEvent_t a, b; };
std::vector<EvPair> g_prof_events;   // recorded pairs not yet read
std::vector<cudaEvent_t> g_event_pool;
thread_local cudaEvent_t t_open_event = nullptr;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

namespace llattn {

void count_launch(int n) { g_total_launches.fetch_add(n); }

void main_kernel_begin(cudaStream_t st) {
  if (!g_profiling.load()) return;
  std::lock_guard<std::mutex> g(g_prof_mu);
  t_open_event = pool_event();
  if (t_open_event) cudaEventRecord(t_open_event, st);
}

void main_kernel_end(cudaStream_t st) {
  if (!g_profiling.load() || t_open_event == nullptr) return;
  std::lock_guard<std::mutex> g(g_prof_mu);
  cudaEvent_t b = pool_event();
  if (b == nullptr) return;
  cudaEventRecord(b, st);
  g_prof_events.push_back({t_open_event, b});
  t_open_event = nullptr;
}

}  // namespace llattn

extern "C" {

llattn_status llattn_profile(int enable) {
  g_profiling.store(enable != 0);
  return LLATTN_OK;
}

llattn_status llattn_profile_read(double* main_kernel_ms, long long* main_launches,
                                  long long* total_launches, int reset) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  double ms = 0.0;
  for (const EvPair& p : g_prof_events) {
    cudaError_t e = cudaEventSynchronize(p.b);
    if (e != cudaSuccess) return cuda_fail(e);
    float x = 0.f;
    if ((e = cudaEventElapsedTime(&x, p.a, p.b)) != cudaSuccess) return cuda_fail(e);
    ms += x;
  }
  if (main_kernel_ms) *main_kernel_ms = ms;
  if (main_launches) *main_launches = (long long)g_prof_events.size();
  if (total_launches) *total_launches = g_total_launches.load();
  if (reset) {
    for (const EvPair& p : g_prof_events) {
      g_event_pool.push_back(p.a);
      g_event_pool.push_back(p.b);
    }
    g_prof_events.clear();
    g_total_launches.store(0);
  }
  return LLATTN_OK;
}


int llattn_abi_version(void) { return 1; }

const char* llattn_status_str(llattn_status s) {
  switch (s) {
    case LLATTN_OK: return "ok";
    case LLATTN_ERR_ARG: return "invalid argument";
    case LLATTN_ERR_SHAPE: return "unsupported or out-of-range shape";
    case LLATTN_ERR_ALIGN: return "misaligned pointer";
    case LLATTN_ERR_DTYPE: return "unsupported dtype";
    case LLATTN_ERR_CUDA: return "CUDA error";
    case LLATTN_ERR_TIMEOUT: return "device-side wait timed out";
    case LLATTN_ERR_WORKSPACE: return "workspace too small or misaligned";
    case LLATTN_ERR_UNSUPPORTED: return "no kernel for this configuration";
    case LLATTN_ERR_NOALLOC_LIMIT:
      return "problem needs more scratch than llattn_fwd_noalloc's fixed array holds";
  }
  return "unknown status";
}

int llattn_num_levels(int T) {
  if (T <= 1) return 1;
  int bits = 0;
  unsigned x = static_cast<unsigned>(T - 1);
  while (x) { ++bits; x >>= 1; }
  return 1 + bits;
}

llattn_status llattn_workspace_bytes(int in_dtype, int path, int chunk, int B, int H, int T,
                                     int dk, int dv, int varlen, size_t* bytes) {
  if (!bytes) return LLATTN_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || T > (1 << 24)) return LLATTN_ERR_SHAPE;
  if (!head_dim_ok(dk) || !head_dim_ok(dv)) return LLATTN_ERR_SHAPE;
  llattn_status s = resolve(in_dtype, &path, &chunk, T, dk, dv);
  if (s != LLATTN_OK) return s;
  *bytes = (B == 0 || H == 0 || T == 0) ? 0 : workspace_for(path, chunk, B, H, T, dk, dv, varlen != 0);
  return LLATTN_OK;
}

llattn_status llattn_fwd(const void* q, const void* k, const void* v, const float* log_a,
                         const float* lam, float* out, int B, int H, int T, int dk, int dv,
                         const int* cu_seqlens, void* stream) {
  return forward(LLATTN_BF16, LLATTN_PATH_AUTO, 0, q, k, v, log_a, lam, out, B, H, T, dk, dv,
                 cu_seqlens, nullptr, 0, stream);
}

llattn_status llattn_fwd_bf16(const void* q, const void* k, const void* v, const float* log_a,
                              const float* lam, float* out, int B, int H, int T, int dk, int dv,
                              const int* cu_seqlens, void* stream) {
  return llattn_fwd(q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens, stream);
}

llattn_status llattn_fwd_f32(const float* q, const float* k, const float* v, const float* log_a,
                             const float* lam, float* out, int B, int H, int T, int dk, int dv,
                             const int* cu_seqlens, void* stream) {
  return forward(LLATTN_F32, LLATTN_PATH_AUTO, 0, q, k, v, log_a, lam, out, B, H, T, dk, dv,
                 cu_seqlens, nullptr, 0, stream);
}

llattn_status llattn_fwd_ex(int in_dtype, int path, int chunk, const void* q, const void* k,
                            const void* v, const float* log_a, const float* lam, float* out,
                            int B, int H, int T, int dk, int dv, const int* cu_seqlens,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return forward(in_dtype, path, chunk, q, k, v, log_a, lam, out, B, H, T, dk, dv, cu_seqlens,
                 workspace, workspace_bytes, stream);
}

llattn_status llattn_fwd_noalloc(int in_dtype, const void* q, const void* k, const void* v,
                                 const float* log_a, const float* lam, float* out, int B, int H,
                                 int T, int dk, int dv, const int* cu_seqlens, void* stream) {
  // Size check first: it needs no device, and a rejected call touches nothing.
  size_t need = 0;
  llattn_status s = llattn_workspace_bytes(in_dtype, LLATTN_PATH_SIMT, 0, B, H, T, dk, dv,
                                           cu_seqlens != nullptr, &need);
  if (s != LLATTN_OK) return s;
  if (need > LLATTN_NOALLOC_SCRATCH_BYTES) return LLATTN_ERR_NOALLOC_LIMIT;
  if (need == 0)  // empty problem: nothing is launched and no scratch is used
    return forward(in_dtype, LLATTN_PATH_SIMT, 0, q, k, v, log_a, lam, out, B, H, T, dk, dv,
                   cu_seqlens, nullptr, 0, stream);
  void* scratch = nullptr;
  cudaError_t e = llattn::noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  // A caller-supplied workspace never reaches the library's allocator.
  return forward(in_dtype, LLATTN_PATH_SIMT, 0, q, k, v, log_a, lam, out, B, H, T, dk, dv,
                 cu_seqlens, scratch, LLATTN_NOALLOC_SCRATCH_BYTES, stream);
}

llattn_status llattn_device_status(unsigned int* flags, int clear) {
  if (!flags) return LLATTN_ERR_ARG;
  DeviceState* ds = nullptr;
  int dev = 0;
  llattn_status s = device_state(&ds, &dev);
  if (s != LLATTN_OK) return s;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int v = 0;
  if ((e = cudaMemcpy(&v, ds->status, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e);
  if (clear && v) {
    if ((e = cudaMemset(ds->status, 0, sizeof(v))) != cudaSuccess) return cuda_fail(e);
  }
  *flags = v;
  return (v & LLATTN_DEV_WAIT_TIMEOUT) ? LLATTN_ERR_TIMEOUT : LLATTN_OK;
}

llattn_status llattn_gdn_fwd(int in_dtype, const void* q, const void* k, const void* v,
                            const float* log_alpha, const float* beta, const float* lam,
                            float* out, int B, int H, int T, int dk, int dv,
                            const int* cu_seqlens, void* stream) {
  if (in_dtype != LLATTN_F32 && in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
  if (B < 0 || H < 0 || T < 0 || H > 65535 || B > 65535) return LLATTN_ERR_SHAPE;
  if (!head_dim_ok(dk) || !head_dim_ok(dv) || !llattn::gdn_supports(dk, dv, T))
    return LLATTN_ERR_SHAPE;
  if (B == 0 || H == 0 || T == 0) return LLATTN_OK;
  if (!q || !k || !v || !log_alpha || !beta || !lam || !out) return LLATTN_ERR_ARG;
  if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(out, 4) ||
      !aligned(log_alpha, 4) || !aligned(beta, 4) || !aligned(lam, 4) ||
      (cu_seqlens && !aligned(cu_seqlens, 4)))
    return LLATTN_ERR_ALIGN;
  const void* ins[6] = {q, k, v, log_alpha, beta, lam};
  for (const void* p : ins)
    if (p == static_cast<const void*>(out)) return LLATTN_ERR_ARG;
  const int L = llattn_num_levels(T);
  if (cu_seqlens == nullptr) {
    const unsigned long long ntok = (unsigned long long)B * T;
    if (ntok * H * (unsigned long long)(dk > dv ? dk : dv) > (1ull << 40)) return LLATTN_ERR_SHAPE;
    const size_t esz = in_dtype == LLATTN_BF16 ? 2 : 4;
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out);
    const uintptr_t o1 = o0 + ntok * H * dv * sizeof(float);
    const struct { const void* p; size_t n; } rng[6] = {
        {q, ntok * H * dk * esz}, {k, ntok * H * dk * esz}, {v, ntok * H * dv * esz},
        {log_alpha, ntok * H * sizeof(float)}, {beta, ntok * H * sizeof(float)},
        {lam, ntok * H * L * sizeof(float)}};
    for (const auto& r : rng) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(r.p), a1 = a0 + r.n;
      if (a0 < o1 && o0 < a1) return LLATTN_ERR_ARG;
    }
  }
  DeviceState* ds = nullptr;
  int dev = 0;
  llattn_status s = device_state(&ds, &dev);
  if (s != LLATTN_OK) return s;
  llattn::GdnProblem p{in_dtype, q, k, v, log_alpha, beta, lam, out, B, H, T, dk, dv, L,
                       cu_seqlens, ds->status};
  const cudaError_t e = llattn::gdn_forward(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return LLATTN_OK;
}

llattn_status llattn_set_segment_chunks(int chunks) {
  if (chunks < 0 || chunks > (1 << 20) || (chunks > 0 && !pow2(chunks)) || chunks == 1)
    return LLATTN_ERR_ARG;
  llattn::tc_set_segment_chunks(chunks);
  return LLATTN_OK;
}

llattn_status llattn_segment_plan(int B, int H, int T, int dk, int dv, int varlen,
                                  int* chunks_per_segment) {
  if (!chunks_per_segment) return LLATTN_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || T > (1 << 24)) return LLATTN_ERR_SHAPE;
  if (!head_dim_ok(dk) || !head_dim_ok(dv)) return LLATTN_ERR_SHAPE;
  *chunks_per_segment = 0;
  if (B == 0 || H == 0 || T == 0 || !llattn::tc_supports(LLATTN_BF16, dk, dv, 128, T))
    return LLATTN_OK;
  *chunks_per_segment = llattn::tc_segment_chunks(B, H, T, dk, dv, varlen != 0);
  return LLATTN_OK;
}

llattn_status llattn_stream_status(unsigned int* flags, int clear, void* stream) {
  if (!flags) return LLATTN_ERR_ARG;
  DeviceState* ds = nullptr;
  int dev = 0;
  llattn_status s = device_state(&ds, &dev);
  if (s != LLATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // stream-ordered copy into a pageable word; the synchronise makes it complete
  unsigned int v = 0;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(&v, ds->status, sizeof(v), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(e);
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e);
  if (clear && v) {
    if ((e = cudaMemsetAsync(ds->status, 0, sizeof(unsigned int), st)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e);
  }
  *flags = v;
  return (v & LLATTN_DEV_WAIT_TIMEOUT) ? LLATTN_ERR_TIMEOUT : LLATTN_OK;
}

llattn_status llattn_fwd_host(int in_dtype, const void* q, const void* k, const void* v,
                              const float* log_a, const float* lam, float* out, int B, int H,
                              int T, int dk, int dv, const int* cu_seqlens, void* stream) {
  if (in_dtype != LLATTN_F32 && in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
  if (B < 0 || H < 0 || T < 0 || T > (1 << 24)) return LLATTN_ERR_SHAPE;
  if (!head_dim_ok(dk) || !head_dim_ok(dv)) return LLATTN_ERR_SHAPE;
  if (B == 0 || H == 0 || T == 0) return LLATTN_OK;
  if (!q || !k || !v || !log_a || !lam || !out) return LLATTN_ERR_ARG;
  long long total = (long long)B * T;
  if (cu_seqlens) {
    if (cu_seqlens[0] != 0) return LLATTN_ERR_ARG;
    for (int i = 0; i < B; ++i) {
      const int len = cu_seqlens[i + 1] - cu_seqlens[i];
      if (len < 0 || len > T) return LLATTN_ERR_SHAPE;
    }
    total = cu_seqlens[B];
  }
  if (total * H * (long long)(dk > dv ? dk : dv) > (1ll << 40)) return LLATTN_ERR_SHAPE;
  const int L = llattn_num_levels(T);
  const size_t esz = in_dtype == LLATTN_BF16 ? 2 : 4;
  const size_t nq = round_up_host((size_t)total * H * dk * esz);
  const size_t nv = round_up_host((size_t)total * H * dv * esz);
  const size_t na = round_up_host((size_t)total * H * sizeof(float));
  const size_t nl = round_up_host((size_t)total * H * L * sizeof(float));
  const size_t no = round_up_host((size_t)total * H * dv * sizeof(float));
  const size_t nc = round_up_host((size_t)(B + 1) * sizeof(int));
  const size_t need = 2 * nq + nv + na + nl + no + nc;
  std::lock_guard<std::mutex> hold(g_host_mu);
  DeviceState* ds = nullptr;
  int dev = 0;
  llattn_status s = device_state(&ds, &dev);
  if (s != LLATTN_OK) return s;
  cudaError_t e;
  if (ds->stage_bytes < need) {
    if (ds->stage) {
      if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e);
      cudaFree(ds->stage);
      ds->stage = nullptr;
      ds->stage_bytes = 0;
    }
    if ((e = cudaMalloc(&ds->stage, need)) != cudaSuccess) {
      ds->stage = nullptr;
      return cuda_fail(e);
    }
    ds->stage_bytes = need;
  }
  char* b = static_cast<char*>(ds->stage);
  char* dq = b; b += nq;
  char* dk_ = b; b += nq;
  char* dv_ = b; b += nv;
  float* da = reinterpret_cast<float*>(b); b += na;
  float* dl = reinterpret_cast<float*>(b); b += nl;
  float* dout = reinterpret_cast<float*>(b); b += no;
  int* dcu = cu_seqlens ? reinterpret_cast<int*>(b) : nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const struct { void* d; const void* h; size_t n; } cp[6] = {
      {dq, q, (size_t)total * H * dk * esz}, {dk_, k, (size_t)total * H * dk * esz},
      {dv_, v, (size_t)total * H * dv * esz}, {da, log_a, (size_t)total * H * sizeof(float)},
      {dl, lam, (size_t)total * H * L * sizeof(float)},
      {dcu, cu_seqlens, (size_t)(B + 1) * sizeof(int)}};
  if (cu_seqlens == nullptr && B >= 2) {
    // Dense batch: each batch row is a contiguous slice of every tensor and an independent
    // problem, so rows are pipelined - row b's upload (stream s_in), forward (the caller's
    // stream) and download (stream s_out) overlap the other rows' copies in both directions.
    if (ds->s_in == nullptr &&
        (e = cudaStreamCreateWithFlags(&ds->s_in, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e);
    if (ds->s_out == nullptr &&
        (e = cudaStreamCreateWithFlags(&ds->s_out, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e);
    const size_t nev = 2 * (size_t)B + 2;
    while (ds->ev.size() < nev) {
      cudaEvent_t x;
      if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail(e);
      ds->ev.push_back(x);
    }
    cudaEvent_t* ev = ds->ev.data();   // [0] start, [1] done, [2 + 2b] uploaded, [3 + 2b] computed
    // on a failure part-way, let the copies already queued finish before the staging memory
    // can be reused by another call
    auto drain = [&](llattn_status r) {
      cudaStreamSynchronize(ds->s_in);
      cudaStreamSynchronize(ds->s_out);
      cudaStreamSynchronize(st);
      return r;
    };
    const size_t rq = (size_t)T * H * dk * esz, rv = (size_t)T * H * dv * esz;
    const size_t ra = (size_t)T * H * sizeof(float), rl = (size_t)T * H * L * sizeof(float);
    const size_t ro = (size_t)T * H * dv * sizeof(float);
    if ((e = cudaEventRecord(ev[0], st)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ds->s_in, ev[0], 0)) != cudaSuccess)
      return drain(cuda_fail(e));
    const char* hq = static_cast<const char*>(q);
    const char* hk = static_cast<const char*>(k);
    const char* hv = static_cast<const char*>(v);
    const char* ha = reinterpret_cast<const char*>(log_a);
    const char* hl = reinterpret_cast<const char*>(lam);
    char* ho = reinterpret_cast<char*>(out);
    for (int r = 0; r < B; ++r) {
      const struct { char* d; const char* h; size_t n; } up[5] = {
          {dq + r * rq, hq + r * rq, rq}, {dk_ + r * rq, hk + r * rq, rq},
          {dv_ + r * rv, hv + r * rv, rv}, {reinterpret_cast<char*>(da) + r * ra, ha + r * ra, ra},
          {reinterpret_cast<char*>(dl) + r * rl, hl + r * rl, rl}};
      for (const auto& c : up)
        if ((e = cudaMemcpyAsync(c.d, c.h, c.n, cudaMemcpyHostToDevice, ds->s_in)) != cudaSuccess)
          return drain(cuda_fail(e));
      if ((e = cudaEventRecord(ev[2 + 2 * r], ds->s_in)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(st, ev[2 + 2 * r], 0)) != cudaSuccess)
        return drain(cuda_fail(e));
      s = forward(in_dtype, LLATTN_PATH_AUTO, 0, dq + r * rq, dk_ + r * rq, dv_ + r * rv,
                  reinterpret_cast<float*>(reinterpret_cast<char*>(da) + r * ra),
                  reinterpret_cast<float*>(reinterpret_cast<char*>(dl) + r * rl),
                  reinterpret_cast<float*>(reinterpret_cast<char*>(dout) + r * ro), 1, H, T, dk,
                  dv, nullptr, nullptr, 0, stream);
      if (s != LLATTN_OK) return drain(s);
      if ((e = cudaEventRecord(ev[3 + 2 * r], st)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(ds->s_out, ev[3 + 2 * r], 0)) != cudaSuccess ||
          (e = cudaMemcpyAsync(ho + r * ro, reinterpret_cast<char*>(dout) + r * ro, ro,
                               cudaMemcpyDeviceToHost, ds->s_out)) != cudaSuccess)
        return drain(cuda_fail(e));
    }
    if ((e = cudaEventRecord(ev[1], ds->s_out)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(st, ev[1], 0)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
      return drain(cuda_fail(e));
    return LLATTN_OK;
  }
  for (const auto& c : cp) {
    if (c.d == nullptr || c.n == 0) continue;
    if ((e = cudaMemcpyAsync(c.d, c.h, c.n, cudaMemcpyHostToDevice, st)) != cudaSuccess)
      return cuda_fail(e);
  }
  s = forward(in_dtype, LLATTN_PATH_AUTO, 0, dq, dk_, dv_, da, dl, dout, B, H, T, dk, dv, dcu,
              nullptr, 0, stream);
  if (s != LLATTN_OK) return s;
  if ((e = cudaMemcpyAsync(out, dout, (size_t)total * H * dv * sizeof(float),
                           cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(e);
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e);
  return LLATTN_OK;
}

llattn_status llattn_decode_state_bytes(int B, int H, int L, int dk, int dv, size_t* bytes) {
  if (!bytes) return LLATTN_ERR_ARG;
  if (B < 0 || H < 0 || B > 65535 || H > 65535 || L < 1 || L > 32) return LLATTN_ERR_SHAPE;
  if (!head_dim_ok(dk) || !head_dim_ok(dv)) return LLATTN_ERR_SHAPE;
  *bytes = llattn::decode_state_bytes(B, H, L, dk, dv);
  return LLATTN_OK;
}

llattn_status llattn_decode_step(int in_dtype, const void* q, const void* k, const void* v,
                                 const float* log_a, const float* lam, const int* pos,
                                 float* state, float* out, int B, int H, int L, int dk, int dv,
                                 void* stream) {
  if (in_dtype != LLATTN_F32 && in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
  size_t state_bytes = 0;
  llattn_status s = llattn_decode_state_bytes(B, H, L, dk, dv, &state_bytes);
  if (s != LLATTN_OK) return s;
  if (B == 0 || H == 0) return LLATTN_OK;  // nothing to compute
  if (!q || !k || !v || !log_a || !lam || !pos || !state || !out) return LLATTN_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(state, 16) ||
      !aligned(out, 16) || !aligned(log_a, 4) || !aligned(lam, 4) || !aligned(pos, 4))
    return LLATTN_ERR_ALIGN;
  // out must not overlap any input or the state
  const size_t bh = (size_t)B * H, esz = in_dtype == LLATTN_BF16 ? 2 : 4;
  const uintptr_t o0 = reinterpret_cast<uintptr_t>(out), o1 = o0 + bh * dv * sizeof(float);
  const struct { const void* p; size_t n; } rng[7] = {
      {q, bh * dk * esz}, {k, bh * dk * esz}, {v, bh * dv * esz}, {log_a, bh * sizeof(float)},
      {lam, bh * L * sizeof(float)}, {pos, (size_t)B * sizeof(int)}, {state, state_bytes}};
  for (const auto& r : rng) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(r.p), a1 = a0 + r.n;
    if (r.n && a0 < o1 && o0 < a1) return LLATTN_ERR_ARG;
  }
  DeviceState* ds = nullptr;
  int dev = 0;
  if ((s = device_state(&ds, &dev)) != LLATTN_OK) return s;
  const size_t nlev = bh * (size_t)(L - 1) * dk * dv;
  llattn::DecodeProblem p{in_dtype, q, k, v, log_a, lam, pos, state, state + nlev, out,
                          B, H, L, dk, dv, ds->status};
  const cudaError_t e = llattn::decode_step(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return LLATTN_OK;
}

llattn_status llattn_prefill_state(int in_dtype, const void* k, const void* v,
                                   const float* log_a, float* state, int B, int H, int T, int L,
                                   int dk, int dv, const int* cu_seqlens, void* stream) {
  if (in_dtype != LLATTN_F32 && in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
  size_t state_bytes = 0;
  llattn_status s = llattn_decode_state_bytes(B, H, L, dk, dv, &state_bytes);
  if (s != LLATTN_OK) return s;
  if (T < 0 || T > (1 << 24)) return LLATTN_ERR_SHAPE;
  if (B == 0 || H == 0) return LLATTN_OK;  // nothing to compute
  if (!state) return LLATTN_ERR_ARG;
  if (T > 0 && (!k || !v || !log_a)) return LLATTN_ERR_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(state, 16) || !aligned(log_a, 4) ||
      (cu_seqlens && !aligned(cu_seqlens, 4)))
    return LLATTN_ERR_ALIGN;
  if (cu_seqlens == nullptr) {   // dense: the inputs' extents are known here
    const size_t rows = (size_t)B * T * H, esz = in_dtype == LLATTN_BF16 ? 2 : 4;
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(state), s1 = s0 + state_bytes;
    const struct { const void* p; size_t n; } rng[3] = {
        {k, rows * dk * esz}, {v, rows * dv * esz}, {log_a, rows * sizeof(float)}};
    for (const auto& r : rng) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(r.p), a1 = a0 + r.n;
      if (r.n && a0 < s1 && s0 < a1) return LLATTN_ERR_ARG;
    }
  }
  DeviceState* ds = nullptr;
  int dev = 0;
  if ((s = device_state(&ds, &dev)) != LLATTN_OK) return s;
  const size_t nlev = (size_t)B * H * (size_t)(L - 1) * dk * dv;
  llattn::PrefillProblem p{in_dtype, k, v, log_a, state, state + nlev, B, H, T, L, dk, dv,
                           cu_seqlens, ds->status};
  const cudaError_t e = llattn::prefill_state(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return LLATTN_OK;
}

llattn_status llattn_bwd_workspace_bytes(int B, int H, int T, int dk, int dv, size_t* bytes) {
  if (!bytes) return LLATTN_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || T > (1 << 24) || H > 65535 || B > 65535) return LLATTN_ERR_SHAPE;
  if (dk != dv || (dk != 32 && dk != 64 && dk != 128)) return LLATTN_ERR_SHAPE;
  *bytes = (B == 0 || H == 0 || T == 0) ? 0 : llattn::bwd_workspace_bytes(B, H, T);
  return LLATTN_OK;
}

llattn_status llattn_bwd(int in_dtype, const void* q, const void* k, const void* v,
                         const float* log_a, const float* lam, const void* dout, float* dq,
                         float* dk, float* dv, float* dlog_a, float* dlam, int B, int H, int T,
                         int dk_dim, int dv_dim, const int* cu_seqlens, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (in_dtype != LLATTN_F32 && in_dtype != LLATTN_BF16) return LLATTN_ERR_DTYPE;
  size_t need = 0;
  llattn_status s = llattn_bwd_workspace_bytes(B, H, T, dk_dim, dv_dim, &need);
  if (s != LLATTN_OK) return s;
  if (B == 0 || H == 0 || T == 0) return LLATTN_OK;  // nothing to compute
  const void* ptrs[12] = {q, k, v, log_a, lam, dout, dq, dk, dv, dlog_a, dlam, nullptr};
  for (int i = 0; i < 11; ++i)
    if (ptrs[i] == nullptr) return LLATTN_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(log_a, 4) ||
      !aligned(lam, 4) || !aligned(dlog_a, 4) || !aligned(dlam, 4) ||
      (cu_seqlens && !aligned(cu_seqlens, 4)))
    return LLATTN_ERR_ALIGN;
  const int L = llattn_num_levels(T);
  if (cu_seqlens == nullptr) {
    // dense: no gradient may overlap an input or another gradient
    const size_t ntok = (size_t)B * T * H, d = (size_t)dk_dim;
    const size_t esz = in_dtype == LLATTN_BF16 ? 2 : 4;
    const struct { const void* p; size_t n; } rng[11] = {
        {q, ntok * d * esz}, {k, ntok * d * esz}, {v, ntok * d * esz}, {dout, ntok * d * esz},
        {log_a, ntok * 4}, {lam, ntok * L * 4}, {dq, ntok * d * 4}, {dk, ntok * d * 4},
        {dv, ntok * d * 4}, {dlog_a, ntok * 4}, {dlam, ntok * L * 4}};
    for (int o = 6; o < 11; ++o) {
      const uintptr_t o0 = reinterpret_cast<uintptr_t>(rng[o].p), o1 = o0 + rng[o].n;
      for (int i = 0; i < 11; ++i) {
        if (i == o) continue;
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(rng[i].p), a1 = a0 + rng[i].n;
        if (a0 < o1 && o0 < a1) return LLATTN_ERR_ARG;
      }
    }
  }
  DeviceState* ds = nullptr;
  int dev = 0;
  if ((s = device_state(&ds, &dev)) != LLATTN_OK) return s;
  void* ws = nullptr;
  std::unique_lock<std::mutex> lock(g_mu, std::defer_lock);
  if ((s = pick_workspace(ds, need, workspace, workspace_bytes, lock, &ws)) != LLATTN_OK) return s;
  llattn::BwdProblem p{in_dtype, q, k, v, dout, log_a, lam, dq, dk, dv, dlog_a, dlam,
                       B, H, T, dk_dim, L, cu_seqlens, ds->status};
  const cudaError_t e = llattn::bwd(p, ws, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return LLATTN_OK;
}

int llattn_last_cuda_error(void) { return t_last_cuda; }

}  // extern "C"
