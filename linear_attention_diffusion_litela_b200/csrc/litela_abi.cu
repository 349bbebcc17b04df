// C ABI of liblitela: argument validation, per-(device, stream) workspace, kernel launches.
// The operation, the layouts and the error behaviour are documented in include/litela.h.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/litela.h"
#include "litela_plan.h"
#include "litela_simt.cuh"

namespace litela {
namespace {

thread_local std::string g_last_error;

litela_status fail(litela_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

litela_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LITELA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// One workspace per (device, stream): partial/prefix states plus arrival counters that the
// kernels always leave at zero.
struct Workspace {
  void* states = nullptr;
  size_t states_bytes = 0;
  unsigned* counters = nullptr;
  size_t counters_len = 0;
};

std::mutex g_ws_mutex;
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;

// Test hook: LITELA_FAIL_ALLOC=1 makes every workspace allocation fail (host-side injection
// of an out-of-memory condition; nothing runs on the GPU).
bool alloc_fault_injected() {
  const char* v = std::getenv("LITELA_FAIL_ALLOC");
  return v != nullptr && v[0] == '1';
}

litela_status get_workspace(const Plan& plan, cudaStream_t stream, Workspace** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  Workspace& ws = g_ws[{dev, reinterpret_cast<uintptr_t>(stream)}];
  const bool grow_states = ws.states_bytes < plan.bytes;
  const bool grow_counters = ws.counters_len < plan.counters;
  if (grow_states || grow_counters) {
    if (alloc_fault_injected())
      return fail(LITELA_ERR_OUT_OF_MEMORY, "workspace allocation failed (injected by LITELA_FAIL_ALLOC)");
    // kernels of earlier calls on this stream may still use the old buffers
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize before workspace growth");
    if (grow_states) {
      if (ws.states) cudaFree(ws.states);
      ws.states = nullptr;
      ws.states_bytes = 0;
      e = cudaMalloc(&ws.states, plan.bytes);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(LITELA_ERR_OUT_OF_MEMORY, std::string("workspace cudaMalloc: ") + cudaGetErrorString(e));
      }
      ws.states_bytes = plan.bytes;
    }
    if (grow_counters) {
      if (ws.counters) cudaFree(ws.counters);
      ws.counters = nullptr;
      ws.counters_len = 0;
      e = cudaMalloc(&ws.counters, plan.counters * sizeof(unsigned));
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(LITELA_ERR_OUT_OF_MEMORY, std::string("counter cudaMalloc: ") + cudaGetErrorString(e));
      }
      e = cudaMemset(ws.counters, 0, plan.counters * sizeof(unsigned));
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemset counters");
      ws.counters_len = plan.counters;
    }
  }
  *out = &ws;
  return LITELA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Host-side validation; on success fills *plan (or returns LITELA_OK with plan->B == 0 for an
// empty problem).
litela_status validate(const void* qkv, const void* out, size_t out_elem, int B, int N, int H,
                       int d, float eps, int tokens_per_block, bool causal, Plan* plan) {
  *plan = Plan{};
  if (B < 0 || N < 0 || H < 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "B, N and H must be >= 0");
  if (d <= 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "d must be positive");
  if (d != kD) return fail(LITELA_ERR_UNSUPPORTED, "only d = 32 is built");
  if (!std::isfinite(eps) || eps < 0.f) return fail(LITELA_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
  if (causal && tokens_per_block < 1) return fail(LITELA_ERR_INVALID_ARGUMENT, "tokens_per_block must be >= 1");
  if (B > 65535 || H > 65535) return fail(LITELA_ERR_INVALID_ARGUMENT, "B and H must be <= 65535");
  if (N > (1 << 30)) return fail(LITELA_ERR_INVALID_ARGUMENT, "N must be <= 2^30");
  if (B == 0 || N == 0 || H == 0) return LITELA_OK;           // empty problem
  if (qkv == nullptr || out == nullptr) return fail(LITELA_ERR_INVALID_ARGUMENT, "null qkv or out");
  if ((reinterpret_cast<uintptr_t>(qkv) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "qkv and out must be 16-byte aligned");
  const double elems = (double)B * (double)N * 3.0 * (double)H * (double)d;
  if (elems > 4.0e18) return fail(LITELA_ERR_INVALID_ARGUMENT, "element count overflows int64");
  const size_t qkv_bytes = (size_t)B * N * 3 * H * d * sizeof(__nv_bfloat16);
  const size_t out_bytes = (size_t)B * N * H * d * out_elem;
  if (overlaps(qkv, qkv_bytes, out, out_bytes)) return fail(LITELA_ERR_INVALID_ARGUMENT, "out overlaps qkv");
  make_plan(B, N, H, causal ? tokens_per_block : 0, plan);
  return LITELA_OK;
}

template <typename OutT>
litela_status run(const void* qkv, OutT* out, int B, int N, int H, int d, float eps,
                  int tokens_per_block, bool causal, cudaStream_t stream,
                  cudaEvent_t* events = nullptr) {
  Plan plan;
  litela_status s = validate(qkv, out, sizeof(OutT), B, N, H, d, eps, tokens_per_block, causal, &plan);
  if (s != LITELA_OK || plan.B == 0) return s;
  Workspace* ws = nullptr;
  s = get_workspace(plan, stream, &ws);
  if (s != LITELA_OK) return s;
  DevPlan dp{plan.B, plan.N, plan.H, plan.T, plan.nblk, plan.chunks_per_block, plan.chunk,
             plan.tiles_per_block, eps};
  char* base = static_cast<char*>(ws->states);
  float* partials = reinterpret_cast<float*>(base + plan.off_partials);
  float* states = reinterpret_cast<float*>(base + plan.off_states);
  const auto* in = static_cast<const __nv_bfloat16*>(qkv);

  cudaError_t e;
  if (events && (e = cudaEventRecord(events[0], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  dim3 rgrid(plan.nblk * plan.chunks_per_block, H, B);
  litela_reduce_simt<<<rgrid, kReduceThreads, 0, stream>>>(in, partials, states, ws->counters, dp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_reduce_simt");
  if (events && (e = cudaEventRecord(events[1], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  dim3 agrid(plan.nblk * plan.tiles_per_block, H, B);
  litela_apply_simt<OutT><<<agrid, kApplyTile, 0, stream>>>(in, states, out, dp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_apply_simt");
  if (events && (e = cudaEventRecord(events[2], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  g_last_error.clear();
  return LITELA_OK;
}

// Fixed scratch of lite_la_fwd_noalloc: one array per device, defined statically so that the
// entry point never allocates.  Host code must not use the symbol as an address; it asks the
// runtime for each device's address once (noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[LITELA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
litela_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LITELA_ERR_UNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return LITELA_OK;
}

litela_status run_noalloc(const void* qkv, __nv_bfloat16* out, int B, int N, int H, int d, float eps,
                          cudaStream_t stream) {
  Plan plan;
  litela_status s = validate(qkv, out, sizeof(__nv_bfloat16), B, N, H, d, eps, 0, false, &plan);
  if (s != LITELA_OK || plan.B == 0) return s;
  const size_t counter_bytes = align_up(plan.counters * sizeof(unsigned), 256);
  const size_t need = counter_bytes + plan.bytes;
  if (need > LITELA_NOALLOC_SCRATCH_BYTES)
    return fail(LITELA_ERR_INVALID_ARGUMENT,
                "problem needs " + std::to_string(need) + " bytes of scratch; lite_la_fwd_noalloc has " +
                    std::to_string((size_t)LITELA_NOALLOC_SCRATCH_BYTES));
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != LITELA_OK) return s;
  char* base = static_cast<char*>(scratch);
  unsigned* counters = reinterpret_cast<unsigned*>(base);
  float* partials = reinterpret_cast<float*>(base + counter_bytes + plan.off_partials);
  float* states = reinterpret_cast<float*>(base + counter_bytes + plan.off_states);
  cudaError_t e = cudaMemsetAsync(counters, 0, plan.counters * sizeof(unsigned), stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-alloc counters)");
  DevPlan dp{plan.B, plan.N, plan.H, plan.T, plan.nblk, plan.chunks_per_block, plan.chunk,
             plan.tiles_per_block, eps};
  const auto* in = static_cast<const __nv_bfloat16*>(qkv);
  dim3 rgrid(plan.nblk * plan.chunks_per_block, H, B);
  litela_reduce_simt<<<rgrid, kReduceThreads, 0, stream>>>(in, partials, states, counters, dp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_reduce_simt");
  dim3 agrid(plan.nblk * plan.tiles_per_block, H, B);
  litela_apply_simt<__nv_bfloat16><<<agrid, kApplyTile, 0, stream>>>(in, states, out, dp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_apply_simt");
  g_last_error.clear();
  return LITELA_OK;
}

}  // namespace
}  // namespace litela

extern "C" {

litela_status lite_la_fwd_noalloc(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                  cudaStream_t stream) {
  return litela::run_noalloc(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, stream);
}


litela_status lite_la_fwd(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                          cudaStream_t stream) {
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, 0, false, stream);
}

litela_status lite_la_block_causal_fwd(const void* qkv, void* out, int B, int N, int H, int d,
                                       float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, tokens_per_block, true,
                     stream);
}

litela_status lite_la_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d, float eps,
                                 cudaStream_t stream) {
  return litela::run(qkv, out, B, N, H, d, eps, 0, false, stream);
}

litela_status lite_la_block_causal_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d,
                                              float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run(qkv, out, B, N, H, d, eps, tokens_per_block, true, stream);
}

litela_status lite_la_fwd_events(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                 cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr || !events[0] || !events[1] || !events[2])
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "events must point to 3 CUDA events");
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, 0, false, stream, events);
}

const char* lite_la_status_string(litela_status status) {
  switch (status) {
    case LITELA_OK: return "LITELA_OK";
    case LITELA_ERR_INVALID_ARGUMENT: return "LITELA_ERR_INVALID_ARGUMENT";
    case LITELA_ERR_UNSUPPORTED: return "LITELA_ERR_UNSUPPORTED";
    case LITELA_ERR_OUT_OF_MEMORY: return "LITELA_ERR_OUT_OF_MEMORY";
    case LITELA_ERR_CUDA: return "LITELA_ERR_CUDA";
  }
  return "LITELA_UNKNOWN_STATUS";
}

const char* lite_la_last_error(void) { return litela::g_last_error.c_str(); }

litela_status lite_la_release_workspace(void) {
  std::lock_guard<std::mutex> lock(litela::g_ws_mutex);
  int cur = 0;
  cudaGetDevice(&cur);
  litela_status s = LITELA_OK;
  for (auto& kv : litela::g_ws) {
    if (cudaSetDevice(kv.first.first) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
      s = litela::fail(LITELA_ERR_CUDA, "device synchronisation before workspace release failed");
    if (kv.second.states) cudaFree(kv.second.states);
    if (kv.second.counters) cudaFree(kv.second.counters);
  }
  litela::g_ws.clear();
  cudaSetDevice(cur);
  return s;
}

size_t lite_la_workspace_bytes(int B, int N, int H, int d, int tokens_per_block) {
  if (B < 0 || N < 0 || H < 0 || d != litela::kD) return 0;
  litela::Plan p;
  if (!litela::make_plan(B, N, H, tokens_per_block, &p)) return 0;
  return p.bytes + p.counters * sizeof(unsigned);
}

}  // extern "C"
