// C ABI of liblitela: argument validation, per-(device, stream) workspace, TMA descriptors and
// kernel launches.  The operation, the layouts and the error behaviour are documented in
// include/litela.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/litela.h"
#include "litela_plan.h"
#include "litela_bwd.cuh"
#include "litela_fused.cuh"
#include "litela_oproj.cuh"
#include "litela_paired.cuh"
#include "litela_tc.cuh"

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

// ---------------------------------------------------------------------------------------
// per-device set-up: SM count, kernel shared-memory limits, the driver's tensor-map encoder

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
};
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

litela_status device_setup(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LITELA_ERR_UNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(compute capability)");
    if (major != 10 || minor != 0)
      return fail(LITELA_ERR_UNSUPPORTED, "liblitela is built for sm_100a (B200); device is sm_" +
                                              std::to_string(major) + std::to_string(minor));
    if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    if ((e = cudaFuncSetAttribute(litela_reduce_tc<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)RedCfg<0>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_reduce_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)RedCfg<1>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_apply_tc<__nv_bfloat16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)ApplyCfg<__nv_bfloat16, 1>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_apply_tc<float, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)ApplyCfg<float, 1>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_apply_tc<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)ApplyCfg<__nv_bfloat16>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_apply_tc<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)ApplyCfg<float>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_fused_tc<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)FusedCfg<__nv_bfloat16>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_fused_tc<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)FusedCfg<float>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_fused_tc<__nv_bfloat16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)FusedCfg<__nv_bfloat16, true>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_fused_tc<float, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)FusedCfg<float, true>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_fused_tc<__nv_bfloat16, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)FusedCfg<__nv_bfloat16, false, 1>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_fused_tc<float, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)FusedCfg<float, false, 1>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_paired_tc<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)PairedCfg<__nv_bfloat16>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_paired_tc<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)PairedCfg<float>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_paired_tc<__nv_bfloat16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)PairedCfg<__nv_bfloat16>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_paired_tc<float, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)PairedCfg<float>::kSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_bwd_q_tc<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBqSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_bwd_q_tc<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBqSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_bwd_kv_tc<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBkSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_bwd_kv_tc<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kBkSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_oproj_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kOpSmemBytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(litela_oproj_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kOpSmemBytes)) != cudaSuccess)
      return cuda_fail(e, "cudaFuncSetAttribute(dynamic shared memory)");
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
        return fail(LITELA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ready = true;
  }
  *num_sms = d.num_sms;
  return LITELA_OK;
}

// 3-D view of the packed qkv buffer for TMA: (channel, token, batch), bf16, boxes of 64
// channels x box_tokens tokens, 128-byte swizzle, zero fill outside the tensor.
// box_channels = 32 gives boxes of one head's 32 channels with 64-byte swizzle (the backward's
// dq stores).
litela_status encode_qkv_map(const void* qkv, int B, int N, int H, int box_tokens, CUtensorMap* map,
                             int box_channels = 64) {
  const cuuint64_t row = 3ull * H * kD;
  const cuuint64_t dims[3] = {row, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[2] = {row * 2, row * 2 * (cuuint64_t)N};
  const cuuint32_t box[3] = {(cuuint32_t)box_channels, (cuuint32_t)box_tokens, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qkv), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_channels == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LITELA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")");
  return LITELA_OK;
}

// 3-D view of the output [B, N, H*d] for TMA stores: (channel, token, batch), boxes of
// 128 bytes of channels x kApTile tokens, 128-byte swizzle.
template <typename OutT>
litela_status encode_out_map(OutT* out, int B, int N, int H, CUtensorMap* map) {
  const CUtensorMapDataType dt =
      sizeof(OutT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const cuuint64_t row = (cuuint64_t)H * kD;
  const cuuint64_t dims[3] = {row, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[2] = {row * sizeof(OutT), row * sizeof(OutT) * (cuuint64_t)N};
  const cuuint32_t box[3] = {(cuuint32_t)(128 / sizeof(OutT)), (cuuint32_t)kApTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, dt, 3, static_cast<void*>(out), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(LITELA_ERR_CUDA, "cuTensorMapEncodeTiled(out) failed (" + std::to_string((int)r) + ")");
  return LITELA_OK;
}

// 3-D view of a bf16 [B, N, C] activation (the output projection's plain input): (channel,
// token, batch), boxes of 64 channels x 128 tokens, 128-byte swizzle, zero fill outside.
litela_status encode_rows_map(const void* x, int B, int N, int C, CUtensorMap* map) {
  const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)C * 2, (cuuint64_t)C * 2 * (cuuint64_t)N};
  const cuuint32_t box[3] = {(cuuint32_t)kOpK, (cuuint32_t)kOpTileM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LITELA_ERR_CUDA, "cuTensorMapEncodeTiled(input) failed (" + std::to_string((int)r) + ")");
  return LITELA_OK;
}

// 2-D view of the projection weight W [C_out, C_in] bf16: (input channel, output channel), boxes
// of 64 input channels x 224 output channels, 128-byte swizzle, zero fill outside.
litela_status encode_weight_map(const void* w, int C_out, int C_in, CUtensorMap* map) {
  const cuuint64_t dims[2] = {(cuuint64_t)C_in, (cuuint64_t)C_out};
  const cuuint64_t strides[1] = {(cuuint64_t)C_in * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kOpK, (cuuint32_t)kOpTileN};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LITELA_ERR_CUDA, "cuTensorMapEncodeTiled(weight) failed (" + std::to_string((int)r) + ")");
  return LITELA_OK;
}

// ---------------------------------------------------------------------------------------
// workspace: one per (device, stream)

struct Workspace {
  void* partials = nullptr;   // partial states (and, for the three-kernel path, state images)
  size_t partials_bytes = 0;
  int* err = nullptr;         // control words: error word, then the fused kernel's counters
  size_t ctl_words = 0;
};

// bytes of partial-state workspace a call with `plan` uses
size_t work_bytes(const Plan& plan) {
  return plan.fused ? (plan.fused_paired ? plan.paired_bytes : plan.fused_bytes) : plan.bytes;
}

// chunk length (tokens) from which the non-causal fused path takes its paired form
std::atomic<int> g_paired_min_chunk{kPairedMinChunk};

std::mutex g_ws_mutex;
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;

// Test hook: LITELA_FAIL_ALLOC=1 makes every workspace allocation fail (host-side injection
// of an out-of-memory condition; nothing runs on the GPU).
bool alloc_fault_injected() {
  const char* v = std::getenv("LITELA_FAIL_ALLOC");
  return v != nullptr && v[0] == '1';
}

// `need`: bytes of partial-state workspace the call uses (work_bytes(plan) for a forward call)
litela_status get_workspace(const Plan& plan, cudaStream_t stream, Workspace** out, size_t need) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  Workspace& ws = g_ws[{dev, reinterpret_cast<uintptr_t>(stream)}];
  const size_t need_ctl = kCounterBase + plan.counters;
  if (ws.partials_bytes < need || ws.ctl_words < need_ctl) {
    if (alloc_fault_injected())
      return fail(LITELA_ERR_OUT_OF_MEMORY, "workspace allocation failed (injected by LITELA_FAIL_ALLOC)");
    // kernels of earlier calls on this stream may still use the old buffers
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize before workspace growth");
    if (ws.ctl_words < need_ctl) {
      int keep = 0;   // a pending error code survives the growth
      if (ws.err) {
        cudaMemcpy(&keep, ws.err, sizeof(int), cudaMemcpyDeviceToHost);
        cudaFree(ws.err);
      }
      ws.err = nullptr;
      ws.ctl_words = 0;
      e = cudaMalloc(&ws.err, need_ctl * sizeof(int));
      if (e != cudaSuccess) {
        cudaGetLastError();
        ws.err = nullptr;
        return fail(LITELA_ERR_OUT_OF_MEMORY, std::string("control-word cudaMalloc: ") + cudaGetErrorString(e));
      }
      e = cudaMemset(ws.err, 0, need_ctl * sizeof(int));
      if (e == cudaSuccess && keep != 0) e = cudaMemcpy(ws.err, &keep, sizeof(int), cudaMemcpyHostToDevice);
      if (e != cudaSuccess) return cuda_fail(e, "initialising control words");
      ws.ctl_words = need_ctl;
    }
    if (ws.partials_bytes < need) {
      if (ws.partials) cudaFree(ws.partials);
      ws.partials = nullptr;
      ws.partials_bytes = 0;
      e = cudaMalloc(&ws.partials, need);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(LITELA_ERR_OUT_OF_MEMORY, std::string("workspace cudaMalloc: ") + cudaGetErrorString(e));
      }
      ws.partials_bytes = need;
    }
  }
  *out = &ws;
  return LITELA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Host-side validation of the arguments (no CUDA call).  Returns LITELA_OK with *empty = true
// for an empty problem.
litela_status validate(const void* qkv, const void* out, size_t out_elem, int B, int N, int H, int d,
                       float eps, int tokens_per_block, bool causal, bool* empty) {
  *empty = false;
  if (B < 0 || N < 0 || H < 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "B, N and H must be >= 0");
  if (d <= 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "d must be positive");
  if (d != kD) return fail(LITELA_ERR_UNSUPPORTED, "only d = 32 is built");
  if (!std::isfinite(eps) || eps < 0.f) return fail(LITELA_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
  if (causal && tokens_per_block < 1) return fail(LITELA_ERR_INVALID_ARGUMENT, "tokens_per_block must be >= 1");
  if (B > 65535 || H > 65535) return fail(LITELA_ERR_INVALID_ARGUMENT, "B and H must be <= 65535");
  if (N > (1 << 30)) return fail(LITELA_ERR_INVALID_ARGUMENT, "N must be <= 2^30");
  if (B == 0 || N == 0 || H == 0) {
    *empty = true;
    return LITELA_OK;
  }
  if (qkv == nullptr || out == nullptr) return fail(LITELA_ERR_INVALID_ARGUMENT, "null qkv or out");
  if ((reinterpret_cast<uintptr_t>(qkv) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "qkv and out must be 16-byte aligned");
  const double elems = (double)B * (double)N * 3.0 * (double)H * (double)d;
  if (elems > 4.0e18) return fail(LITELA_ERR_INVALID_ARGUMENT, "element count overflows int64");
  const size_t qkv_bytes = (size_t)B * N * 3 * H * d * sizeof(__nv_bfloat16);
  const size_t out_bytes = (size_t)B * N * H * d * out_elem;
  if (overlaps(qkv, qkv_bytes, out, out_bytes)) return fail(LITELA_ERR_INVALID_ARGUMENT, "out overlaps qkv");
  return LITELA_OK;
}

TcPlan tc_plan(const Plan& plan, float eps) {
  return TcPlan{plan.B,     plan.N,      plan.H,     plan.T, plan.nblk, plan.ngroups, plan.chunks_per_block,
                plan.chunk, plan.nquads, plan.tiles_per_block, (long long)plan.units, eps, plan.red_bpc};
}


// Launches kernel `k` with `args` as a programmatic dependent of the previous kernel in the
// stream (its prologue overlaps the previous kernel's end) unless `pdl` is false.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}

template <int kMap = 0>
litela_status launch_reduce(const Plan& plan, const void* qkv, float* partials, int* err, cudaStream_t stream,
                            bool pdl) {
  CUtensorMap map;
  litela_status s = encode_qkv_map(qkv, plan.B, plan.N, plan.H, kRedTile, &map);
  if (s != LITELA_OK) return s;
  const int xs = plan.red_bpc > 1 ? (plan.nblk + plan.red_bpc - 1) / plan.red_bpc : plan.nblk * plan.chunks_per_block;
  cudaError_t e = launch_ex(litela_reduce_tc<kMap>, dim3(xs, plan.ngroups, plan.B),
                            dim3(RedCfg<kMap>::kThreads), RedCfg<kMap>::kSmemBytes, stream, pdl, map, partials, err,
                            tc_plan(plan, 0.f));
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_reduce_tc");
  return LITELA_OK;
}

litela_status launch_scan(const Plan& plan, const float* partials, uint8_t* images, float* states, int num_sms,
                          cudaStream_t stream, bool pdl, const float* state_in = nullptr,
                          float* state_out = nullptr, uint8_t* images_t = nullptr, bool reverse = false,
                          int chunks_per_block = 0, bool rows64 = false, float* zrows = nullptr) {
  const int64_t work = ((int64_t)plan.B * plan.H * kStateFloats + kScanElems - 1) / kScanElems;
  int64_t grid = (work + kScanThreads - 1) / kScanThreads;
  if (grid > kScanCtasPerSm * num_sms) grid = kScanCtasPerSm * num_sms;
  TcPlan tp = tc_plan(plan, 0.f);
  if (chunks_per_block > 0) tp.cpb = chunks_per_block;   // partials of another chunking (the backward's)
  cudaError_t e = launch_ex(litela_state_scan, dim3((unsigned)grid), dim3(kScanThreads), 0, stream, pdl,
                            partials, images, images_t, states, state_in, state_out, reverse, rows64, zrows, tp);
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_state_scan");
  return LITELA_OK;
}

// Launches the fused single kernel (non-causal path) for `plan` with the given scratch; phase
// events, if requested, bracket it (events[1] is recorded with events[2], after the kernel).
// kMap 1: the ELU + 1 variant (non-causal plans only).
template <typename OutT, int kMap = 0>
litela_status launch_fused(const Plan& plan, const void* qkv, OutT* out, float eps, float* partials, int* ctl,
                           size_t ctl_words, cudaStream_t stream,
                           cudaEvent_t* events, float* states = nullptr) {
  CUtensorMap map_kv, map_q, map_out;
  litela_status s = encode_qkv_map(qkv, plan.B, plan.N, plan.H, kRedTile, &map_kv);
  if (s != LITELA_OK) return s;
  s = encode_qkv_map(qkv, plan.B, plan.N, plan.H, kApTile, &map_q);
  if (s != LITELA_OK) return s;
  s = encode_out_map(out, plan.B, plan.N, plan.H, &map_out);
  if (s != LITELA_OK) return s;
  cudaError_t e;
  if (events && (e = cudaEventRecord(events[0], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  // the fused kernel's control words: every word after kCounterBase (the last two: finish, ticket)
  const int set_words = (int)(ctl_words - kCounterBase);
  float* totals = plan.fused_causal ? reinterpret_cast<float*>(reinterpret_cast<char*>(partials) + plan.fused_off_totals)
                                    : nullptr;
  const FusedPlan fp{plan.B,   plan.N,    plan.H,     plan.nquads,      plan.fused_cpb, plan.fused_chunk,
                     plan.fused_ntiles, set_words, eps, states, plan.T, plan.nblk,
                     plan.fused_bpc, totals};
  const unsigned grid = (unsigned)(plan.B * plan.nquads * plan.fused_cpb);
  unsigned* counters = reinterpret_cast<unsigned*>(ctl + kCounterBase);
  if (kMap == 0 && plan.fused_paired) {
    FusedPlan pp = fp;
    pp.cpb = plan.paired_cpb;
    pp.chunk = plan.paired_chunk;
    // non-causal: ceil(nq / 2) sibling groups of two quads; block-causal: a group per quad
    const int nq = plan.B * plan.nquads;
    const unsigned pgrid = (unsigned)((plan.fused_causal ? nq : (nq + 1) / 2) * plan.paired_cpb);
    if (plan.fused_causal)
      e = launch_ex(litela_paired_tc<OutT, true>, dim3(pgrid), dim3(PairedCfg<OutT>::kThreads),
                    PairedCfg<OutT>::kSmemBytes, stream, events == nullptr, map_kv, map_q, map_out, partials, counters,
                    ctl, pp);
    else
      e = launch_ex(litela_paired_tc<OutT>, dim3(pgrid), dim3(PairedCfg<OutT>::kThreads), PairedCfg<OutT>::kSmemBytes,
                    stream, events == nullptr, map_kv, map_q, map_out, partials, counters, ctl, pp);
  } else if (kMap != 0) {
    if (plan.fused_causal) return fail(LITELA_ERR_UNSUPPORTED, "the ELU + 1 variant's fused form is non-causal");
    e = launch_ex(litela_fused_tc<OutT, false, 1>, dim3(grid), dim3(FusedCfg<OutT, false, 1>::kThreads),
                  FusedCfg<OutT, false, 1>::kSmemBytes, stream, events == nullptr, map_kv, map_q, map_out, partials,
                  counters, out, ctl, fp);
  } else if (plan.fused_causal) {
    e = launch_ex(litela_fused_tc<OutT, true>, dim3(grid), dim3(FusedCfg<OutT, true>::kThreads),
                  FusedCfg<OutT, true>::kSmemBytes, stream, events == nullptr, map_kv, map_q, map_out, partials,
                  counters, out, ctl, fp);
  } else {
    e = launch_ex(litela_fused_tc<OutT, false>, dim3(grid), dim3(FusedCfg<OutT>::kThreads), FusedCfg<OutT>::kSmemBytes,
                  stream, events == nullptr, map_kv, map_q, map_out, partials, counters, out, ctl, fp);
  }
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_fused_tc");
  if (events && ((e = cudaEventRecord(events[1], stream)) != cudaSuccess ||
                 (e = cudaEventRecord(events[2], stream)) != cudaSuccess))
    return cuda_fail(e, "cudaEventRecord");
  return LITELA_OK;
}

// Launches the state reduction, the scan and the apply for `plan` with the given scratch.  The
// scan and the apply are programmatic dependents (their prologues overlap the preceding
// kernel's end) unless phase events are requested, in which case the kernels run in plain
// stream order with events between the reduction (with the scan) and the apply.
template <typename OutT, int kMap = 0>
litela_status launch(const Plan& plan, const void* qkv, OutT* out, float eps, float* partials, uint8_t* images,
                     int* err, int num_sms, cudaStream_t stream, cudaEvent_t* events,
                     const float* state_in = nullptr, float* state_out = nullptr, float* states = nullptr) {
  CUtensorMap map_q, map_out;
  litela_status s = encode_qkv_map(qkv, plan.B, plan.N, plan.H, kApTile, &map_q);
  if (s != LITELA_OK) return s;
  s = encode_out_map(out, plan.B, plan.N, plan.H, &map_out);
  if (s != LITELA_OK) return s;
  const bool pdl = events == nullptr;
  cudaError_t e;
  if (events && (e = cudaEventRecord(events[0], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  s = launch_reduce<kMap>(plan, qkv, partials, err, stream, pdl);
  if (s != LITELA_OK) return s;
  s = launch_scan(plan, partials, images, states, num_sms, stream, pdl, state_in, state_out);
  if (s != LITELA_OK) return s;
  if (events && (e = cudaEventRecord(events[1], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  // CTAs: a multiple of the head quads when that keeps at least 7/8 of the SMs busy (all quads
  // then advance through the same token rows together), else one per SM
  long long grid = num_sms;
  if (plan.nquads <= num_sms) {
    const long long even = (long long)(num_sms / plan.nquads) * plan.nquads;
    if (8 * even >= 7LL * num_sms) grid = even;
  }
  if (grid > plan.units) grid = plan.units;
  e = launch_ex(litela_apply_tc<OutT, kMap>, dim3((unsigned)grid), dim3(ApplyCfg<OutT, kMap>::kThreads),
                ApplyCfg<OutT, kMap>::kSmemBytes, stream, pdl, map_q, map_out, static_cast<const uint8_t*>(images), out,
                err, tc_plan(plan, eps));
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_apply_tc");
  if (events && (e = cudaEventRecord(events[2], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  return LITELA_OK;
}

// State reduction alone, writing the fp32 prefix states to `states`.
litela_status run_states(const void* qkv, float* states, int B, int N, int H, int d, int tokens_per_block,
                         cudaStream_t stream) {
  bool empty = false;
  litela_status s = validate(qkv, states, 0, B, N, H, d, 0.f, 0, false, &empty);
  if (s != LITELA_OK || empty) return s;
  int num_sms = 0;
  s = device_setup(&num_sms);
  if (s != LITELA_OK) return s;
  Plan plan;
  make_plan(B, N, H, tokens_per_block, num_sms, &plan);
  const size_t state_bytes = (size_t)B * H * plan.nblk * kStateFloats * sizeof(float);
  const size_t qkv_bytes = (size_t)B * N * 3 * H * d * sizeof(__nv_bfloat16);
  if (overlaps(qkv, qkv_bytes, states, state_bytes)) return fail(LITELA_ERR_INVALID_ARGUMENT, "states overlaps qkv");
  Workspace* ws = nullptr;
  s = get_workspace(plan, stream, &ws, plan.bytes);
  if (s != LITELA_OK) return s;
  float* partials = static_cast<float*>(ws->partials);
  s = launch_reduce(plan, qkv, partials, ws->err, stream, true);
  if (s != LITELA_OK) return s;
  s = launch_scan(plan, partials, nullptr, states, num_sms, stream, true);
  if (s != LITELA_OK) return s;
  g_last_error.clear();
  return LITELA_OK;
}

// kMap 0: LiteLA (ReLU, + eps); kMap 1: the ELU + 1 variant (eps is the denominator's clamp),
// always on the three-kernel path.
template <typename OutT, int kMap = 0>
litela_status run(const void* qkv, OutT* out, int B, int N, int H, int d, float eps, int tokens_per_block,
                  bool causal, cudaStream_t stream, cudaEvent_t* events = nullptr, bool carry = false,
                  const float* state_in = nullptr, float* state_out = nullptr, float* save_states = nullptr) {
  bool empty = false;
  litela_status s = validate(qkv, out, sizeof(OutT), B, N, H, d, eps, tokens_per_block, causal, &empty);
  if (s != LITELA_OK || empty) return s;
  if (save_states != nullptr) {   // the states the queries use, fp32 [B][H][nblk][33][32]
    const int nb = (!causal || tokens_per_block >= N) ? 1 : (N + tokens_per_block - 1) / tokens_per_block;
    const size_t sbytes = (size_t)B * H * nb * kStateFloats * sizeof(float);
    const size_t qkv_bytes = (size_t)B * N * 3 * H * d * sizeof(__nv_bfloat16);
    const size_t out_bytes = (size_t)B * N * H * d * sizeof(OutT);
    if (reinterpret_cast<uintptr_t>(save_states) & 15u)
      return fail(LITELA_ERR_INVALID_ARGUMENT, "states must be 16-byte aligned");
    if (overlaps(save_states, sbytes, qkv, qkv_bytes) || overlaps(save_states, sbytes, out, out_bytes))
      return fail(LITELA_ERR_INVALID_ARGUMENT, "states overlaps qkv or out");
  }
  int num_sms = 0;
  s = device_setup(&num_sms);
  if (s != LITELA_OK) return s;
  Plan plan;
  make_plan(B, N, H, causal ? tokens_per_block : 0, num_sms, &plan, g_paired_min_chunk.load());
  // the carried state enters through the scan, and the ELU + 1 variant's block-causal form has
  // no fused kernel: the three-kernel path
  if (carry || (kMap != 0 && plan.fused_causal)) {
    plan.fused = plan.fused_causal = plan.fused_paired = false;
    plan.counters = 0;
  }
  if (kMap != 0) plan.fused_paired = false;   // the paired form is built for ReLU only
  if (carry) {
    const size_t sbytes = (size_t)B * H * kStateFloats * sizeof(float);
    const size_t qkv_bytes = (size_t)B * N * 3 * H * d * sizeof(__nv_bfloat16);
    const size_t out_bytes = (size_t)B * N * H * d * sizeof(OutT);
    if ((state_in && (reinterpret_cast<uintptr_t>(state_in) & 15u)) ||
        (state_out && (reinterpret_cast<uintptr_t>(state_out) & 15u)))
      return fail(LITELA_ERR_INVALID_ARGUMENT, "state_in and state_out must be 16-byte aligned");
    if ((state_in && (overlaps(state_in, sbytes, qkv, qkv_bytes) || overlaps(state_in, sbytes, out, out_bytes))) ||
        (state_out && (overlaps(state_out, sbytes, qkv, qkv_bytes) || overlaps(state_out, sbytes, out, out_bytes))))
      return fail(LITELA_ERR_INVALID_ARGUMENT, "a state buffer overlaps qkv or out");
  }
  Workspace* ws = nullptr;
  s = get_workspace(plan, stream, &ws, work_bytes(plan));
  if (s != LITELA_OK) return s;
  char* base = static_cast<char*>(ws->partials);
  if (carry)
    s = launch<OutT, kMap>(plan, qkv, out, eps, reinterpret_cast<float*>(base),
                           reinterpret_cast<uint8_t*>(base + plan.off_images), ws->err, num_sms, stream, events,
                           state_in, state_out);
  else if (plan.fused)
    s = launch_fused<OutT, kMap>(plan, qkv, out, eps, reinterpret_cast<float*>(base), ws->err, ws->ctl_words, stream,
                                 events, save_states);
  else
    s = launch<OutT, kMap>(plan, qkv, out, eps, reinterpret_cast<float*>(base),
                           reinterpret_cast<uint8_t*>(base + plan.off_images), ws->err, num_sms, stream, events,
                           nullptr, nullptr, save_states);
  if (s == LITELA_OK) g_last_error.clear();
  return s;
}

// ---------------------------------------------------------------------------------------
// backward

// Five kernels: reduction and scan (S, S images, S^T images), dq + partial dS, reverse scan
// (dS images), dk + dv.  Chained with programmatic dependent launch unless phase events are
// requested: then events[0] precedes the reduction, events[1] follows the scan, events[2] the
// dq kernel and events[3] the dk/dv kernel (after the reverse scan).
// states_in (optional): the forward's states, fp32 [B][H][nblk][33][32] (lite_la_fwd_save_state);
// the reduction and the scan are then replaced by their conversion into images.
template <typename OutT>
litela_status run_bwd(const void* qkv, const void* dout, OutT* dqkv, int B, int N, int H, int d, float eps,
                      int tokens_per_block, bool causal, cudaStream_t stream, cudaEvent_t* events = nullptr,
                      const float* states_in = nullptr) {
  bool empty = false;
  // qkv and dout as the forward's qkv and out
  litela_status s = validate(qkv, dout, sizeof(__nv_bfloat16), B, N, H, d, eps, tokens_per_block, causal, &empty);
  if (s != LITELA_OK || empty) return s;
  if (dqkv == nullptr) return fail(LITELA_ERR_INVALID_ARGUMENT, "null dqkv");
  if (reinterpret_cast<uintptr_t>(dqkv) & 15u) return fail(LITELA_ERR_INVALID_ARGUMENT, "dqkv must be 16-byte aligned");
  const size_t qkv_bytes = (size_t)B * N * 3 * H * d * sizeof(__nv_bfloat16);
  const size_t dout_bytes = (size_t)B * N * H * d * sizeof(__nv_bfloat16);
  const size_t dqkv_bytes = (size_t)B * N * 3 * H * d * sizeof(OutT);
  if (overlaps(dqkv, dqkv_bytes, qkv, qkv_bytes) || overlaps(dqkv, dqkv_bytes, dout, dout_bytes))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "dqkv overlaps qkv or dout");
  if (states_in != nullptr) {
    if (reinterpret_cast<uintptr_t>(states_in) & 15u)
      return fail(LITELA_ERR_INVALID_ARGUMENT, "states must be 16-byte aligned");
    const int nb = (!causal || tokens_per_block >= N) ? 1 : (N + tokens_per_block - 1) / tokens_per_block;
    if (overlaps(states_in, (size_t)B * H * nb * kStateFloats * sizeof(float), dqkv, dqkv_bytes))
      return fail(LITELA_ERR_INVALID_ARGUMENT, "states overlaps dqkv");
  }
  int num_sms = 0;
  s = device_setup(&num_sms);
  if (s != LITELA_OK) return s;
  Plan plan;
  make_plan(B, N, H, causal ? tokens_per_block : 0, num_sms, &plan);
  make_bwd_plan(num_sms, &plan);
  Workspace* ws = nullptr;
  s = get_workspace(plan, stream, &ws, plan.bwd_bytes);
  if (s != LITELA_OK) return s;
  char* base = static_cast<char*>(ws->partials);
  float* partials = reinterpret_cast<float*>(base);
  uint8_t* images = reinterpret_cast<uint8_t*>(base + plan.off_images);
  uint8_t* images_t = reinterpret_cast<uint8_t*>(base + plan.off_images_t);
  float* dpartials = reinterpret_cast<float*>(base + plan.off_dpartials);
  uint8_t* dimages = reinterpret_cast<uint8_t*>(base + plan.off_dimages);
  uint8_t* dimages_t = reinterpret_cast<uint8_t*>(base + plan.off_dimages_t);
  float* dzrows = reinterpret_cast<float*>(base + plan.off_dzrows);
  CUtensorMap map_qkv, map_g;
  s = encode_qkv_map(qkv, B, N, H, kApTile, &map_qkv);
  if (s != LITELA_OK) return s;
  s = encode_out_map(static_cast<__nv_bfloat16*>(const_cast<void*>(dout)), B, N, H, &map_g);
  if (s != LITELA_OK) return s;
  // TMA stores of dq (one head per box) and of dk, dv (head pairs) for bf16 output; the fp32
  // output is written row by row and never uses these maps
  CUtensorMap map_dq = map_qkv, map_dqkv = map_qkv;
  if (sizeof(OutT) == 2) {
    s = encode_qkv_map(dqkv, B, N, H, kApTile, &map_dq, 32);
    if (s != LITELA_OK) return s;
    s = encode_qkv_map(dqkv, B, N, H, kApTile, &map_dqkv);
    if (s != LITELA_OK) return s;
  }
  const bool pdl = events == nullptr;
  // one block per quad: the dq and dk/dv kernels sum the partial states into their images
  // themselves (in the scans' order), and the two scan launches are left out
  const int fold_fwd = (plan.nblk == 1 && states_in == nullptr) ? tc_plan(plan, 0.f).cpb : 0;
  const int fold_bwd = plan.nblk == 1 ? plan.bwd_cpb : 0;
  const BwdPlan bp{B, N, H, plan.T, plan.nblk, plan.nquads, plan.bwd_cpb, plan.bwd_chunk, eps, fold_fwd, fold_bwd};
  const dim3 grid((unsigned)(plan.nblk * plan.bwd_cpb), (unsigned)plan.nquads, (unsigned)B);
  cudaError_t e;
  if (events && (e = cudaEventRecord(events[0], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if (states_in == nullptr) {
    s = launch_reduce(plan, qkv, partials, ws->err, stream, pdl);
    if (s != LITELA_OK) return s;
    if (fold_fwd == 0) {
      s = launch_scan(plan, partials, images, nullptr, num_sms, stream, pdl, nullptr, nullptr, images_t, false);
      if (s != LITELA_OK) return s;
    }
  } else {
    const long long nst = (long long)B * H * plan.nblk;
    long long grid = (nst * kStateFloats + kScanThreads - 1) / kScanThreads;
    if (grid > num_sms) grid = num_sms;
    e = launch_ex(litela_state_images, dim3((unsigned)grid), dim3(kScanThreads), 0, stream, pdl, states_in, images,
                  images_t, nst);
    if (e != cudaSuccess) return cuda_fail(e, "launch litela_state_images");
  }
  if (events && (e = cudaEventRecord(events[1], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  e = launch_ex(litela_bwd_q_tc<OutT>, grid, dim3(kBwThreads), kBqSmemBytes, stream, pdl, map_qkv, map_g, map_dq,
                static_cast<const uint8_t*>(images), static_cast<const uint8_t*>(images_t),
                static_cast<const float*>(partials), dpartials, dqkv, ws->err, bp);
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_bwd_q_tc");
  if (events && (e = cudaEventRecord(events[2], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if (fold_bwd == 0) {
    s = launch_scan(plan, dpartials, dimages, nullptr, num_sms, stream, pdl, nullptr, nullptr, dimages_t, true,
                    plan.bwd_cpb, true, dzrows);
    if (s != LITELA_OK) return s;
  }
  e = launch_ex(litela_bwd_kv_tc<OutT>, grid, dim3(kBwThreads), kBkSmemBytes, stream, pdl, map_qkv, map_dqkv,
                static_cast<const uint8_t*>(dimages), static_cast<const uint8_t*>(dimages_t),
                static_cast<const float*>(dzrows), static_cast<const float*>(dpartials), dqkv, ws->err, bp);
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_bwd_kv_tc");
  if (events && (e = cudaEventRecord(events[3], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  g_last_error.clear();
  return LITELA_OK;
}

// ---------------------------------------------------------------------------------------
// output projection: LiteLA with the apply in the projection GEMM's prologue, and the plain
// projection (the unfused chain's second step)

// Validation shared by both: sizes, then (unless the problem is empty) the weight, bias and
// output buffers (host-side, no CUDA call).
litela_status validate_proj(const void* w, const float* bias, const void* y, int C_in, int C_out, bool empty) {
  if (C_out < 0 || C_in < 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "C_in and C_out must be >= 0");
  if (C_out % 8 != 0 || C_in % 8 != 0)
    return fail(LITELA_ERR_INVALID_ARGUMENT, "C_in and C_out must be multiples of 8 (16-byte rows)");
  if (C_out > (1 << 24) || C_in > (1 << 24)) return fail(LITELA_ERR_INVALID_ARGUMENT, "C_in and C_out must be <= 2^24");
  if (C_out == 0 || empty) return LITELA_OK;
  if (w == nullptr || y == nullptr) return fail(LITELA_ERR_INVALID_ARGUMENT, "null weight or output");
  if ((reinterpret_cast<uintptr_t>(w) & 15u) || (reinterpret_cast<uintptr_t>(y) & 15u))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "weight and output must be 16-byte aligned");
  if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 3u))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "bias must be 4-byte aligned");
  return LITELA_OK;
}

OprojPlan oproj_plan(int B, int N, int H, int C_in, int C_out, int T, int nblk, float eps) {
  OprojPlan p{};
  p.B = B; p.N = N; p.H = H; p.C_in = C_in; p.C_out = C_out; p.T = T; p.nblk = nblk; p.eps = eps;
  p.ntn = (C_out + kOpTileN - 1) / kOpTileN;
  p.ntt = (N + kOpTileM - 1) / kOpTileM;
  p.nsteps = (C_in + kOpK - 1) / kOpK;
  p.ntiles = (long long)B * p.ntt * p.ntn;
  return p;
}

// LiteLA (non-causal, or block-causal with a block size that is a multiple of 128 tokens), then
// y = x W^T (+ bias): the state reduction, the prefix scan (the state images) and the fused
// apply + projection kernel.  events (optional): [0] before the reduction, [1] after the scan,
// [2] after the projection kernel (then no programmatic overlap).
litela_status run_oproj(const void* qkv, const void* w, const float* bias, __nv_bfloat16* y, int B, int N, int H, int d,
                        int C_out, float eps, int tokens_per_block, cudaStream_t stream, cudaEvent_t* events) {
  const bool causal = tokens_per_block > 0;
  bool empty = false;
  litela_status s = validate(qkv, y, 0, B, N, H, d, eps, tokens_per_block, causal, &empty);
  if (s != LITELA_OK) return s;
  s = validate_proj(w, bias, y, H * d, C_out, empty);
  if (s != LITELA_OK || empty || C_out == 0) return s;
  if (causal && tokens_per_block < N && tokens_per_block % kOpTileM != 0)
    return fail(LITELA_ERR_UNSUPPORTED, "the fused projection needs tokens_per_block to be a multiple of 128 (or >= N)");
  const size_t qkv_bytes = (size_t)B * N * 3 * H * d * 2, y_bytes = (size_t)B * N * C_out * 2;
  const size_t w_bytes = (size_t)C_out * H * d * 2;
  if (overlaps(y, y_bytes, qkv, qkv_bytes) || overlaps(y, y_bytes, w, w_bytes) ||
      (bias && overlaps(y, y_bytes, bias, (size_t)C_out * 4)))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "the output overlaps an input");
  int num_sms = 0;
  s = device_setup(&num_sms);
  if (s != LITELA_OK) return s;
  Plan plan;
  make_plan(B, N, H, causal ? tokens_per_block : 0, num_sms, &plan);
  plan.fused = plan.fused_causal = plan.fused_paired = false;   // the state images go through the workspace
  plan.counters = 0;
  Workspace* ws = nullptr;
  s = get_workspace(plan, stream, &ws, plan.bytes);
  if (s != LITELA_OK) return s;
  char* base = static_cast<char*>(ws->partials);
  float* partials = reinterpret_cast<float*>(base);
  uint8_t* images = reinterpret_cast<uint8_t*>(base + plan.off_images);
  CUtensorMap map_q, map_w;
  if ((s = encode_qkv_map(qkv, B, N, H, kOpTileM, &map_q)) != LITELA_OK) return s;
  if ((s = encode_weight_map(w, C_out, H * d, &map_w)) != LITELA_OK) return s;
  const bool pdl = events == nullptr;
  cudaError_t e;
  if (events && (e = cudaEventRecord(events[0], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((s = launch_reduce(plan, qkv, partials, ws->err, stream, pdl)) != LITELA_OK) return s;
  if ((s = launch_scan(plan, partials, images, nullptr, num_sms, stream, pdl)) != LITELA_OK) return s;
  if (events && (e = cudaEventRecord(events[1], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  const OprojPlan op = oproj_plan(B, N, H, H * d, C_out, plan.T, plan.nblk, eps);
  const unsigned grid = (unsigned)(op.ntiles < num_sms ? op.ntiles : num_sms);
  e = launch_ex(litela_oproj_tc<true>, dim3(grid), dim3(kOpThreads), kOpSmemBytes, stream, pdl, map_q, map_w,
                static_cast<const uint8_t*>(images), bias, y, ws->err, op);
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_oproj_tc");
  if (events && (e = cudaEventRecord(events[2], stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  g_last_error.clear();
  return LITELA_OK;
}

// y = x W^T (+ bias) on a bf16 [B, N, C_in] input: the same kernel with the input loaded by TMA.
litela_status run_linear(const void* x, const void* w, const float* bias, __nv_bfloat16* y, int B, int N, int C_in,
                         int C_out, cudaStream_t stream) {
  if (B < 0 || N < 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "B and N must be >= 0");
  if (B > 65535 || N > (1 << 30)) return fail(LITELA_ERR_INVALID_ARGUMENT, "B must be <= 65535 and N <= 2^30");
  litela_status s = validate_proj(w, bias, y, C_in, C_out, B == 0 || N == 0);
  if (s != LITELA_OK) return s;
  if (B == 0 || N == 0 || C_out == 0) return LITELA_OK;
  if (C_in == 0) return fail(LITELA_ERR_INVALID_ARGUMENT, "C_in must be positive");
  if (x == nullptr || (reinterpret_cast<uintptr_t>(x) & 15u))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "the input must be non-null and 16-byte aligned");
  const size_t x_bytes = (size_t)B * N * C_in * 2, y_bytes = (size_t)B * N * C_out * 2;
  if (overlaps(y, y_bytes, x, x_bytes) || overlaps(y, y_bytes, w, (size_t)C_out * C_in * 2) ||
      (bias && overlaps(y, y_bytes, bias, (size_t)C_out * 4)))
    return fail(LITELA_ERR_INVALID_ARGUMENT, "the output overlaps an input");
  int num_sms = 0;
  s = device_setup(&num_sms);
  if (s != LITELA_OK) return s;
  Plan plan;
  make_plan(1, 1, 1, 0, num_sms, &plan);   // only for the error word of this stream's workspace
  plan.counters = 0;
  Workspace* ws = nullptr;
  s = get_workspace(plan, stream, &ws, 0);
  if (s != LITELA_OK) return s;
  CUtensorMap map_x, map_w;
  if ((s = encode_rows_map(x, B, N, C_in, &map_x)) != LITELA_OK) return s;
  if ((s = encode_weight_map(w, C_out, C_in, &map_w)) != LITELA_OK) return s;
  const OprojPlan op = oproj_plan(B, N, 0, C_in, C_out, N, 1, 0.f);
  const unsigned grid = (unsigned)(op.ntiles < num_sms ? op.ntiles : num_sms);
  cudaError_t e = launch_ex(litela_oproj_tc<false>, dim3(grid), dim3(kOpThreads), kOpSmemBytes, stream, true, map_x,
                            map_w, static_cast<const uint8_t*>(nullptr), bias, y, ws->err, op);
  if (e != cudaSuccess) return cuda_fail(e, "launch litela_oproj_tc");
  g_last_error.clear();
  return LITELA_OK;
}

// Fixed scratch of lite_la_fwd_noalloc: one array per device, defined statically so that the
// entry point never allocates.  Host code must not use the symbol as an address; it asks the
// runtime for each device's address once (noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[LITELA_NOALLOC_SCRATCH_BYTES];

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
  bool empty = false;
  litela_status s = validate(qkv, out, sizeof(__nv_bfloat16), B, N, H, d, eps, 0, false, &empty);
  if (s != LITELA_OK || empty) return s;
  int num_sms = 0;
  s = device_setup(&num_sms);
  if (s != LITELA_OK) return s;
  Plan plan;
  make_plan(B, N, H, 0, num_sms, &plan, g_paired_min_chunk.load());
  const size_t err_bytes = align_up((kCounterBase + plan.counters) * sizeof(int), 256);
  const size_t need = err_bytes + work_bytes(plan);
  if (need > LITELA_NOALLOC_SCRATCH_BYTES)
    return fail(LITELA_ERR_INVALID_ARGUMENT,
                "problem needs " + std::to_string(need) + " bytes of scratch; lite_la_fwd_noalloc has " +
                    std::to_string((size_t)LITELA_NOALLOC_SCRATCH_BYTES));
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != LITELA_OK) return s;
  char* base = static_cast<char*>(scratch);
  if (plan.fused) {
    // the counters must start at zero: cleared here every call (no state survives between calls)
    cudaError_t e = cudaMemsetAsync(base + kCounterBase * sizeof(int), 0, plan.counters * sizeof(unsigned), stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-alloc counters)");
    s = launch_fused(plan, qkv, out, eps, reinterpret_cast<float*>(base + err_bytes), reinterpret_cast<int*>(base),
                     kCounterBase + plan.counters, stream, nullptr);
    if (s == LITELA_OK) g_last_error.clear();
    return s;
  }
  s = launch(plan, qkv, out, eps, reinterpret_cast<float*>(base + err_bytes),
             reinterpret_cast<uint8_t*>(base + err_bytes + plan.off_images), reinterpret_cast<int*>(base), num_sms,
             stream, nullptr);
  if (s == LITELA_OK) g_last_error.clear();
  return s;
}

}  // namespace
}  // namespace litela

extern "C" {

litela_status lite_la_fwd(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                          cudaStream_t stream) {
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, 0, false, stream);
}

litela_status lite_la_block_causal_fwd(const void* qkv, void* out, int B, int N, int H, int d,
                                       float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, tokens_per_block, true, stream);
}

litela_status lite_la_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d, float eps,
                                 cudaStream_t stream) {
  return litela::run(qkv, out, B, N, H, d, eps, 0, false, stream);
}

litela_status lite_la_block_causal_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d,
                                              float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run(qkv, out, B, N, H, d, eps, tokens_per_block, true, stream);
}

litela_status lite_la_block_causal_fwd_carry(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                             int tokens_per_block, const float* state_in, float* state_out,
                                             cudaStream_t stream) {
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, tokens_per_block, true, stream, nullptr,
                     true, state_in, state_out);
}

litela_status lite_la_block_causal_fwd_carry_f32out(const void* qkv, float* out, int B, int N, int H, int d,
                                                    float eps, int tokens_per_block, const float* state_in,
                                                    float* state_out, cudaStream_t stream) {
  return litela::run(qkv, out, B, N, H, d, eps, tokens_per_block, true, stream, nullptr, true, state_in, state_out);
}

litela_status lite_la_fwd_events(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                 cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr || !events[0] || !events[1] || !events[2])
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "events must point to 3 CUDA events");
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, 0, false, stream, events);
}

litela_status lite_la_block_causal_fwd_events(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                              int tokens_per_block, cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr || !events[0] || !events[1] || !events[2])
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "events must point to 3 CUDA events");
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, tokens_per_block, true, stream, events);
}

litela_status lite_la_state_fwd(const void* qkv, float* states, int B, int N, int H, int d,
                                int tokens_per_block, cudaStream_t stream) {
  return litela::run_states(qkv, states, B, N, H, d, tokens_per_block, stream);
}

litela_status lite_la_fwd_noalloc(const void* qkv, void* out, int B, int N, int H, int d, float eps,
                                  cudaStream_t stream) {
  return litela::run_noalloc(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, stream);
}

litela_status lite_la_fwd_oproj(const void* qkv, const void* w_o, const float* bias, void* y, int B, int N, int H,
                                int d, int C_out, float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run_oproj(qkv, w_o, bias, static_cast<__nv_bfloat16*>(y), B, N, H, d, C_out, eps, tokens_per_block,
                           stream, nullptr);
}

litela_status lite_la_fwd_oproj_events(const void* qkv, const void* w_o, const float* bias, void* y, int B, int N,
                                       int H, int d, int C_out, float eps, int tokens_per_block, cudaStream_t stream,
                                       cudaEvent_t* events) {
  if (events == nullptr || !events[0] || !events[1] || !events[2])
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "events must point to 3 CUDA events");
  return litela::run_oproj(qkv, w_o, bias, static_cast<__nv_bfloat16*>(y), B, N, H, d, C_out, eps, tokens_per_block,
                           stream, events);
}

litela_status lite_la_out_proj(const void* x, const void* w_o, const float* bias, void* y, int B, int N, int C_in,
                               int C_out, cudaStream_t stream) {
  return litela::run_linear(x, w_o, bias, static_cast<__nv_bfloat16*>(y), B, N, C_in, C_out, stream);
}

litela_status lite_la_elu1_fwd(const void* qkv, void* out, int B, int N, int H, int d, float clamp_min,
                               int tokens_per_block, cudaStream_t stream) {
  return litela::run<__nv_bfloat16, 1>(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, clamp_min,
                                       tokens_per_block, tokens_per_block > 0, stream);
}

litela_status lite_la_elu1_fwd_events(const void* qkv, void* out, int B, int N, int H, int d, float clamp_min,
                                      int tokens_per_block, cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr || !events[0] || !events[1] || !events[2])
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "events must point to 3 CUDA events");
  return litela::run<__nv_bfloat16, 1>(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, clamp_min,
                                       tokens_per_block, tokens_per_block > 0, stream, events);
}

litela_status lite_la_elu1_fwd_f32out(const void* qkv, float* out, int B, int N, int H, int d, float clamp_min,
                                      int tokens_per_block, cudaStream_t stream) {
  return litela::run<float, 1>(qkv, out, B, N, H, d, clamp_min, tokens_per_block, tokens_per_block > 0, stream);
}

litela_status lite_la_bwd(const void* qkv, const void* dout, void* dqkv, int B, int N, int H, int d, float eps,
                          cudaStream_t stream) {
  return litela::run_bwd(qkv, dout, static_cast<__nv_bfloat16*>(dqkv), B, N, H, d, eps, 0, false, stream);
}

litela_status lite_la_block_causal_bwd(const void* qkv, const void* dout, void* dqkv, int B, int N, int H, int d,
                                       float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run_bwd(qkv, dout, static_cast<__nv_bfloat16*>(dqkv), B, N, H, d, eps, tokens_per_block, true,
                         stream);
}

litela_status lite_la_fwd_save_state(const void* qkv, void* out, float* states, int B, int N, int H, int d,
                                     float eps, int tokens_per_block, cudaStream_t stream) {
  if (states == nullptr && B > 0 && N > 0 && H > 0)
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "null states");
  return litela::run(qkv, static_cast<__nv_bfloat16*>(out), B, N, H, d, eps, tokens_per_block, tokens_per_block > 0,
                     stream, nullptr, false, nullptr, nullptr, states);
}

litela_status lite_la_bwd_from_state(const void* qkv, const void* dout, const float* states, void* dqkv, int B, int N,
                                     int H, int d, float eps, int tokens_per_block, cudaStream_t stream) {
  if (states == nullptr && B > 0 && N > 0 && H > 0)
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "null states");
  return litela::run_bwd(qkv, dout, static_cast<__nv_bfloat16*>(dqkv), B, N, H, d, eps, tokens_per_block,
                         tokens_per_block > 0, stream, nullptr, states);
}

litela_status lite_la_bwd_f32out(const void* qkv, const void* dout, float* dqkv, int B, int N, int H, int d,
                                 float eps, cudaStream_t stream) {
  return litela::run_bwd(qkv, dout, dqkv, B, N, H, d, eps, 0, false, stream);
}

litela_status lite_la_block_causal_bwd_f32out(const void* qkv, const void* dout, float* dqkv, int B, int N, int H,
                                              int d, float eps, int tokens_per_block, cudaStream_t stream) {
  return litela::run_bwd(qkv, dout, dqkv, B, N, H, d, eps, tokens_per_block, true, stream);
}

litela_status lite_la_bwd_events(const void* qkv, const void* dout, void* dqkv, int B, int N, int H, int d,
                                 float eps, int tokens_per_block, cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr || !events[0] || !events[1] || !events[2] || !events[3])
    return litela::fail(LITELA_ERR_INVALID_ARGUMENT, "events must point to 4 CUDA events");
  return litela::run_bwd(qkv, dout, static_cast<__nv_bfloat16*>(dqkv), B, N, H, d, eps, tokens_per_block,
                         tokens_per_block > 0, stream, events);
}

size_t lite_la_bwd_workspace_bytes(int B, int N, int H, int d, int tokens_per_block) {
  if (B < 0 || N < 0 || H < 0 || d != litela::kD) return 0;
  litela::Plan p;
  if (!litela::make_plan(B, N, H, tokens_per_block, 148, &p)) return 0;
  litela::make_bwd_plan(148, &p);
  return p.bwd_bytes + (litela::kCounterBase + p.counters) * sizeof(int);
}

int lite_la_kernels_per_call(int B, int N, int H, int d, int tokens_per_block) {
  if (B <= 0 || N <= 0 || H <= 0 || d != litela::kD) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  litela::Plan p;
  litela::make_plan(B, N, H, tokens_per_block, sms, &p, litela::g_paired_min_chunk.load());
  return p.fused ? 1 : 3;
}

int lite_la_bwd_kernels_per_call(int B, int N, int H, int d, int tokens_per_block, int from_state) {
  if (B <= 0 || N <= 0 || H <= 0 || d != litela::kD) return 0;
  const bool one_block = tokens_per_block <= 0 || tokens_per_block >= N;
  // the state (reduction, or the saved states' images) + its scan + dq + the reverse scan + dk/dv;
  // with one block per quad the dq and dk/dv kernels do the scans themselves
  if (one_block) return 3;
  return from_state ? 4 : 5;
}

litela_status lite_la_selftest_timeout(cudaStream_t stream) {
  litela::Plan plan;
  litela::make_plan(1, 1, 1, 0, 148, &plan);
  litela::Workspace* ws = nullptr;
  litela_status s = litela::get_workspace(plan, stream, &ws, litela::work_bytes(plan));
  if (s != LITELA_OK) return s;
  litela::litela_selftest_timeout<<<1, 32, 0, stream>>>(ws->err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return litela::cuda_fail(e, "launch litela_selftest_timeout");
  return LITELA_OK;
}

litela_status lite_la_device_status(cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return litela::cuda_fail(e, "cudaGetDevice");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return litela::cuda_fail(e, "cudaStreamSynchronize");
  int* words[2] = {nullptr, nullptr};
  int* words_ws0 = nullptr;
  size_t ctl_words_ws = 0;
  {
    std::lock_guard<std::mutex> lock(litela::g_ws_mutex);
    auto it = litela::g_ws.find({dev, reinterpret_cast<uintptr_t>(stream)});
    if (it != litela::g_ws.end()) {
      words[0] = words_ws0 = it->second.err;
      ctl_words_ws = it->second.ctl_words;
    }
  }
  {
    std::lock_guard<std::mutex> lock(litela::g_noalloc_mutex);
    if (dev < litela::kMaxDevices) words[1] = static_cast<int*>(litela::g_noalloc_ptr[dev]);
  }
  int code = 0;
  for (int* w : words) {
    if (w == nullptr) continue;
    int v = 0;
    if ((e = cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
      return litela::cuda_fail(e, "reading the device error word");
    if (v != 0) {
      if (code == 0) code = v;
      if ((e = cudaMemset(w, 0, sizeof(int))) != cudaSuccess)
        return litela::cuda_fail(e, "clearing the device error word");
      // the fused kernel's last CTA leaves its counters clean even after a time-out; clear them
      // anyway, in case a call ended without reaching that point
      size_t words = 0;
      if (w == words_ws0) words = ctl_words_ws;
      if (words > (size_t)litela::kCounterBase &&
          (e = cudaMemset(w + litela::kCounterBase, 0, (words - litela::kCounterBase) * sizeof(int))) != cudaSuccess)
        return litela::cuda_fail(e, "clearing the counters");
    }
  }
  if (code != 0) {
    char buf[128];
    std::snprintf(buf, sizeof(buf), "a kernel wait timed out (code 0x%x)", code);
    return litela::fail(LITELA_ERR_DEVICE_TIMEOUT, buf);
  }
  return LITELA_OK;
}

const char* lite_la_status_string(litela_status status) {
  switch (status) {
    case LITELA_OK: return "LITELA_OK";
    case LITELA_ERR_INVALID_ARGUMENT: return "LITELA_ERR_INVALID_ARGUMENT";
    case LITELA_ERR_UNSUPPORTED: return "LITELA_ERR_UNSUPPORTED";
    case LITELA_ERR_OUT_OF_MEMORY: return "LITELA_ERR_OUT_OF_MEMORY";
    case LITELA_ERR_CUDA: return "LITELA_ERR_CUDA";
    case LITELA_ERR_DEVICE_TIMEOUT: return "LITELA_ERR_DEVICE_TIMEOUT";
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
    if (kv.second.partials) cudaFree(kv.second.partials);
    if (kv.second.err) cudaFree(kv.second.err);
  }
  litela::g_ws.clear();
  cudaSetDevice(cur);
  return s;
}

size_t lite_la_workspace_bytes(int B, int N, int H, int d, int tokens_per_block) {
  if (B < 0 || N < 0 || H < 0 || d != litela::kD) return 0;
  litela::Plan p;
  if (!litela::make_plan(B, N, H, tokens_per_block, 148, &p, litela::g_paired_min_chunk.load())) return 0;
  return litela::work_bytes(p) + (litela::kCounterBase + p.counters) * sizeof(int);
}

int lite_la_forward_form(int B, int N, int H, int d, int tokens_per_block) {
  if (B <= 0 || N <= 0 || H <= 0 || d != litela::kD) return -1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  litela::Plan p;
  litela::make_plan(B, N, H, tokens_per_block, sms, &p, litela::g_paired_min_chunk.load());
  if (!p.fused) return LITELA_FORM_THREE_KERNEL;
  if (p.fused_causal) return p.fused_paired ? LITELA_FORM_FUSED_PAIRED_CAUSAL : LITELA_FORM_FUSED_CAUSAL;
  return p.fused_paired ? LITELA_FORM_FUSED_PAIRED : LITELA_FORM_FUSED;
}

int lite_la_set_paired_min_chunk(int tokens) {
  return litela::g_paired_min_chunk.exchange(tokens > 0 ? tokens : litela::kPairedMinChunk);
}

}  // extern "C"
