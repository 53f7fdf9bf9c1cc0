// C ABI of libfa.so (declared in include/fa.h): argument checks, tensor-map
// construction and kernel dispatch.  Every entry point validates on the host
// before touching the device, so a bad argument never reaches a kernel.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/fa.h"
#include "fa_device.cuh"
#include "fa_kernels.h"

namespace fa {

static_assert(FA_STAGE_PREPROCESS == kStagePreprocess && FA_STAGE_MAIN == kStageMain &&
                  FA_STAGE_DQ_CONVERT == kStageConvert && FA_STAGE_DETERMINISTIC == kStageDeterministic,
              "stage flags of the header and the kernels differ");

// the device status word g_device_status is defined in fa_device.cuh

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks shared by every entry point; no CUDA call is made.
fa_status check_shape(int B, int H, int N, int d, float scale) {
  if (B <= 0 || H <= 0 || N <= 0) return FA_ERR_INVALID_ARG;
  if ((long long)B * H > 65535LL * 128) return FA_ERR_INVALID_ARG;
  if ((long long)B * H * N * d >= (1LL << 40)) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (p == nullptr) return FA_ERR_INVALID_ARG;
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_MISALIGNED;
  return FA_OK;
}

// Scratch of the bf16 (tcgen05) backward; the fp32 path uses a prefix of it.
size_t ws_bytes_for(int B, int H, int N, int d) {
  const size_t simt = ((size_t)B * H * N * sizeof(float) + 255) / 256 * 256;
  const size_t tc = sm100_backward_workspace(B * H, N, d);
  return simt > tc ? simt : tc;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 3-D bf16 view {d, N, B*H} of a [B,H,N,d] tensor, box {64, rows, 1}, 128-byte
// swizzle; rows past N read as zero (loads) or are not written (stores).
bool make_map(CUtensorMap* map, const void* base, int d, int N, int BH, unsigned rows = 128) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  const cuuint32_t box[3] = {64, rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D e4m3 view {d, N, B*H} of a [B,H,N,d] tensor (uint8 elements), box
// {min(d, 128), 128, 1}, swizzle of min(d, 128) bytes per row (128 or 64);
// rows past N read as zero.
bool make_map_fp8(CUtensorMap* map, const void* base, int d, int N, int BH) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const int sw = d < 128 ? d : 128;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)N * d};
  const cuuint32_t box[3] = {(cuuint32_t)sw, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         sw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D fp32 view {d, N, B*H} of the backward pass's dQ accumulator, box
// {32, 32, 1} (128-byte rows), 128-byte swizzle: the target of the bulk
// reduce-adds.
bool make_dq_map(CUtensorMap* map, void* acc, int d, int N, int BH) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, acc, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The tcgen05 kernels need an sm_100 device (compute capability 10.0).
fa_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

thread_local const char* g_last_error = "no error";

fa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return FA_OK;
  g_last_error = cudaGetErrorString(e);
  return FA_ERR_CUDA;
}

fa_status map_failed() {
  g_last_error = "cuTensorMapEncodeTiled rejected a tensor map";
  return FA_ERR_CUDA;
}

}  // namespace
}  // namespace fa

namespace fa {
namespace {

fa_status forward_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                       void* stream) {
  fa_status s = check_shape(B, H, Nq, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_shape(B, H, Nk, d, scale)) != FA_OK) return s;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, lse})) != FA_OK) return s;
  if ((s = check_device()) != FA_OK) return s;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, d, Nq, B * H) || !make_map(&mk, k, d, Nk, B * Hkv) ||
      !make_map(&mv, v, d, Nk, B * Hkv) || !make_map(&mo, o, d, Nq, B * H, 32))
    return map_failed();
  return from_cuda(sm100_forward(mq, mk, mv, mo, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal ? 1 : 0,
                                 false, 1.0f, 1.0f, static_cast<cudaStream_t>(stream)));
}

fa_status forward_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int Hkv, int Nq, int Nk, int d, float scale, float q_descale,
                      float k_descale, float v_descale, int causal, void* stream) {
  fa_status s = check_shape(B, H, Nq, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_shape(B, H, Nk, d, scale)) != FA_OK) return s;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  const float qk = q_descale * k_descale;
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || !(v_descale > 0.f) || !isfinite(q_descale) ||
      !isfinite(k_descale) || !isfinite(v_descale) || !(qk > 0.f) || !isfinite(qk * scale))
    return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, lse})) != FA_OK) return s;
  if ((s = check_device()) != FA_OK) return s;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_fp8(&mq, q, d, Nq, B * H) || !make_map_fp8(&mk, k, d, Nk, B * Hkv) ||
      !make_map_fp8(&mv, v, d, Nk, B * Hkv) || !make_map(&mo, o, d, Nq, B * H, 32))
    return map_failed();
  return from_cuda(sm100_forward(mq, mk, mv, mo, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal ? 1 : 0,
                                 true, qk, v_descale, static_cast<cudaStream_t>(stream)));
}

fa_status backward_bf16(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        void* workspace, int B, int H, int Hkv, int Nq, int Nk, int d,
                        float scale, int causal, int stages, void* stream) {
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
  if (!make_map(&mq, q, d, Nq, BH) || !make_map(&mk, k, d, Nk, B * Hkv) ||
      !make_map(&mv, v, d, Nk, B * Hkv) || !make_map(&mdo, dout, d, Nq, BH) ||
      !make_dq_map(&mdq, static_cast<char*>(workspace) + sm100_backward_dq_offset(BH, Nq), d, Nq, BH) ||
      !make_map(&mdk, dk, d, Nk, B * Hkv, 32) || !make_map(&mdv, dv, d, Nk, B * Hkv, 32))
    return map_failed();
  return from_cuda(sm100_backward(mq, mk, mv, mdo, mdq, mdk, mdv, o, dout, lse, dq, dk, dv, workspace, B, H,
                                  Hkv, Nq, Nk, d, scale, causal ? 1 : 0, stages,
                                  static_cast<cudaStream_t>(stream)));
}

// Argument checks shared by the bf16 backward entry points, then the launches.
fa_status backward_entry(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq, int Nk,
                         int d, float scale, int causal, int stages, void* stream) {
  fa_status s = check_shape(B, H, Nq, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_shape(B, H, Nk, d, scale)) != FA_OK) return s;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if ((stages & kStageAll) == 0 || (stages & ~(kStageAll | kStageDeterministic)) != 0)
    return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (workspace == nullptr || ws_bytes < ws_bytes_for(B, H, Nq, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;
  return backward_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nk, d, scale,
                       causal, stages, stream);
}

}  // namespace
}  // namespace fa

namespace fa {
// One warp waits on an mbarrier that never completes; the bounded wait gives up,
// records a timeout in the status word and the kernel returns.
__global__ void wait_timeout_probe_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, 0xFF);
  }
}
}  // namespace fa

using namespace fa;

extern "C" {

fa_status fa_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                     int N, int d, float scale, int causal, void* stream) {
  return forward_bf16(q, k, v, o, lse, B, H, H, N, N, d, scale, causal, stream);
}

fa_status fa_forward_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Hkv, int N, int d, float scale, int causal, void* stream) {
  return forward_bf16(q, k, v, o, lse, B, H, Hkv, N, N, d, scale, causal, stream);
}

fa_status fa_forward_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                        void* stream) {
  return forward_bf16(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal, stream);
}

fa_status fa_forward_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Hkv, int Nq, int Nk, int d, float scale, float q_descale,
                         float k_descale, float v_descale, int causal, void* stream) {
  return forward_fp8(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, q_descale, k_descale, v_descale,
                     causal, stream);
}

fa_status fa_forward_fp32(const float* q, const float* k, const float* v, float* o, float* lse, int B,
                          int H, int N, int d, float scale, int causal, void* stream) {
  fa_status s = check_shape(B, H, N, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, lse})) != FA_OK) return s;
  return from_cuda(simt_forward(false, q, k, v, o, lse, B * H, N, d, scale, causal ? 1 : 0,
                                static_cast<cudaStream_t>(stream)));
}

size_t fa_backward_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 1.0f) != FA_OK) return 0;
  return ws_bytes_for(B, H, N, d);
}

fa_status fa_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, void* workspace,
                      size_t ws_bytes, int B, int H, int N, int d, float scale, int causal,
                      void* stream) {
  return backward_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, H, N, N, d,
                        scale, causal, kStageAll, stream);
}

fa_status fa_backward_gqa(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv,
                          void* workspace, size_t ws_bytes, int B, int H, int Hkv, int N, int d,
                          float scale, int causal, void* stream) {
  return backward_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, N, d,
                        scale, causal, kStageAll, stream);
}

fa_status fa_backward_qk(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq, int Nk,
                         int d, float scale, int causal, void* stream) {
  return backward_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, Nq, Nk, d,
                        scale, causal, kStageAll, stream);
}

fa_status fa_backward_deterministic(const void* q, const void* k, const void* v, const void* o,
                                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                   void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq,
                                   int Nk, int d, float scale, int causal, void* stream) {
  return backward_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, Nq, Nk, d,
                        scale, causal, kStageAll | kStageDeterministic, stream);
}

fa_status fa_backward_stages(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv,
                             void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq,
                             int Nk, int d, float scale, int causal, int stages, void* stream) {
  return backward_entry(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, Nq, Nk, d,
                        scale, causal, stages, stream);
}

fa_status fa_backward_fp32(const float* q, const float* k, const float* v, const float* o,
                           const float* dout, const float* lse, float* dq, float* dk, float* dv,
                           void* workspace, size_t ws_bytes, int B, int H, int N, int d, float scale,
                           int causal, void* stream) {
  fa_status s = check_shape(B, H, N, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (workspace == nullptr || ws_bytes < ws_bytes_for(B, H, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* dsum = static_cast<float*>(workspace);
  const int BH = B * H;
  const cudaError_t e = bwd_preprocess(false, o, dout, dsum, (long long)BH * N, d, st);
  if (e != cudaSuccess) return from_cuda(e);
  return from_cuda(simt_backward(false, q, k, v, dout, lse, dsum, dq, dk, dv, BH, N, d, scale,
                                 causal ? 1 : 0, st));
}

fa_status fa_debug_wait_timeout(void* stream) {
  fa::wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return from_cuda(cudaGetLastError());
}

fa_status fa_debug_hold_scheduler(void* stream) {
  fa_status s = check_device();
  if (s != FA_OK) return s;
  return from_cuda(sm100_forward_hold_scheduler(static_cast<cudaStream_t>(stream)));
}

fa_status fa_check_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return from_cuda(e);
  unsigned int word = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word))) != cudaSuccess)
    return from_cuda(e);
  if (word == 0) return FA_OK;
  if ((e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero))) != cudaSuccess)
    return from_cuda(e);
  // a launch that gave up may have left its scheduler slot held
  if ((e = sm100_forward_reset_scheduler()) != cudaSuccess) return from_cuda(e);
  return (word & kTimeoutError) ? FA_ERR_DEVICE_TIMEOUT : FA_ERR_DEVICE_STATE;
}

const char* fa_last_error(void) { return g_last_error; }

const char* fa_status_string(fa_status status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported head dimension or device";
    case FA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_DEVICE_TIMEOUT: return "a kernel wait timed out";
    case FA_ERR_DEVICE_STATE: return "a kernel found inconsistent device state and skipped work";
  }
  return "unknown status";
}

}  // extern "C"

// ------------------------------------------------------------------------
// Allocation-free backward: the scratch of fa_backward in a fixed device
// array.  Host code must not pass the array's name to a kernel (on the host it
// names a stand-in, not device memory); its device address is looked up with
// cudaGetSymbolAddress, while the device is current, on the first call in each
// CUDA context and cached for that context.

namespace fa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_BACKWARD_NOALLOC_MAX_BYTES];

std::mutex g_noalloc_mu;
// Device address of the array per CUDA context.  The key is the context's
// unique id (cuCtxGetId), not the device ordinal: cudaDeviceReset destroys the
// context and a new one may place the module elsewhere, and a new context never
// reuses an id.
constexpr int kCacheEntries = 64;
unsigned long long g_noalloc_ctx[kCacheEntries] = {};
void* g_noalloc_ptr[kCacheEntries] = {};

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// Unique id of the current device's primary context (made current if needed).
fa_status current_context_id(unsigned long long* id) {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (!g_ctx_current || !g_ctx_id) {
    g_last_error = "cuCtxGetCurrent / cuCtxGetId are not available from the driver";
    return FA_ERR_CUDA;
  }
  // cudaSetDevice makes the device's primary context current on this thread
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaSetDevice(dev);
  if (e != cudaSuccess) return from_cuda(e);
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || g_ctx_id(ctx, id) != CUDA_SUCCESS) {
    g_last_error = "could not identify the current CUDA context";
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Device address of the scratch array in the current context.
fa_status noalloc_scratch(void** out) {
  unsigned long long id = 0;
  fa_status s = current_context_id(&id);
  if (s != FA_OK) return s;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  int free_entry = -1;
  for (int i = 0; i < kCacheEntries; ++i) {
    if (g_noalloc_ptr[i] != nullptr && g_noalloc_ctx[i] == id) {
      *out = g_noalloc_ptr[i];
      return FA_OK;
    }
    if (g_noalloc_ptr[i] == nullptr && free_entry < 0) free_entry = i;
  }
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return from_cuda(e);
  if (free_entry < 0) free_entry = (int)(id % kCacheEntries);  // full: replace an entry
  g_noalloc_ctx[free_entry] = id;
  g_noalloc_ptr[free_entry] = ptr;
  *out = ptr;
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_backward_noalloc(const void* q, const void* k, const void* v, const void* o,
                                         const void* dout, const float* lse, void* dq, void* dk,
                                         void* dv, int B, int H, int N, int d, float scale,
                                         int causal, void* stream) {
  fa_status s = check_shape(B, H, N, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (ws_bytes_for(B, H, N, d) > FA_BACKWARD_NOALLOC_MAX_BYTES) return FA_ERR_WORKSPACE;
  if ((s = check_device()) != FA_OK) return s;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  return backward_bf16(q, k, v, o, dout, lse, dq, dk, dv, scratch, B, H, H, N, N, d, scale, causal,
                       kStageAll, stream);
}
