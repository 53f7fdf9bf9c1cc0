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

// 3-D bf16 view {d, N, B*H} of a [B,H,N,d] tensor, box {64, 128, 1}, 128-byte
// swizzle; rows past N read as zero.
bool make_map(CUtensorMap* map, const void* base, int d, int N, int BH) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, d, Nq, B * H) || !make_map(&mk, k, d, Nk, B * Hkv) ||
      !make_map(&mv, v, d, Nk, B * Hkv))
    return map_failed();
  return from_cuda(sm100_forward(mq, mk, mv, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal ? 1 : 0,
                                 static_cast<cudaStream_t>(stream)));
}

fa_status backward_bf16(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        void* workspace, int B, int H, int Hkv, int Nq, int Nk, int d,
                        float scale, int causal, void* stream) {
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_map(&mq, q, d, Nq, BH) || !make_map(&mk, k, d, Nk, B * Hkv) ||
      !make_map(&mv, v, d, Nk, B * Hkv) || !make_map(&mdo, dout, d, Nq, BH) ||
      !make_dq_map(&mdq, static_cast<char*>(workspace) + sm100_backward_dq_offset(BH, Nq), d, Nq, BH))
    return map_failed();
  return from_cuda(sm100_backward(mq, mk, mv, mdo, mdq, o, dout, lse, dq, dk, dv, workspace, B, H,
                                  Hkv, Nq, Nk, d, scale, causal ? 1 : 0,
                                  static_cast<cudaStream_t>(stream)));
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
  fa_status s = check_shape(B, H, N, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (workspace == nullptr || ws_bytes < ws_bytes_for(B, H, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;
  return backward_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, H, N, N, d, scale, causal,
                       stream);
}

fa_status fa_backward_gqa(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv,
                          void* workspace, size_t ws_bytes, int B, int H, int Hkv, int N, int d,
                          float scale, int causal, void* stream) {
  fa_status s = check_shape(B, H, N, d, scale);
  if (s != FA_OK) return s;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (workspace == nullptr || ws_bytes < ws_bytes_for(B, H, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;
  return backward_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, N, N, d, scale, causal,
                       stream);
}

fa_status fa_backward_qk(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq, int Nk,
                         int d, float scale, int causal, void* stream) {
  fa_status s = check_shape(B, H, Nq, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_shape(B, H, Nk, d, scale)) != FA_OK) return s;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (workspace == nullptr || ws_bytes < ws_bytes_for(B, H, Nq, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;
  return backward_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nk, d, scale,
                       causal, stream);
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
  cudaError_t e = bwd_preprocess(false, o, dout, dsum, (long long)BH * N, d, st);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  return from_cuda(simt_backward(false, q, k, v, dout, lse, dsum, dq, dk, dv, BH, N, d, scale,
                                 causal ? 1 : 0, st));
}

fa_status fa_debug_wait_timeout(void* stream) {
  fa::wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return from_cuda(cudaGetLastError());
}

fa_status fa_check_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word)) != cudaSuccess) return FA_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_CUDA;
  return word ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
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
  }
  return "unknown status";
}

}  // extern "C"

// ------------------------------------------------------------------------
// Allocation-free backward: the scratch of fa_backward in a fixed device
// array.  Host code must not pass the array's name to a kernel (on the host it
// names a stand-in, not device memory); its device address is looked up once
// per device with cudaGetSymbolAddress while that device is current.

namespace fa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_BACKWARD_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on error).
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
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
  void* scratch = noalloc_scratch();
  if (scratch == nullptr) return FA_ERR_CUDA;
  return backward_bf16(q, k, v, o, dout, lse, dq, dk, dv, scratch, B, H, H, N, N, d, scale, causal,
                       stream);
}
