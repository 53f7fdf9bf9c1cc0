// Internal launch entry points of the kernels (host side).  Not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// CUDA-core kernels (fa_simt.cu)
cudaError_t simt_forward(bool bf16, const void* q, const void* k, const void* v, void* o, float* lse,
                         int BH, int N, int d, float scale, int causal, cudaStream_t st);
cudaError_t bwd_preprocess(bool bf16, const void* o, const void* dout, float* dsum, long long rows,
                           int d, cudaStream_t st);
cudaError_t simt_backward(bool bf16, const void* q, const void* k, const void* v, const void* dout,
                          const float* lse, const float* dsum, void* dq, void* dk, void* dv, int BH,
                          int N, int d, float scale, int causal, cudaStream_t st);

// tcgen05 forward (fa_fwd_sm100.cu).  Tensor maps: 3-D bf16 views
// {d, Nq, heads} of Q (B*H heads) and {d, Nk, heads} of K and V (B*Hkv heads)
// with a {64, 128, 1} box and 128-byte swizzle.  Hkv divides H (Hkv = H: plain
// multi-head attention).  Under the causal mask key j is visible to query i iff
// j <= i + Nk - Nq.
cudaError_t sm100_forward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          void* o, float* lse, int B, int H, int Hkv, int Nq, int Nk, int d,
                          float scale, int causal, cudaStream_t st);

// tcgen05 backward (fa_bwd_sm100.cu): preprocess, main and dQ-convert kernels.
// Workspace layout (N = query rows): LSE*log2(e) [BH, Npad], D [BH, Npad],
// fp32 dQ [BH, N, d].
size_t sm100_backward_workspace(int BH, int N, int d);
// byte offset of the fp32 dQ accumulator inside the workspace
size_t sm100_backward_dq_offset(int BH, int N);
// mq, mdo, mdq over Nq rows; mk, mv over Nk rows.
// mdq: 3-D fp32 view {d, Nq, B*H} of the accumulator, box {32, 32, 1}, 128-byte swizzle
cudaError_t sm100_backward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mdo, const CUtensorMap& mdq, const void* o,
                           const void* dout, const float* lse,
                           void* dq, void* dk, void* dv, void* workspace, int B, int H, int Hkv,
                           int Nq, int Nk, int d, float scale, int causal, cudaStream_t st);

}  // namespace fa
