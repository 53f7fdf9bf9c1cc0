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
// fp8: Q, K, V are e4m3 (maps of uint8 elements, box {min(d, 128), 128, 1}, swizzle
// of min(d, 128) bytes); the scores are scale * qk_descale * (Q K^T of the stored
// values) and O = v_descale * P V / l.  bf16: qk_descale = v_descale = 1.
// mo: bf16 view {d, Nq, B*H} of O, box {64, 32, 1}, 128-byte swizzle (stores at d = 64)
cudaError_t sm100_forward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mo, void* o, float* lse, int B, int H, int Hkv, int Nq, int Nk, int d,
                          float scale, int causal, bool fp8, float qk_descale, float v_descale,
                          cudaStream_t st);

// Frees every slot of the forward's work-item scheduler on the current device
// (synchronous).  Only for recovery after a reported device error, with no
// forward launch in flight.
cudaError_t sm100_forward_reset_scheduler();
// Diagnostic: enqueues on `st` a write that marks every scheduler slot as held by
// a launch that never finishes, so the next forward launch reports
// kStateTicketOwner instead of computing.
cudaError_t sm100_forward_hold_scheduler(cudaStream_t st);

// tcgen05 backward (fa_bwd_sm100.cu): preprocess, main and dQ-convert kernels.
// Workspace layout (N = query rows): LSE*log2(e) [BH, Npad], D [BH, Npad],
// fp32 dQ [BH, N, d].
size_t sm100_backward_workspace(int BH, int N, int d);
// byte offset of the fp32 dQ accumulator inside the workspace
size_t sm100_backward_dq_offset(int BH, int N);
// `stages` selects the launches (kStagePreprocess | kStageMain | kStageConvert
// for the whole pass); each later stage reads what the earlier ones left in the
// workspace.
// With kStageDeterministic the preprocess leaves the accumulator alone, the main
// stage computes dK and dV only, and the last stage is the separate dQ pass.
constexpr int kStagePreprocess = 1, kStageMain = 2, kStageConvert = 4, kStageAll = 7;
constexpr int kStageDeterministic = 8;
// mq, mdo, mdq over Nq rows; mk, mv over Nk rows.
// mdq: 3-D fp32 view {d, Nq, B*H} of the accumulator, box {32, 32, 1}, 128-byte swizzle
// mdk, mdv: bf16 views {d, Nk, B*Hkv} of dK and dV, box {64, 32, 1}, 128-byte swizzle
cudaError_t sm100_backward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mdo, const CUtensorMap& mdq, const CUtensorMap& mdk,
                           const CUtensorMap& mdv, const void* o,
                           const void* dout, const float* lse,
                           void* dq, void* dk, void* dv, void* workspace, int B, int H, int Hkv,
                           int Nq, int Nk, int d, float scale, int causal, int stages,
                           cudaStream_t st);

}  // namespace fa
