// CUDA-core (SIMT) kernels: the fp32-storage forward and backward passes, and
// the backward preprocess D_i = sum_c dO[i,c] * O[i,c] shared by both backward
// paths.
//
// Forward: one CTA per (64-row query block, batch*head).  Key/value blocks of 64
// rows stream through shared memory; per query row the CTA keeps the running
// maximum m and running sum l and rescales the output accumulator by
// exp(m_old - m_new) when m moves (the tiled loop of the page "Atención Flash:
// Revolucionando la Eficiencia de los Modelos de Transformador", section
// "Detalles de Implementación", with the output kept unnormalised until the
// end).  Exponentials are taken base 2 on pre-scaled scores.
//
// Backward: scores are recomputed block by block from Q, K and the saved LSE
// (the "recomputation" idea of the same page and of "FlashAttention algorithm
// part 3").  One kernel accumulates dK and dV per key block; a second pass
// accumulates dQ per query block.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fa_device.cuh"
#include "fa_kernels.h"

namespace fa {
namespace simt {

constexpr int BQ = 64;
constexpr int BK = 64;
constexpr int NT = 256;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Copies `rows` rows of a [N, D] head slice starting at row r0 into a padded
// fp32 shared tile (row stride D + 1); rows past N are zero.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* dst, const T* src, int r0, int N, int rows) {
  for (int idx = threadIdx.x; idx < rows * D; idx += NT) {
    const int r = idx / D, c = idx % D;
    const int g = r0 + r;
    dst[r * (D + 1) + c] = g < N ? to_f<T>(src[(size_t)g * D + c]) : 0.f;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT) fwd_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                 const T* __restrict__ v, T* __restrict__ o,
                                                 float* __restrict__ lse, int N, float scale,
                                                 int causal) {
  extern __shared__ float sm[];
  float* sQ = sm;                       // [BQ][D+1]
  float* sK = sQ + BQ * (D + 1);        // [BK][D+1]
  float* sV = sK + BK * (D + 1);        // [BK][D+1]
  float* sP = sV + BK * (D + 1);        // [BQ][BK+1]
  float* sM = sP + BQ * (BK + 1);       // running max (raw score units)
  float* sL = sM + BQ;                  // running sum
  float* sA = sL + BQ;                  // per-row rescale factor of this block

  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * BQ;
  const size_t off = (size_t)bh * N * D;
  const float c = scale * kLog2e;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  constexpr int OC = D / 16;  // output columns per thread

  load_tile<T, D>(sQ, q + off, q0, N, BQ);
  if (tid < BQ) {
    sM[tid] = -INFINITY;
    sL[tid] = 0.f;
  }
  float acc[4][OC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < OC; ++j) acc[i][j] = 0.f;

  const int kend = causal ? min(N, q0 + BQ) : N;
  for (int k0 = 0; k0 < kend; k0 += BK) {
    __syncthreads();
    load_tile<T, D>(sK, k + off, k0, N, BK);
    load_tile<T, D>(sV, v + off, k0, N, BK);
    __syncthreads();
    // S block: thread owns rows ty*4.., columns tx + 16*j
    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
    for (int e = 0; e < D; ++e) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sQ[(ty * 4 + i) * (D + 1) + e];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sK[(tx + 16 * j) * (D + 1) + e];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], b[j], s[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int qi = q0 + ty * 4 + i, kj = k0 + tx + 16 * j;
        const bool masked = kj >= N || (causal && kj > qi);
        sP[(ty * 4 + i) * (BK + 1) + tx + 16 * j] = masked ? -INFINITY : s[i][j];
      }
    __syncthreads();
    // online softmax: warp w owns rows w*8 .. w*8+7, lane owns columns lane, lane+32
    {
      const int w = tid / 32, lane = tid % 32;
      for (int rr = 0; rr < 8; ++rr) {
        const int r = w * 8 + rr;
        float x0 = sP[r * (BK + 1) + lane], x1 = sP[r * (BK + 1) + lane + 32];
        float mx = fmaxf(x0, x1);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
        const float m_old = sM[r];
        const float m_new = fmaxf(m_old, mx);
        // a row with no visible key so far keeps m = -inf; use 0 as the pivot
        const float piv = m_new == -INFINITY ? 0.f : m_new;
        const float p0 = exp2f((x0 - piv) * c), p1 = exp2f((x1 - piv) * c);
        float sum = p0 + p1;
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, sh);
        sP[r * (BK + 1) + lane] = p0;
        sP[r * (BK + 1) + lane + 32] = p1;
        __syncwarp();
        if (lane == 0) {
          const float alpha = exp2f((m_old - piv) * c);
          sA[r] = alpha;
          sL[r] = sL[r] * alpha + sum;
          sM[r] = m_new;
        }
      }
    }
    __syncthreads();
    // O block update: thread owns rows ty*4.., columns tx + 16*j
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float alpha = sA[ty * 4 + i];
#pragma unroll
      for (int j = 0; j < OC; ++j) acc[i][j] *= alpha;
    }
    for (int kk = 0; kk < BK; ++kk) {
      float p[4], vv[OC];
#pragma unroll
      for (int i = 0; i < 4; ++i) p[i] = sP[(ty * 4 + i) * (BK + 1) + kk];
#pragma unroll
      for (int j = 0; j < OC; ++j) vv[j] = sV[kk * (D + 1) + tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < OC; ++j) acc[i][j] = fmaf(p[i], vv[j], acc[i][j]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, qi = q0 + r;
    if (qi >= N) continue;
    const float l = sL[r];
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int j = 0; j < OC; ++j) o[off + (size_t)qi * D + tx + 16 * j] = from_f<T>(acc[i][j] * inv);
    if (tx == 0) lse[(size_t)bh * N + qi] = l > 0.f ? sM[r] * scale + logf(l) : -INFINITY;
  }
}

// D_i = sum_c dO[i,c] * O[i,c]; one warp per row.
template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_preprocess_kernel(const T* __restrict__ o,
                                                            const T* __restrict__ dout,
                                                            float* __restrict__ dsum,
                                                            long long rows) {
  const long long row = (long long)blockIdx.x * (NT / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < D; c += 32)
    acc = fmaf(to_f<T>(o[row * D + c]), to_f<T>(dout[row * D + c]), acc);
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
  if (lane == 0) dsum[row] = acc;
}

// Recomputes P^T for one (key block, query block) pair into sP (rows = keys,
// columns = queries) and dS^T into sS.  sLse is LSE * log2(e) per query.
template <int D>
__device__ __forceinline__ void block_p_ds(const float* sK, const float* sV, const float* sQ,
                                           const float* sdO, const float* sLse, const float* sD,
                                           float* sP, float* sS, int k0, int q0, int N,
                                           float c, int causal) {
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float s[4][4], dp[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) s[i][j] = dp[i][j] = 0.f;
  for (int e = 0; e < D; ++e) {
    float kr[4], vr[4], qc[4], oc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kr[i] = sK[(ty * 4 + i) * (D + 1) + e];
      vr[i] = sV[(ty * 4 + i) * (D + 1) + e];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      qc[j] = sQ[(tx + 16 * j) * (D + 1) + e];
      oc[j] = sdO[(tx + 16 * j) * (D + 1) + e];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s[i][j] = fmaf(kr[i], qc[j], s[i][j]);
        dp[i][j] = fmaf(vr[i], oc[j], dp[i][j]);
      }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int kj = k0 + ty * 4 + i, qi = q0 + tx + 16 * j;
      const bool masked = kj >= N || qi >= N || (causal && kj > qi);
      const float p = masked ? 0.f : exp2f(s[i][j] * c - sLse[tx + 16 * j]);
      sP[(ty * 4 + i) * (BQ + 1) + tx + 16 * j] = p;
      sS[(ty * 4 + i) * (BQ + 1) + tx + 16 * j] = p * (dp[i][j] - sD[tx + 16 * j]);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                      const T* __restrict__ v, const T* __restrict__ dout,
                                                      const float* __restrict__ lse,
                                                      const float* __restrict__ dsum, T* __restrict__ dk,
                                                      T* __restrict__ dv, int N, float scale, int causal) {
  extern __shared__ float sm[];
  float* sK = sm;
  float* sV = sK + BK * (D + 1);
  float* sQ = sV + BK * (D + 1);
  float* sdO = sQ + BQ * (D + 1);
  float* sP = sdO + BQ * (D + 1);   // [BK][BQ+1]
  float* sS = sP + BK * (BQ + 1);   // [BK][BQ+1]
  float* sLse = sS + BK * (BQ + 1);
  float* sD = sLse + BQ;

  const int bh = blockIdx.y, k0 = blockIdx.x * BK;
  const size_t off = (size_t)bh * N * D;
  const float c = scale * kLog2e;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  constexpr int OC = D / 16;
  load_tile<T, D>(sK, k + off, k0, N, BK);
  load_tile<T, D>(sV, v + off, k0, N, BK);
  float adk[4][OC], adv[4][OC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < OC; ++j) adk[i][j] = adv[i][j] = 0.f;

  const int qstart = causal ? (k0 / BQ) * BQ : 0;
  for (int q0 = qstart; q0 < N; q0 += BQ) {
    __syncthreads();
    load_tile<T, D>(sQ, q + off, q0, N, BQ);
    load_tile<T, D>(sdO, dout + off, q0, N, BQ);
    if (tid < BQ) {
      const int qi = q0 + tid;
      sLse[tid] = qi < N ? lse[(size_t)bh * N + qi] * kLog2e : 0.f;
      sD[tid] = qi < N ? dsum[(size_t)bh * N + qi] : 0.f;
    }
    __syncthreads();
    block_p_ds<D>(sK, sV, sQ, sdO, sLse, sD, sP, sS, k0, q0, N, c, causal);
    __syncthreads();
    for (int qq = 0; qq < BQ; ++qq) {
      float p[4], ds[4], dov[OC], qv[OC];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        p[i] = sP[(ty * 4 + i) * (BQ + 1) + qq];
        ds[i] = sS[(ty * 4 + i) * (BQ + 1) + qq];
      }
#pragma unroll
      for (int j = 0; j < OC; ++j) {
        dov[j] = sdO[qq * (D + 1) + tx + 16 * j];
        qv[j] = sQ[qq * (D + 1) + tx + 16 * j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < OC; ++j) {
          adv[i][j] = fmaf(p[i], dov[j], adv[i][j]);
          adk[i][j] = fmaf(ds[i], qv[j], adk[i][j]);
        }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int kj = k0 + ty * 4 + i;
    if (kj >= N) continue;
#pragma unroll
    for (int j = 0; j < OC; ++j) {
      dk[off + (size_t)kj * D + tx + 16 * j] = from_f<T>(adk[i][j] * scale);
      dv[off + (size_t)kj * D + tx + 16 * j] = from_f<T>(adv[i][j]);
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(NT) bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                    const T* __restrict__ v, const T* __restrict__ dout,
                                                    const float* __restrict__ lse,
                                                    const float* __restrict__ dsum, T* __restrict__ dq,
                                                    int N, float scale, int causal) {
  extern __shared__ float sm[];
  float* sK = sm;
  float* sV = sK + BK * (D + 1);
  float* sQ = sV + BK * (D + 1);
  float* sdO = sQ + BQ * (D + 1);
  float* sP = sdO + BQ * (D + 1);
  float* sS = sP + BK * (BQ + 1);
  float* sLse = sS + BK * (BQ + 1);
  float* sD = sLse + BQ;

  const int bh = blockIdx.y, q0 = blockIdx.x * BQ;
  const size_t off = (size_t)bh * N * D;
  const float c = scale * kLog2e;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  constexpr int OC = D / 16;
  load_tile<T, D>(sQ, q + off, q0, N, BQ);
  load_tile<T, D>(sdO, dout + off, q0, N, BQ);
  if (tid < BQ) {
    const int qi = q0 + tid;
    sLse[tid] = qi < N ? lse[(size_t)bh * N + qi] * kLog2e : 0.f;
    sD[tid] = qi < N ? dsum[(size_t)bh * N + qi] : 0.f;
  }
  float adq[4][OC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < OC; ++j) adq[i][j] = 0.f;
  const int kend = causal ? min(N, q0 + BQ) : N;
  for (int k0 = 0; k0 < kend; k0 += BK) {
    __syncthreads();
    load_tile<T, D>(sK, k + off, k0, N, BK);
    load_tile<T, D>(sV, v + off, k0, N, BK);
    __syncthreads();
    block_p_ds<D>(sK, sV, sQ, sdO, sLse, sD, sP, sS, k0, q0, N, c, causal);
    __syncthreads();
    // dQ[q][:] += sum_k dS^T[k][q] K[k][:]; thread owns query rows ty*4.., columns tx+16j
    for (int kk = 0; kk < BK; ++kk) {
      float ds[4], kv[OC];
#pragma unroll
      for (int i = 0; i < 4; ++i) ds[i] = sS[kk * (BQ + 1) + ty * 4 + i];
#pragma unroll
      for (int j = 0; j < OC; ++j) kv[j] = sK[kk * (D + 1) + tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < OC; ++j) adq[i][j] = fmaf(ds[i], kv[j], adq[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qi = q0 + ty * 4 + i;
    if (qi >= N) continue;
#pragma unroll
    for (int j = 0; j < OC; ++j) dq[off + (size_t)qi * D + tx + 16 * j] = from_f<T>(adq[i][j] * scale);
  }
}

template <int D>
constexpr size_t fwd_smem() {
  return sizeof(float) * (size_t)(3 * 64 * (D + 1) + 64 * 65 + 3 * 64);
}
template <int D>
constexpr size_t bwd_smem() {
  return sizeof(float) * (size_t)(4 * 64 * (D + 1) + 2 * 64 * 65 + 2 * 64);
}

template <typename T, int D>
cudaError_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int BH,
                       int N, float scale, int causal, cudaStream_t st) {
  const size_t smem = fwd_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(fwd_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((N + BQ - 1) / BQ, BH);
  fwd_kernel<T, D><<<grid, NT, smem, st>>>((const T*)q, (const T*)k, (const T*)v, (T*)o, lse, N,
                                           scale, causal);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_bwd_pre(const void* o, const void* dout, float* dsum, long long rows,
                           cudaStream_t st) {
  const long long blocks = (rows + NT / 32 - 1) / (NT / 32);
  bwd_preprocess_kernel<T, D><<<(unsigned)blocks, NT, 0, st>>>((const T*)o, (const T*)dout, dsum, rows);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                       const float* dsum, void* dq, void* dk, void* dv, int BH, int N, float scale,
                       int causal, cudaStream_t st) {
  const size_t smem = bwd_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((N + 63) / 64, BH);
  bwd_dkdv_kernel<T, D><<<grid, NT, smem, st>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dout,
                                                lse, dsum, (T*)dk, (T*)dv, N, scale, causal);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<T, D><<<grid, NT, smem, st>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dout,
                                              lse, dsum, (T*)dq, N, scale, causal);
  return cudaGetLastError();
}

}  // namespace simt

cudaError_t simt_forward(bool bf16, const void* q, const void* k, const void* v, void* o, float* lse,
                         int BH, int N, int d, float scale, int causal, cudaStream_t st) {
  if (bf16)
    return d == 64 ? simt::launch_fwd<__nv_bfloat16, 64>(q, k, v, o, lse, BH, N, scale, causal, st)
                   : simt::launch_fwd<__nv_bfloat16, 128>(q, k, v, o, lse, BH, N, scale, causal, st);
  return d == 64 ? simt::launch_fwd<float, 64>(q, k, v, o, lse, BH, N, scale, causal, st)
                 : simt::launch_fwd<float, 128>(q, k, v, o, lse, BH, N, scale, causal, st);
}

cudaError_t bwd_preprocess(bool bf16, const void* o, const void* dout, float* dsum, long long rows,
                           int d, cudaStream_t st) {
  if (bf16)
    return d == 64 ? simt::launch_bwd_pre<__nv_bfloat16, 64>(o, dout, dsum, rows, st)
                   : simt::launch_bwd_pre<__nv_bfloat16, 128>(o, dout, dsum, rows, st);
  return d == 64 ? simt::launch_bwd_pre<float, 64>(o, dout, dsum, rows, st)
                 : simt::launch_bwd_pre<float, 128>(o, dout, dsum, rows, st);
}

cudaError_t simt_backward(bool bf16, const void* q, const void* k, const void* v, const void* dout,
                          const float* lse, const float* dsum, void* dq, void* dk, void* dv, int BH,
                          int N, int d, float scale, int causal, cudaStream_t st) {
  if (bf16)
    return d == 64 ? simt::launch_bwd<__nv_bfloat16, 64>(q, k, v, dout, lse, dsum, dq, dk, dv, BH, N,
                                                         scale, causal, st)
                   : simt::launch_bwd<__nv_bfloat16, 128>(q, k, v, dout, lse, dsum, dq, dk, dv, BH, N,
                                                          scale, causal, st);
  return d == 64 ? simt::launch_bwd<float, 64>(q, k, v, dout, lse, dsum, dq, dk, dv, BH, N, scale,
                                               causal, st)
                 : simt::launch_bwd<float, 128>(q, k, v, dout, lse, dsum, dq, dk, dv, BH, N, scale,
                                                causal, st);
}

}  // namespace fa
