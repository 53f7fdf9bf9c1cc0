/*
 * fa.h -- C ABI of libfa.so: exact tiled (FlashAttention-style) attention for
 * NVIDIA B200 (sm_100a).
 *
 * What is computed.  For every batch b and head h, with S = scale * Q K^T
 * (Q, K, V of shape N x d), the exact attention
 *     O   = softmax(S) V
 *     LSE = log(sum_j exp(S_ij))          (natural log, per query row i)
 * as defined by the standard-attention listing of the page "Atención Flash:
 * Revolucionando la Eficiencia de los Modelos de Transformador" (unite.ai),
 * section "Atención Flash", evaluated block by block with a running row maximum
 * m and running sum l (same page, "La Matemática detrás de la Atención Flash",
 * formulas 1-2, and "Detalles de Implementación"; page "FlashAttention
 * algorithm part 3" (nisoo.com), "SafeSoftmax con Calcolo Normalizzatore
 * Online"), so the N x N score matrix never reaches device memory.  With
 * causal != 0, key j is visible to query i only when j <= i (square, top-left
 * aligned).  The backward pass recomputes the score blocks from Q, K and the
 * saved LSE (the "recomputation" idea of both pages) and returns dQ, dK, dV of
 * L = sum(O * dO).
 *
 * Layout.  Q, K, V, O, dO, dQ, dK, dV: [B, H, N, d] contiguous, row-major
 * (d fastest).  LSE: [B, H, N] float32, contiguous.
 *
 * Ownership.  Every pointer is caller-owned DEVICE memory on the current CUDA
 * device.  The library allocates nothing; the backward pass's scratch comes
 * from the caller (fa_backward_workspace_size).
 *
 * Asynchrony.  Work is enqueued on `stream` (a cudaStream_t; 0 = legacy
 * default stream) and the call returns at once.  The returned status covers
 * argument checks and launch errors.  Kernels bound every wait they make; a
 * wait that runs out records FA_ERR_DEVICE_TIMEOUT in a device-side status
 * word instead of hanging, which fa_check_device_status reports.
 *
 * Concurrency.  Calls on different streams may run at the same time.  Each
 * forward launch draws its work items from one of 256 scheduler slots, taken
 * round-robin, under an owner tag of its own; if two launches in flight ever
 * meet on one slot, the later draws stop and FA_ERR_DEVICE_STATE is recorded
 * rather than items being lost silently.  A forward launch captured into a CUDA
 * graph keeps its slot and tag in every replay, so replays of one captured
 * graph must not overlap each other on the GPU (replays in stream order are
 * fine).
 *
 * Limits.  d in {64, 128}; N >= 1 (any N: ragged tails are masked);
 * 1 <= B*H <= 65535*128; pointers 16-byte aligned; scale finite and > 0.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, bad scale */
  FA_ERR_UNSUPPORTED = 2,    /* head dim / device not supported */
  FA_ERR_MISALIGNED = 3,     /* a pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
  FA_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  FA_ERR_DEVICE_TIMEOUT = 6, /* a kernel's bounded wait ran out */
  FA_ERR_DEVICE_STATE = 7    /* a kernel found device-side state it cannot trust
                                (a scheduler slot held by another launch, a
                                misaligned shared-memory base) and skipped work */
} fa_status;

/* Forward pass, bf16 storage, fp32 accumulation and statistics.
 * q, k, v: const bf16 [B,H,N,d]; o: bf16 [B,H,N,d] (written); lse: fp32
 * [B,H,N] (written).  scale multiplies Q K^T (1/sqrt(d) for the pages'
 * scaled dot product).  Runs the tcgen05/TMEM/TMA kernel on sm_100a. */
fa_status fa_forward(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int N, int d, float scale, int causal, void* stream);

/* Grouped-query / multi-query forward: K and V carry Hkv heads, [B,Hkv,N,d];
 * query head h attends with key/value head h / (H / Hkv) (the attention
 * variants named in "Atención Flash-2" of the unite.ai page).  Hkv must divide
 * H; Hkv == H is fa_forward, Hkv == 1 is multi-query attention.  Q, O: [B,H,N,d];
 * LSE: [B,H,N].  Errors as fa_forward, plus FA_ERR_INVALID_ARG for a bad Hkv. */
fa_status fa_forward_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int Hkv, int N, int d, float scale, int causal,
                         void* stream);

/* Forward pass with separate query and key lengths (bf16, grouped-query heads
 * as in fa_forward_gqa).  q, o: [B,H,Nq,d]; k, v: [B,Hkv,Nk,d]; lse: fp32
 * [B,H,Nq].  Nq = Nk is fa_forward_gqa.  Under the causal mask, which the pages
 * define only for square attention, the mask is aligned at the bottom right:
 * key j is visible to query i iff j <= i + (Nk - Nq), so the last query sees
 * every key (the suffix of a longer square problem, e.g. new queries against
 * a key/value cache).  A query that sees no key (i < Nq - Nk) gets O = 0 and
 * LSE = -inf.  Errors as for fa_forward; Nq and Nk must both be >= 1. */
fa_status fa_forward_qk(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                        void* stream);

/* FP8 forward (the FP8 support named in "Atención Flash-3" of the unite.ai page):
 * Q, K, V stored as e4m3 (OCP FP8 E4M3, 1 byte per element) with one scale per
 * tensor, so the values they stand for are q_descale * Q, k_descale * K and
 * v_descale * V.  Both GEMMs run on the tensor cores in e4m3 with fp32
 * accumulation: S = Q K^T, then P (the exponentials, at most 2^8) is rounded to
 * e4m3 for P V.  Results as fa_forward_qk on the values they stand for:
 *   O   = softmax(scale * q_descale * k_descale * Q K^T) (v_descale * V), bf16;
 *   LSE = log sum_j exp(scale * q_descale * k_descale * q_i . k_j), fp32.
 * q: [B,H,Nq,d], k, v: [B,Hkv,Nk,d] (e4m3); o: bf16 [B,H,Nq,d]; lse: fp32
 * [B,H,Nq].  Grouped-query heads, lengths and causal mask as fa_forward_qk.
 * The descales must be finite and > 0 (FA_ERR_INVALID_ARG otherwise); other
 * errors as fa_forward.  The rounding of P to e4m3 (relative error up to 2^-4
 * per element) makes O accurate to about 3 % rather than bf16's 0.5 %. */
fa_status fa_forward_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Hkv, int Nq, int Nk, int d, float scale, float q_descale,
                         float k_descale, float v_descale, int causal, void* stream);

/* Forward pass with fp32 storage (q, k, v, o are float [B,H,N,d]); fp32
 * arithmetic on CUDA cores.  Same definition, same LSE convention. */
fa_status fa_forward_fp32(const float* q, const float* k, const float* v, float* o, float* lse,
                          int B, int H, int N, int d, float scale, int causal, void* stream);

/* Bytes of device scratch fa_backward needs for this shape (0 on bad sizes):
 * -LSE*log2(e) and -D_i = -sum_c dO[i,c] * O[i,c] padded to whole 128-row tiles
 * (fp32, [B,H,Npad]), an fp32 dQ accumulator ([B,H,N,d]) and 256 bytes for the
 * work-item counters of the persistent main kernel, each segment rounded up to
 * 256 bytes. */
size_t fa_backward_workspace_size(int B, int H, int N, int d);

/* Backward pass, bf16 storage, fp32 accumulation.
 * q, k, v, o, dout: const bf16 [B,H,N,d] (o and lse as written by fa_forward
 * for the same q, k, v, scale, causal); lse: const fp32 [B,H,N];
 * dq, dk, dv: bf16 [B,H,N,d] (written);
 * workspace: device scratch of ws_bytes >= fa_backward_workspace_size(...),
 * 16-byte aligned, contents ignored on entry and undefined on return.
 * Computes dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)),
 * dQ = scale * dS K, dK = scale * dS^T Q with P recomputed from Q, K and LSE. */
fa_status fa_backward(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      void* workspace, size_t ws_bytes, int B, int H, int N, int d,
                      float scale, int causal, void* stream);

/* Grouped-query / multi-query backward, the gradient of fa_forward_gqa:
 * k, v, dk, dv are [B,Hkv,N,d]; dK and dV of a key/value head sum the
 * contributions of its H / Hkv query heads.  q, o, dout, dq: [B,H,N,d].
 * Workspace: fa_backward_workspace_size(B, H, N, d) (query heads). */
fa_status fa_backward_gqa(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv,
                          void* workspace, size_t ws_bytes, int B, int H, int Hkv, int N, int d,
                          float scale, int causal, void* stream);

/* Backward pass of fa_forward_qk: q, o, dout, dq: [B,H,Nq,d]; k, v, dk, dv:
 * [B,Hkv,Nk,d]; lse: [B,H,Nq] as written by fa_forward_qk (rows with LSE = -inf
 * have P = 0 and contribute nothing).  Workspace:
 * fa_backward_workspace_size(B, H, Nq, d), i.e. sized by the query rows. */
fa_status fa_backward_qk(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq, int Nk,
                         int d, float scale, int causal, void* stream);

/* Deterministic backward pass: results as fa_backward_qk (Hkv = H and Nq = Nk
 * give fa_backward), computed so that they are the same bit for bit from run to
 * run.  dK and dV come from one CTA per key tile as always; dQ comes from a
 * separate pass, one CTA per 128-row query tile that walks its key tiles in a
 * fixed order and sums dS K in tensor memory, instead of partial sums added
 * into an fp32 accumulator in whatever order the CTAs finish.  It executes
 * 7 N^2 d multiply-adds per head instead of 5 (S and dP are formed twice), and
 * the workspace (same size rule as fa_backward) holds only the LSE and D rows.
 * Errors as fa_backward. */
fa_status fa_backward_deterministic(const void* q, const void* k, const void* v, const void* o,
                                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                   void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq,
                                   int Nk, int d, float scale, int causal, void* stream);

/* Stages of the bf16 backward pass, for callers that schedule or time them one
 * by one (fa_backward runs all three in one call):
 *   FA_STAGE_PREPROCESS  -LSE*log2(e) and -D_i = -sum_c dO[i,c] O[i,c] into the
 *                        workspace, and a zeroed fp32 dQ accumulator there;
 *   FA_STAGE_MAIN        P recomputed from Q, K and LSE; dK and dV written; the
 *                        partial dQ = dS K of every key tile added into the
 *                        accumulator;
 *   FA_STAGE_DQ_CONVERT  dQ = scale * accumulator, rounded to bf16.
 * With FA_STAGE_DETERMINISTIC added, the stages are those of
 * fa_backward_deterministic: the preprocess leaves no accumulator, the main
 * stage writes dK and dV only, and FA_STAGE_DQ_CONVERT runs the separate dQ pass.
 * Arguments as fa_backward_qk (Hkv = H and Nq = Nk for the square multi-head
 * case) plus `stages`, a nonzero OR of the three stage flags, optionally with
 * FA_STAGE_DETERMINISTIC (the same choice for every stage of one backward).  A later stage reads what an
 * earlier one left in the workspace, so run them in this order, on one stream
 * (or ordered by events), with the same arguments and workspace and nothing
 * else writing the workspace in between. */
#define FA_STAGE_PREPROCESS 1
#define FA_STAGE_MAIN 2
#define FA_STAGE_DQ_CONVERT 4
#define FA_STAGE_DETERMINISTIC 8
fa_status fa_backward_stages(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv,
                             void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq,
                             int Nk, int d, float scale, int causal, int stages, void* stream);

/* Backward pass with fp32 storage (all tensors float); CUDA-core arithmetic.
 * Workspace as for fa_backward. */
fa_status fa_backward_fp32(const float* q, const float* k, const float* v, const float* o,
                           const float* dout, const float* lse, float* dq, float* dk, float* dv,
                           void* workspace, size_t ws_bytes, int B, int H, int N, int d,
                           float scale, int causal, void* stream);

/* Largest scratch fa_backward_noalloc can use: 64 MiB, a fixed array inside the
 * library that every GPU which loads the library keeps until process exit. */
#define FA_BACKWARD_NOALLOC_MAX_BYTES ((size_t)64 << 20)

/* Backward pass like fa_backward, for callers that cannot allocate device
 * memory: for example a plug-in that only ever receives the input and output
 * buffers of a host framework which owns all device memory, or a caller that
 * must not issue cudaMalloc/cudaFree because those calls can synchronise the
 * whole device and stall other work.  Same arguments, layout and results as
 * fa_backward minus the workspace: the scratch lives in a fixed device array
 * inside the library (FA_BACKWARD_NOALLOC_MAX_BYTES), so this call allocates
 * nothing.  Shapes whose scratch (fa_backward_workspace_size) exceeds that
 * limit return FA_ERR_WORKSPACE.  The first call in each CUDA context of a
 * device (the first call on the device, and the first one after a
 * cudaDeviceReset) looks up the array's device address there; make that call
 * before any stream capture.
 * All calls share the one array and the kernels re-initialise what they read,
 * but two calls whose work overlaps on the GPU (different streams, no ordering
 * between them) race on it.  The pages have no counterpart to this entry
 * point; it exists only for callers without an allocator. */
fa_status fa_backward_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, float scale, int causal, void* stream);

/* Diagnostic: launches one warp that waits on a barrier nothing ever completes,
 * so the kernels' bounded wait runs out (after about 2 s) and records
 * FA_ERR_DEVICE_TIMEOUT in the status word, then returns; the context stays
 * usable.  Lets callers check their error path; not part of the attention
 * computation (the pages have no counterpart).  Returns FA_OK once launched. */
fa_status fa_debug_wait_timeout(void* stream);

/* Diagnostic: enqueues on `stream` a write that marks every slot of the forward
 * pass's work-item scheduler as held by a launch that never finished, the state
 * a crashed or abandoned launch could leave behind.  The next forward launch on
 * the device then stops drawing work and records FA_ERR_DEVICE_STATE (outputs
 * incomplete) instead of computing with the stale slot, and
 * fa_check_device_status reports it and frees the slots.  Lets callers check
 * that error path; the pages have no counterpart.  Returns FA_OK once enqueued. */
fa_status fa_debug_hold_scheduler(void* stream);

/* Synchronises `stream`, then reads and clears the current device's status
 * word.  FA_ERR_DEVICE_TIMEOUT if a kernel gave up a wait since the last call,
 * FA_ERR_DEVICE_STATE if a kernel skipped work because its device-side state was
 * inconsistent (outputs written since the last call may be incomplete),
 * FA_ERR_CUDA if synchronisation failed, FA_OK otherwise.  After reporting an
 * error it also frees every slot of the forward pass's work-item scheduler, so
 * call it while no other fa_* work is running on the device. */
fa_status fa_check_device_status(void* stream);

/* Text of the most recent CUDA error that an fa_* call on the calling thread
 * ran into (after FA_ERR_CUDA), or "no error".  Valid until the next fa_* call
 * on the same thread. */
const char* fa_last_error(void);

/* Static, NUL-terminated description of a status code. */
const char* fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
