// Backward pass on sm_100a.  The score tiles are recomputed from Q, K and the
// saved LSE instead of being stored (the "recomputation" idea of the page
// "Atención Flash: Revolucionando la Eficiencia de los Modelos de Transformador"
// and of "FlashAttention algorithm part 3"); the gradient formulas are the
// closed form of the softmax Jacobian:
//   P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//   D_i = sum_c dO[i,c] O[i,c],  dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three kernels:
//   preprocess  -D and -LSE * log2(e) (padded to whole 128-row tiles: padding
//               rows get +inf for LSE so their probabilities vanish), a zeroed
//               fp32 dQ accumulator and the main kernel's zeroed ticket counters;
//   main        persistent, one CTA per SM; a work item is one 128-key tile of
//               one key/value head.  For every 128-row query tile it recomputes
//               S^T = K Q^T and dP^T = V dO^T in tensor memory, forms P^T (to
//               tensor memory) and dS (to shared memory), then accumulates
//               dV += P^T dO and dK += dS^T Q in tensor memory and computes the
//               partial dQ = dS K, which a reduce group adds into the fp32
//               accumulator with bulk tensor reduce-adds;
//   convert     dQ = scale * accumulator, rounded to bf16.
//
// Main-kernel CTA layout (512 threads, registers rebalanced with setmaxnreg):
//   warps 0-7   P / dS computation (thread = key row = tensor-memory lane, two
//               warps per row quarter, one per half of the query columns) and
//               the dK / dV epilogue (TMA stores of 32-row boxes)
//   warps 8-11  dQ drain: tensor memory -> registers -> shared staging -> bulk
//               tensor reduce-add into the fp32 accumulator
//   warp  12    TMA producer: draws work items; K, V once per item (prefetched
//               into L2 when the item is drawn); Q_i, dO_i, LSE_i, D_i per
//               query tile
//   warp  13    tensor-memory allocator and MMA issuer (warps 14-15 idle)
// Tensor memory: S^T at column 0 (P^T of query columns 64h.. packed at column 64h),
// dP^T / dQ at 128, dV at 256, dK at 256+d.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>

#include "fa_device.cuh"
#include "fa_kernels.h"

namespace fa {
namespace bwd {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int NTHREADS = 512;     // four warpgroups
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
// Register split (setmaxnreg).  The launch gives every thread 128 registers,
// 512 * 128 = 65536 in all; the shares below sum to 128 * (2*136 + 144 + 96) =
// 65536, exactly that pool.
constexpr int kRegsCompute = 136;  // warpgroups 0 and 1
constexpr int kRegsReduce = 144;   // warpgroup 2
constexpr int kRegsControl = 96;   // warpgroup 3: producer, MMA issuer, two idle warps
static_assert(128 * (2 * kRegsCompute + kRegsReduce + kRegsControl) <= 512 * 128,
              "register split exceeds the launch allocation");
constexpr int kMaxNst = 3;  // Q stages at most (Cfg<D>::NST)
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  // Q stages (with the LSE / D rows): two at d = 128, where shared memory is
  // full; three at d = 64, so Q(i+1) can be loaded one query tile earlier
  static constexpr int NST = D == 64 ? 3 : 2;
  static constexpr int TILE = BN * D * 2;  // bytes of one 128-row bf16 tile
  static constexpr int CHUNK = BN * 128;   // one 64-column swizzle chunk of a tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;                   // stage s at OFF_Q + s * TILE
  static constexpr int OFF_DO = OFF_Q + NST * TILE;        // dO: one buffer
  static constexpr int OFF_DS = OFF_DO + TILE;
  static constexpr int OFF_STG = OFF_DS + BM * BN * 2;     // dQ staging: 4 warps x 2 x 4 KB
  static constexpr int STG_BYTES = 32 * 32 * 4;            // 32 rows x 32 fp32 columns
  static constexpr int OFF_VEC = OFF_STG + 4 * 2 * STG_BYTES;  // LSE2 / D vectors per stage
  static constexpr int OFF_BAR = OFF_VEC + NST * 2 * BM * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;
  // partial dQ: over dP^T at d = 128 (tensor memory is full), in its own
  // columns at d = 64, where dP^T(i+1) then need not wait for dQ(i)'s drain
  static constexpr bool DQ_SHARED = D == 128;
  static constexpr uint32_t T_DQ = DQ_SHARED ? T_DP : 256 + 2 * D;
  static constexpr uint32_t IDESC_S = idesc_bf16(BN, BM, 0, 0);   // K-major x K-major
  static constexpr uint32_t IDESC_DQ = idesc_bf16(BM, D, 1, 1);   // dS (MN) x K (MN)
  static constexpr uint32_t IDESC_DKV = idesc_bf16(BN, D, 0, 1);  // P^T/dS^T (K) x dO/Q (MN)
};

struct Params {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dq_acc;       // [BH, N, d] fp32
  const float* lse2;   // [BH, Npad]  -LSE * log2(e), -inf on padding rows
  const float* dsum;   // [BH, Npad]  -D, 0 on padding rows
  int BH;      // query heads B*H
  int BHkv;    // key/value heads B*Hkv
  int H;       // query heads per batch
  int G;       // query heads per key/value head (H / Hkv; 1 without grouping)
  int Nq;              // query rows
  int Nk;              // key rows
  int off;             // Nk - Nq: under the causal mask key j is visible to query i iff j <= i + off
  int Npad;            // Nq rounded up to whole 128-row tiles (the LSE / D vectors)
  int nq;              // number of query tiles = Npad / 128
  int nkv;             // number of key tiles
  int chunk;           // key/value heads per locality chunk
  int items;           // work items: key tiles x key/value heads
  unsigned long long* tickets;  // [0] items handed out past the first gridDim.x, [1] CTAs done
  float scale;
  float scale_log2;
  int causal;
};

constexpr int kItemRing = 2;  // work items the producer may hand out ahead

struct Bars {
  uint64_t kv_full;
  uint64_t kv_empty;       // the item's last GEMM reading K or V has completed
  uint64_t q_full[kMaxNst];    // Q tile + LSE2 / D vectors of a stage
  uint64_t q_empty[kMaxNst];
  uint64_t do_full;        // dO tile (single buffer)
  uint64_t do_empty;
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t p_full;
  uint64_t ds_full;
  uint64_t ds_free;
  uint64_t dq_full;
  uint64_t dq_empty;
  uint64_t acc_full;       // the item's dK and dV are complete in tensor memory
  uint64_t drain;
  uint64_t it_full[kItemRing];   // the producer has written it_item[s]
  uint64_t it_empty[kItemRing];  // every reader has taken it_item[s]
  int it_item[kItemRing];
  uint32_t tmem_base;
};
static_assert(sizeof(Bars) <= 256, "barrier block over its shared-memory slot");

// Work item -> key tile j and key/value head.  The key/value heads are cut into
// chunks whose K, V, Q, dO and fp32 dQ accumulator fit in L2 together; chunk by
// chunk, items run key-tile-major, so under the causal mask (tile j sees query
// tiles from about j on) the heavy items come first, and CTAs take them in
// this order as they become free.
struct Item {
  int j;      // key tile
  int bkv;    // key/value head
  int i0;     // first query tile with a row that sees a key of tile j
  int nqi;    // query tiles per query head
  int niter;  // query tiles of the item: every query head of the group
  int bhq0;   // first query head of the group
};

__device__ __forceinline__ Item decode_item(const Params& p, int item) {
  const int per_chunk = p.chunk * p.nkv;
  const int chunk_id = item / per_chunk, w_in = item - chunk_id * per_chunk;
  const int h0 = chunk_id * p.chunk, hn = min(p.chunk, p.BHkv - h0);
  Item w;
  w.j = w_in / hn;
  w.bkv = h0 + (w_in - w.j * hn);
  // the causal mask is aligned bottom right: key k is visible to query r iff k <= r + off
  w.i0 = p.causal ? max(0, w.j * BN - p.off) / BM : 0;
  w.nqi = p.nq - w.i0;
  w.niter = p.G * w.nqi;
  w.bhq0 = (w.bkv / (p.H / p.G)) * p.H + (w.bkv % (p.H / p.G)) * p.G;
  return w;
}


// Bulk tensor reduce-add of a shared-memory box into global memory (async proxy).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src_smem, int c0,
                                                  int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src_smem), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float4 ld_shared_v4(uint32_t addr) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "r"(addr));
  return r;
}

// kDQ: also form the partial dQ = dS K of every query tile and add it into the
// fp32 accumulator (the single-pass backward); without it the kernel computes
// dK and dV only and dQ comes from dq_kernel.
//
// Persistent: one CTA per SM takes work items (key/value head, 128-key tile) in
// the order of decode_item, its first item b = blockIdx.x and every later one
// from the launch's ticket counter.  Barrier phases, the Q / dO stages and the
// tensor-memory buffers carry over from item to item, so the next item's loads
// and first GEMMs overlap the current item's last dQ reduction and its dK / dV
// epilogue.
template <int D, bool kDQ>
__global__ void __launch_bounds__(NTHREADS, 1)
    main_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mdo,
                const __grid_constant__ CUtensorMap mdq, const __grid_constant__ CUtensorMap mdk,
                const __grid_constant__ CUtensorMap mdv, const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled tiles need a 1024-byte aligned base and the layout uses the
  // whole opt-in shared memory, so there is no slack to re-align: refuse to run
  // on a misaligned base instead of computing garbage.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_state_error(kStateMisalignedSmem);
    return;
  }
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sDS = smem + C::OFF_DS;
  float* sVec = reinterpret_cast<float*>(smem + C::OFF_VEC);  // [C::NST][2][BM]
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kItemReaders = kDQ ? 13 : 9;  // MMA warp, 8 compute warps (+ 4 reduce warps)

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->do_full, 1);
    mbar_init(&bars->do_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_full, 2 * 128);
    mbar_init(&bars->ds_full, 2 * 128);
    mbar_init(&bars->ds_free, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, 128);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->drain, 1);
    for (int s = 0; s < kItemRing; ++s) {
      mbar_init(&bars->it_full[s], 1);
      mbar_init(&bars->it_empty[s], kItemReaders);
    }
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&mq);
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
    tma_prefetch_desc(&mdo);
    tma_prefetch_desc(&mdq);
    tma_prefetch_desc(&mdk);
    tma_prefetch_desc(&mdv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // The r-th work item of this CTA from the producer's ring (>= p.items: none
  // left).  Every lane of the calling warp reads it; lane 0 then frees the entry.
  auto take_item = [&](int r, int& item, unsigned int site) -> bool {
    const int s = r % kItemRing;
    if (!mbar_wait(&bars->it_full[s], (uint32_t)((r / kItemRing) & 1), site)) return false;
    item = *reinterpret_cast<volatile int*>(&bars->it_item[s]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->it_empty[s]);
    return true;
  };

  if (warp >= 12) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
   if (warp == kProducerWarp) {
    if (lane == 0) {
      bool ok = true;
      int g = 0;      // query tiles (Q, dO) loaded so far, over all items
      int nkv = 0;    // items whose K and V were loaded
      int dog = 0;    // dO tiles loaded
      // loads of one query tile: Q, the LSE2 / D rows into stage g % C::NST, dO
      auto load_tile = [&](const Item& w, int it) -> bool {
        const int st = g % C::NST, round = g / C::NST;
        const int i = w.i0 + it % w.nqi, bh = w.bhq0 + it / w.nqi;
        if (round > 0 && !mbar_wait(&bars->q_empty[st], (round - 1) & 1, 32)) return false;
        uint8_t* sQ = smem + C::OFF_Q + st * C::TILE;
        float* vec = sVec + st * 2 * BM;
        mbar_arrive_expect_tx(&bars->q_full[st], C::TILE + 2 * BM * 4);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ + c * C::CHUNK, &mq, &bars->q_full[st], c * 64, i * BM, bh);
        const size_t voff = (size_t)bh * p.Npad + (size_t)i * BM;
        bulk_load(vec, p.lse2 + voff, BM * 4, &bars->q_full[st]);
        bulk_load(vec + BM, p.dsum + voff, BM * 4, &bars->q_full[st]);
        ++g;
        // dO of a tile reuses the single dO buffer once dV of the tile before has read it
        if (dog > 0 && !mbar_wait(&bars->do_empty, (dog - 1) & 1, 47)) return false;
        mbar_arrive_expect_tx(&bars->do_full, C::TILE);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + C::OFF_DO + c * C::CHUNK, &mdo, &bars->do_full, c * 64, i * BM, bh);
        ++dog;
        return true;
      };
      for (int r = 0; ok; ++r) {
        // A CTA draws its next item once it has issued the loads of the current
        // one, about two query tiles before that item ends.
        const int item = r == 0 ? (int)blockIdx.x : (int)gridDim.x + (int)atomicAdd(p.tickets, 1ull);
        const int s = r % kItemRing;
        if (r >= kItemRing) ok = mbar_wait(&bars->it_empty[s], (uint32_t)((r / kItemRing - 1) & 1), 50);
        if (!ok) break;
        *reinterpret_cast<volatile int*>(&bars->it_item[s]) = item;
        mbar_arrive(&bars->it_full[s]);
        if (item >= p.items) break;
        const Item w = decode_item(p, item);
        // K and V come from DRAM (each key tile is read by one item only); start
        // bringing them into L2 now, while the current item still runs
        if (r > 0)
          for (int c = 0; c < D / 64; ++c) {
            tma_prefetch_l2_3d(&mk, c * 64, w.j * BN, w.bkv);
            tma_prefetch_l2_3d(&mv, c * 64, w.j * BN, w.bkv);
          }
        // the first query tile's Q and dO are fetched before K and V, whose
        // buffers free only when the previous item's last GEMM reading them ends
        ok = load_tile(w, 0);
        if (ok && r > 0) ok = mbar_wait(&bars->kv_empty, (r - 1) & 1, 51);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::TILE);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sK + c * C::CHUNK, &mk, &bars->kv_full, c * 64, w.j * BN, w.bkv);
          tma_load_3d(sV + c * C::CHUNK, &mv, &bars->kv_full, c * 64, w.j * BN, w.bkv);
        }
        ++nkv;
        for (int it = 1; it < w.niter && ok; ++it) ok = load_tile(w, it);
      }
      // This CTA draws no more tickets; the last one to get here resets the
      // counters for the next launch on this workspace.
      __threadfence();
      if (atomicAdd(p.tickets + 1, 1ull) == (unsigned long long)gridDim.x - 1) {
        atomicExch(p.tickets, 0ull);
        atomicExch(p.tickets + 1, 0ull);
      }
      // no copy into this CTA's shared memory may still be in flight at exit
      if (nkv > 0) mbar_wait(&bars->kv_full, (nkv - 1) & 1, 33);
      for (int s = 0; s < C::NST && s < g; ++s) {
        const int last = s + ((g - 1 - s) / C::NST) * C::NST;
        mbar_wait(&bars->q_full[s], (last / C::NST) & 1, 34);
      }
      if (dog > 0) mbar_wait(&bars->do_full, (dog - 1) & 1, 48);
    }
   } else if (warp == kMmaWarp) {
    bool ok = true;
    int g = 0;  // query tiles over all items
    // One descriptor for the start of shared memory (the K tile, K-major); every
    // operand is a compile-time offset from it (one add per MMA), a Q stage a
    // per-tile one, and an MN-major operand differs only in LBO.
    const uint64_t d0 = sdesc_sw128(smem_u32(smem), 16, 1024);
    constexpr uint64_t kToMn = (uint64_t)((C::CHUNK >> 4) - 1) << 16;  // LBO 16 B -> CHUNK
    auto q_desc = [&](int gt) { return sdesc_at(opaque(d0), C::OFF_Q + (gt % C::NST) * C::TILE); };
    // S^T = K Q^T  (keys x queries), K = d
    auto issue_s = [&](int gt) {
      const uint64_t dq = q_desc(gt), dk = opaque(d0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t ko = (kk / 4) * C::CHUNK + (kk % 4) * 32;
        mma_ss(tmem + C::T_S, sdesc_at(dk, C::OFF_K + ko), sdesc_at(dq, ko), C::IDESC_S, kk > 0);
      }
      mma_commit(&bars->s_full);
    };
    // dP^T = V dO^T
    auto issue_dp = [&]() {
      const uint64_t d = opaque(d0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t ko = (kk / 4) * C::CHUNK + (kk % 4) * 32;
        mma_ss(tmem + C::T_DP, sdesc_at(d, C::OFF_V + ko), sdesc_at(d, C::OFF_DO + ko), C::IDESC_S,
               kk > 0);
      }
      mma_commit(&bars->dp_full);
    };
    // dV += P^T dO  (keys x d), K = 128 queries, P^T from tensor memory (queries
    // 64h .. 64h+63 packed at column 64h); the item's first tile starts the sum
    auto issue_dv = [&](bool first) {
      const uint64_t d = opaque(d0) + kToMn;
#pragma unroll
      for (int kk = 0; kk < BM / 16; ++kk)
        mma_ts(tmem + C::T_DV, tmem + C::T_S + 64 * (kk / 4) + 8 * (kk % 4),
               sdesc_at(d, C::OFF_DO + kk * 2048), C::IDESC_DKV, (!first || kk > 0) ? 1u : 0u);
      mma_commit(&bars->do_empty);
    };
    // Order per item: S(0), dP(0), then per query tile i
    //   dV(i) | S(i+1) | dK(i) | dQ(i) | dP(i+1)
    // S(i+1) is issued as soon as dV(i) has read P^T(i) from the S columns (the
    // compute warps no longer touch them in tile i), so it runs while they form
    // dS(i); dK(i) and dQ(i) then run while they form P(i+1), dK first so that
    // Q(i)'s stage is free for Q(i+2) one GEMM earlier.  The next item's
    // S(0) follows the last dQ in issue order; its dP(0) waits, like every dP,
    // until the dQ drawn from the same columns has been drained.
    for (int r = 0; ok; ++r) {
      int item = p.items;
      ok = take_item(r, item, 52);
      if (!ok || item >= p.items) break;
      const Item w = decode_item(p, item);
      if (lane == 0) {
        ok = mbar_wait(&bars->kv_full, r & 1, 35);
        if (ok) ok = mbar_wait(&bars->q_full[g % C::NST], (g / C::NST) & 1, 36);
        if (ok) {
          tc_fence_after();
          issue_s(g);
          if (kDQ && C::DQ_SHARED && g > 0) ok = mbar_wait(&bars->dq_empty, (g - 1) & 1, 37);
        }
        if (ok) ok = mbar_wait(&bars->do_full, g & 1, 49);
        if (ok) {
          tc_fence_after();
          issue_dp();
        }
        for (int it = 0; it < w.niter && ok; ++it, ++g) {
          const int st = g % C::NST;
          const bool more = it + 1 < w.niter;
          ok = mbar_wait(&bars->p_full, g & 1, 46);
          if (!ok) break;
          tc_fence_after();
          issue_dv(it == 0);
          if (!kDQ && !more) mma_commit(&bars->kv_empty);  // the item's last reads of K and V are issued
          if (more) {
            ok = mbar_wait(&bars->q_full[(g + 1) % C::NST], ((g + 1) / C::NST) & 1, 36);
            if (!ok) break;
            tc_fence_after();
            issue_s(g + 1);
          }
          ok = mbar_wait(&bars->ds_full, g & 1, 38);
          if (!ok) break;
          tc_fence_after();
          // dK += dS^T Q  (keys x d), K = 128 queries; before dQ, so that Q's
          // stage frees for the tile after next one GEMM earlier
          const uint64_t dq_mn = q_desc(g) + kToMn, dds = opaque(d0);
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk) {
            const uint32_t ko = (kk / 4) * C::CHUNK + (kk % 4) * 32;
            mma_ss(tmem + C::T_DK, sdesc_at(dds, C::OFF_DS + ko), sdesc_at(dq_mn, kk * 2048), C::IDESC_DKV,
                   (it > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars->q_empty[st]);
          if constexpr (kDQ) {
            // dQ_part = dS K  (queries x d), K = 128 keys; written over dP^T at
            // d = 128.  In its own columns (d = 64) it overwrites the previous
            // tile's partial dQ, once the reduce warps have drained that.
            if (!C::DQ_SHARED && g > 0) {
              ok = mbar_wait(&bars->dq_empty, (g - 1) & 1, 37);
              if (!ok) break;
              tc_fence_after();
            }
            const uint64_t dmn = opaque(d0) + kToMn;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ss(tmem + C::T_DQ, sdesc_at(dmn, C::OFF_DS + kk * 2048), sdesc_at(dmn, C::OFF_K + kk * 2048),
                     C::IDESC_DQ, kk > 0);
            mma_commit(&bars->dq_full);
            if (!more) mma_commit(&bars->kv_empty);
          }
          mma_commit(&bars->ds_free);
          if (!more) mma_commit(&bars->acc_full);  // dK, dV of the item complete
          if (more) {
            // dP^T(i+1) overwrites the columns dQ(i) was drained from; without dQ
            // the compute warps have read dP^T(i) before they published dS(i)
            if constexpr (kDQ && C::DQ_SHARED) ok = mbar_wait(&bars->dq_empty, g & 1, 37);
            if (ok) ok = mbar_wait(&bars->do_full, (g + 1) & 1, 49);
            if (!ok) break;
            tc_fence_after();
            issue_dp();
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      g = __shfl_sync(0xffffffffu, g, 0);
    }
    if (lane == 0) {
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, 39);
    }
    __syncwarp();
  } 
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
    // Compute warps 0-7.  Warp w owns tensor-memory lane quarter w % 4 (key rows
    // 32*(w%4) .. +31 for S^T/dP^T/dK/dV) and column half h = w / 4: query
    // columns 64h .. 64h+63 of P^T and dS, dK / dV columns (d/2)h .. +d/2-1.  Per
    // query tile: P^T -> tensor memory, dS -> shared memory; per item: dK, dV.
    const int qw = warp % 4, h = warp / 4;
    const int r = qw * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S;
    const uint32_t tDP = tmem + lane_off + C::T_DP;
    const float c = p.scale_log2;
    const uint32_t ds_row = smem_u32(sDS) + h * C::CHUNK + r * 128;
    bool ok = true;
    int g = 0;
    for (int ri = 0; ok; ++ri) {
      int item = p.items;
      ok = take_item(ri, item, 53);
      if (!ok || item >= p.items) break;
      const Item w = decode_item(p, item);
      const int kr = w.j * BN + r;
      const bool key_ok = kr < p.Nk;
      for (int it = 0; it < w.niter && ok; ++it, ++g) {
        const int i = w.i0 + it % w.nqi, st = g % C::NST;
        const uint32_t lse2 = smem_u32(sVec + st * 2 * BM) + h * 64 * 4;  // -LSE*log2(e), my columns
        const uint32_t dsv = lse2 + BM * 4;                                // -D, my columns
        ok = mbar_wait(&bars->q_full[st], (g / C::NST) & 1, 40);
        if (ok) ok = mbar_wait(&bars->s_full, g & 1, 41);
        if (!ok) break;
        tc_fence_after();
        float pr[64];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t v[32];
          tmem_ld32(tS + h * 64 + cc * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) pr[cc * 32 + e] = __uint_as_float(v[e]);
        }
        tmem_wait_ld();
        // Masked keys get S = -inf before the exponentials (P = 0): key j*BN + r is
        // hidden from query i*BM + 64h + col iff col < hide (above the causal
        // diagonal), and from every query if it is past Nk.
        {
          const int hide = !key_ok ? 64 : p.causal ? min(max(r + (w.j - i) * BN - p.off - h * 64, 0), 64) : 0;
          if (hide > 0) {
#pragma unroll
            for (int col = 0; col < 64; ++col)
              if (col < hide) pr[col] = -INFINITY;
          }
        }
        const uint64_t c2 = f2_pack(c, c);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l4 = ld_shared_v4(lse2 + c4 * 16);
          // x = s * c - LSE * log2(e) for two columns at a time (the vector holds -LSE * log2(e))
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(pr[4 * c4], pr[4 * c4 + 1]), c2, f2_pack(l4.x, l4.y)), x0, x1);
          f2_unpack(f2_fma(f2_pack(pr[4 * c4 + 2], pr[4 * c4 + 3]), c2, f2_pack(l4.z, l4.w)), x2, x3);
          pr[4 * c4] = ex2(x0);
          pr[4 * c4 + 1] = ex2(x1);
          pr[4 * c4 + 2] = ex2(x2);
          pr[4 * c4 + 3] = ex2(x3);
        }
        {
          uint32_t v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = pack_bf16x2(pr[2 * e], pr[2 * e + 1]);
          // packed P^T of my 64 query columns over the first 32 of my own S columns
          tmem_st32(tS + h * 64, v);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full);
        ok = mbar_wait(&bars->dp_full, g & 1, 42);
        if (ok && g > 0) ok = mbar_wait(&bars->ds_free, (g - 1) & 1, 43);
        if (!ok) break;
        if (it == 0 && ri > 0) {
          // this warp's dK / dV stores of the previous item must have read its
          // part of the dS buffer
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t v[32];
          tmem_ld32(tDP + h * 64 + cc * 32, v);
          tmem_wait_ld();
          uint32_t wv[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const int c0 = cc * 32 + 4 * e4;
            const float4 dd = ld_shared_v4(dsv + c0 * 4);
            // dS = P * (dP - D), two columns per packed instruction (the vector holds -D)
            float d0, d1, d2, d3;
            f2_unpack(f2_mul(f2_pack(pr[c0], pr[c0 + 1]),
                             f2_add(f2_pack(__uint_as_float(v[4 * e4]), __uint_as_float(v[4 * e4 + 1])),
                                    f2_pack(dd.x, dd.y))), d0, d1);
            f2_unpack(f2_mul(f2_pack(pr[c0 + 2], pr[c0 + 3]),
                             f2_add(f2_pack(__uint_as_float(v[4 * e4 + 2]), __uint_as_float(v[4 * e4 + 3])),
                                    f2_pack(dd.z, dd.w))), d2, d3);
            wv[2 * e4] = pack_bf16x2(d0, d1);
            wv[2 * e4 + 1] = pack_bf16x2(d2, d3);
          }
          // row r of the dS^T tile in the 128-byte swizzled layout: chunk h,
          // 16-byte units cc*4 .. cc*4+3 XOR (r % 8)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t unit = (uint32_t)(cc * 4 + u) ^ (uint32_t)(r & 7);
            st_shared_v4(ds_row + unit * 16, wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->ds_full);
      }
      // dK, dV of the item: tensor memory -> bf16 rows.  The next item's first
      // dV and dK overwrite these columns only after this warp has published that
      // item's first P and dS, i.e. after the loads below have completed.
      if (ok) ok = mbar_wait(&bars->acc_full, ri & 1, 44);
      if (!ok) break;
      tc_fence_after();
      // dK, dV of the item: tensor memory -> bf16 -> this warp's 32 x 128-byte
      // part of the dS buffer (the part it writes dS to; the item's last dK and
      // dQ GEMMs have read it) in the 128-byte-swizzled layout -> one TMA store
      // of a 32-row box by lane 0.  Warp (qw, h) stores rows 32qw .. 32qw+31:
      // at d = 128 columns 64h .. 64h+63 of dV, then of dK; at d = 64 all
      // columns of dV (h = 0) or dK (h = 1).  Rows past Nk are clipped by the
      // tensor map, and a box that starts past Nk is not stored.
      {
        constexpr int NT = D == 128 ? 2 : 1;
        const uint32_t region = smem_u32(sDS) + h * C::CHUNK + qw * 32 * 128;
        const int row0 = w.j * BN + qw * 32;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const bool isK = D == 128 ? (t == 1) : (h == 1);
          const uint32_t tsrc = tmem + lane_off + (isK ? C::T_DK : C::T_DV) + (D == 128 ? h * 64 : 0);
          const float mul = isK ? p.scale : 1.f;
          uint32_t wv[32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t v[32];
            tmem_ld32(tsrc + cc * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              wv[cc * 16 + e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
          }
          if (t > 0) {
            // the store of the first tensor must have read the region
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
          }
#pragma unroll
          for (int u = 0; u < 8; ++u)
            st_shared_v4(region + lane * 128 + ((u ^ (lane & 7)) << 4), wv[4 * u], wv[4 * u + 1], wv[4 * u + 2],
                         wv[4 * u + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < p.Nk) tma_store_3d(isK ? &mdk : &mdv, region, D == 128 ? h * 64 : 0, row0, w.bkv);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
      }
      tc_fence_before();
    }
    // no store may still be reading this CTA's shared memory at exit
    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    __syncwarp();
  } else if constexpr (!kDQ) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsReduce));
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsReduce));
    // dQ reduce warps 8-11: warp w drains query rows 32*(w%4) .. +31 of each
    // tile's partial dQ from tensor memory, then, 32 columns at a time, writes
    // them to its own 128-byte-swizzled 4 KB staging buffer (two per warp, used
    // in turn) and lane 0 adds the buffer into the fp32 accumulator with one
    // bulk tensor reduce-add.  No per-thread global atomics.
    const int qw = warp % 4;
    const uint32_t tQ = tmem + ((uint32_t)(qw * 32) << 16) + C::T_DQ;
    const uint32_t stg0 = smem_u32(smem + C::OFF_STG + qw * 2 * C::STG_BYTES);
    bool ok = true;
    int chunk = 0, g = 0;
    for (int ri = 0; ok; ++ri) {
      int item = p.items;
      ok = take_item(ri, item, 54);
      if (!ok || item >= p.items) break;
      const Item w = decode_item(p, item);
      for (int it = 0; it < w.niter && ok; ++it, ++g) {
        ok = mbar_wait(&bars->dq_full, g & 1, 45);
        if (!ok) break;
        tc_fence_after();
        uint32_t v[D / 32][32];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tQ + cc * 32, v[cc]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->dq_empty);
        const int row0 = (w.i0 + it % w.nqi) * BM + qw * 32, bh = w.bhq0 + it / w.nqi;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc, ++chunk) {
          const uint32_t buf = stg0 + (chunk & 1) * C::STG_BYTES;
          if (chunk >= 2) {
            // the reduce that read this buffer two chunks ago must be done with it
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
          }
#pragma unroll
          for (int u = 0; u < 8; ++u)
            st_shared_v4(buf + lane * 128 + ((u ^ (lane & 7)) << 4), v[cc][4 * u], v[cc][4 * u + 1],
                         v[cc][4 * u + 2], v[cc][4 * u + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past N are clipped by the tensor map; a box wholly past N is skipped
            if (row0 < p.Nq) tma_reduce_add_3d(&mdq, buf, cc * 32, row0, bh);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
      }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// -D, -LSE*log2(e) (padded; the main kernel adds them) and, for the single-pass
// backward, a zeroed dQ accumulator.  A row of O and dO is D/8 lanes' worth of
// 16-byte loads, so a warp covers 256/D rows at once; every access is a 16-byte
// vector.  (Four rows per lane with all loads issued first measured slower: the
// 64-bit row arithmetic per pass and the lower occupancy outweighed the extra
// loads in flight.)
template <int D, bool kZeroAcc>
__global__ void __launch_bounds__(256) preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dout,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ lse2,
                                                         float* __restrict__ dsum,
                                                         float* __restrict__ dq_acc,
                                                         unsigned long long* __restrict__ tickets,
                                                         int BH, int N, int Npad) {
  constexpr int L = D / 8;          // lanes per row
  if (blockIdx.x == 0 && threadIdx.x < 2) tickets[threadIdx.x] = 0ull;  // the main kernel's scheduler
  constexpr int RPW = 32 / L;       // rows per warp
  const int lane = threadIdx.x % 32;
  const long long gr = ((long long)blockIdx.x * 8 + threadIdx.x / 32) * RPW + lane / L;
  // BH * Npad is a multiple of 128, hence of RPW: whole warps leave here together
  if (gr >= (long long)BH * Npad) return;
  const int bh = (int)(gr / Npad), row = (int)(gr % Npad);
  const int c = (lane % L) * 8;
  float acc = 0.f;
  if (row < N) {
    const size_t off = ((size_t)bh * N + row) * D + c;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + off);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 af = __bfloat1622float2(a2[i]), gf = __bfloat1622float2(g2[i]);
      acc = fmaf(af.x, gf.x, acc);
      acc = fmaf(af.y, gf.y, acc);
    }
    if constexpr (kZeroAcc) {
      float4* z = reinterpret_cast<float4*>(dq_acc + off);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  // the L lanes of a row are consecutive and L-aligned: reduce within them
#pragma unroll
  for (int sh = L / 2; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
  if (lane % L == 0) {
    if (row >= N) {
      lse2[gr] = -INFINITY;  // padding rows: probability exp2(-inf) = 0
      dsum[gr] = 0.f;
    } else {
      dsum[gr] = -acc;
      // a row that saw no key in the forward (LSE = -inf) gets probability 0 too
      const float l = lse[(size_t)bh * N + row];
      lse2[gr] = l == -INFINITY ? -INFINITY : -l * kLog2e;
    }
  }
}

// dQ = scale * accumulator in bf16: sixteen values per thread (four 16-byte
// loads issued together, two 16-byte stores).
__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ acc,
                                                         __nv_bfloat16* __restrict__ dq, long long n16,
                                                         float scale) {
  for (long long idx = (long long)blockIdx.x * 256 + threadIdx.x; idx < n16;
       idx += (long long)gridDim.x * 256) {
    const float4* src = reinterpret_cast<const float4*>(acc) + 4 * idx;
    float4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __ldcs(src + k);  // read once: streaming
    uint4 w[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      w[k].x = pack_bf16x2(v[2 * k].x * scale, v[2 * k].y * scale);
      w[k].y = pack_bf16x2(v[2 * k].z * scale, v[2 * k].w * scale);
      w[k].z = pack_bf16x2(v[2 * k + 1].x * scale, v[2 * k + 1].y * scale);
      w[k].w = pack_bf16x2(v[2 * k + 1].z * scale, v[2 * k + 1].w * scale);
    }
    uint4* dst = reinterpret_cast<uint4*>(dq) + 2 * idx;
    dst[0] = w[0];
    dst[1] = w[1];
  }
}

// ---------------------------------------------------------------- dQ pass
//
// The deterministic dQ: one CTA per (128-row query tile, query head) walks the
// key tiles the tile sees in a fixed order and accumulates
//   dQ = scale * sum_j dS_j K_j,  dS_j = P_j * (dP_j - D),  P_j = exp2(S_j c - LSE2),
//   S_j = Q K_j^T,  dP_j = dO V_j^T
// in tensor memory, so no partial sums cross CTAs and the result does not
// depend on scheduling.  Q and dO stay in tensor memory for the whole pass
// (copied in once from their TMA tiles), which makes all three GEMMs of a key
// tile tensor-memory-A forms that read only K_j or V_j from shared memory.
//
// CTA layout (384 threads, registers rebalanced as in the forward):
//   warps 0-7  dS (thread = query row = tensor-memory lane; two warps per lane
//              quarter, one per half of the key columns) and the dQ epilogue
//   warp  8    TMA producer: Q, dO and the LSE2 / D rows once, then K_j, V_j
//   warp  9    tensor-memory allocator and MMA issuer (warps 10-11 idle)
// Tensor memory: Q (bf16, D/2 columns) at 0, dO at D/2, S at D, dP at D + 128
// (dS in bf16 written over the first half of each warp's own dP columns), dQ at
// D + 256.
namespace dqp {

constexpr int NTHREADS = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRegsCompute = 208;
constexpr int kRegsControl = 88;
static_assert(128 * (2 * kRegsCompute + kRegsControl) <= NTHREADS * 168,
              "register split exceeds the launch allocation");

template <int D>
struct Cfg {
  static constexpr int TILE = BN * D * 2;
  static constexpr int CHUNK = BN * 128;
  static constexpr int NSLOT = D == 128 ? 5 : 8;  // K/V ring slots
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_RING = 2 * TILE;
  static constexpr int OFF_VEC = OFF_RING + NSLOT * TILE;  // LSE2 row values, then -D
  static constexpr int OFF_BAR = OFF_VEC + 2 * BM * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_Q = 0, T_DO = D / 2, T_S = D, T_DP = D + 128, T_DQ = D + 256;
  static constexpr uint32_t IDESC_S = idesc_bf16(BM, BN, 0, 0);   // Q (tmem) x K (K-major)
  static constexpr uint32_t IDESC_DQ = idesc_bf16(BM, D, 0, 1);   // dS (tmem) x K (MN-major)
  static_assert(T_DQ + D <= TMEM_COLS, "tensor memory over budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory over the per-block limit");
};

struct Params {
  __nv_bfloat16* dq;
  const float* lse2;  // [BH, Npad]  -LSE * log2(e), -inf on padding rows
  const float* dsum;  // [BH, Npad]  -D
  int BH, H, G, Nq, Nk, off, Npad, nq, chunk, causal;
  float scale, scale_log2;
};

struct Bars {
  uint64_t q_full;   // Q, dO tiles and the row vectors
  uint64_t q_ready;  // Q and dO copied into tensor memory
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t s_full, s_free, dp_full, ds_full, dq_done, drain;
  uint32_t tmem_base;
};

// key tiles the query tile starting at row q0 sees (as the forward's tiles_for)
__device__ __forceinline__ int key_tiles(int q0, const Params& p) {
  const int nkv = (p.Nk + BN - 1) / BN;
  if (!p.causal) return nkv;
  const int kmax = min(q0 + BM - 1, p.Nq - 1) + p.off;
  return kmax < 0 ? 0 : min(nkv, kmax / BN + 1);
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    dq_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
              const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mdo,
              const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  float* sVec = reinterpret_cast<float*>(smem + C::OFF_VEC);
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // CTA -> (query head, query tile): heads in L2-sized chunks, within a chunk
  // the tiles that see the most keys first
  const int per_chunk = p.chunk * p.nq;
  const int chunk_id = blockIdx.x / per_chunk, w_in = blockIdx.x - chunk_id * per_chunk;
  const int h0 = chunk_id * p.chunk, hn = min(p.chunk, p.BH - h0);
  const int rank = w_in / hn;
  const int bh = h0 + (w_in - rank * hn);
  const int i = p.causal ? p.nq - 1 - rank : rank;  // query tile
  const int bkv = (bh / p.H) * (p.H / p.G) + (bh % p.H) / p.G;
  const int n = key_tiles(i * BM, p);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_ready, 256);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 256);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->ds_full, 256);
    mbar_init(&bars->dq_done, 1);
    mbar_init(&bars->drain, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&mq);
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
    tma_prefetch_desc(&mdo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (warp == kProducerWarp && lane == 0) {
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE + 2 * BM * 4);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + C::OFF_Q + c * C::CHUNK, &mq, &bars->q_full, c * 64, i * BM, bh);
        tma_load_3d(smem + C::OFF_DO + c * C::CHUNK, &mdo, &bars->q_full, c * 64, i * BM, bh);
      }
      const size_t voff = (size_t)bh * p.Npad + (size_t)i * BM;
      bulk_load(sVec, p.lse2 + voff, BM * 4, &bars->q_full);
      bulk_load(sVec + BM, p.dsum + voff, BM * 4, &bars->q_full);
      bool ok = true;
      // ring sequence K_0, V_0, K_1, V_1, ...
      for (int s2 = 0; s2 < 2 * n && ok; ++s2) {
        const int slot = s2 % C::NSLOT, round = s2 / C::NSLOT;
        if (round > 0) ok = mbar_wait(&bars->kv_empty[slot], (round - 1) & 1, 60);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->kv_full[slot], C::TILE);
        const CUtensorMap* m = (s2 & 1) ? &mv : &mk;
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + C::OFF_RING + slot * C::TILE + c * C::CHUNK, m, &bars->kv_full[slot], c * 64,
                      (s2 >> 1) * BN, bkv);
      }
      // no copy into this CTA's shared memory may be in flight at exit
      mbar_wait(&bars->q_full, 0, 61);
      const int issued = ok ? 2 * n : 0;
      for (int slot = 0; slot < C::NSLOT && slot < issued; ++slot) {
        const int last = slot + ((issued - 1 - slot) / C::NSLOT) * C::NSLOT;
        mbar_wait(&bars->kv_full[slot], (last / C::NSLOT) & 1, 62);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      const uint64_t d0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      constexpr uint64_t kToMn = (uint64_t)((C::CHUNK >> 4) - 1) << 16;
      // a GEMM with A = Q or dO from tensor memory and B = a K-major ring tile
      auto issue_tn = [&](uint32_t d_tmem, uint32_t a_tmem, int slot) {
        const uint64_t b = sdesc_at(opaque(d0), C::OFF_RING + slot * C::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk / 4) * C::CHUNK + (kk % 4) * 32;
          mma_ts(d_tmem, a_tmem + kk * 8, sdesc_at(b, koff), C::IDESC_S, kk > 0);
        }
      };
      bool ok = n > 0 && mbar_wait(&bars->q_ready, 0, 63);
      auto wait_slot = [&](int s2) {
        return mbar_wait(&bars->kv_full[s2 % C::NSLOT], (uint32_t)((s2 / C::NSLOT) & 1), 64);
      };
      if (ok) ok = wait_slot(0);
      if (ok) {
        tc_fence_after();
        issue_tn(tmem + C::T_S, tmem + C::T_Q, 0);  // S_0
        mma_commit(&bars->s_full);
        ok = wait_slot(1);
      }
      if (ok) {
        tc_fence_after();
        issue_tn(tmem + C::T_DP, tmem + C::T_DO, 1 % C::NSLOT);  // dP_0
        mma_commit(&bars->dp_full);
        mma_commit(&bars->kv_empty[1 % C::NSLOT]);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int kslot = (2 * j) % C::NSLOT;
        if (j + 1 < n) {
          // S_{j+1} over S_j once the dS warps have read S_j
          ok = mbar_wait(&bars->s_free, j & 1, 65);
          if (ok) ok = wait_slot(2 * j + 2);
          if (!ok) break;
          tc_fence_after();
          issue_tn(tmem + C::T_S, tmem + C::T_Q, (2 * j + 2) % C::NSLOT);
          mma_commit(&bars->s_full);
        }
        ok = mbar_wait(&bars->ds_full, j & 1, 66);
        if (!ok) break;
        tc_fence_after();
        // dQ += dS_j K_j : A = dS (tensor memory, keys 64h.. at dP + 64h), B = K_j MN-major
        {
          const uint64_t b = sdesc_at(opaque(d0), C::OFF_RING + kslot * C::TILE) + kToMn;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts(tmem + C::T_DQ, tmem + C::T_DP + 64 * (kk / 4) + 8 * (kk % 4), sdesc_at(b, kk * 2048),
                   C::IDESC_DQ, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars->kv_empty[kslot]);
        if (j + 1 < n) {
          // dP_{j+1} over dP_j / dS_j: issued after dQ_j, which reads dS_j first
          ok = wait_slot(2 * j + 3);
          if (!ok) break;
          tc_fence_after();
          issue_tn(tmem + C::T_DP, tmem + C::T_DO, (2 * j + 3) % C::NSLOT);
          mma_commit(&bars->dp_full);
          mma_commit(&bars->kv_empty[(2 * j + 3) % C::NSLOT]);
        }
      }
      mma_commit(&bars->dq_done);
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, 67);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
    const int qw = warp % 4, h = warp / 4;
    const int r = qw * 32 + lane;  // query row in the tile
    const int q_row = i * BM + r;
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    bool ok = mbar_wait(&bars->q_full, 0, 68);
    // Q and dO into tensor memory: this warp copies half of its 32 rows' bytes
    // (the half-h columns) from the 128-byte swizzled TMA tiles
    if (ok) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t base = smem_u32(smem + (which ? C::OFF_DO : C::OFF_Q));
        const uint32_t tdst = tmem + lane_off + (which ? C::T_DO : C::T_Q);
        constexpr int UNITS = D / 16;  // 16-byte units of this warp's half row (D/2 bf16)
        uint32_t v[UNITS * 4];
#pragma unroll
        for (int u = 0; u < UNITS; ++u) {
          const int gu = h * UNITS + u;  // 16-byte unit of the whole row
          const uint32_t chunk = gu / 8, within = gu % 8;
          const float4 f = ld_shared_v4(base + chunk * C::CHUNK + r * 128 + ((within ^ (r & 7)) << 4));
          v[4 * u] = __float_as_uint(f.x);
          v[4 * u + 1] = __float_as_uint(f.y);
          v[4 * u + 2] = __float_as_uint(f.z);
          v[4 * u + 3] = __float_as_uint(f.w);
        }
        if constexpr (D == 128) {
          tmem_st32(tdst + h * 32, v);
        } else {
          tmem_st16(tdst + h * 16, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->q_ready);
    }
    const float lse2 = sVec[r], dsm = sVec[BM + r];
    const float c = p.scale_log2;
    const uint32_t tS = tmem + lane_off + C::T_S + 64 * h;
    const uint32_t tDP = tmem + lane_off + C::T_DP + 64 * h;
    for (int j = 0; j < n && ok; ++j) {
      ok = mbar_wait(&bars->s_full, j & 1, 69);
      if (!ok) break;
      tc_fence_after();
      float pr[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v[32];
        tmem_ld32(tS + cc * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) pr[cc * 32 + e] = __uint_as_float(v[e]);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free);
      // keys j*BN + 64h + col: hidden past Nk, or above the causal diagonal
      const int k0 = j * BN + 64 * h;
      const int lim = p.causal ? min(q_row + 1 + p.off, p.Nk) : p.Nk;  // keys < lim visible
      if (k0 + 64 > lim) {
#pragma unroll
        for (int col = 0; col < 64; ++col)
          if (k0 + col >= lim) pr[col] = -INFINITY;
      }
      const uint64_t c2 = f2_pack(c, c), l2 = f2_pack(lse2, lse2);
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(pr[e], pr[e + 1]), c2, l2), x0, x1);
        pr[e] = ex2(x0);
        pr[e + 1] = ex2(x1);
      }
      ok = mbar_wait(&bars->dp_full, j & 1, 70);
      if (!ok) break;
      tc_fence_after();
      uint32_t w[32];
      const uint64_t d2 = f2_pack(dsm, dsm);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v[32];
        tmem_ld32(tDP + cc * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float a, b;
          f2_unpack(f2_mul(f2_pack(pr[cc * 32 + e], pr[cc * 32 + e + 1]),
                           f2_add(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), d2)),
                    a, b);
          w[cc * 16 + e / 2] = pack_bf16x2(a, b);
        }
      }
      // dS (bf16, 64 keys) over the first 32 of this warp's own dP columns
      tmem_st32(tDP, w);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full);
    }
    if (ok) ok = n == 0 || mbar_wait(&bars->dq_done, 0, 71);
    if (ok) {
      tc_fence_after();
      constexpr int DH = D / 2;  // dQ columns per warp
      const bool row_ok = q_row < p.Nq;
      __nv_bfloat16* dst = p.dq + ((size_t)bh * p.Nq + (row_ok ? q_row : 0)) * D + h * DH;
      if (n == 0) {
        if (row_ok) {
#pragma unroll
          for (int u = 0; u < DH / 8; ++u) reinterpret_cast<uint4*>(dst)[u] = make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
        // every lane takes part in the tensor-memory loads (.sync.aligned);
        // only rows inside the problem store
#pragma unroll
        for (int cc = 0; cc < DH / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::T_DQ + h * DH + cc * 32, v);
          tmem_wait_ld();
          if (row_ok) {
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              o[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * p.scale, __uint_as_float(v[2 * e + 1]) * p.scale);
            uint4* o4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) o4[u] = make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Query heads per locality chunk of the dQ pass: per query head the pass reads
// its Q and dO once and the K and V of its key/value head for every query tile
// (4 Nk d bytes per key/value head); a chunk keeps its K and V near 40 MB of L2
// and holds at least two waves of CTAs.
inline int chunk_heads(int BH, int G, int Nk, int d, int nq, int sms) {
  const long long kv_head = 4LL * Nk * d;
  long long c = std::max(1LL, (40LL << 20) / kv_head) * G;
  c = std::max<long long>(c, (2LL * sms + nq - 1) / nq);
  c = std::min<long long>(((c + G - 1) / G) * G, BH);
  const long long nch = (BH + c - 1) / c;
  c = (BH + nch - 1) / nch;
  return (int)std::min<long long>(((c + G - 1) / G) * G, BH);
}

}  // namespace dqp

// Key/value heads per locality chunk.  Per key/value head the pass touches
// K and V (4 Nk d bytes), the Q and dO of its G query heads (4 G Nq d bytes) and
// their fp32 dQ accumulator (4 G Nq d bytes), which the reduce-adds must find in
// L2; a chunk keeps that near 80 MB of the 126 MB L2.  A chunk also holds at
// least two waves of CTAs so that its light tail balances the SMs, and chunks
// split the heads evenly.
inline int chunk_heads(int BHkv, int G, int Nq, int Nk, int d, int nkv, int sms) {
  const long long per_head = 4LL * d * (Nk + 2LL * G * Nq);
  long long c = std::max(1LL, (80LL << 20) / per_head);
  c = std::max<long long>(c, (2LL * sms + nkv - 1) / nkv);
  c = std::min<long long>(c, BHkv);
  const long long nch = (BHkv + c - 1) / c;
  return (int)((BHkv + nch - 1) / nch);
}

}  // namespace bwd

size_t sm100_backward_workspace(int BH, int N, int d) {
  const size_t npad = (size_t)(N + 127) / 128 * 128;
  const size_t vec = ((size_t)BH * npad * 4 + 255) / 256 * 256;
  const size_t acc = ((size_t)BH * N * d * 4 + 255) / 256 * 256;
  return 2 * vec + acc + 256;  // + the main kernel's two ticket counters
}

size_t sm100_backward_dq_offset(int BH, int N) {
  const size_t npad = (size_t)(N + 127) / 128 * 128;
  return 2 * (((size_t)BH * npad * 4 + 255) / 256 * 256);
}

namespace {

template <int D, bool kDQ>
cudaError_t launch_main(dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const CUtensorMap& mdo, const CUtensorMap& mdq, const CUtensorMap& mdk,
                        const CUtensorMap& mdv, const bwd::Params& p, cudaStream_t st) {
  const int smem = bwd::Cfg<D>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(bwd::main_kernel<D, kDQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd::main_kernel<D, kDQ><<<grid, bwd::NTHREADS, smem, st>>>(mq, mk, mv, mdo, mdq, mdk, mdv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dq(dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const CUtensorMap& mdo, const bwd::dqp::Params& p, cudaStream_t st) {
  const int smem = bwd::dqp::Cfg<D>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(bwd::dqp::dq_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd::dqp::dq_kernel<D><<<grid, bwd::dqp::NTHREADS, smem, st>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t sm100_backward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mdo, const CUtensorMap& mdq, const CUtensorMap& mdk,
                           const CUtensorMap& mdv, const void* o,
                           const void* dout, const float* lse,
                           void* dq, void* dk, void* dv, void* workspace, int B, int H, int Hkv,
                           int Nq, int Nk, int d, float scale, int causal, int stages,
                           cudaStream_t st) {
  const int BH = B * H;
  const int N = Nq;  // the workspace and the preprocess run over query rows
  const bool det = (stages & kStageDeterministic) != 0;
  const int npad = (N + 127) / 128 * 128;
  const size_t vec = ((size_t)BH * npad * 4 + 255) / 256 * 256;
  float* lse2 = static_cast<float*>(workspace);
  float* dsum = reinterpret_cast<float*>(static_cast<char*>(workspace) + vec);
  float* acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + 2 * vec);
  auto* tickets = reinterpret_cast<unsigned long long*>(
      static_cast<char*>(workspace) + 2 * vec + ((size_t)BH * N * d * 4 + 255) / 256 * 256);
  cudaError_t e = cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  sms = std::max(sms, 1);
  if (stages & kStagePreprocess) {
    const long long rows = (long long)BH * npad;
    const long long rows_per_block = 8LL * (256 / d);  // 8 warps of 256/d rows
    const unsigned pblocks = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
    const auto* ob = static_cast<const __nv_bfloat16*>(o);
    const auto* gb = static_cast<const __nv_bfloat16*>(dout);
    if (d == 128) {
      if (det)
        bwd::preprocess_kernel<128, false><<<pblocks, 256, 0, st>>>(ob, gb, lse, lse2, dsum, acc, tickets, BH, N, npad);
      else
        bwd::preprocess_kernel<128, true><<<pblocks, 256, 0, st>>>(ob, gb, lse, lse2, dsum, acc, tickets, BH, N, npad);
    } else {
      if (det)
        bwd::preprocess_kernel<64, false><<<pblocks, 256, 0, st>>>(ob, gb, lse, lse2, dsum, acc, tickets, BH, N, npad);
      else
        bwd::preprocess_kernel<64, true><<<pblocks, 256, 0, st>>>(ob, gb, lse, lse2, dsum, acc, tickets, BH, N, npad);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (stages & kStageMain) {
    bwd::Params p;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.dq_acc = acc;
    p.lse2 = lse2;
    p.dsum = dsum;
    p.BH = BH;
    p.BHkv = B * Hkv;
    p.H = H;
    p.G = H / Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.off = Nk - Nq;
    p.Npad = npad;
    p.nq = npad / 128;
    p.nkv = (Nk + 127) / 128;
    p.scale = scale;
    p.scale_log2 = scale * bwd::kLog2e;
    p.causal = causal;
    p.chunk = bwd::chunk_heads(p.BHkv, p.G, Nq, Nk, d, p.nkv, sms);
    p.items = p.nkv * p.BHkv;
    p.tickets = tickets;
    // persistent: one CTA per SM, each taking items as it becomes free
    const dim3 grid((unsigned)std::min(p.items, sms));
    if (det)
      e = d == 128 ? launch_main<128, false>(grid, mq, mk, mv, mdo, mdq, mdk, mdv, p, st)
                   : launch_main<64, false>(grid, mq, mk, mv, mdo, mdq, mdk, mdv, p, st);
    else
      e = d == 128 ? launch_main<128, true>(grid, mq, mk, mv, mdo, mdq, mdk, mdv, p, st)
                   : launch_main<64, true>(grid, mq, mk, mv, mdo, mdq, mdk, mdv, p, st);
    if (e != cudaSuccess) return e;
  }
  if (!(stages & kStageConvert)) return cudaSuccess;
  if (det) {
    bwd::dqp::Params p;
    p.dq = static_cast<__nv_bfloat16*>(dq);
    p.lse2 = lse2;
    p.dsum = dsum;
    p.BH = BH;
    p.H = H;
    p.G = H / Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.off = Nk - Nq;
    p.Npad = npad;
    p.nq = npad / 128;
    p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * bwd::kLog2e;
    p.chunk = bwd::dqp::chunk_heads(BH, p.G, Nk, d, p.nq, sms);
    const dim3 grid((unsigned)(p.nq * BH));
    return d == 128 ? launch_dq<128>(grid, mq, mk, mv, mdo, p, st)
                    : launch_dq<64>(grid, mq, mk, mv, mdo, p, st);
  }
  const long long n16 = (long long)BH * N * d / 16;
  const unsigned cblocks = (unsigned)std::min<long long>((n16 + 255) / 256, (long long)sms * 16);
  bwd::dq_convert_kernel<<<cblocks, 256, 0, st>>>(acc, static_cast<__nv_bfloat16*>(dq), n16, scale);
  return cudaGetLastError();
}

}  // namespace fa
