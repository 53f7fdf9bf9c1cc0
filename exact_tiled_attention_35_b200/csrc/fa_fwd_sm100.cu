// Forward pass on sm_100a: TMA-fed shared-memory ring, tcgen05 MMAs with fp32
// accumulators in tensor memory, warp-specialised roles.
//
// What it computes is the standard attention of the page "Atención Flash:
// Revolucionando la Eficiencia de los Modelos de Transformador" (unite.ai),
// evaluated tile by tile as in its section "Detalles de Implementación": query
// tiles outside (one CTA owns two 128-row query tiles), key/value tiles inside,
// per-row running maximum m and running sum l, and the output rescaled by
// exp(m_old - m_new) when m moves (formula 2, "Fusión de Softmax", of the same
// page; the online normaliser of "FlashAttention algorithm part 3").  The output
// stays unnormalised until the last tile and is divided by l once.  Tile size
// 128 follows the block size the nisoo.com page reports as typical.
//
// CTA layout (384 threads, registers rebalanced with setmaxnreg):
//   warps 0-3  softmax + epilogue for query tile 0 (tensor-memory lanes 0-127)
//   warps 4-7  softmax + epilogue for query tile 1
//   warp  8    TMA producer: draws the CTA's next work item when it has issued
//              the loads of the current one, hands it to the other roles through
//              a two-entry ring, then loads Q tiles and K_j, V_j into a ring of slots
//   warp  9    tensor-memory allocator and MMA issuer (one elected thread)
//   warps 10-11 idle (they complete the third warpgroup)
// Tensor memory (512 columns): S_t at column 128*t (fp32 128x128, the bf16
// probabilities P_t are written over its first 64 columns), O_t at 256 + D*t.
// MMA order per key tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), so while one
// softmax group works on its scores the tensor core runs the other's GEMMs.  Each
// P V is issued in two halves of 64 keys, as soon as the softmax group has
// written that half of P.
//
// A row's maximum is only raised when it grows by more than 2^8 in the exp2
// domain; P and l then use the same (stale) maximum, so O = O_acc / l and
// LSE = m * scale + ln(l) stay exact up to fp32 rounding, and O is rescaled in
// tensor memory only for those rows' warps.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "fa_device.cuh"
#include "fa_kernels.h"

namespace fa {
namespace fwd {

constexpr int BM = 128;           // query rows per tile
constexpr int BN = 128;           // keys per tile
constexpr int NQT = 2;            // query tiles per CTA
constexpr int NTHREADS = 384;  // three warpgroups
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kItemRing = 2;       // work items the producer may hand out ahead
constexpr int kItemReaders = 9;    // MMA issuer and the 8 softmax warps
constexpr int kSchedSlots = 256;   // ticket counters, one per launch in flight
// Register split (setmaxnreg).  The launch gives every thread 168 registers,
// 384 * 168 = 64512 in all; the shares sum to 128 * (2*208 + 88) = 64512.
constexpr int kRegsSoftmax = 208;  // warpgroups 0 and 1
constexpr int kRegsControl = 88;   // warpgroup 2: producer, MMA issuer, two idle warps
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= NTHREADS * 168,
              "register split exceeds the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
  static constexpr int TILE = BN * D * 2;          // bytes of one 128-row bf16 tile
  static constexpr int CHUNK = BN * 128;           // bytes of one 64-column swizzle chunk
  static constexpr int NSLOT = D == 128 ? 5 : 10;  // K/V ring slots
  static constexpr int SMEM_Q = NQT * TILE;
  static constexpr int SMEM_RING = NSLOT * TILE;
  static constexpr int OFF_BAR = SMEM_Q + SMEM_RING;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;  // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, 0, 1);
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int BH;      // query heads B*H
  int H;       // query heads per batch
  int G;       // query heads per key/value head (1 without grouping)
  int Nq;      // query rows
  int Nk;      // key rows
  int off;     // Nk - Nq: under the causal mask key j is visible to query i iff j <= i + off
  int npairs;  // ceil(Nq / 256)
  int chunk;   // query heads per locality chunk (their K/V stay resident in L2)
  int items;   // work items = query-tile pairs x heads
  int slot;    // ticket counter of this launch
  float scale;
  float scale_log2;
  int causal;
};

struct Bars {
  uint64_t q_full[NQT];
  uint64_t q_empty[NQT];  // the item's last S_t has read Q_t
  uint64_t s_full[NQT];
  uint64_t p_lo[NQT];   // probabilities of keys 0-63 of the tile in tensor memory
  uint64_t p_hi[NQT];   // keys 64-127
  uint64_t o_full[NQT];   // the item's last P_t V has landed in O_t
  uint64_t drain;
  uint64_t kv_full[16];
  uint64_t kv_empty[16];
  uint64_t it_full[kItemRing];   // the producer has written it_item[s]
  uint64_t it_empty[kItemRing];  // every reader has taken it_item[s]
  int it_item[kItemRing];
  uint32_t tmem_base;
};

// Ticket counters of the work-item scheduler: [slot][0] hands out work items past
// the first gridDim.x, [slot][1] counts CTAs that have drawn their last ticket.
// The last such CTA of a launch sets both back to zero, so the next launch that
// draws the same slot starts clean.  The host draws slots round-robin; two launches in flight
// at the same time on one device share a slot only if kSchedSlots launches were
// issued in between.
__device__ unsigned int g_fwd_tickets[kSchedSlots][2];

// Number of key tiles the query tile starting at row q0 needs: 0 past the last
// query, and 0 too when the causal mask hides every key from every row of the
// tile (possible when Nq > Nk; those rows get O = 0 and LSE = -inf).
__device__ __forceinline__ int tiles_for(int q0, const Params& p) {
  if (q0 >= p.Nq) return 0;
  const int nkv = (p.Nk + BN - 1) / BN;
  if (!p.causal) return nkv;
  const int kmax = min(q0 + BM - 1, p.Nq - 1) + p.off;  // last key the tile's last row sees
  return kmax < 0 ? 0 : min(nkv, kmax / BN + 1);
}

// Work item -> (query head, query-tile pair).  The heads are cut into chunks
// whose K and V fit in L2 together; chunk by chunk, the items run pair-major,
// and under the causal mask (where a pair's cost grows with its index) the
// heaviest pairs come first.  CTAs take items in this order as they become
// free, so the light pairs at the end of a chunk fill the gaps.
__device__ __forceinline__ void decode_item(const Params& p, int item, int& bh, int& pair) {
  const int per_chunk = p.chunk * p.npairs;
  const int c = item / per_chunk, w = item - c * per_chunk;
  const int h0 = c * p.chunk, hn = min(p.chunk, p.BH - h0);
  const int rank = w / hn;
  bh = h0 + (w - rank * hn);
  pair = p.causal ? (p.npairs - 1 - rank) : rank;
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
               const __grid_constant__ CUtensorMap mv, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::SMEM_Q;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // per item: query head, key/value head, first query row, key tiles per query tile
  struct Item {
    int bh, bkv, qbase, n[NQT], nmax;
  };
  auto item_info = [&](int item) {
    Item it;
    int pair;
    decode_item(p, item, it.bh, pair);
    // key/value head of query head bh (grouped-query attention; bh itself when G = 1)
    it.bkv = (it.bh / p.H) * (p.H / p.G) + (it.bh % p.H) / p.G;
    it.qbase = pair * (NQT * BM);
#pragma unroll
    for (int t = 0; t < NQT; ++t) it.n[t] = tiles_for(it.qbase + t * BM, p);
    it.nmax = max(it.n[0], it.n[1]);
    return it;
  };

  if (threadIdx.x == 0) {
#pragma unroll
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->q_empty[t], 1);
      mbar_init(&bars->o_full[t], 1);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_lo[t], 128);
      mbar_init(&bars->p_hi[t], 128);
    }
    mbar_init(&bars->drain, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // The k-th work item of this CTA from the producer's ring (>= p.items: none left).
  auto take_item = [&](int k, int& item, int site) -> bool {
    const int s = k % kItemRing;
    if (!mbar_wait(&bars->it_full[s], (uint32_t)((k / kItemRing) & 1), site)) return false;
    item = *reinterpret_cast<volatile int*>(&bars->it_item[s]);
    return true;
  };

  if (warp >= 8) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
   if (warp == kProducerWarp) {
    if (lane == 0) {
      bool ok = true;
      int gseq = 0;           // K/V ring position, continued across items
      int qcnt[NQT] = {0, 0};  // Q_t loads so far
      unsigned int* tickets = &g_fwd_tickets[p.slot][0];
      for (int r = 0; ok; ++r) {
        // The first item of CTA b is b; each later one is drawn from the launch's
        // ticket counter once this CTA's loads for the previous one are issued, so
        // a CTA takes new work about when it is about to run out of it.
        const int item = r == 0 ? (int)blockIdx.x : (int)gridDim.x + (int)atomicAdd(tickets, 1u);
        const int s = r % kItemRing;
        if (r >= kItemRing) ok = mbar_wait(&bars->it_empty[s], (uint32_t)((r / kItemRing - 1) & 1), 24);
        if (!ok) break;
        *reinterpret_cast<volatile int*>(&bars->it_item[s]) = item;
        mbar_arrive(&bars->it_full[s]);
        if (item >= p.items) break;
        const Item w = item_info(item);
        for (int t = 0; t < NQT && ok; ++t) {
          if (w.n[t] == 0) continue;
          if (qcnt[t] > 0) ok = mbar_wait(&bars->q_empty[t], (qcnt[t] - 1) & 1, 10);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars->q_full[t], C::TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sQ + t * C::TILE + c * C::CHUNK, &mq, &bars->q_full[t], c * 64,
                        w.qbase + t * BM, w.bh);
          ++qcnt[t];
        }
        // ring sequence: K_0, V_0, K_1, V_1, ...
        for (int s2 = 0; s2 < 2 * w.nmax && ok; ++s2) {
          const int seq = gseq + s2;
          const int slot = seq % C::NSLOT, round = seq / C::NSLOT;
          if (round > 0) ok = mbar_wait(&bars->kv_empty[slot], (round - 1) & 1, 1);
          if (!ok) break;
          const int j = s2 >> 1;
          const CUtensorMap* m = (s2 & 1) ? &mv : &mk;
          uint8_t* dst = sRing + slot * C::TILE;
          mbar_arrive_expect_tx(&bars->kv_full[slot], C::TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(dst + c * C::CHUNK, m, &bars->kv_full[slot], c * 64, j * BN, w.bkv);
        }
        gseq += 2 * w.nmax;
      }
      // This CTA draws no more tickets (it has drawn one past the last item, or
      // given up on a wait); the last CTA to get here resets the slot.
      __threadfence();
      if (atomicAdd(tickets + 1, 1u) == gridDim.x - 1) {
        atomicExch(tickets, 0u);
        atomicExch(tickets + 1, 0u);
      }
      // make sure no copy into this CTA's shared memory is still in flight at exit
      for (int slot = 0; slot < C::NSLOT && slot < gseq; ++slot) {
        const int last = slot + ((gseq - 1 - slot) / C::NSLOT) * C::NSLOT;
        mbar_wait(&bars->kv_full[slot], (last / C::NSLOT) & 1, 2);
      }
      for (int t = 0; t < NQT; ++t)
        if (qcnt[t] > 0) mbar_wait(&bars->q_full[t], (qcnt[t] - 1) & 1, 11);
    }
   } else if (warp == kMmaWarp) {
    if (lane == 0) {
      bool ok = true;
      // Descriptors are built once; each MMA moves them by a compile-time offset
      // (one add), and ring positions advance incrementally, so the issuing thread
      // spends few instructions per MMA.
      // One descriptor for the start of shared memory (Q_0, K-major); the ring
      // follows the Q tiles, and an MN-major operand differs only in LBO.
      const uint64_t d0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      constexpr uint64_t kToMn = (uint64_t)((C::CHUNK >> 4) - 1) << 16;  // LBO 16 B -> CHUNK
      // S_t = Q_t K_j^T : A = Q_t (K-major), B = K_j (K-major), K = D in steps of 16
      auto issue_s = [&](int t, uint32_t kslot) {
        const uint64_t d = opaque(d0);
        const uint64_t a = sdesc_at(d, t * C::TILE), b = sdesc_at(d, C::SMEM_Q + kslot * C::TILE);
        const uint32_t d_tmem = tmem + t * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk / 4) * C::CHUNK + (kk % 4) * 32;
          mma_ss(d_tmem, sdesc_at(a, koff), sdesc_at(b, koff), C::IDESC_QK, kk > 0);
        }
      };
      // O_t += P_t V_j : A = P_t (tensor memory), B = V_j (MN-major), K = 128 keys,
      // issued in two halves (keys 0-63, 64-127) as the softmax group publishes them
      auto issue_pv = [&](int t, uint32_t vslot, int j, int half) {
        const uint64_t b = sdesc_at(opaque(d0), C::SMEM_Q + vslot * C::TILE) + kToMn;
        const uint32_t d_tmem = tmem + 2 * BN + t * D;
        const uint32_t a_tmem = tmem + t * BN;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int kk = half * 4 + q;
          mma_ts(d_tmem, a_tmem + kk * 8, sdesc_at(b, kk * 16 * 128), C::IDESC_PV,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      auto advance = [](uint32_t& slot, uint32_t& phase) {
        if (++slot == (uint32_t)C::NSLOT) {
          slot = 0;
          phase ^= 1u;
        }
      };
      uint32_t kslot = 0, kphase = 0;  // ring position of the next K tile (the item's K_0)
      int gt[NQT] = {0, 0};         // S_t tiles issued before this item
      int qcnt[NQT] = {0, 0};       // items with a tile t before this one
      for (int r = 0; ok; ++r) {
        int item = p.items;
        ok = take_item(r, item, 25);
        if (ok) mbar_arrive(&bars->it_empty[r % kItemRing]);
        if (!ok || item >= p.items) break;
        const Item w = item_info(item);
        if (w.nmax == 0) continue;  // every key hidden from both tiles: nothing to multiply
        for (int t = 0; t < NQT && ok; ++t)
          if (w.n[t] > 0) ok = mbar_wait(&bars->q_full[t], qcnt[t] & 1, 3);
        if (ok) ok = mbar_wait(&bars->kv_full[kslot], kphase, 4);
        if (!ok) break;
        tc_fence_after();
        // first S of the item; the previous item's last P_t V has already been
        // issued, so overwriting S_t (where P_t lived) is ordered after it
        for (int t = 0; t < NQT; ++t)
          if (w.n[t] > 0) {
            issue_s(t, kslot);
            mma_commit(&bars->s_full[t]);
            if (w.n[t] == 1) mma_commit(&bars->q_empty[t]);
          }
        mma_commit(&bars->kv_empty[kslot]);
        for (int j = 0; j < w.nmax && ok; ++j) {
          uint32_t vslot = kslot, vphase = kphase;
          advance(vslot, vphase);  // V_j
          uint32_t nslot = vslot, nphase = vphase;
          advance(nslot, nphase);  // K_{j+1} (the next item's K_0 after the last j)
          ok = mbar_wait(&bars->kv_full[vslot], vphase, 5);
          bool k_next_ready = false;
          for (int t = 0; t < NQT && ok; ++t) {
            if (j >= w.n[t]) continue;
            const uint32_t par = (uint32_t)((gt[t] + j) & 1);
            // P of the item's first tile is published only after this softmax
            // group has read the previous item's O_t, so the overwrite is safe
            ok = mbar_wait(&bars->p_lo[t], par, 6);
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, vslot, j, 0);
            ok = mbar_wait(&bars->p_hi[t], par, 9);
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, vslot, j, 1);
            if (j + 1 < w.n[t]) {
              if (!k_next_ready) {
                ok = mbar_wait(&bars->kv_full[nslot], nphase, 7);
                if (!ok) break;
                tc_fence_after();
                k_next_ready = true;
              }
              issue_s(t, nslot);
              mma_commit(&bars->s_full[t]);
              if (j + 2 == w.n[t]) mma_commit(&bars->q_empty[t]);  // last S_t of the item
            } else {
              mma_commit(&bars->o_full[t]);  // last P_t V of the item
            }
          }
          if (!ok) break;
          mma_commit(&bars->kv_empty[vslot]);
          if (k_next_ready) mma_commit(&bars->kv_empty[nslot]);
          kslot = nslot;
          kphase = nphase;
        }
        for (int t = 0; t < NQT; ++t) {
          gt[t] += w.n[t];
          qcnt[t] += w.n[t] > 0;
        }
      }
      // wait for every MMA this thread issued before tensor memory is released
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, 8);
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // softmax / epilogue groups
    const int t = warp / 4;
    const int row = (warp % 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * BN;
    const uint32_t tO = tmem + lane_off + 2 * BN + t * D;
    const float c = p.scale_log2;
    bool ok = true;
    int gtile = 0, icnt = 0;  // S_t tiles and items with a tile t so far
    for (int r = 0; ok; ++r) {
    int item = p.items;
    ok = take_item(r, item, 27);
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&bars->it_empty[r % kItemRing]);
    if (!ok || item >= p.items) break;
    const Item w = item_info(item);
    const int n = w.n[t];
    const int bh = w.bh;
    const int q_row = w.qbase + t * BM + row;
    if (n == 0) {
      // no key visible to any row of this tile (or no tile): O = 0, LSE = -inf
      if (q_row < p.Nq) {
        uint4* orow = reinterpret_cast<uint4*>(p.o + ((size_t)bh * p.Nq + q_row) * D);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) orow[i] = make_uint4(0u, 0u, 0u, 0u);
        p.lse[(size_t)bh * p.Nq + q_row] = -INFINITY;
      }
      continue;
    }
    const int q_tile0 = w.qbase + t * BM;
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < n && ok; ++j) {
      ok = mbar_wait(&bars->s_full[t], (gtile + j) & 1, 16 + t);
      if (!ok) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tS + cc * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
      }
      tmem_wait_ld();
      const int k0 = j * BN;
      // masked keys in this tile: past Nk, or above the causal diagonal of some row
      const bool need_mask = (p.causal && k0 + BN - 1 > q_tile0 + p.off) || (k0 + BN > p.Nk);
      if (need_mask) {
        const int lim = p.causal ? min(q_row + 1 + p.off, p.Nk) : p.Nk;  // keys < lim are visible
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (k0 + i >= lim) s[i] = -INFINITY;
      }
      float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int i = 4; i < BN; i += 2) mx4[(i / 2) % 4] = fmax3(mx4[(i / 2) % 4], s[i], s[i + 1]);
      const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      const float m_new = fmaxf(m_used, mx);
      const bool need = (m_new - m_used) * c > kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = ex2((m_used - m_new) * c);
        m_used = m_new;
      }
      // O picks up the new maximum before this tile's P V is accumulated into it
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tO + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + cc * 32, r);
        }
      }
      // a row that has seen no visible key keeps m = -inf; pivot on 0 then
      const float mc = m_used == -INFINITY ? 0.f : m_used * c;
      const uint64_t c2 = f2_pack(c, c), nmc2 = f2_pack(-mc, -mc);
      uint64_t sum2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
      // Exponentials in two halves of 64 keys; each half goes to tensor memory and
      // is published at once so the P V MMA can start on it.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = half * 64 + 2 * i;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), c2, nmc2), x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          sum2[i % 2] = f2_add(sum2[i % 2], f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + half * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(half ? &bars->p_hi[t] : &bars->p_lo[t]);
      }
      float s0, s1, s2, s3;
      f2_unpack(sum2[0], s0, s1);
      f2_unpack(sum2[1], s2, s3);
      l = l * alpha + ((s0 + s1) + (s2 + s3));
    }
    if (ok) ok = mbar_wait(&bars->o_full[t], icnt & 1, 20 + t);
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + ((size_t)bh * p.Nq + (size_t)(q_row < p.Nq ? q_row : 0)) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tO + cc * 32, r);
        tmem_wait_ld();
        if (q_row < p.Nq) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (q_row < p.Nq)
        p.lse[(size_t)bh * p.Nq + q_row] = l > 0.f ? m_used * p.scale + logf(l) : -INFINITY;
    }
    gtile += n;
    ++icnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Query heads per locality chunk.  A chunk's K and V (4 N d bytes per key/value
// head) should fit in about 40 MB of the 126 MB L2, a chunk should hold at least
// two items per CTA so that its light tail balances the CTAs, chunks split the
// heads evenly, and a group of query heads sharing a key/value head never
// straddles two chunks.
inline int chunk_heads(int BH, int G, int N, int d, int npairs, int grid) {
  const long long kv_head = 4LL * N * d;
  long long c = std::max(1LL, (40LL << 20) / kv_head) * G;
  c = std::max<long long>(c, (2LL * grid + npairs - 1) / npairs);
  c = std::min<long long>(((c + G - 1) / G) * G, BH);
  const long long nch = (BH + c - 1) / c;
  c = (BH + nch - 1) / nch;
  c = std::min<long long>(((c + G - 1) / G) * G, BH);
  return (int)c;
}

}  // namespace fwd

cudaError_t sm100_forward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          void* o, float* lse, int B, int H, int Hkv, int Nq, int Nk, int d,
                          float scale, int causal, cudaStream_t st) {
  const int BH = B * H;
  fwd::Params p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.BH = BH;
  p.H = H;
  p.G = H / Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.off = Nk - Nq;
  p.npairs = (Nq + 2 * fwd::BM - 1) / (2 * fwd::BM);
  p.scale = scale;
  p.scale_log2 = scale * fwd::kLog2e;
  p.causal = causal;
  p.items = p.npairs * BH;
  // persistent: one CTA per SM, each taking items as it becomes free
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const dim3 grid((unsigned)std::min(p.items, std::max(sms, 1)));
  p.chunk = fwd::chunk_heads(BH, p.G, Nk, d, p.npairs, (int)grid.x);
  static std::atomic<unsigned int> launches{0};
  p.slot = (int)(launches.fetch_add(1u, std::memory_order_relaxed) % fwd::kSchedSlots);
  cudaError_t e;
  if (d == 128) {
    const int smem = fwd::Cfg<128>::SMEM_BYTES;
    e = cudaFuncSetAttribute(fwd::fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fwd::fwd_kernel<128><<<grid, fwd::NTHREADS, smem, st>>>(mq, mk, mv, p);
  } else {
    const int smem = fwd::Cfg<64>::SMEM_BYTES;
    e = cudaFuncSetAttribute(fwd::fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fwd::fwd_kernel<64><<<grid, fwd::NTHREADS, smem, st>>>(mq, mk, mv, p);
  }
  return cudaGetLastError();
}

}  // namespace fa
