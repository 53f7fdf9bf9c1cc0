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
//   warps 4-7  softmax + epilogue for query tile 1 (the epilogue stages O in
//              shared memory and stores it with TMA, one 32-row box of 64
//              columns at a time per warp; e4m3 at d = 128 has no room and
//              stores rows directly)
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
constexpr unsigned int kHeldTag = 0xFFFFFFFFu;  // owner tag of no launch (diagnostics)
// Register split (setmaxnreg).  The launch gives every thread 168 registers,
// 384 * 168 = 64512 in all; the shares sum to 128 * (2*216 + 72) = 64512.
// 216 per softmax thread leaves its code without spills (208 spilled 20 bytes);
// the producer and the MMA issuer fit in 72.
constexpr int kRegsSoftmax = 216;  // warpgroups 0 and 1
constexpr int kRegsControl = 72;   // warpgroup 2: producer, MMA issuer, two idle warps
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= NTHREADS * 168,
              "register split exceeds the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Tile geometry for head dimension D and element type (F8: e4m3, else bf16).
// A 128-row tile is stored as NCHUNK column chunks of SW bytes per row, each in
// the SW-byte swizzled layout TMA writes (SW = 128, or 64 for e4m3 with D = 64).
template <int D, bool F8>
struct Cfg {
  static constexpr int EB = F8 ? 1 : 2;                 // bytes per element
  static constexpr int ROWB = D * EB;                   // bytes per tile row
  static constexpr int SW = ROWB < 128 ? ROWB : 128;    // swizzle span
  static constexpr int NCHUNK = ROWB / SW;
  static constexpr int CHUNK = BN * SW;                 // bytes of one column chunk
  static constexpr int TILE = BN * ROWB;                // bytes of one 128-row tile
  static constexpr uint32_t LAYOUT = SW == 128 ? 2u : 4u;  // descriptor layout type
  static constexpr int SBO = 8 * SW;                    // 8-row group stride
  static constexpr int KSTEP = 32 / EB;                 // K elements per MMA (32 bytes)
  static constexpr int S_STEPS = D / KSTEP;             // MMAs per S tile
  static constexpr int PV_STEPS = BN / KSTEP;           // MMAs per P V (all 128 keys)
  static constexpr int PCOLS = BN * EB / 4;             // tensor-memory columns of P
  static constexpr int NSLOT = F8 ? (D == 128 ? 12 : 16) : (D == 128 ? 4 : 10);  // K/V ring slots
  static constexpr int SMEM_Q = NQT * TILE;
  static constexpr int SMEM_RING = NSLOT * TILE;
  // O staging, 4 KB per softmax warp: it converts 64 columns of its 32 rows
  // there and stores them with one TMA store (twice at d = 128).  bf16 at d =
  // 128 makes room with a 4-slot ring, which measured no slower than 5 slots;
  // e4m3 at d = 128 has none and stores rows directly.
  static constexpr bool O_STAGED = !F8 || D == 64;
  static constexpr int OFF_O = SMEM_Q + SMEM_RING;
  static constexpr int SMEM_O = O_STAGED ? NQT * BM * 128 : 0;
  static constexpr int OFF_BAR = OFF_O + SMEM_O;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;  // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_QK = F8 ? idesc_e4m3(BM, BN, 0, 0) : idesc_bf16(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = F8 ? idesc_e4m3(BM, D, 0, 1) : idesc_bf16(BM, D, 0, 1);
  static_assert(SMEM_BYTES <= 232448, "shared memory over the per-block limit");
  static_assert(NSLOT <= 16, "K/V ring larger than its barrier arrays");
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
  unsigned int tag;  // this launch's owner tag for the slot (nonzero)
  float scale;       // multiplies the stored Q K^T to give the scores (LSE)
  float scale_log2;  // the same times log2(e)
  float o_scale;     // multiplies P V / l (the stored V's scale; 1 for bf16)
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

// Ticket counters of the work-item scheduler, three words per slot: [0] hands
// out work items past the first gridDim.x, [1] counts CTAs that have drawn
// their last ticket, [2] holds the owner tag of the launch using the slot (0 =
// free).  Every launch carries a nonzero tag of its own, and each CTA claims the
// slot for it (compare-and-swap from 0, or finding its own tag) once, before its
// first draw; a slot left held by a launch that never finished, or shared with a
// launch still in flight, fails the claim and is reported (kStateTicketOwner in
// the status word) instead of handing out wrong items.  The draws themselves are
// single atomic adds.  The last CTA of a launch zeroes the counters, then frees
// the tag.  The host draws slots round-robin.
__device__ unsigned long long g_fwd_tickets[kSchedSlots][3];

// Claims the slot for the launch tagged `tag`; false (recorded) if another
// launch holds it.
__device__ __forceinline__ bool ticket_claim(unsigned long long* slot, unsigned int tag) {
  const unsigned long long old = atomicCAS(slot + 2, 0ull, (unsigned long long)tag);
  if (old == 0ull || old == (unsigned long long)tag) return true;
  record_state_error(kStateTicketOwner);
  return false;
}

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

template <int D, bool F8>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
               const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mo,
               const Params p) {
  using C = Cfg<D, F8>;
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
    if (C::O_STAGED) tma_prefetch_desc(&mo);
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
      bool owner = true;      // false if the slot turned out to be held by another launch
      bool claimed = false;
      int gseq = 0;           // K/V ring position, continued across items
      int qcnt[NQT] = {0, 0};  // Q_t loads so far
      unsigned long long* tickets = &g_fwd_tickets[p.slot][0];
      for (int r = 0; ok; ++r) {
        // The first item of CTA b is b; each later one is drawn from the launch's
        // ticket counter once this CTA's loads for the previous one are issued, so
        // a CTA takes new work about when it is about to run out of it.  A slot
        // held by another launch ends this CTA's work (and is reported).
        int item = (int)blockIdx.x;
        if (r == 1) {
          owner = ticket_claim(tickets, p.tag);
          claimed = true;
        }
        if (r > 0) item = owner ? (int)gridDim.x + (int)atomicAdd(tickets, 1ull) : p.items;
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
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_3d(sQ + t * C::TILE + c * C::CHUNK, &mq, &bars->q_full[t], c * (C::SW / C::EB),
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
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_3d(dst + c * C::CHUNK, m, &bars->kv_full[slot], c * (C::SW / C::EB), j * BN, w.bkv);
        }
        gseq += 2 * w.nmax;
      }
      // This CTA draws no more tickets (it has drawn one past the last item, or
      // given up on a wait); the last CTA to get here frees the slot.  A CTA that
      // gave up before its first draw still claims the slot, so the count of
      // CTAs done stays that of the launch.
      if (!claimed) owner = ticket_claim(tickets, p.tag);
      __threadfence();
      if (owner && atomicAdd(tickets + 1, 1ull) == (unsigned long long)gridDim.x - 1) {
        atomicExch(tickets, 0ull);
        atomicExch(tickets + 1, 0ull);
        __threadfence();
        atomicExch(tickets + 2, 0ull);
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
      const uint64_t d0 = sdesc_swz(smem_u32(sQ), 16, C::SBO, C::LAYOUT);
      constexpr uint64_t kToMn = (uint64_t)((C::CHUNK >> 4) - 1) << 16;  // LBO 16 B -> CHUNK
      // S_t = Q_t K_j^T : A = Q_t (K-major), B = K_j (K-major), K = D in steps of 32 bytes
      auto issue_s = [&](int t, uint32_t kslot) {
        const uint64_t d = opaque(d0);
        const uint64_t a = sdesc_at(d, t * C::TILE), b = sdesc_at(d, C::SMEM_Q + kslot * C::TILE);
        const uint32_t d_tmem = tmem + t * BN;
#pragma unroll
        for (int kk = 0; kk < C::S_STEPS; ++kk) {
          const uint32_t koff = ((kk * 32) / C::SW) * C::CHUNK + (kk * 32) % C::SW;
          if constexpr (F8)
            mma_ss_f8(d_tmem, sdesc_at(a, koff), sdesc_at(b, koff), C::IDESC_QK, kk > 0);
          else
            mma_ss(d_tmem, sdesc_at(a, koff), sdesc_at(b, koff), C::IDESC_QK, kk > 0);
        }
      };
      // O_t += P_t V_j : A = P_t (tensor memory, 8 columns per 32 bytes of keys),
      // B = V_j (MN-major), K = 128 keys, issued in two halves (keys 0-63, 64-127)
      // as the softmax group publishes them
      auto issue_pv = [&](int t, uint32_t vslot, int j, int half) {
        const uint64_t b = sdesc_at(opaque(d0), C::SMEM_Q + vslot * C::TILE) + kToMn;
        const uint32_t d_tmem = tmem + 2 * BN + t * D;
        const uint32_t a_tmem = tmem + t * BN;
#pragma unroll
        for (int q = 0; q < C::PV_STEPS / 2; ++q) {
          const int kk = half * (C::PV_STEPS / 2) + q;
          if constexpr (F8)
            mma_ts_f8(d_tmem, a_tmem + kk * 8, sdesc_at(b, kk * C::KSTEP * C::SW), C::IDESC_PV,
                      (j > 0 || kk > 0) ? 1u : 0u);
          else
            mma_ts(d_tmem, a_tmem + kk * 8, sdesc_at(b, kk * C::KSTEP * C::SW), C::IDESC_PV,
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
      // Exponentials of one half (64 keys), packed for the P V MMA (bf16 pairs, or
      // e4m3 quadruples).
      auto exps = [&](int half, uint32_t(&pk)[32]) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = half * 64 + 2 * i;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), c2, nmc2), x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          sum2[i % 2] = f2_add(sum2[i % 2], f2_pack(p0, p1));
          if constexpr (F8) {
            const uint32_t h = pack_e4m3x2(p0, p1);
            pk[i / 2] = (i % 2) ? (pk[i / 2] | (h << 16)) : h;
          } else {
            pk[i] = pack_bf16x2(p0, p1);
          }
        }
      };
      // Exponentials in two halves of 64 keys; each half goes to tensor memory and
      // is published at once so the P V MMA can start on it.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
        exps(half, pk);
        if constexpr (F8) {
          uint32_t pk16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk16[i] = pk[i];
          tmem_st16(tS + half * 16, pk16);
        } else {
          tmem_st32(tS + half * 32, pk);
        }
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
      const float inv = l > 0.f ? p.o_scale / l : 0.f;
      if constexpr (C::O_STAGED) {
        // rows 32*(warp%4) .. +31 of the tile: bf16 into this warp's 4 KB of the
        // O staging area (128-byte swizzled), then one TMA store by lane 0; rows
        // past Nq are clipped by the tensor map, a box starting past Nq skipped
        const uint32_t region = smem_u32(smem + C::OFF_O) + t * (BM * 128) + (warp % 4) * 4096;
        const int row0 = q_tile0 + (warp % 4) * 32;
        // 64 columns (one 128-byte swizzle chunk) per round: one round at d = 64,
        // two at d = 128 through the same 4 KB
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          uint32_t wv[32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t r[32];
            tmem_ld32(tO + ch * 64 + cc * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              wv[cc * 16 + i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
          }
          // the previous store from this region must have read it
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 8; ++u)
            st_shared_v4(region + lane * 128 + ((u ^ (lane & 7)) << 4), wv[4 * u], wv[4 * u + 1], wv[4 * u + 2],
                           wv[4 * u + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < p.Nq) tma_store_3d(&mo, region, ch * 64, row0, bh);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
      } else {
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
      }
      if (q_row < p.Nq)
        p.lse[(size_t)bh * p.Nq + q_row] = l > 0.f ? m_used * p.scale + logf(l) : -INFINITY;
    }
    gtile += n;
    ++icnt;
    }
    // no O store may still be reading this CTA's shared memory at exit
    if (C::O_STAGED && lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Query heads per locality chunk.  A chunk's K and V (2 N row_bytes per key/value
// head) should fit in about 40 MB of the 126 MB L2, a chunk should hold at least
// two items per CTA so that its light tail balances the CTAs, chunks split the
// heads evenly, and a group of query heads sharing a key/value head never
// straddles two chunks.
inline int chunk_heads(int BH, int G, int N, int row_bytes, int npairs, int grid) {
  const long long kv_head = 2LL * N * row_bytes;
  long long c = std::max(1LL, (40LL << 20) / kv_head) * G;
  c = std::max<long long>(c, (2LL * grid + npairs - 1) / npairs);
  c = std::min<long long>(((c + G - 1) / G) * G, BH);
  const long long nch = (BH + c - 1) / c;
  c = (BH + nch - 1) / nch;
  c = std::min<long long>(((c + G - 1) / G) * G, BH);
  return (int)c;
}

}  // namespace fwd

namespace fwd {
// Marks every scheduler slot as held by a launch that never finishes (owner tag
// kHeldTag, which no launch is given).
__global__ void hold_scheduler_kernel() {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < kSchedSlots) {
    g_fwd_tickets[i][0] = 0ull;
    g_fwd_tickets[i][1] = 0ull;
    g_fwd_tickets[i][2] = (unsigned long long)kHeldTag;
  }
}
}  // namespace fwd

cudaError_t sm100_forward_hold_scheduler(cudaStream_t st) {
  fwd::hold_scheduler_kernel<<<1, fwd::kSchedSlots, 0, st>>>();
  return cudaGetLastError();
}

cudaError_t sm100_forward_reset_scheduler() {
  static const unsigned long long zeros[fwd::kSchedSlots][3] = {};
  return cudaMemcpyToSymbol(fwd::g_fwd_tickets, zeros, sizeof(zeros));
}

namespace {

template <int D, bool F8>
cudaError_t launch_fwd(dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mo, const fwd::Params& p, cudaStream_t st) {
  const int smem = fwd::Cfg<D, F8>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(fwd::fwd_kernel<D, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  fwd::fwd_kernel<D, F8><<<grid, fwd::NTHREADS, smem, st>>>(mq, mk, mv, mo, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t sm100_forward(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mo, void* o, float* lse, int B, int H, int Hkv, int Nq, int Nk, int d,
                          float scale, int causal, bool fp8, float qk_descale, float v_descale,
                          cudaStream_t st) {
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
  p.scale = scale * qk_descale;
  p.scale_log2 = p.scale * fwd::kLog2e;
  p.o_scale = v_descale;
  p.causal = causal;
  p.items = p.npairs * BH;
  // persistent: one CTA per SM, each taking items as it becomes free
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const dim3 grid((unsigned)std::min(p.items, std::max(sms, 1)));
  p.chunk = fwd::chunk_heads(BH, p.G, Nk, d * (fp8 ? 1 : 2), p.npairs, (int)grid.x);
  static std::atomic<unsigned long long> launches{0};
  const unsigned long long seq = launches.fetch_add(1ull, std::memory_order_relaxed);
  p.slot = (int)(seq % fwd::kSchedSlots);
  p.tag = (unsigned int)(seq % (unsigned long long)(fwd::kHeldTag - 1u)) + 1u;  // 1 .. kHeldTag-1
  if (fp8)
    return d == 128 ? launch_fwd<128, true>(grid, mq, mk, mv, mo, p, st)
                    : launch_fwd<64, true>(grid, mq, mk, mv, mo, p, st);
  return d == 128 ? launch_fwd<128, false>(grid, mq, mk, mv, mo, p, st)
                  : launch_fwd<64, false>(grid, mq, mk, mv, mo, p, st);
}

}  // namespace fa
