// Block-sparse causal attention forward for B200 (sm_100a).
//
// What one CTA computes: one work item = (query tile, query block i).  A query
// tile holds 128 query rows: one block of B = 128 tokens of one head, or, for
// B = 64, the same block of two query heads that share a key/value head and a
// layout row (grouped-query packing), else the block once plus a discarded
// copy.  The CTA walks the CSR row of kept key blocks j ("Block Sparse
// Attention in LLMs", section 6: for each query block, for each allowed key
// block, a dense product; "Block-Sparse Attention", How It Works: dense work
// inside an allowed block, skipped blocks never scored) and keeps a running
// (FlashAttention-style, same page section 7) softmax so the n x n score
// matrix never exists.
//
// Per kept block j:
//   S = Q K_j^T                (tcgen05.mma, bf16 x bf16 -> fp32 in TMEM)
//   diagonal block only: s[r][c] = -inf for key c > query r (the within-chunk
//                        causal mask of "bsbr", Solution; BF1 section 3.1)
//   m' = max(m, rowmax S); P = exp2((S - m') * scale*log2 e) as bf16 into TMEM
//   O += P V_j                 (tcgen05.mma with A = P read from TMEM)
// then o = O / l (bf16, stored row by row) and lse = (m + log2 l) * ln 2.
// The running max is only moved when a block's max exceeds it by more than
// 8 in exp2 units (a factor of 2^8), which keeps P <= 256 and skips
// almost every rescale of O; the final normalisation uses the same max as the
// sum, so the result is the plain softmax.
//
// Roles (192 threads): warp 0 issues TMA loads (Q once, then K_j and V_j into
// two rings of shared-memory slots); warp 1 owns TMEM and issues the MMAs from one
// thread; warps 2-5 do the softmax, one query row per thread (a warp can only
// reach its own quarter of the TMEM lanes: warp w serves rows 32*(w%4) ..).
// Every wait on an mbarrier is bounded; when one runs out the kernel records
// a status bit, every role stops issuing work, in-flight copies and MMAs are
// drained, TMEM is released and the CTA returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "bsa_device.cuh"
#include "bsa_tmap.h"
#include "bsa_internal.h"

namespace bsa {
namespace dev {

using namespace ptx;

constexpr int kThreads = 192;
constexpr int kTileM = 128;          // query rows per CTA (one tcgen05 M=128 tile)
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.693147180559945309f;

struct Params {
  const int4* work;            // per (layout head, rank): {query block, first CSR entry, kept blocks, diagonal last}
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  uint32_t* status;
  uint32_t* work_counter;   // [0]: items claimed beyond the first one of each CTA, [1]: CTAs done;
                            // both zero at launch, set back to zero by the last CTA
  int n, nb, heads, L, group;
  int items;         // work items in the longest-first list
  int pack;          // distinct heads per tile (1 or 2)
  float scale_log2;  // scale * log2(e)
  uint64_t timeout_ns;
  int debug_never;
};

// Two fp32 lanes at once (sm_100 packed FP32): each lane rounds exactly as
// the scalar instruction would.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rd, {%0, %1};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}
__device__ __forceinline__ void mul2(float& d0, float& d1, float b) {
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %2};\n\t"
      "mul.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(b));
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---------------------------------------------------------------- the kernel
// Every kept key block is processed in chunks of 64 keys (one chunk for
// B = 64, two for B = 128), so S is a 128 x 64 fp32 tile, two S buffers and the
// O accumulator fit in 256 TMEM columns, and two CTAs share each SM.
constexpr int kChunk = 64;
constexpr int kItemSlots = 8;  // items claimed by the producer, handed to the other roles

// K_c lives in K slot c % KS and V_c in V slot c % VS; PV_c completes
// o_done[c % VS] (the V slot of chunk c frees when PV_c is done).
template <int BLK, int HD, int KS, int VS>
struct KernelShape {
  static constexpr int kKSlots = KS;
  static constexpr int kVSlots = VS;
  static constexpr int kODone = VS;
  static constexpr int kCPB = BLK / kChunk;                  // chunks per kept block
  static constexpr int kSubs = kTileM / BLK;                 // query blocks stacked in the tile
  static constexpr int kAtoms = HD / 64;                     // 128-byte swizzle atoms along d
  static constexpr int kQBytes = kTileM * HD * 2;
  static constexpr int kTileBytes = kChunk * HD * 2;         // one 64-key chunk of K or V
  static constexpr int kAtomRowsQ = kTileM * 128;            // bytes of one Q atom column
  static constexpr int kAtomRowsKV = kChunk * 128;           // bytes of one K/V atom column
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKSlots * kTileBytes;
  static constexpr int kOffBar = kOffV + kVSlots * kTileBytes;
  // barriers: q_full, q_free, k_full[2], v_full[3], s_full[2], p_full[2],
  //           o_done[VS], o_free, drain, never, item_full[8], k_free[KS],
  //           stage_free[8]
  static constexpr int kPend = 8;                            // producer's pending-staging FIFO
  static constexpr int kNumBars = 2 + kKSlots + kVSlots + 2 + 2 + kODone + 3 + kItemSlots + kKSlots + kPend;
  static constexpr int kWarpStage = 32 * 128;                // one warp's 32 rows x 64 columns of o
  static_assert(4 * (HD / 64) * kWarpStage == 2 * kTileBytes, "o staging fills two V slots");
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffPend = kOffMisc + 16;
  static constexpr int kOffItems = kOffPend + 8 * kPend;     // claimed, decoded items, ring of 8
  static constexpr int kSmemUsed = kOffItems + 32 * kItemSlots;
  static constexpr int kColS = 0;                            // S buffers: columns 0..63, 64..127
  static constexpr int kColO = 2 * kChunk;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kIdescQK = idesc_bf16(kTileM, kChunk, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16(kTileM, HD, 0, 1);
  static_assert(2 * kChunk + HD <= 256, "TMEM budget");
  static_assert(BLK == 64 || BLK == 128, "block size");
  static_assert(KS >= 2 && VS >= 3, "the rings hold at least the two K and three V chunks of the issue order");
  // at most VS items are waiting for their staging slots at any time
  static_assert(VS <= kPend, "pending-staging FIFO");
  static_assert(kSmemUsed <= 227 * 1024, "shared memory");
  static_assert(HD == 64 || HD == 128, "head dim");
};

// One work item = (head group, rank in its layout head's longest-first order).
struct Item {
  int row, start, len, h0, kvh;
  bool diag_last;
};

// The work-table entry of item t (one 16-byte load; the producer issues it
// for the next item while the current one is still loading).
__device__ __forceinline__ int4 load_work(const Params& p, int t) {
  const int hg = t / p.nb;
  const int rank = t - hg * p.nb;
  const int lh = (hg * p.pack) % p.L;
  return __ldg(p.work + size_t(lh) * p.nb + rank);
}

__device__ __forceinline__ Item decode_item(const Params& p, int t, int4 w) {
  Item it;
  it.h0 = (t / p.nb) * p.pack;
  it.kvh = it.h0 / p.group;
  it.row = w.x;
  it.start = w.y;
  it.len = w.z;
  it.diag_last = w.w != 0;
  return it;
}

// Persistent schedule: CTA b starts with item b of the longest-first list
// (no atomic on the way to its first loads); after that the producer of each
// CTA claims the next unclaimed item with one atomic add (greedy list
// scheduling, so every CTA ends within about one item of the others) and
// hands its index to the MMA and softmax roles through a ring of slots in
// shared memory; -1 ends the stream.
__device__ __forceinline__ int first_item(int n_items) {
  return int(blockIdx.x) < n_items ? int(blockIdx.x) : -1;
}
__device__ __forceinline__ int claim_item(const Params& p, int n_items) {
  if (n_items <= 0) return -1;
  const int t = int(gridDim.x) + int(atomicAdd(p.work_counter, 1u));
  return t < n_items ? t : -1;
}

__device__ __forceinline__ void st_global_v4(void* ptr, const uint32_t* u) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(ptr), "r"(u[0]), "r"(u[1]), "r"(u[2]),
               "r"(u[3])
               : "memory");
}

// The last CTA of a launch to finish puts the work counter back to zero for the
// next launch that uses it (launches on one counter are ordered by the host).
__device__ __forceinline__ void release_counter(uint32_t* counter) {
  __threadfence();
  if (atomicAdd(counter + 1, 1u) == gridDim.x - 1) {
    atomicExch(counter, 0u);
    atomicExch(counter + 1, 0u);
  }
}

// Chunk c (counted over all items of the CTA) uses S buffer c & 1, K slot
// c % KS and V slot c % VS.  MMAs are issued in the order QK_0, QK_1, PV_0,
// QK_2, PV_1, ..., and the producer loads in the same order (K_{q+1} before
// V_q).  A K slot frees when QK_{c-KS} completes (k_free[c % KS]; with two
// K slots the s_full commit of that QK^T), a V slot when PV_{c-VS} completes
// (o_done[c % VS]).  Each such barrier completes
// once per product of its residue class, and the load that waits on it is
// the one the next product of that class needs, so a parity wait can be
// neither one phase early nor two phases late.
template <int BLK, int HD, int MIN_CTAS, int KS, int VS>
__global__ void __launch_bounds__(kThreads, MIN_CTAS)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const Params p) {
  using S = KernelShape<BLK, HD, KS, VS>;
  constexpr int CPB = S::kCPB;
  constexpr int kKSlots = S::kKSlots;
  constexpr int kVSlots = S::kVSlots;
  constexpr int kODone = S::kODone;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    // The 128-byte swizzle needs 1024-byte aligned tiles; refuse to run rather
    // than compute garbage (never expected: dynamic shared memory starts aligned).
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  uint8_t* gbase = smem_raw;

  const uint32_t sQ = base;
  const uint32_t sK = base + S::kOffK;
  const uint32_t sV = base + S::kOffV;
  const uint32_t bar0 = base + S::kOffBar;
  const uint32_t bQFull = bar0;
  const uint32_t bQFree = bar0 + 8u;
  const uint32_t bKFull0 = bar0 + 16u;
  const uint32_t bVFull0 = bKFull0 + 8u * kKSlots;
  const uint32_t bSFull0 = bVFull0 + 8u * kVSlots;
  const uint32_t bPFull0 = bSFull0 + 16u;
  const uint32_t bODone0 = bPFull0 + 16u;
  const uint32_t bOFree = bODone0 + 8u * kODone;
  const uint32_t bDrain = bOFree + 8u;
  const uint32_t bNever = bOFree + 16u;
  const uint32_t bItemFull0 = bOFree + 24u;
  auto bItemFull = [&](int k) { return bItemFull0 + 8u * (k % kItemSlots); };
  // k_free[s] completes when the QK^T that read K slot s has finished.  With
  // two K slots and two S buffers s_full of QK^T_c is already the completion
  // of slot c % 2's reader, so the producer waits on it and QK^T commits
  // nothing more (each commit costs tensor-pipe time).
  constexpr bool kKFreeIsSFull = (kKSlots == 2);
  const uint32_t bKFree0 = bItemFull0 + 8u * kItemSlots;
  auto bKFree = [&](int c) { return bKFree0 + 8u * (c % kKSlots); };
  // The epilogue of an item stages o in the V slots of its last two chunks
  // (free once its last PV is done); stage_free[e % 8] completes when the TMA
  // stores out of them have read them, e counting the items with at least one
  // chunk.  Eight barriers in turn: the producer waits for item e only when a
  // V load reaches its slots, at most VS - 1 <= 7 chunks after its last one,
  // and eight later items (at least one chunk each) cannot all finish in that
  // span, so the wait never sees its barrier two phases on.
  const uint32_t bStageFree0 = bKFree0 + 8u * kKSlots;
  auto bStageFree = [&](int e) { return bStageFree0 + 8u * (e % S::kPend); };
  auto parStage = [](int e) { return uint32_t(e / S::kPend) & 1u; };
  // slot k % 8: {valid, row, start, len, h0, kvh, diag_last}
  volatile int* item_ring = reinterpret_cast<volatile int*>(gbase + S::kOffItems);
  auto read_item = [&](int k, Item& it) -> bool {
    volatile int* e = item_ring + 8 * (k % kItemSlots);
    if (!e[0]) return false;
    it.row = e[1];
    it.start = e[2];
    it.len = e[3];
    it.h0 = e[4];
    it.kvh = e[5];
    it.diag_last = e[6] != 0;
    return true;
  };
  auto bKFull = [&](int c) { return bKFull0 + 8u * (c % kKSlots); };
  auto bVFull = [&](int c) { return bVFull0 + 8u * (c % kVSlots); };
  auto bSFull = [&](int c) { return bSFull0 + 8u * (c & 1); };
  auto bPFull = [&](int c) { return bPFull0 + 8u * (c & 1); };
  auto bODone = [&](int c) { return bODone0 + 8u * (c % kODone); };
  // phase parities of chunk c's barriers
  auto parK = [](int c) { return uint32_t(c / kKSlots) & 1u; };
  auto parV = [](int c) { return uint32_t(c / kVSlots) & 1u; };
  auto parS = [](int c) { return uint32_t(c >> 1) & 1u; };
  auto parO = [](int c) { return uint32_t(c / kODone) & 1u; };
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(gbase + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + S::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};
  const int n_items = p.debug_never ? 0 : p.items;

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(bQFull, 1);
    mbar_init(bQFree, 1);
    for (int s = 0; s < kKSlots; ++s) mbar_init(bKFull0 + 8u * s, 1);
    for (int s = 0; s < kVSlots; ++s) mbar_init(bVFull0 + 8u * s, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bSFull0 + 8u * s, 1);
      mbar_init(bPFull0 + 8u * s, 128);
    }
    for (int s = 0; s < kODone; ++s) mbar_init(bODone0 + 8u * s, 1);
    mbar_init(bOFree, 128);
    mbar_init(bDrain, 1);
    mbar_init(bNever, 1);
    for (int s = 0; s < S::kPend; ++s) mbar_init(bStageFree0 + 8u * s, 4);
    for (int s = 0; s < kItemSlots; ++s) mbar_init(bItemFull0 + 8u * s, 1);
    for (int s = 0; s < kKSlots; ++s) mbar_init(bKFree0 + 8u * s, 1);
    *abort_flag = 0;
    fence_barrier_init();
    if (!p.debug_never) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      tma_prefetch(&tmO);
    }
  }
  if (warp == 1) {
    tmem_alloc(base + S::kOffMisc, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      int kc = 0;            // K chunk loads issued (global chunk index of the next one)
      int vc = 0;            // V chunk loads issued
      int q_loads = 0;       // Q tile loads issued
      // Items with chunks whose staging slots the producer has not yet seen
      // freed: (ordinal among items with chunks, global index of last chunk).
      int* pend_ord = reinterpret_cast<int*>(gbase + S::kOffPend);
      int* pend_last = pend_ord + S::kPend;
      int pend_head = 0, pend_tail = 0, n_nonempty = 0;
      bool ok = true;
      if (p.debug_never) ok = ctl.wait(bNever, 0);
      int next_t = ok ? first_item(n_items) : -1;
      int4 next_w = next_t >= 0 ? load_work(p, next_t) : make_int4(0, 0, 0, 0);
      for (int k = 0; ok; ++k) {
        const int t = next_t;
        Item it{};
        if (t >= 0) it = decode_item(p, t, next_w);
        volatile int* e = item_ring + 8 * (k % kItemSlots);
        e[0] = t >= 0;
        e[1] = it.row;
        e[2] = it.start;
        e[3] = it.len;
        e[4] = it.h0;
        e[5] = it.kvh;
        e[6] = it.diag_last;
        mbar_arrive(bItemFull(k));           // publishes the slot (release)
        if (t < 0) break;
        next_t = claim_item(p, n_items);     // the atomic's latency overlaps this item's loads
        // the previous item's last QK^T has finished reading the Q buffer
        if (k > 0 && !(ok = ctl.wait(bQFree, (k - 1) & 1))) break;
        mbar_expect_tx(bQFull, S::kQBytes);
        // For B = 64 without a partner head the second block of the tile is
        // the next head's (or zeros past the last head): its rows are discarded.
        tma_load_q<BLK, HD>(sQ, &tmQ, bQFull, it.row * BLK, it.h0);
        ++q_loads;
        const int nch = it.len * CPB;
        if (nch > 0) {
          pend_ord[pend_tail % S::kPend] = n_nonempty++;
          pend_last[pend_tail % S::kPend] = kc + nch - 1;
          ++pend_tail;
        }
        auto key0 = [&](int q) { return __ldg(p.col_idx + it.start + q / CPB) * BLK + (q % CPB) * kChunk; };
        auto load_k = [&](int q) -> bool {
          const int c = kc;
          if (c >= kKSlots) {
            const bool freed = kKFreeIsSFull ? ctl.wait(bSFull(c), parS(c - kKSlots))
                                             : ctl.wait(bKFree(c), parK(c - kKSlots));
            if (!freed) return false;
          }
          const uint32_t dst = sK + (c % kKSlots) * S::kTileBytes;
          mbar_expect_tx(bKFull(c), S::kTileBytes);
          const int r0 = key0(q);
          tma_load_kv<HD>(dst, &tmK, bKFull(c), r0, it.kvh);
          ++kc;
          return true;
        };
        auto load_v = [&](int q) -> bool {
          const int c = vc;
          if (c >= kVSlots && !ctl.wait(bODone(c), parO(c - kVSlots))) return false;
          // V_c refills the slot of chunk c - VS; if that chunk or the one
          // after it was the last of an item, its epilogue staged o there.
          while (pend_head != pend_tail && c >= pend_last[pend_head % S::kPend] + kVSlots - 1) {
            const int e = pend_ord[pend_head % S::kPend];
            if (!ctl.wait(bStageFree(e), parStage(e))) return false;
            ++pend_head;
          }
          const uint32_t dst = sV + (c % kVSlots) * S::kTileBytes;
          mbar_expect_tx(bVFull(c), S::kTileBytes);
          const int r0 = key0(q);
          tma_load_kv<HD>(dst, &tmV, bVFull(c), r0, it.kvh);
          ++vc;
          return true;
        };
        if (nch > 0) ok = load_k(0);
        // the claim above has returned by now: fetch the next item's entry
        // while this item's loads wait for their slots
        if (next_t >= 0) next_w = load_work(p, next_t);
        for (int q = 0; q < nch && ok; ++q) {
          if (q + 1 < nch) ok = load_k(q + 1);
          if (ok) ok = load_v(q);
        }
      }
      // Never leave the CTA with copies in flight into its shared memory.
      if (q_loads > 0) wait_drain(bQFull, (q_loads - 1) & 1, 200000000ull);
      for (int c = (kc > kKSlots ? kc - kKSlots : 0); c < kc; ++c) wait_drain(bKFull(c), parK(c), 200000000ull);
      for (int c = (vc > kVSlots ? vc - kVSlots : 0); c < vc; ++c) wait_drain(bVFull(c), parV(c), 200000000ull);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int c0 = 0;            // chunks of earlier items (global chunk index base)
      // Operand descriptors as fixed bits plus (address >> 4): each product
      // adds its tile's offset to one of these low words.
      constexpr uint64_t kFixKMajor = sw128_fixed(16, 1024);              // Q and K, read along d
      constexpr uint64_t kFixV = sw128_fixed(S::kAtomRowsKV, 1024);       // V, read along the keys
      const uint32_t q_lo = uint32_t(kFixKMajor) + (sQ >> 4);
      const uint32_t k_lo = uint32_t(kFixKMajor) + (sK >> 4);
      const uint32_t v_lo = uint32_t(kFixV) + (sV >> 4);
      constexpr uint32_t kHiKMajor = uint32_t(kFixKMajor >> 32);
      constexpr uint32_t kHiV = uint32_t(kFixV >> 32);
      if (p.debug_never) ok = ctl.wait(bNever, 0);
      for (int k = 0; ok; ++k) {
        if (!(ok = ctl.wait(bItemFull(k), uint32_t(k / kItemSlots) & 1u))) break;
        Item it;
        if (!read_item(k, it)) break;
        const int nch = it.len * CPB;
        if (!(ok = ctl.wait(bQFull, k & 1))) break;
        tc_fence_after();
        auto issue_qk = [&](int q) -> bool {
          const int c = c0 + q;
          if (!ctl.wait(bKFull(c), parK(c))) return false;
          tc_fence_after();
          const uint32_t d = tmem + S::kColS + (c & 1) * kChunk;
          const uint32_t kb_lo = k_lo + uint32_t(c % kKSlots) * (S::kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t a = desc_from(q_lo + ((kk >> 2) * S::kAtomRowsQ + (kk & 3) * 32) / 16, kHiKMajor);
            const uint64_t b = desc_from(kb_lo + ((kk >> 2) * S::kAtomRowsKV + (kk & 3) * 32) / 16, kHiKMajor);
            mma_ss(d, a, b, S::kIdescQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(bSFull(c));
          if constexpr (!kKFreeIsSFull) tc_commit(bKFree(c));
          if (q == nch - 1) tc_commit(bQFree);      // last reader of this Q tile
          return true;
        };
        auto issue_pv = [&](int q) -> bool {
          const int c = c0 + q;
          // V and the O hand-over first: they are normally ready long before
          // the softmax hands over P, so their barrier tests do not sit
          // between P and the products
          if (!ctl.wait(bVFull(c), parV(c))) return false;
          if (q == 0 && k > 0) {
            // the previous item's epilogue has read O out of TMEM
            if (!ctl.wait(bOFree, (k - 1) & 1)) return false;
          }
          if (!ctl.wait(bPFull(c), parS(c))) return false;
          tc_fence_after();
          const uint32_t pa = tmem + S::kColS + (c & 1) * kChunk;
          const uint32_t vb_lo = v_lo + uint32_t(c % kVSlots) * (S::kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            const uint64_t b = desc_from(vb_lo + kk * 16 * 128 / 16, kHiV);
            mma_ts(tmem + S::kColO, pa + kk * 8, b, S::kIdescPV, (q > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bODone(c));
          return true;
        };
        if (nch == 0) {
          // keep the O hand-over in step with the softmax warps
          if (k > 0 && !(ok = ctl.wait(bOFree, (k - 1) & 1))) break;
          tc_commit(bQFree);
        } else {
          ok = issue_qk(0);
          for (int q = 0; q < nch && ok; ++q) {
            if (q + 1 < nch) ok = issue_qk(q + 1);
            if (ok) ok = issue_pv(q);
          }
        }
        c0 += nch;
      }
      // Wait for every MMA this thread issued before TMEM can be released.
      tc_commit(bDrain);
      wait_drain(bDrain, 0, 200000000ull);
    }
  } else {
    // ================================================================ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;            // tile row = TMEM lane
    const int sub = r / BLK;
    const int rl = r - sub * BLK;            // row inside its query block
    const uint32_t lane_base = tmem + (uint32_t(q4 * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    int s_cnt = 0;                           // chunks seen (global chunk index base)
    bool stage_pending = false;              // this warp's last staging stores not yet released
    int n_staged = 0;                        // items with at least one chunk staged so far
    // Once the TMA stores of the previous epilogue have read the staging box,
    // tell the producer (one arrival per warp); deferred so the store drains
    // while this warp already works on the next item.
    auto release_stage = [&]() {
      if (stage_pending) {
        if (lane == 0) {
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          mbar_arrive(bStageFree(n_staged - 1));
        }
        __syncwarp();
        stage_pending = false;
      }
    };
    if (p.debug_never) ok = __all_sync(0xffffffffu, ctl.wait(bNever, 0));
    for (int k = 0; ok; ++k) {
      ok = __all_sync(0xffffffffu, ctl.wait(bItemFull(k), uint32_t(k / kItemSlots) & 1u));
      if (!ok) break;
      Item it;
      if (!read_item(k, it)) break;
      const int nch = it.len * CPB;
      const int diag_first = it.diag_last ? nch - CPB : nch;   // first chunk of the diagonal block
      if (nch == 0) release_stage();
      float m2 = -INFINITY;                  // running max, in exp2 units
      float l = 0.f;                         // running sum of P
      for (int q = 0; ok && q < nch; ++q) {
        const int sc = s_cnt + q, s = sc & 1;
        ok = __all_sync(0xffffffffu, ctl.wait(bSFull(sc), parS(sc)));
        if (!ok) break;
        if (q == 0) release_stage();
        tc_fence_after();
        float sv[kChunk];
        const uint32_t s_col = lane_base + S::kColS + s * kChunk;
        const bool masked = q >= diag_first;
        // causal mask inside the diagonal block: key (chunk offset + c) > row
        const int lim = rl - (q - diag_first) * kChunk;
        auto load_s = [&]() {
          tmem_ld32(s_col, sv);
          tmem_ld32(s_col + 32, sv + 32);
          tmem_wait_ld();
          if (masked) {
#pragma unroll
            for (int c = 0; c < kChunk; ++c)
              if (c > lim) sv[c] = -INFINITY;
          }
        };
        // P = exp2(S * scale * log2 e - m) in place, with four running sums
        float s0, s1, s2, s3;
        auto exp_pass = [&](float neg_m) {
          s0 = s1 = s2 = s3 = 0.f;
#pragma unroll
          for (int c = 0; c < kChunk; c += 4) {
            float x0, x1, x2, x3;
            fma2(x0, x1, sv[c], sv[c + 1], sl2, neg_m);
            fma2(x2, x3, sv[c + 2], sv[c + 3], sl2, neg_m);
            sv[c] = ex2(x0);
            sv[c + 1] = ex2(x1);
            sv[c + 2] = ex2(x2);
            sv[c + 3] = ex2(x3);
            add2(s0, s1, sv[c], sv[c + 1]);
            add2(s2, s3, sv[c + 2], sv[c + 3]);
          }
        };
        load_s();
        float m_new = m2, alpha = 1.f;
        bool need = false;
        if (q == 0) {
          float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int c = 0; c < kChunk; c += 4) {
            mx0 = max3(mx0, sv[c], sv[c + 1]);
            mx1 = max3(mx1, sv[c + 2], sv[c + 3]);
          }
          m_new = fmaxf(mx0, mx1) * sl2;
          exp_pass((m_new == -INFINITY) ? 0.f : -m_new);
        } else {
          // The running max is finite after the first chunk (its key 0 is
          // never masked).  Exponentiate with it while this chunk's max is
          // reduced alongside; a row moves its max only when the chunk's max
          // exceeds it by more than the threshold, and then this chunk is
          // recomputed from S (still in TMEM) with the new max.
          const float neg_m = -m2;
          float mx0 = -INFINITY, mx1 = -INFINITY;
          s0 = s1 = s2 = s3 = 0.f;
#pragma unroll
          for (int c = 0; c < kChunk; c += 4) {
            mx0 = max3(mx0, sv[c], sv[c + 1]);
            mx1 = max3(mx1, sv[c + 2], sv[c + 3]);
            float x0, x1, x2, x3;
            fma2(x0, x1, sv[c], sv[c + 1], sl2, neg_m);
            fma2(x2, x3, sv[c + 2], sv[c + 3], sl2, neg_m);
            sv[c] = ex2(x0);
            sv[c + 1] = ex2(x1);
            sv[c + 2] = ex2(x2);
            sv[c + 3] = ex2(x3);
            add2(s0, s1, sv[c], sv[c + 1]);
            add2(s2, s3, sv[c + 2], sv[c + 3]);
          }
          const float mb = fmaxf(mx0, mx1) * sl2;
          // Each row moves its own max (so rows never influence each other's
          // rounding); the warp recomputes and passes over O when any moved.
          need = mb > m2 + kRescaleThreshold;
          if (need) {
            m_new = mb;
            alpha = ex2(m2 - m_new);
          }
          if (__any_sync(0xffffffffu, need)) {
            load_s();
            exp_pass(-m_new);
          }
        }
        const bool resc = __any_sync(0xffffffffu, need);
        l = l * alpha + ((s0 + s1) + (s2 + s3));
        if (resc) {
          // O must hold PV_{sc-1} before it is rescaled; only rescaling chunks wait.
          ok = __all_sync(0xffffffffu, ctl.wait(bODone(sc - 1), parO(sc - 1)));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            float ov[32];
            tmem_ld32(lane_base + S::kColO + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2) mul2(ov[e], ov[e + 1], alpha);
            tmem_st32(lane_base + S::kColO + c * 32, ov);
          }
        }
#pragma unroll
        for (int c = 0; c < kChunk / 32; ++c) {
          uint32_t u[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) u[e] = pack_bf16(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]);
          tmem_st16(lane_base + S::kColS + s * kChunk + c * 16, u);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bPFull(sc));
        m2 = m_new;
      }
      if (!ok) break;
      if (nch > 0) {
        const int last = s_cnt + nch - 1;
        ok = __all_sync(0xffffffffu, ctl.wait(bODone(last), parO(last)));
        if (!ok) break;
        tc_fence_after();
      }
      // ---- epilogue: o = O / l as bf16 through this warp's 32-row staging box
      // in a V slot of the item's last two chunks and a TMA store (o rows past
      // n are clipped by the store); lse straight to global
      const int tok = it.row * BLK + rl;
      const int head = it.h0 + (p.pack == 2 ? sub : 0);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (nch > 0) {
        const int last = s_cnt + nch - 1;
        const int r0 = q4 * 32;              // first row of this warp
        const int sub0 = r0 / BLK;
        const int tok0 = it.row * BLK + (r0 - sub0 * BLK);
        const int head0 = it.h0 + (p.pack == 2 ? sub0 : 0);
        const bool warp_stores = sub0 < p.pack;
#pragma unroll
        for (int a = 0; a < S::kAtoms; ++a) {
          float ov[64];
          tmem_ld32(lane_base + S::kColO + a * 64, ov);
          tmem_ld32(lane_base + S::kColO + a * 64 + 32, ov + 32);
          tmem_wait_ld();
          if (a == S::kAtoms - 1) {
            // O has been read: the next item's first PV may overwrite it
            tc_fence_before();
            mbar_arrive(bOFree);
          }
          // the two slots as one 2 x tile area: warp q4, atom a at (q4 * atoms + a) boxes
          const int off = (q4 * S::kAtoms + a) * S::kWarpStage;
          const int j = off / S::kTileBytes;                       // 0: chunk last, 1: chunk last - 1
          const uint32_t stage = sV + ((last - j + kVSlots) % kVSlots) * S::kTileBytes + off % S::kTileBytes;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            st_shared_v4(stage + lane * 128 + ((ch ^ (lane & 7)) << 4),
                         pack_bf16(ov[8 * ch] * inv, ov[8 * ch + 1] * inv),
                         pack_bf16(ov[8 * ch + 2] * inv, ov[8 * ch + 3] * inv),
                         pack_bf16(ov[8 * ch + 4] * inv, ov[8 * ch + 5] * inv),
                         pack_bf16(ov[8 * ch + 6] * inv, ov[8 * ch + 7] * inv));
          fence_proxy_async();
          __syncwarp();
          if (warp_stores && lane == 0 && !*abort_flag) tma_store_3d(&tmO, stage, a * 64, tok0, head0);
        }
        if (lane == 0) asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        stage_pending = true;
        ++n_staged;
      } else {
        // an item without kept blocks: o = 0 (rare; plain stores)
        if (sub < p.pack && tok < p.n && !*abort_flag) {
          uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) + (size_t(head) * p.n + tok) * HD * 2;
          const uint32_t z[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int w4 = 0; w4 < HD / 8; ++w4) st_global_v4(orow + w4 * 16, z);
        }
        tc_fence_before();
        mbar_arrive(bOFree);
      }
      if (sub < p.pack && tok < p.n)
        p.lse[size_t(head) * p.n + tok] = l > 0.f ? (m2 + __log2f(l)) * kLn2 : -INFINITY;
      s_cnt += nch;
    }
    release_stage();
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
  if (threadIdx.x == 0) release_counter(p.work_counter);
}

}  // namespace dev

// ==================================================================== host side
namespace {

using namespace tmap;

template <int BLK, int HD, int MIN_CTAS, int KS = 2, int VS = 3>
int launch_instance(const ForwardArgs& a, dev::Params p) {
  using S = dev::KernelShape<BLK, HD, KS, VS>;
  auto kern = dev::bsa_fwd_kernel<BLK, HD, MIN_CTAS, KS, VS>;
  // Ask for enough shared memory that no more than MIN_CTAS CTAs share an SM,
  // so every resident CTA's TMEM allocation succeeds at once.
  int smem = S::kSmemUsed;
  const int floor_bytes = (228 * 1024) / (MIN_CTAS + 1) + 1024;
  if (smem < floor_bytes) smem = floor_bytes;
  // The shared-memory attribute belongs to the function and the SM count to
  // the device: both are set / queried once per device.
  static std::mutex mu;
  static int sm_count[64] = {};
  int dev_id = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess || dev_id < 0 || dev_id >= 64) return set_error(BSA_ERR_CUDA, "cannot query the device");
  {
    std::lock_guard<std::mutex> lock(mu);
    if (sm_count[dev_id] == 0) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id);
      if (e != cudaSuccess || sms < 1) return set_error(BSA_ERR_CUDA, "cannot query the SM count");
      sm_count[dev_id] = sms;
    }
    sms = sm_count[dev_id];
  }
  CUtensorMap mq, mk, mv, mo;
  std::memset(&mo, 0, sizeof(mo));
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  int grid;
  if (!a.debug_never) {
    int st = encode_q(&mq, a.q, a.heads, a.n, HD, BLK);
    if (st == BSA_OK) st = encode_kv(&mk, a.k, a.kv_heads, a.n, HD);
    if (st == BSA_OK) st = encode_kv(&mv, a.v, a.kv_heads, a.n, HD);
    if (st == BSA_OK) st = encode_o(&mo, a.o, a.heads, a.n, HD);
    if (st != BSA_OK) return st;
    grid = p.items < sms * MIN_CTAS ? p.items : sms * MIN_CTAS;
  } else {
    grid = 8;
  }
  kern<<<grid, dev::kThreads, smem, static_cast<cudaStream_t>(a.stream)>>>(mq, mk, mv, mo, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
  return BSA_OK;
}

// The kernel instance for (B, d): CTAs per SM and the depth of the K and V rings.
int launch_shape(const ForwardArgs& a, const dev::Params& p) {
  if (a.B == 128 && a.d == 128) return launch_instance<128, 128, 2>(a, p);
  if (a.B == 128 && a.d == 64) return launch_instance<128, 64, 2>(a, p);
  if (a.B == 64 && a.d == 128) return launch_instance<64, 128, 2>(a, p);
  if (a.B == 64 && a.d == 64) return launch_instance<64, 64, 2>(a, p);
  return set_error(BSA_ERR_UNSUPPORTED, "unsupported (B, d)");
}

}  // namespace

int launch_forward(const ForwardArgs& a) {
  int st = get_encoder();
  if (st != BSA_OK) return st;
  const bsa_layout* L = a.layout;
  dev::Params p{};
  p.work = reinterpret_cast<const int4*>(L->d_work);
  p.col_idx = L->d_col_idx;
  p.lse = a.lse;
  p.status = L->d_status;
  p.n = a.n;
  p.nb = L->nb;
  p.heads = a.heads;
  p.L = L->L;
  p.group = a.heads / a.kv_heads;
  p.pack = (a.B == 64 && p.group % 2 == 0 && L->L == 1) ? 2 : 1;
  p.scale_log2 = float(double(a.scale) * 1.4426950408889634);
  p.timeout_ns = a.debug_never ? a.timeout_ns : 1000000000ull;   // 1 s: never reached in a correct run
  p.debug_never = a.debug_never;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.items = (a.heads / p.pack) * L->nb;
  if (p.items < 1) return set_error(BSA_ERR_SHAPE, "no work items");
  return with_work_counter(L, static_cast<cudaStream_t>(a.stream), [&](uint32_t* counter) {
    p.work_counter = counter;
    return launch_shape(a, p);
  });
}

int launch_forward_with(const ForwardArgs& a, const int32_t* work, const int32_t* col_idx, uint32_t* status) {
  int st = get_encoder();
  if (st != BSA_OK) return st;
  const bsa_layout* L = a.layout;
  dev::Params p{};
  p.work = reinterpret_cast<const int4*>(work);
  p.col_idx = col_idx;
  p.lse = a.lse;
  p.status = status;
  p.work_counter = status + kScratchCounterWord;
  p.n = a.n;
  p.nb = L->nb;
  p.heads = a.heads;
  p.L = L->L;
  p.group = a.heads / a.kv_heads;
  p.pack = (a.B == 64 && p.group % 2 == 0 && L->L == 1) ? 2 : 1;
  p.scale_log2 = float(double(a.scale) * 1.4426950408889634);
  p.timeout_ns = 1000000000ull;
  p.debug_never = 0;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.items = (a.heads / p.pack) * L->nb;
  if (p.items < 1) return set_error(BSA_ERR_SHAPE, "no work items");
  return launch_shape(a, p);
}

}  // namespace bsa
