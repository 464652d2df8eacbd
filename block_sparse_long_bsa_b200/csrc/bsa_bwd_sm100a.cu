// Block-sparse causal attention backward for B200 (sm_100a): the gradients
// dq, dk, dv of the forward's o with respect to q, k and v, for the same
// block layouts ("BF1: A Causal Dyadic Sparse-Attention Retrofit for
// Efficient Long-Context Transformers", section 4: the operator is gated on
// its gradients as well as its outputs, and adaptation trains through the
// route).  With P_tu = exp(s_tu - lse_t) over the allowed pairs and
// s_tu = scale <q_t, k_u>:
//   D_t = <dO_t, o_t>,  dP_tu = <dO_t, v_u>,  dS_tu = P_tu (dP_tu - D_t),
//   dq_t = scale sum_u dS_tu k_u,  dk_u = scale sum_t dS_tu q_t,
//   dv_u = sum_t P_tu dO_t.
// P is rebuilt from the forward's lse, so no n x n matrix is stored.
//
// Launches on the caller's stream: a clear of the dk / dv rows that are
// summed by several CTAs (or of all of dk, dv), D (one warp per row), then the
// dq kernel (query tiles, each walking its CSR row of kept blocks) and the
// dk/dv kernel (segments of a key block's column of the transposed layout,
// each walking the query tiles that read it).  Both product kernels are
// persistent, one CTA per SM, 320 threads: warp 0 decodes the CTA's work
// items into a ring of shared-memory slots and issues the TMA loads; one
// thread of warp 1 issues the tcgen05 products, each as soon as its inputs
// are ready (two kinds of product interleave, so neither waits behind the
// other; the thread polls with non-blocking barrier tests, which reacts
// faster than suspending waits); warps 2-9 rebuild P and dS, two threads per
// tile row (warp w reaches TMEM lanes 32 (w % 4) ..; warps 2-5 take the first
// 32 keys of each 64-key chunk, warps 6-9 the other 32).  Every product is a
// 128-row bf16 x bf16 -> fp32 tcgen05 MMA accumulating in TMEM.  Every
// mbarrier wait is bounded: one that runs out sets the layout's status word,
// the CTA drains what it has in flight, releases TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>

#include "bsa_device.cuh"
#include "bsa_tmap.h"
#include "bsa_internal.h"

namespace bsa {
namespace bwd {

// The last CTA of a launch to finish puts the work counter back to zero for the
// next launch that uses it (the dq and dk/dv kernels of one call share one
// counter one after the other; launches on one counter are ordered by the host).
__device__ __forceinline__ void release_counter(uint32_t* counter) {
  __threadfence();
  if (atomicAdd(counter + 1, 1u) == gridDim.x - 1) {
    atomicExch(counter, 0u);
    atomicExch(counter + 1, 0u);
  }
}

using namespace ptx;


// ---------------------------------------------------------------- shared
constexpr int kThreads = 320;        // warp 0: item ring and loads; warp 1: products; warps 2-9: rows
constexpr int kRowThreads = 256;     // two threads per tile row, one per half of a 64-key chunk
constexpr int kRowWarps = 8;
constexpr int kTileM = 128;          // rows of every product tile (tcgen05 M = 128)
constexpr int kChunk = 64;           // keys per chunk
constexpr int kHalf = 32;            // keys per row thread
constexpr int kRing = 8;             // decoded work items in flight
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kDrainNs = 200000000ull;


struct Params {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* order;
  const int32_t* col_ptr;
  const int32_t* row_idx;
  const int32_t* seg_ptr;
  const int32_t* segs;
  const float* lse;      // forward lse (natural log)
  const float* dsum;     // D = rowsum(dO * o)
  float* dq;
  float* dk;
  float* dv;
  uint32_t* status;
  uint32_t* work_counter;   // [0]: next unclaimed item of the launched kernel, [1]: its CTAs done;
                            // both zero at launch, set back to zero by the last CTA
  int n, nb, L, heads, kv_heads, group, pack, n_steps;   // n_steps = group / pack head steps per key/value head
  int items;         // work items of the launched kernel
  float scale, scale_log2;
  uint64_t timeout_ns;
};

// A 128-row query tile: block i of head h0 (B = 128), or block i of heads h0
// and h0 + 1 stacked (B = 64; with pack = 1 the second half is not a row of
// this tile and is left out).
struct QTile {
  int i, h0;
};

// Row r of a tile: its head and token, and whether it is a real row.
template <int BLK>
__device__ __forceinline__ bool tile_row(const Params& p, const QTile& t, int r, int& head, int& tok) {
  const int sub = r / BLK;
  head = t.h0 + sub;
  tok = t.i * BLK + (r - sub * BLK);
  return sub < p.pack && tok < p.n;
}

// P and dS of one row against 32 keys of a chunk, from the raw scores s (q.k)
// and dP (dO.v): P = exp(scale s - lse), dS = P (dP - D).  Keys past `lim`
// (causal, diagonal block) and rows that are not live get 0.  dS overwrites s.
__device__ __forceinline__ void p_ds_half(float* s, const float* dp, float* pv, float sl2, float lse2, float dd,
                                          int lim, bool live) {
#pragma unroll
  for (int c = 0; c < kHalf; ++c) {
    const bool keep = live && c <= lim;
    const float pr = keep ? ex2(fmaf(s[c], sl2, -lse2)) : 0.f;
    pv[c] = pr;
    s[c] = pr * (dp[c] - dd);
  }
}

// Row-thread coordinates: warps 2-9, warp w reaching TMEM lanes 32 (w % 4);
// warps 2-5 take keys 0-31 of each chunk, warps 6-9 keys 32-63.
struct RowRole {
  int r, hf;
  uint32_t lane_base;
};
__device__ __forceinline__ RowRole row_role(uint32_t tmem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;
  RowRole rr;
  rr.r = q4 * 32 + lane;
  rr.hf = (warp - 2) >> 2;
  rr.lane_base = tmem + (uint32_t(q4 * 32) << 16);
  return rr;
}

// Bounded polling of several conditions by one thread: true while it may go
// on; after `timeout_ns` without progress it raises the abort flag.
struct Idle {
  uint64_t since = 0;
  __device__ __forceinline__ bool step(bool progress, const Ctl& ctl) {
    if (progress) {
      since = 0;
      return true;
    }
    if (*ctl.abort) return false;
    const uint64_t now = globaltimer();
    if (since == 0) since = now;
    if (now - since > ctl.timeout_ns) {
      *ctl.abort = 1;
      atomicOr(ctl.status, kStatusTimeout);
      return false;
    }
    return true;
  }
};

// ---------------------------------------------------------------- D = rowsum(dO * o)
// D_t = sum_u P_tu dP_tu, which equals <dO_t, o_t>.  A row is read with
// 16-byte loads by HD / 8 lanes; a warp takes kRowdotPasses groups of rows and
// issues all of their loads before any arithmetic, so each thread keeps
// several loads in flight (the pass is bound by HBM).
constexpr int kRowdotPasses = 4;
template <int HD>
__host__ __device__ constexpr int rowdot_rows_per_cta() {
  return 8 * (32 / (HD / 8)) * kRowdotPasses;   // 8 warps x rows per pass x passes
}
template <int HD>
__global__ void __launch_bounds__(256) bsa_bwd_rowdot_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                             float* dsum, size_t rows) {
  constexpr int kLanesPerRow = HD / 8;
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  const int lane = threadIdx.x & 31, sub = lane / kLanesPerRow, part = lane % kLanesPerRow;
  const size_t row0 = size_t(blockIdx.x) * rowdot_rows_per_cta<HD>() +
                      size_t(threadIdx.x >> 5) * (kRowsPerPass * kRowdotPasses);
  uint4 a[kRowdotPasses], b[kRowdotPasses];
#pragma unroll
  for (int ps = 0; ps < kRowdotPasses; ++ps) {
    const size_t row = row0 + size_t(ps) * kRowsPerPass + sub;
    if (row < rows) {
      a[ps] = *reinterpret_cast<const uint4*>(o + row * HD + part * 8);
      b[ps] = *reinterpret_cast<const uint4*>(dout + row * HD + part * 8);
    } else {
      a[ps] = make_uint4(0u, 0u, 0u, 0u);
      b[ps] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int ps = 0; ps < kRowdotPasses; ++ps) {
    const uint32_t wa[4] = {a[ps].x, a[ps].y, a[ps].z, a[ps].w};
    const uint32_t wb[4] = {b[ps].x, b[ps].y, b[ps].z, b[ps].w};
    float acc = 0.f;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wa[h]));
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb[h]));
      acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
    }
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    const size_t row = row0 + size_t(ps) * kRowsPerPass + sub;
    if (part == 0 && row < rows) dsum[row] = acc;
  }
}

// ---------------------------------------------------------------- dk, dv clear
// Zeroes the dk and dv rows of key blocks that do not get exactly one
// store: blocks no query reads (no segment) and blocks whose column is cut
// into several segments (their sums are added by several CTAs).  Used when
// each key/value head has one head step; otherwise all of dk, dv are cleared.
template <int HD>
__global__ void __launch_bounds__(256) bsa_bwd_clear_kernel(const Params p, int B) {
  const int kvh = blockIdx.x / p.nb, j = blockIdx.x - kvh * p.nb;
  const int lh = (kvh * p.group) % p.L;
  const int len = p.col_ptr[size_t(lh) * p.nb + j + 1] - p.col_ptr[size_t(lh) * p.nb + j];
  if (len >= 1 && len <= kColumnSegment) return;
  const int t0 = j * B, t1 = min(p.n, t0 + B);
  float4* dk = reinterpret_cast<float4*>(p.dk + (size_t(kvh) * p.n + t0) * HD);
  float4* dv = reinterpret_cast<float4*>(p.dv + (size_t(kvh) * p.n + t0) * HD);
  const int count = (t1 - t0) * HD / 4;
  for (int e = threadIdx.x; e < count; e += blockDim.x) {
    dk[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    dv[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ---------------------------------------------------------------- dQ
// Persistent: one CTA per SM walks query tiles (head group by head group,
// longest row first inside one; CTAs claim them in order through a counter).  Warp 0 decodes each tile
// into a ring of shared-memory slots (read by the other warps) and loads its
// Q, dO, K and V tiles.  A tile's kept blocks are taken 128 keys at a time
// (two 64-key chunks: two blocks for B = 64, one for B = 128; a lone last
// chunk is paired with zero rows): S = Q K^T and dP = dO V^T as N = 128
// products into single TMEM buffers; the row threads (two per row, 64 keys
// each) read both, release S, turn them into dS = P (dP - D), rounded to bf16
// and packed over the dP columns they read; then dQ += dS K (A = dS read from
// TMEM, B = K read along d) into the tile's accumulator (two TMEM
// accumulators, so one tile's read-out overlaps the next tile's products).
// The products go S(s + 1), dQ(s), dP(s + 1): the next scores are formed while
// the row threads work on the current ones.  Steps are numbered across the
// CTA's tiles: K of step s sits in slot s % 2 until dQ(s) is done, V in the
// single V slot until dP(s) is done, a tile's Q and dO in buffer (tile & 1)
// until its last dP is done.
template <int BLK, int HD>
struct DqShape {
  static constexpr int kCPB = BLK / kChunk;
  static constexpr int kStep = 2 * kChunk;                 // keys per step
  static constexpr int kQBytes = kTileM * HD * 2;
  static constexpr int kKV = kStep * HD * 2;               // one step's K (or V): [atom][128 rows][64 columns]
  static constexpr int kAtomQ = kTileM * 128;
  static constexpr int kAtomKV = kStep * 128;
  static constexpr int kOffK = 4 * kQBytes;                // Q, dO of buffer b at b * 2 * kQBytes
  static constexpr int kOffV = kOffK + 2 * kKV;
  static constexpr int kOffBar = kOffV + kKV;
  static constexpr int kBQ = 0, kBQFree = 2, kBK = 4, kBKFree = 6, kBV = 8, kBS = 9, kBDP = 10, kBRead = 11,
                       kBDS = 12, kBAcc = 13, kBAccFree = 15, kBItem = 17, kBItemFree = 17 + kRing,
                       kBDrain = 17 + 2 * kRing, kNumBars = 18 + 2 * kRing;
  static constexpr int kOffRing = ((kOffBar + kNumBars * 8 + 15) / 16) * 16;
  static constexpr int kOffMisc = kOffRing + kRing * 32;
  static constexpr int kSmem = kOffMisc + 16;
  static constexpr int kColS = 0, kColDP = 128, kColQ = 256;
  static constexpr uint32_t kIdescS = idesc_bf16(kTileM, kStep, 0, 0);
  static constexpr uint32_t kIdescDQ = idesc_bf16(kTileM, HD, 0, 1);
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kColQ + 2 * HD <= 512, "TMEM columns");
};

// One decoded query tile (a ring slot).  last = 1 marks the end of the CTA's list.
struct DqSlot {
  int i, h0, kvh, start, nch, diag_first, last, pad;
};

template <int BLK>
__device__ __forceinline__ DqSlot dq_decode(const Params& p, int x) {
  constexpr int CPB = BLK / kChunk;
  DqSlot s;
  s.pad = 0;
  if (x >= p.items) {
    s.last = 1;
    s.i = s.h0 = s.kvh = s.start = s.nch = s.diag_first = 0;
    return s;
  }
  s.last = 0;
  // head group by head group (the K / V working set in flight is about one
  // key/value head and stays in L2), longest row first inside a head group
  const int hg = x / p.nb, rank = x - hg * p.nb;
  s.h0 = hg * p.pack;
  const int lh = s.h0 % p.L;
  s.i = p.order[size_t(lh) * p.nb + rank];
  s.kvh = s.h0 / p.group;
  const size_t lrow = size_t(lh) * p.nb + s.i;
  s.start = p.row_ptr[lrow];
  const int len = p.row_ptr[lrow + 1] - s.start;
  s.nch = len * CPB;
  const bool diag_last = len > 0 && p.col_idx[s.start + len - 1] == s.i;
  s.diag_first = diag_last ? s.nch - CPB : s.nch;
  return s;
}

__device__ __forceinline__ DqSlot read_slot(const uint8_t* ring, int k) {
  const volatile int* v = reinterpret_cast<const volatile int*>(ring + (k % kRing) * 32);
  DqSlot s;
  s.i = v[0];
  s.h0 = v[1];
  s.kvh = v[2];
  s.start = v[3];
  s.nch = v[4];
  s.diag_first = v[5];
  s.last = v[6];
  s.pad = 0;
  return s;
}

// A position in a CTA's stream of steps: ring item k, step c of it, global
// step number g, and the count of non-empty items before it.
struct DqCursor {
  int k, c, g, xi;
  DqSlot it;
  bool valid;
};

__device__ __forceinline__ int dq_steps(const DqSlot& it) { return (it.nch + 1) >> 1; }

template <int BLK, int HD>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const Params p) {
  using S = DqShape<BLK, HD>;
  constexpr int CPB = S::kCPB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  const uint32_t bar0 = base + S::kOffBar;
  auto bar = [&](int idx) { return bar0 + 8u * uint32_t(idx); };
  auto sQ = [&](int b) { return base + uint32_t(b) * 2 * S::kQBytes; };
  auto sK = [&](int g) { return base + S::kOffK + uint32_t(g & 1) * S::kKV; };
  const uint32_t sV = base + S::kOffV;
  uint8_t* ring = smem_raw + S::kOffRing;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem_raw + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + S::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int b = 0; b < S::kNumBars; ++b) {
      uint32_t count = 1;
      if (b == S::kBRead || b == S::kBDS || b == S::kBAccFree || b == S::kBAccFree + 1) count = kRowThreads;
      if (b >= S::kBItemFree && b < S::kBItemFree + kRing) count = kRowWarps + 1;
      mbar_init(bar(b), count);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + S::kOffMisc, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---- item ring and loads
    if (lane == 0) {
      bool ok = true;
      int nk = 0, nv = 0, xi = 0;   // K, V and Q / dO loads issued (step g's K is load g)
      // one step's K or V: for each 64-key half and 64-column atom, one box
      // landing at [atom][half * 64 + row][64 columns]; a half past the
      // tile's chunks reads rows at n (zero-filled)
      auto load_step = [&](uint32_t dst, const CUtensorMap* m, uint32_t b, const DqSlot& it, int step) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = 2 * step + h;
          const int key0 = c < it.nch ? p.col_idx[it.start + c / CPB] * BLK + (c % CPB) * kChunk : p.n;
#pragma unroll
          for (int a = 0; a < HD / 64; ++a)
            tma_load_3d(dst + a * S::kAtomKV + h * kChunk * 128, m, b, a * 64, key0, it.kvh);
        }
      };
      // items are claimed in list order through the counter, so every CTA
      // ends within about one item of the others
      int x = int(atomicAdd(p.work_counter, 1u));
      for (int k = 0; ok; ++k) {
        if (k >= kRing && !(ok = ctl.wait(bar(S::kBItemFree + k % kRing), uint32_t((k - kRing) / kRing) & 1u))) break;
        const DqSlot it = dq_decode<BLK>(p, x);
        // the next claim's latency overlaps this item's hand-over and loads
        const int x_next = it.last ? x : int(atomicAdd(p.work_counter, 1u));
        volatile int* v = reinterpret_cast<volatile int*>(ring + (k % kRing) * 32);
        v[0] = it.i;
        v[1] = it.h0;
        v[2] = it.kvh;
        v[3] = it.start;
        v[4] = it.nch;
        v[5] = it.diag_first;
        v[6] = it.last;
        mbar_arrive(bar(S::kBItem + k % kRing));
        if (it.last) break;
        x = x_next;
        if (it.nch == 0) continue;
        const int b = xi & 1;
        if (xi >= 2 && !(ok = ctl.wait(bar(S::kBQFree + b), uint32_t((xi - 2) >> 1) & 1u))) break;
        mbar_expect_tx(bar(S::kBQ + b), 2 * S::kQBytes);
        tma_load_q<BLK, HD>(sQ(b), &tmQ, bar(S::kBQ + b), it.i * BLK, it.h0);
        tma_load_q<BLK, HD>(sQ(b) + S::kQBytes, &tmDO, bar(S::kBQ + b), it.i * BLK, it.h0);
        ++xi;
        for (int st = 0; st < dq_steps(it); ++st) {
          const int g = nk;
          // K slot g % 2 held step g - 2 until its dQ product; the V slot held
          // step g - 1 until its dP product
          if (g >= 2 && !(ok = ctl.wait(bar(S::kBKFree + (g & 1)), uint32_t((g - 2) >> 1) & 1u))) break;
          mbar_expect_tx(bar(S::kBK + (g & 1)), S::kKV);
          load_step(sK(g), &tmK, bar(S::kBK + (g & 1)), it, st);
          ++nk;
          if (g >= 1 && !(ok = ctl.wait(bar(S::kBDP), uint32_t(g - 1) & 1u))) break;
          mbar_expect_tx(bar(S::kBV), S::kKV);
          load_step(sV, &tmV, bar(S::kBV), it, st);
          ++nv;
        }
      }
      if (!ok) {
        // let the copies in flight land before the CTA exits
        for (int e = (nk > 2 ? nk - 2 : 0); e < nk; ++e) wait_drain(bar(S::kBK + (e & 1)), uint32_t(e >> 1) & 1u, kDrainNs);
        if (nv > 0) wait_drain(bar(S::kBV), uint32_t(nv - 1) & 1u, kDrainNs);
        for (int e = (xi > 2 ? xi - 2 : 0); e < xi; ++e) wait_drain(bar(S::kBQ + (e & 1)), uint32_t(e >> 1) & 1u, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---- products
    if (lane == 0) {
      bool ok = true;
      // cursor load: the next non-empty item from ring item k on; the dQ
      // cursor, the later of the two, hands each slot back once copied
      auto seek = [&](DqCursor& cu, bool release) {
        while (ok) {
          if (!(ok = ctl.wait(bar(S::kBItem + cu.k % kRing), uint32_t(cu.k / kRing) & 1u))) break;
          cu.it = read_slot(ring, cu.k);
          if (release) mbar_arrive(bar(S::kBItemFree + cu.k % kRing));
          if (cu.it.last) {
            cu.valid = false;
            return;
          }
          if (cu.it.nch > 0) {
            cu.valid = true;
            return;
          }
          ++cu.k;
        }
        cu.valid = false;
      };
      auto advance = [&](DqCursor& cu, bool release) {
        ++cu.g;
        if (++cu.c < dq_steps(cu.it)) return;
        cu.c = 0;
        ++cu.xi;
        ++cu.k;
        seek(cu, release);
      };
      // Every wait for a load (or an accumulator hand-back) is taken before
      // the wait for the row threads that precedes the product, so no
      // barrier test sits between the row threads' hand-over and the
      // product (the tensor core's instruction queue is short).
      auto loads_s = [&](const DqCursor& cs) -> bool {
        return (cs.c != 0 || ctl.wait(bar(S::kBQ + (cs.xi & 1)), uint32_t(cs.xi >> 1) & 1u)) &&
               ctl.wait(bar(S::kBK + (cs.g & 1)), uint32_t(cs.g >> 1) & 1u);
      };
      // S of step s (cursor cs) into the S buffer
      auto issue_s = [&](const DqCursor& cs) {
        tc_fence_after();
        const uint32_t qb = sQ(cs.xi & 1), kb = sK(cs.g);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * S::kAtomQ + (kk & 3) * 32, bo = (kk >> 2) * S::kAtomKV + (kk & 3) * 32;
          mma_ss(tmem + S::kColS, sw128<16, 1024>(qb + ao), sw128<16, 1024>(kb + bo), S::kIdescS, kk > 0);
        }
        tc_commit(bar(S::kBS));
      };
      // dP of step s into the dP buffer
      auto issue_dp = [&](const DqCursor& cs) {
        tc_fence_after();
        const uint32_t qb = sQ(cs.xi & 1) + S::kQBytes;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * S::kAtomQ + (kk & 3) * 32, bo = (kk >> 2) * S::kAtomKV + (kk & 3) * 32;
          mma_ss(tmem + S::kColDP, sw128<16, 1024>(qb + ao), sw128<16, 1024>(sV + bo), S::kIdescS, kk > 0);
        }
        tc_commit(bar(S::kBDP));
        if (cs.c == dq_steps(cs.it) - 1) tc_commit(bar(S::kBQFree + (cs.xi & 1)));   // last reader of Q, dO
      };
      DqCursor cd{0, 0, 0, 0, {}, false};
      seek(cd, true);
      if (cd.valid) {
        ok = loads_s(cd) && ctl.wait(bar(S::kBV), uint32_t(cd.g) & 1u);
        if (ok) {
          issue_s(cd);
          issue_dp(cd);
        }
      }
      while (ok && cd.valid) {
        DqCursor nx = cd;                      // the next step (same item or the next one)
        {
          ++nx.g;
          if (++nx.c >= dq_steps(nx.it)) {
            nx.c = 0;
            ++nx.xi;
            ++nx.k;
            seek(nx, false);
          }
        }
        if (nx.valid && !(ok = loads_s(nx))) break;
        // the row threads have read S(s) and dP(s): S(s + 1) may overwrite S
        if (!(ok = ctl.wait(bar(S::kBRead), uint32_t(cd.g) & 1u))) break;
        if (nx.valid) issue_s(nx);
        // dQ(s) once dS(s) is in TMEM (and, for a tile's first step, its
        // accumulator has been read out for the tile two before); dP(s + 1)
        // overwrites the dP buffer after dQ(s) has read it (same queue)
        if (nx.valid && !(ok = ctl.wait(bar(S::kBV), uint32_t(nx.g) & 1u))) break;
        if (cd.c == 0 && cd.xi >= 2 &&
            !(ok = ctl.wait(bar(S::kBAccFree + (cd.xi & 1)), uint32_t((cd.xi - 2) >> 1) & 1u)))
          break;
        if (!(ok = ctl.wait(bar(S::kBDS), uint32_t(cd.g) & 1u))) break;
        tc_fence_after();
        {
          const uint32_t kb = sK(cd.g);
          const uint32_t acc = tmem + S::kColQ + uint32_t(cd.xi & 1) * HD;
          // dS of keys 64 h + 16 j (j < 4) is packed at dP columns 64 h + 8 j
#pragma unroll
          for (int kk = 0; kk < S::kStep / 16; ++kk)
            mma_ts(acc, tmem + S::kColDP + (kk >> 2) * 64 + (kk & 3) * 8,
                   sw128<S::kAtomKV, 1024>(kb + kk * 16 * 128), S::kIdescDQ, (cd.c > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(S::kBKFree + (cd.g & 1)));
          if (cd.c == dq_steps(cd.it) - 1) tc_commit(bar(S::kBAcc + (cd.xi & 1)));
        }
        if (nx.valid) issue_dp(nx);
        advance(cd, true);
      }
      tc_commit(bar(S::kBDrain));
      wait_drain(bar(S::kBDrain), 0, kDrainNs);
    }
  } else {
    // ---- rows: dS, then each tile's dQ read-out (half of the keys and of the
    // dQ columns per thread)
    const RowRole rr = row_role(tmem);
    const int rl = rr.r - (rr.r / BLK) * BLK;
    constexpr int kCols = HD / 2;
    bool ok = true;
    int g = 0, xi = 0;
    // the row's lse and D of the next item are fetched while the current one ends
    float nlse2 = 0.f, ndd = 0.f;
    bool have_next = false;
    for (int k = 0; ok; ++k) {
      ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBItem + k % kRing), uint32_t(k / kRing) & 1u));
      if (!ok) break;
      const DqSlot it = read_slot(ring, k);
      if (it.last) break;
      int head, tok;
      const bool real = tile_row<BLK>(p, QTile{it.i, it.h0}, rr.r, head, tok);
      const size_t rowi = size_t(head) * p.n + (real ? tok : 0);
      float* out = p.dq + rowi * HD + rr.hf * kCols;
      float lse2, dd;
      if (have_next) {
        lse2 = nlse2;
        dd = ndd;
      } else {
        lse2 = real ? p.lse[rowi] * kLog2e : 0.f;
        dd = real ? p.dsum[rowi] : 0.f;
      }
      have_next = false;
      if (it.nch == 0) {
        if (real) {
#pragma unroll
          for (int e = 0; e < kCols; e += 4) *reinterpret_cast<float4*>(out + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      } else {
        const bool live = real && lse2 > -INFINITY;
        const int steps = dq_steps(it);
        for (int st = 0; st < steps; ++st, ++g) {
          ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBS), uint32_t(g) & 1u) && ctl.wait(bar(S::kBDP), uint32_t(g) & 1u));
          if (!ok) break;
          tc_fence_after();
          float s[kChunk], dp[kChunk];
          const uint32_t cs = rr.lane_base + S::kColS + rr.hf * kChunk;
          const uint32_t cdp = rr.lane_base + S::kColDP + rr.hf * kChunk;
          tmem_ld32(cs, s);
          tmem_ld32(cs + 32, s + 32);
          tmem_ld32(cdp, dp);
          tmem_ld32(cdp + 32, dp + 32);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(S::kBRead));
          // keys of chunk c = 2 st + hf: none past the tile's chunks; in the
          // diagonal block, key (chunk offset + j) > row is dropped
          const int c = 2 * st + rr.hf;
          const int lim = c >= it.nch ? -1 : (c >= it.diag_first ? rl - (c - it.diag_first) * kChunk : kChunk);
#pragma unroll
          for (int j = 0; j < kChunk; ++j) {
            const bool keep = live && j <= lim;
            const float pr = keep ? ex2(fmaf(s[j], p.scale_log2, -lse2)) : 0.f;
            s[j] = pr * (dp[j] - dd);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t u[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) u[e] = pack_bf16(s[h * 32 + 2 * e], s[h * 32 + 2 * e + 1]);
            tmem_st16(cdp + h * 16, u);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(S::kBDS));
        }
        if (!ok) break;
        // prefetch the next item's row values
        if (__all_sync(0xffffffffu, ctl.wait(bar(S::kBItem + (k + 1) % kRing), uint32_t((k + 1) / kRing) & 1u))) {
          const DqSlot nx = read_slot(ring, k + 1);
          if (!nx.last) {
            int nh, nt;
            const bool nreal = tile_row<BLK>(p, QTile{nx.i, nx.h0}, rr.r, nh, nt);
            const size_t nrow = size_t(nh) * p.n + (nreal ? nt : 0);
            nlse2 = nreal ? p.lse[nrow] * kLog2e : 0.f;
            ndd = nreal ? p.dsum[nrow] : 0.f;
            have_next = true;
          }
        }
        ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBAcc + (xi & 1)), uint32_t(xi >> 1) & 1u));
        if (!ok) break;
        tc_fence_after();
        float v[kCols];
        const uint32_t acc = rr.lane_base + S::kColQ + uint32_t(xi & 1) * HD + rr.hf * kCols;
#pragma unroll
        for (int a = 0; a < kCols / 32; ++a) tmem_ld32(acc + a * 32, v + a * 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(S::kBAccFree + (xi & 1)));
        ++xi;
        if (real) {
#pragma unroll
          for (int e = 0; e < kCols; e += 4)
            *reinterpret_cast<float4*>(out + e) =
                make_float4(v[e] * p.scale, v[e + 1] * p.scale, v[e + 2] * p.scale, v[e + 3] * p.scale);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(S::kBItemFree + k % kRing));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) release_counter(p.work_counter);
}

// ---------------------------------------------------------------- dK, dV
// Persistent: one CTA per SM walks work items (key/value head, column
// segment, query-head step, 64-key chunk of a key block; head by head,
// longest segments first inside one; CTAs claim them in order through a counter).  A segment lists up to 16 query blocks whose rows keep
// the key block (the transposed layout).  Warp 0 decodes each item into a
// ring of shared-memory slots and loads its tiles.  Per query tile t:
// S = Q K^T and dP = dO V^T (M = 128 query rows) into TMEM buffer t & 1; the
// row threads write P and dS = P (dP - D) as bf16 [query][key] tiles into
// shared memory; then dV^T += dO^T P and dK^T += Q^T dS (M = 128 along d: A
// is the dO / Q tile read along d, B the P / dS tile read along the keys; for
// d = 64 the upper 64 rows of M read the neighbouring tile and are never
// stored) into the item's accumulators (two TMEM pairs, so one item's
// read-out overlaps the next item's products).  An item that holds a whole
// column, when each key/value head has a single head step, stores its sums;
// otherwise they are added into dk and dv (cleared first).  Tiles are
// numbered across the CTA's items: a tile's Q and dO sit in buffer t & 1
// until its dV / dK products are done; an item's K and V in buffer
// (item & 1) until its last S / dP are done.
template <int BLK, int HD>
struct DkvShape {
  static constexpr int kQBytes = kTileM * HD * 2;
  static constexpr int kTile = kChunk * HD * 2;
  static constexpr int kAtomQ = kTileM * 128;
  static constexpr int kAtomKV = kChunk * 128;
  static constexpr int kPBytes = kTileM * kChunk * 2;      // one [128 queries][64 keys] bf16 tile
  static constexpr int kOffKV = 4 * kQBytes;               // Q, dO of buffer b at b * 2 * kQBytes
  static constexpr int kOffP = kOffKV + 4 * kTile;         // K, V of buffer b at kOffKV + b * 2 * kTile
  static constexpr int kOffBar = kOffP + 2 * kPBytes;      // P, dS
  static constexpr int kBKV = 0, kBKVFree = 2, kBQ = 4, kBS = 6, kBPDS = 8, kBDone = 9, kBAcc = 11,
                       kBAccFree = 13, kBItem = 15, kBItemFree = 15 + kRing, kBDrain = 15 + 2 * kRing,
                       kNumBars = 16 + 2 * kRing;
  static constexpr int kSlotBytes = 96;                    // 8 ints + 16 query blocks
  static constexpr int kOffRing = ((kOffBar + kNumBars * 8 + 15) / 16) * 16;
  static constexpr int kOffMisc = kOffRing + kRing * kSlotBytes;
  static constexpr int kSmem = kOffMisc + 16;
  static constexpr int kColS = 0, kColDP = 128, kColAcc = 256;   // acc pair b: dV at 256 + 128 b, dK 64 further
  static constexpr uint32_t kIdescS = idesc_bf16(kTileM, kChunk, 0, 0);
  static constexpr uint32_t kIdescT = idesc_bf16(kTileM, kChunk, 1, 1);
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct DkvSlot {
  int kvh, h0, j, key0, total, sole, last;
};

template <int BLK>
__device__ __forceinline__ bool dkv_decode(const Params& p, int x, DkvSlot& s, int& e0) {
  constexpr int CPB = BLK / kChunk;
  // key/value head by key/value head (the Q / dO tiles in flight stay in
  // L2), longest segment first inside a head
  const int inner = p.n_steps * CPB;
  const int per_head = p.items / p.kv_heads;     // segment ranks x inner
  s.kvh = x / per_head;
  int rem = x - s.kvh * per_head;
  const int rank = rem / inner;
  rem -= rank * inner;
  const int hs = rem / CPB, hh = rem - hs * CPB;
  s.h0 = s.kvh * p.group + hs * p.pack;
  const int lh = s.h0 % p.L;
  const int seg = p.seg_ptr[lh] + rank;
  if (seg >= p.seg_ptr[lh + 1]) return false;
  s.j = p.segs[3 * seg];
  e0 = p.segs[3 * seg + 1];
  s.total = p.segs[3 * seg + 2];
  s.key0 = s.j * BLK + hh * kChunk;
  const int col_len = p.col_ptr[size_t(lh) * p.nb + s.j + 1] - p.col_ptr[size_t(lh) * p.nb + s.j];
  s.sole = (p.n_steps == 1 && col_len == s.total) ? 1 : 0;
  s.last = 0;
  return true;
}

__device__ __forceinline__ DkvSlot read_dkv_slot(const uint8_t* ring, int k, int slot_bytes) {
  const volatile int* v = reinterpret_cast<const volatile int*>(ring + (k % kRing) * slot_bytes);
  DkvSlot s;
  s.kvh = v[0];
  s.h0 = v[1];
  s.j = v[2];
  s.key0 = v[3];
  s.total = v[4];
  s.sole = v[5];
  s.last = v[6];
  return s;
}
__device__ __forceinline__ int slot_tile(const uint8_t* ring, int k, int slot_bytes, int e) {
  return reinterpret_cast<const volatile int*>(ring + (k % kRing) * slot_bytes)[8 + e];
}

struct DkvCursor {
  int k, e, t, y;
  DkvSlot it;
  bool valid;
};

template <int BLK, int HD>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params p) {
  using S = DkvShape<BLK, HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  const uint32_t bar0 = base + S::kOffBar;
  auto bar = [&](int idx) { return bar0 + 8u * uint32_t(idx); };
  auto sQ = [&](int t) { return base + uint32_t(t & 1) * 2 * S::kQBytes; };
  auto sKV = [&](int y) { return base + S::kOffKV + uint32_t(y & 1) * 2 * S::kTile; };
  const uint32_t sP = base + S::kOffP, sDS = sP + S::kPBytes;
  uint8_t* ring = smem_raw + S::kOffRing;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem_raw + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + S::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int b = 0; b < S::kNumBars; ++b) {
      uint32_t count = 1;
      if (b == S::kBPDS || b == S::kBAccFree || b == S::kBAccFree + 1) count = kRowThreads;
      if (b >= S::kBItemFree && b < S::kBItemFree + kRing) count = kRowWarps + 1;
      mbar_init(bar(b), count);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + S::kOffMisc, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---- item ring and loads
    if (lane == 0) {
      bool ok = true;
      int t = 0, y = 0;
      int k = 0;
      // items are claimed in list order through the counter, so every CTA
      // ends within about one item of the others
      int x = int(atomicAdd(p.work_counter, 1u));
      while (ok) {
        DkvSlot it{};
        int e0 = 0;
        const bool end = x >= p.items;
        if (!end && !dkv_decode<BLK>(p, x, it, e0)) {
          x = int(atomicAdd(p.work_counter, 1u));
          continue;
        }
        // the next claim's latency overlaps this item's hand-over and loads
        const int x_next = end ? x : int(atomicAdd(p.work_counter, 1u));
        if (k >= kRing && !(ok = ctl.wait(bar(S::kBItemFree + k % kRing), uint32_t((k - kRing) / kRing) & 1u))) break;
        volatile int* v = reinterpret_cast<volatile int*>(ring + (k % kRing) * S::kSlotBytes);
        v[0] = it.kvh;
        v[1] = it.h0;
        v[2] = it.j;
        v[3] = it.key0;
        v[4] = it.total;
        v[5] = it.sole;
        v[6] = end ? 1 : 0;
        for (int e = 0; e < (end ? 0 : it.total); ++e) v[8 + e] = p.row_idx[e0 + e];
        mbar_arrive(bar(S::kBItem + k % kRing));
        if (end) break;
        if (y >= 2 && !(ok = ctl.wait(bar(S::kBKVFree + (y & 1)), uint32_t((y - 2) >> 1) & 1u))) break;
        mbar_expect_tx(bar(S::kBKV + (y & 1)), 2 * S::kTile);
        tma_load_kv<HD>(sKV(y), &tmK, bar(S::kBKV + (y & 1)), it.key0, it.kvh);
        tma_load_kv<HD>(sKV(y) + S::kTile, &tmV, bar(S::kBKV + (y & 1)), it.key0, it.kvh);
        ++y;
        for (int e = 0; e < it.total; ++e) {
          if (t >= 2 && !(ok = ctl.wait(bar(S::kBDone + (t & 1)), uint32_t((t - 2) >> 1) & 1u))) break;
          const int i = v[8 + e];
          mbar_expect_tx(bar(S::kBQ + (t & 1)), 2 * S::kQBytes);
          tma_load_q<BLK, HD>(sQ(t), &tmQ, bar(S::kBQ + (t & 1)), i * BLK, it.h0);
          tma_load_q<BLK, HD>(sQ(t) + S::kQBytes, &tmDO, bar(S::kBQ + (t & 1)), i * BLK, it.h0);
          ++t;
        }
        ++k;
        x = x_next;
      }
      if (!ok) {
        for (int e = (t > 2 ? t - 2 : 0); e < t; ++e) wait_drain(bar(S::kBQ + (e & 1)), uint32_t(e >> 1) & 1u, kDrainNs);
        for (int e = (y > 2 ? y - 2 : 0); e < y; ++e) wait_drain(bar(S::kBKV + (e & 1)), uint32_t(e >> 1) & 1u, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---- products, issued as their inputs become ready
    if (lane == 0) {
      bool ok = true;
      auto seek = [&](DkvCursor& cu, bool release) {
        if (!(ok = ctl.wait(bar(S::kBItem + cu.k % kRing), uint32_t(cu.k / kRing) & 1u))) {
          cu.valid = false;
          return;
        }
        cu.it = read_dkv_slot(ring, cu.k, S::kSlotBytes);
        if (release) mbar_arrive(bar(S::kBItemFree + cu.k % kRing));
        cu.valid = !cu.it.last;
      };
      auto advance = [&](DkvCursor& cu, bool release) {
        ++cu.t;
        if (++cu.e < cu.it.total) return;
        cu.e = 0;
        ++cu.y;
        ++cu.k;
        seek(cu, release);
      };
      DkvCursor cs{0, 0, 0, 0, {}, false}, cd{0, 0, 0, 0, {}, false};
      seek(cs, false);
      seek(cd, true);
      Idle idle;
      while (cd.valid && ok) {
        bool progress = false;
        // dV^T += dO^T P, dK^T += Q^T dS for tile t, once its P / dS are written
        if ((cd.t < cs.t || !cs.valid) && mbar_test(bar(S::kBPDS), uint32_t(cd.t) & 1u) &&
            (cd.e > 0 || cd.y < 2 ||
             mbar_test(bar(S::kBAccFree + (cd.y & 1)), uint32_t((cd.y - 2) >> 1) & 1u))) {
          tc_fence_after();
          const uint32_t qb = sQ(cd.t);
          const uint32_t accv = tmem + S::kColAcc + uint32_t(cd.y & 1) * 128, acck = accv + 64;
#pragma unroll
          for (int kk = 0; kk < kTileM / 16; ++kk) {
            const uint32_t off = kk * 16 * 128;
            const uint32_t acc = (cd.e > 0 || kk > 0) ? 1u : 0u;
            mma_ss(accv, sw128<S::kAtomQ, 1024>(qb + S::kQBytes + off), sw128<S::kPBytes, 1024>(sP + off),
                   S::kIdescT, acc);
            mma_ss(acck, sw128<S::kAtomQ, 1024>(qb + off), sw128<S::kPBytes, 1024>(sDS + off), S::kIdescT,
                   acc);
          }
          tc_commit(bar(S::kBDone + (cd.t & 1)));
          if (cd.e == cd.it.total - 1) tc_commit(bar(S::kBAcc + (cd.y & 1)));
          advance(cd, true);
          progress = true;
        }
        // S(t), dP(t): TMEM buffer t & 1 is free once tile t - 2's dV / dK are issued
        if (cs.valid && cs.t < cd.t + 2 &&
            (cs.e > 0 || mbar_test(bar(S::kBKV + (cs.y & 1)), uint32_t(cs.y >> 1) & 1u)) &&
            mbar_test(bar(S::kBQ + (cs.t & 1)), uint32_t(cs.t >> 1) & 1u)) {
          tc_fence_after();
          const uint32_t qb = sQ(cs.t), kb = sKV(cs.y), vb = kb + S::kTile;
          const uint32_t ds = tmem + S::kColS + (cs.t & 1) * kChunk, ddp = tmem + S::kColDP + (cs.t & 1) * kChunk;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t ao = (kk >> 2) * S::kAtomQ + (kk & 3) * 32, bo = (kk >> 2) * S::kAtomKV + (kk & 3) * 32;
            mma_ss(ds, sw128<16, 1024>(qb + ao), sw128<16, 1024>(kb + bo), S::kIdescS, kk > 0);
            mma_ss(ddp, sw128<16, 1024>(qb + S::kQBytes + ao), sw128<16, 1024>(vb + bo), S::kIdescS,
                   kk > 0);
          }
          tc_commit(bar(S::kBS + (cs.t & 1)));
          if (cs.e == cs.it.total - 1) tc_commit(bar(S::kBKVFree + (cs.y & 1)));
          advance(cs, false);
          progress = true;
        }
        ok = ok && idle.step(progress, ctl);
      }
      tc_commit(bar(S::kBDrain));
      wait_drain(bar(S::kBDrain), 0, kDrainNs);
    }
  } else {
    // ---- rows: P and dS per tile (half of the keys per thread), then each
    // item's dV (warps 2-5) or dK (warps 6-9) read-out
    const RowRole rr = row_role(tmem);
    const int rl = rr.r - (rr.r / BLK) * BLK;
    bool ok = true;
    int t = 0, y = 0;
    for (int k = 0; ok; ++k) {
      ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBItem + k % kRing), uint32_t(k / kRing) & 1u));
      if (!ok) break;
      const DkvSlot it = read_dkv_slot(ring, k, S::kSlotBytes);
      if (it.last) break;
      const int hh = (it.key0 - it.j * BLK) / kChunk;
      // the row's lse and D for tile e + 1 are fetched while tile e is computed
      auto row_vals = [&](int e, float& lse2, float& dd, bool& live) {
        int head, tok;
        const bool real = tile_row<BLK>(p, QTile{slot_tile(ring, k, S::kSlotBytes, e), it.h0}, rr.r, head, tok);
        const size_t rowi = size_t(head) * p.n + (real ? tok : 0);
        lse2 = real ? p.lse[rowi] * kLog2e : 0.f;
        dd = real ? p.dsum[rowi] : 0.f;
        live = real;
      };
      float lse2, dd;
      bool live;
      row_vals(0, lse2, dd, live);
      for (int e = 0; e < it.total; ++e, ++t) {
        float nlse2 = 0.f, ndd = 0.f;
        bool nlive = false;
        if (e + 1 < it.total) row_vals(e + 1, nlse2, ndd, nlive);
        const int i = slot_tile(ring, k, S::kSlotBytes, e);
        // causal: in the diagonal block, key (chunk offset + c) > row is dropped
        const int lim = ((i == it.j) ? rl - hh * kChunk : kChunk) - rr.hf * kHalf;
        ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBS + (t & 1)), uint32_t(t >> 1) & 1u));
        if (!ok) break;
        tc_fence_after();
        float s[kHalf], dp[kHalf], pv[kHalf];
        tmem_ld32(rr.lane_base + S::kColS + (t & 1) * kChunk + rr.hf * kHalf, s);
        tmem_ld32(rr.lane_base + S::kColDP + (t & 1) * kChunk + rr.hf * kHalf, dp);
        tmem_wait_ld();
        p_ds_half(s, dp, pv, p.scale_log2, lse2, dd, lim, live && lse2 > -INFINITY);
        // the P / dS tiles were last read by tile t - 1's products
        if (t >= 1) {
          ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBDone + ((t - 1) & 1)), uint32_t((t - 1) >> 1) & 1u));
          if (!ok) break;
        }
        // row r, keys 32 hf .. 32 hf + 31 of the [query][key] tiles, 128-byte swizzled
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = rr.hf * 4 + q;
          const uint32_t off = uint32_t(rr.r) * 128 + ((ch ^ (rr.r & 7)) << 4);
          st_shared_v4(sP + off, pack_bf16(pv[8 * q], pv[8 * q + 1]), pack_bf16(pv[8 * q + 2], pv[8 * q + 3]),
                       pack_bf16(pv[8 * q + 4], pv[8 * q + 5]), pack_bf16(pv[8 * q + 6], pv[8 * q + 7]));
          st_shared_v4(sDS + off, pack_bf16(s[8 * q], s[8 * q + 1]), pack_bf16(s[8 * q + 2], s[8 * q + 3]),
                       pack_bf16(s[8 * q + 4], s[8 * q + 5]), pack_bf16(s[8 * q + 6], s[8 * q + 7]));
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(S::kBPDS));
        lse2 = nlse2;
        dd = ndd;
        live = nlive;
      }
      if (!ok) break;
      // TMEM lane r holds element d = r of the chunk's 64 key rows
      ok = __all_sync(0xffffffffu, ctl.wait(bar(S::kBAcc + (y & 1)), uint32_t(y >> 1) & 1u));
      if (!ok) break;
      tc_fence_after();
      float vals[kChunk];
      const uint32_t acc = rr.lane_base + S::kColAcc + uint32_t(y & 1) * 128 + rr.hf * 64;
      tmem_ld32(acc, vals);
      tmem_ld32(acc + 32, vals + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(S::kBAccFree + (y & 1)));
      ++y;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(S::kBItemFree + k % kRing));
      if (rr.r < HD) {
        float* dst = rr.hf ? p.dk : p.dv;
        const float mul = rr.hf ? p.scale : 1.f;
        const size_t row0 = size_t(it.kvh) * p.n;
        if (it.sole) {
#pragma unroll
          for (int c = 0; c < kChunk; ++c)
            if (it.key0 + c < p.n) dst[(row0 + it.key0 + c) * HD + rr.r] = vals[c] * mul;
        } else {
#pragma unroll
          for (int c = 0; c < kChunk; ++c)
            if (it.key0 + c < p.n) atomicAdd(dst + (row0 + it.key0 + c) * HD + rr.r, vals[c] * mul);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) release_counter(p.work_counter);
}

}  // namespace bwd

// ==================================================================== host side
namespace {

using namespace tmap;

struct Launch {
  const void *q, *k, *v, *o, *dout;
  int heads, kv_heads, n, items_dq, items_dkv, sms;
  size_t dq_rows;
  float* dsum;
  cudaStream_t stream;
};

// Set a kernel's shared-memory size once per device (the attribute belongs
// to the function; several layouts and streams may call at once).
template <typename K>
int prepare(K kern, int smem, int slot) {
  static std::mutex mu;
  static bool done[64][8] = {};
  int dev_id = 0;
  cudaError_t e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess || dev_id < 0 || dev_id >= 64) return set_error(BSA_ERR_CUDA, "cannot query the device");
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev_id][slot]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    done[dev_id][slot] = true;
  }
  return BSA_OK;
}

template <int BLK, int HD>
int launch_instance(const Launch& a, const bwd::Params& p) {
  using SQ = bwd::DqShape<BLK, HD>;
  using SK = bwd::DkvShape<BLK, HD>;
  constexpr int slot = (BLK == 128 ? 2 : 0) + (HD == 128 ? 1 : 0);
  auto kq = bwd::bsa_bwd_dq_kernel<BLK, HD>;
  auto kkv = bwd::bsa_bwd_dkv_kernel<BLK, HD>;
  // both kernels take a whole SM (512 TMEM columns): ask for more than half
  // of its shared memory so a second CTA never lands beside one
  const int floor_bytes = 116 * 1024;
  const int smem_q = SQ::kSmem > floor_bytes ? SQ::kSmem : floor_bytes;
  const int smem_kv = SK::kSmem > floor_bytes ? SK::kSmem : floor_bytes;
  int st = prepare(kq, smem_q, slot);
  if (st == BSA_OK) st = prepare(kkv, smem_kv, 4 + slot);
  if (st != BSA_OK) return st;
  CUtensorMap mq, mdo, mk, mv;
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mdo, 0, sizeof(mdo));
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  CUtensorMap mk2, mv2;   // the dq kernel's K and V: 64-row x 64-column boxes, one per atom
  std::memset(&mk2, 0, sizeof(mk2));
  std::memset(&mv2, 0, sizeof(mv2));
  st = encode_q(&mq, a.q, a.heads, a.n, HD, BLK);
  if (st == BSA_OK) st = encode_q(&mdo, a.dout, a.heads, a.n, HD, BLK);
  if (st == BSA_OK) st = encode_kv(&mk, a.k, a.kv_heads, a.n, HD);
  if (st == BSA_OK) st = encode_kv(&mv, a.v, a.kv_heads, a.n, HD);
  if (st == BSA_OK) st = encode_atoms(&mk2, a.k, a.kv_heads, a.n, HD, 64);
  if (st == BSA_OK) st = encode_atoms(&mv2, a.v, a.kv_heads, a.n, HD, 64);
  if (st != BSA_OK) return st;
  cudaError_t e = cudaSuccess;
  if (p.n_steps == 1) {
    // only rows that several CTAs add into, or that nothing writes, are cleared
    bwd::bsa_bwd_clear_kernel<HD><<<a.kv_heads * p.nb, 256, 0, a.stream>>>(p, BLK);
  } else {
    const size_t grad_kv = size_t(a.kv_heads) * a.n * HD * sizeof(float);
    e = cudaMemsetAsync(p.dk, 0, grad_kv, a.stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.dv, 0, grad_kv, a.stream);
    if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("clearing dk, dv: ") + cudaGetErrorString(e));
  }
  const unsigned rows_grid = unsigned((a.dq_rows + bwd::rowdot_rows_per_cta<HD>() - 1) / bwd::rowdot_rows_per_cta<HD>());
  bwd::bsa_bwd_rowdot_kernel<HD><<<rows_grid, 256, 0, a.stream>>>(
      static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.dsum, a.dq_rows);
  bwd::Params pq = p, pk = p;
  pq.items = a.items_dq;
  pk.items = a.items_dkv;
  // the two product kernels share one item counter, one after the other
  if (a.items_dq > 0)
    kq<<<a.items_dq < a.sms ? a.items_dq : a.sms, bwd::kThreads, smem_q, a.stream>>>(mq, mdo, mk2, mv2, pq);
  if (a.items_dkv > 0) {
    kkv<<<a.items_dkv < a.sms ? a.items_dkv : a.sms, bwd::kThreads, smem_kv, a.stream>>>(mq, mdo, mk, mv, pk);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_backward(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dout, const bsa_layout* layout, int B, int n, int heads, int kv_heads,
                            int d, float scale, float* dq, float* dk, float* dv, float* workspace,
                            void* stream) {
  using namespace bsa;
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (layout->device < 0 || !layout->d_base)
    return set_error(BSA_ERR_INVALID_ARG, "layout was built host-only (device = -1)");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (cur != layout->device) return set_error(BSA_ERR_INVALID_ARG, "layout lives on another device");
  if (B != layout->B || n != layout->n) return set_error(BSA_ERR_SHAPE, "B/n differ from the layout's");
  if (B != 64 && B != 128) return set_error(BSA_ERR_UNSUPPORTED, "B must be 64 or 128");
  if (d != 64 && d != 128) return set_error(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (heads < 1 || kv_heads < 1) return set_error(BSA_ERR_SHAPE, "heads and kv_heads must be >= 1");
  if (heads % kv_heads) return set_error(BSA_ERR_SHAPE, "heads must be a multiple of kv_heads");
  if (heads % layout->L) return set_error(BSA_ERR_SHAPE, "heads must be a multiple of layout_heads");
  if (!(std::isfinite(scale) && scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return set_error(BSA_ERR_INVALID_ARG, "null pointer");
  auto aligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; };
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return set_error(BSA_ERR_INVALID_ARG, "q, k, v, o, dout, dq, dk and dv must be 16-byte aligned");
  if (!aligned(lse, 4) || !aligned(workspace, 4))
    return set_error(BSA_ERR_INVALID_ARG, "lse and workspace must be 4-byte aligned");
  const int group = heads / kv_heads;
  const int pack = (B == 64 && group % 2 == 0 && layout->L == 1) ? 2 : 1;
  const int n_steps = group / pack, cpb = B / 64;
  const int64_t items_dq = int64_t(heads / pack) * layout->nb;
  const int64_t items_dkv = int64_t(layout->max_segs) * kv_heads * n_steps * cpb;
  if (items_dq > INT32_MAX || items_dkv > INT32_MAX) return set_error(BSA_ERR_SHAPE, "too many work items");
  int st = get_encoder();
  if (st != BSA_OK) return st;
  bwd::Params p{};
  p.row_ptr = layout->d_row_ptr;
  p.col_idx = layout->d_col_idx;
  p.order = layout->d_order;
  p.col_ptr = layout->d_col_ptr;
  p.row_idx = layout->d_row_idx;
  p.seg_ptr = layout->d_seg_ptr;
  p.segs = layout->d_segs;
  p.lse = lse;
  p.dsum = workspace;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = layout->d_status;
  p.n = n;
  p.nb = layout->nb;
  p.L = layout->L;
  p.heads = heads;
  p.kv_heads = kv_heads;
  p.group = group;
  p.pack = pack;
  p.n_steps = n_steps;
  p.scale = scale;
  p.scale_log2 = float(double(scale) * 1.4426950408889634);
  p.timeout_ns = 1000000000ull;   // 1 s: never reached in a correct run
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, cur);
  if (e != cudaSuccess || sms < 1) return set_error(BSA_ERR_CUDA, "cannot query the SM count");
  Launch a{q, k, v, o, dout, heads, kv_heads, n, int(items_dq), int(items_dkv), sms, size_t(heads) * n, workspace,
           static_cast<cudaStream_t>(stream)};
  // one of the layout's work counters, taken in turn with its forwards
  return with_work_counter(layout, a.stream, [&](uint32_t* counter) {
    p.work_counter = counter;
    if (B == 64 && d == 128) return launch_instance<64, 128>(a, p);
    if (B == 64 && d == 64) return launch_instance<64, 64>(a, p);
    if (B == 128 && d == 128) return launch_instance<128, 128>(a, p);
    return launch_instance<128, 64>(a, p);
  });
}
