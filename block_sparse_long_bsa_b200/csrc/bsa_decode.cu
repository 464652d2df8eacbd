// Selected-page decode for B200 (sm_100a): one new query token per sequence
// over a key/value cache paged by blocks, reading the block route that the
// layout holds for the token's block row ("BF1: A Causal Dyadic
// Sparse-Attention Retrofit for Efficient Long-Context Transformers",
// section 5, selected-page decode: the route is planned once and reused for
// every token, so a step only gathers its kept pages).
//
// A query row is a single vector, so the step is a stream over the kept
// pages' keys and values (HBM/L2 bound, no matrix product to hand to the
// tensor cores).  The unit of work is a task: 16 consecutive key rows of one
// kept page, i.e. one contiguous K run and one contiguous V run of the page's
// tile for the key/value head.  A thread-block cluster of C CTAs (C = 1..8,
// chosen on the host from the layout's longest row and the number of query
// groups, so that short rows spread over many SMs and long batches do not
// exceed the CTAs the GPU holds at once) serves G query rows of one key/value
// head (G = 2 when two rows of a group share a route, else 1); the row's tasks
// are dealt round-robin over the cluster's warps.  A warp brings a task's K and
// V rows into its own buffer with two bulk copies on an mbarrier; small tasks
// and small buffers keep 24 warps on an SM, which is what hides the copies'
// latency.  The page numbers of a warp's next 32 tasks are fetched at once by
// its lanes.  Scoring: 8 lanes per key row, four rows per step, q held in
// registers, packed fp32 FMAs; a warp keeps an fp32 online softmax per query
// (P is not rounded to bf16) and accumulates P V with lanes across d.  The
// warps' partial (max, sum, o) are merged in shared memory, each CTA stores
// its merged state into CTA 0's (then idle) tile buffers through distributed
// shared memory, and CTA 0 merges those; o is stored as bf16 and lse in fp32.
//
// Positions and page numbers come from device memory: a position outside
// [0, n) or a page outside [0, num_pages) is not read; the kernel records a
// status bit (reported by bsa_get_status) and writes o = 0, lse = -inf for
// the rows of that cluster.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "bsa_internal.h"

namespace bsa {
namespace dec {

constexpr int kRows = 16;                           // key rows per task
constexpr int kMaxCluster = 8;                      // CTAs per cluster at most (portable size)
constexpr uint64_t kWaitLimitNs = 1000000000ull;    // a copy that takes longer than 1 s is abandoned
constexpr float kLn2 = 0.693147180559945309f;
constexpr int kFlagBadIndex = 1, kFlagTimeout = 2;

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const int32_t* page_table;
  const int32_t* positions;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  uint32_t* status;
  int n, nb, L, max_blocks, num_pages;
  int H, hkv, g;        // query heads and key/value heads per sequence, H / hkv
  int C;                // CTAs per cluster (the grid's x extent is query groups * C)
  float scale_log2;
};

// Warps per CTA, each with one buffer for its current task's K and V rows.
constexpr int kWarps = 6;
template <int HD>
__host__ __device__ constexpr uint32_t task_tile_bytes() {   // one task's K (or V) rows
  return uint32_t(kRows) * HD * 2;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// One contiguous run global -> shared by the bulk-copy engine (no multicast),
// completing the given mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// Bounded wait for a phase of an mbarrier; false if it did not complete in time.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = gtimer();
  while (true) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}\n"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    if (ok) return true;
    if (gtimer() - t0 > kWaitLimitNs) return false;
  }
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// (d0, d1) += (a0, a1) * (b0, b1), two fp32 lanes in one instruction, each
// rounded as the scalar fma would be.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// bf16 pair (low half first) to two floats: a bf16 is the high half of an fp32.
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}
__device__ __forceinline__ int cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return int(r);
}
// Cluster barrier in two halves: every thread of every CTA arrives, then waits
// for all of them.  With release/acquire, writes before the arrival (shared
// memory of other CTAs included) are visible after the wait.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, int rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ void st_peer_f32(uint32_t a, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void st_peer_s32(uint32_t a, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

template <int BLK, int HD, int G>
__global__ void __launch_bounds__(kWarps * 32, 4) bsa_decode_kernel(const DecodeParams p) {
  constexpr int W = kWarps;
  constexpr int PB = BLK / kRows;     // tasks per page
  constexpr int CPL = HD / 8;         // key columns per lane (8 lanes per key row)
  constexpr int DPL = HD / 32;        // o columns per lane
  constexpr uint32_t kTile = task_tile_bytes<HD>();
  constexpr unsigned kAll = 0xffffffffu;
  static_assert(kRows <= 32 && kRows % 4 == 0, "a task's rows map onto a warp's lanes");
  // Per warp: the K and V rows of its current task.  After the last task the
  // same buffer holds the warp's partial o (G x HD fp32) and, at CTA 0, two of
  // the cluster's CTA partial states (o[HD], max, sum per query) behind it.
  constexpr uint32_t kPartialBytes = G * (HD + 2) * 4;
  static_assert(G * HD * 4 + 2 * kPartialBytes <= 2 * kTile && (kMaxCluster + 1) / 2 <= W,
                "a warp's buffer holds its partial o and two CTA partial states");
  extern __shared__ __align__(128) uint8_t dyn[];
  __shared__ __align__(8) uint64_t bars[W];
  __shared__ float sp[W][G][kRows];               // scores, then P, of a warp's task
  __shared__ float sm[W][G], sl[W][G];
  __shared__ int xflags[kMaxCluster];             // at CTA 0: each CTA's flags
  __shared__ int s_flags, s_start, s_len, s_t;

  const int C = p.C;
  const int rank = cluster_rank();
  const int f0 = (blockIdx.x / C) * G;            // the cluster's rows f0 .. f0 + G - 1
  const int b = f0 / p.H;
  const int hk = (f0 - b * p.H) / p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float sl2 = p.scale_log2;
  // CTA r's partial state for query gq, at CTA 0
  auto partial = [&](int r, int gq) -> float* {
    return reinterpret_cast<float*>(dyn + size_t(r >> 1) * 2 * kTile + G * HD * 4 + (r & 1) * kPartialBytes) +
           gq * (HD + 2);
  };
  if (threadIdx.x == 0) {
    const int t = p.positions[b];
    int start = 0, len = 0, flags = 0;
    if (t >= 0 && t < p.n) {
      const size_t row = size_t(f0 % p.L) * p.nb + t / BLK;
      start = p.row_ptr[row];
      len = p.row_ptr[row + 1] - start;
    } else {
      flags = kFlagBadIndex;
    }
    s_t = t;
    s_start = start;
    s_len = len;
    s_flags = flags;
  }
  if (lane == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[warp])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // this lane's query columns, in registers
  const int sub = lane >> 3, pc = lane & 7;       // key row within a step of 4, column slice
  float qr[G][CPL];
#pragma unroll
  for (int gq = 0; gq < G; ++gq) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + size_t(f0 + gq) * HD + pc * CPL);
#pragma unroll
    for (int c8 = 0; c8 < CPL / 8; ++c8) {
      const uint4 w = src[c8];
      bf16x2_to_f32(w.x, qr[gq][c8 * 8 + 0], qr[gq][c8 * 8 + 1]);
      bf16x2_to_f32(w.y, qr[gq][c8 * 8 + 2], qr[gq][c8 * 8 + 3]);
      bf16x2_to_f32(w.z, qr[gq][c8 * 8 + 4], qr[gq][c8 * 8 + 5]);
      bf16x2_to_f32(w.w, qr[gq][c8 * 8 + 6], qr[gq][c8 * 8 + 7]);
    }
  }
  __syncthreads();

  const int t = s_t, start = s_start, len = s_len;
  const int T = len * PB;                         // tasks of the row
  const int gw = rank * W + warp, S = C * W;      // this warp's first task, stride
  const int mine = T > gw ? (T - gw + S - 1) / S : 0;
  uint8_t* wbase = dyn + size_t(warp) * 2 * kTile;
  const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(wbase);
  const __nv_bfloat16* vt = kt + kRows * HD;
  const uint32_t bar = smem_u32(&bars[warp]);
  float m[G], l[G], acc[G][DPL];
#pragma unroll
  for (int gq = 0; gq < G; ++gq) {
    m[gq] = -INFINITY;
    l[gq] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[gq][e] = 0.f;
  }
  // lane x holds the key block and page of local task m0 + x
  int m0 = -32, idx_j = 0, idx_page = -1;
  uint32_t phase = 0;                             // parity of the buffer's next completion
  bool live = false;                              // copies in flight into the buffer
  int flags = 0;

  for (int mt = 0; mt < mine; ++mt) {
    if (mt - m0 >= 32) {                          // page numbers of the next 32 tasks
      m0 = mt;
      const int x = mt + lane;
      idx_j = 0;
      idx_page = -1;
      if (x < mine) {
        const int k = gw + x * S;
        idx_j = p.col_idx[start + k / PB];
        idx_page = p.page_table[size_t(b) * p.max_blocks + idx_j];
      }
    }
    const int j = __shfl_sync(kAll, idx_j, mt - m0);
    const int page = __shfl_sync(kAll, idx_page, mt - m0);
    const int u0 = j * BLK + ((gw + mt * S) % PB) * kRows;   // the task's first key
    if (page < 0 || page >= p.num_pages) {
      flags |= kFlagBadIndex;
      continue;
    }
    if (u0 > t) continue;                         // every key of the task is after the token
    if (lane == 0) {                              // every lane is done with the last task (warp barrier below)
      const size_t off = (size_t(page) * p.hkv + hk) * BLK * HD + size_t(u0 - j * BLK) * HD;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // earlier reads before the copy
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2 * kTile) : "memory");
      bulk_load(smem_u32(kt), p.kc + off, kTile, bar);
      bulk_load(smem_u32(vt), p.vc + off, kTile, bar);
    }
    live = true;
    const bool landed = bar_wait(bar, phase);
    if (!__all_sync(kAll, landed)) {              // the drain below waits on the same phase
      flags |= kFlagTimeout;
      break;
    }
    phase ^= 1u;
    live = false;
    // ---- scores: rows 4 * step + sub, columns pc * CPL ..
#pragma unroll 2
    for (int step = 0; step < kRows / 4; ++step) {
      const int r = step * 4 + sub;
      const uint4* kr = reinterpret_cast<const uint4*>(kt + size_t(r) * HD + pc * CPL);
      float d0[G], d1[G];
#pragma unroll
      for (int gq = 0; gq < G; ++gq) d0[gq] = d1[gq] = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < CPL / 8; ++c8) {
        const uint4 w = kr[c8];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          float k0, k1;
          bf16x2_to_f32(ws[e2], k0, k1);
#pragma unroll
          for (int gq = 0; gq < G; ++gq)
            fma2(d0[gq], d1[gq], k0, k1, qr[gq][c8 * 8 + 2 * e2], qr[gq][c8 * 8 + 2 * e2 + 1]);
        }
      }
#pragma unroll
      for (int gq = 0; gq < G; ++gq) {
        float dot = d0[gq] + d1[gq];
        dot += __shfl_xor_sync(kAll, dot, 1);
        dot += __shfl_xor_sync(kAll, dot, 2);
        dot += __shfl_xor_sync(kAll, dot, 4);
        if (pc == 0) sp[warp][gq][r] = (u0 + r <= t) ? dot * sl2 : -INFINITY;
      }
    }
    __syncwarp();
    // ---- online softmax per query; lane x < kRows owns key row x of the task
#pragma unroll
    for (int gq = 0; gq < G; ++gq) {
      const float s = lane < kRows ? sp[warp][gq][lane] : -INFINITY;
      float bm = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(kAll, bm, off));
      const float m_new = fmaxf(m[gq], bm);        // finite: the task's first key is allowed
      const float alpha = ex2(m[gq] - m_new);      // 0 while m is -inf
      const float pv = ex2(s - m_new);             // 0 for a disallowed key or an idle lane
      if (lane < kRows) sp[warp][gq][lane] = pv;
      float psum = pv;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(kAll, psum, off);
      l[gq] = l[gq] * alpha + psum;
      m[gq] = m_new;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[gq][e] *= alpha;
    }
    __syncwarp();
    // ---- O += P V: lane owns columns lane * DPL ..
#pragma unroll 8
    for (int r = 0; r < kRows; ++r) {
      const __nv_bfloat16* vr = vt + size_t(r) * HD + lane * DPL;
      float vv[DPL];
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vr);
        bf16x2_to_f32(w.x, vv[0], vv[1]);
        bf16x2_to_f32(w.y, vv[2], vv[3]);
      } else {
        bf16x2_to_f32(*reinterpret_cast<const uint32_t*>(vr), vv[0], vv[1]);
      }
#pragma unroll
      for (int gq = 0; gq < G; ++gq) {
        const float pu = sp[warp][gq][r];
#pragma unroll
        for (int e2 = 0; e2 < DPL; e2 += 2) fma2(acc[gq][e2], acc[gq][e2 + 1], pu, pu, vv[e2], vv[e2 + 1]);
      }
    }
    __syncwarp();
  }
  // leave no copy in flight into shared memory
  if (lane == 0 && live && !bar_wait(bar, phase)) flags |= kFlagTimeout;
  __syncwarp();
  flags = __reduce_or_sync(kAll, flags);
  if (lane == 0 && flags) atomicOr(&s_flags, flags);
  // ---- merge the warps' partial softmax states (o over the warp's own buffer)
  float* so = reinterpret_cast<float*>(wbase);
#pragma unroll
  for (int gq = 0; gq < G; ++gq) {
    if (lane == 0) {
      sm[warp][gq] = m[gq];
      sl[warp][gq] = l[gq];
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) so[gq * HD + lane * DPL + e] = acc[gq][e];
  }
  __syncthreads();
  // Every CTA of the cluster is done with its tiles (CTA 0's buffers take the
  // partial states next).
  cluster_arrive();
  cluster_wait();
  for (int c = threadIdx.x; c < G * HD; c += W * 32) {
    const int gq = c / HD, col = c % HD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, sm[w][gq]);
    float Lsum = 0.f, v = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float wt = (M == -INFINITY) ? 0.f : ex2(sm[w][gq] - M);
      Lsum += wt * sl[w][gq];
      v += wt * reinterpret_cast<const float*>(dyn + size_t(w) * 2 * kTile)[gq * HD + col];
    }
    // this CTA's partial state into CTA 0's shared memory
    float* dst = partial(rank, gq);
    st_peer_f32(peer_addr(dst + col, 0), v);
    if (col == 0) {
      st_peer_f32(peer_addr(dst + HD, 0), M);
      st_peer_f32(peer_addr(dst + HD + 1, 0), Lsum);
    }
  }
  if (threadIdx.x == 0) st_peer_s32(peer_addr(&xflags[rank], 0), s_flags);
  cluster_arrive();
  cluster_wait();                                 // the partial states have landed at CTA 0
  if (rank != 0) return;
  int all_flags = 0;
  for (int r = 0; r < C; ++r) all_flags |= xflags[r];
  for (int c = threadIdx.x; c < G * HD; c += W * 32) {
    const int gq = c / HD, col = c % HD;
    float M = -INFINITY;
    for (int r = 0; r < C; ++r) M = fmaxf(M, partial(r, gq)[HD]);
    float Lsum = 0.f, v = 0.f;
    for (int r = 0; r < C; ++r) {
      const float* x = partial(r, gq);
      const float wt = (M == -INFINITY) ? 0.f : ex2(x[HD] - M);
      Lsum += wt * x[HD + 1];
      v += wt * x[col];
    }
    const bool ok = Lsum > 0.f && all_flags == 0;
    p.o[size_t(f0 + gq) * HD + col] = __float2bfloat16_rn(ok ? v / Lsum : 0.f);
    if (col == 0) p.lse[f0 + gq] = ok ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
  }
  if (threadIdx.x == 0 && all_flags)
    atomicOr(p.status, (all_flags & kFlagTimeout ? kStatusTimeout : 0u) |
                           (all_flags & kFlagBadIndex ? kStatusBadIndex : 0u));
}

// CTAs per cluster: enough warps for one task each on the longest row, cut
// back while the grid would exceed the CTAs the GPU holds at once.
inline int cluster_size(int groups, int max_row, int tasks_per_page, int warps, int resident) {
  const int tasks = std::max(1, max_row * tasks_per_page);
  int c = std::min(kMaxCluster, (tasks + warps - 1) / warps);
  while (c > 1 && size_t(groups) * c > size_t(resident)) c = (c + 1) / 2;
  return std::max(c, 1);
}

template <int BLK, int HD, int G>
int launch_g(DecodeParams p, int heads, int max_row, cudaStream_t s) {
  auto kern = bsa_decode_kernel<BLK, HD, G>;
  constexpr int W = kWarps;
  const int smem = W * 2 * int(task_tile_bytes<HD>());
  // the attribute is a property of the function: set it once per device
  static std::mutex mu;
  static bool done[64] = {};
  static int resident[64] = {};                   // CTAs the GPU holds at once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return set_error(BSA_ERR_CUDA, "cannot query the device");
  int n_resident = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("decode smem: ") + cudaGetErrorString(e));
      int n_sm = 0, per_sm = 0;
      e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
      if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, W * 32, smem);
      if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("decode occupancy: ") + cudaGetErrorString(e));
      resident[dev] = std::max(1, n_sm * per_sm);
      done[dev] = true;
    }
    n_resident = resident[dev];
  }
  const int groups = heads / G;
  p.C = cluster_size(groups, max_row, BLK / kRows, W, n_resident);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(groups * p.C), 1, 1);
  cfg.blockDim = dim3(W * 32, 1, 1);
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(p.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
  return BSA_OK;
}

template <int BLK, int HD>
int launch(const DecodeParams& p, int heads, int max_row, cudaStream_t s) {
  // two query rows of a key/value head's group per cluster when they share a route
  return (p.L == 1 && p.g % 2 == 0) ? launch_g<BLK, HD, 2>(p, heads, max_row, s)
                                    : launch_g<BLK, HD, 1>(p, heads, max_row, s);
}

}  // namespace dec
}  // namespace bsa

extern "C" int bsa_decode(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* page_table, int max_blocks, int num_pages,
                          const int32_t* positions, const bsa_layout* layout, int batch, int heads,
                          int kv_heads, int d, float scale, void* o, float* lse, void* stream) {
  using namespace bsa;
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (layout->device < 0 || !layout->d_base)
    return set_error(BSA_ERR_INVALID_ARG, "layout was built host-only (device = -1)");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (cur != layout->device) return set_error(BSA_ERR_INVALID_ARG, "layout lives on another device");
  const int B = layout->B;
  if (B != 64 && B != 128) return set_error(BSA_ERR_UNSUPPORTED, "B must be 64 or 128");
  if (d != 64 && d != 128) return set_error(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (batch < 1 || heads < 1 || kv_heads < 1) return set_error(BSA_ERR_SHAPE, "batch, heads and kv_heads must be >= 1");
  if (heads % batch || kv_heads % batch)
    return set_error(BSA_ERR_SHAPE, "heads and kv_heads must be multiples of batch");
  const int H = heads / batch, hkv = kv_heads / batch;
  if (H % hkv) return set_error(BSA_ERR_SHAPE, "query heads per sequence must be a multiple of its kv heads");
  if (H % layout->L) return set_error(BSA_ERR_SHAPE, "query heads per sequence must be a multiple of layout_heads");
  if (max_blocks < layout->nb) return set_error(BSA_ERR_SHAPE, "max_blocks is smaller than the layout's blocks");
  if (num_pages < 1) return set_error(BSA_ERR_SHAPE, "num_pages must be >= 1");
  if (!(std::isfinite(scale) && scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!q || !k_cache || !v_cache || !page_table || !positions || !o || !lse)
    return set_error(BSA_ERR_INVALID_ARG, "null pointer");
  auto aligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16))
    return set_error(BSA_ERR_INVALID_ARG, "q, k_cache, v_cache and o must be 16-byte aligned");
  if (!aligned(lse, 4) || !aligned(page_table, 4) || !aligned(positions, 4))
    return set_error(BSA_ERR_INVALID_ARG, "lse, page_table and positions must be 4-byte aligned");
  dec::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(k_cache);
  p.vc = static_cast<const __nv_bfloat16*>(v_cache);
  p.page_table = page_table;
  p.positions = positions;
  p.row_ptr = layout->d_row_ptr;
  p.col_idx = layout->d_col_idx;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = layout->d_status;
  p.n = layout->n;
  p.nb = layout->nb;
  p.L = layout->L;
  p.max_blocks = max_blocks;
  p.num_pages = num_pages;
  p.H = H;
  p.hkv = hkv;
  p.g = H / hkv;
  p.scale_log2 = float(double(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int mr = layout->max_row;
  if (B == 64 && d == 128) return dec::launch<64, 128>(p, heads, mr, s);
  if (B == 64 && d == 64) return dec::launch<64, 64>(p, heads, mr, s);
  if (B == 128 && d == 128) return dec::launch<128, 128>(p, heads, mr, s);
  return dec::launch<128, 64>(p, heads, mr, s);
}
