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
// Three launches on the caller's stream: D (one warp per row), then the dq
// kernel (one CTA per query tile, walking the tile's CSR row of kept blocks)
// and the dk/dv kernel (one CTA per segment of a key block's column of the
// transposed layout, walking the query tiles that read it).  Both product
// kernels use 160 threads: warp 0 issues the TMA loads and, from one thread,
// the tcgen05 products; warps 1-4 hold one tile row per thread (warp w reaches
// TMEM lanes 32 (w % 4) ..) and rebuild P and dS.  Every product is a
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

#include "bsa_internal.h"

namespace bsa {
namespace bwd {

constexpr uint32_t kSuspendHintNs = 1000000;   // longest single suspension inside a wait

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Slow path of a bounded wait: poll (each try suspends the thread for up to
// kSuspendHintNs or until the phase completes) until the phase completes, the
// CTA's abort flag is raised, or `limit_ns` passes; on time-out record the
// status bit and raise the abort flag.
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       uint32_t* status, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

struct Ctl {
  volatile int* abort;   // shared: set once any wait of this CTA ran out
  uint32_t* status;      // global status word
  uint64_t timeout_ns;
  // Bounded wait for the completion of the phase with the given parity.
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, abort, status, timeout_ns);
  }
};

// Bounded wait that ignores the abort flag (used while draining on exit).
__device__ __noinline__ void wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return;
  }
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// TMA (no multicast anywhere in this library).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// One 64-key chunk of K or V (rows r0 .. r0+63 of head h, all d columns) as a
// single box: the tensor map's third dimension walks the 64-column swizzle
// atoms, so the box lands as [atom][row][64 columns], the layout the MMA
// descriptors read.
template <int HD>
__device__ __forceinline__ void tma_load_kv(uint32_t dst, const CUtensorMap* m, uint32_t bar, int r0, int h) {
  if constexpr (HD == 128) tma_load_4d(dst, m, bar, 0, r0, 0, h);
  else tma_load_3d(dst, m, bar, 0, r0, h);
}
// The whole 128-row Q tile as a single box: for B = 64 the box spans two
// consecutive heads (the two stacked query blocks), for B = 128 one block.
template <int BLK, int HD>
__device__ __forceinline__ void tma_load_q(uint32_t dst, const CUtensorMap* m, uint32_t bar, int r0, int h) {
  if constexpr (HD == 128 && BLK == 64) tma_load_4d(dst, m, bar, 0, r0, h, 0);
  else if constexpr (HD == 128) tma_load_4d(dst, m, bar, 0, r0, 0, h);
  else tma_load_3d(dst, m, bar, 0, r0, h);
}

// tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc)
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc)
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 consecutive 32-bit columns (each holding two bf16 values).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* u) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]),
      "r"(u[8]), "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((addr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// ---------------------------------------------------------------- shared
constexpr int kThreads = 160;        // warp 0: loads and products; warps 1-4: one tile row per thread
constexpr int kTileM = 128;          // rows of every product tile (tcgen05 M = 128)
constexpr int kChunk = 64;           // keys per chunk
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kDrainNs = 200000000ull;

// Instruction descriptor of a kind::f16 product with bf16 operands and an fp32
// accumulator; a_mn / b_mn select operands stored along M / N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

struct Params {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* order;
  const int32_t* row_idx;
  const int32_t* seg_ptr;
  const int32_t* segs;
  const float* lse;      // forward lse (natural log)
  const float* dsum;     // D = rowsum(dO * o)
  float* dq;
  float* dk;
  float* dv;
  uint32_t* status;
  int n, nb, L, kv_heads, group, pack, n_steps;   // n_steps = group / pack head steps per key/value head
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

// P and dS of one tile row against one 64-key chunk, from the raw scores s
// (q.k) and dP (dO.v): P = exp(scale s - lse), dS = P (dP - D).  Keys past
// `lim` (causal, diagonal block) and rows that are not real get 0.  dS
// overwrites s.
__device__ __forceinline__ void p_ds_row(float* s, const float* dp, float* pv, float sl2, float lse2, float dd,
                                         int lim, bool live) {
#pragma unroll
  for (int c = 0; c < kChunk; ++c) {
    const bool keep = live && c <= lim;
    const float pr = keep ? ex2(fmaf(s[c], sl2, -lse2)) : 0.f;
    pv[c] = pr;
    s[c] = pr * (dp[c] - dd);
  }
}

// ---------------------------------------------------------------- D = rowsum(dO * o)
// One warp per query row: D_t = sum_u P_tu dP_tu, which equals <dO_t, o_t>.
template <int HD>
__global__ void __launch_bounds__(256) bsa_bwd_rowdot_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                             float* dsum, size_t rows) {
  const size_t row = size_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
#pragma unroll
  for (int c = lane * 4; c < HD; c += 128) {
    const uint2 a = *reinterpret_cast<const uint2*>(o + row * HD + c);
    const uint2 b = *reinterpret_cast<const uint2*>(dout + row * HD + c);
    const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.x));
    const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.y));
    const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.x));
    const float2 b1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.y));
    acc = fmaf(a0.x, b0.x, fmaf(a0.y, b0.y, fmaf(a1.x, b1.x, fmaf(a1.y, b1.y, acc))));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dsum[row] = acc;
}

// ---------------------------------------------------------------- dQ
// One CTA per query tile, tiles longest row first.  Per 64-key chunk c of the
// tile's kept blocks: S = Q K_c^T and dP = dO V_c^T into TMEM buffer c & 1;
// the row threads turn them into dS = P (dP - D), rounded to bf16 over the S
// buffer; then dQ += dS K_c (A = dS read from TMEM, B = K_c read along d).
// K_c and V_c stay in shared-memory slot c % 3 until dQ_c is done.
template <int BLK, int HD>
struct DqShape {
  static constexpr int kCPB = BLK / kChunk;
  static constexpr int kQBytes = kTileM * HD * 2;
  static constexpr int kTile = kChunk * HD * 2;
  static constexpr int kAtomQ = kTileM * 128;
  static constexpr int kAtomKV = kChunk * 128;
  static constexpr int kOffDO = kQBytes;
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + 3 * kTile;
  static constexpr int kOffBar = kOffV + 3 * kTile;
  // q_full, kv_full[3], s_full[2], ds_full[2], dq_done[3], drain
  static constexpr int kNumBars = 12;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16;
  static constexpr int kColS = 0, kColDP = 128, kColQ = 256;
  static constexpr uint32_t kIdescS = idesc_bf16(kTileM, kChunk, 0, 0);
  static constexpr uint32_t kIdescDQ = idesc_bf16(kTileM, HD, 0, 1);
  static_assert(4 * 32 * 33 * 4 <= 3 * kTile, "epilogue staging fits the K ring");
};

template <int BLK, int HD>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const Params p) {
  using S = DqShape<BLK, HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  const uint32_t sQ = base, sDO = base + S::kOffDO, sK = base + S::kOffK, sV = base + S::kOffV;
  const uint32_t bar0 = base + S::kOffBar;
  const uint32_t bQ = bar0;
  auto bKV = [&](int c) { return bar0 + 8u * (1 + c % 3); };
  auto bS = [&](int c) { return bar0 + 8u * (4 + (c & 1)); };
  auto bDS = [&](int c) { return bar0 + 8u * (6 + (c & 1)); };
  auto bDQ = [&](int c) { return bar0 + 8u * (8 + c % 3); };
  const uint32_t bDrain = bar0 + 8u * 11;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem_raw + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + S::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};

  // item -> (rank in the longest-first order, head group): every head
  // group's longest rows go first
  const int n_hg = gridDim.x / p.nb;
  const int rank = blockIdx.x / n_hg, hg = blockIdx.x - rank * n_hg;
  const int h0 = hg * p.pack;
  const int lh = h0 % p.L;
  const QTile tile{p.order[size_t(lh) * p.nb + rank], h0};
  const int kvh = h0 / p.group;
  const size_t lrow = size_t(lh) * p.nb + tile.i;
  const int start = p.row_ptr[lrow], len = p.row_ptr[lrow + 1] - start;
  const bool diag_last = len > 0 && p.col_idx[start + len - 1] == tile.i;
  const int nch = len * S::kCPB;
  const int diag_first = diag_last ? nch - S::kCPB : nch;

  if (threadIdx.x == 0) {
    mbar_init(bQ, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar0 + 8u * (1 + s), 1);
      mbar_init(bar0 + 8u * (8 + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar0 + 8u * (4 + s), 1);
      mbar_init(bar0 + 8u * (6 + s), 128);
    }
    mbar_init(bDrain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(base + S::kOffMisc, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0 && nch > 0) {
      bool ok = true;
      int loaded = 0;
      auto key0 = [&](int c) { return p.col_idx[start + c / S::kCPB] * BLK + (c % S::kCPB) * kChunk; };
      auto load = [&](int c) -> bool {
        if (c >= 3 && !ctl.wait(bDQ(c), uint32_t((c - 3) / 3) & 1u)) return false;   // dQ_{c-3} done
        mbar_expect_tx(bKV(c), 2 * S::kTile);
        const uint32_t slot = uint32_t(c % 3) * S::kTile;
        const int k0 = key0(c);
        tma_load_kv<HD>(sK + slot, &tmK, bKV(c), k0, kvh);
        tma_load_kv<HD>(sV + slot, &tmV, bKV(c), k0, kvh);
        ++loaded;
        return true;
      };
      auto products_s = [&](int c) -> bool {
        if (!ctl.wait(bKV(c), uint32_t(c / 3) & 1u)) return false;
        tc_fence_after();
        const uint32_t slot = uint32_t(c % 3) * S::kTile;
        const uint32_t ds = tmem + S::kColS + (c & 1) * kChunk, ddp = tmem + S::kColDP + (c & 1) * kChunk;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * S::kAtomQ + (kk & 3) * 32, bo = (kk >> 2) * S::kAtomKV + (kk & 3) * 32;
          mma_ss(ds, sw128_desc(sQ + ao, 16, 1024), sw128_desc(sK + slot + bo, 16, 1024), S::kIdescS, kk > 0);
          mma_ss(ddp, sw128_desc(sDO + ao, 16, 1024), sw128_desc(sV + slot + bo, 16, 1024), S::kIdescS, kk > 0);
        }
        tc_commit(bS(c));
        return true;
      };
      auto product_dq = [&](int c) -> bool {
        if (!ctl.wait(bDS(c), uint32_t(c >> 1) & 1u)) return false;
        tc_fence_after();
        const uint32_t slot = uint32_t(c % 3) * S::kTile;
        const uint32_t pa = tmem + S::kColS + (c & 1) * kChunk;
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_ts(tmem + S::kColQ, pa + kk * 8, sw128_desc(sK + slot + kk * 16 * 128, S::kAtomKV, 1024), S::kIdescDQ,
                 (c > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bDQ(c));
        return true;
      };
      mbar_expect_tx(bQ, 2 * S::kQBytes);
      tma_load_q<BLK, HD>(sQ, &tmQ, bQ, tile.i * BLK, tile.h0);
      tma_load_q<BLK, HD>(sDO, &tmDO, bQ, tile.i * BLK, tile.h0);
      for (int c = 0; c < nch && c < 3 && ok; ++c) ok = load(c);
      if (ok) ok = ctl.wait(bQ, 0);
      if (ok) ok = products_s(0);
      if (ok && nch > 1) ok = products_s(1);
      for (int c = 0; c < nch && ok; ++c) {
        ok = product_dq(c);
        if (ok && c + 2 < nch) ok = products_s(c + 2);
        if (ok && c + 3 < nch) ok = load(c + 3);
      }
      tc_commit(bDrain);
      wait_drain(bDrain, 0, kDrainNs);
      wait_drain(bQ, 0, kDrainNs);
      for (int c = (loaded > 3 ? loaded - 3 : 0); c < loaded; ++c) wait_drain(bKV(c), uint32_t(c / 3) & 1u, kDrainNs);
    }
  } else {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(q4 * 32) << 16);
    int head, tok;
    const bool real = tile_row<BLK>(p, tile, r, head, tok);
    const int rl = r - (r / BLK) * BLK;
    const size_t rowi = size_t(head) * p.n + (real ? tok : 0);
    const float lse2 = real ? p.lse[rowi] * kLog2e : 0.f;
    const float dd = real ? p.dsum[rowi] : 0.f;
    const bool live = real && lse2 > -INFINITY;
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      ok = __all_sync(0xffffffffu, ctl.wait(bS(c), uint32_t(c >> 1) & 1u));
      if (!ok) break;
      tc_fence_after();
      float s[kChunk], dp[kChunk], pv[kChunk];
      const uint32_t cs = lane_base + S::kColS + (c & 1) * kChunk, cd = lane_base + S::kColDP + (c & 1) * kChunk;
      tmem_ld32(cs, s);
      tmem_ld32(cs + 32, s + 32);
      tmem_ld32(cd, dp);
      tmem_ld32(cd + 32, dp + 32);
      tmem_wait_ld();
      const int lim = c >= diag_first ? rl - (c - diag_first) * kChunk : kChunk;
      p_ds_row(s, dp, pv, p.scale_log2, lse2, dd, lim, live);
#pragma unroll
      for (int h = 0; h < kChunk / 32; ++h) {
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(s[h * 32 + 2 * e], s[h * 32 + 2 * e + 1]);
        tmem_st16(cs + h * 16, u);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bDS(c));
    }
    if (ok && nch > 0) ok = __all_sync(0xffffffffu, ctl.wait(bDQ(nch - 1), uint32_t((nch - 1) / 3) & 1u));
    if (ok) {
      // dQ = scale * acc, through a per-warp [32 rows][33] staging tile in the
      // (idle) K ring so each row is written as whole 128-byte lines
      tc_fence_after();
      float* stage = reinterpret_cast<float*>(smem_raw + S::kOffK) + q4 * 32 * 33;
      const int row0 = q4 * 32;
#pragma unroll 1
      for (int a = 0; a < HD / 32; ++a) {
        float v[32];
        if (nch > 0) {
          tmem_ld32(lane_base + S::kColQ + a * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) stage[lane * 33 + e] = v[e] * p.scale;
        __syncwarp();
        for (int rr = 0; rr < 32; ++rr) {
          int hh, tt;
          if (tile_row<BLK>(p, tile, row0 + rr, hh, tt))
            p.dq[(size_t(hh) * p.n + tt) * HD + a * 32 + lane] = stage[rr * 33 + lane];
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV
// One CTA per (key/value head, query-head step, 64-key chunk of a key block,
// column segment): the segment lists up to 16 query blocks whose rows keep
// the key block (the transposed layout).  Per query tile t of the segment:
// S = Q K^T and dP = dO V^T (M = 128 query rows) into TMEM buffer t & 1; the
// row threads write P and dS = P (dP - D) as bf16 [query][key] tiles into
// shared-memory buffer t & 1; then dV^T += dO^T P and dK^T += Q^T dS (M = 128
// along d: A is the dO / Q tile read along d, B the P / dS tile read along
// the keys; for d = 64 the upper 64 rows of M read the neighbouring tile and
// are never stored).  The sums are added into dk and dv (zeroed first), as
// segments of one column run on several CTAs.
template <int BLK, int HD>
struct DkvShape {
  static constexpr int kQBytes = kTileM * HD * 2;
  static constexpr int kTile = kChunk * HD * 2;
  static constexpr int kAtomQ = kTileM * 128;
  static constexpr int kAtomKV = kChunk * 128;
  static constexpr int kPBytes = kTileM * kChunk * 2;      // one [128 queries][64 keys] bf16 tile
  static constexpr int kOffK = 4 * kQBytes;                // Q, dO of tile t at (t & 1) * 2 * kQBytes
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffP = kOffV + kTile;              // P[2], dS[2]
  static constexpr int kOffBar = kOffP + 4 * kPBytes;
  // kv_full, q_full[2], s_full[2], pds_full[2], done[2], drain
  static constexpr int kNumBars = 10;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffTiles = kOffMisc + 16;          // the segment's query blocks
  static constexpr int kSmem = kOffTiles + kColumnSegment * 4;
  static constexpr int kColS = 0, kColDP = 128, kColV = 256, kColK = 320;
  static constexpr uint32_t kIdescS = idesc_bf16(kTileM, kChunk, 0, 0);
  static constexpr uint32_t kIdescT = idesc_bf16(kTileM, kChunk, 1, 1);
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int BLK, int HD>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params p) {
  using S = DkvShape<BLK, HD>;
  constexpr int CPB = BLK / kChunk;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  // item -> (segment rank, key/value head, head step, chunk): the longest
  // segments of every head go first
  const int inner = p.n_steps * CPB;                     // (head step, chunk) per key/value head
  const int kv_heads = p.kv_heads;
  const int rank = blockIdx.x / (kv_heads * inner);
  int rem = blockIdx.x - rank * (kv_heads * inner);
  const int kvh = rem / inner;
  rem -= kvh * inner;
  const int hs = rem / CPB, hh = rem - hs * CPB;
  const int h0 = kvh * p.group + hs * p.pack;
  const int lh = h0 % p.L;
  const int seg = p.seg_ptr[lh] + rank;
  if (seg >= p.seg_ptr[lh + 1]) return;                  // this layout head has fewer segments
  const int j = p.segs[3 * seg], e0 = p.segs[3 * seg + 1], total = p.segs[3 * seg + 2];
  const int key0 = j * BLK + hh * kChunk;

  auto sQ = [&](int t) { return base + uint32_t(t & 1) * 2 * S::kQBytes; };
  auto sDO = [&](int t) { return sQ(t) + S::kQBytes; };
  const uint32_t sK = base + S::kOffK, sV = base + S::kOffV;
  auto sP = [&](int t) { return base + S::kOffP + uint32_t(t & 1) * S::kPBytes; };
  auto sDS = [&](int t) { return base + S::kOffP + uint32_t(2 + (t & 1)) * S::kPBytes; };
  const uint32_t bar0 = base + S::kOffBar;
  const uint32_t bKV = bar0;
  auto bQ = [&](int t) { return bar0 + 8u * (1 + (t & 1)); };
  auto bS = [&](int t) { return bar0 + 8u * (3 + (t & 1)); };
  auto bPDS = [&](int t) { return bar0 + 8u * (5 + (t & 1)); };
  auto bDone = [&](int t) { return bar0 + 8u * (7 + (t & 1)); };
  const uint32_t bDrain = bar0 + 8u * 9;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem_raw + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + S::kOffMisc + 4);
  int* tiles = reinterpret_cast<int*>(smem_raw + S::kOffTiles);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int b = 0; b < 9; ++b) mbar_init(bar0 + 8u * b, (b == 5 || b == 6) ? 128u : 1u);
    mbar_init(bDrain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < total) tiles[threadIdx.x] = p.row_idx[e0 + threadIdx.x];
  if (warp == 0) {
    tmem_alloc(base + S::kOffMisc, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int q_loads = 0;
      auto load_q = [&](int t) {
        mbar_expect_tx(bQ(t), 2 * S::kQBytes);
        tma_load_q<BLK, HD>(sQ(t), &tmQ, bQ(t), tiles[t] * BLK, h0);
        tma_load_q<BLK, HD>(sDO(t), &tmDO, bQ(t), tiles[t] * BLK, h0);
        ++q_loads;
      };
      auto products_s = [&](int t) -> bool {
        if (!ctl.wait(bQ(t), uint32_t(t >> 1) & 1u)) return false;
        tc_fence_after();
        const uint32_t ds = tmem + S::kColS + (t & 1) * kChunk, ddp = tmem + S::kColDP + (t & 1) * kChunk;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * S::kAtomQ + (kk & 3) * 32, bo = (kk >> 2) * S::kAtomKV + (kk & 3) * 32;
          mma_ss(ds, sw128_desc(sQ(t) + ao, 16, 1024), sw128_desc(sK + bo, 16, 1024), S::kIdescS, kk > 0);
          mma_ss(ddp, sw128_desc(sDO(t) + ao, 16, 1024), sw128_desc(sV + bo, 16, 1024), S::kIdescS, kk > 0);
        }
        tc_commit(bS(t));
        return true;
      };
      mbar_expect_tx(bKV, 2 * S::kTile);
      tma_load_kv<HD>(sK, &tmK, bKV, key0, kvh);
      tma_load_kv<HD>(sV, &tmV, bKV, key0, kvh);
      load_q(0);
      if (total > 1) load_q(1);
      ok = ctl.wait(bKV, 0);
      if (ok) ok = products_s(0);
      if (ok && total > 1) ok = products_s(1);
      for (int t = 0; t < total && ok; ++t) {
        // P, dS of tile t are in shared memory, and S, dP of tile t have been read
        if (!(ok = ctl.wait(bPDS(t), uint32_t(t >> 1) & 1u))) break;
        tc_fence_after();
        // dV^T += dO^T P, dK^T += Q^T dS over the tile's 128 query rows
#pragma unroll
        for (int kk = 0; kk < kTileM / 16; ++kk) {
          const uint32_t off = kk * 16 * 128;
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tmem + S::kColV, sw128_desc(sDO(t) + off, S::kAtomQ, 1024), sw128_desc(sP(t) + off, S::kPBytes, 1024),
                 S::kIdescT, acc);
          mma_ss(tmem + S::kColK, sw128_desc(sQ(t) + off, S::kAtomQ, 1024), sw128_desc(sDS(t) + off, S::kPBytes, 1024),
                 S::kIdescT, acc);
        }
        tc_commit(bDone(t));
        if (t + 2 < total) {
          // tile t + 2 into buffer t & 1 once tile t's products have read it
          if (!(ok = ctl.wait(bDone(t), uint32_t(t >> 1) & 1u))) break;
          load_q(t + 2);
          if (!(ok = products_s(t + 2))) break;
        }
      }
      tc_commit(bDrain);
      wait_drain(bDrain, 0, kDrainNs);
      wait_drain(bKV, 0, kDrainNs);
      for (int t = (q_loads > 2 ? q_loads - 2 : 0); t < q_loads; ++t) wait_drain(bQ(t), uint32_t(t >> 1) & 1u, kDrainNs);
    }
  } else {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(q4 * 32) << 16);
    const int rl = r - (r / BLK) * BLK;
    bool ok = true;
    // the row's lse and D for tile t + 1 are fetched while tile t is computed
    auto row_of = [&](int t, float& lse2, float& dd, bool& live) {
      int head, tok;
      const bool real = tile_row<BLK>(p, QTile{tiles[t], h0}, r, head, tok);
      const size_t rowi = size_t(head) * p.n + (real ? tok : 0);
      lse2 = real ? p.lse[rowi] * kLog2e : 0.f;
      dd = real ? p.dsum[rowi] : 0.f;
      live = real;
    };
    float lse2 = 0.f, dd = 0.f;
    bool live = false;
    if (total > 0) row_of(0, lse2, dd, live);
    for (int t = 0; t < total && ok; ++t) {
      float nlse2 = 0.f, ndd = 0.f;
      bool nlive = false;
      if (t + 1 < total) row_of(t + 1, nlse2, ndd, nlive);
      // causal: in the diagonal block, key (chunk offset + c) > row is dropped
      const int lim = (tiles[t] == j) ? rl - hh * kChunk : kChunk;
      ok = __all_sync(0xffffffffu, ctl.wait(bS(t), uint32_t(t >> 1) & 1u));
      if (!ok) break;
      tc_fence_after();
      float s[kChunk], dp[kChunk], pv[kChunk];
      const uint32_t cs = lane_base + S::kColS + (t & 1) * kChunk, cd = lane_base + S::kColDP + (t & 1) * kChunk;
      tmem_ld32(cs, s);
      tmem_ld32(cs + 32, s + 32);
      tmem_ld32(cd, dp);
      tmem_ld32(cd + 32, dp + 32);
      tmem_wait_ld();
      p_ds_row(s, dp, pv, p.scale_log2, lse2, dd, lim, live && lse2 > -INFINITY);
      // buffer t & 1 was last read by tile t - 2's products
      if (t >= 2) {
        ok = __all_sync(0xffffffffu, ctl.wait(bDone(t), uint32_t((t - 2) >> 1) & 1u));
        if (!ok) break;
      }
      // row r of the [query][key] tiles, 128-byte swizzled
      const uint32_t tp = sP(t), td = sDS(t);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t off = uint32_t(r) * 128 + ((ch ^ (r & 7)) << 4);
        st_shared_v4(tp + off, pack_bf16(pv[8 * ch], pv[8 * ch + 1]), pack_bf16(pv[8 * ch + 2], pv[8 * ch + 3]),
                     pack_bf16(pv[8 * ch + 4], pv[8 * ch + 5]), pack_bf16(pv[8 * ch + 6], pv[8 * ch + 7]));
        st_shared_v4(td + off, pack_bf16(s[8 * ch], s[8 * ch + 1]), pack_bf16(s[8 * ch + 2], s[8 * ch + 3]),
                     pack_bf16(s[8 * ch + 4], s[8 * ch + 5]), pack_bf16(s[8 * ch + 6], s[8 * ch + 7]));
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bPDS(t));
      lse2 = nlse2;
      dd = ndd;
      live = nlive;
    }
    // TMEM lane r holds element d = r of the chunk's 64 key rows
    if (ok && total > 0) ok = __all_sync(0xffffffffu, ctl.wait(bDone(total - 1), uint32_t((total - 1) >> 1) & 1u));
    if (ok && total > 0) {
      tc_fence_after();
      float vk[kChunk], vv[kChunk];
      tmem_ld32(lane_base + S::kColK, vk);
      tmem_ld32(lane_base + S::kColK + 32, vk + 32);
      tmem_ld32(lane_base + S::kColV, vv);
      tmem_ld32(lane_base + S::kColV + 32, vv + 32);
      tmem_wait_ld();
      if (r < HD) {
#pragma unroll
        for (int c = 0; c < kChunk; ++c) {
          const int key = key0 + c;
          if (key < p.n) {
            const size_t at = (size_t(kvh) * p.n + key) * HD + r;
            atomicAdd(p.dk + at, vk[c] * p.scale);
            atomicAdd(p.dv + at, vv[c]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd

// ==================================================================== host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
int g_encode_status = BSA_OK;
std::string g_encode_msg;

int get_encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q{};
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
      g_encode_status = BSA_ERR_CUDA;
      g_encode_msg = std::string("cuTensorMapEncodeTiled unavailable: ") + cudaGetErrorString(e);
      return;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode_status != BSA_OK) return set_error(g_encode_status, g_encode_msg);
  return BSA_OK;
}

int encode_tiled(CUtensorMap* m, const void* ptr, cuuint32_t rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
  return BSA_OK;
}

// K or V [kv_heads][n][d]: a 64-row chunk of one head per box, landing as
// [64-column atom][row][64 columns] (d = 128: the atom is a tensor dimension
// of stride 128 bytes, so one box holds both atoms).
int encode_kv(CUtensorMap* m, const void* ptr, int slices, int n, int d) {
  const cuuint64_t row = cuuint64_t(d) * 2, slice = cuuint64_t(n) * row;
  if (d == 128) {
    const cuuint64_t dims[4] = {64, cuuint64_t(n), 2, cuuint64_t(slices)};
    const cuuint64_t str[3] = {row, 128, slice};
    const cuuint32_t box[4] = {64, 64, 2, 1};
    return encode_tiled(m, ptr, 4, dims, str, box);
  }
  const cuuint64_t dims[3] = {64, cuuint64_t(n), cuuint64_t(slices)};
  const cuuint64_t str[2] = {row, slice};
  const cuuint32_t box[3] = {64, 64, 1};
  return encode_tiled(m, ptr, 3, dims, str, box);
}

// Q or dO [heads][n][d]: one 128-row tile per box (B = 128: one block of one
// head; B = 64: the same block of two consecutive heads), landing as
// [64-column atom][128 rows][64 columns].
int encode_q(CUtensorMap* m, const void* ptr, int heads, int n, int d, int blk) {
  const cuuint64_t row = cuuint64_t(d) * 2, slice = cuuint64_t(n) * row;
  if (d == 128 && blk == 64) {
    const cuuint64_t dims[4] = {64, cuuint64_t(n), cuuint64_t(heads), 2};
    const cuuint64_t str[3] = {row, slice, 128};
    const cuuint32_t box[4] = {64, 64, 2, 2};
    return encode_tiled(m, ptr, 4, dims, str, box);
  }
  if (d == 128) {
    const cuuint64_t dims[4] = {64, cuuint64_t(n), 2, cuuint64_t(heads)};
    const cuuint64_t str[3] = {row, 128, slice};
    const cuuint32_t box[4] = {64, 128, 2, 1};
    return encode_tiled(m, ptr, 4, dims, str, box);
  }
  const cuuint64_t dims[3] = {64, cuuint64_t(n), cuuint64_t(heads)};
  const cuuint64_t str[2] = {row, slice};
  const cuuint32_t box[3] = {64, cuuint32_t(blk), cuuint32_t(blk == 64 ? 2 : 1)};
  return encode_tiled(m, ptr, 3, dims, str, box);
}

struct Launch {
  const void *q, *k, *v, *o, *dout;
  int heads, kv_heads, n, items_dq, items_dkv;
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
  st = encode_q(&mq, a.q, a.heads, a.n, HD, BLK);
  if (st == BSA_OK) st = encode_q(&mdo, a.dout, a.heads, a.n, HD, BLK);
  if (st == BSA_OK) st = encode_kv(&mk, a.k, a.kv_heads, a.n, HD);
  if (st == BSA_OK) st = encode_kv(&mv, a.v, a.kv_heads, a.n, HD);
  if (st != BSA_OK) return st;
  const size_t grad_kv = size_t(a.kv_heads) * a.n * HD * sizeof(float);
  cudaError_t e = cudaMemsetAsync(p.dk, 0, grad_kv, a.stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(p.dv, 0, grad_kv, a.stream);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("clearing dk, dv: ") + cudaGetErrorString(e));
  const unsigned rows_grid = unsigned((a.dq_rows + 7) / 8);
  bwd::bsa_bwd_rowdot_kernel<HD><<<rows_grid, 256, 0, a.stream>>>(
      static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.dsum, a.dq_rows);
  if (a.items_dq > 0) kq<<<a.items_dq, bwd::kThreads, smem_q, a.stream>>>(mq, mdo, mk, mv, p);
  if (a.items_dkv > 0) kkv<<<a.items_dkv, bwd::kThreads, smem_kv, a.stream>>>(mq, mdo, mk, mv, p);
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
  p.kv_heads = kv_heads;
  p.group = group;
  p.pack = pack;
  p.n_steps = n_steps;
  p.scale = scale;
  p.scale_log2 = float(double(scale) * 1.4426950408889634);
  p.timeout_ns = 1000000000ull;   // 1 s: never reached in a correct run
  Launch a{q, k, v, o, dout, heads, kv_heads, n, int(items_dq), int(items_dkv), size_t(heads) * n, workspace,
           static_cast<cudaStream_t>(stream)};
  if (B == 64 && d == 128) return launch_instance<64, 128>(a, p);
  if (B == 64 && d == 64) return launch_instance<64, 64>(a, p);
  if (B == 128 && d == 128) return launch_instance<128, 128>(a, p);
  return launch_instance<128, 64>(a, p);
}
