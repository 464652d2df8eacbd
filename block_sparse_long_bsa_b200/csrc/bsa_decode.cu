// Selected-page decode for B200 (sm_100a): one new query token per sequence
// over a key/value cache paged by blocks, reading the block route that the
// layout holds for the token's block row ("BF1: A Causal Dyadic
// Sparse-Attention Retrofit for Efficient Long-Context Transformers",
// section 5, selected-page decode: the route is planned once and reused for
// every token, so a step only gathers its kept pages).
//
// A query row is a single vector, so the step is a stream over the kept
// pages' keys and values (HBM/L2 bound, no matrix product to hand to the
// tensor cores).  One CTA serves two query rows of a key/value head's group
// when they share a route (one layout head, an even group), else one row, so
// a group's rows read each kept page once.  Its 16 warps take the kept blocks in turn.  For a
// block, 8 lanes cooperate on each key row (16-byte loads, the row read as
// one coalesced line; a 3-step shuffle tree sums the dot product), four rows
// per step, scoring the row against all G queries held in shared memory; the
// scores go through shared memory for the block's max, exponentials and sum
// (an fp32 online softmax per query), and P V is accumulated with lanes across
// d.  The warps' partial (max, sum, o) are then merged in shared memory.
// Everything is fp32 (P is not rounded to bf16); o is stored as bf16 and lse
// in fp32.
//
// Positions and page numbers come from device memory: a position outside
// [0, n) or a page outside [0, num_pages) is not read; the kernel records a
// status bit (reported by bsa_get_status) and writes o = 0, lse = -inf for
// the rows of that CTA.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>
#include <string>

#include "bsa_internal.h"

namespace bsa {
namespace dec {

constexpr int kTileBudget = 192 * 1024;   // shared memory for the warps' K/V tiles
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // a copy that takes longer than 1 s is abandoned
constexpr float kLn2 = 0.693147180559945309f;

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
  float scale_log2;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// One contiguous tile global -> shared by the bulk-copy engine (no multicast),
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

// G query rows per CTA (2 when the rows of a group share a route, else 1).
template <int BLK, int HD>
__host__ __device__ constexpr int warps_for() {   // as many warps as K and V tiles of a page fit the budget, at most 6
  return kTileBudget / (2 * BLK * HD * 2) < 6 ? kTileBudget / (2 * BLK * HD * 2) : 6;
}

template <int BLK, int HD, int G>
__global__ void __launch_bounds__(warps_for<BLK, HD>() * 32) bsa_decode_kernel(const DecodeParams p) {
  constexpr int kWarps = warps_for<BLK, HD>();
  constexpr int CPL = HD / 8;         // key columns per lane (8 lanes per key row)
  constexpr int DPL = HD / 32;        // o columns per lane
  constexpr uint32_t kTile = BLK * HD * 2;   // one page's K (or V) tile of one head
  extern __shared__ __align__(128) uint8_t dyn[];   // per warp: K tile, V tile
  __shared__ __align__(8) uint64_t tile_bar[kWarps];
  __shared__ float sq[G][HD];
  __shared__ float sp[kWarps][G][BLK];          // scores, then P, of a warp's block
  __shared__ float sm[kWarps][G], sl[kWarps][G];
  __shared__ float so[kWarps][G][HD];
  __shared__ int s_bad;
  // the CTA's rows f0 .. f0 + G - 1 (G divides g, so they share a key/value head)
  const int f0 = blockIdx.x * G;
  const int b = f0 / p.H;
  const int hk = (f0 - b * p.H) / p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float sl2 = p.scale_log2;
  for (int c = threadIdx.x; c < G * HD; c += blockDim.x)
    sq[c / HD][c % HD] = __bfloat162float(p.q[size_t(f0) * HD + c]);
  if (threadIdx.x == 0) s_bad = 0;
  if (lane == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&tile_bar[warp])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const uint32_t bar = smem_u32(&tile_bar[warp]);
  const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(dyn + size_t(warp) * 2 * kTile);
  const __nv_bfloat16* vt = kt + BLK * HD;
  int loads = 0;                      // tiles pairs this warp has brought in (barrier phases)

  const int t = p.positions[b];
  const bool pos_ok = t >= 0 && t < p.n;
  float m[G], l[G], acc[G][DPL];
#pragma unroll
  for (int gq = 0; gq < G; ++gq) {
    m[gq] = -INFINITY;
    l[gq] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[gq][e] = 0.f;
  }
  if (pos_ok) {
    const int i = t / BLK;
    const size_t row = size_t(f0 % p.L) * p.nb + i;
    const int start = p.row_ptr[row], len = p.row_ptr[row + 1] - start;
    const int sub = lane >> 3, part = lane & 7;   // key row within a step of 4, column slice
    for (int e = warp; e < len; e += kWarps) {
      const int j = p.col_idx[start + e];
      const int page = p.page_table[size_t(b) * p.max_blocks + j];
      if (page < 0 || page >= p.num_pages) {
        if (lane == 0) s_bad = 1;
        continue;
      }
      const size_t tile = (size_t(page) * p.hkv + hk) * BLK * HD;
      // this block's K and V tiles into the warp's buffers, one bulk copy each
      __syncwarp();                      // every lane is done with the previous tiles
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // earlier reads before the copy
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2 * kTile)
                     : "memory");
        bulk_load(smem_u32(kt), p.kc + tile, kTile, bar);
        bulk_load(smem_u32(vt), p.vc + tile, kTile, bar);
      }
      const bool landed = bar_wait(bar, uint32_t(loads) & 1u);
      ++loads;
      if (!__all_sync(0xffffffffu, landed)) {
        if (lane == 0) s_bad = 2;
        break;
      }
      // ---- scores: rows 4 * step + sub, columns part * CPL ..
#pragma unroll 4
      for (int step = 0; step < BLK / 4; ++step) {
        const int r = step * 4 + sub;
        const uint4* kr = reinterpret_cast<const uint4*>(kt + size_t(r) * HD + part * CPL);
        float dot[G];
#pragma unroll
        for (int gq = 0; gq < G; ++gq) dot[gq] = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < CPL / 8; ++c8) {
          const uint4 w = kr[c8];
          const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 kv = __bfloat1622float2(pr[e2]);
            const int c = part * CPL + c8 * 8 + 2 * e2;
#pragma unroll
            for (int gq = 0; gq < G; ++gq) {
              dot[gq] = fmaf(kv.x, sq[gq][c], dot[gq]);
              dot[gq] = fmaf(kv.y, sq[gq][c + 1], dot[gq]);
            }
          }
        }
#pragma unroll
        for (int gq = 0; gq < G; ++gq) {
          dot[gq] += __shfl_xor_sync(0xffffffffu, dot[gq], 1);
          dot[gq] += __shfl_xor_sync(0xffffffffu, dot[gq], 2);
          dot[gq] += __shfl_xor_sync(0xffffffffu, dot[gq], 4);
        }
        if (part == 0) {
          const bool allowed = j * BLK + r <= t;   // causal; other blocks of the route are earlier
#pragma unroll
          for (int gq = 0; gq < G; ++gq) sp[warp][gq][r] = allowed ? dot[gq] * sl2 : -INFINITY;
        }
      }
      __syncwarp();
      // ---- online softmax per query over this block's keys
      float alpha[G];
      bool any = false;
#pragma unroll
      for (int gq = 0; gq < G; ++gq) {
        float bm = -INFINITY;
#pragma unroll
        for (int r = lane; r < BLK; r += 32) bm = fmaxf(bm, sp[warp][gq][r]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
        const float m_new = fmaxf(m[gq], bm);
        alpha[gq] = (m_new == -INFINITY) ? 1.f : ex2(m[gq] - m_new);   // 0 when m was -inf
        float psum = 0.f;
#pragma unroll
        for (int r = lane; r < BLK; r += 32) {
          const float pv = (m_new == -INFINITY) ? 0.f : ex2(sp[warp][gq][r] - m_new);
          sp[warp][gq][r] = pv;
          psum += pv;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l[gq] = l[gq] * alpha[gq] + psum;
        m[gq] = m_new;
        any = any || bm != -INFINITY;
      }
      __syncwarp();
      if (!any) continue;                        // nothing allowed in this block
      // ---- O += P V: lane owns columns lane * DPL ..
#pragma unroll
      for (int gq = 0; gq < G; ++gq)
#pragma unroll
        for (int e2 = 0; e2 < DPL; ++e2) acc[gq][e2] *= alpha[gq];
#pragma unroll 8
      for (int r = 0; r < BLK; ++r) {
        const __nv_bfloat16* vr = vt + size_t(r) * HD + lane * DPL;
        float vv[DPL];
        if constexpr (DPL == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(vr);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
          const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
          vv[0] = a.x;
          vv[1] = a.y;
          vv[2] = c.x;
          vv[3] = c.y;
        } else {
          const uint32_t w = *reinterpret_cast<const unsigned int*>(vr);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
          vv[0] = a.x;
          vv[1] = a.y;
        }
#pragma unroll
        for (int gq = 0; gq < G; ++gq) {
          const float pu = sp[warp][gq][r];
#pragma unroll
          for (int e2 = 0; e2 < DPL; ++e2) acc[gq][e2] = fmaf(pu, vv[e2], acc[gq][e2]);
        }
      }
      __syncwarp();
    }
  } else if (threadIdx.x == 0) {
    s_bad = 1;
  }
  // merge the warps' partial softmax states
#pragma unroll
  for (int gq = 0; gq < G; ++gq) {
    if (lane == 0) {
      sm[warp][gq] = m[gq];
      sl[warp][gq] = l[gq];
    }
#pragma unroll
    for (int e2 = 0; e2 < DPL; ++e2) so[warp][gq][lane * DPL + e2] = acc[gq][e2];
  }
  __syncthreads();
  // a refused index (or a copy that never landed): the CTA's rows are o = 0,
  // lse = -inf.  Leave no copy in flight into shared memory.
  if (lane == 0 && loads > 0) bar_wait(bar, uint32_t(loads - 1) & 1u);
  __syncwarp();
  const bool bad = s_bad != 0;
  for (int c = threadIdx.x; c < G * HD; c += blockDim.x) {
    const int gq = c / HD, col = c % HD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm[w][gq]);
    float Lsum = 0.f, v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float wt = (M == -INFINITY) ? 0.f : ex2(sm[w][gq] - M);
      Lsum += wt * sl[w][gq];
      v += wt * so[w][gq][col];
    }
    const bool ok = Lsum > 0.f && !bad;
    p.o[size_t(f0 + gq) * HD + col] = __float2bfloat16_rn(ok ? v / Lsum : 0.f);
    if (col == 0) p.lse[f0 + gq] = ok ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
  }
  if (threadIdx.x == 0 && bad) atomicOr(p.status, s_bad == 2 ? kStatusTimeout : kStatusBadIndex);
}

template <int BLK, int HD, int G>
int launch_g(const DecodeParams& p, int heads, cudaStream_t s) {
  auto kern = bsa_decode_kernel<BLK, HD, G>;
  constexpr int kWarps = warps_for<BLK, HD>();
  const int smem = kWarps * 2 * BLK * HD * 2;
  // the attribute is a property of the function: set it once per device
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return set_error(BSA_ERR_CUDA, "cannot query the device");
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("decode smem: ") + cudaGetErrorString(e));
      done[dev] = true;
    }
  }
  kern<<<heads / G, kWarps * 32, smem, s>>>(p);
  return BSA_OK;
}

template <int BLK, int HD>
int launch(const DecodeParams& p, int heads, cudaStream_t s) {
  // two query rows of a key/value head's group per CTA when they share a route
  const int st = (p.L == 1 && p.g % 2 == 0) ? launch_g<BLK, HD, 2>(p, heads, s) : launch_g<BLK, HD, 1>(p, heads, s);
  if (st != BSA_OK) return st;
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
  return BSA_OK;
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
  if (B == 64 && d == 128) return dec::launch<64, 128>(p, heads, s);
  if (B == 64 && d == 64) return dec::launch<64, 64>(p, heads, s);
  if (B == 128 && d == 128) return dec::launch<128, 128>(p, heads, s);
  return dec::launch<128, 64>(p, heads, s);
}
