// Selected-page decode for B200 (sm_100a): one new query token per sequence
// over a key/value cache paged by blocks, reading the block route that the
// layout holds for the token's block row ("BF1: A Causal Dyadic
// Sparse-Attention Retrofit for Efficient Long-Context Transformers",
// section 5, selected-page decode: the route is planned once and reused for
// every token, so a step only gathers its kept pages).
//
// A query row is a single vector, so the step is a stream over the kept
// pages' keys and values (HBM/L2 bound, no matrix product to hand to the
// tensor cores).  One CTA per query row; its 8 warps take the kept blocks in
// turn.  For each block a warp scores its keys (lane l owns keys l, l + 32,
// ..., reading each key row in 16-byte pieces against q held in shared
// memory), folds them into its running max and sum, and accumulates
// P V with lanes across d (each key row read as one coalesced line).  The
// warps' partial (max, sum, o) are then merged in shared memory.  Everything is
// fp32 (P is not rounded to bf16); o is stored as bf16 and lse in fp32.
//
// Positions and page numbers come from device memory: a position outside
// [0, n) or a page outside [0, num_pages) is not read; the kernel records a
// status bit (reported by bsa_get_status) and writes o = 0, lse = -inf for
// that row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <string>

#include "bsa_internal.h"

namespace bsa {
namespace dec {

constexpr int kWarps = 8;
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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int BLK, int HD>
__global__ void __launch_bounds__(kWarps * 32) bsa_decode_kernel(const DecodeParams p) {
  constexpr int KPL = BLK / 32;       // keys per lane in a block
  constexpr int DPL = HD / 32;        // o columns per lane
  __shared__ float sq[HD];
  __shared__ float sm[kWarps], sl[kWarps];
  __shared__ float so[kWarps][HD];
  __shared__ int s_bad;
  const int f = blockIdx.x;
  const int b = f / p.H, h = f - b * p.H;
  const int hk = h / p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float sl2 = p.scale_log2;
  for (int c = threadIdx.x; c < HD; c += blockDim.x) sq[c] = __bfloat162float(p.q[size_t(f) * HD + c]);
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();

  const int t = p.positions[b];
  const bool pos_ok = t >= 0 && t < p.n;
  float m = -INFINITY, l = 0.f;       // this warp's running max (exp2 units) and sum
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  if (pos_ok) {
    const int i = t / BLK;
    const size_t row = size_t(f % p.L) * p.nb + i;
    const int start = p.row_ptr[row], len = p.row_ptr[row + 1] - start;
    for (int e = warp; e < len; e += kWarps) {
      const int j = p.col_idx[start + e];
      const int page = p.page_table[size_t(b) * p.max_blocks + j];
      if (page < 0 || page >= p.num_pages) {
        if (lane == 0) s_bad = 1;
        continue;
      }
      const size_t tile = (size_t(page) * p.hkv + hk) * BLK * HD;
      const __nv_bfloat16* kt = p.kc + tile;
      const __nv_bfloat16* vt = p.vc + tile;
      // scores of this lane's keys
      float s[KPL];
      float bm = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < KPL; ++kk) {
        const int r = lane + 32 * kk;
        const uint4* kr = reinterpret_cast<const uint4*>(kt + size_t(r) * HD);
        float dot = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < HD / 8; ++c8) {
          const uint4 w = __ldg(kr + c8);
          const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 kv = __bfloat1622float2(pr[e]);
            dot = fmaf(kv.x, sq[c8 * 8 + 2 * e], dot);
            dot = fmaf(kv.y, sq[c8 * 8 + 2 * e + 1], dot);
          }
        }
        const bool allowed = j * BLK + r <= t;   // causal; other blocks of the route are earlier
        s[kk] = allowed ? dot * sl2 : -INFINITY;
        bm = fmaxf(bm, s[kk]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      if (bm == -INFINITY) continue;             // nothing allowed in this block
      const float m_new = fmaxf(m, bm);
      const float alpha = ex2(m - m_new);        // 0 when m = -inf
      float psum = 0.f;
#pragma unroll
      for (int kk = 0; kk < KPL; ++kk) {
        s[kk] = ex2(s[kk] - m_new);
        psum += s[kk];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      l = l * alpha + psum;
      m = m_new;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] *= alpha;
      // O += P V: lane owns columns lane * DPL ..
#pragma unroll
      for (int kk = 0; kk < KPL; ++kk) {
#pragma unroll 8
        for (int src = 0; src < 32; ++src) {
          const float pu = __shfl_sync(0xffffffffu, s[kk], src);
          const __nv_bfloat16* vr = vt + size_t(src + 32 * kk) * HD + lane * DPL;
          if constexpr (DPL == 4) {
            const uint2 w = __ldg(reinterpret_cast<const uint2*>(vr));
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
            const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
            acc[0] = fmaf(pu, a.x, acc[0]);
            acc[1] = fmaf(pu, a.y, acc[1]);
            acc[2] = fmaf(pu, c.x, acc[2]);
            acc[3] = fmaf(pu, c.y, acc[3]);
          } else {
            const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(vr));
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
            acc[0] = fmaf(pu, a.x, acc[0]);
            acc[1] = fmaf(pu, a.y, acc[1]);
          }
        }
      }
    }
  } else if (threadIdx.x == 0) {
    s_bad = 1;
  }
  // merge the warps' partial softmax states
  if (lane == 0) {
    sm[warp] = m;
    sl[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) so[warp][lane * DPL + e] = acc[e];
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm[w]);
  float Lsum = 0.f;
  float wgt[kWarps];
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    wgt[w] = (M == -INFINITY) ? 0.f : ex2(sm[w] - M);
    Lsum += wgt[w] * sl[w];
  }
  const bool bad = s_bad != 0;           // a refused index: the whole row is o = 0, lse = -inf
  const float inv = (Lsum > 0.f && !bad) ? 1.f / Lsum : 0.f;
  for (int c = threadIdx.x; c < HD; c += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += wgt[w] * so[w][c];
    p.o[size_t(f) * HD + c] = __float2bfloat16_rn(v * inv);
  }
  if (threadIdx.x == 0) {
    p.lse[f] = (Lsum > 0.f && !bad) ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
    if (bad) atomicOr(p.status, kStatusBadIndex);
  }
}

template <int BLK, int HD>
int launch(const DecodeParams& p, int heads, cudaStream_t s) {
  bsa_decode_kernel<BLK, HD><<<heads, kWarps * 32, 0, s>>>(p);
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
