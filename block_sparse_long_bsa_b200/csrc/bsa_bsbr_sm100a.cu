// BSBR's between-chunk retrieval term for B200 (sm_100a) ("bsbr",
// jvboid.dev/projects/bsbr, section "Solution"): each chunk of B tokens is
// compressed into the state F_c = K_c^T V_c; chunk c retrieves from the
// states of the chunks before it with softmax weights of its meta query
// against their meta keys (R_c, H_c: means of q and k over a chunk), and its
// tokens read the retrieved d x d state with their queries.  The result is
// added to the within-chunk attention output (the block-diagonal layout of
// the forward) already in o.
//
// Two launches: the state kernel (one CTA per key/value head and chunk:
// F_c by one tcgen05 product, H_c by column sums) and the retrieval kernel
// (one CTA per query head and chunk >= 1: meta weights, the weighted sum of
// earlier states in fp32, and o += Q_c S_c by tcgen05 products with S split
// into bf16 hi + lo parts).  The work is small and bound by memory traffic
// and latency; the products go to the tensor cores so no fp32 ALU loop over
// B x d x d sits on the path.  Every mbarrier wait is bounded (the layout's
// status word records a wait that ran out).
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
namespace bsbr {

using namespace ptx;


constexpr uint64_t kDrainNs = 200000000ull;


struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __nv_bfloat16* o;
  float* F;        // [kv_heads][chunks][d][d]
  float* H;        // [kv_heads][chunks][d]
  uint32_t* status;
  int n, chunks, heads, kv_heads, group;
  float scale;
  uint64_t timeout_ns;
};

// ---------------------------------------------------------------- chunk states
// One CTA per (key/value head g, chunk c): F_c = K_c^T V_c as one tcgen05
// product with M along d (A = the K tile read along d, B = the V tile read
// along d, the reduction over the chunk's tokens; for d = 64 the upper 64
// rows of M read the neighbouring tile and are never stored), and H_c = the
// mean of k over the chunk's tokens.  Tokens past n are zero-filled by the
// tensor map and left out of the mean.
template <int BLK, int HD>
struct StateShape {
  static constexpr int kBox = 64 * HD * 2;                // one 64-token box: [atom][64 rows][64 columns]
  static constexpr int kTile = BLK * HD * 2;
  static constexpr int kOffV = kTile;
  static constexpr int kOffBar = 2 * kTile;
  static constexpr int kOffMisc = kOffBar + 16;
  static constexpr int kOffRed = kOffMisc + 16;            // [128] partial column sums
  static constexpr int kSmem = kOffRed + 128 * 4;
  static constexpr uint32_t kIdesc = idesc_bf16(128, HD, 1, 1);
};

// Element (row t, column x) of a bf16 tile landed by the tensor maps as
// [64-row box][64-column atom][row][128-byte swizzled line].
template <int HD>
__device__ __forceinline__ float tile_elem(const uint8_t* tile, int rows_per_box, int t, int x) {
  const int box = t / rows_per_box, row = t - box * rows_per_box;
  const int off = box * rows_per_box * HD * 2 + (x >> 6) * rows_per_box * 128 + row * 128 +
                  ((((x & 63) >> 3) ^ (row & 7)) << 4) + (x & 7) * 2;
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + off));
}

// Column means of the first `count` rows of a tile in shared memory, by all
// threads of the block (blockDim.x a multiple of HD); out[x] for x < HD.
template <int HD>
__device__ __forceinline__ void tile_column_means(const uint8_t* tile, int rows_per_box, int count, float* part,
                                                  float* out) {
  const int groups = int(blockDim.x) / HD;
  const int x = threadIdx.x % HD, gr = threadIdx.x / HD;
  float acc = 0.f;
  for (int t = gr; t < count; t += groups) acc += tile_elem<HD>(tile, rows_per_box, t, x);
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < HD) {
    float sum = 0.f;
    for (int k = 0; k < groups; ++k) sum += part[k * HD + threadIdx.x];
    out[threadIdx.x] = sum / float(count);
  }
}

template <int BLK, int HD>
__global__ void __launch_bounds__(128) bsbr_state_kernel(const __grid_constant__ CUtensorMap tmK,
                                                         const __grid_constant__ CUtensorMap tmV, const Params p) {
  using S = StateShape<BLK, HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  const int g = blockIdx.x / p.chunks, c = blockIdx.x - g * p.chunks;
  const uint32_t sK = base, sV = base + S::kOffV;
  const uint32_t bLoad = base + S::kOffBar, bDone = bLoad + 8;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem_raw + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + S::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};
  const int t0 = c * BLK;
  const int count = min(BLK, p.n - t0);

  if (threadIdx.x == 0) {
    mbar_init(bLoad, 1);
    mbar_init(bDone, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(base + S::kOffMisc, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (threadIdx.x == 0) {
    mbar_expect_tx(bLoad, 2 * S::kTile);
#pragma unroll
    for (int b = 0; b < BLK / 64; ++b) {
      tma_load_kv<HD>(sK + b * S::kBox, &tmK, bLoad, t0 + b * 64, g);
      tma_load_kv<HD>(sV + b * S::kBox, &tmV, bLoad, t0 + b * 64, g);
    }
  }
  const bool loaded = __syncthreads_and(ctl.wait(bLoad, 0));
  if (threadIdx.x == 0) {
    if (loaded) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BLK / 16; ++kk) {
        const uint32_t off = (kk >> 2) * S::kBox + (kk & 3) * 2048;
        mma_ss(tmem, sw128_desc(sK + off, 8192, 1024), sw128_desc(sV + off, 8192, 1024), S::kIdesc, kk > 0);
      }
    } else {
      wait_drain(bLoad, 0, kDrainNs);
    }
    tc_commit(bDone);
  }
  // H_c: column means of the K tile
  if (loaded)
    tile_column_means<HD>(smem_raw, 64, count, reinterpret_cast<float*>(smem_raw + S::kOffRed),
                          p.H + (size_t(g) * p.chunks + c) * HD);
  // F_c: TMEM lane r holds row r (element r of d) of K_c^T V_c
  const bool ok = __all_sync(0xffffffffu, ctl.wait(bDone, 0));
  const int r = warp * 32 + lane;
  if (ok && !*abort_flag) {
    tc_fence_after();
    float* out = p.F + ((size_t(g) * p.chunks + c) * HD + (r < HD ? r : 0)) * HD;
#pragma unroll
    for (int a = 0; a < HD / 32; ++a) {
      float v[32];
      tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + a * 32, v);
      tmem_wait_ld();
      if (r < HD) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(out + a * 32 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------- retrieval
// One CTA per (query head f, chunk c >= 1): R_c = mean of q over the chunk;
// a_c' = scale <R_c, H_c'> and A = softmax over c' < c; S_c = sum A_c' F_c'
// in fp32, split into bf16 hi + lo parts (S = hi + lo to 2^-16); then
// o_t += q_t S_c for the chunk's tokens as two tcgen05 products
// (M = 128 tile rows, A = the Q tile, B = S read along d), added to the
// within-chunk output already in o.  For B = 64 the tile's upper 64 rows are
// the next chunk's queries and are never stored.
template <int BLK, int HD>
struct RetrShape {
  static constexpr int kQBytes = 128 * HD * 2;
  static constexpr int kAtomQ = 128 * 128;
  static constexpr int kSBytes = HD * HD * 2;             // one bf16 S part: [atom][HD rows][64 columns]
  static constexpr int kAtomS = HD * 128;
  static constexpr int kOffS = kQBytes;                   // hi, then lo
  static constexpr int kOffR = kOffS + 2 * kSBytes;       // R_c [HD] fp32
  static constexpr int kOffRed = kOffR + HD * 4;          // block reduction scratch [8]
  static constexpr int kOffPart = kOffRed + 64;           // [256] partial column sums
  static constexpr int kOffBar = kOffPart + 256 * 4;
  static constexpr int kOffMisc = kOffBar + 16;
  static constexpr int kOffA = kOffMisc + 16;             // meta weights [chunks] fp32
  static constexpr uint32_t kIdesc = idesc_bf16(128, HD, 0, 1);
};

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < int(blockDim.x >> 5); ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

template <int BLK, int HD>
__global__ void __launch_bounds__(256) bsbr_retrieve_kernel(const __grid_constant__ CUtensorMap tmQ, const Params p) {
  using S = RetrShape<BLK, HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_addr(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
    return;
  }
  const int per_head = p.chunks - 1;
  const int f = blockIdx.x / per_head, c = blockIdx.x - f * per_head + 1;
  const int g = f / p.group;
  const int t0 = c * BLK;
  const int count = min(BLK, p.n - t0);
  const uint32_t sQ = base, sS = base + S::kOffS;
  float* R = reinterpret_cast<float*>(smem_raw + S::kOffR);
  float* red = reinterpret_cast<float*>(smem_raw + S::kOffRed);
  float* A = reinterpret_cast<float*>(smem_raw + S::kOffA);
  const uint32_t bLoad = base + S::kOffBar, bDone = bLoad + 8;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem_raw + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + S::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(bLoad, 1);
    mbar_init(bDone, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(base + S::kOffMisc, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (threadIdx.x == 0) {
    mbar_expect_tx(bLoad, S::kQBytes);
    tma_load_q<128, HD>(sQ, &tmQ, bLoad, t0, f);
  }
  // R_c: column means of the Q tile (one 128-row box)
  const bool loaded = __syncthreads_and(ctl.wait(bLoad, 0));
  if (loaded) tile_column_means<HD>(smem_raw, 128, count, reinterpret_cast<float*>(smem_raw + S::kOffPart), R);
  __syncthreads();
  // meta scores of the earlier chunks, one warp per chunk, four chunks' loads in flight
  const float* Hg = p.H + size_t(g) * p.chunks * HD;
  for (int cp0 = warp; cp0 < c; cp0 += 32) {
    float sc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cp = cp0 + 8 * u;
      float s = 0.f;
      if (cp < c) {
#pragma unroll
        for (int x = lane; x < HD; x += 32) s = fmaf(R[x], Hg[size_t(cp) * HD + x], s);
      }
      sc[u] = s;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], off);
      if (lane == 0 && cp0 + 8 * u < c) A[cp0 + 8 * u] = sc[u] * p.scale;
    }
  }
  __syncthreads();
  float m = -INFINITY;
  for (int cp = threadIdx.x; cp < c; cp += blockDim.x) m = fmaxf(m, A[cp]);
  m = block_reduce(m, red, true);
  float z = 0.f;
  for (int cp = threadIdx.x; cp < c; cp += blockDim.x) {
    const float e = __expf(A[cp] - m);
    A[cp] = e;
    z += e;
  }
  z = block_reduce(z, red, false);   // its barriers also publish A
  const float inv = 1.f / z;
  // S_c: thread owns float4 columns j4 of rows r = threadIdx.x / (HD/4) + k * (256 / (HD/4))
  constexpr int kV4 = HD / 4;                 // float4 per row
  constexpr int kRowsPerPass = 256 / kV4;
  constexpr int kPasses = HD / kRowsPerPass;
  const int j4 = threadIdx.x % kV4, r0 = threadIdx.x / kV4;
  float4 acc[kPasses];
#pragma unroll
  for (int k = 0; k < kPasses; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* Fg = p.F + size_t(g) * p.chunks * HD * HD;
  // U earlier states per step, their loads issued together
  constexpr int U = HD == 64 ? 4 : 2;
  for (int cp0 = 0; cp0 < c; cp0 += U) {
    float4 x[U][kPasses];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int cp = cp0 + u < c ? cp0 + u : c - 1;
      const float4* src = reinterpret_cast<const float4*>(Fg + size_t(cp) * HD * HD);
#pragma unroll
      for (int k = 0; k < kPasses; ++k) x[u][k] = src[(r0 + k * kRowsPerPass) * kV4 + j4];
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float w = cp0 + u < c ? A[cp0 + u] * inv : 0.f;
#pragma unroll
      for (int k = 0; k < kPasses; ++k) {
        acc[k].x = fmaf(w, x[u][k].x, acc[k].x);
        acc[k].y = fmaf(w, x[u][k].y, acc[k].y);
        acc[k].z = fmaf(w, x[u][k].z, acc[k].z);
        acc[k].w = fmaf(w, x[u][k].w, acc[k].w);
      }
    }
  }
  // S as bf16 hi and lo, [K = d rows][N = d columns] in 64-column swizzled atoms
#pragma unroll
  for (int k = 0; k < kPasses; ++k) {
    const int row = r0 + k * kRowsPerPass, col = j4 * 4;
    const uint32_t off = uint32_t(col >> 6) * S::kAtomS + uint32_t(row) * 128 +
                         ((uint32_t(((col & 63) >> 3) ^ (row & 7))) << 4) + uint32_t(col & 7) * 2;
    const float vals[4] = {acc[k].x, acc[k].y, acc[k].z, acc[k].w};
    float lo[4];
    __nv_bfloat16 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      h[e] = __float2bfloat16_rn(vals[e]);
      lo[e] = vals[e] - __bfloat162float(h[e]);
    }
    const uint32_t hi01 = uint32_t(__bfloat16_as_ushort(h[0])) | (uint32_t(__bfloat16_as_ushort(h[1])) << 16);
    const uint32_t hi23 = uint32_t(__bfloat16_as_ushort(h[2])) | (uint32_t(__bfloat16_as_ushort(h[3])) << 16);
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sS + off), "r"(hi01), "r"(hi23) : "memory");
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sS + S::kSBytes + off), "r"(pack_bf16(lo[0], lo[1])),
                 "r"(pack_bf16(lo[2], lo[3]))
                 : "memory");
  }
  fence_proxy_async();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (loaded) {
      tc_fence_after();
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * S::kAtomQ + (kk & 3) * 32;
          mma_ss(tmem, sw128_desc(sQ + ao, 16, 1024),
                 sw128_desc(sS + part * S::kSBytes + kk * 16 * 128, S::kAtomS, 1024), S::kIdesc,
                 (part > 0 || kk > 0) ? 1u : 0u);
        }
    } else {
      wait_drain(bLoad, 0, kDrainNs);
    }
    tc_commit(bDone);
  }
  if (warp < 4) {
    const bool ok = __all_sync(0xffffffffu, ctl.wait(bDone, 0));
    const int r = warp * 32 + lane;
    if (ok && !*abort_flag) {
      tc_fence_after();
      __nv_bfloat16* op = p.o + (size_t(f) * p.n + t0 + r) * HD;
      const bool mine = r < count;
#pragma unroll
      for (int a = 0; a < HD / 32; ++a) {
        float v[32];
        tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + a * 32, v);
        tmem_wait_ld();
        if (mine) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w = *reinterpret_cast<const uint4*>(op + a * 32 + e);
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wp[h]));
              wp[h] = pack_bf16(x.x + v[e + 2 * h], x.y + v[e + 2 * h + 1]);
            }
            *reinterpret_cast<uint4*>(op + a * 32 + e) = w;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}
}  // namespace bsbr

namespace {

using namespace tmap;

template <typename K>
int prepare(K kern, int smem, int slot) {
  static std::mutex mu;
  static int done[64][8] = {};
  int dev_id = 0;
  cudaError_t e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess || dev_id < 0 || dev_id >= 64) return set_error(BSA_ERR_CUDA, "cannot query the device");
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev_id][slot] < smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    done[dev_id][slot] = smem;
  }
  return BSA_OK;
}

template <int BLK, int HD>
int launch_instance(const void* q, const void* k, const void* v, const bsbr::Params& p, cudaStream_t stream) {
  using SS = bsbr::StateShape<BLK, HD>;
  using SR = bsbr::RetrShape<BLK, HD>;
  constexpr int slot = (BLK == 128 ? 2 : 0) + (HD == 128 ? 1 : 0);
  auto ks = bsbr::bsbr_state_kernel<BLK, HD>;
  auto kr = bsbr::bsbr_retrieve_kernel<BLK, HD>;
  // no more than four CTAs per SM, so each one's 128 TMEM columns are free at once
  const int floor_bytes = 46 * 1024;
  const int smem_s = SS::kSmem > floor_bytes ? SS::kSmem : floor_bytes;
  const int need_r = SR::kOffA + 4 * p.chunks;
  const int smem_r = need_r > floor_bytes ? need_r : floor_bytes;
  if (smem_r > 227 * 1024) return set_error(BSA_ERR_SHAPE, "too many chunks for the retrieval kernel's weights");
  int st = prepare(ks, smem_s, slot);
  if (st == BSA_OK) st = prepare(kr, smem_r, 4 + slot);
  if (st != BSA_OK) return st;
  CUtensorMap mq, mk, mv;
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  st = encode_rows(&mq, q, p.heads, p.n, HD, 128);
  if (st == BSA_OK) st = encode_rows(&mk, k, p.kv_heads, p.n, HD, 64);
  if (st == BSA_OK) st = encode_rows(&mv, v, p.kv_heads, p.n, HD, 64);
  if (st != BSA_OK) return st;
  ks<<<p.kv_heads * p.chunks, 128, smem_s, stream>>>(mk, mv, p);
  kr<<<p.heads * (p.chunks - 1), 256, smem_r, stream>>>(mq, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" size_t bsa_bsbr_workspace_bytes(int n, int B, int kv_heads, int d) {
  if (n < 1 || B < 1 || kv_heads < 1 || d < 1) return 0;
  const size_t chunks = size_t((int64_t(n) + B - 1) / B);
  return size_t(kv_heads) * chunks * size_t(d) * size_t(d + 1) * sizeof(float);
}

extern "C" int bsa_bsbr_retrieval(const void* q, const void* k, const void* v, const bsa_layout* layout, int B,
                                  int n, int heads, int kv_heads, int d, float scale, void* o, void* workspace,
                                  size_t workspace_bytes, void* stream) {
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
  if (!(std::isfinite(scale) && scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!q || !k || !v || !o || !workspace) return set_error(BSA_ERR_INVALID_ARG, "null pointer");
  auto aligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; };
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(workspace, 16))
    return set_error(BSA_ERR_INVALID_ARG, "q, k, v, o and workspace must be 16-byte aligned");
  if (workspace_bytes < bsa_bsbr_workspace_bytes(n, B, kv_heads, d))
    return set_error(BSA_ERR_SHAPE, "workspace smaller than bsa_bsbr_workspace_bytes");
  const int64_t chunks = (int64_t(n) + B - 1) / B;
  if (int64_t(heads) * chunks > INT32_MAX) return set_error(BSA_ERR_SHAPE, "too many (head, chunk) items");
  if (chunks < 2) return BSA_OK;   // one chunk: nothing to retrieve
  int st = get_encoder();
  if (st != BSA_OK) return st;
  bsbr::Params p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.F = static_cast<float*>(workspace);
  p.H = p.F + size_t(kv_heads) * size_t(chunks) * d * d;
  p.status = layout->d_status;
  p.n = n;
  p.chunks = int(chunks);
  p.heads = heads;
  p.kv_heads = kv_heads;
  p.group = heads / kv_heads;
  p.scale = scale;
  p.timeout_ns = 1000000000ull;   // 1 s: never reached in a correct run
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 64 && d == 128) return launch_instance<64, 128>(q, k, v, p, s);
  if (B == 64 && d == 64) return launch_instance<64, 64>(q, k, v, p, s);
  if (B == 128 && d == 128) return launch_instance<128, 128>(q, k, v, p, s);
  return launch_instance<128, 64>(q, k, v, p, s);
}
