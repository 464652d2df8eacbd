// bsa_forward_noalloc: the forward pass for callers that cannot allocate
// device memory.
//
// Who needs it: a process whose device memory is owned by someone else -- for
// example a serving framework that reserved the GPU's memory in its own pool
// at start-up, or a host application that lends this library only the buffers
// it passes in -- and code that must not allocate once it is running, because
// cudaMalloc/cudaFree can synchronise the whole device and stall other work.
// bsa_build_layout with a device index allocates the layout's device arrays, so
// such a caller builds the layout host-only (device = -1) and calls this entry
// point, which needs no allocation at all: the layout arrays and the kernel's
// status word are staged in one fixed block of device memory that this
// library declares statically (it exists on every GPU that loads the library,
// for as long as the process lives).
//
// Because every call uses that same block, calls that overlap on the GPU (on
// different streams, or from several host threads without ordering) race with
// each other; each call overwrites what the previous one left there.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "bsa_internal.h"

namespace {

// Layout of the static scratch, in 32-bit words: word 0 is the kernel's status
// word (cleared at every call; bsa_get_status with a host-only layout reads
// it), words 32 and 33 the kernel's work counter (left at zero by every
// launch); words from kLayoutBase on (256 bytes in, so 16-byte aligned) hold
// the layout's work table (four words per query block, longest row first)
// and then col_idx.
constexpr size_t kScratchWords = (size_t(4) << 20) / 4 + 64;   // 4 MiB of layout + 256 B head
constexpr size_t kLayoutBase = 64;
constexpr size_t kLayoutWordsMax = kScratchWords - kLayoutBase;

static __device__ __align__(256) uint32_t g_noalloc_scratch[kScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
uint32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device.  The symbol's
// name in host code is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached for the life of the
// process; after a cudaDeviceReset of that device the cached address is stale,
// so this entry point must not be used on a device once it has been reset.
int scratch_on_current_device(uint32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return bsa::set_error(BSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return bsa::set_error(BSA_ERR_INVALID_ARG, "device index out of range");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return bsa::set_error(BSA_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") +
                                              cudaGetErrorString(e));
    g_scratch_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return BSA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

namespace bsa {
int noalloc_status_word(uint32_t** out) { return scratch_on_current_device(out); }
}  // namespace bsa

extern "C" int bsa_forward_noalloc(const void* q, const void* k, const void* v,
                                   const bsa_layout* layout, int B, int n, int heads, int kv_heads,
                                   int d, float scale, void* o, float* lse, void* stream) {
  using bsa::set_error;
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (B != layout->B || n != layout->n) return set_error(BSA_ERR_SHAPE, "B/n differ from the layout's");
  if (B != 64 && B != 128) return set_error(BSA_ERR_UNSUPPORTED, "B must be 64 or 128");
  if (d != 64 && d != 128) return set_error(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (heads < 1 || kv_heads < 1) return set_error(BSA_ERR_SHAPE, "heads and kv_heads must be >= 1");
  if (heads % kv_heads) return set_error(BSA_ERR_SHAPE, "heads must be a multiple of kv_heads");
  if (heads % layout->L) return set_error(BSA_ERR_SHAPE, "heads must be a multiple of layout_heads");
  if (!(scale > 0.f && scale < 3.0e38f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!q || !k || !v || !o || !lse) return set_error(BSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return set_error(BSA_ERR_INVALID_ARG, "q, k, v and o must be 16-byte aligned");
  if (!aligned(lse, 4)) return set_error(BSA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  const size_t words = layout->work.size() + layout->col_idx.size();
  if (words > kLayoutWordsMax)
    return set_error(BSA_ERR_SHAPE, "layout needs " + std::to_string(words) +
                                        " words of device scratch; the static scratch of this entry "
                                        "point holds " + std::to_string(kLayoutWordsMax) +
                                        " (4 MiB): use bsa_forward with a device layout instead");
  if (int64_t(heads) * layout->nb > INT32_MAX) return set_error(BSA_ERR_SHAPE, "too many work items");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The layout is copied from the caller's host vectors while the call runs; a
  // graph captured around that copy would read them again at every replay,
  // after they may have been freed, so a capturing stream is refused.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t ce = cudaStreamIsCapturing(s, &cap);
  if (ce != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaStreamIsCapturing: ") + cudaGetErrorString(ce));
  if (cap != cudaStreamCaptureStatusNone)
    return set_error(BSA_ERR_UNSUPPORTED,
                     "bsa_forward_noalloc copies the layout from host memory at every call and is refused "
                     "on a capturing stream; capture bsa_forward with a device layout instead");
  uint32_t* scratch = nullptr;
  int st = scratch_on_current_device(&scratch);
  if (st != BSA_OK) return st;
  int32_t* d_work = reinterpret_cast<int32_t*>(scratch + kLayoutBase);
  int32_t* d_col_idx = d_work + layout->work.size();
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s);   // status word starts at zero
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(d_work, layout->work.data(), layout->work.size() * sizeof(int32_t),
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !layout->col_idx.empty())
    e = cudaMemcpyAsync(d_col_idx, layout->col_idx.data(), layout->col_idx.size() * sizeof(int32_t),
                        cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("staging the layout: ") + cudaGetErrorString(e));
  bsa::ForwardArgs a{q, k, v, o, lse, layout, B, n, heads, kv_heads, d, scale, stream, 0, 0};
  return bsa::launch_forward_with(a, d_work, d_col_idx, scratch);
}
