// C ABI entry points: argument validation, layout ownership, device upload and
// status reporting.  The arithmetic runs in the sm_100a kernel
// (bsa_fwd_sm100a.cu); nothing here computes attention.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <new>
#include <string>

#include "bsa_internal.h"

namespace {
thread_local std::string g_last_error;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
}  // namespace

namespace bsa {
int set_error(int status, const std::string& msg) {
  g_last_error = msg;
  return status;
}
}  // namespace bsa

using bsa::set_error;

extern "C" {

const char* bsa_last_error(void) { return g_last_error.c_str(); }

int bsa_build_layout(const bsa_pattern* spec, int n, int B, int layout_heads, int device,
                     bsa_layout** out) {
  if (!out) return set_error(BSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!spec) return set_error(BSA_ERR_INVALID_ARG, "spec is NULL");
  if (n < 1) return set_error(BSA_ERR_SHAPE, "n must be >= 1");
  if (B < 1) return set_error(BSA_ERR_SHAPE, "B must be >= 1");
  if (layout_heads < 1) return set_error(BSA_ERR_SHAPE, "layout_heads must be >= 1");
  if (device < -1) return set_error(BSA_ERR_INVALID_ARG, "device must be -1 or a device index");
  const int64_t nb = (int64_t(n) + B - 1) / B;
  if (int64_t(layout_heads) * nb + 1 > INT32_MAX)
    return set_error(BSA_ERR_SHAPE, "layout_heads * blocks exceeds 2^31-1 rows");
  switch (spec->kind) {
    case BSA_PATTERN_BAND_GLOBAL:
    case BSA_PATTERN_DYADIC:
      if (spec->window < 0) return set_error(BSA_ERR_INVALID_ARG, "window must be >= 0");
      if (spec->kind == BSA_PATTERN_DYADIC && spec->dyadic_kmin < 0)
        return set_error(BSA_ERR_INVALID_ARG, "dyadic_kmin must be >= 0");
      break;
    case BSA_PATTERN_RANDOM:
      if (!(spec->density >= 0.0 && spec->density <= 1.0))
        return set_error(BSA_ERR_INVALID_ARG, "density must lie in [0, 1]");
      break;
    case BSA_PATTERN_EXPLICIT:
      if (!spec->mask) return set_error(BSA_ERR_INVALID_ARG, "explicit pattern needs a mask");
      if (nb > 65536) return set_error(BSA_ERR_SHAPE, "explicit masks are limited to 65536 blocks");
      break;
    default:
      return set_error(BSA_ERR_INVALID_ARG, "unknown pattern kind");
  }

  bsa_layout* lay = new (std::nothrow) bsa_layout();
  if (!lay) return set_error(BSA_ERR_OOM, "host allocation failed");
  int st;
  try {
    st = bsa::compile_layout(*spec, n, B, layout_heads, lay);
  } catch (const std::bad_alloc&) {
    st = set_error(BSA_ERR_OOM, "host allocation failed while compiling the layout");
  }
  if (st != BSA_OK) {
    delete lay;
    return st;
  }

  if (device >= 0) {
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    cudaError_t e = cudaSetDevice(device);
    if (e != cudaSuccess) {
      delete lay;
      return set_error(BSA_ERR_CUDA, std::string("cudaSetDevice: ") + cudaGetErrorString(e));
    }
    const size_t b_rp = lay->row_ptr.size() * sizeof(int32_t);
    const size_t b_ci = std::max<size_t>(1, lay->col_idx.size()) * sizeof(int32_t);
    const size_t b_or = lay->order.size() * sizeof(int32_t);
    const size_t o_ci = round_up(b_rp, 256), o_or = o_ci + round_up(b_ci, 256);
    const size_t b_cp = lay->col_ptr.size() * sizeof(int32_t);
    const size_t b_ri = std::max<size_t>(1, lay->row_idx.size()) * sizeof(int32_t);
    const size_t o_cp = o_or + round_up(b_or, 256), o_ri = o_cp + round_up(b_cp, 256);
    const size_t b_sp = lay->seg_ptr.size() * sizeof(int32_t);
    const size_t b_sg = std::max<size_t>(1, lay->segs.size()) * sizeof(int32_t);
    const size_t o_sp = o_ri + round_up(b_ri, 256), o_sg = o_sp + round_up(b_sp, 256);
    const size_t o_st = o_sg + round_up(b_sg, 256), total = o_st + bsa::kStatusBlockBytes;
    void* base = nullptr;
    e = cudaMalloc(&base, total);
    if (e != cudaSuccess) {
      delete lay;
      if (prev >= 0) cudaSetDevice(prev);
      cudaGetLastError();
      return set_error(e == cudaErrorMemoryAllocation ? BSA_ERR_OOM : BSA_ERR_CUDA,
                       std::string("cudaMalloc: ") + cudaGetErrorString(e));
    }
    char* c = static_cast<char*>(base);
    e = cudaMemcpy(c, lay->row_ptr.data(), b_rp, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !lay->col_idx.empty())
      e = cudaMemcpy(c + o_ci, lay->col_idx.data(), lay->col_idx.size() * sizeof(int32_t),
                     cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(c + o_or, lay->order.data(), b_or, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(c + o_cp, lay->col_ptr.data(), b_cp, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !lay->row_idx.empty())
      e = cudaMemcpy(c + o_ri, lay->row_idx.data(), lay->row_idx.size() * sizeof(int32_t),
                     cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(c + o_sp, lay->seg_ptr.data(), b_sp, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !lay->segs.empty())
      e = cudaMemcpy(c + o_sg, lay->segs.data(), lay->segs.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(c + o_st, 0, bsa::kStatusBlockBytes);
    if (e != cudaSuccess) {
      cudaFree(base);
      delete lay;
      if (prev >= 0) cudaSetDevice(prev);
      return set_error(BSA_ERR_CUDA, std::string("layout upload: ") + cudaGetErrorString(e));
    }
    lay->d_base = base;
    lay->d_row_ptr = reinterpret_cast<const int32_t*>(c);
    lay->d_col_idx = reinterpret_cast<const int32_t*>(c + o_ci);
    lay->d_order = reinterpret_cast<const int32_t*>(c + o_or);
    lay->d_col_ptr = reinterpret_cast<const int32_t*>(c + o_cp);
    lay->d_row_idx = reinterpret_cast<const int32_t*>(c + o_ri);
    lay->d_seg_ptr = reinterpret_cast<const int32_t*>(c + o_sp);
    lay->d_segs = reinterpret_cast<const int32_t*>(c + o_sg);
    lay->d_status = reinterpret_cast<uint32_t*>(c + o_st);
    lay->device = device;
    if (prev >= 0 && prev != device) cudaSetDevice(prev);
  }
  *out = lay;
  return BSA_OK;
}

int bsa_layout_csr(const bsa_layout* layout, const int32_t** row_ptr, const int32_t** col_idx,
                   int* rows, int* nnz) {
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (row_ptr) *row_ptr = layout->row_ptr.data();
  if (col_idx) *col_idx = layout->col_idx.data();
  if (rows) *rows = int(layout->row_ptr.size()) - 1;
  if (nnz) *nnz = int(layout->col_idx.size());
  return BSA_OK;
}

int bsa_layout_order(const bsa_layout* layout, const int32_t** order, int* count) {
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (order) *order = layout->order.data();
  if (count) *count = int(layout->order.size());
  return BSA_OK;
}

int bsa_layout_csc(const bsa_layout* layout, const int32_t** col_ptr, const int32_t** row_idx,
                   int* cols, int* nnz) {
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (col_ptr) *col_ptr = layout->col_ptr.data();
  if (row_idx) *row_idx = layout->row_idx.data();
  if (cols) *cols = int(layout->col_ptr.size()) - 1;
  if (nnz) *nnz = int(layout->row_idx.size());
  return BSA_OK;
}

static int check_device(const bsa_layout* layout) {
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (layout->device < 0 || !layout->d_base)
    return set_error(BSA_ERR_INVALID_ARG, "layout was built host-only (device = -1)");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (cur != layout->device)
    return set_error(BSA_ERR_INVALID_ARG, "layout lives on device " + std::to_string(layout->device) +
                                              " but the current device is " + std::to_string(cur));
  return BSA_OK;
}

int bsa_layout_segments(const bsa_layout* layout, const int32_t** seg_ptr, const int32_t** segs,
                        int* layout_heads, int* count) {
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (seg_ptr) *seg_ptr = layout->seg_ptr.data();
  if (segs) *segs = layout->segs.data();
  if (layout_heads) *layout_heads = layout->L;
  if (count) *count = int(layout->segs.size() / 3);
  return BSA_OK;
}

int bsa_forward(const void* q, const void* k, const void* v, const bsa_layout* layout, int B,
                int n, int heads, int kv_heads, int d, float scale, void* o, float* lse,
                void* stream) {
  int st = check_device(layout);
  if (st != BSA_OK) return st;
  if (B != layout->B || n != layout->n)
    return set_error(BSA_ERR_SHAPE, "B/n differ from the layout's (" + std::to_string(layout->B) +
                                        ", " + std::to_string(layout->n) + ")");
  if (B != 64 && B != 128) return set_error(BSA_ERR_UNSUPPORTED, "B must be 64 or 128");
  if (d != 64 && d != 128) return set_error(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (heads < 1 || kv_heads < 1) return set_error(BSA_ERR_SHAPE, "heads and kv_heads must be >= 1");
  if (heads % kv_heads) return set_error(BSA_ERR_SHAPE, "heads must be a multiple of kv_heads");
  if (heads % layout->L) return set_error(BSA_ERR_SHAPE, "heads must be a multiple of layout_heads");
  if (!(std::isfinite(scale) && scale > 0.f)) return set_error(BSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!q || !k || !v || !o || !lse) return set_error(BSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return set_error(BSA_ERR_INVALID_ARG, "q, k, v and o must be 16-byte aligned");
  if (!aligned(lse, 4)) return set_error(BSA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (int64_t(heads) * (int64_t(n + B - 1) / B) > INT32_MAX)
    return set_error(BSA_ERR_SHAPE, "too many (head, block) work items");
  bsa::ForwardArgs a{q, k, v, o, lse, layout, B, n, heads, kv_heads, d, scale, stream, 0, 0};
  return bsa::launch_forward(a);
}

int bsa_debug_timeout_probe(const bsa_layout* layout, int d, uint64_t timeout_ns, void* stream) {
  int st = check_device(layout);
  if (st != BSA_OK) return st;
  if (layout->B != 64 && layout->B != 128) return set_error(BSA_ERR_UNSUPPORTED, "B must be 64 or 128");
  if (d != 64 && d != 128) return set_error(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (timeout_ns == 0 || timeout_ns > 1000000000ull)
    return set_error(BSA_ERR_INVALID_ARG, "timeout_ns must lie in [1, 1e9]");
  bsa::ForwardArgs a{nullptr, nullptr, nullptr, nullptr, nullptr, layout, layout->B, layout->n,
                     layout->L, layout->L, d, 1.f, stream, 1, timeout_ns};
  return bsa::launch_forward(a);
}

int bsa_get_status(const bsa_layout* layout, void* stream) {
  int st = check_device(layout);
  if (st != BSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, layout->d_status, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(layout->d_status, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("status read: ") + cudaGetErrorString(e));
  if (word & bsa::kStatusTimeout)
    return set_error(BSA_ERR_DEVICE_TIMEOUT, "a device-side wait ran out; the kernel returned early");
  if (word & bsa::kStatusBadIndex)
    return set_error(BSA_ERR_SHAPE, "a decode position or page number was out of range; its row got o = 0");
  return BSA_OK;
}

void bsa_free(bsa_layout* layout) {
  if (!layout) return;
  if (layout->d_base) {
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    cudaSetDevice(layout->device);
    cudaFree(layout->d_base);
    if (prev >= 0 && prev != layout->device) cudaSetDevice(prev);
  }
  delete layout;
}

}  // extern "C"
