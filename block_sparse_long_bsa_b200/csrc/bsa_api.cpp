// C ABI entry points: argument validation, layout ownership, device upload and
// status reporting.  The arithmetic runs in the sm_100a kernel
// (bsa_fwd_sm100a.cu); nothing here computes attention.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

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
int counter_error(const char* what, cudaError_t e) {
  return set_error(BSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
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
    const size_t b_wk = lay->work.size() * sizeof(int32_t);
    const size_t o_wk = o_sg + round_up(b_sg, 256);
    const size_t o_st = o_wk + round_up(b_wk, 256), total = o_st + bsa::kStatusBlockBytes;
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
    if (e == cudaSuccess) e = cudaMemcpy(c + o_wk, lay->work.data(), b_wk, cudaMemcpyHostToDevice);
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
    lay->d_work = reinterpret_cast<const int32_t*>(c + o_wk);
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

int bsa_layout_work(const bsa_layout* layout, const int32_t** work, int* count) {
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  if (work) *work = layout->work.data();
  if (count) *count = int(layout->work.size() / 4);
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

static int check_forward(const void* q, const void* k, const void* v, const bsa_layout* layout, int B, int n,
                         int heads, int kv_heads, int d, float scale, const void* o, const float* lse) {
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
  return BSA_OK;
}

int bsa_forward(const void* q, const void* k, const void* v, const bsa_layout* layout, int B,
                int n, int heads, int kv_heads, int d, float scale, void* o, float* lse,
                void* stream) {
  const int st = check_forward(q, k, v, layout, B, n, heads, kv_heads, d, scale, o, lse);
  if (st != BSA_OK) return st;
  bsa::ForwardArgs a{q, k, v, o, lse, layout, B, n, heads, kv_heads, d, scale, stream, 0, 0};
  return bsa::launch_forward(a);
}

// Two copy streams per device (host to device, device to host), created on
// first use and kept for the process; every call orders its copies against
// the caller's stream with events, so calls may share them.
static int copy_streams(int dev, cudaStream_t* up, cudaStream_t* down) {
  static std::mutex mu;
  static cudaStream_t streams[64][2] = {};
  if (dev < 0 || dev >= 64) return set_error(BSA_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 2; ++i) {
    if (!streams[dev][i]) {
      const cudaError_t e = cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking);
      if (e != cudaSuccess) return set_error(BSA_ERR_CUDA, std::string("copy stream: ") + cudaGetErrorString(e));
    }
  }
  *up = streams[dev][0];
  *down = streams[dev][1];
  return BSA_OK;
}

int bsa_forward_host(const void* q_host, const void* k_host, const void* v_host, const bsa_layout* layout,
                     int B, int n, int heads, int kv_heads, int d, float scale, void* q, void* k, void* v,
                     void* o, float* lse, void* o_host, float* lse_host, int groups, void* stream) {
  int st = check_forward(q, k, v, layout, B, n, heads, kv_heads, d, scale, o, lse);
  if (st != BSA_OK) return st;
  if (!q_host || !k_host || !v_host || !o_host || !lse_host)
    return set_error(BSA_ERR_INVALID_ARG, "null host pointer");
  if (groups < 1) return set_error(BSA_ERR_INVALID_ARG, "groups must be >= 1");
  // Groups are runs of whole key/value heads whose first query head maps to
  // layout head 0, so each group is a forward of its own: `unit` key/value
  // heads is the smallest such step.
  const int g = heads / kv_heads;
  int a0 = g, b0 = layout->L;
  while (b0) {
    const int t = a0 % b0;
    a0 = b0;
    b0 = t;
  }
  const int unit = layout->L / a0;
  const int units = kv_heads / unit;
  const int G = groups < units ? groups : units;
  cudaStream_t up = nullptr, down = nullptr;
  st = copy_streams(layout->device, &up, &down);
  if (st != BSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t q_head = size_t(n) * d * 2, kv_head = q_head, lse_head = size_t(n) * sizeof(float);
  std::vector<cudaEvent_t> ev(2 * size_t(G) + 2, nullptr);
  cudaError_t e = cudaSuccess;
  for (auto& x : ev)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
  auto fail = [&](const char* what) {
    for (auto x : ev)
      if (x) cudaEventDestroy(x);
    return set_error(BSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  };
  if (e != cudaSuccess) return fail("events");
  // the copies start after the caller's earlier work on its stream
  e = cudaEventRecord(ev[0], s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(up, ev[0], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(down, ev[0], 0);
  if (e != cudaSuccess) return fail("ordering the copies");
  auto at = [](const void* p, size_t off) { return static_cast<const char*>(p) + off; };
  auto at_mut = [](void* p, size_t off) { return static_cast<char*>(p) + off; };
  for (int i = 0; i < G; ++i) {
    const int u0 = int(int64_t(units) * i / G), u1 = int(int64_t(units) * (i + 1) / G);
    const int kv0 = u0 * unit, kvn = (u1 - u0) * unit, h0 = kv0 * g, hn = kvn * g;
    const size_t qo = size_t(h0) * q_head, qb = size_t(hn) * q_head;
    const size_t ko = size_t(kv0) * kv_head, kb = size_t(kvn) * kv_head;
    e = cudaMemcpyAsync(at_mut(q, qo), at(q_host, qo), qb, cudaMemcpyHostToDevice, up);
    if (e == cudaSuccess) e = cudaMemcpyAsync(at_mut(k, ko), at(k_host, ko), kb, cudaMemcpyHostToDevice, up);
    if (e == cudaSuccess) e = cudaMemcpyAsync(at_mut(v, ko), at(v_host, ko), kb, cudaMemcpyHostToDevice, up);
    if (e == cudaSuccess) e = cudaEventRecord(ev[1 + 2 * i], up);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev[1 + 2 * i], 0);
    if (e != cudaSuccess) return fail("host-to-device copy");
    bsa::ForwardArgs a{at(q, qo), at(k, ko), at(v, ko), at_mut(o, qo),
                       reinterpret_cast<float*>(at_mut(lse, size_t(h0) * lse_head)), layout, B, n, hn, kvn, d,
                       scale, stream, 0, 0};
    st = bsa::launch_forward(a);
    if (st != BSA_OK) {
      for (auto x : ev) cudaEventDestroy(x);
      return st;
    }
    e = cudaEventRecord(ev[2 + 2 * i], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(down, ev[2 + 2 * i], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(at_mut(o_host, qo), at(o, qo), qb, cudaMemcpyDeviceToHost, down);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(at_mut(lse_host, size_t(h0) * lse_head), at(lse, size_t(h0) * lse_head),
                          size_t(hn) * lse_head, cudaMemcpyDeviceToHost, down);
    if (e != cudaSuccess) return fail("device-to-host copy");
  }
  // the caller's stream completes after the last copy back
  e = cudaEventRecord(ev[2 * size_t(G) + 1], down);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev[2 * size_t(G) + 1], 0);
  if (e != cudaSuccess) return fail("ordering the copies back");
  for (auto x : ev) cudaEventDestroy(x);   // released once their work completes
  return BSA_OK;
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
  if (!layout) return set_error(BSA_ERR_INVALID_ARG, "layout is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* d_word = nullptr;
  if (layout->device < 0) {
    // a host-only layout: the status word of the allocation-free entry point's
    // static block on the current device
    const int st = bsa::noalloc_status_word(&d_word);
    if (st != BSA_OK) return st;
  } else {
    const int st = check_device(layout);
    if (st != BSA_OK) return st;
    d_word = layout->d_status;
  }
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, d_word, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_word, 0, sizeof(uint32_t), s);
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
    for (cudaEvent_t& ev : layout->counter_event)
      if (ev) cudaEventDestroy(ev);
    cudaFree(layout->d_base);
    if (prev >= 0 && prev != layout->device) cudaSetDevice(prev);
  }
  delete layout;
}

}  // extern "C"
