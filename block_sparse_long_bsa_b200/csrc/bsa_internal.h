// Internal declarations shared by the host layout compiler, the C ABI and the
// sm_100a kernel launcher.  Not part of the public interface.
#pragma once

#include <cuda_runtime_api.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include "bsa.h"

namespace bsa {
// Work counters of a layout.  Call number c of a layout (a forward or a
// backward launched eagerly) uses counter c % kWorkCounters; a call captured
// into a CUDA graph takes one of kGraphCounters counters for good.  Each
// counter sits on its own 128-byte line of the layout's status block: word 0
// is the next unclaimed work item, word 1 counts the CTAs that have finished;
// the last CTA of a launch sets both back to zero, so no clear is enqueued.
constexpr int kWorkCounters = 64;
constexpr int kGraphCounters = 192;
}  // namespace bsa

struct bsa_layout {
  int n = 0;             // tokens per sequence
  int B = 0;             // tokens per block
  int nb = 0;            // blocks per sequence, ceil(n / B)
  int L = 0;             // layout heads
  int device = -1;       // device holding the uploaded arrays, -1 for host-only
  int max_row = 0;       // longest row (kept blocks)
  std::vector<int32_t> row_ptr;   // [L*nb + 1]
  std::vector<int32_t> col_idx;   // [nnz]
  std::vector<int32_t> order;     // [L*nb], longest row first per layout head
  // [L*nb][4]: the forward's work table, per (layout head, rank in order):
  // query block, first CSR entry, kept blocks, and 1 when the last kept block
  // is the diagonal one, so one 16-byte load decodes a work item
  std::vector<int32_t> work;
  std::vector<int32_t> col_ptr;   // [L*nb + 1]: transposed layout (CSC), per layout head
  std::vector<int32_t> row_idx;   // [nnz]: query blocks keeping each key block, ascending
  std::vector<int32_t> seg_ptr;   // [L + 1]: column segments of layout head h are seg_ptr[h] .. seg_ptr[h+1]
  std::vector<int32_t> segs;      // [3 * segments]: (key block j, first row_idx entry, entries <= kColumnSegment)
  int max_segs = 0;               // most segments of one layout head
  void* d_base = nullptr;         // single device allocation holding the arrays below
  const int32_t* d_row_ptr = nullptr;
  const int32_t* d_col_idx = nullptr;
  const int32_t* d_order = nullptr;
  const int32_t* d_work = nullptr;   // 16-byte aligned
  const int32_t* d_col_ptr = nullptr;
  const int32_t* d_row_idx = nullptr;
  const int32_t* d_seg_ptr = nullptr;
  const int32_t* d_segs = nullptr;
  uint32_t* d_status = nullptr;   // bit 0: a device wait ran out
  // Work-counter bookkeeping (see bsa::kWorkCounters): the next eager slot, the
  // graph slots handed out, and per eager slot the event recorded after its
  // last launch, which the next call that wraps onto the slot waits for.
  mutable std::mutex counter_mu;
  mutable uint32_t next_counter = 0;
  mutable int graph_counters_used = 0;
  mutable cudaEvent_t counter_event[bsa::kWorkCounters] = {};
};

namespace bsa {

// Thread-local error message; returns the status for convenience.
int set_error(int status, const std::string& msg);

// Host layout compiler (bsa_layout.cpp).  Fills row_ptr/col_idx/order/work/max_row.
int compile_layout(const bsa_pattern& spec, int n, int B, int L, bsa_layout* out);

// Longest run of query blocks one key/value-gradient work item takes from a
// column of the transposed layout.
constexpr int kColumnSegment = 16;

// Device status bits.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadIndex = 2u;   // a decode position or page number was out of range
// The status block that follows a layout's arrays holds the status word at
// word 0 and, from byte 256 on, the work counters (kWorkCounters eager ones,
// then kGraphCounters for captured calls), one per 128-byte line.  The
// allocation-free scratch has one counter line, at word 32.
constexpr size_t kStatusBlockBytes = 256 + size_t(kWorkCounters + kGraphCounters) * 128;
constexpr int kScratchCounterWord = 32;

// Runs `launch(counter)` with one of the layout's work counters, under the
// layout's lock.  An eager call first makes `stream` wait for the previous
// launch that used the same counter (an event recorded after it), and records
// the counter's event after `launch` has enqueued its work, so calls on one
// layout never share a counter while both run, however many are in flight.  A
// call made while `stream` is capturing a CUDA graph gets a counter of its own
// that no other call uses (BSA_ERR_UNSUPPORTED once they run out).
template <class F>
int with_work_counter(const bsa_layout* L, cudaStream_t stream, F&& launch);

// Launch description handed to the kernel launcher (bsa_fwd_sm100a.cu).
struct ForwardArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const bsa_layout* layout;
  int B, n, heads, kv_heads, d;
  float scale;
  void* stream;
  // diagnostics: every thread waits on a never-completed barrier
  int debug_never;
  uint64_t timeout_ns;
};

int launch_forward(const ForwardArgs& a);

// Same launch with the forward's layout arrays (the work table, 16-byte
// aligned, and col_idx) and the status word at explicit device addresses (the
// allocation-free entry point stages them itself).
int launch_forward_with(const ForwardArgs& a, const int32_t* work, const int32_t* col_idx, uint32_t* status);

// Device address of the allocation-free entry point's status word on the
// current device (bsa_noalloc.cu).
int noalloc_status_word(uint32_t** out);

// Implementation of with_work_counter (a template, so it lives here).
int counter_error(const char* what, cudaError_t e);

template <class F>
int with_work_counter(const bsa_layout* L, cudaStream_t stream, F&& launch) {
  std::lock_guard<std::mutex> lock(L->counter_mu);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return counter_error("cudaStreamIsCapturing", e);
  uint32_t* const lines = L->d_status + 64;   // counter lines start at byte 256
  if (cap != cudaStreamCaptureStatusNone) {
    if (L->graph_counters_used >= kGraphCounters)
      return set_error(BSA_ERR_UNSUPPORTED, "this layout's counters for captured calls are used up (" +
                                                std::to_string(kGraphCounters) + "); build another layout");
    const int slot = kWorkCounters + L->graph_counters_used;
    const int st = launch(lines + size_t(slot) * 32);
    if (st == BSA_OK) ++L->graph_counters_used;
    return st;
  }
  const int slot = int(L->next_counter % kWorkCounters);
  cudaEvent_t& ev = L->counter_event[slot];
  if (ev) {
    e = cudaStreamWaitEvent(stream, ev, 0);
  } else {
    e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
  }
  if (e != cudaSuccess) return counter_error("ordering against the counter's last user", e);
  const int st = launch(lines + size_t(slot) * 32);
  if (st != BSA_OK) return st;
  ++L->next_counter;
  e = cudaEventRecord(ev, stream);
  if (e != cudaSuccess) return counter_error("recording the counter's event", e);
  return BSA_OK;
}

}  // namespace bsa

