// Internal declarations shared by the host layout compiler, the C ABI and the
// sm_100a kernel launcher.  Not part of the public interface.
#pragma once

#include <atomic>
#include <cstdint>
#include <string>
#include <vector>

#include "bsa.h"

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
  std::vector<int32_t> col_ptr;   // [L*nb + 1]: transposed layout (CSC), per layout head
  std::vector<int32_t> row_idx;   // [nnz]: query blocks keeping each key block, ascending
  std::vector<int32_t> seg_ptr;   // [L + 1]: column segments of layout head h are seg_ptr[h] .. seg_ptr[h+1]
  std::vector<int32_t> segs;      // [3 * segments]: (key block j, first row_idx entry, entries <= kColumnSegment)
  int max_segs = 0;               // most segments of one layout head
  void* d_base = nullptr;         // single device allocation holding the arrays below
  const int32_t* d_row_ptr = nullptr;
  const int32_t* d_col_idx = nullptr;
  const int32_t* d_order = nullptr;
  const int32_t* d_col_ptr = nullptr;
  const int32_t* d_row_idx = nullptr;
  const int32_t* d_seg_ptr = nullptr;
  const int32_t* d_segs = nullptr;
  uint32_t* d_status = nullptr;   // bit 0: a device wait ran out
  std::atomic<uint32_t> calls{0};  // forwards and backwards launched (picks each call's work counter)
};

namespace bsa {

// Thread-local error message; returns the status for convenience.
int set_error(int status, const std::string& msg);

// Host layout compiler (bsa_layout.cpp).  Fills row_ptr/col_idx/order/max_row.
int compile_layout(const bsa_pattern& spec, int n, int B, int L, bsa_layout* out);

// Longest run of query blocks one key/value-gradient work item takes from a
// column of the transposed layout.
constexpr int kColumnSegment = 16;

// Device status bits.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadIndex = 2u;   // a decode position or page number was out of range
// The status block that follows a layout's arrays holds the status word at
// word 0 and, from byte 256 on, kWorkCounters work counters, one per 128-byte
// line: call number c of a layout (forward or backward) uses counter
// c % kWorkCounters, so up to that many calls on one layout may be in flight
// at once.  The
// allocation-free scratch has one counter, at word 32.
constexpr int kWorkCounters = 64;
constexpr size_t kStatusBlockBytes = 256 + size_t(kWorkCounters) * 128;
constexpr int kScratchCounterWord = 32;

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

// Same launch with the layout arrays and status word at explicit device
// addresses (the allocation-free entry point stages them itself).
int launch_forward_with(const ForwardArgs& a, const int32_t* row_ptr, const int32_t* col_idx,
                        const int32_t* order, uint32_t* status);

}  // namespace bsa
