// Host layout compiler: pattern spec -> sorted CSR of kept key blocks per
// (layout head, query block) -> longest-row-first processing order.
//
// Families (rules stated in include/bsa.h):
//   band + global first block -- "Block-Sparse Attention" (How It Works);
//     "Block Sparse Attention in LLMs", section 5B; window 0 without block 0
//     is the within-chunk term of "bsbr" (Solution).
//   dyadic -- "BF1: A Causal Dyadic Sparse-Attention Retrofit ...", Method and
//     section 3.1.
//   static random -- BF1's static-random control (sections 5, 8); the
//     generator is this library's reading, driven by SplitMix64 (Steele, Lea,
//     Flood 2014).
//   explicit -- the block mask M_B of "Block-Sparse Attention" (Math Or
//     Compute Schema).
// The planning step is timed separately from the kernel, as BF1 does
// (section 4, "separate topology timing").
#include <algorithm>
#include <cmath>
#include <numeric>

#include "bsa_internal.h"

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

struct SplitMix64 {
  uint64_t state;
  explicit SplitMix64(uint64_t s) : state(s) {}
  uint64_t next() {
    state += kGolden;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

// Appends the sorted kept blocks of query block i to `row` using a scratch
// flag array `mark` (size nb, all zero on entry and on exit).
void band_dyadic_row(int i, int window, bool global_first, bool dyadic, int kmin,
                     std::vector<uint8_t>& mark, std::vector<int32_t>& row) {
  row.clear();
  auto keep = [&](int j) {
    if (j >= 0 && j <= i && !mark[j]) {
      mark[j] = 1;
      row.push_back(j);
    }
  };
  for (int j = std::max(0, i - window); j <= i; ++j) keep(j);
  if (global_first) keep(0);
  if (dyadic) {
    for (int k = kmin; k < 62; ++k) {
      const int64_t off = int64_t(1) << k;
      if (int64_t(i) - off < 0) break;
      keep(int(int64_t(i) - off));
    }
  }
  std::sort(row.begin(), row.end());
  for (int j : row) mark[j] = 0;
}

}  // namespace

namespace bsa {

int compile_layout(const bsa_pattern& spec, int n, int B, int L, bsa_layout* out) {
  const int64_t nb64 = (int64_t(n) + B - 1) / B;
  const int nb = int(nb64);
  out->n = n;
  out->B = B;
  out->nb = nb;
  out->L = L;
  out->row_ptr.assign(size_t(L) * nb + 1, 0);
  out->col_idx.clear();
  out->max_row = 0;

  std::vector<uint8_t> mark(nb, 0);
  std::vector<int32_t> row;
  row.reserve(nb);
  std::vector<int32_t> cand;
  size_t r = 0;

  int64_t ppm = 0;
  if (spec.kind == BSA_PATTERN_RANDOM) ppm = std::llround(spec.density * 1e6);

  for (int h = 0; h < L; ++h) {
    SplitMix64 rng(spec.seed + uint64_t(h + 1) * kGolden);
    for (int i = 0; i < nb; ++i) {
      switch (spec.kind) {
        case BSA_PATTERN_BAND_GLOBAL:
          band_dyadic_row(i, spec.window, spec.global_first != 0, false, 0, mark, row);
          break;
        case BSA_PATTERN_DYADIC:
          band_dyadic_row(i, spec.window, spec.global_first != 0, true, spec.dyadic_kmin,
                          mark, row);
          break;
        case BSA_PATTERN_RANDOM: {
          const int mandatory = (i == 0) ? 1 : 2;
          const int64_t target = (ppm * int64_t(i + 1) + 500000) / 1000000;
          const int total = int(std::min<int64_t>(i + 1, std::max<int64_t>(mandatory, target)));
          const int draws = total - mandatory;
          cand.resize(i > 1 ? i - 1 : 0);
          std::iota(cand.begin(), cand.end(), 1);   // blocks 1 .. i-1
          for (int t = 0; t < draws; ++t) {
            const uint64_t span = uint64_t(cand.size()) - uint64_t(t);
            const int j = t + int(rng.next() % span);
            std::swap(cand[t], cand[j]);
          }
          row.assign(cand.begin(), cand.begin() + draws);
          row.push_back(0);
          if (i > 0) row.push_back(i);
          std::sort(row.begin(), row.end());
          break;
        }
        case BSA_PATTERN_EXPLICIT: {
          row.clear();
          const uint8_t* m = spec.mask + (size_t(h) * nb + i) * nb;
          for (int j = 0; j < nb; ++j) {
            if (m[j]) {
              if (j > i)
                return set_error(BSA_ERR_NONCAUSAL,
                                 "explicit block mask keeps block " + std::to_string(j) +
                                     " for query block " + std::to_string(i) +
                                     " of layout head " + std::to_string(h));
              row.push_back(j);
            }
          }
          break;
        }
        default:
          return set_error(BSA_ERR_INVALID_ARG, "unknown pattern kind");
      }
      out->col_idx.insert(out->col_idx.end(), row.begin(), row.end());
      if (out->col_idx.size() > size_t(INT32_MAX))
        return set_error(BSA_ERR_SHAPE, "layout has more than 2^31-1 kept blocks");
      out->row_ptr[r + 1] = int32_t(out->col_idx.size());
      out->max_row = std::max<int>(out->max_row, int(row.size()));
      ++r;
    }
  }

  // The transposed layout (for gradients of keys and values): for layout head
  // h and key block j, the query blocks whose rows keep j, ascending.
  out->col_ptr.assign(size_t(L) * nb + 1, 0);
  out->row_idx.assign(out->col_idx.size(), 0);
  for (int h = 0; h < L; ++h)
    for (int i = 0; i < nb; ++i) {
      const size_t r = size_t(h) * nb + i;
      for (int32_t e = out->row_ptr[r]; e < out->row_ptr[r + 1]; ++e)
        ++out->col_ptr[size_t(h) * nb + out->col_idx[e] + 1];
    }
  for (size_t c = 0; c + 1 < out->col_ptr.size(); ++c) out->col_ptr[c + 1] += out->col_ptr[c];
  {
    std::vector<int32_t> fill(out->col_ptr.begin(), out->col_ptr.end() - 1);
    for (int h = 0; h < L; ++h)
      for (int i = 0; i < nb; ++i) {
        const size_t r = size_t(h) * nb + i;
        for (int32_t e = out->row_ptr[r]; e < out->row_ptr[r + 1]; ++e)
          out->row_idx[fill[size_t(h) * nb + out->col_idx[e]]++] = i;
      }
  }

  // Column segments (the work list of the key/value gradients): each column
  // cut into runs of at most kColumnSegment query blocks, so a key block read
  // by every query block (a global first block) is shared out like any other;
  // per layout head, longest segment first, equal lengths in column order.
  out->seg_ptr.assign(size_t(L) + 1, 0);
  out->segs.clear();
  for (int h = 0; h < L; ++h) {
    const size_t first = out->segs.size() / 3;
    for (int j = 0; j < nb; ++j) {
      const int32_t c0 = out->col_ptr[size_t(h) * nb + j], c1 = out->col_ptr[size_t(h) * nb + j + 1];
      for (int32_t e = c0; e < c1; e += kColumnSegment) {
        out->segs.push_back(j);
        out->segs.push_back(e);
        out->segs.push_back(std::min<int32_t>(kColumnSegment, c1 - e));
      }
    }
    const size_t count = out->segs.size() / 3 - first;
    std::vector<int32_t> idx(count);
    std::iota(idx.begin(), idx.end(), 0);
    const int32_t* sg = out->segs.data() + first * 3;
    std::stable_sort(idx.begin(), idx.end(), [sg](int32_t a, int32_t b) { return sg[3 * a + 2] > sg[3 * b + 2]; });
    std::vector<int32_t> sorted(count * 3);
    for (size_t x = 0; x < count; ++x)
      for (int w = 0; w < 3; ++w) sorted[3 * x + w] = sg[3 * idx[x] + w];
    std::copy(sorted.begin(), sorted.end(), out->segs.begin() + first * 3);
    if (out->segs.size() / 3 > size_t(INT32_MAX)) return set_error(BSA_ERR_SHAPE, "too many column segments");
    out->seg_ptr[h + 1] = int32_t(out->segs.size() / 3);
    out->max_segs = std::max<int>(out->max_segs, int(count));
  }

  // Longest row first within each layout head; equal lengths keep block order.
  out->order.resize(size_t(L) * nb);
  for (int h = 0; h < L; ++h) {
    int32_t* ord = out->order.data() + size_t(h) * nb;
    const int32_t* rp = out->row_ptr.data() + size_t(h) * nb;
    std::iota(ord, ord + nb, 0);
    std::stable_sort(ord, ord + nb, [rp](int32_t a, int32_t b) {
      return (rp[a + 1] - rp[a]) > (rp[b + 1] - rp[b]);
    });
  }
  // The forward's work table: each (layout head, rank) decoded once here.
  out->work.resize(size_t(4) * L * nb);
  for (int h = 0; h < L; ++h) {
    for (int rank = 0; rank < nb; ++rank) {
      const int32_t row = out->order[size_t(h) * nb + rank];
      const size_t r = size_t(h) * nb + row;
      const int32_t start = out->row_ptr[r], len = out->row_ptr[r + 1] - start;
      int32_t* w = out->work.data() + 4 * (size_t(h) * nb + rank);
      w[0] = row;
      w[1] = start;
      w[2] = len;
      w[3] = (len > 0 && out->col_idx[size_t(start) + len - 1] == row) ? 1 : 0;
    }
  }
  return BSA_OK;
}

}  // namespace bsa
