// CPU oracle for the strided indexer top-k. TEST INFRASTRUCTURE ONLY.
//
// Only the test suite, the smoke check and the benchmark's CPU-baseline leg
// may load this file's library. The product (the CUDA library) never calls it
// and shares no code, header or table with it.
//
// What it computes, per row r (plain definition, no blocking or reordering):
//   1. L = clamp(lengths[r], 0, row_stride), m = min(k, L).
//      Row r's entry j lives at logits[r * row_stride + j]; the stride is the
//      tensor's row stride, not the valid width (vLLM PR #42169, "实现拆解" 1-2:
//      the top-k must use logits.stride(0) rather than logits.size(1), since the
//      padded DeepGEMM logits are not contiguous).
//   2. Stable-sort the indices 0..L-1 by value, descending: equal values keep
//      ascending index order.
//   3. out[r*k + t] = index at sorted position t for t < m; -1 for m <= t < k.
// The indices are row-local (SGLang PR #34167 code excerpt: idx = chunk_start +
// local_idx), and the "gt" / "eq" split around a threshold value in that
// excerpt is what the stable sort resolves exactly: every value above the k-th
// is taken, and among values equal to it the lowest indices win.
//
// Total order used for "descending" (the pages do not fix these cases):
//   NaN (any payload) ranks above +inf, all NaNs equal to each other;
//   -0.0 == +0.0; otherwise IEEE order. Comparisons are done in fp64, which
//   is exact for fp32 inputs.
//
// Parity status: pinned by brute force, special cases, library sorts and
// invariants in tests/test_oracle.py; the pages print no worked example.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <thread>
#include <vector>

namespace {

// true when value a ranks strictly above value b
bool ranks_above(float fa, float fb) {
  const double a = static_cast<double>(fa);
  const double b = static_cast<double>(fb);
  const bool na = std::isnan(a), nb = std::isnan(b);
  if (na || nb) return na && !nb;
  return a > b;  // -0.0 > +0.0 is false both ways: equal
}

void one_row(const float* row, int64_t row_stride, int32_t len, int32_t k, int32_t* out) {
  int64_t L = len;
  if (L < 0) L = 0;
  if (L > row_stride) L = row_stride;
  const int64_t m = std::min<int64_t>(k, L);
  std::vector<int32_t> order(static_cast<size_t>(L));
  for (int64_t j = 0; j < L; ++j) order[static_cast<size_t>(j)] = static_cast<int32_t>(j);
  std::stable_sort(order.begin(), order.end(),
                   [row](int32_t a, int32_t b) { return ranks_above(row[a], row[b]); });
  for (int64_t t = 0; t < k; ++t) out[t] = (t < m) ? order[static_cast<size_t>(t)] : -1;
}

}  // namespace

extern "C" {

// Returns 0 on success, -1 on a bad argument. num_threads <= 0 uses every
// hardware thread. Rows are split into contiguous blocks across threads.
int oracle_dsa_topk(const float* logits, int64_t row_stride, const int32_t* lengths,
                    int64_t num_rows, int32_t k, int32_t* out, int32_t num_threads) {
  if (num_rows < 0 || k < 1 || row_stride < 1) return -1;
  if (num_rows == 0) return 0;
  if (!logits || !lengths || !out) return -1;
  int64_t nt = num_threads > 0 ? num_threads : static_cast<int64_t>(std::thread::hardware_concurrency());
  if (nt < 1) nt = 1;
  if (nt > num_rows) nt = num_rows;
  auto work = [&](int64_t r0, int64_t r1) {
    for (int64_t r = r0; r < r1; ++r)
      one_row(logits + r * row_stride, row_stride, lengths[r], k, out + r * static_cast<int64_t>(k));
  };
  if (nt == 1) {
    work(0, num_rows);
    return 0;
  }
  std::vector<std::thread> pool;
  for (int64_t t = 0; t < nt; ++t) {
    const int64_t r0 = num_rows * t / nt, r1 = num_rows * (t + 1) / nt;
    pool.emplace_back(work, r0, r1);
  }
  for (auto& th : pool) th.join();
  return 0;
}

int oracle_hardware_threads(void) { return static_cast<int>(std::thread::hardware_concurrency()); }

}  // extern "C"
