// hsel.cuh -- the running digit histogram of an online top-K filter.
//
// A candidate's digit is the top 12 bits of its order key (sign, exponent and
// three mantissa bits of the score: bins an eighth of an octave wide).  A
// filter (select.cuh) that also keeps the histogram of its buffer -- one
// shared-memory atomic per appended entry, plus one on a 128-bin coarse copy
// (digit >> 5) -- gets a running threshold cheaply: the highest digit b with
// at least K buffered entries in bins >= b bounds the K-th largest value from
// below, so "keep digit >= b" is exact.  One lane reads it off the coarse and
// fine histograms in a few instructions, from a racy snapshot (counts only
// grow, so a snapshot under-counts, which keeps the bound valid), without
// stopping the others; the buffer then rarely needs a compaction.  At the end
// of a segment the same floor tells the fine select (fsel.cuh) where the top K
// starts.  The digit histogram is the radix-select machinery of "Iterate Topk"
// (radix family) and of qsa_topk2 ("Round 18 Track C", section 1 Target 1),
// kept as a running statistic of the stream instead of recomputed in passes
// over the row.
#pragma once

#include "select.cuh"

namespace idx {

constexpr int kHBits = 12;
constexpr int kHBins = 1 << kHBits;          // 4096 fine bins
constexpr int kHShift = 32 - kHBits;         // digit = key >> kHShift
constexpr int kHCoarse = kHBins / 32;        // 128 coarse bins of 32 fine bins

__device__ __forceinline__ uint32_t hdigit_v(uint64_t v) {
  return (uint32_t)(v >> (32 + kHShift));
}

// filter_offer that also counts every appended entry in the fine and coarse
// histograms of the buffer (hist: kHBins words, chist: kHCoarse words).  Each
// taking lane claims its slot with its own shared-memory atomic: after the
// first few hundred offers only a few lanes of a warp take, and a ballot and
// shuffle per warp cost more than those atomics.
__device__ __forceinline__ void filter_offer_h(FilterState& fs, uint32_t* fb, uint32_t* fi,
                                               uint32_t* hist, uint32_t* chist, uint32_t bits,
                                               uint32_t index, bool valid) {
  const uint64_t v = valid ? rank_value(bits, index) : 0ull;
  if (v > fs.thr) {
    const int pos = atomicAdd(&fs.count, 1);
    fb[pos] = bits;
    fi[pos] = index;
    const uint32_t d = hdigit_v(v);
    atomicAdd(&hist[d], 1u);
    atomicAdd(&chist[d >> 5], 1u);
  }
}

// Clear the fine and coarse histograms (all NT threads; caller syncs after).
template <int NT>
__device__ __forceinline__ void hist_clear(uint32_t* hist, uint32_t* chist) {
  for (int i = threadIdx.x; i < kHBins; i += NT) hist[i] = 0u;
  for (int i = threadIdx.x; i < kHCoarse; i += NT) chist[i] = 0u;
}

// Recount the histograms from the buffer's fs.count entries (after a radix
// compaction dropped entries).  All NT threads; ends with a barrier.
template <int NT>
__device__ void hist_rebuild(const FilterState& fs, const uint32_t* fb, const uint32_t* fi,
                             uint32_t* hist, uint32_t* chist) {
  hist_clear<NT>(hist, chist);
  group_sync(NT);
  const int n = fs.count;
  for (int i = threadIdx.x; i < n; i += NT) {
    const uint32_t d = hdigit_v(rank_value(fb[i], fi[i]));
    atomicAdd(&hist[d], 1u);
    atomicAdd(&chist[d >> 5], 1u);
  }
  group_sync(NT);
}

// The highest digit b >= 1 with at least K entries counted in bins >= b, from
// a snapshot of histograms that other warps keep incrementing; 0 when fewer
// than K entries are counted.  Every count read is a lower bound of the
// buffer's true count, so the answer is a valid lower bound of the digit of
// the K-th largest buffered value.  One thread: coarse bins from the top
// (16-byte loads) until K entries are reached, then the 32 fine bins of the
// coarse bin that got there (no warp-synchronous steps: on this part a shuffle
// or ballot in a loop costs more than a short scan by one lane).
__device__ __forceinline__ uint32_t hist_floor_1t(const uint32_t* hist, const uint32_t* chist,
                                                  uint32_t K) {
  uint32_t cum = 0;
  for (int c4 = kHCoarse / 4 - 1; c4 >= 0; --c4) {
    const uint4 q = reinterpret_cast<const uint4*>(chist)[c4];
    const uint32_t h[4] = {q.w, q.z, q.y, q.x};  // coarse bins 4*c4+3 .. 4*c4
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (cum + h[k] >= K) {
        const int c = 4 * c4 + 3 - k;
        // fine bins of coarse bin c, top down; the coarse count alone
        // already guarantees bin 32 * c
        const uint4* f4 = reinterpret_cast<const uint4*>(hist + 32 * c);
        for (int f = 7; f >= 0; --f) {
          const uint4 w = f4[f];
          const uint32_t g[4] = {w.w, w.z, w.y, w.x};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            cum += g[e];
            if (cum >= K) return (uint32_t)(32 * c + 4 * f + 3 - e);
          }
        }
        return (uint32_t)(32 * c);
      }
      cum += h[k];
    }
  }
  return 0u;
}

// hist_floor_1t computed by a whole warp (every lane gets the result): lane l
// reads the 4 coarse bins 4(31 - l) .. 4(31 - l) + 3 (lane 0 the top ones),
// one inclusive scan finds the coarse bin that reaches K, and one more over
// its 32 fine bins the digit.  About a dozen dependent steps instead of a
// serial walk down the bins.
__device__ __forceinline__ uint32_t hist_floor_warp(const uint32_t* hist, const uint32_t* chist,
                                                    uint32_t K) {
  const uint32_t lane = lane_id();
  const uint4 q = reinterpret_cast<const uint4*>(chist)[31 - lane];
  const uint32_t ch[4] = {q.w, q.z, q.y, q.x};
  const uint32_t s4 = q.x + q.y + q.z + q.w;
  const uint32_t incl = warp_incl_scan(s4);
  const uint32_t hit = __ballot_sync(0xFFFFFFFFu, incl - s4 < K && incl >= K);
  if (!hit) return 0u;  // fewer than K entries counted
  const int l = __ffs(hit) - 1;
  uint32_t cum = incl - s4, cb = 0, before = 0;
  bool found = false;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (!found && cum + ch[e] >= K) {
      cb = 4 * (31 - lane) + 3 - e;
      before = cum;
      found = true;
    }
    cum += ch[e];
  }
  cb = __shfl_sync(0xFFFFFFFFu, cb, l);
  before = __shfl_sync(0xFFFFFFFFu, before, l);
  const uint32_t fi = warp_incl_scan(hist[32 * cb + 31 - lane]) + before;
  const uint32_t fh = __ballot_sync(0xFFFFFFFFu, fi >= K);
  // counts only grow while the warp reads them: a racy read may find K only
  // in the coarse count, and bin 32 cb is then still a valid floor
  return fh ? 32 * cb + 31 - (uint32_t)(__ffs(fh) - 1) : 32 * cb;
}

// Raise a filter's threshold to "digit >= b" (one thread).  A racing raise by
// another warp may win with a lower value: that only admits more entries.
__device__ __forceinline__ void raise_threshold_1t(FilterState& fs, const uint32_t* hist,
                                                   const uint32_t* chist, int K) {
  const uint32_t b = hist_floor_1t(hist, chist, (uint32_t)K);
  if (b != 0u) {
    const unsigned long long t = ((unsigned long long)b << (32 + kHShift)) - 1ull;
    if (t > fs.thr) fs.thr = t;
  }
}

// Load a filter buffer's n entries into registers (entry i = tid + k * NT).
template <int NT, int E>
__device__ __forceinline__ int load_buffer(const uint32_t* fb, const uint32_t* fi, int n,
                                           uint64_t (&v)[E], uint32_t (&bits)[E]) {
  const int nk = (n + NT - 1) / NT;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = (int)threadIdx.x + k * NT;
    v[k] = 0ull;
    bits[k] = 0u;
    if (k < nk && i < n) {
      bits[k] = fb[i];
      v[k] = rank_value(bits[k], fi[i]);
    }
  }
  return nk;
}

}  // namespace idx
