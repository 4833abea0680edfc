// fsel.cuh -- exact ordered top-K of a candidate set by one fine histogram.
//
// The candidates (rank values v = key << 32 | ~index, select.cuh) sit in
// registers, E per thread.  The caller knows a lower bound vlo of the K-th
// largest candidate (the digit floor of the K-th largest buffered entry, or a
// row's shared threshold) and an upper bound khi of every key; candidates
// below vlo are dropped.  The key span [key(vlo), khi] is cut into 1024 equal
// bins,
//     digit(v) = (key(v) - key(vlo)) >> s,   s the least shift with span >> s < 1024,
// so the bins follow the candidates' own range instead of the fixed top bits
// of the key: a top K squeezed into a fraction of an octave still spreads
// over hundreds of bins.  One counting pass and one suffix scan of that
// histogram give the bin b holding the K-th largest candidate; every winner
// above it lands at "winners in higher bins + its rank inside its own (small)
// bin", and the members of bin b are ranked among themselves.  There is no
// sort and no second pass over the candidates.
//
// Cost is set by barriers and shared-memory round trips, not by arithmetic,
// so the steps are laid out for them: each thread owns 4 consecutive bins
// (one conflict-free 16-byte access), the histogram is left zeroed for the
// next call by the pass that last reads it, and the result is out 3 barriers
// after the counting pass.
//
// This is the radix-select family of "Iterate Topk" and of qsa_topk2
// ("Round 18 Track C", section 1 Target 1): a digit histogram over order
// keys whose suffix sums locate the K-th largest; here the digit is taken
// relative to known bounds rather than from the top bits, and one level
// suffices unless the K-th largest shares its bin with more than
// kFineBoundaryMax others (heavy ties), where the caller falls back to the
// radix compaction of select.cuh.
#pragma once

#include "hsel.cuh"

namespace idx {

constexpr int kFineBins = 1024;
constexpr int kFineBoundaryMax = 256;

// Shared-memory areas of a fine select (all distinct, 16-byte aligned).
struct FineArea {
  uint32_t* hist;   // kFineBins words, zero between calls
  uint32_t* start;  // kFineBins words: bin offsets, then bin ends
  uint64_t* tv;     // >= K entries: winners grouped by bin
  uint32_t* tb;     // >= K entries
  uint64_t* bl_v;   // kFineBoundaryMax + 2 entries: members of the boundary bin
  uint32_t* bl_b;   // kFineBoundaryMax + 2 entries
  uint32_t* wsum;   // one word per warp
  uint32_t* bcast;  // 4 words
};

// Zero the histogram of a fine area (all NT threads; a barrier must follow
// before the first fine_select).
template <int NT>
__device__ __forceinline__ void fine_clear(const FineArea& ar) {
  for (int i = threadIdx.x; i < kFineBins / 4; i += NT)
    reinterpret_cast<uint4*>(ar.hist)[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Shift that maps the key span [klo, khi] into kFineBins bins.
__device__ __forceinline__ int fine_shift(uint32_t klo, uint32_t khi) {
  const uint32_t span = khi > klo ? khi - klo : 0u;
  return span < (uint32_t)kFineBins ? 0 : (32 - __clz(span)) - 10;
}

// Exact top K of the register-held candidates (v[k] for k < nk, 0 = none;
// bits[k] their fp32 bits), in order.  Keeps v >= vlo; kept keys are expected
// to be <= khi (a larger one is still placed correctly, in the top bin).  Calls emit(pos, v, bits) once for each of the min(K, #kept)
// winners with its final position (0 = best), and pad(pos) for every
// position from there up to K - 1.  NT = kFineBins / 4 threads take part
// (each owns 4 bins).  The caller puts a barrier between its last use of the
// areas (other than the zeroed histogram) and this call.  Returns false,
// uniformly and having emitted nothing, when the boundary bin holds more than
// kFineBoundaryMax candidates; the histogram is zero again either way.  Ends
// after the emits, with no barrier.
template <int NT, int E, class Emit, class Pad>
__device__ bool fine_select(const uint64_t (&v)[E], const uint32_t (&bits)[E], int nk, uint64_t vlo,
                            uint32_t khi, int K, const FineArea& ar, Emit emit, Pad pad) {
  static_assert(kFineBins == 4 * NT, "each thread owns 4 bins");
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t klo = (uint32_t)(vlo >> 32);
  const int s = fine_shift(klo, khi);
  // (clamped: a key above khi only joins the top bin, which keeps the order)
  auto digit = [&](uint64_t x) {
    return min(((uint32_t)(x >> 32) - klo) >> s, (uint32_t)kFineBins - 1u);
  };
  auto kept = [&](int k) { return k < nk && v[k] >= vlo && v[k] != 0; };
  // P1: count.
#pragma unroll
  for (int k = 0; k < E; ++k)
    if (kept(k)) atomicAdd(&ar.hist[digit(v[k])], 1u);
  group_sync(NT);
  IDX_TRACE(21);
  // P2: suffix scan.  Thread t owns bins 4u .. 4u + 3 with u = NT - 1 - t, so
  // thread order is descending bin order; dh[0] is its highest bin.
  const int u = NT - 1 - tid;
  const uint4 q = reinterpret_cast<const uint4*>(ar.hist)[u];
  const uint32_t dh[4] = {q.w, q.z, q.y, q.x};
  const uint32_t s4 = q.x + q.y + q.z + q.w;
  const uint32_t incl = warp_incl_scan(s4);
  if (lane_id() == 31) ar.wsum[warp] = incl;
  group_sync(NT);
  uint32_t excl = incl - s4, total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t x = ar.wsum[w];
    if (w < warp) excl += x;
    total += x;
  }
  {
    uint32_t st[4], cum = excl;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      st[e] = cum;
      if (total > (uint32_t)K && cum < (uint32_t)K && cum + dh[e] >= (uint32_t)K) {
        ar.bcast[0] = (uint32_t)(4 * u + 3 - e);
        ar.bcast[1] = cum;
        ar.bcast[2] = dh[e];
      }
      cum += dh[e];
    }
    reinterpret_cast<uint4*>(ar.start)[u] = make_uint4(st[3], st[2], st[1], st[0]);
  }
  group_sync(NT);
  IDX_TRACE(22);
  // P3: winners grouped by bin (highest bin first), boundary members listed;
  // the histogram is zeroed for the next call.
  const bool all = total <= (uint32_t)K;
  const uint32_t b = all ? 0xFFFFFFFFu : ar.bcast[0];
  const int above = all ? (int)total : (int)ar.bcast[1];
  const int cnt = all ? 0 : (int)ar.bcast[2];
  reinterpret_cast<uint4*>(ar.hist)[u] = make_uint4(0u, 0u, 0u, 0u);
  if (!all && cnt > kFineBoundaryMax) return false;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    if (!kept(k)) continue;
    const uint32_t d = digit(v[k]);
    if (all || d > b) {
      const uint32_t p = atomicAdd(&ar.start[d], 1u);
      ar.tv[p] = v[k];
      ar.tb[p] = bits[k];
    } else if (d == b) {
      const uint32_t p = atomicAdd(&ar.start[d], 1u) - (uint32_t)above;
      ar.bl_v[p] = v[k];
      ar.bl_b[p] = bits[k];
    }
  }
  if (tid == 0) ar.bl_v[cnt] = 0ull;  // members are read two at a time
  group_sync(NT);
  IDX_TRACE(23);
  // P4: bins above b are full, so bin d occupies [end(d + 1), end(d)) with
  // end = the start[] counters after P3 (end(kFineBins) = 0).
  for (int i = tid; i < above; i += NT) {
    const uint64_t x = ar.tv[i];
    const uint32_t d = digit(x);
    const int hi = (int)ar.start[d];
    const int lo = d + 1 < (uint32_t)kFineBins ? (int)ar.start[d + 1] : 0;
    int pos = lo;
    for (int j = lo; j < hi; ++j) pos += ar.tv[j] > x;
    emit(pos, x, ar.tb[i]);
  }
  const int r = K - above;
  const int half = (cnt + 1) >> 1;
  for (int t = tid; t < cnt; t += NT) {
    const uint64_t x = ar.bl_v[t];
    int rank = 0;
    for (int j = 0; j < half; ++j) {
      const ulonglong2 w2 = reinterpret_cast<const ulonglong2*>(ar.bl_v)[j];
      rank += (w2.x > x) + (w2.y > x);
    }
    if (rank < r) emit(above + rank, x, ar.bl_b[t]);
  }
  for (int k = min((int)total, K) + tid; k < K; k += NT) pad(k);
  IDX_TRACE(24);
  return true;
}

// Bounds of the K-th largest entry of a filter buffer from its exact digit
// histogram (hsel.cuh: hist kHBins words, chist kHCoarse words), computed by
// one whole warp: out[0] = the digit holding the K-th largest entry (0 when
// fewer than K entries), out[1] = the highest nonzero digit (0 when empty),
// out[3] = max(out[0], dmin) (a floor raised by a bound known from elsewhere),
// out[2] = the number of entries with digit >= out[3].  Every entry of the
// buffer's top K then has digit >= out[0], and every entry has digit <= out[1].
__device__ __forceinline__ void warp_hist_bounds(const uint32_t* hist, const uint32_t* chist,
                                                 uint32_t K, uint32_t dmin, uint32_t* out) {
  const uint32_t lane = lane_id();
  // coarse bins, lane l owning 4(31 - l) .. 4(31 - l) + 3 (lane 0 the top)
  const uint4 q = reinterpret_cast<const uint4*>(chist)[31 - lane];
  const uint32_t ch[4] = {q.w, q.z, q.y, q.x};
  const uint32_t s4 = q.x + q.y + q.z + q.w;
  const uint32_t incl = warp_incl_scan(s4);
  const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  // highest nonzero coarse bin, then its highest nonzero fine bin
  const uint32_t nz = __ballot_sync(0xFFFFFFFFu, s4 != 0);
  uint32_t bmax = 0;
  if (nz) {
    const int l = __ffs(nz) - 1;
    const uint32_t c4 = __shfl_sync(0xFFFFFFFFu, ch[0] ? 0u : ch[1] ? 1u : ch[2] ? 2u : 3u, l);
    const uint32_t c = 4 * (31 - l) + 3 - c4;
    const uint32_t f = hist[32 * c + 31 - lane];
    const uint32_t fz = __ballot_sync(0xFFFFFFFFu, f != 0);
    bmax = 32 * c + 31 - (__ffs(fz) - 1);
  }
  uint32_t b0 = 0, n0 = total;
  if (total >= K) {
    // the lane whose coarse bins reach K, then the coarse bin inside it
    const uint32_t hit = __ballot_sync(0xFFFFFFFFu, incl - s4 < K && incl >= K);
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
    // fine bins of coarse bin cb, lane l owning bin 32 cb + 31 - l
    const uint32_t f = hist[32 * cb + 31 - lane];
    const uint32_t fi = warp_incl_scan(f) + before;
    const uint32_t fh = __ballot_sync(0xFFFFFFFFu, fi >= K);
    b0 = 32 * cb + 31 - (__ffs(fh) - 1);
    n0 = __shfl_sync(0xFFFFFFFFu, fi, __ffs(fh) - 1);
  }
  if (dmin > b0) {
    // entries at or above dmin: coarse bins above its own, then its fine bins
    const uint32_t cd = dmin >> 5;
    uint32_t part = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (4 * (31 - lane) + 3 - e > cd) part += ch[e];
    const uint32_t f = hist[32 * cd + 31 - lane];
    if (31 - lane >= (dmin & 31)) part += f;
    n0 = __reduce_add_sync(0xFFFFFFFFu, part);
  }
  if (lane == 0) {
    out[0] = b0;
    out[1] = bmax;
    out[2] = n0;
    out[3] = max(b0, dmin);
  }
}

// Copy published candidate lists (list i at bits/index + slot_of(i) * stride,
// L entries each, L a multiple of 4, lists 16-byte aligned) into shared
// memory: entry e of list i goes to sb[i * L + e] and si[i * L + e].  All NT
// threads; every copy is in flight at once (16-byte asynchronous copies), and
// the call ends with a barrier.
template <int NT, class SlotOf>
__device__ __forceinline__ void stage_lists(int nslots, SlotOf slot_of, const uint32_t* cand_bits,
                                            const int32_t* cand_idx, int64_t stride, int L,
                                            uint32_t* sb, uint32_t* si) {
  const int per = L / 4;
  const int nch = nslots * per;
  for (int c = threadIdx.x; c < nch; c += NT) {
    const int i = c / per, e = (c - i * per) * 4;
    const int64_t off = slot_of(i) * stride + e;
    cp_async16(sb + i * L + e, cand_bits + off);
    cp_async16(si + i * L + e, cand_idx + off);
  }
  cp_async_wait_all();
  group_sync(NT);
}

}  // namespace idx
