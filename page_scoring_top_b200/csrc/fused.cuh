// fused.cuh -- the select side of the fused score + top-K kernels.
//
// A decode kernel cuts the valid pages of a batch into one chunk per CTA; a
// chunk covers the tail of one request, whole requests, the head of another.
// Each (chunk, request) piece is a segment.  Per segment and token the kernel
// feeds every page score to an exact online filter (select.cuh; with one
// token per row the filter also keeps its digit histogram, hsel.cuh) and at
// the segment's end either writes the row (the request lies inside the chunk)
// or publishes the segment's top K to a candidate slot; the last CTA to
// publish for a request merges the slots into the final row.  Top-K
// selection ("Iterate Topk", opening description) over the page scores of
// "Iterate Centroids Score"; the tie rule of "Round 18 Track C", section 2.
#pragma once

#include "fsel.cuh"
#include "hsel.cuh"
#include "kernels.h"

namespace idx {

constexpr int kSelThreads = 256;  // threads 0..255 run every select step
static_assert(2 * (kSelThreads / 32) <= 32, "per-warp key maxima and minima fit the scratch");
constexpr int kMaxFusedT = 4;
// Virtual pages charged per request in fused mode: about what a segment-end
// select step costs in streaming time (a few microseconds at one SM's share
// of HBM bandwidth, minus what the stage ring absorbs; measured best among
// 256 .. 2304 on the decode workloads).
constexpr int kSegmentPages = 512;

// Shared-memory state of the fused select (pointers into the kernel's layout).
struct FusedSel {
  uint32_t* fbuf;       // per token: cap bits, then cap indices
  FilterState* fst;     // per token
  SelectScratch* sc;
  uint64_t* sortv;      // kMaxK + 2 entries
  uint32_t* sortb;      // kMaxK + 4 entries
  uint32_t* hist;       // kHBins + kHCoarse words (single-token rows only)
  int cap;              // filter entries per token
  int* s_flag;
  // single-token rows: the last polled high word of the request's shared
  // threshold (its key part), copied in asynchronously while streaming
  uint32_t* s_row;
};

// Filter entries per token for T tokens, the buffer holding `bufs` x
// kFilterCap entries in all (at most kFilterCap per token: a filter is
// loaded into registers whole).
__host__ __device__ inline int fused_cap(int T, int bufs = 1) {
  int tp = 1;
  while (tp < T) tp <<= 1;
  const int c = bufs * kFilterCap / tp;
  return c < kFilterCap ? c : kFilterCap;
}

// Segment start (all select threads; the caller syncs after).
template <bool HIST>
__device__ __forceinline__ void fused_begin(const FusedSel& f, int T) {
  if ((int)threadIdx.x < T) filter_reset(f.fst[threadIdx.x]);
  if (HIST) {
    hist_clear<kSelThreads>(f.hist, f.hist + kHBins);
    if (threadIdx.x == 0) *f.s_row = 0u;
  }
}

// One warp offers its 32 lanes' scores of token t.
template <bool HIST>
__device__ __forceinline__ void fused_offer(const FusedSel& f, int t, uint32_t bits, uint32_t index,
                                            bool valid) {
  if (HIST) {
    filter_offer_h(f.fst[0], f.fbuf, f.fbuf + f.cap, f.hist, f.hist + kHBins, bits, index, valid);
  } else {
    uint32_t* fb = f.fbuf + t * 2 * f.cap;
    filter_offer_lane(f.fst[t], fb, fb + f.cap, bits, index, valid);
  }
}

// The calling warp (all lanes) reads the floor off the histogram, then lane 0
// lifts the single-token filter's threshold to it, and shares it with the other CTAs streaming the same
// request: the filter's floor raises the request's threshold *row_thr
// (atomic max; a segment's K-th largest bounds its request's from below),
// and the request's threshold as last polled raises the filter's, so a
// segment stops buffering what another segment has already beaten.  The poll
// is an asynchronous 4-byte copy of the threshold's key half into s_row,
// read at the next raise: never a stall on global memory.
__device__ __forceinline__ void fused_raise(const FusedSel& f, int K,
                                            unsigned long long* row_thr) {
  const uint32_t b = hist_floor_warp(f.hist, f.hist + kHBins, (uint32_t)K);
  if (lane_id() != 0) return;
  FilterState& fs = f.fst[0];
  unsigned long long t = fs.thr;
  if (b != 0u) {
    const unsigned long long fl = (unsigned long long)b << (32 + kHShift);
    t = max(t, fl - 1ull);
    atomicMax(row_thr, fl);
  }
  const uint32_t hi = *reinterpret_cast<volatile uint32_t*>(f.s_row);
  if (hi != 0u) t = max(t, ((unsigned long long)hi << 32) - 1ull);
  if (t > fs.thr) fs.thr = t;
  cp_async4(f.s_row, reinterpret_cast<const uint32_t*>(row_thr) + 1);
}

// Overflow guard at a check point (all select threads, after a barrier that
// completed every offer): compact each filter holding more than compact_at.
// Every thread reads the counts before a second barrier, so all of them take
// the same decision even when fast warps go back to offering right after.
// Returns the smallest free room (cap - count) over the filters afterwards.
template <bool HIST>
__device__ __forceinline__ int fused_check(const FusedSel& f, int T, int K, int compact_at) {
  uint32_t over = 0;
  int used = 0;
  for (int t = 0; t < T; ++t) {
    const int n = f.fst[t].count;
    if (n > compact_at) over |= 1u << t;
    else used = max(used, n);
  }
  group_sync(kSelThreads);
  for (int t = 0; t < T; ++t)
    if (over >> t & 1u) {
      uint32_t* fb = f.fbuf + t * 2 * f.cap;
      filter_compact<kSelThreads>(f.fst[t], fb, fb + f.cap, K, *f.sc);
      if (HIST) hist_rebuild<kSelThreads>(f.fst[0], f.fbuf, f.fbuf + f.cap, f.hist, f.hist + kHBins);
      used = max(used, min(K, f.fst[t].count));
    }
  return f.cap - used;
}

// Check period (in rounds of 256 offers per token) and compaction mark: a
// check comes before a filter could overflow; without a histogram the
// compaction is also what raises the threshold, so it starts once a filter
// holds a few K entries.
__device__ __forceinline__ int fused_rounds(int cap, int K) {
  return max(1, min(4, (cap - K) / kSelThreads));
}
template <bool HIST>
__device__ __forceinline__ int fused_compact_at(int cap, int K) {
  const int guard = cap - fused_rounds(cap, K) * kSelThreads;
  return HIST ? guard : min(guard, max(4 * K, 1024));
}

// Where a single-token row's selection goes: the output row, and the
// candidate slots, threshold and arrival counter used when the row is split
// into segments over several CTAs.
struct RowOut {
  int32_t* idx_out;  // [rows][K]
  float* val_out;    // [rows][K] or null
  int K;
  uint32_t* cand_bits;
  int32_t* cand_idx;
  int64_t slot_stride;
  unsigned long long* row_thr;  // per row, zero between calls
  int32_t* arrive;              // per row, zero between calls
};

// The merge of a request row's published lists by the last CTA to arrive,
// when they fit the filter buffer together (nslots * lcap <= kFilterCap; every
// filter of the CTA is spent): the lists are staged into the buffer, then the
// fine select runs over the candidates' key span floored by the row's
// threshold.  When no threshold was raised or the boundary bin is crowded, the
// candidates' own digit histogram (in `dhist`, kHBins + kHCoarse words; null
// to skip this step) bounds the K-th largest first; heavy ties go to the
// radix compaction.  Writes the row, resets *row_thr.  All select threads.
template <class SlotOf>
__device__ bool merge_staged(const FusedSel& f, int nslots, SlotOf slot_of, const uint32_t* cand_bits,
                             const int32_t* cand_idx, int64_t stride, int lcap, int K,
                             unsigned long long* row_thr, uint32_t* dhist, int32_t* out_i,
                             float* out_v) {
  SelectScratch& sc = *f.sc;
  FilterState& fs = f.fst[0];
  uint32_t* fb = f.fbuf;
  uint32_t* fi = f.fbuf + kFilterCap;
  uint32_t* fine = &sc.hist[1][0];
  const FineArea ar{fine,    fine + kFineBins, f.sortv, f.sortb,
                    reinterpret_cast<uint64_t*>(f.fbuf), f.fbuf + 2 * (kFineBoundaryMax + 2),
                    sc.wsum, sc.bcast};
  constexpr int E = kFilterCap / kSelThreads;
  uint64_t v[E];
  uint32_t bits[E];
  auto out_emit = [&](int pos, uint64_t x, uint32_t xb) {
    out_i[pos] = (int32_t)~(uint32_t)x;
    if (out_v) out_v[pos] = __uint_as_float(xb);
  };
  auto out_pad = [&](int pos) {
    out_i[pos] = -1;
    if (out_v) out_v[pos] = __uint_as_float(kNegInfBits);
  };
  bool done = false;
  // the request's final threshold, read while the lists are staged
  unsigned long long rt = 0ull;
  if (threadIdx.x == 0) {
    rt = __ldcg(row_thr);
    *row_thr = 0ull;  // zero for the next call
  }
  // the buffer (already published) receives every list
  stage_lists<kSelThreads>(nslots, slot_of, cand_bits, cand_idx, stride, lcap, fb, fi);
  IDX_TRACE(25);
  const int nkm = load_buffer<kSelThreads, E>(fb, fi, nslots * lcap, v, bits);
  // The fine select over the candidates' key span, floored by the
  // request's threshold: with a threshold raised by the segments the span
  // is narrow.  When it is not (short segments) or the boundary bin is
  // crowded all the same, the candidates' own digit histogram bounds the
  // K-th largest as a segment's does, and the fine select runs again over
  // the digits from there up.
  uint32_t km = 0, kn = 0xFFFFFFFFu;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    km = max(km, (uint32_t)(v[k] >> 32));
    if (v[k] != 0) kn = min(kn, (uint32_t)(v[k] >> 32));
  }
  km = __reduce_max_sync(0xFFFFFFFFu, km);
  kn = __reduce_min_sync(0xFFFFFFFFu, kn);
  if (lane_id() == 0) {
    sc.wsum[threadIdx.x >> 5] = km;
    sc.wsum[kSelThreads / 32 + (threadIdx.x >> 5)] = kn;
  }
  if (threadIdx.x == 0) *reinterpret_cast<unsigned long long*>(&sc.bcast[0]) = rt;
  fine_clear<kSelThreads>(ar);
  group_sync(kSelThreads);
  IDX_TRACE(26);
  km = 0;
  kn = 0xFFFFFFFFu;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) {
    km = max(km, sc.wsum[w]);
    kn = min(kn, sc.wsum[kSelThreads / 32 + w]);
  }
  const uint64_t thr0 = *reinterpret_cast<const unsigned long long*>(&sc.bcast[0]);
  uint64_t thr = thr0 > ((uint64_t)kn << 32) ? thr0 : ((uint64_t)kn << 32);
  // (every thread has read wsum and bcast before fine_select's first barrier)
  if (thr0 != 0 || !dhist)
    done = fine_select<kSelThreads, E>(v, bits, nkm, thr, km, K, ar, out_emit, out_pad);
  if (!done && dhist) {
    // (a spent digit histogram: the next segment clears it)
    hist_clear<kSelThreads>(dhist, dhist + kHBins);
    group_sync(kSelThreads);
#pragma unroll
    for (int k = 0; k < E; ++k)
      if (k < nkm && v[k] >= thr0 && v[k] != 0) {
        const uint32_t d = (uint32_t)(v[k] >> (32 + kHShift));
        atomicAdd(&dhist[d], 1u);
        atomicAdd(&dhist[kHBins + (d >> 5)], 1u);
      }
    group_sync(kSelThreads);
    if ((threadIdx.x >> 5) == 0)
      warp_hist_bounds(dhist, dhist + kHBins, (uint32_t)K, 0u, sc.bcast);
    group_sync(kSelThreads);
    const uint32_t mb0 = sc.bcast[0], mbmax = sc.bcast[1];
    const uint64_t mlo = (uint64_t)mb0 << (32 + kHShift);
    thr = thr0 > mlo ? thr0 : mlo;
    const uint32_t mhi =
        mbmax + 1 >= (uint32_t)kHBins ? 0xFFFFFFFFu : ((mbmax + 1) << kHShift) - 1u;
    done = fine_select<kSelThreads, E>(v, bits, nkm, thr, mhi, K, ar, out_emit, out_pad);
  }
  if (!done) {
    // a crowded boundary bin (heavy ties): the entries at or above the
    // threshold go back to the buffer for the exact radix compaction
    if (threadIdx.x == 0) sc.ctr = 0;
    group_sync(kSelThreads);
#pragma unroll
    for (int k = 0; k < E; ++k)
      if (k < nkm && v[k] >= thr && v[k] != 0) {
        const int p = atomicAdd(&sc.ctr, 1);
        fb[p] = bits[k];
        fi[p] = ~(uint32_t)v[k];
      }
    group_sync(kSelThreads);
    if (threadIdx.x == 0) {
      fs.count = sc.ctr;
      fs.thr = 0ull;
    }
    group_sync(kSelThreads);
    filter_compact<kSelThreads>(fs, fb, fi, K, sc);
    sort_and_write<kSelThreads>(fb, fi, fs.count, K, f.sortv, f.sortb, out_i, out_v);
    done = true;
  }
  return done;
}

// Segment end of single-token row b in chunk j, the row spanning chunks
// j0..j1 (all select threads, after a barrier that completed every offer).
// The filter's digit histogram is exact for its buffer: one warp reads from
// it the digit b0 of the segment's K-th largest entry, so every entry of the
// segment's top K is >= vlo = b0's floor.  A segment that holds its whole row
// takes the exact ordered top K above vlo from registers (fine select,
// fsel.cuh).  Otherwise it publishes every entry >= vlo, unordered (about K
// plus one digit bin's worth), raises the row's threshold to vlo, and the
// last segment to arrive runs the fine select over all published entries.
static __device__ void hist_finalize(const FusedSel& f, const RowOut& o, int b, int j, int j0,
                                     int j1) {
  SelectScratch& sc = *f.sc;
  FilterState& fs = f.fst[0];
  uint32_t* fb = f.fbuf;
  uint32_t* fi = f.fbuf + f.cap;
  const bool single = j0 == j1;
  const int nslots = j1 - j0 + 1;
  int32_t* out_i = o.idx_out + (int64_t)b * o.K;
  float* out_v = o.val_out ? o.val_out + (int64_t)b * o.K : nullptr;
  const int64_t slot = (int64_t)(j + b);
  uint32_t* cbits = o.cand_bits + slot * o.slot_stride;
  int32_t* cidx = o.cand_idx + slot * o.slot_stride;
  unsigned long long* row_thr = o.row_thr + b;
  // Entries per published list: as many as the merge can hold in registers
  // (kFilterCap over all lists), at least K, at most a slot, a multiple of 4
  // (lists are copied 16 bytes at a time).
  const int lcap = max((o.K + 3) & ~3, min((int)o.slot_stride, kFilterCap / nslots) & ~3);
  // The areas: the fine histogram and its bin offsets in the second radix
  // histogram of the scratch, the winners in the sort staging, the boundary
  // list at the front of the buffer once the buffer is in registers.
  uint32_t* fine = &sc.hist[1][0];
  const FineArea ar{fine,    fine + kFineBins, f.sortv, f.sortb,
                    reinterpret_cast<uint64_t*>(f.fbuf), f.fbuf + 2 * (kFineBoundaryMax + 2),
                    sc.wsum, sc.bcast};
  constexpr int E = kFilterCap / kSelThreads;
  uint64_t v[E];
  uint32_t bits[E];
  auto out_emit = [&](int pos, uint64_t x, uint32_t xb) {
    out_i[pos] = (int32_t)~(uint32_t)x;
    if (out_v) out_v[pos] = __uint_as_float(xb);
  };
  auto out_pad = [&](int pos) {
    out_i[pos] = -1;
    if (out_v) out_v[pos] = __uint_as_float(kNegInfBits);
  };
  // (A poll of the request's threshold may still be landing in s_row: either
  // value is a floor of this request's K-th largest.  The wait for it comes
  // at the end, before the next segment resets s_row.)
  if ((threadIdx.x >> 5) == 0)
    warp_hist_bounds(f.hist, f.hist + kHBins, (uint32_t)o.K, single ? 0u : *f.s_row >> kHShift,
                     sc.bcast);
  if (threadIdx.x == 0) {
    sc.ctr = 0;
    if (single) *row_thr = 0ull;  // raised while streaming, read by nobody else
  }
  fine_clear<kSelThreads>(ar);
  const int nk = load_buffer<kSelThreads, E>(fb, fi, fs.count, v, bits);
  IDX_TRACE(19);
  group_sync(kSelThreads);
  // b0: the digit of the segment's K-th largest; bp >= b0: the publish
  // floor, raised to the request's threshold; n0: entries at or above bp.
  const uint32_t b0 = sc.bcast[0], bmax = sc.bcast[1], n0 = sc.bcast[2], bp = sc.bcast[3];
  const uint64_t vlo = (uint64_t)b0 << (32 + kHShift);
  const uint64_t vpub = (uint64_t)bp << (32 + kHShift);
  IDX_TRACE(13);
  bool ok = true;
  const uint32_t khi = bmax + 1 >= (uint32_t)kHBins ? 0xFFFFFFFFu : ((bmax + 1) << kHShift) - 1u;
  if (single) {
    ok = fine_select<kSelThreads, E>(v, bits, nk, vlo, khi, o.K, ar, out_emit, out_pad);
  } else if (n0 > (uint32_t)lcap) {
    // more entries at or above the publish floor than a list holds (the
    // boundary digit is wide): publish the segment's exact top K instead
    auto pub_emit = [&](int pos, uint64_t x, uint32_t xb) {
      cbits[pos] = xb;
      cidx[pos] = (int32_t)~(uint32_t)x;
    };
    auto pub_pad = [&](int pos) {
      cbits[pos] = kNegInfBits;
      cidx[pos] = -1;
    };
    ok = fine_select<kSelThreads, E>(v, bits, nk, vlo, khi, o.K, ar, pub_emit, pub_pad);
    if (ok) {
      for (int p = o.K + (int)threadIdx.x; p < lcap; p += kSelThreads) pub_pad(p);
      if (threadIdx.x == 0 && b0 != 0) atomicMax(row_thr, (unsigned long long)vlo);
    }
  } else {
#pragma unroll
    for (int k = 0; k < E; ++k)
      if (k < nk && v[k] >= vpub && v[k] != 0) {
        const int p = atomicAdd(&sc.ctr, 1);
        cbits[p] = bits[k];
        cidx[p] = (int32_t)~(uint32_t)v[k];
      }
    for (int p = (int)n0 + (int)threadIdx.x; p < lcap; p += kSelThreads) {
      cbits[p] = kNegInfBits;
      cidx[p] = -1;
    }
    // with b0 > 0 the segment holds K entries >= vlo: so does its row
    if (threadIdx.x == 0 && b0 != 0) atomicMax(row_thr, (unsigned long long)vlo);
  }
  if (!ok) {
    // a crowded digit bin (heavy ties): exact radix compaction first
    group_sync(kSelThreads);
    filter_compact<kSelThreads>(fs, fb, fi, o.K, sc);
    if (single) {
      sort_and_write<kSelThreads>(fb, fi, fs.count, o.K, f.sortv, f.sortb, out_i, out_v);
    } else {
      publish_candidates<kSelThreads>(fb, fi, fs.count, o.K, fs.thr, cbits, cidx, row_thr);
      for (int p = o.K + (int)threadIdx.x; p < lcap; p += kSelThreads) {
        cbits[p] = kNegInfBits;
        cidx[p] = -1;
      }
    }
  }
  IDX_TRACE(14);
  if (!single && arrive_last<kSelThreads>(o.arrive + b, nslots, f.s_flag)) {
    IDX_TRACE(15);
    auto slot_of = [=](int i) { return (int64_t)(j0 + i + b); };
    bool done = false;
    if (nslots * lcap <= kFilterCap)
      done = merge_staged(f, nslots, slot_of, o.cand_bits, o.cand_idx, o.slot_stride, lcap, o.K,
                          row_thr, f.hist, out_i, out_v);
    if (!done)
      merge_candidates<kSelThreads>(nslots, slot_of, o.cand_bits, o.cand_idx, o.slot_stride,
                                    lcap, o.K, row_thr, fs, f.fbuf, f.fbuf + kFilterCap,
                                    kFilterCap, sc, f.sortv, f.sortb, out_i, out_v);
    IDX_TRACE(16);
  }
  // every poll of the threshold has landed before the next segment (maybe of
  // another request) resets s_row, and before the CTA exits
  cp_async_wait_all();
  group_sync(kSelThreads);
}

// Segment end for request b, chunk j (all select threads, after a barrier
// that completed every offer).  The request's pages span chunks j0..j1.
template <bool HIST>
__device__ void fused_finalize(const FusedSel& f, const DecodeArgs& a, int T, int b, int j, int j0,
                               int j1) {
  SelectScratch& sc = *f.sc;
  if (HIST) {
    const RowOut o{a.idx_out,     a.val_out, a.K,       a.cand_bits,
                   a.cand_idx,    a.slot_stride, a.row_thr, a.arrive};
    hist_finalize(f, o, b, j, j0, j1);
    return;
  } else {
    for (int t = 0; t < T; ++t) {
      uint32_t* fb = f.fbuf + t * 2 * f.cap;
      uint32_t* fi = fb + f.cap;
      filter_compact<kSelThreads>(f.fst[t], fb, fi, a.K, sc);
      const int kk = f.fst[t].count;
      const int64_t orow = (int64_t)b * T + t;
      if (j0 == j1) {
        sort_and_write<kSelThreads>(fb, fi, kk, a.K, f.sortv, f.sortb, a.idx_out + orow * a.K,
                                    a.val_out ? a.val_out + orow * a.K : nullptr);
      } else {
        const int64_t slot = (int64_t)(j + b) * T + t;
        uint32_t* cb = a.cand_bits + slot * a.slot_stride;
        int32_t* ci = a.cand_idx + slot * a.slot_stride;
        publish_candidates<kSelThreads>(fb, fi, kk, a.K, f.fst[t].thr, cb, ci, a.row_thr + orow);
        // padded to a multiple of 4 entries for the staged merge's 16-byte copies
        for (int p = a.K + (int)threadIdx.x; p < ((a.K + 3) & ~3); p += kSelThreads) {
          cb[p] = kNegInfBits;
          ci[p] = -1;
        }
      }
    }
    if (j0 != j1 && arrive_last<kSelThreads>(a.arrive + b, j1 - j0 + 1, f.s_flag)) {
      const int nslots = j1 - j0 + 1, lcap = (a.K + 3) & ~3;
      for (int t = 0; t < T; ++t) {
        const int64_t orow = (int64_t)b * T + t;
        auto slot_of = [=](int i) { return (int64_t)(j0 + i + b) * T + t; };
        int32_t* out_i = a.idx_out + orow * a.K;
        float* out_v = a.val_out ? a.val_out + orow * a.K : nullptr;
        // (every filter of the CTA is spent: the whole buffer stages the lists)
        if (nslots * lcap <= kFilterCap)
          merge_staged(f, nslots, slot_of, a.cand_bits, a.cand_idx, a.slot_stride, lcap, a.K,
                       a.row_thr + orow, nullptr, out_i, out_v);
        else
          merge_candidates<kSelThreads>(nslots, slot_of, a.cand_bits, a.cand_idx, a.slot_stride,
                                        a.K, a.K, a.row_thr + orow, f.fst[0], f.fbuf,
                                        f.fbuf + kFilterCap, kFilterCap, sc, f.sortv, f.sortb,
                                        out_i, out_v);
        group_sync(kSelThreads);
      }
    }
  }
  group_sync(kSelThreads);
}

// Rows with no valid page get all-padding output (-1 / -inf), requests dealt
// round-robin over the grid (all select threads).
__device__ __forceinline__ void fused_empty_rows(const DecodeArgs& a, const int* s_off, int g,
                                                 int G) {
  for (int b = g; b < a.B; b += G) {
    if (s_off[b + 1] != s_off[b]) continue;
    for (int x = threadIdx.x; x < a.T * a.K; x += kSelThreads) {
      const int64_t o = ((int64_t)b * a.T) * a.K + x;
      a.idx_out[o] = -1;
      if (a.val_out) a.val_out[o] = __uint_as_float(kNegInfBits);
    }
  }
}

// Score mode: -inf for the padded pages p >= len[b] of every token row; rows
// are cut into 4096-entry pieces dealt round-robin over the grid.
__device__ __forceinline__ void score_padding(const DecodeArgs& a, const int* s_off, int g, int G) {
  constexpr int kPiece = 4096;
  const int N = a.N, T = a.T;
  const int ppr = (N + kPiece - 1) / kPiece;  // pieces per row
  const int64_t npieces = (int64_t)a.B * T * ppr;
  for (int64_t pc = g; pc < npieces; pc += G) {
    const int rowi = (int)(pc / ppr);
    const int b = rowi / T;
    const int lb = s_off[b + 1] - s_off[b];
    const int p_lo = max(lb, (int)(pc - (int64_t)rowi * ppr) * kPiece);
    const int p_hi = min(N, (int)(pc - (int64_t)rowi * ppr) * kPiece + kPiece);
    float* dst = a.scores + (int64_t)rowi * N;
    for (int p = p_lo + (int)threadIdx.x; p < p_hi; p += kSelThreads)
      dst[p] = __uint_as_float(kNegInfBits);
  }
}

// Valid pages of token t of request b when the call carries per-token
// counts (clamped to [0, N]; an out-of-range value is reported).
__device__ __forceinline__ int tok_length(const DecodeArgs& a, int b, int t) {
  int len = __ldg(a.tok_lengths + (int64_t)b * a.T + t);
  if (len < 0 || len > a.N) {
    if (blockIdx.x == 0) atomicOr(a.status, kErrLengthClamped);
    len = len < 0 ? 0 : a.N;
  }
  return len;
}

// Prefix sums of the clamped request lengths: s_off[b] = first global page of
// request b, s_off[B] = all valid pages (all nthreads threads; s_wsum holds
// one word per warp).  A length outside [0, N] is clamped and reported.
__device__ __forceinline__ void length_prefix(const DecodeArgs& a, int* s_off, uint32_t* s_wsum,
                                              int nthreads) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int running = 0;
  if (tid == 0) {
    s_off[0] = 0;
    s_off[a.B + 1] = 0;  // the longest (clamped) length
  }
  for (int base = 0; base < a.B; base += nthreads) {
    const int i = base + tid;
    int len = 0;
    if (i < a.B) {
      if (a.tok_lengths) {  // a request streams the pages of its longest token row
        for (int t = 0; t < a.T; ++t) len = max(len, tok_length(a, i, t));
      } else {
        len = a.lengths ? a.lengths[i] : a.N;
        if (len < 0 || len > a.N) {
          if (blockIdx.x == 0) atomicOr(a.status, kErrLengthClamped);
          len = len < 0 ? 0 : a.N;
        }
      }
    }
    const uint32_t incl = warp_incl_scan((uint32_t)len);
    const uint32_t wmax = __reduce_max_sync(0xFFFFFFFFu, (uint32_t)len);
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    if (lane == 0) atomicMax(&s_off[a.B + 1], (int)wmax);
    uint32_t excl = incl - (uint32_t)len, total = 0;
    for (int w = 0; w < nthreads / 32; ++w) {
      if (w < warp) excl += s_wsum[w];
      total += s_wsum[w];
    }
    if (i < a.B) s_off[i + 1] = running + (int)excl + len;
    __syncthreads();
    running += (int)total;
  }
}

// Work split of a decode launch.  The valid pages of the batch are laid end
// to end; in fused mode every request is also charged W pages of virtual
// work up front (a segment end costs a select step, which a CTA whose chunk
// ends a request pays while its stream waits), and the resulting virtual
// page range is cut into equal chunks, one per CTA.  Request b occupies the
// virtual range [voff(b), voff(b+1)), its real pages the last len(b) of it.
// Each (chunk, request) piece is a segment; its real pages run from
// snap(b, chunk start) to snap(b, chunk end), both multiples of 32, so the
// arithmetic of a page's score does not depend on how the batch was cut.
struct Chunking {
  const int* s_off;  // prefix sums of the clamped lengths
  int B, W, PV, Lc, nchunks;

  __device__ __forceinline__ int voff(int b) const { return s_off[b] + b * W; }
  __device__ __forceinline__ int len(int b) const { return s_off[b + 1] - s_off[b]; }
  // First request whose virtual range extends past x.
  __device__ __forceinline__ int row(int x) const {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (voff(mid + 1) > x) hi = mid;
      else lo = mid + 1;
    }
    return lo;
  }
  // Real page of request b at virtual position x, snapped down to 32 (or
  // clamped to the row's ends).
  __device__ __forceinline__ int snap(int b, int x) const {
    const int n = len(b);
    const int r = x - voff(b) - W;
    if (r >= n) return n;
    return r <= 0 ? 0 : (r & ~31);
  }
  // Chunks holding a segment of request b (a nonempty page range):
  // first(b) .. last(b).  The chunk holding b's first real page may see
  // fewer than 32 of them, which snap to none; its segment then starts in the
  // next chunk.  With chunks of at least 64 pages every chunk in between
  // holds a nonempty segment.
  __device__ __forceinline__ int first(int b) const {
    const int x = voff(b) + W + min(len(b), 32);  // first virtual end with a real page
    return min((x - 1) / Lc, nchunks - 1);
  }
  __device__ __forceinline__ int last(int b) const { return (voff(b + 1) - 1) / Lc; }
  __device__ __forceinline__ int chunk_begin(int j) const { return j * Lc; }
  __device__ __forceinline__ int chunk_end(int j) const { return min(j * Lc + Lc, PV); }
};

// s_off must be complete (after the barrier that ends length_prefix).
__device__ __forceinline__ Chunking make_chunking(const int* s_off, int B, int G, int W, int lmin) {
  Chunking c;
  c.s_off = s_off;
  c.B = B;
  c.W = W;
  c.PV = s_off[B] + B * W;
  int Lc = (c.PV + G - 1) / G;
  Lc = Lc < lmin ? lmin : Lc;
  c.Lc = Lc < 1 ? 1 : Lc;
  c.nchunks = (c.PV + c.Lc - 1) / c.Lc;
  return c;
}

// The work split of a fused launch: chunks of at least `lmin` pages, and
// long enough that no request is cut into more segments than the merge
// stages at once (kFilterCap entries, at least K from each segment): a
// request of L pages spans at most ceil(L / Lc) + 1 chunks.  s_off[B + 1]
// holds the longest length (length_prefix).
__device__ __forceinline__ Chunking make_fused_chunking(const int* s_off, int B, int G, int W,
                                                        int lmin, int K) {
  int smax = kFilterCap / ((K + 3) & ~3);
  smax = smax < 2 ? 2 : smax;
  const int lk = (s_off[B + 1] + smax - 2) / (smax - 1);
  return make_chunking(s_off, B, G, W, lmin > lk ? lmin : lk);
}

}  // namespace idx
