// select.cuh -- exact block-level top-K machinery (sm_100a).
//
// Ranking.  Every candidate (fp32 bits, index) gets a 64-bit rank value
//     v = (order_key(bits) << 32) | ~index        (0 for -inf, NaN, padding)
// so larger v = better: higher score first, and on equal scores the lower
// index ("Iterate Topk", opening description, with the tie rule of the
// "Round 18 Track C" section 2 adversarial-tie tests).  Rank values are
// unique, so "the top K" is always one well-defined set, whatever order the
// candidates are visited in.
//
// Online filter.  A CTA keeps a candidate buffer in shared memory and a
// threshold thr (initially 0).  Warps offer candidates 32 at a time; one with
// v > thr is appended (warp-aggregated atomic slot).  When the buffer passes
// its high-water mark the CTA compacts it: the K-th largest rank value T is
// found by a radix select over registers (11/11/10-bit digits of the key,
// then of ~index, stopping as soon as the boundary bin is taken whole), the
// entries >= T stay, and thr = T.  Anything offered later with v < T is beaten
// by K kept entries and can never be in the top K, so the filter is exact.
// This is the radix-select family of "Iterate Topk" (8-bit radix seed),
// widened to 11-bit digits, run on a candidate set that the threshold keeps
// small instead of on the whole row.
#pragma once

#include "common.cuh"

namespace idx {

constexpr int kFilterCap = 4096;  // buffer entries per filter (K <= 2048 leaves room)

__device__ __forceinline__ uint64_t rank_value(uint32_t bits, uint32_t index) {
  const uint32_t key = order_key(bits);
  return key ? (((uint64_t)key << 32) | (uint64_t)(~index)) : 0ull;
}

struct SelectScratch {
  uint32_t hist[2][2048];  // passes alternate between the two
  uint32_t wsum[32];
  uint32_t bcast[4];
  int ctr;
  int pad[3];
};

struct FilterState {
  unsigned long long thr;  // accept v > thr
  int count;               // entries in the buffer
  int pad;
};

// Among bins hist[0..NB) find b with suffix(b+1) < r <= suffix(b), where
// suffix(x) = sum_{y >= x} hist[y].  Broadcasts b (bcast[0]), suffix(b+1)
// (bcast[1]) and hist[b] (bcast[2]).  Each thread owns NB/NT consecutive bins
// (thread 0 the top ones), read with 16-byte loads and searched in registers.
template <int NT, int NB>
__device__ __forceinline__ void find_rank_bin(const uint32_t* hist, uint32_t r, SelectScratch& sc) {
  constexpr int BPT = NB / NT;
  static_assert(NB % NT == 0 && BPT % 4 == 0, "bins per thread must be a multiple of 4");
  const int tid = threadIdx.x;
  const int lo = NB - (tid + 1) * BPT;  // this thread's bins: lo .. lo + BPT - 1
  uint32_t h[BPT];
#pragma unroll
  for (int k = 0; k < BPT; k += 4) {
    const uint4 q = *reinterpret_cast<const uint4*>(hist + lo + k);
    h[k] = q.x;
    h[k + 1] = q.y;
    h[k + 2] = q.z;
    h[k + 3] = q.w;
  }
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) s += h[k];
  const uint32_t incl = warp_incl_scan(s);
  const int warp = tid >> 5;
  if (lane_id() == 31) sc.wsum[warp] = incl;
  group_sync(NT);
  uint32_t excl = incl - s;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w)
    if (w < warp) excl += sc.wsum[w];
  if (excl < r && r <= excl + s) {
    uint32_t cum = excl;
    bool found = false;
#pragma unroll
    for (int k = BPT - 1; k >= 0; --k) {  // descending bin order
      if (!found && cum + h[k] >= r) {
        sc.bcast[0] = (uint32_t)(lo + k);
        sc.bcast[1] = cum;
        sc.bcast[2] = h[k];
        found = true;
      }
      cum += h[k];
    }
  }
  group_sync(NT);
}

// The K-th largest of the nonzero values held E per thread by NT threads
// (count of them: n).  Returns T with #{v >= T, v != 0} == min(K, n); when
// n <= K that is T = 1.  Values must be unique.
// The K-th largest of the nonzero values held E per thread by NT threads
// (count of them: n).  Returns T with #{v >= T, v != 0} == min(K, n); when
// n <= K that is T = 1.  Values must be unique.  Both histograms of sc must be
// zero on entry (filter_compact clears them under its first barrier); a pass
// leaves its histogram dirty and pass p uses hist[p & 1], re-cleared when a
// third pass is needed.
template <int NT, int E>
__device__ uint64_t block_kth_largest(const uint64_t (&v)[E], int K, int n, SelectScratch& sc) {
  if (n <= K) return 1ull;
  const int tid = threadIdx.x;
  const int nk = (n + NT - 1) / NT;  // register slots in use (uniform)
  uint64_t prefix = 0;
  uint32_t r = (uint32_t)K;
  int shift = 64;
#pragma unroll 1
  for (int p = 0; p < 6; ++p) {
    const int w = (p == 2 || p == 5) ? 10 : 11;
    shift -= w;
    const uint32_t mask = (1u << w) - 1u;
    uint32_t* hist = sc.hist[p & 1];
    if (p >= 2) {  // the histogram was used two passes ago
      for (int i = tid; i < 2048; i += NT) hist[i] = 0u;
      group_sync(NT);
    }
#pragma unroll
    for (int k = 0; k < E; ++k) {
      if (k >= nk) break;
      const uint64_t x = v[k];
      const bool match = x != 0 && (p == 0 || (x >> (shift + w)) == prefix);
      if (match) atomicAdd(&hist[(uint32_t)(x >> shift) & mask], 1u);
    }
    group_sync(NT);
    if (w == 11) find_rank_bin<NT, 2048>(hist, r, sc);
    else find_rank_bin<NT, 1024>(hist, r, sc);
    const uint32_t b = sc.bcast[0];
    const uint32_t above = sc.bcast[1];
    const uint32_t cnt = sc.bcast[2];
    r -= above;
    prefix = (prefix << w) | b;
    if (cnt == r) return prefix << shift;  // the boundary bin is taken whole
  }
  return prefix;  // shift == 0: T is the exact K-th value
}

__device__ __forceinline__ void filter_reset(FilterState& fs) {
  fs.thr = 0ull;
  fs.count = 0;
}

// One warp offers 32 candidates (one per lane).  All lanes call it.
__device__ __forceinline__ void filter_offer(FilterState& fs, uint32_t* fb, uint32_t* fi,
                                             uint32_t bits, uint32_t index, bool valid) {
  const uint64_t v = valid ? rank_value(bits, index) : 0ull;
  const bool take = v > fs.thr;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
  if (m) {
    const int leader = __ffs(m) - 1;
    int base = 0;
    if ((int)lane_id() == leader) base = atomicAdd(&fs.count, __popc(m));
    base = __shfl_sync(0xFFFFFFFFu, base, leader);
    if (take) {
      const int pos = base + __popc(m & lanemask_lt());
      fb[pos] = bits;
      fi[pos] = index;
    }
  }
}

// filter_offer without the warp vote: each lane that beats the threshold
// claims its own slot.  Cheaper once the threshold rejects most offers (no
// warp-wide step for the lanes that append nothing); lanes need not call it
// together.
__device__ __forceinline__ void filter_offer_lane(FilterState& fs, uint32_t* fb, uint32_t* fi,
                                                  uint32_t bits, uint32_t index, bool valid) {
  const uint64_t v = valid ? rank_value(bits, index) : 0ull;
  if (v > fs.thr) {
    const int pos = atomicAdd(&fs.count, 1);
    fb[pos] = bits;
    fi[pos] = index;
  }
}

// Keep only the top K of the buffer (all NT threads; every offer made before
// the call must be complete, i.e. the caller syncs the group first).
template <int NT>
__device__ void filter_compact(FilterState& fs, uint32_t* fb, uint32_t* fi, int K,
                               SelectScratch& sc) {
  constexpr int E = kFilterCap / NT;
  const int tid = threadIdx.x;
  const int n = fs.count;
  if (n <= K) return;  // uniform: n was read after the caller's barrier
  const int nk = (n + NT - 1) / NT;  // register slots in use (uniform)
  uint64_t v[E];
  uint32_t bb[E];
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = tid + k * NT;
    bb[k] = 0u;
    v[k] = 0ull;
    if (k < nk && i < n) {
      bb[k] = fb[i];
      v[k] = rank_value(bb[k], fi[i]);
    }
  }
  if (tid == 0) sc.ctr = 0;
  for (int i = tid; i < 2 * 2048; i += NT) (&sc.hist[0][0])[i] = 0u;
  group_sync(NT);  // all entries are in registers; the buffer may be rewritten
  IDX_TRACE(0);
  const uint64_t T = block_kth_largest<NT, E>(v, K, n, sc);
  IDX_TRACE(1);
#pragma unroll
  for (int k = 0; k < E; ++k) {
    if (k >= nk) break;
    const bool win = v[k] != 0 && v[k] >= T;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, win);
    if (m) {
      const int leader = __ffs(m) - 1;
      int base = 0;
      if ((int)lane_id() == leader) base = atomicAdd(&sc.ctr, __popc(m));
      base = __shfl_sync(0xFFFFFFFFu, base, leader);
      if (win) {
        const int pos = base + __popc(m & lanemask_lt());
        fb[pos] = bb[k];
        fi[pos] = ~(uint32_t)v[k];
      }
    }
  }
  group_sync(NT);
  if (tid == 0) {
    fs.count = sc.ctr;
    fs.thr = T;
  }
  group_sync(NT);
  IDX_TRACE(2);
}

// One compare-exchange of a bitonic network between this lane's entry (x, xb)
// at network position p and the partner lane (lane ^ s) in the same warp.
__device__ __forceinline__ void cmpx_lane(uint64_t& x, uint32_t& xb, int p, int s, int size) {
  const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, x, s);
  const uint32_t yb = __shfl_xor_sync(0xFFFFFFFFu, xb, s);
  const bool lower = (p & s) == 0;
  const bool desc = (p & size) == 0;
  const bool want_larger = (lower == desc);
  if (want_larger ? (y > x) : (y < x)) {
    x = y;
    xb = yb;
  }
}

// Compare-exchange of the two entries a thread holds (positions p and p + 32).
__device__ __forceinline__ void cmpx_pair(uint64_t& a, uint32_t& ab, uint64_t& b, uint32_t& bbits,
                                          int p, int size) {
  const bool desc = (p & size) == 0;
  if (desc ? (b > a) : (a > b)) {
    const uint64_t t = a;
    a = b;
    b = t;
    const uint32_t tb = ab;
    ab = bbits;
    bbits = tb;
  }
}

// Bitonic sort (descending) of sv/sb[0..P2), P2 a power of two >= 64.  Warp w
// owns 64-entry blocks w, w + NT/32, ...; every stage of stride <= 32 runs in
// registers (shuffles and in-thread swaps, no barrier); only strides >= 64
// go through shared memory with a barrier per stage.
template <int NT>
__device__ void block_bitonic_desc(uint64_t* sv, uint32_t* sb, int P2) {
  constexpr int NW = NT / 32;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto local_stages = [&](int size_lo, int size_hi, int first_stride) {
    for (int blk = warp; blk * 64 < P2; blk += NW) {
      const int base = blk * 64;
      uint64_t a = sv[base + lane], b = sv[base + lane + 32];
      uint32_t ab = sb[base + lane], bbits = sb[base + lane + 32];
      for (int size = size_lo; size <= size_hi; size <<= 1) {
        int stride = size == size_lo ? first_stride : (size >> 1);
        if (stride > 32) stride = 32;
        for (; stride > 0; stride >>= 1) {
          if (stride == 32) {
            cmpx_pair(a, ab, b, bbits, base + lane, size);
          } else {
            cmpx_lane(a, ab, base + lane, stride, size);
            cmpx_lane(b, bbits, base + lane + 32, stride, size);
          }
        }
      }
      sv[base + lane] = a;
      sv[base + lane + 32] = b;
      sb[base + lane] = ab;
      sb[base + lane + 32] = bbits;
    }
    group_sync(NT);
  };
  local_stages(2, 64, 1);  // every size up to 64 stays inside a block
  for (int size = 128; size <= P2; size <<= 1) {
    for (int stride = size >> 1; stride >= 64; stride >>= 1) {
      for (int i = threadIdx.x; i < (P2 >> 1); i += NT) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t x = sv[lo], y = sv[hi];
        if ((x < y) == desc) {
          sv[lo] = y;
          sv[hi] = x;
          const uint32_t t = sb[lo];
          sb[lo] = sb[hi];
          sb[hi] = t;
        }
      }
      group_sync(NT);
    }
    local_stages(size, size, 32);
  }
}

// Sort the kk buffer entries by rank value (descending) and write the first K
// as one output row: idx_out[k] = index, val_out[k] = the entry's exact fp32
// bits; slots past kk get -1 / -inf.  sv / sb hold max(64, next_pow2(K)) + 1
// entries.  Up to 2*NT entries are placed by counting (the rank of an entry is
// how many rank values exceed it -- they are unique -- and only ranks < K are
// written), which needs two barriers; more entries (then kk <= K) go through
// the bitonic network.
template <int NT>
__device__ void sort_and_write(const uint32_t* fb, const uint32_t* fi, int kk, int K,
                               uint64_t* sv, uint32_t* sb, int32_t* idx_out, float* val_out) {
  const int tid = threadIdx.x;
  if (kk <= 2 * NT) {
    for (int i = tid; i <= kk; i += NT) sv[i] = i < kk ? rank_value(fb[i], fi[i]) : 0ull;
    group_sync(NT);
    const uint64_t v0 = tid < kk ? sv[tid] : 0ull;
    const uint64_t v1 = tid + NT < kk ? sv[tid + NT] : 0ull;
    uint32_t r0 = 0, r1 = 0;
    const int kk2 = (kk + 1) & ~1;
    if (kk <= NT) {
#pragma unroll 8
      for (int j = 0; j < kk2; j += 2) {
        const ulonglong2 u = *reinterpret_cast<const ulonglong2*>(sv + j);
        r0 += (u.x > v0) + (u.y > v0);
      }
    } else {
#pragma unroll 8
      for (int j = 0; j < kk2; j += 2) {
        const ulonglong2 u = *reinterpret_cast<const ulonglong2*>(sv + j);
        r0 += (u.x > v0) + (u.y > v0);
        r1 += (u.x > v1) + (u.y > v1);
      }
    }
    if (tid < kk && r0 < (uint32_t)K) {
      idx_out[r0] = (int32_t)~(uint32_t)v0;
      if (val_out) val_out[r0] = __uint_as_float(fb[tid]);
    }
    if (tid + NT < kk && r1 < (uint32_t)K) {
      idx_out[r1] = (int32_t)~(uint32_t)v1;
      if (val_out) val_out[r1] = __uint_as_float(fb[tid + NT]);
    }
    for (int k = min(kk, K) + tid; k < K; k += NT) {
      idx_out[k] = -1;
      if (val_out) val_out[k] = __uint_as_float(kNegInfBits);
    }
    group_sync(NT);
    return;
  }
  int P2 = 64;
  while (P2 < kk) P2 <<= 1;
  for (int i = tid; i < P2; i += NT) {
    sv[i] = i < kk ? rank_value(fb[i], fi[i]) : 0ull;
    sb[i] = i < kk ? fb[i] : 0u;
  }
  group_sync(NT);
  block_bitonic_desc<NT>(sv, sb, P2);
  for (int k = tid; k < K; k += NT) {
    if (k < kk) {
      idx_out[k] = (int32_t)~(uint32_t)sv[k];
      if (val_out) val_out[k] = __uint_as_float(sb[k]);
    } else {
      idx_out[k] = -1;
      if (val_out) val_out[k] = __uint_as_float(kNegInfBits);
    }
  }
  group_sync(NT);
}

// Publish a range's kk <= K winners as one candidate list of exactly K entries
// (unused entries invalid: -inf, index -1), so a merger can fetch every list
// without reading a count first.  A nonzero filter threshold thr is a lower
// bound of the range's K-th rank value, hence of its row's: it raises the
// row's shared threshold (atomic max), which the merger uses to drop
// candidates early.
template <int NT>
__device__ void publish_candidates(const uint32_t* fb, const uint32_t* fi, int kk, int K,
                                   uint64_t thr, uint32_t* cbits, int32_t* cidx,
                                   unsigned long long* row_thr) {
  for (int k = threadIdx.x; k < K; k += NT) {
    cbits[k] = k < kk ? fb[k] : kNegInfBits;
    cidx[k] = k < kk ? (int32_t)fi[k] : -1;
  }
  if (threadIdx.x == 0 && thr != 0) atomicMax(row_thr, (unsigned long long)thr);
}

// Merge nslots published lists (list i at bits/index + slot_of(i) * stride,
// L entries each, unused entries invalid) into one final row of K.  All lists are fetched with every
// thread's loads in flight together; entries below the row threshold are
// dropped on arrival; the survivors are placed by the counting sort when few
// enough remain, else compacted first.  Resets *row_thr to zero for the next
// call.  fb/fi is a filter buffer of cap >= K + NT * 8 entries.
template <int NT, class SlotOf>
__device__ void merge_candidates(int nslots, SlotOf slot_of, const uint32_t* cand_bits,
                                 const int32_t* cand_idx, int64_t stride, int L, int K,
                                 unsigned long long* row_thr, FilterState& fs, uint32_t* fb,
                                 uint32_t* fi, int cap, SelectScratch& sc, uint64_t* sv,
                                 uint32_t* sb, int32_t* idx_out, float* val_out) {
  constexpr int U = 8;
  const int tid = threadIdx.x;
  IDX_TRACE(7);
  if (tid == 0) {
    const unsigned long long t = __ldcg(row_thr);
    fs.thr = t ? t - 1 : 0ull;  // keep v >= t
    fs.count = 0;
    *row_thr = 0ull;
  }
  group_sync(NT);
  const int total = nslots * L;
  for (int f0 = 0; f0 < total; f0 += NT * U) {
    uint32_t bits[U], index[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int f = f0 + u * NT + tid;
      bits[u] = kNegInfBits;
      index[u] = 0xFFFFFFFFu;
      if (f < total) {
        const int i = f / L;
        const int e = f - i * L;
        const int64_t off = slot_of(i) * stride + e;
        bits[u] = __ldcg(cand_bits + off);
        index[u] = (uint32_t)__ldcg(cand_idx + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) filter_offer(fs, fb, fi, bits[u], index[u], index[u] != 0xFFFFFFFFu);
    group_sync(NT);
    // every thread reads the count before anyone offers again: one decision
    const int n = fs.count;
    group_sync(NT);
    if (n > cap - NT * U) filter_compact<NT>(fs, fb, fi, K, sc);
  }
  IDX_TRACE(3);
  if (fs.count > 2 * NT) filter_compact<NT>(fs, fb, fi, K, sc);
  IDX_TRACE(4);
  sort_and_write<NT>(fb, fi, fs.count, K, sv, sb, idx_out, val_out);
  IDX_TRACE(5);
}

// All threads of the group: count one arrival on *counter once this CTA's
// global stores are visible GPU-wide.  Returns true (to every thread) in the
// CTA that arrives last (the expected-th arrival), which also resets the
// counter to zero.  The barrier orders every thread's stores before thread
// 0's arrival, a GPU-scope acquire-release atomic: its release half publishes
// them (release is cumulative over what the barrier ordered before it), its
// acquire half orders the other CTAs' published stores before this CTA's
// later reads, which the second barrier extends to every thread.
template <int NT>
__device__ bool arrive_last(int32_t* counter, int expected, int* s_flag) {
  group_sync(NT);
  if (threadIdx.x == 0) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(old) : "l"(counter) : "memory");
    const bool last = old == expected - 1;
    if (last) *counter = 0;  // no CTA of this launch touches it again
    *s_flag = last;
  }
  group_sync(NT);
  return *s_flag != 0;
}

}  // namespace idx
