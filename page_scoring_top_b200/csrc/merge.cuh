// merge.cuh -- exact merge of per-range top-K candidate lists (last CTA of a row).
//
// Every range of a row publishes its own exact top-K' (value, index) list, in
// index order.  The row's top-K is contained in the union of those lists: an
// entry beaten by fewer than K entries of its row is beaten by fewer than K
// entries of its own range.  The merge concatenates the lists in range order
// (so buffer position order is index order, which keeps "equal scores go to
// the lower index" exact), selects, and compacts in rounds when the lists do
// not fit the buffer at once.
#pragma once

#include "common.cuh"

namespace idx {

// Move the winners s_bits[win_pos[k]], s_idx[win_pos[k]] (k < kk, ascending
// positions) to the front of the buffers, keeping their order.
template <int NT>
__device__ void compact_front(uint32_t* s_bits, int32_t* s_idx, const int* win_pos, int kk) {
  constexpr int PER = (2048 + NT - 1) / NT;  // kk <= IDX_MAX_K = 2048
  uint32_t rb[PER];
  int32_t ri[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int k = threadIdx.x + u * NT;
    if (k < kk) {
      rb[u] = s_bits[win_pos[k]];
      ri[u] = s_idx[win_pos[k]];
    }
  }
  group_sync(NT);
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int k = threadIdx.x + u * NT;
    if (k < kk) {
      s_bits[k] = rb[u];
      s_idx[k] = ri[u];
    }
  }
  group_sync(NT);
}

// Merge nslots candidate lists (slot i: cnt[slot_of(i)] entries at
// bits/idx + slot_of(i) * stride) into the final row.  cap >= 2 * K.
template <int NT, class SlotOf>
__device__ void merge_candidates(int nslots, SlotOf slot_of, const uint32_t* cand_bits,
                                 const int32_t* cand_idx, const int32_t* cand_cnt,
                                 int64_t stride, int K, int cap, uint32_t* s_bits, int32_t* s_idx,
                                 int* win_pos, SelectScratch& sc, uint64_t* sortbuf,
                                 int32_t* idx_out, float* val_out) {
  int have = 0;
  int next = 0;
  for (;;) {
    int fill = have;
    while (next < nslots) {
      const int64_t slot = slot_of(next);
      int cnt = __ldcg(cand_cnt + slot);
      cnt = cnt < 0 ? 0 : (cnt > K ? K : cnt);  // a published count is <= K
      if (fill + cnt > cap) break;
      const uint32_t* sb = cand_bits + slot * stride;
      const int32_t* si = cand_idx + slot * stride;
      for (int k = threadIdx.x; k < cnt; k += NT) {
        s_bits[fill + k] = __ldcg(sb + k);
        s_idx[fill + k] = __ldcg(si + k);
      }
      fill += cnt;
      ++next;
    }
    group_sync(NT);
    const int kk = block_select<NT>(s_bits, fill, K, win_pos, sc);
    if (next >= nslots) {
      sort_and_write<NT>(s_bits, s_idx, 0, win_pos, kk, K, sortbuf, idx_out, val_out);
      return;
    }
    compact_front<NT>(s_bits, s_idx, win_pos, kk);
    have = kk;
  }
}

// All threads of the group: publish this CTA's stores, then count one arrival
// on *counter.  Returns true (to every thread) in the CTA that arrives last
// (the expected-th arrival); that CTA also resets the counter to zero.
template <int NT>
__device__ bool arrive_last(int32_t* counter, int expected, int* s_flag) {
  __threadfence();
  group_sync(NT);
  if (threadIdx.x == 0) {
    const int old = atomicAdd(counter, 1);
    *s_flag = (old == expected - 1);
  }
  group_sync(NT);
  const bool last = *s_flag != 0;
  if (last) {
    __threadfence();
    if (threadIdx.x == 0) *counter = 0;
  }
  group_sync(NT);
  return last;
}

}  // namespace idx
