// topk_stream.cu -- standalone exact top-K over fp32 score rows, streamed.
//
// What is computed ("Iterate Topk", opening description: given per-segment
// scores, return the top-K indices): for every row r, the K positions of
// largest score among its first len[r] entries, by descending score, equal
// scores to the lower position ("Round 18 Track C", section 2 ties), -inf and
// NaN never selected.
//
// One persistent CTA per SM, the work split of the fused decode kernels
// (fused.cuh): the valid entries of all rows are laid end to end, each row is
// also charged kTsRowCharge virtual entries for its segment-end select, and
// the range is cut into one equal chunk per CTA; a (chunk, row) piece is a
// segment.
//  * warp 8, the producer: 32 KB stages of a segment, 1-D bulk copies (TMA
//    engine) into a 4-stage ring, stages of a segment visited in bit-reversed
//    order (a row sorted either way then raises the threshold early; the
//    consumers walk the same order).  Four lanes issue, stage k by lane k % 4.
//  * warps 0-7 consume each stage together: every thread offers 32 scores
//    (eight 16-byte shared-memory reads) to the single-token online filter
//    of fused.cuh, whose digit histogram raises the threshold while the
//    stream runs (and shares it with the other CTAs of the row).  A score
//    that passes the threshold while the buffer is full is kept back (a bit
//    per score); one barrier per stage finds whether any was, and only then
//    does the CTA compact its buffer and offer those scores again, from the
//    stage still in the ring.  At a
//    segment end the filter's exact ordered top K is written (whole row in
//    the chunk) or its candidates published for the last CTA of the row to
//    merge (hist_finalize).
// Every score is read from HBM once; the scores of a row's ragged end that
// do not fill 16 bytes are read by the consumers directly.
#include "common.cuh"
#include "fused.cuh"
#include "kernels.h"

namespace idx {

namespace {

constexpr int kTsConsumerWarps = 8;
constexpr int kTsConsumers = kTsConsumerWarps * 32;
static_assert(kTsConsumers == kSelThreads, "the consumer warps run the select steps");
constexpr int kTsThreads = kTsConsumers + 32;
constexpr int kTsStage = 8192;  // scores per stage (32 KB)
constexpr int kTsStages = 4;
constexpr int kTsLanes = 4;       // producer lanes
constexpr int kTsRound = kTsConsumers * 4;  // scores per offer round (16 bytes a thread)
constexpr int kTsRowCharge = 49152;  // virtual scores charged per row (a segment-end select and merge)
constexpr int kTsLMin = kTsStage;    // smallest chunk
constexpr int kTsMaxRows = kDecodeMaxB;
constexpr int kTsMaxSegments = 8;    // CTAs per row, for the launch's grid

__host__ __device__ inline size_t ts_al16(size_t x) { return (x + 15) & ~(size_t)15; }

struct TsLayout {
  size_t bars, misc, off, fbuf, fstate, scratch, sortv, sortb, hist, ring, total;
};

__host__ __device__ inline TsLayout ts_layout() {
  TsLayout L;
  size_t o = 0;
  L.bars = o;  // full[4], empty[4]
  o += 64;
  L.misc = o;  // abort, arrival flag, -, overflow flag, warp sums, [14] polled row threshold
  o += 64;
  L.off = o;
  o += ts_al16((size_t)(kTsMaxRows + 1) * 4);
  L.fbuf = o;
  o += (size_t)kFilterCap * 8;
  L.fstate = o;
  o += 16;
  L.scratch = o;
  o += ts_al16(sizeof(SelectScratch));
  L.sortv = o;
  o += (size_t)(kMaxK + 2) * 8;
  L.sortb = o;
  o += (size_t)(kMaxK + 4) * 4;
  L.hist = o;
  o += (size_t)(kHBins + kHCoarse) * 4;
  o = (o + 127) & ~(size_t)127;
  L.ring = o;
  o += (size_t)kTsStages * kTsStage * 4;
  L.total = o;
  return L;
}

// The float whose order key is the key half of a filter threshold (-inf for
// a zero threshold): every score that can pass the threshold is >= it.
__device__ __forceinline__ float thr_key_float(unsigned long long thr) {
  const uint32_t k = (uint32_t)(thr >> 32);
  if (k == 0u) return __uint_as_float(kNegInfBits);
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

__device__ __forceinline__ uint32_t ts_bitrev(uint32_t x, int bits) {
  return bits ? (__brev(x) >> (32 - bits)) : 0u;
}

// Stage q of a segment of n scores in visiting order: the bit-reversed
// permutation of 0 .. 2^bits - 1 with indices past the stage count skipped.
struct StageOrder {
  int nst, bits, seq;
  __device__ void init(int n) {
    nst = (n + kTsStage - 1) / kTsStage;
    bits = 0;
    while ((1 << bits) < nst) ++bits;
    seq = 0;
  }
  __device__ int next() {
    while (seq < (1 << bits)) {
      const int s = (int)ts_bitrev((uint32_t)seq++, bits);
      if (s < nst) return s;
    }
    return -1;
  }
};

// Prefix sums of the clamped row lengths (all nthreads threads); a length
// outside [0, N] is clamped and reported.
__device__ void ts_row_prefix(const TopkStreamArgs& a, int* s_off, uint32_t* s_wsum, int nthreads) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int running = 0;
  if (tid == 0) s_off[0] = 0;
  for (int base = 0; base < a.rows; base += nthreads) {
    const int i = base + tid;
    int len = 0;
    if (i < a.rows) {
      len = a.lengths ? a.lengths[i / a.len_div] : a.N;
      if (len < 0 || len > a.N) {
        if (blockIdx.x == 0) atomicOr(a.status, kErrLengthClamped);
        len = len < 0 ? 0 : a.N;
      }
    }
    const uint32_t incl = warp_incl_scan((uint32_t)len);
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    uint32_t excl = incl - (uint32_t)len, total = 0;
    for (int w = 0; w < nthreads / 32; ++w) {
      if (w < warp) excl += s_wsum[w];
      total += s_wsum[w];
    }
    if (i < a.rows) s_off[i + 1] = running + (int)excl + len;
    __syncthreads();
    running += (int)total;
  }
}

__global__ void __launch_bounds__(kTsThreads, 1) topk_stream_kernel(const TopkStreamArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const TsLayout L = ts_layout();
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kTsStages;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  volatile int* s_abort = misc;
  volatile int* s_over = misc + 3;  // a score found the buffer full this stage
  uint32_t* s_wsum = reinterpret_cast<uint32_t*>(misc + 4);  // 9 warp sums
  int* s_off = reinterpret_cast<int*>(smem + L.off);
  float* ring = reinterpret_cast<float*>(smem + L.ring);
  const FusedSel fsel{reinterpret_cast<uint32_t*>(smem + L.fbuf),
                      reinterpret_cast<FilterState*>(smem + L.fstate),
                      reinterpret_cast<SelectScratch*>(smem + L.scratch),
                      reinterpret_cast<uint64_t*>(smem + L.sortv),
                      reinterpret_cast<uint32_t*>(smem + L.sortb),
                      reinterpret_cast<uint32_t*>(smem + L.hist),
                      kFilterCap,
                      misc + 1,
                      reinterpret_cast<uint32_t*>(misc + 14)};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < kTsStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kTsConsumerWarps);  // one arrival per consumer warp
    }
    *s_abort = 0;
    *s_over = 0;
    fence_mbar_init();
  }
  ts_row_prefix(a, s_off, s_wsum, kTsThreads);
  __syncthreads();
  const Chunking ch = make_chunking(s_off, a.rows, G, kTsRowCharge, kTsLMin);
  const int nchunks = ch.nchunks;

  if (warp == kTsConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane < kTsLanes) {
      const uint64_t pol = policy_evict_first();
      uint32_t stage = 0;
      int64_t last = -1;  // last stage this lane filled
      for (int j = g; j < nchunks; j += G) {
        const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
        const int b_last = ch.row(ce - 1);
        for (int b = ch.row(cb); b <= b_last; ++b) {
          if (ch.len(b) == 0) continue;
          const int p0 = ch.snap(b, cb);
          const int n = ch.snap(b, ce) - p0;
          if (n <= 0) continue;
          const float* src = a.scores + (int64_t)b * a.lds + p0;
          StageOrder order;
          order.init(n);
          for (int s = order.next(); s >= 0; s = order.next(), ++stage) {
            if ((int)(stage % kTsLanes) != lane) continue;
            const int slot = (int)(stage % kTsStages);
            const uint32_t round = stage / kTsStages;
            if (round > 0) mbar_wait_bounded(&empty[slot], (round - 1) & 1, s_abort, a.status);
            if (*s_abort) continue;
            const int o = s * kTsStage;
            const int cnt = min(kTsStage, n - o);
            const int n4 = cnt & ~3;  // whole 16-byte groups (the rest is read directly)
            if (n4 > 0) {
              mbar_arrive_expect_tx(&full[slot], (uint32_t)n4 * 4u);
              bulk_g2s(ring + (size_t)slot * kTsStage, src + o, (uint32_t)n4 * 4u, &full[slot], pol);
            } else {
              mbar_arrive(&full[slot]);
            }
            last = stage;
          }
        }
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int64_t t = last; t >= 0 && t > last - kTsStages; t -= kTsLanes)
        mbar_wait_drain(&full[t % kTsStages], (uint32_t)(t / kTsStages) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  IDX_TRACE(10);
  // rows with no valid score: all-padding output (rows dealt round-robin)
  for (int b = g; b < a.rows; b += G) {
    if (s_off[b + 1] != s_off[b]) continue;
    for (int x = tid; x < a.K; x += kTsConsumers) {
      a.idx_out[(int64_t)b * a.K + x] = -1;
      if (a.val_out) a.val_out[(int64_t)b * a.K + x] = __uint_as_float(kNegInfBits);
    }
  }
  const RowOut out{a.idx_out, a.val_out, a.K, a.cand_bits, a.cand_idx, a.slot_stride,
                   a.row_thr, a.arrive};
  uint32_t stage = 0;
  for (int j = g; j < nchunks; j += G) {
    const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
    const int b_last = ch.row(ce - 1);
    for (int b = ch.row(cb); b <= b_last; ++b) {
      if (ch.len(b) == 0) continue;
      const int p0 = ch.snap(b, cb);
      const int n = ch.snap(b, ce) - p0;
      if (n <= 0) continue;
      fused_begin<true>(fsel, 1);
      group_sync(kTsConsumers);
      const float* rowp = a.scores + (int64_t)b * a.lds;
      StageOrder order;  // the producer's order
      order.init(n);
      FilterState& fs = fsel.fst[0];
      bool first = true;  // the segment's first stage (in visiting order)
      for (int s = order.next(); s >= 0; s = order.next(), ++stage) {
        const int slot = (int)(stage % kTsStages);
        mbar_wait_bounded(&full[slot], (stage / kTsStages) & 1, s_abort, a.status);
        IDX_TRACE(40);
        const int o = p0 + s * kTsStage;
        const int cnt = min(kTsStage, n - s * kTsStage), n4 = cnt & ~3;
        const float4* sb = reinterpret_cast<const float4*>(ring + (size_t)slot * kTsStage);
        // score k of round r of this thread: stage position 4 (256 r + tid) + k
        auto load4 = [&](int r, uint32_t (&w)[4]) {
          const int e0 = (r * kTsConsumers + tid) * 4;
          if (e0 + 4 <= n4) {
            const float4 x = sb[r * kTsConsumers + tid];
            w[0] = __float_as_uint(x.x);
            w[1] = __float_as_uint(x.y);
            w[2] = __float_as_uint(x.z);
            w[3] = __float_as_uint(x.w);
          } else {
            // the row's ragged end, not in the copied 16-byte groups
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w[k] = e0 + k < cnt ? __float_as_uint(__ldg(rowp + o + e0 + k)) : kNegInfBits;
          }
        };
        // Offer scores to the filter; a score that passes the threshold but
        // finds the buffer full is remembered in `failed` (one bit per score).
        // score k of round r (bits w) against the current threshold
        auto offer_one = [&](int r, int k, uint32_t w, uint32_t& failed) {
          const unsigned long long thr = *reinterpret_cast<volatile unsigned long long*>(&fs.thr);
          const uint32_t thi = (uint32_t)(thr >> 32), tlo = (uint32_t)thr;
          const uint32_t key = order_key(w);
          const uint32_t index = (uint32_t)(o + (r * kTsConsumers + tid) * 4 + k);
          if (key != 0u && (key > thi || (key == thi && ~index > tlo))) {
            const int pos = atomicAdd(&fs.count, 1);
            if (pos < fsel.cap) {
              fsel.fbuf[pos] = w;
              fsel.fbuf[fsel.cap + pos] = index;
              const uint32_t d = key >> kHShift;
              atomicAdd(&fsel.hist[d], 1u);
              atomicAdd(&fsel.hist[kHBins + (d >> 5)], 1u);
            } else {
              failed |= 1u << (4 * r + k);
            }
          }
        };
        auto offer = [&](int r, const uint32_t (&w)[4], uint32_t mask, uint32_t& failed) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (mask >> k & 1u) offer_one(r, k, w[k], failed);
        };
        const int nrounds = (cnt + kTsRound - 1) / kTsRound;
        uint32_t failed = 0;
        // Fast rejection: a score can pass the threshold only if its order
        // key reaches the threshold's key half, i.e. (order keys being
        // monotone) only if it is >= that key's float.  Four scores cost one
        // 16-byte read, three max and one compare; the few that pass take
        // the exact offer.  The threshold is read once a stage (a stale one
        // is lower, so it only lets more through).
        const unsigned long long thr_now = *reinterpret_cast<volatile unsigned long long*>(&fs.thr);
        float tf = thr_key_float(thr_now);
        // a score equal to tf (its key the threshold's key half) passes only
        // below this index (ties go to the lower index)
        uint32_t ilim = ~(uint32_t)thr_now;
        {
          // All 32 scores first (a bit per score that may pass), then the
          // exact offers of the few that may: a warp walks the slow path
          // once a stage, not once for every 16 bytes that one lane needs.
          // A partial stage reads its ragged end directly; missing scores
          // are -inf.
          static_assert(kTsStage / kTsRound * 4 == 32, "a bit per score of a stage");
          float4 x[kTsStage / kTsRound];
          if (cnt == kTsStage) {
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r) x[r] = sb[r * kTsConsumers + tid];
          } else {
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r) {
              uint32_t w[4];
              load4(r, w);
              x[r] = make_float4(__uint_as_float(w[0]), __uint_as_float(w[1]),
                                 __uint_as_float(w[2]), __uint_as_float(w[3]));
            }
          }
          if (first && n > kTsStage) {
            // A segment of several stages starts from a threshold before its
            // first offer: the digit of the first stage's K-th largest score,
            // from the stage's own digit histogram (counted into the filter's,
            // still empty, then cleared again).  Every score of the stage's
            // top K is at or above that digit's floor, so the floor is <= the
            // segment's K-th largest.  Without it the first stages would fill
            // the buffer and force compactions.
            uint32_t* hh = fsel.hist;
            uint32_t* hc = fsel.hist + kHBins;
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r) {
              const uint32_t kk[4] = {order_key(__float_as_uint(x[r].x)), order_key(__float_as_uint(x[r].y)),
                                      order_key(__float_as_uint(x[r].z)), order_key(__float_as_uint(x[r].w))};
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if (kk[k] != 0u && (r * kTsConsumers + tid) * 4 + k < cnt) {
                  const uint32_t d = kk[k] >> kHShift;
                  atomicAdd(&hh[d], 1u);
                  atomicAdd(&hc[d >> 5], 1u);
                }
            }
            group_sync(kTsConsumers);
            if (warp == 0) {
              const uint32_t bfl = hist_floor_warp(hh, hc, (uint32_t)a.K);
              if (lane == 0) s_wsum[0] = bfl;
            }
            group_sync(kTsConsumers);
            const uint32_t bfl = s_wsum[0];
            hist_clear<kTsConsumers>(hh, hc);
            group_sync(kTsConsumers);
            if (bfl != 0u) {
              const unsigned long long t = ((unsigned long long)bfl << (32 + kHShift)) - 1ull;
              tf = thr_key_float(t);
              ilim = 0u;
              if (tid == 0 && t > fs.thr) fs.thr = t;
            }
            first = false;
          } else if (first) {
            // A one-stage segment takes a cheaper starting threshold: cut the
            // stage into at least K groups (gp groups of 32 / gp scores a thread); every
            // group's maximum is a distinct score, so the smallest group
            // maximum is <= the segment's K-th largest.  Without it the
            // first stage would fill the buffer and force a compaction.
            const int gp = a.K <= 256 ? 1 : a.K <= 512 ? 2 : a.K <= 1024 ? 4 : 8;
            uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r) {
              gmax = max(gmax, max(max(order_key(__float_as_uint(x[r].x)),
                                       order_key(__float_as_uint(x[r].y))),
                                   max(order_key(__float_as_uint(x[r].z)),
                                       order_key(__float_as_uint(x[r].w)))));
              // a group ends every 8 / gp rounds
              if (((r + 1) * gp) % (kTsStage / kTsRound) == 0) {
                gmin = min(gmin, gmax);
                gmax = 0u;
              }
            }
            gmin = __reduce_min_sync(0xFFFFFFFFu, gmin);
            if (lane == 0) s_wsum[warp] = gmin;
            group_sync(kTsConsumers);
#pragma unroll
            for (int w = 0; w < kTsConsumerWarps; ++w) gmin = min(gmin, s_wsum[w]);
            if (gmin != 0u) {  // every group holds a valid score
              const unsigned long long t = ((unsigned long long)gmin << 32) - 1ull;
              tf = thr_key_float(t);
              ilim = 0u;
              if (tid == 0 && t > fs.thr) fs.thr = t;
            }
            first = false;
          }
          uint32_t maybe = 0;
          if ((uint32_t)o >= ilim) {
            // no score of the stage that ties the threshold's key can pass
            // (heavy ties would otherwise all take the exact offer)
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r)
              maybe |= ((uint32_t)(x[r].x > tf) | (uint32_t)(x[r].y > tf) << 1 |
                        (uint32_t)(x[r].z > tf) << 2 | (uint32_t)(x[r].w > tf) << 3)
                       << (4 * r);
          } else {
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r)
              maybe |= ((uint32_t)(x[r].x >= tf) | (uint32_t)(x[r].y >= tf) << 1 |
                        (uint32_t)(x[r].z >= tf) << 2 | (uint32_t)(x[r].w >= tf) << 3)
                       << (4 * r);
          }
          if (cnt < kTsStage) {  // only positions that hold a score
#pragma unroll
            for (int r = 0; r < kTsStage / kTsRound; ++r)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if ((r * kTsConsumers + tid) * 4 + k >= cnt) maybe &= ~(1u << (4 * r + k));
          }
          const uint32_t* sw = reinterpret_cast<const uint32_t*>(sb);
          while (maybe) {
            const int bit = __ffs(maybe) - 1;
            maybe &= maybe - 1u;
            const int r = bit >> 2, k = bit & 3;
            const int e = (r * kTsConsumers + tid) * 4 + k;  // < cnt: -inf never passes
            offer_one(r, k, e < n4 ? sw[e] : __float_as_uint(__ldg(rowp + o + e)), failed);
          }
        }
        if (failed) *s_over = 1;
        group_sync(kTsConsumers);
        IDX_TRACE(41);
        // A full buffer (rare: the stage's first offers, or a rising row):
        // compact it to the exact top K, then offer the scores that found it
        // full again, until none does.  The stage stays in the ring meanwhile.
        while (*s_over) {
          group_sync(kTsConsumers);  // every thread has read the flag
          if (tid == 0) {
            fs.count = min(fs.count, fsel.cap);
            *s_over = 0;
          }
          group_sync(kTsConsumers);
          filter_compact<kTsConsumers>(fs, fsel.fbuf, fsel.fbuf + fsel.cap, a.K, *fsel.sc);
          hist_rebuild<kTsConsumers>(fs, fsel.fbuf, fsel.fbuf + fsel.cap, fsel.hist,
                                     fsel.hist + kHBins);
          const uint32_t retry = failed;
          failed = 0;
          for (int r = 0; r < nrounds; ++r) {
            const uint32_t m = retry >> (4 * r) & 0xFu;
            if (!m) continue;
            uint32_t w[4];
            load4(r, w);
            offer(r, w, m, failed);
          }
          if (failed) *s_over = 1;
          group_sync(kTsConsumers);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        // one warp a stage lifts the threshold from the histogram (rotating)
        if ((int)(stage % kTsConsumerWarps) == warp) fused_raise(fsel, a.K, a.row_thr + b);
      }
      group_sync(kTsConsumers);  // every offer of the segment is complete
      IDX_TRACE(12);
      hist_finalize(fsel, out, b, j, ch.first(b), ch.last(b));
    }
  }
  // polls of a row threshold issued by the last raises have landed
  cp_async_wait_all();
}

}  // namespace

bool topk_stream_supported(const float* scores, int64_t lds) {
  return (reinterpret_cast<uintptr_t>(scores) & 15) == 0 && (lds % 4) == 0;
}

int64_t topk_stream_slots(int rows, int num_sms) {
  return (int64_t)num_sms + 1 + (rows < kTsMaxRows ? rows : kTsMaxRows);
}

int topk_stream_max_rows(int N) {
  const int64_t fit = (int64_t)INT32_MAX / ((int64_t)N + kTsRowCharge);
  return fit < kTsMaxRows ? (int)fit : kTsMaxRows;
}

cudaError_t launch_topk_stream(const TopkStreamArgs& a, int num_sms, cudaStream_t stream) {
  const TsLayout L = ts_layout();
  cudaError_t e = cudaFuncSetAttribute(topk_stream_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  // One CTA per SM, fewer when the rows hold fewer than a chunk each, and at
  // most kTsMaxSegments CTAs per row: a row's merge then holds every
  // published list in registers.
  const int64_t work = (int64_t)a.rows * a.N + (int64_t)a.rows * kTsRowCharge;
  int64_t grid = (work + kTsLMin - 1) / kTsLMin;
  if (grid > (int64_t)a.rows * kTsMaxSegments) grid = (int64_t)a.rows * kTsMaxSegments;
  if (grid > num_sms) grid = num_sms;
  if (grid < 1) grid = 1;
  topk_stream_kernel<<<(int)grid, kTsThreads, L.total, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace idx
