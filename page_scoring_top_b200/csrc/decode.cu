// decode.cu -- page scoring on CUDA cores, alone or fused with the top-K select.
//
// The decode shapes the tensor-core kernel (decode_tc.cu) does not take --
// D = 256 or not a multiple of 64, more than 64 query rows -- run here; both
// kernels share the work split and the select steps (fused.cuh).
//
// What is computed ("Iterate Centroids Score", opening description;
// "Round 18 Track C", section 1 Target 2, qsa_score):
//     s[b,t,p] = sum_h sum_d q[b,t,h,d] * c[b,p,d]   for p < len[b]
// with bf16 inputs and fp32 arithmetic.  The heads are summed first, in fp32:
// qs[t,d] = sum_h q[b,t,h,d], then s = sum_d qs[t,d] * c[b,p,d].  That keeps
// the query in registers (the register-hoisting result of qsa_score vB) and
// cuts the work per centroid byte by Q; the fp32 error stays far inside
// 1e-5 * sum_h sum_d |q*c| because sum_d |qs_d * c_d| <= sum_h sum_d |q*c|.
//
// Work decomposition (B200: 148 SMs, one persistent CTA per SM):
//  * The valid pages of all requests are laid end to end (prefix sums of the
//    ragged lengths, computed in every CTA; in fused mode each request is also
//    charged a fixed number of virtual pages for its segment-end select) and
//    cut into equal chunks, so a CTA's load is balanced however ragged the
//    batch is; padded pages are never read.
//  * Warp 8 is the producer: four lanes stream 32-page stages of the centroid
//    table into a shared-memory ring with 1-D bulk copies (TMA engine), an
//    mbarrier pair per slot, L2 evict-first.
//  * Warps 0..7 consume stages round-robin.  Four lanes share a page (8 pages
//    per warp instruction); lane c of page-group p reads the page's 16-byte
//    chunks c, c+4, ... starting at a rotation (p mod chunks-per-lane) that
//    makes every 128-byte shared-memory wavefront hit 32 distinct banks.  Each
//    lane keeps its pre-summed query chunks in registers; a two-step butterfly
//    of shuffles leaves each lane with one page's full score.
//  * Score mode writes the scores (and -inf padding) to HBM.  Fused mode offers
//    each score to an exact online top-K filter in shared memory (fused.cuh:
//    the digit-histogram filter of hsel.cuh for single-token rows, radix
//    compaction filters per token otherwise); at the end of a row's part of
//    the chunk the filter's exact top K is published, and the last CTA to
//    finish the row merges the row's candidates and writes the final indices.
//    The score row never reaches HBM and the producer keeps prefetching
//    through every select step.
// Both modes run the same arithmetic, so fused and score-mode scores are
// bit-identical.
#include "common.cuh"
#include "kernels.h"
#include "fused.cuh"

namespace idx {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
static_assert(kConsumers == kSelThreads, "the consumer warps run the select steps");
constexpr int kDecodeThreads = kConsumers + 32;
constexpr int kStagePages = 32;
constexpr int kMaxStages = 32;
constexpr int kLMin = 256;
constexpr int kSmemMax = 227 * 1024;
constexpr int kProducerLanes = 4;
constexpr size_t kRingTargetBytes = 128 * 1024;

struct DecodeLayout {
  size_t ring, fbuf, fstate, scratch, sortv, sortb, hist, off, bar, misc, total;
  int nstage;
  int cap;  // filter entries per token
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

// Shared-memory layout; identical on host (launch size) and device.
__host__ __device__ inline DecodeLayout decode_layout(bool fused, int D, int T) {
  DecodeLayout L;
  const size_t stage_bytes = (size_t)kStagePages * D * 2;
  L.cap = fused ? fused_cap(T) : 0;
  size_t o = 0;
  L.fbuf = o;  // per token: cap bits then cap indices; 2 * kFilterCap words in all
  o += fused ? (size_t)kFilterCap * 8 : 0;
  L.fstate = o;
  o += fused ? align16(sizeof(FilterState) * kMaxFusedT) : 0;
  L.scratch = o;
  o += fused ? align16(sizeof(SelectScratch)) : 0;
  L.sortv = o;
  o += fused ? (size_t)(kMaxK + 2) * 8 : 0;
  L.sortb = o;
  o += fused ? (size_t)(kMaxK + 4) * 4 : 0;
  L.hist = o;  // single-token filters also keep their digit histograms
  o += (fused && T == 1) ? (size_t)(kHBins + kHCoarse) * 4 : 0;
  L.off = o;
  o += align16((size_t)(kDecodeMaxB + 2) * 4);  // prefix sums + the longest length
  L.bar = o;
  o += (size_t)2 * kMaxStages * 8;
  L.misc = o;
  o += 64;
  o = (o + 127) & ~(size_t)127;
  L.ring = o;  // the ring takes what is left
  int ns = (int)(((size_t)kSmemMax - o) / stage_bytes);
  if (ns > kMaxStages) ns = kMaxStages;
  // About 128 KB in flight per SM streams at the HBM rate; deeper rings only
  // add queueing.
  const int ns_cap = (int)(kRingTargetBytes / stage_bytes);
  if (ns > ns_cap && ns_cap >= kConsumerWarps) ns = ns_cap;
  // A multiple of the consumer-warp count: slot s is then only ever consumed
  // by warp s % 8, which waits on its full barrier's phases strictly in order
  // (a waiter two phases ahead would see an old phase as complete).
  ns -= ns % kConsumerWarps;
  L.nstage = ns;
  o += (size_t)ns * stage_bytes;
  L.total = o;
  return L;
}

// Unpack 8 bf16 (one 16-byte chunk) to fp32; element 2k is the low half of word k.
__device__ __forceinline__ void unpack8(const uint4 v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

// D_T: head dim as a template constant (64, 128, 256), or 0 for any D % 8 == 0.
template <int D_T, int TT, bool FUSED>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  // One token per row: its filter keeps a digit histogram (hsel.cuh), which
  // supplies the running threshold, the winners and the output order.
  constexpr bool HIST = FUSED && TT == 1;
  constexpr int CPL = D_T ? D_T / 32 : 8;  // 16-byte chunks per lane (max)
  const int D = D_T ? D_T : a.D;
  const DecodeLayout L = decode_layout(FUSED, D, a.T);
  unsigned char* ring = smem + L.ring;
  uint32_t* fbuf = reinterpret_cast<uint32_t*>(smem + L.fbuf);
  FilterState* fst = reinterpret_cast<FilterState*>(smem + L.fstate);
  SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem + L.scratch);
  uint64_t* sortv = reinterpret_cast<uint64_t*>(smem + L.sortv);
  uint32_t* sortb = reinterpret_cast<uint32_t*>(smem + L.sortb);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L.hist);
  int* s_off = reinterpret_cast<int*>(smem + L.off);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + kMaxStages;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  volatile int* s_abort = misc;
  uint32_t* s_wsum = reinterpret_cast<uint32_t*>(misc + 4);  // 9 warp sums
  const FusedSel fsel{fbuf, fst,   &sc,    sortv, sortb, hist, L.cap, misc + 1,
                      reinterpret_cast<uint32_t*>(misc + 14)};

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = gridDim.x;
  const int g = blockIdx.x;
  const int B = a.B, T = a.T, N = a.N, Q = a.Q;
  const int nst = L.nstage;
  const int cap = L.cap;
  const uint32_t page_bytes = (uint32_t)D * 2;
  const uint32_t stage_bytes = page_bytes * kStagePages;

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  length_prefix(a, s_off, s_wsum, kDecodeThreads);
  __syncthreads();
  const Chunking ch = FUSED ? make_fused_chunking(s_off, B, G, kSegmentPages, kLMin, a.K)
                            : make_chunking(s_off, B, G, 0, 1);
  const int nchunks = ch.nchunks;

  // ------------------------------------------------------------------ producer
  // Lanes 0..kProducerLanes-1 issue the stages round-robin (stage k by lane
  // k % kProducerLanes): one issuing thread alone caps the copy rate well
  // below HBM bandwidth.  The ring depth is a multiple of kProducerLanes, so a
  // slot is always refilled by the same lane, in order.
  if (warp == kConsumerWarps && a.page_table) {
    // Paged table: the whole warp fills each stage, lane i copying page i of
    // the stage from its block-pool row (no L2 hint: pool rows are shared
    // across requests and stay hot).  Entries outside the pool are clamped.
    uint32_t stage = 0;
    int64_t last = -1;  // last stage this warp filled
    for (int j = g; j < nchunks; j += G) {
      const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
      const int b_last = ch.row(ce - 1);
      for (int b = ch.row(cb); b <= b_last; ++b) {
        if (ch.len(b) == 0) continue;
        const int p0 = ch.snap(b, cb);
        const int np = ch.snap(b, ce) - p0;
        const int32_t* pt = a.page_table + (int64_t)b * a.ld_pt + p0;
        for (int sp = 0; sp < np; sp += kStagePages, ++stage) {
          const int slot = (int)(stage % (uint32_t)nst);
          const uint32_t round = stage / (uint32_t)nst;
          int go = 1;
          if (lane == 0) {
            if (round > 0) mbar_wait_bounded(&empty[slot], (round - 1) & 1, s_abort, a.status);
            go = *s_abort == 0;
          }
          go = __shfl_sync(0xFFFFFFFFu, go, 0);
          if (!go) continue;
          const int n = min(kStagePages, np - sp);
          if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)n * page_bytes);
          if (lane < n) {
            int blk = __ldg(pt + sp + lane);
            if (blk < 0 || blk >= a.n_blocks) {
              atomicOr(a.status, kErrPageClamped);
              blk = blk < 0 ? 0 : a.n_blocks - 1;
            }
            bulk_g2s_nohint(ring + (size_t)slot * stage_bytes + (size_t)lane * page_bytes,
                            a.c + (int64_t)blk * D, page_bytes, &full[slot]);
          }
          last = stage;
        }
      }
    }
    // Nothing may still be landing in shared memory when the CTA exits (this
    // matters only after an abort): wait for the last stages' copies.
    if (lane == 0)
      for (int64_t t = last; t >= 0 && t > last - nst; --t)
        mbar_wait_drain(&full[t % nst], (uint32_t)(t / nst) & 1);
    return;
  }
  if (warp == kConsumerWarps) {
    if (lane < kProducerLanes) {
      const uint64_t pol = policy_evict_first();
      uint32_t stage = 0;
      int64_t last = -1;  // last stage this lane issued
      for (int j = g; j < nchunks; j += G) {
        const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
        const int b_last = ch.row(ce - 1);
        for (int b = ch.row(cb); b <= b_last; ++b) {
          if (ch.len(b) == 0) continue;
          const int p0 = ch.snap(b, cb);
          const int np = ch.snap(b, ce) - p0;
          const uint16_t* src = a.c + (int64_t)b * a.ldc_b + (int64_t)p0 * D;
          for (int sp = 0; sp < np; sp += kStagePages, ++stage) {
            if ((int)(stage % kProducerLanes) != lane) continue;
            const int slot = (int)(stage % (uint32_t)nst);
            const uint32_t round = stage / (uint32_t)nst;
            if (round > 0) mbar_wait_bounded(&empty[slot], (round - 1) & 1, s_abort, a.status);
            if (*s_abort) continue;
            const uint32_t bytes = (uint32_t)min(kStagePages, np - sp) * page_bytes;
            mbar_arrive_expect_tx(&full[slot], bytes);
#ifdef IDX_NO_L2_HINT
            bulk_g2s_nohint(ring + (size_t)slot * stage_bytes, src + (int64_t)sp * D, bytes,
                            &full[slot]);
            (void)pol;
#else
            bulk_g2s(ring + (size_t)slot * stage_bytes, src + (int64_t)sp * D, bytes, &full[slot],
                     pol);
#endif
            last = stage;
          }
        }
      }
      // As above: wait for this lane's copies still in flight before exiting.
      for (int64_t t = last; t >= 0 && t > last - nst; t -= kProducerLanes)
        mbar_wait_drain(&full[t % nst], (uint32_t)(t / nst) & 1);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  if (!FUSED) score_padding(a, s_off, g, G);
  else fused_empty_rows(a, s_off, g, G);

  // Lane geometry: lane = 4 * pg + c4; page-group pg (0..7) of each 8-page
  // instruction, lane c4 (0..3) within the page.
  const int pg = lane >> 2;
  const int c4 = lane & 3;
  const int nchunk = D >> 3;  // 16-byte chunks per page
  const int cpl = D_T ? CPL : (nchunk + 3) / 4;
  uint32_t lane_off[CPL];
  bool chunk_ok[CPL];
  int chunk_of[CPL];
#pragma unroll
  for (int jj = 0; jj < CPL; ++jj) {
    const int ch = c4 + 4 * ((jj + pg) % cpl);
    chunk_of[jj] = ch;
    chunk_ok[jj] = (jj < cpl) && (ch < nchunk);
    lane_off[jj] = (uint32_t)pg * page_bytes + (uint32_t)ch * 16u;
  }
  const int my_page = c4 * 8 + pg;  // page this lane holds after the butterfly
  // Filter checks every `rounds` rounds of 8 stages (a round appends at most
  // 256 entries per token).
  const int rounds = FUSED ? fused_rounds(cap, a.K) : 1;
  const int compact_at = FUSED ? fused_compact_at<HIST>(cap, a.K) : 0;
  const int check_period = rounds * kConsumerWarps;
  const bool q_resident = (T <= TT);

  float qr[TT][CPL][8];
  uint32_t stage = 0;

  for (int j = g; j < nchunks; j += G) {
    const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
    const int b_last = ch.row(ce - 1);
    for (int b = ch.row(cb); b <= b_last; ++b) {
      if (ch.len(b) == 0) continue;
      const int p0 = ch.snap(b, cb);
      const int np = ch.snap(b, ce) - p0;
      if (np <= 0) continue;  // no real page of b in this chunk: not a segment
      if (FUSED) {
        fused_begin<HIST>(fsel, T);
        group_sync(kConsumers);
      }
      for (int sp = 0; sp < np; sp += kStagePages, ++stage) {
        if ((int)(stage % kConsumerWarps) == warp) {
          const int slot = (int)(stage % (uint32_t)nst);
          mbar_wait_bounded(&full[slot], (stage / (uint32_t)nst) & 1, s_abort, a.status);
          const unsigned char* sb = ring + (size_t)slot * stage_bytes;
          const int n_here = min(kStagePages, np - sp);
          for (int t0 = 0; t0 < T; t0 += TT) {
            if (!q_resident || sp < kConsumerWarps * kStagePages) {
              // pre-summed query chunks (first stage of this warp in the
              // segment, or every stage when the tokens do not fit registers)
#pragma unroll
              for (int t = 0; t < TT; ++t)
#pragma unroll
                for (int jj = 0; jj < CPL; ++jj) {
#pragma unroll
                  for (int e = 0; e < 8; ++e) qr[t][jj][e] = 0.f;
                  if (t0 + t < T && chunk_ok[jj]) {
                    const uint16_t* qp =
                        a.q + ((int64_t)b * T + t0 + t) * Q * D + chunk_of[jj] * 8;
                    for (int h = 0; h < Q; ++h) {
                      float f[8];
                      unpack8(*reinterpret_cast<const uint4*>(qp + (int64_t)h * D), f);
#pragma unroll
                      for (int e = 0; e < 8; ++e) qr[t][jj][e] += f[e];
                    }
                  }
                }
            }
            float acc[TT][4];
#pragma unroll
            for (int t = 0; t < TT; ++t)
#pragma unroll
              for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;
#pragma unroll
            for (int jj = 0; jj < CPL; ++jj) {
              if (D_T || chunk_ok[jj]) {
                uint4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  v[i] = *reinterpret_cast<const uint4*>(sb + lane_off[jj] + i * 8 * page_bytes);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float f[8];
                  unpack8(v[i], f);
#pragma unroll
                  for (int t = 0; t < TT; ++t)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[t][i] = fmaf(qr[t][jj][e], f[e], acc[t][i]);
                }
              }
            }
            // butterfly over the 4 lanes of a page: lane c4 ends with group c4's sum
            const bool u2 = (lane & 2) != 0, u1 = (lane & 1) != 0;
#pragma unroll
            for (int t = 0; t < TT; ++t) {
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {
                const float send = u2 ? acc[t][jj] : acc[t][jj + 2];
                const float keep = u2 ? acc[t][jj + 2] : acc[t][jj];
                acc[t][jj] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 2);
              }
              const float send = u1 ? acc[t][0] : acc[t][1];
              const float keep = u1 ? acc[t][1] : acc[t][0];
              acc[t][0] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 1);
            }
            const bool mine = my_page < n_here;
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              if (t0 + t < T) {
                const int page = p0 + sp + my_page;
                // per-token counts: a token row ends before the request's longest
                const bool ok = !a.tok_lengths || page < tok_length(a, b, t0 + t);
                if (FUSED) {
                  fused_offer<HIST>(fsel, t0 + t, __float_as_uint(acc[t][0]), (uint32_t)page,
                                    mine && ok);
                } else if (mine) {
                  a.scores[((int64_t)b * T + t0 + t) * N + page] =
                      ok ? acc[t][0] : __uint_as_float(kNegInfBits);
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[slot]);
          // Every fourth of its stages, a warp lifts the threshold to the
          // histogram's top-K bin; two warps of each round do it.
          if (HIST && ((stage >> 3) & 3) == (uint32_t)(warp & 3)) fused_raise(fsel, a.K, a.row_thr + b);
        }
        if (FUSED && ((stage % check_period) == check_period - 1 || sp + kStagePages >= np)) {
          group_sync(kConsumers);  // this round's offers are complete
          fused_check<HIST>(fsel, T, a.K, compact_at);
        }
      }
      if (FUSED)
        fused_finalize<HIST>(fsel, a, T, b, j, ch.first(b), ch.last(b));
    }
  }
}

int decode_grid(int num_sms) { return num_sms; }

int decode_fused_max_k(int T) {
  if (T > kMaxFusedT) return 0;
  int tp = 1;
  while (tp < T) tp <<= 1;
  const int k = kFilterCap / tp - kConsumers;
  return k < kMaxK ? k : kMaxK;
}

int64_t decode_fused_slots(int64_t B, int64_t T, int64_t N, int grid) {
  // The fused chunk length is at least ceil(virtual pages / grid), so there
  // are at most `grid` chunks; the pair (chunk j, request b) owns slot (j + b)
  // per token.
  (void)N;
  return ((int64_t)grid + 1 + B) * T;
}

template <int D_T, int TT, bool FUSED>
static cudaError_t launch_one(const DecodeArgs& a, int grid, cudaStream_t stream) {
  const DecodeLayout L = decode_layout(FUSED, a.D, a.T);
  if (L.nstage < kConsumerWarps || L.total > (size_t)kSmemMax) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D_T, TT, FUSED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  decode_kernel<D_T, TT, FUSED><<<grid, kDecodeThreads, L.total, stream>>>(a);
  return cudaGetLastError();
}

template <int D_T, bool FUSED>
static cudaError_t launch_tt(const DecodeArgs& a, int grid, cudaStream_t stream) {
  if (a.T == 1) return launch_one<D_T, 1, FUSED>(a, grid, stream);
  return launch_one<D_T, 2, FUSED>(a, grid, stream);
}

cudaError_t launch_decode(const DecodeArgs& a, bool fused, int num_sms, cudaStream_t stream) {
  // Head dims 64 and 128 with up to 64 query rows take the tensor-core kernel
  // (decode_tc.cu), contiguous or paged, in both modes so that fused and
  // score-mode scores stay bit-identical; the CUDA-core kernel takes every
  // other shape (its paged producer copies page by page).
  if (decode_tc_supported(a.T, a.Q, a.D, a.page_table ? a.D : a.ldc_b, a.c))
    return launch_decode_tc(a, fused, num_sms, stream);
  const int grid = decode_grid(num_sms);
  if (fused) {
    if (a.D == 128) return launch_tt<128, true>(a, grid, stream);
    if (a.D == 64) return launch_tt<64, true>(a, grid, stream);
    if (a.D == 256) return launch_tt<256, true>(a, grid, stream);
    return launch_tt<0, true>(a, grid, stream);
  }
  if (a.D == 128) return launch_tt<128, false>(a, grid, stream);
  if (a.D == 64) return launch_tt<64, false>(a, grid, stream);
  if (a.D == 256) return launch_tt<256, false>(a, grid, stream);
  return launch_tt<0, false>(a, grid, stream);
}

}  // namespace idx
