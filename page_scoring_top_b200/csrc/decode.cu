// decode.cu -- page scoring on CUDA cores, alone or fused with the top-K select.
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
//    ragged lengths, computed in every CTA) and cut into equal chunks, so a
//    CTA's load is balanced to within one page however ragged the batch is;
//    padded pages are never read.
//  * Warp 8 is the producer: one lane streams 32-page stages of the centroid
//    table into a shared-memory ring with 1-D bulk copies (TMA engine), an
//    mbarrier pair per slot, L2 evict-first.
//  * Warps 0..7 consume stages round-robin.  D/8 lanes cover one page's
//    16-byte chunks (32/(D/8) pages per warp instruction, conflict-free), each
//    lane keeps its 8 pre-summed query values in registers, and a transposed
//    butterfly of shuffles leaves lane l holding one page's full score.
//  * Score mode writes the scores (and -inf padding) to HBM.  Fused mode keeps
//    the chunk's scores in shared memory; when a row's part of the chunk is
//    done, the consumer warps select its exact top-K' there, publish the
//    candidates, and the last CTA to finish the row merges all of the row's
//    candidates and writes the final indices.  The full score row never
//    reaches HBM, and the producer keeps prefetching during the select.
// Both modes run the same arithmetic, so fused and score-mode scores are
// bit-identical.
#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"

namespace idx {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kDecodeThreads = kConsumers + 32;
constexpr int kStagePages = 32;
constexpr int kMaxStages = 32;
constexpr int kLMin = 128;
constexpr int kSmemMax = 227 * 1024;

struct DecodeLayout {
  size_t ring, score, win, scratch, off, bar, misc, total;
  int nstage;
};

__host__ __device__ inline DecodeLayout decode_layout(bool fused, int D) {
  DecodeLayout L;
  const size_t stage_bytes = (size_t)kStagePages * D * 2;
  size_t fixed = 0;
  fixed += fused ? (size_t)kDecodeScoreCap * 4 : 0;                       // score
  fixed += fused ? 2048 * 4 : 0;                                          // win_pos
  fixed += fused ? ((sizeof(SelectScratch) + 15) & ~(size_t)15) : 0;     // scratch / sort
  fixed += (size_t)(kDecodeMaxB + 1) * 4 + 12;                            // off (+pad)
  fixed += (size_t)2 * kMaxStages * 8;                                    // barriers
  fixed += 64;                                                            // misc
  size_t ring_cap = (size_t)kSmemMax - fixed;
  int ns = (int)(ring_cap / stage_bytes);
  if (ns > kMaxStages) ns = kMaxStages;
  L.nstage = ns;
  size_t o = 0;
  L.ring = o;
  o += (size_t)ns * stage_bytes;
  L.score = o;
  o += fused ? (size_t)kDecodeScoreCap * 4 : 0;
  L.win = o;
  o += fused ? 2048 * 4 : 0;
  L.scratch = o;
  o += fused ? ((sizeof(SelectScratch) + 15) & ~(size_t)15) : 0;
  L.off = o;
  o += ((size_t)(kDecodeMaxB + 1) * 4 + 15) & ~(size_t)15;
  L.bar = o;
  o += (size_t)2 * kMaxStages * 8;
  L.misc = o;
  o += 64;
  L.total = o;
  return L;
}

// First request b whose pages extend past global page gp (s_off[b+1] > gp).
__device__ __forceinline__ int row_of(const int* s_off, int B, int gp) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (s_off[mid + 1] > gp) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

// Unpack 8 bf16 (one 16-byte chunk) to fp32.
__device__ __forceinline__ void unpack8(const uint4 v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

template <int LPP, int TT, bool FUSED>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DecodeLayout L = decode_layout(FUSED, a.D);
  unsigned char* ring = smem + L.ring;
  uint32_t* s_score = reinterpret_cast<uint32_t*>(smem + L.score);
  int* win_pos = reinterpret_cast<int*>(smem + L.win);
  SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem + L.scratch);
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(smem + L.scratch);
  int* s_off = reinterpret_cast<int*>(smem + L.off);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + kMaxStages;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  volatile int* s_abort = misc;
  int* s_flag = misc + 1;
  uint32_t* s_wsum = reinterpret_cast<uint32_t*>(misc + 4);  // 9 warp sums

  constexpr int PPI = 32 / LPP;  // pages per warp instruction
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = gridDim.x;
  const int g = blockIdx.x;
  const int B = a.B, T = a.T, N = a.N, D = a.D, Q = a.Q;
  const int nst = L.nstage;
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
  // Prefix sums of the clamped lengths: s_off[b] = first global page of request b.
  {
    int running = 0;
    if (tid == 0) s_off[0] = 0;
    for (int base = 0; base < B; base += kDecodeThreads) {
      const int i = base + tid;
      int len = 0;
      if (i < B) {
        len = a.lengths ? a.lengths[i] : N;
        if (len < 0 || len > N) {
          if (g == 0) atomicOr(a.status, kErrLengthClamped);
          len = len < 0 ? 0 : N;
        }
      }
      const uint32_t incl = warp_incl_scan((uint32_t)len);
      if (lane == 31) s_wsum[warp] = incl;
      __syncthreads();
      uint32_t excl = incl - (uint32_t)len, total = 0;
      for (int w = 0; w < kDecodeThreads / 32; ++w) {
        if (w < warp) excl += s_wsum[w];
        total += s_wsum[w];
      }
      if (i < B) s_off[i + 1] = running + (int)excl + len;
      __syncthreads();
      running += (int)total;
    }
  }
  __syncthreads();
  const int P = s_off[B];
  int Lc;
  if (FUSED) {
    Lc = (P + G - 1) / G;
    Lc = Lc < kLMin ? kLMin : Lc;
    const int lmax = kDecodeScoreCap / T;
    Lc = Lc > lmax ? lmax : Lc;
  } else {
    Lc = (P + G - 1) / G;
    Lc = Lc < 1 ? 1 : Lc;
  }
  const int nchunks = (P + Lc - 1) / Lc;

  // ------------------------------------------------------------------ producer
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t stage = 0;
      for (int j = g; j < nchunks; j += G) {
        const int cb = j * Lc, ce = min(cb + Lc, P);
        int b = row_of(s_off, B, cb);
        for (int gp = cb; gp < ce;) {
          while (s_off[b + 1] <= gp) ++b;
          const int se = min(ce, s_off[b + 1]);
          const int p0 = gp - s_off[b];
          const int np = se - gp;
          const uint16_t* src = a.c + (int64_t)b * a.ldc_b + (int64_t)p0 * D;
          for (int sp = 0; sp < np; sp += kStagePages, ++stage) {
            const int slot = (int)(stage % (uint32_t)nst);
            const uint32_t round = stage / (uint32_t)nst;
            if (round > 0) mbar_wait_bounded(&empty[slot], (round - 1) & 1, s_abort, a.status);
            if (*s_abort) continue;
            const uint32_t bytes = (uint32_t)min(kStagePages, np - sp) * page_bytes;
            mbar_arrive_expect_tx(&full[slot], bytes);
            bulk_g2s(ring + (size_t)slot * stage_bytes, src + (int64_t)sp * D, bytes, &full[slot],
                     pol);
          }
          gp = se;
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  if (!FUSED) {
    // -inf for the padded pages p >= len[b] of every token row, balanced over CTAs.
    const int64_t per_tok_total = (int64_t)B * N - P;
    const int64_t tot = per_tok_total * T;
    const int64_t beg = tot * g / G, end = tot * (g + 1) / G;
    if (beg < end) {
      // first request whose padding extends past beg
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int64_t pad_next = (int64_t)T * ((int64_t)(mid + 1) * N - s_off[mid + 1]);
        if (pad_next > beg) hi = mid;
        else lo = mid + 1;
      }
      int64_t x = beg;
      for (int b = lo; x < end && b < B; ++b) {
        const int lb = s_off[b + 1] - s_off[b];
        const int64_t per = N - lb;
        const int64_t rb = (int64_t)T * ((int64_t)b * N - s_off[b]);
        const int64_t re = rb + per * T;
        const int64_t e = end < re ? end : re;
        for (int64_t y = x + tid; y < e; y += kConsumers) {
          const int64_t r = y - rb;
          const int t = (int)(r / per);
          const int p = lb + (int)(r % per);
          a.scores[((int64_t)b * T + t) * N + p] = __uint_as_float(kNegInfBits);
        }
        if (e > x) x = e;
      }
    }
  } else {
    // Rows with no valid page: their output is all padding.
    for (int b = g; b < B; b += G) {
      if (s_off[b + 1] != s_off[b]) continue;
      for (int x = tid; x < T * a.K; x += kConsumers) {
        const int64_t o = ((int64_t)b * T) * a.K + x;
        a.idx_out[o] = -1;
        if (a.val_out) a.val_out[o] = __uint_as_float(kNegInfBits);
      }
    }
  }

  const int nchunks_d = D >> 3;  // 16-byte chunks per page
  const int chunk_id = lane & (LPP - 1);
  const int sub = lane / LPP;
  const int my_page = chunk_id * PPI + sub;  // page this lane holds after the butterfly
  uint32_t stage = 0;
  int cur_b = -1;
  float qs[TT][8];

  for (int j = g; j < nchunks; j += G) {
    const int cb = j * Lc, ce = min(cb + Lc, P);
    int b = row_of(s_off, B, cb);
    for (int gp = cb; gp < ce;) {
      while (s_off[b + 1] <= gp) ++b;
      const int se = min(ce, s_off[b + 1]);
      const int p0 = gp - s_off[b];
      const int np = se - gp;
      const int local = gp - cb;
      for (int sp = 0; sp < np; sp += kStagePages, ++stage) {
        if ((int)(stage % kConsumerWarps) != warp) continue;
        const int slot = (int)(stage % (uint32_t)nst);
        mbar_wait_bounded(&full[slot], (stage / (uint32_t)nst) & 1, s_abort, a.status);
        const unsigned char* sb = ring + (size_t)slot * stage_bytes;
        const int n_here = min(kStagePages, np - sp);
        for (int t0 = 0; t0 < T; t0 += TT) {
          // pre-summed query of tokens t0..t0+TT-1 for this lane's 8 dims
          if (b != cur_b || T > TT) {
#pragma unroll
            for (int t = 0; t < TT; ++t) {
#pragma unroll
              for (int e = 0; e < 8; ++e) qs[t][e] = 0.f;
              if (t0 + t < T && chunk_id < nchunks_d) {
                const uint16_t* qp = a.q + (((int64_t)b * T + t0 + t) * Q) * D + chunk_id * 8;
                for (int h = 0; h < Q; ++h) {
                  float f[8];
                  unpack8(*reinterpret_cast<const uint4*>(qp + (int64_t)h * D), f);
#pragma unroll
                  for (int e = 0; e < 8; ++e) qs[t][e] += f[e];
                }
              }
            }
            cur_b = b;
          }
          float acc[TT][LPP];
#pragma unroll
          for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int i = 0; i < LPP; ++i) acc[t][i] = 0.f;
#pragma unroll
          for (int i = 0; i < LPP; ++i) {
            const int page = i * PPI + sub;
            if (page < n_here && chunk_id < nchunks_d) {
              const uint4 v = *reinterpret_cast<const uint4*>(sb + (size_t)page * page_bytes +
                                                              chunk_id * 16);
              float f[8];
              unpack8(v, f);
#pragma unroll
              for (int t = 0; t < TT; ++t)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[t][i] = fmaf(qs[t][e], f[e], acc[t][i]);
            }
          }
          // transposed butterfly over the LPP lanes of a page
#pragma unroll
          for (int m = LPP / 2; m >= 1; m >>= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int t = 0; t < TT; ++t) {
#pragma unroll
              for (int jj = 0; jj < m; ++jj) {
                const float send = upper ? acc[t][jj] : acc[t][jj + m];
                const float keep = upper ? acc[t][jj + m] : acc[t][jj];
                acc[t][jj] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, m);
              }
            }
          }
          if (my_page < n_here) {
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              if (t0 + t < T) {
                if (FUSED) {
                  s_score[(t0 + t) * Lc + local + sp + my_page] = __float_as_uint(acc[t][0]);
                } else {
                  a.scores[((int64_t)b * T + t0 + t) * N + p0 + sp + my_page] = acc[t][0];
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      if (FUSED) {
        group_sync(kConsumers);  // every stage of this row segment is scored
        const int j0 = s_off[b] / Lc;
        const int j1 = (s_off[b + 1] - 1) / Lc;
        const bool single = (j0 == j1);
        for (int t = 0; t < T; ++t) {
          const uint32_t* row = s_score + t * Lc + local;
          const int kk = block_select<kConsumers>(row, np, a.K, win_pos, sc);
          const int64_t orow = (int64_t)b * T + t;
          if (single) {
            sort_and_write<kConsumers>(row, nullptr, p0, win_pos, kk, a.K, sortbuf,
                                       a.idx_out + orow * a.K,
                                       a.val_out ? a.val_out + orow * a.K : nullptr);
          } else {
            const int64_t slot = (int64_t)(j + b) * T + t;
            uint32_t* cbits = a.cand_bits + slot * a.slot_stride;
            int32_t* cidx = a.cand_idx + slot * a.slot_stride;
            for (int k = tid; k < kk; k += kConsumers) {
              const int p = win_pos[k];
              cbits[k] = row[p];
              cidx[k] = p0 + p;
            }
            if (tid == 0) a.cand_cnt[slot] = kk;
          }
        }
        if (!single && arrive_last<kConsumers>(a.arrive + b, j1 - j0 + 1, s_flag)) {
          const int cap = kDecodeScoreCap / 2;
          uint32_t* m_bits = s_score;
          int32_t* m_idx = reinterpret_cast<int32_t*>(s_score + cap);
          for (int t = 0; t < T; ++t) {
            const int64_t orow = (int64_t)b * T + t;
            merge_candidates<kConsumers>(
                j1 - j0 + 1, [=](int i) { return (int64_t)(j0 + i + b) * T + t; }, a.cand_bits,
                a.cand_idx, a.cand_cnt, a.slot_stride, a.K, cap, m_bits, m_idx, win_pos, sc,
                sortbuf, a.idx_out + orow * a.K, a.val_out ? a.val_out + orow * a.K : nullptr);
          }
        }
      }
      gp = se;
    }
  }
}

int decode_grid(int num_sms) { return num_sms; }

int64_t decode_fused_slots(int64_t B, int64_t T, int64_t N, int grid) {
  // The kernel's chunk length is clamp(ceil(P/grid), kLMin, floor(cap/T)), so
  // chunks <= max(grid, ceil(B*N / floor(cap/T))); the pair (chunk j,
  // request b) owns slot (j + b) for each of its T tokens.
  const int64_t lmax = kDecodeScoreCap / T;
  int64_t chunks = (B * N + lmax - 1) / lmax;
  if (chunks < grid) chunks = grid;
  return (chunks + 1 + B) * T;
}

template <int LPP, int TT, bool FUSED>
static cudaError_t launch_one(const DecodeArgs& a, int grid, cudaStream_t stream) {
  const DecodeLayout L = decode_layout(FUSED, a.D);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<LPP, TT, FUSED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  decode_kernel<LPP, TT, FUSED><<<grid, kDecodeThreads, L.total, stream>>>(a);
  return cudaGetLastError();
}

template <int LPP, bool FUSED>
static cudaError_t launch_tt(const DecodeArgs& a, int grid, cudaStream_t stream) {
  // register budget: TT * LPP accumulators
  if (a.T == 1) return launch_one<LPP, 1, FUSED>(a, grid, stream);
  if (a.T == 2 || LPP == 32) return launch_one<LPP, 2, FUSED>(a, grid, stream);
  return launch_one<LPP, 4, FUSED>(a, grid, stream);
}

cudaError_t launch_decode(const DecodeArgs& a, bool fused, int num_sms, cudaStream_t stream) {
  const int grid = decode_grid(num_sms);
  const int chunks = a.D / 8;
  if (fused) {
    if (chunks <= 8) return launch_tt<8, true>(a, grid, stream);
    if (chunks <= 16) return launch_tt<16, true>(a, grid, stream);
    return launch_tt<32, true>(a, grid, stream);
  }
  if (chunks <= 8) return launch_tt<8, false>(a, grid, stream);
  if (chunks <= 16) return launch_tt<16, false>(a, grid, stream);
  return launch_tt<32, false>(a, grid, stream);
}

}  // namespace idx
