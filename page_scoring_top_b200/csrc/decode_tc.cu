// decode_tc.cu -- page scoring on the tensor cores (tcgen05 / TMEM), alone or
// fused with the top-K select.
//
// What is computed ("Iterate Centroids Score", opening description;
// "Round 18 Track C", section 1 Target 2, qsa_score):
//     s[b,t,p] = sum_h sum_d q[b,t,h,d] * c[b,p,d]   for p < len[b]
// bf16 inputs, fp32 arithmetic.  Per 128-page tile of request b this is the
// matrix product Acc[p, t*Q + h] = sum_d c[b,p,d] * q[b,t,h,d]: M = 128 pages,
// N = T*Q query rows (zero-padded to a multiple of 16), K = D.  The tensor
// cores take the dot products (exact bf16 products, fp32 accumulation); the
// head-sum s = sum_h Acc[p, t*Q + h] is taken in fp32, in head order, on the
// accumulators as they leave TMEM.  The CUDA cores are left with one TMEM load
// and Q - 1 adds per page and token, so the kernel streams the centroids at
// the HBM rate with the select running alongside.
//
// One persistent CTA per SM, 10 warps:
//  * warp 8   TMA: 128-page tiles of c (128-byte swizzled, K-major) into a
//             ring of stages; a segment's ragged tail goes in 32-page boxes.
//             Up to four lanes issue, stage k by lane k % lanes; L2
//             evict-first (the centroids are read once).  A paged table
//             (page p of request b = block-pool row page_table[b][p]) is
//             gathered four rows per copy (tile::gather4), the whole warp
//             filling each tile.
//  * warp 9   MMA: writes the request's query rows into the B operand when
//             the request changes, then one thread issues D/16 tcgen05.mma
//             (M128, N = T*Q rounded up to 16, K16) per tile into one of four
//             TMEM accumulators and commits: the commit frees the stage and
//             hands the accumulator to the epilogue.
//  * warps 0-7 epilogue, two warpgroups taking alternate tiles: each warp
//             loads its 32 TMEM lanes (= 32 pages) and head-sums them; score
//             mode stores the scores, fused mode offers them to the online
//             top-K filter (fused.cuh) and runs the select steps.
// The work split (chunks of equal valid-page counts over the CTAs, segment
// boundaries on 32-page multiples) is the one of the CUDA-core decode kernel.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "fused.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace idx {

PFN_cuTensorMapEncodeTiled_v12000 get_encode();

namespace {

constexpr int kTcEpiWarps = 8;
constexpr int kTcEpi = kTcEpiWarps * 32;
static_assert(kTcEpi == kSelThreads, "the epilogue warps run the select steps");
constexpr int kTcProducerWarp = kTcEpiWarps;
constexpr int kTcMmaWarp = kTcEpiWarps + 1;
constexpr int kTcThreads = kTcEpi + 64;
constexpr int kTcTile = 128;      // pages per tile (MMA M)
constexpr int kTcSub = 32;        // pages per tail box
constexpr int kTcAcc = 4;         // TMEM accumulators, two per epilogue warpgroup
constexpr int kTcMaxNP = 64;      // query rows per request (MMA N)
constexpr int kTcMaxStages = 8;
constexpr int kTcSmemMax = 227 * 1024;
constexpr size_t kTcRingTarget = 128 * 1024;
constexpr int kTcLMin = 256;

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~(size_t)15; }

struct TcLayout {
  size_t bars, misc, off, fbuf, fstate, scratch, sortv, sortb, hist, qop, ring, total;
  int nstage, lanes, cap, np;
};

// Shared-memory layout (offsets from the 1024-aligned base; identical on host and device).
__host__ __device__ inline TcLayout tc_layout(bool fused, int D, int T, int Q) {
  TcLayout L;
  L.np = ((T * Q + 15) / 16) * 16;
  // multi-token rows (no digit histogram) get twice the buffer: their
  // compactions, which raise the thresholds, come half as often
  const int bufs = (fused && T > 1) ? 2 : 1;
  L.cap = fused ? fused_cap(T, bufs) : 0;
  size_t o = 0;
  L.bars = o;  // full[8], empty[8], acc_full[4], acc_empty[4], q_free
  o += 256;
  L.misc = o;  // abort, flag, TMEM base, warp sums
  o += 64;
  L.off = o;
  o += al16((size_t)(kDecodeMaxB + 2) * 4);  // prefix sums + the longest length
  L.fbuf = o;
  o += fused ? (size_t)bufs * kFilterCap * 8 : 0;
  L.fstate = o;
  o += fused ? al16(sizeof(FilterState) * kMaxFusedT) : 0;
  L.scratch = o;
  o += fused ? al16(sizeof(SelectScratch)) : 0;
  L.sortv = o;
  o += fused ? (size_t)(kMaxK + 2) * 8 : 0;
  L.sortb = o;
  o += fused ? (size_t)(kMaxK + 4) * 4 : 0;
  L.hist = o;
  o += (fused && T == 1) ? (size_t)(kHBins + kHCoarse) * 4 : 0;
  o = (o + 1023) & ~(size_t)1023;
  L.qop = o;  // B operand: D/64 blocks of np rows x 128 B
  o += (size_t)L.np * D * 2;
  L.ring = o;
  const size_t stage_bytes = (size_t)kTcTile * D * 2;
  const size_t room = (size_t)kTcSmemMax - 1024 - o;  // 1024: base alignment slack
  int ns = (int)(room / stage_bytes);
  const int ns_cap = (int)(kTcRingTarget / stage_bytes);
  if (ns > ns_cap) ns = ns_cap;
  if (ns > kTcMaxStages) ns = kTcMaxStages;
  L.nstage = ns;
  // Issuing lanes: a slot is always refilled by the same lane (the lane count
  // divides the ring depth), which waits on its empty barrier strictly in order.
  L.lanes = ns % 4 == 0 ? 4 : (ns % 3 == 0 ? 3 : (ns % 2 == 0 ? 2 : 1));
  o += (size_t)(ns > 0 ? ns : 0) * stage_bytes;
  L.total = o + 1024;
  return L;
}

// D: head dim (64 or 128).  NC: query rows the epilogue unrolls (16 or 64).
// HIST: single-token fused rows with the histogram select.  PAGED: page p of
// request b is row page_table[b][p] of a block pool (map_tile is then the
// pool as [n_blocks][D] with one-row boxes, and map_sub is unused).
template <int D, int NC, bool FUSED, bool HIST, bool PAGED>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap map_tile,
                     const __grid_constant__ CUtensorMap map_sub, const DecodeArgs a) {
  static_assert(!HIST || FUSED, "the histogram select is a fused-mode path");
  constexpr int KB = D / 64;                  // 64-column K blocks
  constexpr uint32_t kBlock = kTcTile * 128;  // bytes of one K block of a tile
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const TcLayout L = tc_layout(FUSED, D, a.T, a.Q);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* acc_full = empty + kTcMaxStages;
  uint64_t* acc_empty = acc_full + kTcAcc;
  uint64_t* q_free = acc_empty + kTcAcc;
  int* misc = reinterpret_cast<int*>(smem + L.misc);
  volatile int* s_abort = misc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 2);
  uint32_t* s_wsum = reinterpret_cast<uint32_t*>(misc + 4);  // 10 warp sums
  int* s_off = reinterpret_cast<int*>(smem + L.off);
  unsigned char* qop = smem + L.qop;
  unsigned char* ring = smem + L.ring;
  const FusedSel fsel{reinterpret_cast<uint32_t*>(smem + L.fbuf),
                      reinterpret_cast<FilterState*>(smem + L.fstate),
                      reinterpret_cast<SelectScratch*>(smem + L.scratch),
                      reinterpret_cast<uint64_t*>(smem + L.sortv),
                      reinterpret_cast<uint32_t*>(smem + L.sortb),
                      reinterpret_cast<uint32_t*>(smem + L.hist),
                      L.cap,
                      misc + 1,
                      reinterpret_cast<uint32_t*>(misc + 14)};

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int B = a.B, T = a.T, Q = a.Q, N = a.N;
  const int nst = L.nstage, np = L.np;
  const uint32_t stage_bytes = (uint32_t)kTcTile * D * 2;
  uint32_t tcols = 32;
  while (tcols < (uint32_t)(kTcAcc * np)) tcols <<= 1;

  // The next launch may start taking SMs as this grid's CTAs finish; the
  // shared-memory and TMEM setup below overlaps the previous grid's tail,
  // and nothing in global memory is touched before griddep_wait.
  griddep_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kTcAcc; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrival per warp of the owning warpgroup
    }
    mbar_init(q_free, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kTcMmaWarp) tmem_alloc(tmem_slot, tcols);
  // Query rows past T*Q stay zero for the whole launch.
  for (int i = tid; i < np * D * 2 / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(qop)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  griddep_wait();
  length_prefix(a, s_off, s_wsum, kTcThreads);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Chunking ch = FUSED ? make_fused_chunking(s_off, B, G, kSegmentPages, kTcLMin, a.K)
                            : make_chunking(s_off, B, G, 0, 1);
  const int nchunks = ch.nchunks;

  if (PAGED && warp == kTcProducerWarp) {
    // ------------------------------------------------------------ TMA gather producer
    // The whole warp fills each tile: lane i reads the block ids of pages
    // 4i .. 4i+3 of the tile and gathers the four pool rows per 64-column K
    // block (tile::gather4), which land where a tile load of those rows would
    // put them.  A last group past the segment end repeats its first page.
    // Ids outside the pool are clamped and reported.  No L2 hint: pool rows
    // are shared across requests and stay hot.
    uint32_t tile = 0;
    int64_t last = -1;  // last tile this warp filled
    for (int j = g; j < nchunks; j += G) {
      const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
      const int b_last = ch.row(ce - 1);
      for (int b = ch.row(cb); b <= b_last; ++b) {
        if (ch.len(b) == 0) continue;
        const int p0 = ch.snap(b, cb);
        const int nps = ch.snap(b, ce) - p0;
        const int32_t* pt = a.page_table + (int64_t)b * a.ld_pt + p0;
        for (int r0 = 0; r0 < nps; r0 += kTcTile, ++tile) {
          const int slot = (int)(tile % (uint32_t)nst);
          const uint32_t round = tile / (uint32_t)nst;
          int go = 1;
          if (lane == 0) {
            if (round > 0) mbar_wait_bounded(&empty[slot], (round - 1) & 1, s_abort, a.status);
            go = *s_abort == 0;
          }
          go = __shfl_sync(0xFFFFFFFFu, go, 0);
          if (!go) continue;
          const int rem = min(kTcTile, nps - r0);
          const int ngr = (rem + 3) >> 2;  // 4-row groups
          if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)ngr * 4u * 128u * KB);
          __syncwarp();
          if (lane < ngr) {
            int y[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int r = 4 * lane + u;
              int blk = __ldg(pt + r0 + (r < rem ? r : 4 * lane));
              if (blk < 0 || blk >= a.n_blocks) {
                atomicOr(a.status, kErrPageClamped);
                blk = blk < 0 ? 0 : a.n_blocks - 1;
              }
              y[u] = blk;
            }
            unsigned char* dst = ring + (size_t)slot * stage_bytes + (size_t)lane * 4 * 128;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb)
              tma_gather4(dst + kb * kBlock, &map_tile, kb * 64, y[0], y[1], y[2], y[3],
                          &full[slot]);
          }
          last = tile;
        }
      }
    }
    // Nothing may still be landing in shared memory when the CTA exits (this
    // matters only after an abort): wait for the last tiles' copies.
    if (lane == 0)
      for (int64_t t = last; t >= 0 && t > last - nst; --t)
        mbar_wait_drain(&full[t % nst], (uint32_t)(t / nst) & 1);
  } else if (warp == kTcProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    const int lanes = L.lanes;
    if (lane < lanes) {
      const uint64_t pol = policy_evict_first();
      uint32_t tile = 0;
      int64_t last = -1;  // last tile this lane issued
      for (int j = g; j < nchunks; j += G) {
        const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
        const int b_last = ch.row(ce - 1);
        for (int b = ch.row(cb); b <= b_last; ++b) {
          if (ch.len(b) == 0) continue;
          const int p0 = ch.snap(b, cb);
          const int nps = ch.snap(b, ce) - p0;
          for (int r0 = 0; r0 < nps; r0 += kTcTile, ++tile) {
            if ((int)(tile % (uint32_t)lanes) != lane) continue;
            const int slot = (int)(tile % (uint32_t)nst);
            const uint32_t round = tile / (uint32_t)nst;
            if (round > 0) mbar_wait_bounded(&empty[slot], (round - 1) & 1, s_abort, a.status);
            if (*s_abort) continue;
            unsigned char* dst = ring + (size_t)slot * stage_bytes;
            const int rem = nps - r0;
            if (rem >= kTcTile) {
              mbar_arrive_expect_tx(&full[slot], stage_bytes);
#pragma unroll
              for (int kb = 0; kb < KB; ++kb)
                tma_load_3d_hint(dst + kb * kBlock, &map_tile, kb * 64, p0 + r0, b, &full[slot],
                                 pol);
            } else {
              const int nsub = (rem + kTcSub - 1) / kTcSub;
              mbar_arrive_expect_tx(&full[slot], (uint32_t)(nsub * kTcSub * D * 2));
              for (int u = 0; u < nsub; ++u)
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                  tma_load_3d_hint(dst + kb * kBlock + u * kTcSub * 128, &map_sub, kb * 64,
                                   p0 + r0 + u * kTcSub, b, &full[slot], pol);
            }
            last = tile;
          }
        }
      }
      // Nothing may still be landing in shared memory when the CTA exits (this
      // matters only after an abort): wait for this lane's last copies.
      for (int64_t t = last; t >= 0 && t > last - nst; t -= lanes)
        mbar_wait_drain(&full[t % nst], (uint32_t)(t / nst) & 1);
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc_bf16(kTcTile, np);
    const uint32_t q_base = smem_u32(qop);
    const uint32_t ring_base = smem_u32(ring);
    const int rows = T * Q;
    uint32_t tile = 0;
    int seg = 0;
    for (int j = g; j < nchunks; j += G) {
      const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
      const int b_last = ch.row(ce - 1);
      for (int b = ch.row(cb); b <= b_last; ++b) {
        if (ch.len(b) == 0) continue;
        const int p0 = ch.snap(b, cb);
        const int nps = ch.snap(b, ce) - p0;
        if (nps <= 0) continue;
        // The previous request's MMAs must be done reading the query rows.
        if (seg > 0 && lane == 0) mbar_wait_bounded(q_free, (uint32_t)(seg - 1) & 1, s_abort, a.status);
        __syncwarp();
        // q[b] as [T*Q rows][D] into the swizzled K-major B operand
        const uint16_t* qb = a.q + (int64_t)b * rows * D;
        for (int x = lane; x < rows * (D / 8); x += 32) {
          const int r = x / (D / 8), c = x % (D / 8);
          const int kb = c >> 3, cc = c & 7;
          const uint4 v = *reinterpret_cast<const uint4*>(qb + (int64_t)r * D + c * 8);
          *reinterpret_cast<uint4*>(qop + (size_t)kb * np * 128 + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int ntl = (nps + kTcTile - 1) / kTcTile;
        if (lane == 0) {
          for (int tt = 0; tt < ntl; ++tt, ++tile) {
            const int slot = (int)(tile % (uint32_t)nst);
            const int acc = (int)(tile % kTcAcc);
            mbar_wait_bounded(&full[slot], (tile / (uint32_t)nst) & 1, s_abort, a.status);
            if (tile >= (uint32_t)kTcAcc)
              mbar_wait_bounded(&acc_empty[acc], ((tile / kTcAcc) - 1) & 1, s_abort, a.status);
            tc_fence_after();
            if (!*s_abort) {
              const uint32_t d_tmem = tmem_base + (uint32_t)(acc * np);
              const uint32_t a_base = ring_base + (uint32_t)slot * stage_bytes;
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint32_t kb = (uint32_t)(k >> 2), ks = (uint32_t)(k & 3);
                const uint64_t ad = umma_desc_sw128(a_base + kb * kBlock + ks * 32u);
                const uint64_t bd = umma_desc_sw128(q_base + kb * (uint32_t)np * 128u + ks * 32u);
                umma_bf16(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
              }
            }
            umma_commit(&empty[slot]);
            umma_commit(&acc_full[acc]);
          }
          umma_commit(q_free);
        }
        tile = __shfl_sync(0xFFFFFFFFu, tile, 0);
        __syncwarp();
        ++seg;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = warp >> 2;    // warpgroup: takes tiles with (tile & 1) == wg
    const int quad = warp & 3;   // TMEM lanes quad*32 .. quad*32+31 = pages of the tile
    IDX_TRACE(10);
    if (!FUSED) score_padding(a, s_off, g, G);
    else fused_empty_rows(a, s_off, g, G);
    const int rows = T * Q;
    // Filter checks: a tile appends at most 128 entries per token, so after a
    // check that leaves `room` free entries the next one comes within
    // room / 128 tiles.  With the histogram the compaction is only the
    // overflow guard; without it, it also raises the threshold.
    // (without it, a filter compacts once it holds twice K entries -- the
    // threshold then tracks the K-th value -- and always before the room
    // runs out; small per-token filters would otherwise compact every check)
    const int compact_at =
        FUSED ? (HIST ? L.cap - 2 * kTcTile
                      : max(fused_compact_at<HIST>(L.cap, a.K), min(L.cap - 2 * kTcTile, 2 * a.K)))
              : 0;
    uint32_t tile = 0;
    for (int j = g; j < nchunks; j += G) {
      const int cb = ch.chunk_begin(j), ce = ch.chunk_end(j);
      const int b_last = ch.row(ce - 1);
      for (int b = ch.row(cb); b <= b_last; ++b) {
        if (ch.len(b) == 0) continue;
        const int p0 = ch.snap(b, cb);
        const int nps = ch.snap(b, ce) - p0;
        if (nps <= 0) continue;  // no real page of b in this chunk: not a segment
        if (FUSED) {
          fused_begin<HIST>(fsel, T);
          group_sync(kTcEpi);
        }
        const int ntl = (nps + kTcTile - 1) / kTcTile;
        int next_check = FUSED ? (L.cap - a.K) / kTcTile - 1 : 0;
        for (int tt = 0; tt < ntl; ++tt, ++tile) {
          if ((int)(tile & 1) == wg) {
            const int acc = (int)(tile % kTcAcc);
            mbar_wait_bounded(&acc_full[acc], (tile / kTcAcc) & 1, s_abort, a.status);
            tc_fence_after();
            uint32_t v[NC];
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * np);
#pragma unroll
            for (int c16 = 0; c16 < NC / 16; ++c16)
              if (c16 * 16 < rows) tmem_ld16_nowait(taddr + c16 * 16, v + c16 * 16);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            const int row = tt * kTcTile + quad * 32 + lane;
            const bool mine = row < nps;
            const int page = p0 + row;
            // head-sums in head order, one token after another (starting from
            // -0, which adds exactly: the same bits in both modes)
            if (FUSED) {
              constexpr int TM = HIST ? 1 : kMaxFusedT;
              float st[TM];
#pragma unroll
              for (int t = 0; t < TM; ++t) st[t] = -0.f;
#pragma unroll
              for (int col = 0; col < NC; ++col) {
                if (col < rows) {
                  const float x = __uint_as_float(v[col]);
#pragma unroll
                  for (int t = 0; t < TM; ++t)
                    if (col >= t * Q && col < t * Q + Q) st[t] += x;
                }
              }
#pragma unroll
              for (int t = 0; t < TM; ++t)
                if (t < T) {
                  // per-token counts: a token row ends before the request's longest
                  const bool ok = mine && (!a.tok_lengths || page < tok_length(a, b, t));
                  fused_offer<HIST>(fsel, t, __float_as_uint(st[t]), (uint32_t)page, ok);
                }
            } else {
              float s = -0.f;
              int h = 0, t = 0;
#pragma unroll
              for (int col = 0; col < NC; ++col) {
                if (col < rows) {
                  s += __uint_as_float(v[col]);
                  if (++h == Q) {
                    if (mine)
                      a.scores[((int64_t)b * T + t) * N + page] =
                          (!a.tok_lengths || page < tok_length(a, b, t))
                              ? s
                              : __uint_as_float(kNegInfBits);
                    s = -0.f;
                    h = 0;
                    ++t;
                  }
                }
              }
            }
            // twice per 8 tiles (once per warpgroup), one warp lifts the
            // threshold from the histogram
            if (HIST && (tile & 7) == (wg ? 5u : 0u) && (int)((tile >> 3) & 3) == quad)
              fused_raise(fsel, a.K, a.row_thr + b);
          }
          if (FUSED && (tt == next_check || tt + 1 == ntl)) {
            group_sync(kTcEpi);  // every offer so far is complete
            next_check = tt + max(1, fused_check<HIST>(fsel, T, a.K, compact_at) / kTcTile);
          }
        }
        IDX_TRACE(12);
        if (FUSED) fused_finalize<HIST>(fsel, a, T, b, j, ch.first(b), ch.last(b));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
}

template <int D, int NC, bool FUSED, bool HIST, bool PAGED>
cudaError_t launch_tc(const CUtensorMap& mt, const CUtensorMap& ms, const DecodeArgs& a, int grid,
                      size_t smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<D, NC, FUSED, HIST, PAGED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // Launched as a programmatic dependent of the previous kernel in the
  // stream: its setup overlaps that kernel's tail, its global reads wait.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<D, NC, FUSED, HIST, PAGED>, mt, ms, a);
}

template <int D, bool FUSED, bool HIST, bool PAGED>
cudaError_t launch_nc(const CUtensorMap& mt, const CUtensorMap& ms, const DecodeArgs& a, int grid,
                      size_t smem, cudaStream_t stream) {
  if (a.T * a.Q <= 16) return launch_tc<D, 16, FUSED, HIST, PAGED>(mt, ms, a, grid, smem, stream);
  return launch_tc<D, 64, FUSED, HIST, PAGED>(mt, ms, a, grid, smem, stream);
}

template <int D, bool PAGED>
cudaError_t launch_modes(const CUtensorMap& mt, const CUtensorMap& ms, const DecodeArgs& a,
                         bool fused, int grid, size_t smem, cudaStream_t stream) {
  if (!fused) return launch_nc<D, false, false, PAGED>(mt, ms, a, grid, smem, stream);
  if (a.T == 1) return launch_nc<D, true, true, PAGED>(mt, ms, a, grid, smem, stream);
  return launch_nc<D, true, false, PAGED>(mt, ms, a, grid, smem, stream);
}

}  // namespace

bool decode_tc_supported(int T, int Q, int D, int64_t ldc_b, const void* c) {
  if (!(D == 64 || D == 128) || T < 1 || Q < 1 || T * Q > kTcMaxNP) return false;
  if ((ldc_b % 8) != 0 || (reinterpret_cast<uintptr_t>(c) & 15) != 0) return false;
  const TcLayout L = tc_layout(true, D, T, Q);
  return L.nstage >= 2 && L.total <= (size_t)kTcSmemMax;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, bool fused, int num_sms, cudaStream_t stream) {
  if (!decode_tc_supported(a.T, a.Q, a.D, a.page_table ? a.D : a.ldc_b, a.c))
    return cudaErrorNotSupported;
  auto encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  const TcLayout L = tc_layout(fused, a.D, a.T, a.Q);
  const int grid = num_sms;
  if (a.page_table) {
    // the block pool as [n_blocks][D] bf16; one-row boxes of 64 columns
    // (128 B, 128-byte swizzle) for the four-row gathers
    CUtensorMap mp;
    const cuuint64_t dims[2] = {(cuuint64_t)a.D, (cuuint64_t)a.n_blocks};
    const cuuint64_t strides[1] = {(cuuint64_t)a.D * 2};
    const cuuint32_t estr[2] = {1, 1};
    const cuuint32_t box[2] = {64, 1};
    if (encode(&mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.c), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if (a.D == 128) return launch_modes<128, true>(mp, mp, a, fused, grid, L.total, stream);
    return launch_modes<64, true>(mp, mp, a, fused, grid, L.total, stream);
  }
  // c as [B][N][D] bf16 with request stride ldc_b; boxes of 64 columns (128 B,
  // 128-byte swizzle) x 128 pages (whole tiles) or x 32 pages (ragged tails)
  CUtensorMap mt, ms;
  const cuuint64_t dims[3] = {(cuuint64_t)a.D, (cuuint64_t)a.N, (cuuint64_t)a.B};
  const cuuint64_t strides[2] = {(cuuint64_t)a.D * 2, (cuuint64_t)a.ldc_b * 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t box_t[3] = {64, (cuuint32_t)kTcTile, 1};
  const cuuint32_t box_s[3] = {64, (cuuint32_t)kTcSub, 1};
  if (encode(&mt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(a.c), dims, strides,
             box_t, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode(&ms, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(a.c), dims, strides,
             box_s, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (a.D == 128) return launch_modes<128, false>(mt, ms, a, fused, grid, L.total, stream);
  return launch_modes<64, false>(mt, ms, a, fused, grid, L.total, stream);
}

}  // namespace idx
