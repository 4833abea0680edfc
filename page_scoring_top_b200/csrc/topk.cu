// topk.cu -- standalone exact top-K over fp32 score rows ("Iterate Topk",
// opening description: given per-segment scores, return the top-K indices).
//
// Grid (chunks, rows).  Each CTA streams one chunk of a row from HBM with
// coalesced 16-byte loads (one round prefetched ahead) and offers every
// element to the exact online top-K filter of select.cuh; rounds are visited
// in bit-reversed order, so a row sorted ascending or descending still raises
// the threshold early.  A row that fits one chunk is sorted and written by
// its CTA; otherwise each chunk publishes its K' candidates and the last CTA
// of the row to arrive merges them.  Every score is read from HBM once.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace idx {

constexpr int kTopkThreads = 256;
constexpr int kTopkMaxChunk = 16384;
constexpr int kTopkMinChunk = 2048;
constexpr int kTopkVec = 4;                               // float4 loads per thread per round
constexpr int kTopkRound = kTopkThreads * 4 * kTopkVec;  // elements per round

struct TopkLayout {
  size_t fbuf, fstate, scratch, sortv, sortb, flag, total;
};

__host__ __device__ inline TopkLayout topk_layout() {
  TopkLayout L;
  size_t o = 0;
  L.fbuf = o;
  o += (size_t)kFilterCap * 8;
  L.fstate = o;
  o += 16;
  L.scratch = o;
  o += (sizeof(SelectScratch) + 15) & ~(size_t)15;
  L.sortv = o;
  o += (size_t)(kMaxK + 2) * 8;
  L.sortb = o;
  o += (size_t)(kMaxK + 4) * 4;
  L.flag = o;
  o += 16;
  L.total = o;
  return L;
}

__device__ __forceinline__ int clamp_len(const int32_t* lengths, int r, int N, int* status,
                                         bool report) {
  if (!lengths) return N;
  int l = lengths[r];
  if (l < 0 || l > N) {
    if (report) atomicOr(status, kErrLengthClamped);
    l = l < 0 ? 0 : N;
  }
  return l;
}

__device__ __forceinline__ uint32_t bit_reverse(uint32_t x, int bits) {
  return bits ? (__brev(x) >> (32 - bits)) : 0u;
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_chunk_kernel(const TopkArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const TopkLayout L = topk_layout();
  uint32_t* fb = reinterpret_cast<uint32_t*>(smem + L.fbuf);
  uint32_t* fi = fb + kFilterCap;
  FilterState& fs = *reinterpret_cast<FilterState*>(smem + L.fstate);
  SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem + L.scratch);
  uint64_t* sortv = reinterpret_cast<uint64_t*>(smem + L.sortv);
  uint32_t* sortb = reinterpret_cast<uint32_t*>(smem + L.sortb);
  int* s_flag = reinterpret_cast<int*>(smem + L.flag);

  const int tid = threadIdx.x;
  const int row = blockIdx.y;
  const int ch = blockIdx.x;
  const int len = clamp_len(a.lengths, row / a.len_div, a.N, a.status, ch == 0 && tid == 0);
  const int nch = len > 0 ? (len + a.chunk - 1) / a.chunk : 1;
  if (ch >= nch) return;
  const int c0 = ch * a.chunk;
  const int n = max(0, min(a.chunk, len - c0));
  const float* src = a.scores + (int64_t)row * a.lds + c0;
  const bool vec = (reinterpret_cast<uintptr_t>(src) & 15) == 0;

  int32_t* io = a.idx_out + (int64_t)row * a.K;
  float* vo = a.val_out ? a.val_out + (int64_t)row * a.K : nullptr;

  if (tid == 0) filter_reset(fs);
  group_sync(NT);
  // compact once the filter holds a few K entries (the threshold then rises
  // early), and always before the next 4*NT offers could overflow it
  const int compact_at = min(kFilterCap - 4 * NT, max(4 * a.K, 1024));

  // Round r covers elements [r * kTopkRound, (r+1) * kTopkRound) of the chunk;
  // thread tid loads float4 number tid + u * NT (u < kTopkVec) of the round.
  const int rounds = (n + kTopkRound - 1) / kTopkRound;
  int rbits = 0;
  while ((1 << rbits) < rounds) ++rbits;
  uint4 cur[kTopkVec], nxt[kTopkVec];
  int seq = 0;
  // next round index in bit-reversed order, skipping indices past `rounds`
  auto next_round = [&]() {
    while (seq < (1 << rbits)) {
      const int cand = (int)bit_reverse((uint32_t)seq++, rbits);
      if (cand < rounds) return cand;
    }
    return -1;
  };
  auto load_round = [&](int r, uint4 (&buf)[kTopkVec]) {
#pragma unroll
    for (int u = 0; u < kTopkVec; ++u) {
      const int e0 = r * kTopkRound + 4 * (tid + u * NT);
      if (vec && e0 + 3 < n) {
        buf[u] = __ldcs(reinterpret_cast<const uint4*>(src + e0));
      } else {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          w[k] = (e0 + k < n) ? __float_as_uint(__ldcs(src + e0 + k)) : kNegInfBits;
        buf[u] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  };
  int r = rounds > 0 ? next_round() : -1;
  if (r >= 0) load_round(r, cur);
  while (r >= 0) {
    const int rn = next_round();
    if (rn >= 0) load_round(rn, nxt);
#pragma unroll
    for (int u = 0; u < kTopkVec; ++u) {
      const int e0 = r * kTopkRound + 4 * (tid + u * NT);
      const uint32_t w[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        filter_offer(fs, fb, fi, w[k], (uint32_t)(c0 + e0 + k), e0 + k < n);
      group_sync(NT);
      // every thread reads the count before anyone offers again: one decision
      const int cnt = fs.count;
      group_sync(NT);
      if (cnt > compact_at) filter_compact<NT>(fs, fb, fi, a.K, sc);
    }
#pragma unroll
    for (int u = 0; u < kTopkVec; ++u) cur[u] = nxt[u];
    r = rn;
  }
  group_sync(NT);
  filter_compact<NT>(fs, fb, fi, a.K, sc);
  const int kk = fs.count;
  if (nch == 1) {
    sort_and_write<NT>(fb, fi, kk, a.K, sortv, sortb, io, vo);
    return;
  }
  const int64_t slot = (int64_t)row * a.max_chunks + ch;
  publish_candidates<NT>(fb, fi, kk, a.K, fs.thr, a.cand_bits + slot * a.slot_stride,
                         a.cand_idx + slot * a.slot_stride, a.row_thr + row);
  if (!arrive_last<NT>(a.arrive + row, nch, s_flag)) return;
  const int64_t base = (int64_t)row * a.max_chunks;
  merge_candidates<NT>(
      nch, [base](int i) { return base + i; }, a.cand_bits, a.cand_idx, a.slot_stride, a.K, a.K,
      a.row_thr + row, fs, fb, fi, kFilterCap, sc, sortv, sortb, io, vo);
}

int topk_plan_chunk(int rows, int N, int K, int num_sms) {
  (void)K;
  int chunk = kTopkMaxChunk;
  while (chunk > kTopkMinChunk &&
         (int64_t)rows * ((N + chunk - 1) / chunk) < 3 * (int64_t)num_sms)
    chunk >>= 1;
  return chunk;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream) {
  const TopkLayout L = topk_layout();
  cudaError_t e = cudaFuncSetAttribute(topk_chunk_kernel<kTopkThreads>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  const int nch = a.N > 0 ? (a.N + a.chunk - 1) / a.chunk : 1;
  dim3 grid(nch, a.rows);
  topk_chunk_kernel<kTopkThreads><<<grid, kTopkThreads, L.total, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace idx
