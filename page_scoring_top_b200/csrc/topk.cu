// topk.cu -- standalone exact top-K over fp32 score rows ("Iterate Topk",
// opening description: given per-segment scores, return the top-K indices).
//
// Grid (chunks, rows).  Each CTA loads one chunk of a row into shared memory
// with coalesced 16-byte loads, selects the chunk's exact top-K' with the
// block radix select, and either writes the final row directly (a row that
// fits one chunk) or publishes its candidates; the last CTA of the row to
// arrive merges them.  Short rows therefore take one CTA and one HBM read;
// long rows spread over many SMs and still read every score exactly once.
#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"

namespace idx {

constexpr int kTopkThreads = 512;
constexpr int kTopkMaxChunk = 8192;
constexpr int kTopkMinChunk = 2048;

struct TopkLayout {
  size_t bits, gidx, win, scratch, flag, total;
};

__host__ __device__ inline TopkLayout topk_layout(int cap, int K) {
  TopkLayout L;
  size_t o = 0;
  L.bits = o;
  o += (size_t)cap * 4;
  L.gidx = o;
  o += (size_t)cap * 4;
  L.win = o;
  o += ((size_t)K * 4 + 15) & ~(size_t)15;
  L.scratch = o;
  size_t sortb = (size_t)next_pow2(K) * 8;
  o += (sizeof(SelectScratch) > sortb ? sizeof(SelectScratch) : sortb);
  o = (o + 15) & ~(size_t)15;
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

// Copy n fp32 bit patterns from global memory into shared memory.
template <int NT>
__device__ __forceinline__ void load_bits(uint32_t* dst, const float* src, int n) {
  const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    const int n4 = n >> 2;
    const uint4* s4 = reinterpret_cast<const uint4*>(s);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    constexpr int U = 4;
    for (int base = threadIdx.x; base < n4; base += NT * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (base + u * NT < n4) v[u] = __ldcs(s4 + base + u * NT);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (base + u * NT < n4) d4[base + u * NT] = v[u];
    }
    for (int i = (n4 << 2) + threadIdx.x; i < n; i += NT) dst[i] = __ldcs(s + i);
  } else {
    for (int i = threadIdx.x; i < n; i += NT) dst[i] = __ldcs(s + i);
  }
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_chunk_kernel(const TopkArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int cap = a.chunk > 2 * a.K ? a.chunk : 2 * a.K;
  const TopkLayout L = topk_layout(cap, a.K);
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + L.bits);
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem + L.gidx);
  int* win_pos = reinterpret_cast<int*>(smem + L.win);
  SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem + L.scratch);
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(smem + L.scratch);
  int* s_flag = reinterpret_cast<int*>(smem + L.flag);

  const int row = blockIdx.y;
  const int ch = blockIdx.x;
  const int len =
      clamp_len(a.lengths, row / a.len_div, a.N, a.status, ch == 0 && threadIdx.x == 0);
  const int nch = len > 0 ? (len + a.chunk - 1) / a.chunk : 1;
  if (ch >= nch) return;
  const int c0 = ch * a.chunk;
  const int n = max(0, min(a.chunk, len - c0));

  int32_t* io = a.idx_out + (int64_t)row * a.K;
  float* vo = a.val_out ? a.val_out + (int64_t)row * a.K : nullptr;

  load_bits<NT>(s_bits, a.scores + (int64_t)row * a.lds + c0, n);
  group_sync(NT);
  const int kk = block_select<NT>(s_bits, n, a.K, win_pos, sc);
  if (nch == 1) {
    sort_and_write<NT>(s_bits, nullptr, 0, win_pos, kk, a.K, sortbuf, io, vo);
    return;
  }
  const int64_t slot = (int64_t)row * a.max_chunks + ch;
  uint32_t* cb = a.cand_bits + slot * a.slot_stride;
  int32_t* ci = a.cand_idx + slot * a.slot_stride;
  for (int k = threadIdx.x; k < kk; k += NT) {
    const int p = win_pos[k];
    cb[k] = s_bits[p];
    ci[k] = c0 + p;
  }
  if (threadIdx.x == 0) a.cand_cnt[slot] = kk;
  if (!arrive_last<NT>(a.arrive + row, nch, s_flag)) return;
  const int64_t base = (int64_t)row * a.max_chunks;
  merge_candidates<NT>(
      nch, [base](int i) { return base + i; }, a.cand_bits, a.cand_idx, a.cand_cnt,
      a.slot_stride, a.K, cap, s_bits, s_idx, win_pos, sc, sortbuf, io, vo);
}

int topk_plan_chunk(int rows, int N, int K, int num_sms) {
  int chunk = kTopkMaxChunk;
  const int floor_chunk = kTopkMinChunk > 2 * K ? kTopkMinChunk : next_pow2(2 * K);
  while (chunk > floor_chunk &&
         (int64_t)rows * ((N + chunk - 1) / chunk) < 2 * (int64_t)num_sms)
    chunk >>= 1;
  if (chunk < floor_chunk) chunk = floor_chunk;
  return chunk;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream) {
  const int cap = a.chunk > 2 * a.K ? a.chunk : 2 * a.K;
  const TopkLayout L = topk_layout(cap, a.K);
  cudaError_t e = cudaFuncSetAttribute(topk_chunk_kernel<kTopkThreads>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  const int nch = a.N > 0 ? (a.N + a.chunk - 1) / a.chunk : 1;
  dim3 grid(nch, a.rows);
  topk_chunk_kernel<kTopkThreads><<<grid, kTopkThreads, L.total, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace idx
