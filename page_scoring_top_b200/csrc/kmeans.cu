// kmeans.cu -- KMeans assignment on the tensor cores (tcgen05 / TMEM).
//
// What is computed ("Export Cake KMeans plan-runtime suite", summary:
// assignments = compute(x, centroids) on raw bf16 inputs): every point goes
// to its nearest centroid.  |x - c|^2 = |x|^2 - 2 s[i,c] with
//     s[i,c] = sum_d x[i,d] * c[c,d] - h[c],   h[c] = (sum_d c[c,d]^2) / 2,
// so the assignment is argmax_c s[i,c], equal scores to the lower centroid.
// The dot products are a dense contraction, points x centroids x D: bf16
// operands, fp32 accumulation in TMEM.  h is computed once per call in fp32
// (kmeans_norms_kernel) and subtracted as the accumulators leave TMEM.
//
// One persistent CTA per SM over 128-point tiles, 10 warps:
//  * warp 0   TMA producer: the point tile (double-buffered) and 256-centroid
//             tiles (2-stage ring), 128-byte swizzled K-major; columns past
//             D (and rows past M or C) arrive as zeros;
//  * warp 1   MMA issuer: one thread issues D/16 tcgen05.mma (M128 N256 K16)
//             per (point tile, centroid tile) into one of two TMEM
//             accumulators of 256 fp32 columns;
//  * warps 2-9 epilogue, two warpgroups: warpgroup g reads columns
//             128 g .. 128 g + 127 of each accumulator (each warp its
//             32-lane quadrant = 32 points), adds -h with paired adds, and
//             keeps a running best per point (-h is staged in shared memory
//             by the same warps, one tile ahead): the maximum of each
//             32-column chunk is a tree of three-input maxima, and only a
//             chunk that beats the best so far is searched for its first
//             maximal column.  At the end of a point tile the two halves
//             are combined (the lower columns win ties) and the assignment
//             (and its score) written.
// Score mode writes s[i,c] instead, from the same arithmetic, so an
// assignment equals the row argmax of the score matrix bit for bit.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace idx {

PFN_cuTensorMapEncodeTiled_v12000 get_encode();

namespace {

constexpr int kKmThreads = 320;
constexpr int kKmEpiWarps = 8;
constexpr int kKmM = 128;       // points per tile (MMA M)
constexpr int kKmN = 256;       // centroids per tile (MMA N)
constexpr int kKmMaxD = 128;    // two 64-column K blocks
constexpr int kKmBStages = 2;
constexpr uint32_t kKmABytes = kKmM * kKmMaxD * 2;   // 32 KB
constexpr uint32_t kKmBBytes = kKmN * kKmMaxD * 2;   // 64 KB
constexpr uint32_t kKmBlockA = kKmM * 128;           // one 64-column K block of A
constexpr uint32_t kKmBlockB = kKmN * 128;           // one 64-column K block of B
constexpr uint32_t kKmIdesc = umma_idesc_bf16(kKmM, kKmN);

// Shared-memory layout (offsets from the 1024-aligned base).
struct KmSmem {
  // full[2], empty[2], a_full[2], a_empty[2], acc_full[2], acc_empty[2]
  static constexpr size_t bars = 0;
  static constexpr size_t tmem_slot = bars + 16 * 8;
  static constexpr size_t misc = tmem_slot + 16;      // abort flag
  static constexpr size_t best = misc + 64;           // [kKmM] value + [kKmM] index, upper half
  static constexpr size_t hn = 2048;                  // [2][kKmN] floats (by accumulator)
  static constexpr size_t a = 4096;                   // [2] point tiles
  static constexpr size_t b = a + 2 * (size_t)kKmABytes;  // [kKmBStages] centroid tiles
  static constexpr size_t total = b + (size_t)kKmBStages * kKmBBytes + 1024;  // + alignment slack
  static_assert(best + 2 * kKmM * 4 <= hn, "small state overflows");
  static_assert(hn + 2 * (size_t)kKmN * 4 <= a, "h area overflows");
};

// x0 += y0, x1 += y1: one paired fp32 add (add.rn.f32x2), each lane rounded
// to nearest like a scalar add.
__device__ __forceinline__ void add_pair(float& x0, float& x1, float y0, float y1) {
  asm("{\n\t.reg .b64 u, v;\n\t"
      "mov.b64 u, {%0, %1};\n\t"
      "mov.b64 v, {%2, %3};\n\t"
      "add.rn.f32x2 u, u, v;\n\t"
      "mov.b64 {%0, %1}, u;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(y0), "f"(y1));
}

// The largest of three (a NaN input is ignored, as by fmaxf).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The largest of 32: three-input maxima 32 -> 11 -> 4 -> 1.
__device__ __forceinline__ float max32(const float (&v)[32]) {
  float t[11];
#pragma unroll
  for (int j = 0; j < 10; ++j) t[j] = max3(v[3 * j], v[3 * j + 1], v[3 * j + 2]);
  t[10] = fmaxf(v[30], v[31]);
  const float u0 = max3(t[0], t[1], t[2]), u1 = max3(t[3], t[4], t[5]);
  const float u2 = max3(t[6], t[7], t[8]), u3 = fmaxf(t[9], t[10]);
  return fmaxf(max3(u0, u1, u2), u3);
}

// h[c] = (sum_d c[c,d]^2) / 2 in fp32, d in order; one thread per centroid.
__global__ void kmeans_norms_kernel(const uint16_t* cent, int C, int D, float* hn) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  const uint16_t* row = cent + (int64_t)c * D;
  float s = 0.f;
  for (int d = 0; d < D; d += 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + d);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
      s = fmaf(lo, lo, s);
      s = fmaf(hi, hi, s);
    }
  }
  hn[c] = -0.5f * s;  // stored negated: the epilogue adds it
}

// The main kernel.  SCORES: write s[i,c] to a.scores instead of assigning.
template <bool SCORES>
__global__ void __launch_bounds__(kKmThreads, 1)
    kmeans_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_c,
                  const KmeansArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KmSmem::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + 2;
  uint64_t* a_full = bars + 4;
  uint64_t* a_empty = bars + 6;
  uint64_t* acc_full = bars + 8;
  uint64_t* acc_empty = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + KmSmem::tmem_slot);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + KmSmem::misc);
  float* s_h = reinterpret_cast<float*>(smem + KmSmem::hn);
  float* s_bval = reinterpret_cast<float*>(smem + KmSmem::best);
  int* s_bidx = reinterpret_cast<int*>(smem + KmSmem::best + kKmM * 4);
  unsigned char* sA = smem + KmSmem::a;
  unsigned char* sB = smem + KmSmem::b;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int M = a.M, C = a.C;
  const int KB = (a.D + 63) / 64;  // 64-column K blocks (the last zero-filled past D)
  const int nmt = (M + kKmM - 1) / kKmM, nct = (C + kKmN - 1) / kKmN;
  const int my_tiles = nmt > g ? (nmt - g + G - 1) / G : 0;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kKmEpiWarps);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512u);  // two 256-column fp32 accumulators
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int i = 0;
      for (int lt = 0; lt < my_tiles && !*s_abort; ++lt) {
        const int m = g + lt * G, buf = lt & 1;
        if (lt >= 2) mbar_wait_bounded(&a_empty[buf], ((lt >> 1) - 1) & 1, s_abort, a.status);
        unsigned char* dA = sA + (size_t)buf * kKmABytes;
        mbar_arrive_expect_tx(&a_full[buf], (uint32_t)KB * kKmBlockA);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(dA + kb * kKmBlockA, &map_x, kb * 64, m * kKmM, &a_full[buf]);
        for (int n = 0; n < nct; ++n, ++i) {
          const int s = i & 1;
          if (i >= 2) mbar_wait_bounded(&empty[s], ((i >> 1) - 1) & 1, s_abort, a.status);
          unsigned char* dB = sB + (size_t)s * kKmBBytes;
          mbar_arrive_expect_tx(&full[s], (uint32_t)KB * kKmBlockB);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(dB + kb * kKmBlockB, &map_c, kb * 64, n * kKmN, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int i = 0;
      for (int lt = 0; lt < my_tiles && !*s_abort; ++lt) {
        const int buf = lt & 1;
        mbar_wait_bounded(&a_full[buf], (lt >> 1) & 1, s_abort, a.status);
        const uint32_t a_base = smem_u32(sA + (size_t)buf * kKmABytes);
        for (int n = 0; n < nct; ++n, ++i) {
          const int s = i & 1, acc = i & 1;
          mbar_wait_bounded(&full[s], (i >> 1) & 1, s_abort, a.status);
          if (i >= 2) mbar_wait_bounded(&acc_empty[acc], ((i >> 1) - 1) & 1, s_abort, a.status);
          tc_fence_after();
          if (!*s_abort) {
            const uint32_t b_base = smem_u32(sB + (size_t)s * kKmBBytes);
            const uint32_t d_tmem = tmem_base + (uint32_t)acc * kKmN;
            for (int k = 0; k < KB * 4; ++k) {
              const uint32_t kb = (uint32_t)(k >> 2), ks = (uint32_t)(k & 3);
              const uint64_t ad = umma_desc_sw128(a_base + kb * kKmBlockA + ks * 32u);
              const uint64_t bd = umma_desc_sw128(b_base + kb * kKmBlockB + ks * 32u);
              umma_bf16(d_tmem, ad, bd, kKmIdesc, k > 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty[s]);
          umma_commit(&acc_full[acc]);
        }
        umma_commit(&a_empty[buf]);  // the point tile is free once its MMAs are done
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int te = tid - 64;                 // 0..255
    const int wg = (warp - 2) >> 2;          // column half of each accumulator
    const int quad = warp & 3;               // TMEM lanes quad*32 .. quad*32+31
    const int row = quad * 32 + lane;        // point of the tile
    const int cbase = wg * (kKmN / 2);
    int i = 0;
    // h of the next centroid tile, loaded a tile ahead (each thread one value)
    float h_next = te < C ? __ldg(a.hn + te) : 0.f;
    // (no early exit on abort: every epilogue thread must reach every barrier;
    // after an abort the waits return at once and the loops run out)
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int m = g + lt * G;
      const int point = m * kKmM + row;
      float best = __uint_as_float(kNegInfBits);
      int bidx = -1;
      for (int n = 0; n < nct; ++n, ++i) {
        const int acc = i & 1;
        float* hs = s_h + acc * kKmN;
        hs[te] = h_next;
        {
          const int nn = n + 1 < nct ? n + 1 : 0;  // the next tile (the first, for the next point tile)
          const int c = nn * kKmN + te;
          h_next = c < C ? __ldg(a.hn + c) : 0.f;
        }
        group_sync(kKmEpiWarps * 32);  // h staged; the tile two back is done with this slice
        mbar_wait_bounded(&acc_full[acc], (i >> 1) & 1, s_abort, a.status);
        tc_fence_after();
        const int c0 = n * kKmN + cbase;
        // 32 columns: subtract h, then (score mode) store, or (assignment)
        // a tree maximum and, only if it beats the best so far, the first
        // column that reaches it
        auto process = [&](const uint32_t (&raw)[32], int ch) {
          float sv[32];
          const float4* h4 = reinterpret_cast<const float4*>(hs + cbase + ch * 32);
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 hv = h4[j4];  // -h
#pragma unroll
            for (int q = 0; q < 4; ++q) sv[4 * j4 + q] = __uint_as_float(raw[4 * j4 + q]);
            add_pair(sv[4 * j4 + 0], sv[4 * j4 + 1], hv.x, hv.y);
            add_pair(sv[4 * j4 + 2], sv[4 * j4 + 3], hv.z, hv.w);
          }
          const int cc = c0 + ch * 32;  // centroid of sv[0]
          if (SCORES) {
            if (point < M) {
              float* dst = a.scores + (int64_t)point * C + cc;
              if (cc + 32 <= C && (C & 3) == 0) {
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4)
                  reinterpret_cast<float4*>(dst)[j4] =
                      make_float4(sv[4 * j4], sv[4 * j4 + 1], sv[4 * j4 + 2], sv[4 * j4 + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (cc + j < C) dst[j] = sv[j];
              }
            }
          } else {
            if (cc + 32 > C) {  // the table's ragged end: columns past C never win
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (cc + j >= C) sv[j] = __uint_as_float(kNegInfBits);
            }
            const float mx = max32(sv);
            if (mx > best) {  // strictly: an earlier chunk keeps its ties
              int jj = 31;
#pragma unroll
              for (int j = 31; j >= 0; --j)
                if (sv[j] == mx) jj = j;
              best = mx;
              bidx = cc + jj;
            }
          }
        };
        // two chunks' TMEM loads in flight per wait; the accumulator is free
        // once the last two are in registers
        const uint32_t taddr =
            tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kKmN + cbase);
        {
          uint32_t ra[32], rb[32];
          tmem_ld32_nowait(taddr, ra);
          tmem_ld32_nowait(taddr + 32, rb);
          tmem_ld_wait();
          process(ra, 0);
          process(rb, 1);
        }
        {
          uint32_t ra[32], rb[32];
          tmem_ld32_nowait(taddr + 64, ra);
          tmem_ld32_nowait(taddr + 96, rb);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[acc]);
          process(ra, 2);
          process(rb, 3);
        }
      }
      if (!SCORES) {
        // the two column halves of every point: the upper half hands its best
        // to the lower, which keeps its own on ties (lower centroids)
        if (wg == 1) {
          s_bval[row] = best;
          s_bidx[row] = bidx;
        }
        group_sync(kKmEpiWarps * 32);
        if (wg == 0 && point < M) {
          const float ob = s_bval[row];
          if (ob > best) {
            best = ob;
            bidx = s_bidx[row];
          }
          a.assign[point] = bidx;
          if (a.score) a.score[point] = best;
        }
        // (the next write of s_bval comes after this tile's readers have
        // passed the next tile's h barrier)
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512u);
  }
}

template <bool SCORES>
cudaError_t launch_km(const CUtensorMap& mx, const CUtensorMap& mc, const KmeansArgs& a, int grid,
                      cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kmeans_kernel<SCORES>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)KmSmem::total);
  if (e != cudaSuccess) return e;
  kmeans_kernel<SCORES><<<grid, kKmThreads, KmSmem::total, stream>>>(mx, mc, a);
  return cudaGetLastError();
}

}  // namespace

bool kmeans_supported(int D) { return D >= 8 && D <= kKmMaxD && (D % 8) == 0; }

cudaError_t launch_kmeans(const KmeansArgs& a, bool scores, int num_sms, cudaStream_t stream) {
  static_assert(KmSmem::total <= 227 * 1024, "kmeans shared memory");
  if (!kmeans_supported(a.D)) return cudaErrorNotSupported;
  auto encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  // h = |c|^2 / 2 for every centroid
  kmeans_norms_kernel<<<(a.C + 255) / 256, 256, 0, stream>>>(a.cent, a.C, a.D, a.hn);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // x as [M rows][D] and the centroids as [C rows][D], bf16; boxes of 64
  // columns (128 B, 128-byte swizzle) x 128 points / 256 centroids
  CUtensorMap mx, mc;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.D, (cuuint64_t)a.M};
    const cuuint64_t strides[1] = {(cuuint64_t)a.D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kKmM};
    if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.x), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.D, (cuuint64_t)a.C};
    const cuuint64_t strides[1] = {(cuuint64_t)a.D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kKmN};
    if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.cent), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int nmt = (a.M + kKmM - 1) / kKmM;
  const int grid = nmt < num_sms ? nmt : num_sms;
  return scores ? launch_km<true>(mx, mc, a, grid, stream) : launch_km<false>(mx, mc, a, grid, stream);
}

}  // namespace idx
