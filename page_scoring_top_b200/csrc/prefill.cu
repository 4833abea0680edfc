// prefill.cu -- tensor-core (tcgen05 / TMEM) scoring of multi-token prefill chunks.
//
// "Round 15 Track C Audit", section 1 Target 1 item 3: a prefill chunk scores
// every token of a 16-token tile against the same pages with one matrix
// product (qsa_score_mm's matmul2d).  Here, per request b,
//     Acc[m, p] = sum_d A[m, d] * c[b, p, d],   A = q[b] viewed as [T*Q, D]
// (row m = t*Q + h), is a real dense contraction: bf16 operands, fp32
// accumulation, M = T*Q <= 128 rows, N = pages, K = D = 128.  The score is the
// head-sum s[b, t, p] = sum_h Acc[t*Q + h, p], taken on the fp32 accumulators
// as they leave TMEM (pre-summing the heads in bf16 would round them).
//
// sm_100a design, one persistent CTA per SM, 6 warps:
//  * warp 0   TMA producer: the request's A tile (32 KB, loaded when the
//             request changes) and 256-page B tiles (64 KB) into a 3-stage
//             ring, both in the 128-byte-swizzled K-major layout;
//  * warp 1   MMA issuer: one thread issues 8 tcgen05.mma (M128 N256 K16)
//             per tile into one of two TMEM accumulators (2 x 256 fp32
//             columns = all 512), then tcgen05.commit frees the B stage and
//             hands the accumulator to the epilogue;
//  * warps 2-5 epilogue: tcgen05.ld 32 columns at a time (each warp owns one
//             32-lane TMEM quadrant = 32/Q tokens), head-sum across the Q
//             lanes of a token with a transposed shuffle butterfly, 16-byte
//             stores of the scores, then free the accumulator.
// The contraction is HBM-bound at this shape (128 flop per byte of c, below
// the B200 ridge), so the MMA and the epilogue hide under the TMA stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace idx {

constexpr int kPfThreads = 192;
constexpr int kPfTileN = 256;   // pages per tile (MMA N)
constexpr int kPfM = 128;       // MMA M (rows t*Q + h, zero-padded)
constexpr int kPfD = 128;       // head dim (MMA K in total)
constexpr int kPfStages = 3;
constexpr int kPfMaxB = 256;  // requests per launch (the host splits larger batches)
constexpr uint32_t kPfABytes = kPfM * kPfD * 2;          // 32 KB
constexpr uint32_t kPfBBytes = kPfTileN * kPfD * 2;      // 64 KB
constexpr uint32_t kPfBlockA = kPfM * 128;               // one 64-column K-block of A
constexpr uint32_t kPfBlockB = kPfTileN * 128;           // one 64-column K-block of B

struct PfSmem {
  // offsets from the 1024-aligned dynamic smem base: the small state first,
  // then the swizzled operand buffers on 1024-byte boundaries
  static constexpr size_t bars = 0;  // full[3], empty[3], a_full, a_empty, acc_full[2], acc_empty[2]
  static constexpr size_t tmem_slot = bars + 16 * 8;
  static constexpr size_t misc = tmem_slot + 16;               // abort flag, warp sums
  static constexpr size_t tiles = misc + 64;                   // tile prefix [kPfMaxB + 1]
  static constexpr size_t a = 2048;
  static constexpr size_t b = a + kPfABytes;
  static constexpr size_t total = b + (size_t)kPfStages * kPfBBytes + 1024;  // + alignment slack
  static_assert(tiles + (kPfMaxB + 1) * 4 <= a, "small state overflows");
};

constexpr uint32_t kPfIdesc = umma_idesc_bf16(kPfM, kPfTileN);

struct PfParams {
  PrefillArgs a;
  int rows_per_req;  // T * Q
};

// Tile t of this CTA's sequence -> (request, first page).  s_tiles[b] is the
// number of 256-page tiles before request b.
__device__ __forceinline__ void tile_coords(const int* s_tiles, int B, int tile, int& b, int& p0) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (s_tiles[mid + 1] > tile) hi = mid;
    else lo = mid + 1;
  }
  b = lo;
  p0 = (tile - s_tiles[lo]) * kPfTileN;
}

template <int Q>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_c,
                   const PfParams pp) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const PrefillArgs& a = pp.a;
  unsigned char* sA = smem + PfSmem::a;
  unsigned char* sB = smem + PfSmem::b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PfSmem::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kPfStages;
  uint64_t* a_full = bars + 2 * kPfStages;
  uint64_t* a_empty = a_full + 1;
  uint64_t* acc_full = a_full + 2;
  uint64_t* acc_empty = a_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PfSmem::tmem_slot);
  int* s_tiles = reinterpret_cast<int*>(smem + PfSmem::tiles);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + PfSmem::misc);
  uint32_t* s_wsum = reinterpret_cast<uint32_t*>(smem + PfSmem::misc + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int B = a.B, N = a.N, T = a.T;
  const int R = pp.rows_per_req;

  if (tid == 0) {
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrival per epilogue warp
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {  // TMEM: two 256-column fp32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // Per-request tile counts (ceil(len/256)) and their prefix, plus clamped lengths.
  {
    int running = 0;
    if (tid == 0) s_tiles[0] = 0;
    for (int base = 0; base < B; base += kPfThreads) {
      const int i = base + tid;
      int nt = 0;
      if (i < B) {
        int len = a.lengths ? a.lengths[i] : N;
        if (len < 0 || len > N) {
          if (g == 0) atomicOr(a.status, kErrLengthClamped);
          len = len < 0 ? 0 : N;
        }
        nt = (len + kPfTileN - 1) / kPfTileN;
      }
      const uint32_t incl = warp_incl_scan((uint32_t)nt);
      if (lane == 31) s_wsum[warp] = incl;
      __syncthreads();
      uint32_t excl = incl - (uint32_t)nt, total = 0;
      for (int w = 0; w < kPfThreads / 32; ++w) {
        if (w < warp) excl += s_wsum[w];
        total += s_wsum[w];
      }
      if (i < B) s_tiles[i + 1] = running + (int)excl + nt;
      __syncthreads();
      running += (int)total;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = s_tiles[B];
  const int my_tiles = ntiles > g ? (ntiles - g + G - 1) / G : 0;

  // -inf for the padded pages p >= len[b] of every token row (4096-entry
  // pieces dealt round-robin to the CTAs), by the epilogue warps.
  if (warp >= 2) {
    constexpr int kPiece = 4096;
    const int ppr = (N + kPiece - 1) / kPiece;
    const int64_t npieces = (int64_t)B * T * ppr;
    for (int64_t pc = g; pc < npieces; pc += G) {
      const int rowi = (int)(pc / ppr);
      const int b = rowi / T;
      int lb = a.lengths ? a.lengths[b] : N;
      lb = lb < 0 ? 0 : (lb > N ? N : lb);
      const int k0 = (int)(pc - (int64_t)rowi * ppr) * kPiece;
      const int p_lo = max(lb, k0), p_hi = min(N, k0 + kPiece);
      float* dst = a.scores + (int64_t)rowi * N;
      for (int p = p_lo + tid - 64; p < p_hi; p += 128) dst[p] = __uint_as_float(kNegInfBits);
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int cur_b = -1, a_loads = 0;
      for (int i = 0; i < my_tiles && !*s_abort; ++i) {
        int b, p0;
        tile_coords(s_tiles, B, g + i * G, b, p0);
        if (b != cur_b) {
          if (a_loads > 0) mbar_wait_bounded(a_empty, (a_loads - 1) & 1, s_abort, a.status);
          mbar_arrive_expect_tx(a_full, kPfABytes);
          tma_load_2d(sA, &map_q, 0, b * R, a_full);
          tma_load_2d(sA + kPfBlockA, &map_q, 64, b * R, a_full);
          ++a_loads;
          cur_b = b;
        }
        const int s = i % kPfStages;
        if (i >= kPfStages) mbar_wait_bounded(&empty[s], ((i / kPfStages) - 1) & 1, s_abort, a.status);
        unsigned char* dst = sB + (size_t)s * kPfBBytes;
        mbar_arrive_expect_tx(&full[s], kPfBBytes);
        tma_load_3d(dst, &map_c, 0, p0, b, &full[s]);
        tma_load_3d(dst + kPfBlockB, &map_c, 64, p0, b, &full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int cur_b = -1, a_loads = 0;
      const uint32_t a_base = smem_u32(sA);
      for (int i = 0; i < my_tiles && !*s_abort; ++i) {
        int b, p0;
        tile_coords(s_tiles, B, g + i * G, b, p0);
        if (b != cur_b) {
          if (a_loads > 0) umma_commit(a_empty);  // previous A is free once its MMAs finish
          mbar_wait_bounded(a_full, a_loads & 1, s_abort, a.status);
          ++a_loads;
          cur_b = b;
        }
        const int s = i % kPfStages;
        const int acc = i & 1;
        mbar_wait_bounded(&full[s], (i / kPfStages) & 1, s_abort, a.status);
        if (i >= 2) mbar_wait_bounded(&acc_empty[acc], ((i >> 1) - 1) & 1, s_abort, a.status);
        tc_fence_after();
        const uint32_t b_base = smem_u32(sB + (size_t)s * kPfBBytes);
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * kPfTileN;
#pragma unroll
        for (int k = 0; k < kPfD / 16; ++k) {
          const uint32_t kb = (uint32_t)(k >> 2), ks = (uint32_t)(k & 3);
          const uint64_t ad = umma_desc_sw128(a_base + kb * kPfBlockA + ks * 32u);
          const uint64_t bd = umma_desc_sw128(b_base + kb * kPfBlockB + ks * 32u);
          umma_bf16(d_tmem, ad, bd, kPfIdesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        umma_commit(&acc_full[acc]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes quad*32 .. quad*32+31
    constexpr int TPW = 32 / Q;     // tokens per warp
    constexpr int VPL = 32 / Q;     // columns each lane keeps after the head-sum
    const int t_local = lane / Q;   // token of this lane within the warp
    for (int i = 0; i < my_tiles && !*s_abort; ++i) {
      int b, p0;
      tile_coords(s_tiles, B, g + i * G, b, p0);
      int lb = a.lengths ? a.lengths[b] : N;
      lb = lb < 0 ? 0 : (lb > N ? N : lb);
      const int acc = i & 1;
      mbar_wait_bounded(&acc_full[acc], (i >> 1) & 1, s_abort, a.status);
      tc_fence_after();
      const int t = quad * TPW + t_local;  // token whose heads this lane's row belongs to
#pragma unroll 1
      for (int chunk = 0; chunk < kPfTileN / 32; ++chunk) {
        uint32_t raw[32];
        tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)acc * kPfTileN +
                      (uint32_t)chunk * 32,
                  raw);
        float v[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(raw[k]);
        // transposed butterfly over the Q lanes of a token: after it, lane
        // (token, j) holds the head-sums of columns j*VPL .. j*VPL+VPL-1
#pragma unroll
        for (int m = Q / 2, half = 16; m >= 1; m >>= 1, half >>= 1) {
          const bool up = (lane & m) != 0;
#pragma unroll
          for (int k = 0; k < half; ++k) {
            const float send = up ? v[k] : v[k + half];
            const float keep = up ? v[k + half] : v[k];
            v[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, m);
          }
        }
        const int j = lane & (Q - 1);
        int col0 = 0;  // column block this lane holds: bit-reversed order of the steps
#pragma unroll
        for (int m = Q / 2, blk = VPL * (Q / 2); m >= 1; m >>= 1, blk >>= 1)
          if (j & m) col0 += blk;
        const int p = p0 + chunk * 32 + col0;
        if (t < T && p < lb) {
          float* dst = a.scores + ((int64_t)b * T + t) * N + p;
          if ((VPL % 4) == 0 && p + VPL <= lb && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
            for (int k = 0; k < VPL; k += 4)
              *reinterpret_cast<float4*>(dst + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
          } else {
#pragma unroll
            for (int k = 0; k < VPL; ++k)
              if (p + k < lb) dst[k] = v[k];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512u)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool prefill_supported(int T, int Q, int D, int64_t ldc_b) {
  const bool q_pow2 = Q == 1 || Q == 2 || Q == 4 || Q == 8 || Q == 16 || Q == 32;
  return D == kPfD && q_pow2 && T * Q >= 32 && T * Q <= kPfM && (ldc_b % 8) == 0;
}

template <int Q>
static cudaError_t launch_q(const CUtensorMap& mq, const CUtensorMap& mc, const PfParams& pp, int grid,
                            cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<Q>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PfSmem::total);
  if (e != cudaSuccess) return e;
  prefill_kernel<Q><<<grid, kPfThreads, PfSmem::total, stream>>>(mq, mc, pp);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillArgs& a, int num_sms, cudaStream_t stream) {
  static_assert(PfSmem::total <= 227 * 1024, "prefill shared memory");
  if (!prefill_supported(a.T, a.Q, a.D, a.ldc_b) || a.B > kPfMaxB) return cudaErrorNotSupported;
  auto encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap mq, mc;
  // q as [B*T*Q rows][D] bf16; box 64 columns (128 B) x 128 rows, 128-byte swizzle
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.D, (cuuint64_t)a.B * a.T * a.Q};
    const cuuint64_t strides[1] = {(cuuint64_t)a.D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kPfM};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // c as [B][N][D] bf16 with request stride ldc_b; box 64 x 256 pages x 1
  {
    const cuuint64_t dims[3] = {(cuuint64_t)a.D, (cuuint64_t)a.N, (cuuint64_t)a.B};
    const cuuint64_t strides[2] = {(cuuint64_t)a.D * 2, (cuuint64_t)a.ldc_b * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kPfTileN, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(a.c), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  PfParams pp;
  pp.a = a;
  pp.rows_per_req = a.T * a.Q;
  const int grid = num_sms;
  switch (a.Q) {
    case 1: return launch_q<1>(mq, mc, pp, grid, stream);
    case 2: return launch_q<2>(mq, mc, pp, grid, stream);
    case 4: return launch_q<4>(mq, mc, pp, grid, stream);
    case 8: return launch_q<8>(mq, mc, pp, grid, stream);
    case 16: return launch_q<16>(mq, mc, pp, grid, stream);
    default: return launch_q<32>(mq, mc, pp, grid, stream);
  }
}

}  // namespace idx
