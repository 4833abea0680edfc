// kernels.h -- internal launch interface between the C ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace idx {

constexpr int kMaxK = 2048;  // the ABI's IDX_MAX_K

// ---------------------------------------------------------------- top-K select
struct TopkArgs {
  const float* scores;
  const int32_t* lengths;  // or null (all N); row r uses lengths[r / len_div]
  int len_div;
  int rows, N;
  int64_t lds;
  int K;
  int chunk;       // elements per CTA (power of two)
  int max_chunks;  // candidate slots per row
  int64_t slot_stride;  // entries per candidate slot (>= K)
  int32_t* idx_out;
  float* val_out;  // may be null
  uint32_t* cand_bits;
  int32_t* cand_idx;
  unsigned long long* row_thr;  // per-row shared thresholds, zero between calls
  int32_t* arrive;  // per-row arrival counters, zero between calls
  int* status;
};
// Candidate slots the launch needs: rows * max_chunks, each of K entries.
int topk_plan_chunk(int rows, int N, int K, int num_sms);
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream);

// Streamed top-K (topk_stream.cu): one persistent CTA per SM over the rows laid
// end to end.  Needs 16-byte aligned scores and lds % 4 == 0; at most
// topk_stream_max_rows(N) rows of N entries per launch (the entries of a
// launch, with their per-row charges, are counted in 32 bits; 0 when even one
// row does not fit); candidate slots (chunk + row) of
// slot_stride entries, and per-row thresholds and arrival counters that are
// zero between calls.
struct TopkStreamArgs {
  const float* scores;
  const int32_t* lengths;  // or null (all N); row r uses lengths[r / len_div]
  int len_div;
  int rows, N;
  int64_t lds;
  int K;
  int32_t* idx_out;
  float* val_out;  // may be null
  uint32_t* cand_bits;
  int32_t* cand_idx;
  int64_t slot_stride;
  unsigned long long* row_thr;
  int32_t* arrive;
  int* status;
};
bool topk_stream_supported(const float* scores, int64_t lds);
int64_t topk_stream_slots(int rows, int num_sms);
int topk_stream_max_rows(int N);
cudaError_t launch_topk_stream(const TopkStreamArgs& a, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- decode score / fused select
struct DecodeArgs {
  const uint16_t* q;
  const uint16_t* c;
  const int32_t* lengths;      // per request, or null
  const int32_t* tok_lengths;  // per (request, token) [B*T] instead of lengths, or null
  // paged centroids: page p of request b is row page_table[b*ld_pt + p] of
  // the block pool `c` ([n_blocks][D]); null for contiguous per-request rows
  const int32_t* page_table;
  int64_t ld_pt;
  int n_blocks;
  int B, T, Q, D, N;
  int64_t ldc_b;
  int K;
  float* scores;    // score mode: [B][T][N]
  int32_t* idx_out; // fused mode: [B*T][K]
  float* val_out;   // fused mode, may be null
  uint32_t* cand_bits;
  int32_t* cand_idx;
  int64_t slot_stride;          // entries per candidate slot (>= K)
  unsigned long long* row_thr;  // per-row shared thresholds, zero between calls
  int32_t* arrive;              // per-request arrival counters, zero between calls
  int* status;
};
constexpr int kDecodeMaxB = 1024;       // requests per launch (host splits larger batches)
constexpr int kDecodeMaxTFused = 4;     // tokens per request on the fused CUDA-core path
// Candidate slots a fused launch of B requests x T tokens can use.
int64_t decode_fused_slots(int64_t B, int64_t T, int64_t N, int grid);
// Largest K the fused CUDA-core path takes for T tokens (its on-chip filter).
int decode_fused_max_k(int T);
int decode_grid(int num_sms);
cudaError_t launch_decode(const DecodeArgs& a, bool fused, int num_sms, cudaStream_t stream);
// Tensor-core decode kernel (decode_tc.cu): D in {64, 128}, T*Q <= 64,
// 16-byte aligned request rows.  launch_decode routes these shapes to it.
bool decode_tc_supported(int T, int Q, int D, int64_t ldc_b, const void* c);
cudaError_t launch_decode_tc(const DecodeArgs& a, bool fused, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- prefill (tcgen05) score
struct PrefillArgs {
  const uint16_t* q;
  const uint16_t* c;
  const int32_t* lengths;
  int B, T, Q, D, N;
  int64_t ldc_b;
  float* scores;  // [B][T][N]
  int* status;
};
constexpr int kPrefillMaxB = 256;  // requests per launch (host splits larger batches)
bool prefill_supported(int T, int Q, int D, int64_t ldc_b);
cudaError_t launch_prefill(const PrefillArgs& a, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- KMeans assignment
struct KmeansArgs {
  const uint16_t* x;     // bf16 [M][D], 16-byte aligned rows
  const uint16_t* cent;  // bf16 [C][D]
  int M, C, D;
  float* hn;             // [C] workspace: -|c|^2 / 2
  int32_t* assign;       // [M] (assignment mode)
  float* score;          // [M] or null (assignment mode)
  float* scores;         // [M][C] (score mode)
  int* status;
};
bool kmeans_supported(int D);
// Computes hn, then the assignment (scores == false) or the score matrix.
cudaError_t launch_kmeans(const KmeansArgs& a, bool scores, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- page centroids
struct PoolArgs {
  const uint16_t* keys;        // bf16, key i of request b at keys + b*ldk_b + i*D
  const int32_t* key_counts;   // [B] valid keys per request
  int B, D, P, N;              // P keys per page, N pages per request
  int64_t ldk_b, ldc_b;
  uint16_t* c;                 // bf16 [B][N][D] with request stride ldc_b
  int* status;
};
cudaError_t launch_pool(const PoolArgs& a, int num_sms, cudaStream_t stream);

}  // namespace idx
