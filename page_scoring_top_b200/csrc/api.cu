// api.cu -- the C ABI of libidx.so: argument checks, workspace, dispatch.
//
// The context follows the two-stage runtime shape of "Export Cake KMeans
// plan-runtime suite" (summary: init() once, then compute() many times): all
// device memory the kernels need is sized from the caller's limits and
// allocated in idx_init; every later call only validates, picks a kernel and
// launches it on the caller's stream.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "idx.h"
#include "kernels.h"

struct idx_ctx {
  int device;
  int max_rows, max_n, max_k;
  int num_sms;
  void* ws;  // one allocation holding everything below
  size_t ws_bytes;
  uint32_t* cand_bits;  // standalone select: cand_slots lists of max_k entries
  int32_t* cand_idx;
  int64_t cand_slots;
  uint32_t* fcand_bits;  // fused decode: fused_slots lists of fused_stride entries
  int32_t* fcand_idx;
  int64_t fused_slots, fused_stride;
  unsigned long long* row_thr;
  int32_t* arrive;
  int* status;
  float* scratch;  // fp32 scores for the score-then-select route
  int64_t scratch_elems;
};

namespace {

// Runs the body with ctx->device current, restoring the caller's device.
class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev_) != cudaSuccess) prev_ = -1;
    if (prev_ != dev) ok_ = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev_ >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev_) cudaSetDevice(prev_);
  }
  bool ok() const { return ok_; }

 private:
  int prev_ = -1;
  bool ok_ = true;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int check_score_args(const idx_ctx* ctx, const uint16_t* q, const uint16_t* c, int B, int T,
                     int Q, int D, int N, int64_t ldc_b) {
  if (!ctx || !q || !c) return IDX_EINVAL;
  if (B <= 0 || T <= 0 || Q <= 0 || D <= 0 || N <= 0) return IDX_EINVAL;
  if (!aligned16(q) || !aligned16(c)) return IDX_EINVAL;
  if (ldc_b < (int64_t)N * D || (ldc_b % 8) != 0) return IDX_EINVAL;
  if ((D % 8) != 0 || D > 256) return IDX_EUNSUPPORTED;
  if ((int64_t)B * T > ctx->max_rows || N > ctx->max_n) return IDX_ENOWORKSPACE;
  // page counts, plus the per-request work charge of the fused split, are ints
  if ((int64_t)B * ((int64_t)N + 1024) > INT32_MAX) return IDX_EUNSUPPORTED;
  return IDX_OK;
}

int check_k(const idx_ctx* ctx, int K) {
  if (K <= 0) return IDX_EINVAL;
  if (K > IDX_MAX_K) return IDX_EUNSUPPORTED;
  if (K > ctx->max_k) return IDX_ENOWORKSPACE;
  return IDX_OK;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? IDX_OK : IDX_ECUDA; }

int run_topk(idx_ctx* ctx, const float* scores, const int32_t* lengths, int len_div, int rows,
             int N, int64_t lds, int K, int32_t* idx_out, float* val_out, cudaStream_t stream) {
  if (idx::topk_stream_supported(scores, lds) && idx::topk_stream_max_rows(N) >= len_div) {
    // the streamed kernel, in blocks of rows; its candidate slots are the
    // fused path's (chunk + row per launch)
    // (a block is a whole number of length groups: rows r use lengths[r / len_div])
    const int rmax = (idx::topk_stream_max_rows(N) / len_div) * len_div;
    for (int r0 = 0; r0 < rows; r0 += rmax) {
      const int nr = std::min(rmax, rows - r0);
      if (idx::topk_stream_slots(nr, ctx->num_sms) > ctx->fused_slots) return IDX_ENOWORKSPACE;
      idx::TopkStreamArgs s{};
      s.scores = scores + (int64_t)r0 * lds;
      s.lengths = lengths ? lengths + r0 / len_div : nullptr;
      s.len_div = len_div;
      s.rows = nr;
      s.N = N;
      s.lds = lds;
      s.K = K;
      s.idx_out = idx_out + (int64_t)r0 * K;
      s.val_out = val_out ? val_out + (int64_t)r0 * K : nullptr;
      s.cand_bits = ctx->fcand_bits;
      s.cand_idx = ctx->fcand_idx;
      s.slot_stride = ctx->fused_stride;
      s.row_thr = ctx->row_thr + r0;
      s.arrive = ctx->arrive + r0;
      s.status = ctx->status;
      const int rc = status_of(idx::launch_topk_stream(s, ctx->num_sms, stream));
      if (rc != IDX_OK) return rc;
    }
    return IDX_OK;
  }
  idx::TopkArgs a{};
  a.scores = scores;
  a.lengths = lengths;
  a.len_div = len_div;
  a.rows = rows;
  a.N = N;
  a.lds = lds;
  a.K = K;
  a.chunk = idx::topk_plan_chunk(rows, N, K, ctx->num_sms);
  a.max_chunks = (int)ceil_div(N, a.chunk);
  if ((int64_t)rows * a.max_chunks > ctx->cand_slots) return IDX_ENOWORKSPACE;
  a.idx_out = idx_out;
  a.val_out = val_out;
  a.cand_bits = ctx->cand_bits;
  a.cand_idx = ctx->cand_idx;
  a.row_thr = ctx->row_thr;
  a.slot_stride = ctx->max_k;
  a.arrive = ctx->arrive;
  a.status = ctx->status;
  return status_of(idx::launch_topk(a, stream));
}

// Scores into `scores` [B][T][N].  Per-token page counts (tok_lengths
// [B*T], lengths unused) always take the decode kernels, which mask each
// token row; the prefill kernel serves whole-request lengths only.
// A paged table (page_table, non-null) also takes the decode kernels.
struct Paged {
  const int32_t* page_table = nullptr;
  int64_t ld_pt = 0;
  int n_blocks = 0;
};

int run_score(idx_ctx* ctx, const uint16_t* q, const uint16_t* c, const int32_t* lengths,
              const int32_t* tok_lengths, int B, int T, int Q, int D, int N, int64_t ldc_b,
              float* scores, cudaStream_t stream, const Paged& pg = Paged()) {
  if (!tok_lengths && !pg.page_table && idx::prefill_supported(T, Q, D, ldc_b)) {
    for (int b0 = 0; b0 < B; b0 += idx::kPrefillMaxB) {
      idx::PrefillArgs p{};
      p.q = q + (int64_t)b0 * T * Q * D;
      p.c = c + (int64_t)b0 * ldc_b;
      p.lengths = lengths ? lengths + b0 : nullptr;
      p.B = std::min(idx::kPrefillMaxB, B - b0);
      p.T = T;
      p.Q = Q;
      p.D = D;
      p.N = N;
      p.ldc_b = ldc_b;
      p.scores = scores + (int64_t)b0 * T * N;
      p.status = ctx->status;
      const int rc = status_of(idx::launch_prefill(p, ctx->num_sms, stream));
      if (rc != IDX_OK) return rc;
    }
    return IDX_OK;
  }
  for (int b0 = 0; b0 < B; b0 += idx::kDecodeMaxB) {
    const int nb = std::min(idx::kDecodeMaxB, B - b0);
    idx::DecodeArgs a{};
    a.q = q + (int64_t)b0 * T * Q * D;
    a.c = c + (int64_t)b0 * ldc_b;
    a.lengths = (lengths && !tok_lengths) ? lengths + b0 : nullptr;
    a.tok_lengths = tok_lengths ? tok_lengths + (int64_t)b0 * T : nullptr;
    if (pg.page_table) {
      a.c = c;  // the shared pool, not offset by request
      a.page_table = pg.page_table + (int64_t)b0 * pg.ld_pt;
      a.ld_pt = pg.ld_pt;
      a.n_blocks = pg.n_blocks;
    }
    a.B = nb;
    a.T = T;
    a.Q = Q;
    a.D = D;
    a.N = N;
    a.ldc_b = ldc_b;
    a.scores = scores + (int64_t)b0 * T * N;
    a.status = ctx->status;
    const int rc = status_of(idx::launch_decode(a, false, ctx->num_sms, stream));
    if (rc != IDX_OK) return rc;
  }
  return IDX_OK;
}

}  // namespace

extern "C" {

IDX_API int idx_init(idx_ctx** out, int device, int max_rows, int max_n, int max_k) {
  if (!out) return IDX_EINVAL;
  *out = nullptr;
  if (max_rows <= 0 || max_n <= 0 || max_k <= 0) return IDX_EINVAL;
  if (max_k > IDX_MAX_K) return IDX_EUNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return IDX_ECUDA;
  DeviceGuard guard(device);
  if (!guard.ok()) return IDX_ECUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return IDX_ECUDA;

  idx_ctx* ctx = new idx_ctx();
  ctx->device = device;
  ctx->max_rows = max_rows;
  ctx->max_n = max_n;
  ctx->max_k = max_k;
  ctx->num_sms = sms;
  // Candidate slots of the standalone select: rows x chunks of at least 2048
  // entries, K entries each.  The fused decode path has its own slots (chunks
  // + requests), wider: a segment publishes about K entries plus one digit
  // bin's worth.
  ctx->cand_slots = (int64_t)max_rows * ceil_div(max_n, 2048);
  int64_t fused_slots = 0;
  for (int t = 1; t <= idx::kDecodeMaxTFused; ++t) {
    const int64_t b = std::min<int64_t>(max_rows / t, idx::kDecodeMaxB);
    if (b > 0)
      fused_slots = std::max(fused_slots,
                             idx::decode_fused_slots(b, t, max_n, idx::decode_grid(sms)));
  }
  ctx->fused_slots = fused_slots;
  // (a multiple of 4 entries: lists are copied 16 bytes at a time)
  ctx->fused_stride = ((int64_t)max_k + std::max(max_k, 256) + 3) & ~(int64_t)3;
  ctx->scratch_elems = (int64_t)max_rows * max_n;
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t o_bits = carve((size_t)ctx->cand_slots * max_k * 4);
  const size_t o_idx = carve((size_t)ctx->cand_slots * max_k * 4);
  const size_t o_fbits = carve((size_t)ctx->fused_slots * ctx->fused_stride * 4);
  const size_t o_fidx = carve((size_t)ctx->fused_slots * ctx->fused_stride * 4);
  const size_t o_thr = carve((size_t)max_rows * 8);
  const size_t o_arr = carve((size_t)max_rows * 4);
  const size_t o_st = carve(16);
  const size_t o_scr = carve((size_t)ctx->scratch_elems * 4);
  ctx->ws_bytes = off;
  char* base = nullptr;
  if (cudaMalloc(&base, off) != cudaSuccess) {
    delete ctx;
    return IDX_ECUDA;
  }
  // Thresholds, counters and the status word start at zero; kernels return
  // them to zero.
  if (cudaMemset(base + o_thr, 0, o_scr - o_thr) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(base);
    delete ctx;
    return IDX_ECUDA;
  }
  ctx->ws = base;
  ctx->cand_bits = reinterpret_cast<uint32_t*>(base + o_bits);
  ctx->cand_idx = reinterpret_cast<int32_t*>(base + o_idx);
  ctx->fcand_bits = reinterpret_cast<uint32_t*>(base + o_fbits);
  ctx->fcand_idx = reinterpret_cast<int32_t*>(base + o_fidx);
  ctx->row_thr = reinterpret_cast<unsigned long long*>(base + o_thr);
  ctx->arrive = reinterpret_cast<int32_t*>(base + o_arr);
  ctx->status = reinterpret_cast<int*>(base + o_st);
  ctx->scratch = reinterpret_cast<float*>(base + o_scr);
  *out = ctx;
  return IDX_OK;
}

IDX_API int idx_destroy(idx_ctx* ctx) {
  if (!ctx) return IDX_OK;
  int rc = IDX_OK;
  {
    DeviceGuard guard(ctx->device);
    if (cudaDeviceSynchronize() != cudaSuccess) rc = IDX_ECUDA;
    if (cudaFree(ctx->ws) != cudaSuccess) rc = IDX_ECUDA;
  }
  delete ctx;
  return rc;
}

IDX_API int centroid_score(idx_ctx* ctx, const uint16_t* q, const uint16_t* c,
                           const int32_t* lengths, int B, int T, int Q, int D, int N,
                           int64_t ldc_b, float* scores, idx_stream stream) {
  int rc = check_score_args(ctx, q, c, B, T, Q, D, N, ldc_b);
  if (rc != IDX_OK) return rc;
  if (!scores || !aligned16(scores)) return IDX_EINVAL;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  return run_score(ctx, q, c, lengths, nullptr, B, T, Q, D, N, ldc_b, scores,
                   (cudaStream_t)stream);
}

IDX_API int centroid_score_tokens(idx_ctx* ctx, const uint16_t* q, const uint16_t* c,
                                  const int32_t* token_lengths, int B, int T, int Q, int D,
                                  int N, int64_t ldc_b, float* scores, idx_stream stream) {
  int rc = check_score_args(ctx, q, c, B, T, Q, D, N, ldc_b);
  if (rc != IDX_OK) return rc;
  if (!token_lengths || !scores || !aligned16(scores)) return IDX_EINVAL;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  return run_score(ctx, q, c, nullptr, token_lengths, B, T, Q, D, N, ldc_b, scores,
                   (cudaStream_t)stream);
}

IDX_API int topk_select(idx_ctx* ctx, const float* scores, const int32_t* lengths, int rows,
                        int N, int64_t lds, int K, int32_t* idx_out, float* val_out,
                        idx_stream stream) {
  if (!ctx || !scores || !idx_out) return IDX_EINVAL;
  if (rows <= 0 || N <= 0 || lds < N) return IDX_EINVAL;
  if ((reinterpret_cast<uintptr_t>(scores) & 3) != 0) return IDX_EINVAL;
  int rc = check_k(ctx, K);
  if (rc != IDX_OK) return rc;
  if (rows > ctx->max_rows || N > ctx->max_n) return IDX_ENOWORKSPACE;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  return run_topk(ctx, scores, lengths, 1, rows, N, lds, K, idx_out, val_out,
                  (cudaStream_t)stream);
}

// score_topk_fused with whole-request lengths or, when tok_lengths is set,
// a valid page count per (request, token) row.
static int fused_impl(idx_ctx* ctx, const uint16_t* q, const uint16_t* c,
                      const int32_t* lengths, const int32_t* tok_lengths, int B, int T, int Q,
                      int D, int N, int64_t ldc_b, int K, int32_t* idx_out, float* val_out,
                      idx_stream stream, const Paged& pg = Paged()) {
  int rc = check_score_args(ctx, q, c, B, T, Q, D, N, ldc_b);
  if (rc != IDX_OK) return rc;
  if (!idx_out) return IDX_EINVAL;
  rc = check_k(ctx, K);
  if (rc != IDX_OK) return rc;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (T <= idx::kDecodeMaxTFused && K <= idx::decode_fused_max_k(T) &&
      (tok_lengths || pg.page_table || !idx::prefill_supported(T, Q, D, ldc_b))) {
    for (int b0 = 0; b0 < B; b0 += idx::kDecodeMaxB) {
      const int nb = std::min(idx::kDecodeMaxB, B - b0);
      idx::DecodeArgs a{};
      a.q = q + (int64_t)b0 * T * Q * D;
      a.c = c + (int64_t)b0 * ldc_b;
      a.lengths = (lengths && !tok_lengths) ? lengths + b0 : nullptr;
      a.tok_lengths = tok_lengths ? tok_lengths + (int64_t)b0 * T : nullptr;
      if (pg.page_table) {
        a.c = c;  // the shared pool, not offset by request
        a.page_table = pg.page_table + (int64_t)b0 * pg.ld_pt;
        a.ld_pt = pg.ld_pt;
        a.n_blocks = pg.n_blocks;
      }
      a.B = nb;
      a.T = T;
      a.Q = Q;
      a.D = D;
      a.N = N;
      a.ldc_b = ldc_b;
      a.K = K;
      a.idx_out = idx_out + (int64_t)b0 * T * K;
      a.val_out = val_out ? val_out + (int64_t)b0 * T * K : nullptr;
      a.cand_bits = ctx->fcand_bits;
      a.cand_idx = ctx->fcand_idx;
      a.row_thr = ctx->row_thr;
      a.slot_stride = ctx->fused_stride;
      a.arrive = ctx->arrive;
      a.status = ctx->status;
      if (idx::decode_fused_slots(nb, T, N, idx::decode_grid(ctx->num_sms)) > ctx->fused_slots)
        return IDX_ENOWORKSPACE;
      rc = status_of(idx::launch_decode(a, true, ctx->num_sms, st));
      if (rc != IDX_OK) return rc;
    }
    return IDX_OK;
  }
  // Prefill chunks (and token counts beyond the fused CUDA-core path): score
  // into the context's scratch, then select each (request, token) row.
  if ((int64_t)B * T * N > ctx->scratch_elems) return IDX_ENOWORKSPACE;
  rc = run_score(ctx, q, c, lengths, tok_lengths, B, T, Q, D, N, ldc_b, ctx->scratch, st, pg);
  if (rc != IDX_OK) return rc;
  if (tok_lengths)  // one length per row
    return run_topk(ctx, ctx->scratch, tok_lengths, 1, B * T, N, N, K, idx_out, val_out, st);
  return run_topk(ctx, ctx->scratch, lengths, T, B * T, N, N, K, idx_out, val_out, st);
}

IDX_API int centroid_pool(idx_ctx* ctx, const uint16_t* keys, const int32_t* key_counts, int B,
                          int D, int P, int N, int64_t ldk_b, uint16_t* c, int64_t ldc_b,
                          idx_stream stream) {
  if (!ctx || !keys || !key_counts || !c) return IDX_EINVAL;
  if (B <= 0 || D <= 0 || P <= 0 || N <= 0) return IDX_EINVAL;
  if (!aligned16(keys) || !aligned16(c) || (ldk_b % 8) != 0 || (ldc_b % 8) != 0) return IDX_EINVAL;
  if (ldc_b < (int64_t)N * D || ldk_b < D) return IDX_EINVAL;
  if ((D % 8) != 0 || D > 256) return IDX_EUNSUPPORTED;
  if ((int64_t)N * P > INT32_MAX || (int64_t)B * N > INT32_MAX) return IDX_EUNSUPPORTED;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  idx::PoolArgs a{};
  a.keys = keys;
  a.key_counts = key_counts;
  a.B = B;
  a.D = D;
  a.P = P;
  a.N = N;
  a.ldk_b = ldk_b;
  a.ldc_b = ldc_b;
  a.c = c;
  a.status = ctx->status;
  return status_of(idx::launch_pool(a, ctx->num_sms, (cudaStream_t)stream));
}

IDX_API int score_topk_fused(idx_ctx* ctx, const uint16_t* q, const uint16_t* c,
                             const int32_t* lengths, int B, int T, int Q, int D, int N,
                             int64_t ldc_b, int K, int32_t* idx_out, float* val_out,
                             idx_stream stream) {
  return fused_impl(ctx, q, c, lengths, nullptr, B, T, Q, D, N, ldc_b, K, idx_out, val_out,
                    stream);
}

// Paged entry points: `pool` holds n_blocks centroid rows of D values; the
// row stride check of check_score_args is applied to a request stride of
// N*D (the pool has no per-request rows).
static int check_paged(const idx_ctx* ctx, const uint16_t* pool, const int32_t* page_table,
                       int64_t ld_pt, int n_blocks, int N, int D) {
  if (!ctx || !pool || !page_table) return IDX_EINVAL;
  if (n_blocks <= 0 || ld_pt < N || N <= 0 || D <= 0) return IDX_EINVAL;
  if (!aligned16(pool)) return IDX_EINVAL;
  if ((D % 8) != 0 || D > 256) return IDX_EUNSUPPORTED;
  return IDX_OK;
}

IDX_API int centroid_score_paged(idx_ctx* ctx, const uint16_t* q, const uint16_t* pool,
                                 int n_blocks, const int32_t* page_table, int64_t ld_pt,
                                 const int32_t* lengths, int B, int T, int Q, int D, int N,
                                 float* scores, idx_stream stream) {
  int rc = check_paged(ctx, pool, page_table, ld_pt, n_blocks, N, D);
  if (rc != IDX_OK) return rc;
  rc = check_score_args(ctx, q, pool, B, T, Q, D, N, (int64_t)N * D);
  if (rc != IDX_OK) return rc;
  if (!scores || !aligned16(scores)) return IDX_EINVAL;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  Paged pg;
  pg.page_table = page_table;
  pg.ld_pt = ld_pt;
  pg.n_blocks = n_blocks;
  return run_score(ctx, q, pool, lengths, nullptr, B, T, Q, D, N, (int64_t)N * D, scores,
                   (cudaStream_t)stream, pg);
}

IDX_API int score_topk_fused_paged(idx_ctx* ctx, const uint16_t* q, const uint16_t* pool,
                                   int n_blocks, const int32_t* page_table, int64_t ld_pt,
                                   const int32_t* lengths, int B, int T, int Q, int D, int N,
                                   int K, int32_t* idx_out, float* val_out, idx_stream stream) {
  const int rc = check_paged(ctx, pool, page_table, ld_pt, n_blocks, N, D);
  if (rc != IDX_OK) return rc;
  Paged pg;
  pg.page_table = page_table;
  pg.ld_pt = ld_pt;
  pg.n_blocks = n_blocks;
  return fused_impl(ctx, q, pool, lengths, nullptr, B, T, Q, D, N, (int64_t)N * D, K, idx_out,
                    val_out, stream, pg);
}

IDX_API int score_topk_fused_tokens(idx_ctx* ctx, const uint16_t* q, const uint16_t* c,
                                    const int32_t* token_lengths, int B, int T, int Q, int D,
                                    int N, int64_t ldc_b, int K, int32_t* idx_out,
                                    float* val_out, idx_stream stream) {
  if (!token_lengths) return IDX_EINVAL;
  return fused_impl(ctx, q, c, nullptr, token_lengths, B, T, Q, D, N, ldc_b, K, idx_out, val_out,
                    stream);
}

// KMeans assignment and scores: x [M][D], centroids [C][D] (bf16, 16-byte
// aligned), h = |c|^2/2 in the context's score scratch (C floats).
static int kmeans_impl(idx_ctx* ctx, const uint16_t* x, const uint16_t* cent, int M, int C, int D,
                       int32_t* assign, float* score, float* scores, idx_stream stream) {
  if (!ctx || !x || !cent) return IDX_EINVAL;
  if (M <= 0 || C <= 0 || D <= 0) return IDX_EINVAL;
  if (!aligned16(x) || !aligned16(cent)) return IDX_EINVAL;
  if ((D % 8) != 0) return IDX_EINVAL;
  if (!idx::kmeans_supported(D)) return IDX_EUNSUPPORTED;
  if ((int64_t)C > ctx->scratch_elems) return IDX_ENOWORKSPACE;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  idx::KmeansArgs a{};
  a.x = x;
  a.cent = cent;
  a.M = M;
  a.C = C;
  a.D = D;
  a.hn = ctx->scratch;
  a.assign = assign;
  a.score = score;
  a.scores = scores;
  a.status = ctx->status;
  return status_of(idx::launch_kmeans(a, scores != nullptr, ctx->num_sms, (cudaStream_t)stream));
}

IDX_API int kmeans_assign(idx_ctx* ctx, const uint16_t* x, const uint16_t* centroids, int M, int C,
                          int D, int32_t* assign_out, float* score_out, idx_stream stream) {
  if (!assign_out) return IDX_EINVAL;
  return kmeans_impl(ctx, x, centroids, M, C, D, assign_out, score_out, nullptr, stream);
}

IDX_API int kmeans_scores(idx_ctx* ctx, const uint16_t* x, const uint16_t* centroids, int M, int C,
                          int D, float* scores, idx_stream stream) {
  if (!scores || !aligned16(scores)) return IDX_EINVAL;
  if ((int64_t)M * C > INT32_MAX * 4ll) return IDX_EUNSUPPORTED;
  return kmeans_impl(ctx, x, centroids, M, C, D, nullptr, nullptr, scores, stream);
}

IDX_API int idx_get_status(idx_ctx* ctx, idx_stream stream, int* bits) {
  if (!ctx) return IDX_EINVAL;
  DeviceGuard guard(ctx->device);
  if (!guard.ok()) return IDX_ECUDA;
  int h = 0;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return IDX_ECUDA;
  if (cudaMemcpy(&h, ctx->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return IDX_ECUDA;
  if (cudaMemset(ctx->status, 0, sizeof(int)) != cudaSuccess) return IDX_ECUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return IDX_ECUDA;
  if (bits) *bits = h;
  return h ? IDX_EDEVICE : IDX_OK;
}

IDX_API const char* idx_strerror(int code) {
  switch (code) {
    case IDX_OK: return "ok";
    case IDX_EINVAL: return "invalid argument (null pointer, size, alignment or stride)";
    case IDX_EUNSUPPORTED: return "unsupported shape (D must be a multiple of 8 up to 256; K up to 2048)";
    case IDX_ENOWORKSPACE: return "rows, N or K exceed the limits given to idx_init";
    case IDX_ECUDA: return "CUDA runtime error or kernel launch failure";
    case IDX_EDEVICE: return "device-side status raised (clamped length or expired wait)";
    default: return "unknown status";
  }
}

IDX_API int idx_num_sms(const idx_ctx* ctx) { return ctx ? ctx->num_sms : 0; }

}  // extern "C"
