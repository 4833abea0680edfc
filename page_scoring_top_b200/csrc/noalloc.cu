// noalloc.cu -- topk_select for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: serving engines that plan every byte
// of device memory up front and forbid allocations on the request path, and
// plugin hosts that hand a library device pointers but no allocator.  topk_select needs scratch for the
// per-chunk candidate lists of long rows and for the per-row counters; this
// variant keeps that scratch in one file-scope static device array instead of
// an idx_ctx workspace, so the call itself allocates nothing.
//
// The array is kNoAllocScratchBytes (8 MiB); every GPU that loads the library
// holds it until the process exits.  Its device address is looked up once per
// device (cudaGetSymbolAddress) on the first call made with that device
// current, so that first call should come before any stream capture.  All
// calls share the array and it keeps the last call's contents: each call
// clears the counters it needs (cudaMemsetAsync on the caller's stream), and
// calls that overlap on the GPU (other streams, other host threads) race.
#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "idx.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Per-device set-up results.  Host threads may make their first calls at the
// same time: the set-up runs under a mutex, and the address is published with
// release order after the SM count, so a thread that reads a non-null address
// (acquire) also sees that device's SM count.
std::atomic<unsigned char*> g_scratch_addr[kMaxDevices] = {};
int g_scratch_sms[kMaxDevices] = {};
std::mutex g_setup_mutex;

// The device address of the scratch array on the current device `dev`
// (looked up once per device), or null on a CUDA error.
unsigned char* scratch_on(int dev) {
  unsigned char* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return nullptr;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return nullptr;
  g_scratch_sms[dev] = sms;
  p = static_cast<unsigned char*>(addr);
  g_scratch_addr[dev].store(p, std::memory_order_release);
  return p;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

extern "C" IDX_API int topk_select_noalloc(const float* scores, const int32_t* lengths, int rows,
                                           int N, int64_t lds, int K, int32_t* idx_out,
                                           float* val_out, idx_stream stream) {
  if (!scores || !idx_out) return IDX_EINVAL;
  if (rows <= 0 || N <= 0 || lds < N || K <= 0) return IDX_EINVAL;
  if ((reinterpret_cast<uintptr_t>(scores) & 3) != 0) return IDX_EINVAL;
  if (K > IDX_MAX_K) return IDX_EUNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return IDX_ECUDA;
  unsigned char* base = scratch_on(dev);  // set-up, once per device, with that device current
  if (!base) return IDX_ECUDA;
  idx::TopkArgs a{};
  a.chunk = idx::topk_plan_chunk(rows, N, K, g_scratch_sms[dev]);
  a.max_chunks = (N + a.chunk - 1) / a.chunk;
  // scratch: status word | arrival counters | row thresholds | candidate bits | indices
  const size_t o_arrive = 256;
  const size_t o_thr = o_arrive + round256((size_t)rows * 4);
  const size_t o_bits = o_thr + round256((size_t)rows * 8);
  const size_t cand = (size_t)rows * a.max_chunks * K * 4;
  const size_t o_idx = o_bits + round256(cand);
  if (o_idx + cand > kNoAllocScratchBytes) return IDX_ENOWORKSPACE;  // rows x chunks x K too large
  // counters and thresholds must start at zero whatever the last call left
  if (cudaMemsetAsync(base, 0, o_bits, (cudaStream_t)stream) != cudaSuccess) return IDX_ECUDA;
  a.scores = scores;
  a.lengths = lengths;
  a.len_div = 1;
  a.rows = rows;
  a.N = N;
  a.lds = lds;
  a.K = K;
  a.slot_stride = K;
  a.idx_out = idx_out;
  a.val_out = val_out;
  a.status = reinterpret_cast<int*>(base);
  a.arrive = reinterpret_cast<int32_t*>(base + o_arrive);
  a.row_thr = reinterpret_cast<unsigned long long*>(base + o_thr);
  a.cand_bits = reinterpret_cast<uint32_t*>(base + o_bits);
  a.cand_idx = reinterpret_cast<int32_t*>(base + o_idx);
  return idx::launch_topk(a, (cudaStream_t)stream) == cudaSuccess ? IDX_OK : IDX_ECUDA;
}
