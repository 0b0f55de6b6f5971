// Dispatch for callers that cannot allocate device memory.
//
// Some callers of this library hold only the tensors they were handed and a
// stream: a plugin running inside another inference engine's enqueue step,
// a serving loop that has a fixed device-memory budget and must not
// allocate (cudaMalloc can synchronise the device and stall every stream)
// after start-up, or a host program with no allocator of its own.  They
// cannot provide the scratch workspace that switch_dispatch takes.  This
// entry point runs the same three dispatch kernels with their scratch in a
// file-scope device array instead.  It calls no cudaMalloc, cudaFree or
// other allocating routine.
//
// The array is fixed when the library loads: every GPU that loads the
// library holds kNoAllocScratchBytes (2 MiB) of it until the process exits.
// All calls on a device share it, and it keeps the last call's contents.
// Every scratch word is written before it is read within a call, so nothing
// needs to start at zero; but two calls that overlap on the GPU (different
// streams, no ordering between them) race on the array and give wrong
// results.
#include <climits>
#include <mutex>

#include "kernels.cuh"

namespace {

constexpr int64_t kNoAllocMaxTokens = 131072;       // T limit
constexpr int64_t kNoAllocMaxTileCounts = 131072;   // N * ceil(T / 128) limit
constexpr size_t kNoAllocScratchBytes =
    sizeof(int) * (2 * kNoAllocMaxTileCounts + 2 * kNoAllocMaxTokens);   // 2 MiB

// hist [N][tiles] | base [N][tiles] | local_rank [T] | idx [T]
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};

// Device address of the array on the current device.  In host code the name
// g_noalloc_scratch is only a host-side stand-in, so the address is looked
// up once per device with that device current.
switch_status_t scratch_on_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SWITCH_ERR_CUDA;
  if (dev < 0 || dev >= 64) return SWITCH_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SWITCH_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_ptr[dev]);
  return SWITCH_OK;
}

}  // namespace

extern "C" switch_status_t switch_dispatch_noalloc(const switch_config_t* cfg,
                                                   const int32_t* idx, const float* probs,
                                                   int32_t* rank, uint8_t* drop,
                                                   int32_t* counts, int32_t* slot_token,
                                                   void* stream) {
  if (cfg == nullptr) return SWITCH_ERR_INVALID_ARG;
  const int64_t T = cfg->T;
  const int N = cfg->n_experts;
  if (T < 0 || N < 1 || N > 1024) return SWITCH_ERR_INVALID_ARG;
  if (cfg->flags & SWITCH_FLAG_TOP2) return SWITCH_ERR_UNSUPPORTED;   // one route only
  const int64_t C = switch_capacity(T, N, cfg->capacity_factor);
  if (C < 0) return SWITCH_ERR_INVALID_ARG;
  if (C > INT_MAX / N) return SWITCH_ERR_UNSUPPORTED;
  const int64_t ntiles = (T + smoe::kTileTok - 1) / smoe::kTileTok;
  if (T > kNoAllocMaxTokens || static_cast<int64_t>(N) * ntiles > kNoAllocMaxTileCounts)
    return SWITCH_ERR_UNSUPPORTED;            // beyond the fixed scratch array
  if (T == 0) return SWITCH_OK;
  if ((!idx && !probs) || !rank || !drop || !counts || !slot_token)
    return SWITCH_ERR_INVALID_ARG;

  unsigned char* base = nullptr;
  switch_status_t s = scratch_on_current_device(&base);
  if (s != SWITCH_OK) return s;
  int* hist = reinterpret_cast<int*>(base);
  int* scan = hist + kNoAllocMaxTileCounts;
  int* local_rank = scan + kNoAllocMaxTileCounts;
  int* idx_scratch = local_rank + kNoAllocMaxTokens;
  int* idx_src = idx ? const_cast<int*>(idx) : idx_scratch;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nt = static_cast<int>(ntiles);

  // Expert ids outside [0, N) are treated as dropped; there is no device
  // error word here (nullptr), so they are not reported.
  if (smoe::launch_tile_rank(T, N, idx, probs, idx ? nullptr : idx_src, local_rank, hist, nt,
                             nullptr, st) != cudaSuccess)
    return SWITCH_ERR_CUDA;
  if (smoe::launch_scan(N, nt, hist, scan, counts, st) != cudaSuccess) return SWITCH_ERR_CUDA;
  if (smoe::launch_finalize(T, N, C, nt, idx_src, local_rank, scan, counts, rank, drop,
                            slot_token, nullptr, 0, st) != cudaSuccess)
    return SWITCH_ERR_CUDA;
  return SWITCH_OK;
}
