// kda_noalloc.cu -- kda_prefill_noalloc: the packed variable-length chunked
// prefill with its scratch memory held by the library, for callers that
// cannot allocate device memory.
//
// The chunked prefill over packed sequences needs a small scratch buffer (the
// longest-first order of the sequences, one int32 per sequence) that
// kda_prefill takes from a caller-provided workspace. Some callers cannot
// provide one: plugins and runtime hooks that are handed device pointers but
// own no allocator, serving runtimes whose device memory is already reserved
// by their own pool, and latency-critical paths where an allocation (and the
// device synchronisation it can imply) is not acceptable. This entry point
// serves them: the scratch lives in a file-scope device array of fixed size,
// so nothing is allocated per call.
//
// Limits and rules (also stated in include/kda.h):
//   - at most KDA_NOALLOC_MAX_SEQS sequences per call; larger calls are
//     rejected with KDA_ERR_UNSUPPORTED before anything is launched;
//   - the array is one per device that loads the library and lives until the
//     process exits;
//   - all calls on a device share it: calls whose work overlaps on the GPU
//     (different streams without ordering between them) race on it; calls on
//     one stream, or otherwise ordered, are safe;
//   - the first call on a device looks up the array's device address (a
//     runtime call, done once per device with that device current); make
//     that first call before any stream capture begins. The address is kept
//     until the process exits; a cudaDeviceReset of the device unloads the
//     library's device code and leaves it stale, so the entry point must not
//     be called on a device that was reset.
// The kernel writes every entry it later reads (the order kernel fills
// entries 0..n_seq-1 each call), so nothing has to be cleared between calls.
#include <mutex>

#include "../../include/kda.h"
#include "kda_common.cuh"

namespace kda {

bool chunk_pointers_aligned(const void* q, const void* k, const void* v, const float* la,
                            const void* o, const float* sT);
cudaError_t launch_chunk64(const void* q, const void* k, const void* v, const float* la,
                           const float* beta, const float* s0, const int32_t* cu, int n_seq,
                           int T, int H, void* o, float* sT, float* xfer, int32_t* order,
                           int gate, unsigned flags, cudaStream_t stream);

namespace noalloc {

// The scratch itself. Host code must not use this name as a device address:
// on the host it is only a stand-in object, so its device address is looked
// up with cudaGetSymbolAddress below.
static __device__ __align__(256) int32_t g_order_scratch[KDA_NOALLOC_MAX_SEQS];

constexpr int kMaxDevices = 64;
static std::mutex g_mutex;
static int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once
// per device).
static cudaError_t scratch_for_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_order_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace noalloc
}  // namespace kda

extern "C" kda_status kda_prefill_noalloc(const void* q, const void* k, const void* v,
                                          const float* log_alpha, const float* beta,
                                          const float* init_state, const int32_t* cu_seqlens,
                                          int n_seq, int T, int H, void* o, float* final_state,
                                          cudaStream_t stream) {
  // Same argument rules as kda_prefill for the packed, chunked, bf16 path.
  if (!cu_seqlens || n_seq < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (n_seq > KDA_NOALLOC_MAX_SEQS) return KDA_ERR_UNSUPPORTED;
  if (T > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_INVALID_ARG;
  if ((long long)T * H * 128 >= (1LL << 40)) return KDA_ERR_UNSUPPORTED;
  if ((long long)n_seq * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if (T > 0 && !kda::chunk_pointers_aligned(q, k, v, log_alpha, o, final_state))
    return KDA_ERR_INVALID_ARG;
  if (n_seq == 0) return KDA_OK;
  int32_t* scratch = nullptr;
  if (kda::noalloc::scratch_for_current_device(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
  // With few chains the ring of CTAs hands the state over through each
  // chain's own final_state slot (no other memory is available here).
  const cudaError_t err = kda::launch_chunk64(q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                              n_seq, T, H, o, final_state, final_state, scratch,
                                              0, 0u, stream);
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
