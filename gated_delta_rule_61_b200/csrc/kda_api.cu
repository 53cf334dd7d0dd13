// kda_api.cu -- the C ABI of libkda.so: argument checks, kernel choice,
// launch on the caller's stream, device status word. See include/kda.h.
#include "../../include/kda.h"
#include "kda_common.cuh"

namespace kda {

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* la,
                          const float* beta, float* state, int dk, int dv, bool bf16,
                          void* o, int n_heads, cudaStream_t stream);
cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const float* la,
                             const float* beta, const float* s0, const int32_t* cu,
                             int n_seq, int T, int H, int dk, int dv, bool bf16, void* o,
                             float* sT, cudaStream_t stream);
cudaError_t launch_chunk64(const void* q, const void* k, const void* v, const float* la,
                           const float* beta, const float* s0, const int32_t* cu,
                           int n_seq, int T, int H, void* o, float* sT, int32_t* order,
                           cudaStream_t stream);

static bool head_size_ok(int d) { return d == 64 || d == 128; }

// The chunked kernel moves q, k, v, o, log_alpha and the state hand-over in
// 8- and 16-byte vectors.
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool chunk_pointers_aligned(const void* q, const void* k, const void* v, const float* la,
                            const void* o, const float* sT) {
  return aligned16(q) && aligned16(k) && aligned16(v) && aligned16(la) && aligned16(o) &&
         (!sT || aligned16(sT));
}

}  // namespace kda

extern "C" {

const char* kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported configuration";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int kda_version(void) { return 100; }

size_t kda_prefill_workspace_bytes(int n_seq, int has_cu_seqlens) {
  if (!has_cu_seqlens || n_seq <= 0) return 0;
  const size_t bytes = sizeof(int32_t) * (size_t)n_seq;
  return (bytes + 255) / 256 * 256;
}

kda_status kda_prefill(const void* q, const void* k, const void* v, const float* log_alpha,
                       const float* beta, const float* init_state, const int32_t* cu_seqlens,
                       int n_seq, int B, int T, int H, int dk, int dv, kda_dtype dtype,
                       int chunk, void* o, float* final_state, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || T < 0 || H <= 0 || n_seq < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!kda::head_size_ok(dk) || !kda::head_size_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (cu_seqlens) {
    if (B != 1) return KDA_ERR_INVALID_ARG;
  } else {
    if (n_seq == 0) n_seq = B;
    if (n_seq != B) return KDA_ERR_INVALID_ARG;
  }
  const long long tokens = (long long)B * T;
  if (tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_INVALID_ARG;
  if (tokens * H * (dk > dv ? dk : dv) >= (1LL << 40)) return KDA_ERR_UNSUPPORTED;
  if (chunk != 0 && chunk != 64) return KDA_ERR_UNSUPPORTED;
  if (n_seq == 0) return KDA_OK;
  // Chains are (sequence, head) pairs; grid sizes are 32-bit.
  if ((long long)n_seq * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;

  const bool bf16 = dtype == KDA_BF16;
  const bool use_chunk = bf16 && chunk == 64;
  cudaError_t err;
  if (use_chunk) {
    if (dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
    if (tokens > 0 && !kda::chunk_pointers_aligned(q, k, v, log_alpha, o, final_state))
      return KDA_ERR_INVALID_ARG;
    const size_t need = kda_prefill_workspace_bytes(n_seq, cu_seqlens != nullptr);
    if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255)) return KDA_ERR_WORKSPACE;
    err = kda::launch_chunk64(q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, T, H,
                              o, final_state, cu_seqlens ? (int32_t*)workspace : nullptr,
                              stream);
  } else {
    err = kda::launch_recurrent(q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, T, H,
                                dk, dv, bf16, o, final_state, stream);
  }
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, float* state, int B, int H, int dk, int dv,
                           kda_dtype dtype, void* o, cudaStream_t stream) {
  if (B < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!kda::head_size_ok(dk) || !kda::head_size_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (B == 0) return KDA_OK;
  if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
  if ((long long)B * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(state) & 15)) return KDA_ERR_INVALID_ARG;
  const cudaError_t err = kda::launch_decode(q, k, v, log_alpha, beta, state, dk, dv,
                                             dtype == KDA_BF16, o, B * H, stream);
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_get_device_status(int reset, int* detail, cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
  kda::DeviceStatus st;
  if (cudaMemcpyFromSymbol(&st, kda::g_status, sizeof(st)) != cudaSuccess) return KDA_ERR_CUDA;
  if (reset) {
    const kda::DeviceStatus zero = {0, 0};
    if (cudaMemcpyToSymbol(kda::g_status, &zero, sizeof(zero)) != cudaSuccess)
      return KDA_ERR_CUDA;
  }
  if (detail) *detail = st.flags ? st.detail : 0;
  return (st.flags & kda::kStatusTimeout) ? KDA_ERR_TIMEOUT : KDA_OK;
}

}  // extern "C"
