// kda_api.cu -- the C ABI of libkda.so: argument checks, kernel choice,
// launch on the caller's stream, device status word. See include/kda.h.
#include "../../include/kda.h"
#include "kda_common.cuh"

namespace kda {

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* la,
                          const float* beta, float* state, int dk, int dv, bool bf16,
                          void* o, int n_heads, int T, int H, int gate, unsigned flags,
                          cudaStream_t stream);
cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const float* la,
                             const float* beta, const float* s0, const int32_t* cu,
                             int n_seq, int T, int H, int dk, int dv, bool bf16, void* o,
                             float* sT, int gate, unsigned flags, cudaStream_t stream);
cudaError_t launch_chunk64(const void* q, const void* k, const void* v, const float* la,
                           const float* beta, const float* s0, const int32_t* cu,
                           int n_seq, int T, int H, void* o, float* sT, float* xfer,
                           int32_t* order, int gate, unsigned flags, cudaStream_t stream);

cudaError_t launch_backward(const void* q, const void* k, const void* v, const float* la,
                            const float* beta, const float* s0, const int32_t* cu,
                            const void* d_o, const float* d_final, int n_seq, int T, int H,
                            int dk, int dv, bool bf16, int gate, unsigned flags,
                            long long tokens, float* dq, float* dkk, float* dvv, float* dla,
                            float* dbeta, float* d_init, void* workspace, cudaStream_t stream);
size_t backward_workspace_bytes(int n_seq, long long tokens, int H, int dk, int dv);

static bool head_size_ok(int d) { return d == 64 || d == 128; }
static bool gate_ok(kda_gate g) {
  return g == KDA_GATE_CHANNEL || g == KDA_GATE_SCALAR || g == KDA_GATE_NONE;
}
constexpr unsigned kAllFlags = KDA_RAW_QK | KDA_RAW_BETA | KDA_RAW_GATE;

// Workspace of a prefill call: the longest-first order of packed sequences
// (one int32 each) and, when the chains are few enough that a ring of CTAs
// may serve each chain, one dk x dv fp32 hand-over slot per chain. Each part
// starts on a 256-byte boundary.
struct WorkspaceLayout {
  bool chunked;        // the chunked tensor-core kernel serves the call
  size_t order_off, order_bytes, xfer_off, xfer_bytes, total;
};
constexpr long long kRingMaxChains = 128;   // 2 x chains <= SMs on any GPU up to 256 SMs

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

void workspace_layout(int n_seq, int H, int dk, int dv, kda_dtype dtype, int chunk,
                      bool has_cu, WorkspaceLayout* w) {
  *w = WorkspaceLayout{};
  if (n_seq < 0) n_seq = 0;
  if (H < 0) H = 0;
  w->chunked = dtype == KDA_BF16 && chunk == 64 && dk == 128 && dv == 128;
  if (!w->chunked || n_seq == 0) return;
  w->order_bytes = has_cu ? round256(sizeof(int32_t) * (size_t)n_seq) : 0;
  const long long chains = (long long)n_seq * H;
  w->xfer_off = w->order_bytes;
  w->xfer_bytes = chains <= kRingMaxChains ? (size_t)chains * dk * dv * sizeof(float) : 0;
  w->total = w->xfer_off + w->xfer_bytes;
}

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

size_t kda_prefill_workspace_bytes(int n_seq, int H, int dk, int dv, kda_dtype dtype,
                                   int chunk, int has_cu_seqlens) {
  kda::WorkspaceLayout w;
  kda::workspace_layout(n_seq, H, dk, dv, dtype, chunk, has_cu_seqlens != 0, &w);
  return w.total;
}

kda_status kda_prefill_ex(const void* q, const void* k, const void* v, const float* log_alpha,
                          const float* beta, const float* init_state,
                          const int32_t* cu_seqlens, int n_seq, int B, int T, int H, int dk,
                          int dv, kda_dtype dtype, kda_gate gate, unsigned flags, int chunk,
                          void* o, float* final_state, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || T < 0 || H <= 0 || n_seq < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!kda::gate_ok(gate) || (flags & ~kda::kAllFlags)) return KDA_ERR_INVALID_ARG;
  if (!kda::head_size_ok(dk) || !kda::head_size_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (cu_seqlens) {
    if (B != 1) return KDA_ERR_INVALID_ARG;
  } else {
    if (n_seq == 0) n_seq = B;
    if (n_seq != B) return KDA_ERR_INVALID_ARG;
  }
  const long long tokens = (long long)B * T;
  if (tokens > 0 && (!q || !k || !v || !beta || !o)) return KDA_ERR_INVALID_ARG;
  if (tokens > 0 && gate != KDA_GATE_NONE && !log_alpha) return KDA_ERR_INVALID_ARG;
  if (tokens * H * (dk > dv ? dk : dv) >= (1LL << 40)) return KDA_ERR_UNSUPPORTED;
  if (chunk != 0 && chunk != 64) return KDA_ERR_UNSUPPORTED;
  if (n_seq == 0) return KDA_OK;
  // Chains are (sequence, head) pairs; grid sizes are 32-bit.
  if ((long long)n_seq * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;

  const bool bf16 = dtype == KDA_BF16;
  kda::WorkspaceLayout w;
  kda::workspace_layout(n_seq, H, dk, dv, dtype, chunk, cu_seqlens != nullptr, &w);
  cudaError_t err;
  if (w.chunked) {
    // token coordinates of the tensor-map copies are 32-bit
    if (tokens > 0x7fffffffLL - 256) return KDA_ERR_UNSUPPORTED;
    // (a scalar or absent gate is read one float at a time)
    if (tokens > 0 &&
        !kda::chunk_pointers_aligned(q, k, v, gate == KDA_GATE_CHANNEL ? log_alpha : nullptr,
                                     o, final_state))
      return KDA_ERR_INVALID_ARG;
    if (w.total > 0 && (!workspace || workspace_bytes < w.total)) return KDA_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255)) return KDA_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* order = w.order_bytes ? reinterpret_cast<int32_t*>(ws + w.order_off) : nullptr;
    float* xfer = w.xfer_bytes ? reinterpret_cast<float*>(ws + w.xfer_off) : nullptr;
    err = kda::launch_chunk64(q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, T, H,
                              o, final_state, xfer, order, (int)gate, flags, stream);
  } else {
    err = kda::launch_recurrent(q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, T, H,
                                dk, dv, bf16, o, final_state, (int)gate, flags, stream);
  }
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_prefill(const void* q, const void* k, const void* v, const float* log_alpha,
                       const float* beta, const float* init_state, const int32_t* cu_seqlens,
                       int n_seq, int B, int T, int H, int dk, int dv, kda_dtype dtype,
                       int chunk, void* o, float* final_state, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  if (B * (long long)T > 0 && !log_alpha) return KDA_ERR_INVALID_ARG;
  return kda_prefill_ex(q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, B, T, H, dk,
                        dv, dtype, KDA_GATE_CHANNEL, 0u, chunk, o, final_state, workspace,
                        workspace_bytes, stream);
}

kda_status kda_decode_ex(const void* q, const void* k, const void* v, const float* log_alpha,
                         const float* beta, float* state, int B, int T, int H, int dk, int dv,
                         kda_dtype dtype, kda_gate gate, unsigned flags, void* o,
                         cudaStream_t stream) {
  if (B < 0 || H <= 0 || T < 1) return KDA_ERR_INVALID_ARG;
  if (T > KDA_DECODE_MAX_TOKENS) return KDA_ERR_UNSUPPORTED;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!kda::gate_ok(gate) || (flags & ~kda::kAllFlags)) return KDA_ERR_INVALID_ARG;
  if (!kda::head_size_ok(dk) || !kda::head_size_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (B == 0) return KDA_OK;
  if (!q || !k || !v || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
  if (gate != KDA_GATE_NONE && !log_alpha) return KDA_ERR_INVALID_ARG;
  if ((long long)B * H * 2 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(state) & 15)) return KDA_ERR_INVALID_ARG;
  const cudaError_t err = kda::launch_decode(q, k, v, log_alpha, beta, state, dk, dv,
                                             dtype == KDA_BF16, o, B * H, T, H, (int)gate,
                                             flags, stream);
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, float* state, int B, int H, int dk, int dv,
                           kda_dtype dtype, void* o, cudaStream_t stream) {
  if (B > 0 && !log_alpha) return KDA_ERR_INVALID_ARG;
  return kda_decode_ex(q, k, v, log_alpha, beta, state, B, 1, H, dk, dv, dtype,
                       KDA_GATE_CHANNEL, 0u, o, stream);
}

size_t kda_backward_workspace_bytes(int n_seq, int64_t tokens, int H, int dk, int dv) {
  if (n_seq <= 0 || tokens < 0 || H <= 0 || !kda::head_size_ok(dk) || !kda::head_size_ok(dv))
    return 0;
  return kda::backward_workspace_bytes(n_seq, (long long)tokens, H, dk, dv);
}

kda_status kda_backward_ex(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* init_state,
                           const int32_t* cu_seqlens, int n_seq, int B, int T, int H, int dk,
                           int dv, kda_dtype dtype, kda_gate gate, unsigned flags,
                           const void* d_o, const float* d_final, float* dq, float* dk_out,
                           float* dv_out, float* dlog_alpha, float* dbeta, float* d_init,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || T < 0 || H <= 0 || n_seq < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (!kda::gate_ok(gate) || (flags & ~kda::kAllFlags)) return KDA_ERR_INVALID_ARG;
  if (!kda::head_size_ok(dk) || !kda::head_size_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (cu_seqlens) {
    if (B != 1) return KDA_ERR_INVALID_ARG;
  } else {
    if (n_seq == 0) n_seq = B;
    if (n_seq != B) return KDA_ERR_INVALID_ARG;
  }
  const long long tokens = (long long)B * T;
  if (tokens > 0 && (!q || !k || !v || !beta || !d_o || !dq || !dk_out || !dv_out || !dbeta))
    return KDA_ERR_INVALID_ARG;
  if (tokens > 0 && gate != KDA_GATE_NONE && (!log_alpha || !dlog_alpha))
    return KDA_ERR_INVALID_ARG;
  if (tokens * H * (dk > dv ? dk : dv) >= (1LL << 40)) return KDA_ERR_UNSUPPORTED;
  if (n_seq == 0) return KDA_OK;
  if ((long long)n_seq * H * 4 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
  // the states are moved in 16-byte vectors
  if ((reinterpret_cast<uintptr_t>(init_state) | reinterpret_cast<uintptr_t>(d_final) |
       reinterpret_cast<uintptr_t>(d_init)) & 15)
    return KDA_ERR_INVALID_ARG;
  const size_t need = kda::backward_workspace_bytes(n_seq, tokens, H, dk, dv);
  if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return KDA_ERR_WORKSPACE;
  const cudaError_t err = kda::launch_backward(
      q, k, v, log_alpha, beta, init_state, cu_seqlens, d_o, d_final, n_seq, T, H, dk, dv,
      dtype == KDA_BF16, (int)gate, flags, tokens, dq, dk_out, dv_out, dlog_alpha, dbeta,
      d_init, workspace, stream);
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_backward(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* init_state, const int32_t* cu_seqlens,
                        int n_seq, int B, int T, int H, int dk, int dv, kda_dtype dtype,
                        kda_gate gate, const void* d_o, const float* d_final, float* dq,
                        float* dk_out, float* dv_out, float* dlog_alpha, float* dbeta,
                        float* d_init, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  return kda_backward_ex(q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, B, T, H, dk,
                         dv, dtype, gate, 0u, d_o, d_final, dq, dk_out, dv_out, dlog_alpha,
                         dbeta, d_init, workspace, workspace_bytes, stream);
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
