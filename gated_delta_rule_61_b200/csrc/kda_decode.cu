// kda_decode.cu -- single-token KDA decode step, state updated in place.
//
// Pages: "22580: from GPT-2 to Kimi K3, explained", section "DeltaNet, or
// Fast Weight Programmers" (forward with a cache and one token: read at the
// key, delta, outer-product write, read-out) with the per-channel decay of
// "Gated Delta Net" / "KDA / Kimi Linear". One step per (sequence, head):
//     S' = Diag(alpha) S;  r = S'^T k;  p = S'^T q;  d = beta (v - r)
//     S  = S' + k d^T;     o = S^T q = p + (k . q) d
// The last identity lets both reductions over the key index run in the same
// pass over S, so the state is read once and written once: the kernel is
// bound by HBM bandwidth (about 2 * dk * dv * 4 bytes per head).
//
// Layout: one CTA per (sequence, head); 256 threads = 8 warps. Lane l owns
// value columns [VPL*l, VPL*l + VPL) (VPL = dv / 32, one 128-bit or 64-bit
// vector); warp w owns key rows w, w + 8, ... (dk / 8 rows). A warp therefore
// reads whole contiguous rows of S (coalesced 512-byte rows for dv = 128).
#include "kda_common.cuh"

namespace kda {

template <int N> struct VecF;
template <> struct VecF<4> {
  using T = float4;
  static __device__ __forceinline__ void unpack(const T& v, float* e) {
    e[0] = v.x; e[1] = v.y; e[2] = v.z; e[3] = v.w;
  }
  static __device__ __forceinline__ T pack(const float* e) { return make_float4(e[0], e[1], e[2], e[3]); }
};
template <> struct VecF<2> {
  using T = float2;
  static __device__ __forceinline__ void unpack(const T& v, float* e) { e[0] = v.x; e[1] = v.y; }
  static __device__ __forceinline__ T pack(const float* e) { return make_float2(e[0], e[1]); }
};

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                   const TIn* __restrict__ v, const float* __restrict__ log_alpha,
                   const float* __restrict__ beta, float* __restrict__ state,
                   TIn* __restrict__ o) {
  constexpr int kWarps = 8;
  constexpr int VPL = DV / 32;          // value columns per lane
  constexpr int RPW = DK / kWarps;      // key rows per warp
  using V = VecF<VPL>;
  using VT = typename V::T;

  const int head = blockIdx.x;          // flat (b, h)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  __shared__ float s_k[DK], s_q[DK], s_a[DK];
  __shared__ float s_red[kWarps][2][DV];
  __shared__ float s_kq[kWarps];

  float* S = state + (size_t)head * DK * DV;

  // Issue the state loads first: they are the bytes that matter.
  float s[RPW][VPL];
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int row = warp + i * kWarps;
    V::unpack(__ldcs(reinterpret_cast<const VT*>(S + (size_t)row * DV) + lane), s[i]);
  }

  // Small per-head vectors: k, q, alpha = exp(log_alpha); k . q per warp.
  float kq_part = 0.f;
  for (int i = threadIdx.x; i < DK; i += blockDim.x) {
    const float kk = Io<TIn>::load(k + (size_t)head * DK + i);
    const float qq = Io<TIn>::load(q + (size_t)head * DK + i);
    s_k[i] = kk;
    s_q[i] = qq;
    s_a[i] = expf(__ldg(log_alpha + (size_t)head * DK + i));
    kq_part += kk * qq;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kq_part += __shfl_xor_sync(0xffffffffu, kq_part, off);
  if (lane == 0) s_kq[warp] = kq_part;
  __syncthreads();

  // Decay rows and accumulate partial r = S'^T k and p = S'^T q.
  float r[VPL], p[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) r[j] = p[j] = 0.f;
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int row = warp + i * kWarps;
    const float a = s_a[row], kk = s_k[row], qq = s_q[row];
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      s[i][j] *= a;
      r[j] = fmaf(s[i][j], kk, r[j]);
      p[j] = fmaf(s[i][j], qq, p[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    s_red[warp][0][lane * VPL + j] = r[j];
    s_red[warp][1][lane * VPL + j] = p[j];
  }
  __syncthreads();

  float kq = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) kq += s_kq[w];
  const float b = __ldg(beta + head);
  float d[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    float rr = 0.f, pp = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      rr += s_red[w][0][lane * VPL + j];
      pp += s_red[w][1][lane * VPL + j];
    }
    const int col = lane * VPL + j;
    d[j] = b * (Io<TIn>::load(v + (size_t)head * DV + col) - rr);
    if (warp == 0) Io<TIn>::store(o + (size_t)head * DV + col, fmaf(kq, d[j], pp));
  }

  // S = S' + k d^T, written once.
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int row = warp + i * kWarps;
    const float kk = s_k[row];
#pragma unroll
    for (int j = 0; j < VPL; ++j) s[i][j] = fmaf(kk, d[j], s[i][j]);
    __stcs(reinterpret_cast<VT*>(S + (size_t)row * DV) + lane, V::pack(s[i]));
  }
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v,
                                   const float* la, const float* beta, float* state,
                                   void* o, int n_heads, cudaStream_t stream) {
  decode_step_kernel<TIn, DK, DV><<<n_heads, 256, 0, stream>>>(
      (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, state, (TIn*)o);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_decode_dtype(const void* q, const void* k, const void* v,
                                       const float* la, const float* beta, float* state,
                                       int dk, int dv, void* o, int n_heads,
                                       cudaStream_t stream) {
  if (dk == 128 && dv == 128)
    return launch_decode_t<TIn, 128, 128>(q, k, v, la, beta, state, o, n_heads, stream);
  if (dk == 128 && dv == 64)
    return launch_decode_t<TIn, 128, 64>(q, k, v, la, beta, state, o, n_heads, stream);
  if (dk == 64 && dv == 128)
    return launch_decode_t<TIn, 64, 128>(q, k, v, la, beta, state, o, n_heads, stream);
  return launch_decode_t<TIn, 64, 64>(q, k, v, la, beta, state, o, n_heads, stream);
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* la,
                          const float* beta, float* state, int dk, int dv, bool bf16,
                          void* o, int n_heads, cudaStream_t stream) {
  if (n_heads == 0) return cudaSuccess;
  if (bf16)
    return launch_decode_dtype<__nv_bfloat16>(q, k, v, la, beta, state, dk, dv, o,
                                              n_heads, stream);
  return launch_decode_dtype<float>(q, k, v, la, beta, state, dk, dv, o, n_heads, stream);
}

}  // namespace kda
