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
// Layout: SPLIT CTAs per (sequence, head), each owning a slice of the value
// columns; 256 threads = 8 warps; every lane streams 128-bit vectors of whole
// contiguous rows, holds its rows in registers between the read and the
// write, and the two column reductions go through shuffles and one small
// shared-memory exchange.
#include "kda_common.cuh"

namespace kda {

// SPLIT CTAs share a head: CTA (head, slice) owns value columns
// [slice * DV / SPLIT, +DV / SPLIT) (value columns evolve independently given
// k, alpha, beta and their v entries). Within a CTA each lane owns one 4-column
// group; LPR = columns / 4 lanes cover a row, so a warp instruction reads RPI =
// 32 / LPR whole rows (512 contiguous bytes per warp for 128 columns).
template <typename TIn, int DK, int DV, int SPLIT>
__global__ void __launch_bounds__(256, 2 * SPLIT)
decode_step_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                   const TIn* __restrict__ v, const float* __restrict__ log_alpha,
                   const float* __restrict__ beta, float* __restrict__ state,
                   TIn* __restrict__ o) {
  constexpr int kWarps = 8;
  constexpr int CW = DV / SPLIT;          // value columns of this CTA
  constexpr int LPR = CW / 4;             // lanes per row (one float4 each)
  constexpr int RPI = 32 / LPR;           // rows per warp instruction
  constexpr int NI = DK / (kWarps * RPI); // float4 per thread
  static_assert(CW % 4 == 0 && 32 % LPR == 0 && DK % (kWarps * RPI) == 0, "shape");

  const int head = blockIdx.x / SPLIT, slice = blockIdx.x % SPLIT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cg = lane % LPR, sub = lane / LPR;
  const int col = slice * CW + 4 * cg;

  __shared__ float s_k[DK], s_q[DK], s_a[DK];
  __shared__ float4 s_red[kWarps][2][LPR];
  __shared__ float s_kq[kWarps];

  float* S = state + (size_t)head * DK * DV;

  // Issue the state loads first: they are the bytes that matter.
  float4 s[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)row * DV + col));
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
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    const float a = s_a[row], kk = s_k[row], qq = s_q[row];
    s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
    r.x = fmaf(s[i].x, kk, r.x); r.y = fmaf(s[i].y, kk, r.y);
    r.z = fmaf(s[i].z, kk, r.z); r.w = fmaf(s[i].w, kk, r.w);
    p.x = fmaf(s[i].x, qq, p.x); p.y = fmaf(s[i].y, qq, p.y);
    p.z = fmaf(s[i].z, qq, p.z); p.w = fmaf(s[i].w, qq, p.w);
  }
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {   // lanes holding the same columns
    r.x += __shfl_xor_sync(0xffffffffu, r.x, off); r.y += __shfl_xor_sync(0xffffffffu, r.y, off);
    r.z += __shfl_xor_sync(0xffffffffu, r.z, off); r.w += __shfl_xor_sync(0xffffffffu, r.w, off);
    p.x += __shfl_xor_sync(0xffffffffu, p.x, off); p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
    p.z += __shfl_xor_sync(0xffffffffu, p.z, off); p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
  }
  if (sub == 0) {
    s_red[warp][0][cg] = r;
    s_red[warp][1][cg] = p;
  }
  __syncthreads();

  float kq = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) kq += s_kq[w];
  r = make_float4(0.f, 0.f, 0.f, 0.f);
  p = r;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float4 a = s_red[w][0][cg], b = s_red[w][1][cg];
    r.x += a.x; r.y += a.y; r.z += a.z; r.w += a.w;
    p.x += b.x; p.y += b.y; p.z += b.z; p.w += b.w;
  }
  const float bb = __ldg(beta + head);
  const float rr[4] = {r.x, r.y, r.z, r.w}, pp[4] = {p.x, p.y, p.z, p.w};
  float d[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    d[j] = bb * (Io<TIn>::load(v + (size_t)head * DV + col + j) - rr[j]);
    if (warp == 0 && sub == 0)
      Io<TIn>::store(o + (size_t)head * DV + col + j, fmaf(kq, d[j], pp[j]));
  }

  // S = S' + k d^T, written once.
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    const float kk = s_k[row];
    s[i].x = fmaf(kk, d[0], s[i].x); s[i].y = fmaf(kk, d[1], s[i].y);
    s[i].z = fmaf(kk, d[2], s[i].z); s[i].w = fmaf(kk, d[3], s[i].w);
    __stcs(reinterpret_cast<float4*>(S + (size_t)row * DV + col), s[i]);
  }
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v,
                                   const float* la, const float* beta, float* state,
                                   void* o, int n_heads, cudaStream_t stream) {
  constexpr int kSplit = DV == 128 ? 2 : 1;
  decode_step_kernel<TIn, DK, DV, kSplit><<<n_heads * kSplit, 256, 0, stream>>>(
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
