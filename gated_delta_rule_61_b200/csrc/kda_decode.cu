// kda_decode.cu -- KDA decode against a cached state, updated in place: one
// token per sequence (the pages' decode step), or a few tokens per sequence
// in one pass over the state (multi-token decode).
//
// Pages: "22580: from GPT-2 to Kimi K3, explained", section "DeltaNet, or
// Fast Weight Programmers" (forward with a cache: read at the key, delta,
// outer-product write, read-out; q and k through SiLU and L2 normalisation,
// beta through a sigmoid) with the decay of "Gated Delta Net" (one scalar per
// token) and "KDA / Kimi Linear" (one per key channel). Each token applies
//     S' = Diag(alpha) S;  r = S'^T k;  p = S'^T q;  d = beta (v - r)
//     S  = S' + k d^T;     o = S^T q = p + (k . q) d
// The last identity lets both reductions over the key index run in the same
// pass over S. The state is read once and written once per call whatever the
// number of tokens, so a call is bound by HBM bandwidth (about
// 2 * dk * dv * 4 bytes per head).
//
// Layout: SPLIT CTAs per (sequence, head), each owning a slice of the value
// columns (value columns evolve independently given k, alpha, beta and their
// own v entries); 256 threads = 8 warps; every lane streams 128-bit vectors of
// whole contiguous rows, holds its rows in registers for the whole call, and
// the two column reductions go through shuffles and one small shared-memory
// exchange per token.
#include "kda_common.cuh"

namespace kda {

// Gate forms (kda_gate in include/kda.h) and prologue flags.
constexpr int kGateChannel = 0, kGateScalar = 1, kGateNone = 2;
constexpr unsigned kRawQK = 1u, kRawBeta = 2u, kRawGate = 4u;

__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }

// The decay alpha of key channel i from the stored gate: exp(log_alpha), or
// sigmoid(x) when the gate holds logits (exp(log sigmoid(x)) = sigmoid(x)).
__device__ __forceinline__ float decay_from(float g, unsigned flags) {
  return (flags & kRawGate) ? sigmoid_f(g) : expf(g);
}

// CTA (head, slice) owns value columns [slice * DV / SPLIT, +DV / SPLIT).
// Within a CTA each lane owns one 4-column group; LPR = columns / 4 lanes
// cover a row, so a warp instruction reads RPI = 32 / LPR whole rows (512
// contiguous bytes per warp for 128 columns).
template <typename TIn, int DK, int DV, int SPLIT>
__global__ void __launch_bounds__(256, 2 * SPLIT)
decode_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
              const float* __restrict__ log_alpha, const float* __restrict__ beta,
              float* __restrict__ state, TIn* __restrict__ o, int T, int H, int gate,
              unsigned flags) {
  constexpr int kWarps = 8;
  constexpr int CW = DV / SPLIT;          // value columns of this CTA
  constexpr int LPR = CW / 4;             // lanes per row (one float4 each)
  constexpr int RPI = 32 / LPR;           // rows per warp instruction
  constexpr int NI = DK / (kWarps * RPI); // float4 per thread
  static_assert(CW % 4 == 0 && 32 % LPR == 0 && DK % (kWarps * RPI) == 0, "shape");

  const int head = blockIdx.x / SPLIT, slice = blockIdx.x % SPLIT;   // head = b * H + h
  const int b = head / H, h = head - (head / H) * H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cg = lane % LPR, sub = lane / LPR;
  const int col = slice * CW + 4 * cg;
  const bool raw_qk = flags & kRawQK;

  __shared__ float s_k[2][DK], s_q[2][DK], s_a[2][DK];
  __shared__ float4 s_red[2][kWarps][2][LPR];
  __shared__ float s_sum[2][kWarps][3];   // k.q and, for raw inputs, |k|^2 and |q|^2

  float* S = state + (size_t)head * DK * DV;

  // Issue the state loads first: they are the bytes that matter.
  float4 s[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)row * DV + col));
  }

  for (int t = 0; t < T; ++t) {
    const int buf = t & 1;
    const size_t tok = ((size_t)b * T + t) * H + h;      // token index in [B, T, H]
    // Per-token vectors: k, q (after the prologue when raw), alpha per key row.
    float part[3] = {0.f, 0.f, 0.f};
    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
      float kk = Io<TIn>::load(k + tok * DK + i);
      float qq = Io<TIn>::load(q + tok * DK + i);
      if (raw_qk) {
        kk = silu_f(kk);
        qq = silu_f(qq);
        part[1] += kk * kk;
        part[2] += qq * qq;
      }
      s_k[buf][i] = kk;
      s_q[buf][i] = qq;
      float a = 1.f;
      if (gate == kGateChannel) a = decay_from(__ldg(log_alpha + tok * DK + i), flags);
      else if (gate == kGateScalar) a = decay_from(__ldg(log_alpha + tok), flags);
      s_a[buf][i] = a;
      part[0] += kk * qq;
    }
#pragma unroll
    for (int j = 0; j < 3; ++j)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], off);
    if (lane == 0) {
      s_sum[buf][warp][0] = part[0];
      s_sum[buf][warp][1] = part[1];
      s_sum[buf][warp][2] = part[2];
    }
    __syncthreads();

    // Decay rows and accumulate partial r = S'^T k and p = S'^T q.
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int row = (warp + i * kWarps) * RPI + sub;
      const float a = s_a[buf][row], kk = s_k[buf][row], qq = s_q[buf][row];
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
      s_red[buf][warp][0][cg] = r;
      s_red[buf][warp][1][cg] = p;
    }
    __syncthreads();

    float kq = 0.f, nk2 = 0.f, nq2 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      kq += s_sum[buf][w][0];
      nk2 += s_sum[buf][w][1];
      nq2 += s_sum[buf][w][2];
    }
    // L2 normalisation of SiLU(k), SiLU(q) folded into the reductions:
    // x / max(|x|, 1e-12).
    const float ik = raw_qk ? 1.f / fmaxf(sqrtf(nk2), 1e-12f) : 1.f;
    const float iq = raw_qk ? 1.f / fmaxf(sqrtf(nq2), 1e-12f) : 1.f;
    kq *= ik * iq;
    r = make_float4(0.f, 0.f, 0.f, 0.f);
    p = r;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float4 x = s_red[buf][w][0][cg], y = s_red[buf][w][1][cg];
      r.x += x.x; r.y += x.y; r.z += x.z; r.w += x.w;
      p.x += y.x; p.y += y.y; p.z += y.z; p.w += y.w;
    }
    float bb = __ldg(beta + tok);
    if (flags & kRawBeta) bb = sigmoid_f(bb);
    const float rr[4] = {r.x * ik, r.y * ik, r.z * ik, r.w * ik};
    const float pp[4] = {p.x * iq, p.y * iq, p.z * iq, p.w * iq};
    float d[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      d[j] = bb * (Io<TIn>::load(v + tok * DV + col + j) - rr[j]);
      if (warp == 0 && sub == 0) Io<TIn>::store(o + tok * DV + col + j, fmaf(kq, d[j], pp[j]));
    }
    // S = S' + k d^T (k normalised).
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int row = (warp + i * kWarps) * RPI + sub;
      const float kk = s_k[buf][row] * ik;
      s[i].x = fmaf(kk, d[0], s[i].x); s[i].y = fmaf(kk, d[1], s[i].y);
      s[i].z = fmaf(kk, d[2], s[i].z); s[i].w = fmaf(kk, d[3], s[i].w);
    }
  }

  // Written once.
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    __stcs(reinterpret_cast<float4*>(S + (size_t)row * DV + col), s[i]);
  }
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v,
                                   const float* la, const float* beta, float* state, void* o,
                                   int n_heads, int T, int H, int gate, unsigned flags,
                                   cudaStream_t stream) {
  constexpr int kSplit = DV == 128 ? 2 : 1;
  decode_kernel<TIn, DK, DV, kSplit><<<n_heads * kSplit, 256, 0, stream>>>(
      (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, state, (TIn*)o, T, H, gate, flags);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_decode_dtype(const void* q, const void* k, const void* v,
                                       const float* la, const float* beta, float* state,
                                       int dk, int dv, void* o, int n_heads, int T, int H,
                                       int gate, unsigned flags, cudaStream_t stream) {
  if (dk == 128 && dv == 128)
    return launch_decode_t<TIn, 128, 128>(q, k, v, la, beta, state, o, n_heads, T, H, gate,
                                          flags, stream);
  if (dk == 128 && dv == 64)
    return launch_decode_t<TIn, 128, 64>(q, k, v, la, beta, state, o, n_heads, T, H, gate,
                                         flags, stream);
  if (dk == 64 && dv == 128)
    return launch_decode_t<TIn, 64, 128>(q, k, v, la, beta, state, o, n_heads, T, H, gate,
                                         flags, stream);
  return launch_decode_t<TIn, 64, 64>(q, k, v, la, beta, state, o, n_heads, T, H, gate, flags,
                                      stream);
}

// n_heads = B * H; T tokens per sequence.
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* la,
                          const float* beta, float* state, int dk, int dv, bool bf16,
                          void* o, int n_heads, int T, int H, int gate, unsigned flags,
                          cudaStream_t stream) {
  if (n_heads == 0 || T == 0) return cudaSuccess;
  if (bf16)
    return launch_decode_dtype<__nv_bfloat16>(q, k, v, la, beta, state, dk, dv, o, n_heads,
                                              T, H, gate, flags, stream);
  return launch_decode_dtype<float>(q, k, v, la, beta, state, dk, dv, o, n_heads, T, H, gate,
                                    flags, stream);
}

}  // namespace kda
