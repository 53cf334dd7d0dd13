// kda_recurrent.cu -- token-recurrent KDA prefill (fp32 state in registers).
//
// Pages: "22580: from GPT-2 to Kimi K3, explained", section "DeltaNet, or
// Parallelizing Linear Transformers with Delta Rule" (the direct prefill is a
// token loop carrying S), with the per-channel decay of "Gated Delta Net" /
// "KDA / Kimi Linear". Every token applies
//     S' = Diag(alpha_t) S; r = S'^T k; d = beta (v - r); S = S' + k d^T;
//     o = S^T q = S'^T q + (k . q) d
// exactly as written (fp32, exact gate, log_alpha = -inf clears). This is the
// path for fp32 inputs and serves as an independent GPU cross-check of the
// chunked tensor-core kernel. It takes every gate form (per key channel, one
// scalar per token as in "Gated Delta Net", or none) and the optional input
// prologue of the cached forward in "DeltaNet, or Fast Weight Programmers"
// (SiLU and L2 normalisation of q and k, sigmoid of beta; a gate given as
// logits x decays by sigmoid(x)).
//
// Layout: one CTA per (sequence, head, 32-column slice of dv); 128 threads.
// Lane j owns value column j of the slice; warp g owns key rows
// [g * dk/4, (g+1) * dk/4). The per-token vectors (k, q, alpha) are staged
// through double-buffered shared memory, and the next token's inputs are
// loaded into registers while the current token is computed.
#include "kda_common.cuh"

namespace kda {

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(128)
recurrent_prefill_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                         const TIn* __restrict__ v, const float* __restrict__ log_alpha,
                         const float* __restrict__ beta, const float* __restrict__ init_state,
                         const int32_t* __restrict__ cu_seqlens, int T, int H,
                         TIn* __restrict__ o, float* __restrict__ final_state, int gate,
                         unsigned flags) {
  constexpr int kGroups = 4;
  constexpr int RPT = DK / kGroups;     // key rows per thread
  constexpr int kSlices = DV / 32;

  const int slice = blockIdx.x % kSlices;
  const int head = (blockIdx.x / kSlices) % H;
  const int seq = blockIdx.x / (kSlices * H);
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int col = slice * 32 + lane;
  const int row0 = g * RPT;

  long long t_begin, t_end;
  seq_bounds(cu_seqlens, seq, T, &t_begin, &t_end);

  __shared__ float s_k[2][DK], s_q[2][DK], s_a[2][DK];
  __shared__ float s_red[2][2][kGroups][32];
  __shared__ float s_kq[2][kGroups][3];   // k.q and, for raw inputs, |k|^2 and |q|^2
  const bool raw_qk = flags & kRawQK;

  const size_t state_off = ((size_t)seq * H + head) * DK * DV;
  float s[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
    s[i] = init_state ? init_state[state_off + (size_t)(row0 + i) * DV + col] : 0.f;

  // Registers holding the next token's inputs.
  float nk = 0.f, nq = 0.f, nla = 0.f, nv = 0.f, nb = 0.f;
  auto fetch = [&](long long t) {
    const size_t tok = (size_t)t * H + head;
    if (threadIdx.x < DK) {
      nk = Io<TIn>::load(k + tok * DK + threadIdx.x);
      nq = Io<TIn>::load(q + tok * DK + threadIdx.x);
      nla = gate == kGateChannel ? __ldg(log_alpha + tok * DK + threadIdx.x)
          : gate == kGateScalar  ? __ldg(log_alpha + tok) : 0.f;
    }
    nv = Io<TIn>::load(v + tok * DV + col);
    nb = __ldg(beta + tok);
  };
  if (t_begin < t_end) fetch(t_begin);

  for (long long t = t_begin; t < t_end; ++t) {
    const int buf = (int)(t & 1);
    float part[3] = {0.f, 0.f, 0.f};
    if (threadIdx.x < DK) {
      float kk = nk, qq = nq;
      if (raw_qk) {
        kk = silu_f(kk);
        qq = silu_f(qq);
        part[1] = kk * kk;
        part[2] = qq * qq;
      }
      s_k[buf][threadIdx.x] = kk;
      s_q[buf][threadIdx.x] = qq;
      s_a[buf][threadIdx.x] = gate == kGateNone ? 1.f : decay_from(nla, flags);
      part[0] = kk * qq;
    }
#pragma unroll
    for (int j = 0; j < 3; ++j)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], off);
    if (lane == 0) {
      s_kq[buf][g][0] = part[0];
      s_kq[buf][g][1] = part[1];
      s_kq[buf][g][2] = part[2];
    }
    const float vv = nv, bb = (flags & kRawBeta) ? sigmoid_f(nb) : nb;
    __syncthreads();
    if (t + 1 < t_end) fetch(t + 1);

    float r = 0.f, p = 0.f;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      s[i] *= s_a[buf][row0 + i];
      r = fmaf(s[i], s_k[buf][row0 + i], r);
      p = fmaf(s[i], s_q[buf][row0 + i], p);
    }
    s_red[buf][0][g][lane] = r;
    s_red[buf][1][g][lane] = p;
    __syncthreads();

    r = 0.f;
    p = 0.f;
    float kq = 0.f, nk2 = 0.f, nq2 = 0.f;
#pragma unroll
    for (int w = 0; w < kGroups; ++w) {
      r += s_red[buf][0][w][lane];
      p += s_red[buf][1][w][lane];
      kq += s_kq[buf][w][0];
      nk2 += s_kq[buf][w][1];
      nq2 += s_kq[buf][w][2];
    }
    // L2 normalisation of SiLU(k), SiLU(q), folded into the reductions.
    const float ik = raw_qk ? 1.f / fmaxf(sqrtf(nk2), 1e-12f) : 1.f;
    const float iq = raw_qk ? 1.f / fmaxf(sqrtf(nq2), 1e-12f) : 1.f;
    const float d = bb * (vv - r * ik);
    if (g == 0)
      Io<TIn>::store(o + ((size_t)t * H + head) * DV + col, fmaf(kq * ik * iq, d, p * iq));
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = fmaf(s_k[buf][row0 + i] * ik, d, s[i]);
  }

  if (final_state) {
#pragma unroll
    for (int i = 0; i < RPT; ++i) final_state[state_off + (size_t)(row0 + i) * DV + col] = s[i];
  }
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_rec_t(const void* q, const void* k, const void* v, const float* la,
                                const float* beta, const float* s0, const int32_t* cu,
                                int n_seq, int T, int H, void* o, float* sT, int gate,
                                unsigned flags, cudaStream_t stream) {
  const long long blocks = (long long)n_seq * H * (DV / 32);
  recurrent_prefill_kernel<TIn, DK, DV><<<(unsigned)blocks, 128, 0, stream>>>(
      (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, s0, cu, T, H, (TIn*)o, sT, gate,
      flags);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_rec_dtype(const void* q, const void* k, const void* v,
                                    const float* la, const float* beta, const float* s0,
                                    const int32_t* cu, int n_seq, int T, int H, int dk,
                                    int dv, void* o, float* sT, int gate, unsigned flags,
                                    cudaStream_t stream) {
  if (dk == 128 && dv == 128)
    return launch_rec_t<TIn, 128, 128>(q, k, v, la, beta, s0, cu, n_seq, T, H, o, sT, gate,
                                       flags, stream);
  if (dk == 128 && dv == 64)
    return launch_rec_t<TIn, 128, 64>(q, k, v, la, beta, s0, cu, n_seq, T, H, o, sT, gate,
                                      flags, stream);
  if (dk == 64 && dv == 128)
    return launch_rec_t<TIn, 64, 128>(q, k, v, la, beta, s0, cu, n_seq, T, H, o, sT, gate,
                                      flags, stream);
  return launch_rec_t<TIn, 64, 64>(q, k, v, la, beta, s0, cu, n_seq, T, H, o, sT, gate, flags,
                                   stream);
}

cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const float* la,
                             const float* beta, const float* s0, const int32_t* cu,
                             int n_seq, int T, int H, int dk, int dv, bool bf16, void* o,
                             float* sT, int gate, unsigned flags, cudaStream_t stream) {
  if (n_seq == 0) return cudaSuccess;
  if (bf16)
    return launch_rec_dtype<__nv_bfloat16>(q, k, v, la, beta, s0, cu, n_seq, T, H, dk, dv,
                                           o, sT, gate, flags, stream);
  return launch_rec_dtype<float>(q, k, v, la, beta, s0, cu, n_seq, T, H, dk, dv, o, sT, gate,
                                 flags, stream);
}

}  // namespace kda
