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
// exchange per token. Two kernels: the single step (any gate form and
// prologue; the plain form compiled on its own), and the several-token one.
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

// The decode step (one token; any gate form; the prologue flags applied to
// the small per-head vectors).
// CTA (head, slice) owns value columns [slice * DV / SPLIT, +DV / SPLIT).
// Within a CTA each lane owns one 4-column group; LPR = columns / 4 lanes
// cover a row, so a warp instruction reads RPI = 32 / LPR whole rows (512
// contiguous bytes per warp for 128 columns). With SPLIT >= 2, 64 registers
// per thread keep four CTAs per SM in flight.
template <int SPLIT>
constexpr int decode_min_blocks() { return SPLIT == 1 ? 2 : 4; }

// kForms: the gate form and prologue flags are read (gate, flags); without
// it the kernel is the plain step (per-channel gate, ready inputs).
template <typename TIn, int DK, int DV, int SPLIT, bool kForms>
__global__ void __launch_bounds__(256, decode_min_blocks<SPLIT>())
decode_step_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                   const TIn* __restrict__ v, const float* __restrict__ log_alpha,
                   const float* __restrict__ beta, float* __restrict__ state,
                   TIn* __restrict__ o, int gate_arg, unsigned flags_arg) {
  constexpr int kWarps = 8;
  constexpr int CW = DV / SPLIT;          // value columns of this CTA
  const int gate = kForms ? gate_arg : kGateChannel;
  const unsigned flags = kForms ? flags_arg : 0u;
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
  __shared__ float s_kq[kWarps], s_nk[kWarps], s_nq[kWarps];
  const bool raw_qk = flags & kRawQK;

  float* S = state + (size_t)head * DK * DV;

  // Launched with programmatic dependent launch, this grid can be scheduled
  // while the previous kernel on the stream finishes; nothing is read before
  // that kernel's writes are visible (it may have produced q, k, v or the
  // state), so the wait comes first.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Issue the state loads first: they are the bytes that matter.
  float4 s[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)row * DV + col));
  }
  float kk0 = 0.f, qq0 = 0.f, la0 = 0.f;
  if (threadIdx.x < DK) {
    kk0 = Io<TIn>::load(k + (size_t)head * DK + threadIdx.x);
    qq0 = Io<TIn>::load(q + (size_t)head * DK + threadIdx.x);
    if (gate == kGateChannel) la0 = __ldg(log_alpha + (size_t)head * DK + threadIdx.x);
    else if (gate == kGateScalar) la0 = __ldg(log_alpha + head);
  }

  // Small per-head vectors: k, q (SiLU of raw projections; their norms are
  // applied as scales below), the decay alpha; k . q (and the squared norms)
  // per warp.
  float kq_part = 0.f, nk_part = 0.f, nq_part = 0.f;
  if (threadIdx.x < DK) {
    if (raw_qk) {
      kk0 = silu_f(kk0);
      qq0 = silu_f(qq0);
      nk_part = kk0 * kk0;
      nq_part = qq0 * qq0;
    }
    s_k[threadIdx.x] = kk0;
    s_q[threadIdx.x] = qq0;
    s_a[threadIdx.x] = gate == kGateNone ? 1.f : decay_from(la0, flags);
    kq_part = kk0 * qq0;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kq_part += __shfl_xor_sync(0xffffffffu, kq_part, off);
  if (raw_qk) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      nk_part += __shfl_xor_sync(0xffffffffu, nk_part, off);
      nq_part += __shfl_xor_sync(0xffffffffu, nq_part, off);
    }
  }
  if (lane == 0) {
    s_kq[warp] = kq_part;
    s_nk[warp] = nk_part;
    s_nq[warp] = nq_part;
  }
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
  // L2 normalisation of SiLU(k), SiLU(q) (x / max(|x|, 1e-12)) as scales of
  // r, p, k . q and k (exactly 1 without the prologue)
  float ik = 1.f, iq = 1.f;
  if (raw_qk) {
    float nk = 0.f, nq = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      nk += s_nk[w];
      nq += s_nq[w];
    }
    ik = 1.f / fmaxf(sqrtf(nk), 1e-12f);
    iq = 1.f / fmaxf(sqrtf(nq), 1e-12f);
    kq = kq * ik * iq;
  }
  float bb = __ldg(beta + head);
  if (flags & kRawBeta) bb = sigmoid_f(bb);
  const float rr[4] = {r.x, r.y, r.z, r.w}, pp[4] = {p.x, p.y, p.z, p.w};
  float d[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    d[j] = bb * (Io<TIn>::load(v + (size_t)head * DV + col + j) - rr[j] * ik);
    if (warp == 0 && sub == 0)
      Io<TIn>::store(o + (size_t)head * DV + col + j, fmaf(kq, d[j], pp[j] * iq));
  }

  // S = S' + k d^T, written once.
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    const float kk = s_k[row] * ik;
    s[i].x = fmaf(kk, d[0], s[i].x); s[i].y = fmaf(kk, d[1], s[i].y);
    s[i].z = fmaf(kk, d[2], s[i].z); s[i].w = fmaf(kk, d[3], s[i].w);
    __stcs(reinterpret_cast<float4*>(S + (size_t)row * DV + col), s[i]);
  }
  // the next kernel on the stream may be scheduled now (its reads still wait
  // for this grid to finish)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Calls with 2 to 16 tokens (any gate form, prologue flags):
// the same state pass, with all T tokens' inputs staged into shared memory
// first (k, q and the decay per key row after the prologue; v of this CTA's
// columns; beta, k.q and the normalisation scales per token), which also
// overlaps those loads with the state loads. The token loop then needs two
// CTA barriers per token (the cross-warp part of r and p is added once per
// value, not by every warp; double-buffered).
template <typename TIn, int DK, int DV, int SPLIT>
__global__ void __launch_bounds__(256, decode_min_blocks<SPLIT>())
decode_multi_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                    const TIn* __restrict__ v, const float* __restrict__ log_alpha,
                    const float* __restrict__ beta, float* __restrict__ state,
                    TIn* __restrict__ o, int T, int H, int gate, unsigned flags) {
  constexpr int kWarps = 8, kMaxT = 16;
  constexpr int CW = DV / SPLIT;
  constexpr int LPR = CW / 4;
  constexpr int RPI = 32 / LPR;
  constexpr int NI = DK / (kWarps * RPI);
  static_assert(CW % 4 == 0 && 32 % LPR == 0 && DK % (kWarps * RPI) == 0, "shape");

  const int head = blockIdx.x / SPLIT, slice = blockIdx.x % SPLIT;   // head = b * H + h
  const int b = head / H, h = head - b * H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cg = lane % LPR, sub = lane / LPR;
  const int col = slice * CW + 4 * cg;
  const bool raw_qk = flags & kRawQK;

  // per token and key row: {decay, k, q, unused}, one 16-byte load per row
  __shared__ float4 s_akq[kMaxT][DK];
  __shared__ __align__(16) float s_v[kMaxT][CW];
  __shared__ float s_beta[kMaxT], s_kq[kMaxT], s_ik[kMaxT], s_iq[kMaxT];
  __shared__ float4 s_red[2][kWarps][2][LPR];
  __shared__ __align__(16) float s_fin[2][2][4 * LPR];   // r and p of the CTA's columns

  // programmatic dependent launch: wait for the previous kernel on the stream
  // (it may update this state) before reading anything
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float* S = state + (size_t)head * DK * DV;
  float4 s[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)row * DV + col));
  }

  // Stage the tokens: warp w takes tokens w, w + 8.
  for (int t = warp; t < T; t += kWarps) {
    const size_t tok = ((size_t)b * T + t) * H + h;
    // k . q is summed in the plain step's order (a warp tree over each 32
    // channels, then the groups in turn), so a call over T tokens matches T
    // single-token calls bit for bit.
    float kqg[DK / 32], nk = 0.f, nq = 0.f;
#pragma unroll
    for (int g = 0; g < DK / 32; ++g) {
      const int i = lane + 32 * g;
      float kk = Io<TIn>::load(k + tok * DK + i);
      float qq = Io<TIn>::load(q + tok * DK + i);
      if (raw_qk) {
        kk = silu_f(kk);
        qq = silu_f(qq);
        nk = fmaf(kk, kk, nk);
        nq = fmaf(qq, qq, nq);
      }
      float a = 1.f;
      if (gate == kGateChannel) a = decay_from(__ldg(log_alpha + tok * DK + i), flags);
      else if (gate == kGateScalar) a = decay_from(__ldg(log_alpha + tok), flags);
      s_akq[t][i] = make_float4(a, kk, qq, 0.f);
      kqg[g] = kk * qq;
    }
    for (int j = lane; j < CW; j += 32) s_v[t][j] = Io<TIn>::load(v + tok * DV + slice * CW + j);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int g = 0; g < DK / 32; ++g) kqg[g] += __shfl_xor_sync(0xffffffffu, kqg[g], off);
      nk += __shfl_xor_sync(0xffffffffu, nk, off);
      nq += __shfl_xor_sync(0xffffffffu, nq, off);
    }
    float kq = 0.f;
#pragma unroll
    for (int g = 0; g < DK / 32; ++g) kq += kqg[g];
    if (lane == 0) {
      // L2 normalisation of SiLU(k), SiLU(q): x / max(|x|, 1e-12)
      const float ik = raw_qk ? 1.f / fmaxf(sqrtf(nk), 1e-12f) : 1.f;
      const float iq = raw_qk ? 1.f / fmaxf(sqrtf(nq), 1e-12f) : 1.f;
      float bb = __ldg(beta + tok);
      if (flags & kRawBeta) bb = sigmoid_f(bb);
      s_ik[t] = ik;
      s_iq[t] = iq;
      s_kq[t] = kq * ik * iq;
      s_beta[t] = bb;
    }
  }
  __syncthreads();

  for (int t = 0; t < T; ++t) {
    const int buf = t & 1;
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int row = (warp + i * kWarps) * RPI + sub;
      const float4 akq = s_akq[t][row];
      const float a = akq.x, kk = akq.y, qq = akq.z;
      s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
      r.x = fmaf(s[i].x, kk, r.x); r.y = fmaf(s[i].y, kk, r.y);
      r.z = fmaf(s[i].z, kk, r.z); r.w = fmaf(s[i].w, kk, r.w);
      p.x = fmaf(s[i].x, qq, p.x); p.y = fmaf(s[i].y, qq, p.y);
      p.z = fmaf(s[i].z, qq, p.z); p.w = fmaf(s[i].w, qq, p.w);
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
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
    // The warps' partial sums, added once per value (in warp order, as the
    // plain step does) by the first 8 LPR threads, then read by all.
    if (threadIdx.x < 8 * LPR) {
      const int rp = threadIdx.x / (4 * LPR), cc = threadIdx.x % (4 * LPR);
      const float* part = reinterpret_cast<const float*>(&s_red[buf][0][rp][0]) + cc;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) acc += part[w * 8 * LPR];
      s_fin[buf][rp][cc] = acc;
    }
    __syncthreads();
    r = *reinterpret_cast<const float4*>(&s_fin[buf][0][4 * cg]);
    p = *reinterpret_cast<const float4*>(&s_fin[buf][1][4 * cg]);
    const float ik = s_ik[t], iq = s_iq[t], kq = s_kq[t], bb = s_beta[t];
    const float4 vv = *reinterpret_cast<const float4*>(&s_v[t][4 * cg]);
    const float d[4] = {bb * (vv.x - r.x * ik), bb * (vv.y - r.y * ik), bb * (vv.z - r.z * ik),
                        bb * (vv.w - r.w * ik)};
    if (warp == 0 && sub == 0) {
      const size_t tok = ((size_t)b * T + t) * H + h;
      Io<TIn>::store(o + tok * DV + col, fmaf(kq, d[0], p.x * iq));
      Io<TIn>::store(o + tok * DV + col + 1, fmaf(kq, d[1], p.y * iq));
      Io<TIn>::store(o + tok * DV + col + 2, fmaf(kq, d[2], p.z * iq));
      Io<TIn>::store(o + tok * DV + col + 3, fmaf(kq, d[3], p.w * iq));
    }
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int row = (warp + i * kWarps) * RPI + sub;
      const float kk = s_akq[t][row].y * ik;
      s[i].x = fmaf(kk, d[0], s[i].x); s[i].y = fmaf(kk, d[1], s[i].y);
      s[i].z = fmaf(kk, d[2], s[i].z); s[i].w = fmaf(kk, d[3], s[i].w);
    }
  }
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int row = (warp + i * kWarps) * RPI + sub;
    __stcs(reinterpret_cast<float4*>(S + (size_t)row * DV + col), s[i]);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename TIn, int DK, int DV, int kSplit>
static cudaError_t launch_decode_split(const void* q, const void* k, const void* v,
                                       const float* la, const float* beta, float* state,
                                       void* o, int n_heads, int T, int H, int gate,
                                       unsigned flags, cudaStream_t stream) {
  // programmatic dependent launch: scheduled while the previous kernel on
  // the stream finishes (the kernels wait for it before reading anything)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(n_heads * kSplit));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (T == 1) {
    const bool forms = gate != kGateChannel || flags != 0u;
    if (forms)
      return cudaLaunchKernelEx(&cfg, decode_step_kernel<TIn, DK, DV, kSplit, true>,
                                (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, state,
                                (TIn*)o, gate, flags);
    return cudaLaunchKernelEx(&cfg, decode_step_kernel<TIn, DK, DV, kSplit, false>,
                              (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, state,
                              (TIn*)o, gate, flags);
  }
  return cudaLaunchKernelEx(&cfg, decode_multi_kernel<TIn, DK, DV, kSplit>, (const TIn*)q,
                            (const TIn*)k, (const TIn*)v, la, beta, state, (TIn*)o, T, H, gate,
                            flags);
}

// Value slices per head: 2 (dv = 128) or 1 (dv = 64) fill the GPU once there
// are a few hundred CTAs; with fewer heads (small-batch decode, latency-bound)
// 16-column slices spread the state over eight or four times as many SMs.
constexpr int kFewHeads = 128;

template <typename TIn, int DK, int DV>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v,
                                   const float* la, const float* beta, float* state, void* o,
                                   int n_heads, int T, int H, int gate, unsigned flags,
                                   cudaStream_t stream) {
  if (n_heads < kFewHeads)
    return launch_decode_split<TIn, DK, DV, DV / 16>(q, k, v, la, beta, state, o, n_heads, T,
                                                     H, gate, flags, stream);
  return launch_decode_split<TIn, DK, DV, DV == 128 ? 2 : 1>(q, k, v, la, beta, state, o,
                                                             n_heads, T, H, gate, flags, stream);
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
