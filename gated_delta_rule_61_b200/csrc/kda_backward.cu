// kda_backward.cu -- reverse mode of the KDA recurrence (the gradients a
// training step needs), token-recurrent with state checkpoints.
//
// Pages: "22580: from GPT-2 to Kimi K3, explained", section "DeltaNet, or
// Parallelizing Linear Transformers with Delta Rule" (the chunk-wise form
// exists for hardware-efficient training), with the recurrence of "DeltaNet,
// or Fast Weight Programmers" and the decay of "Gated Delta Net" / "KDA /
// Kimi Linear". Forward, per token:
//     S' = Diag(a) S;  r = S'^T k;  d = beta (v - r);  S_t = S' + k d^T;  o = S_t^T q
// Backward, with G = dL/dS_t (starting from dL/dS_final), per token in
// reverse:
//     G += q do^T;             dq = S_t do
//     dd = G^T k;              dk = G d
//     dbeta = dd . (v - r);    dv = beta dd;    dr = -beta dd
//     G' = G + k dr^T;         dk += S' dr
//     dlog_alpha_i = sum_j S'_ij G'_ij;         G = Diag(a) G'
// and dL/dS_0 = G at the end.
//
// Layout: one CTA per (sequence, head, slice of kCols value columns: 32, or
// 8 when chains are few, so that enough CTAs are resident to hide the
// per-token latency); thread i owns key row i of the slice's columns of S
// and of G (registers). Sums over
// the value columns (dq, dk, dlog_alpha) stay inside a thread; the two sums
// over key rows per token (r in the recomputation, dd in the reverse step)
// are a halving-exchange reduction over the warp's lanes plus one shared-
// memory exchange across warps. Column slices of one head add their partial
// dq, dk, dlog_alpha and dbeta into the fp32 outputs (red.add; the slices'
// order is not fixed, so these gradients can differ between runs in the
// last bits). dv and dL/dS_0 are written by their slice alone.
//
// The states are not stored per token: a first forward pass writes the
// slice of S at the start of every block of kBlk tokens to the workspace;
// then, block by block from the last, the block's states are recomputed from
// its checkpoint into a per-CTA scratch (kBlk x dk x kCols fp32, L2-resident)
// and walked backwards (the next token's state is loaded while the current
// one is processed). S' is recovered as S_t - k d^T with d kept from the
// recomputation. Each block's inputs are staged in shared memory once, so
// the per-token steps wait on no global load.
//
// Input prologue (raw projections, as in the forward's flags): a small first
// kernel stores each (token, head) row's 1 / max(|SiLU(q)|, 1e-12) and the
// same for k in the workspace; the staging applies the prologue with them
// (q and k through SiLU and that scale, beta and the decay through the
// sigmoid), the token steps then give the gradients with respect to the
// transformed inputs, and a last kernel carries them back to the raw ones:
// through the normalisation's
// Jacobian (I - n n^T) / max(|u|, 1e-12) and SiLU's derivative
// s (1 + x (1 - s)) for q and k, sigmoid's s (1 - s) for beta, and
// d log sigmoid(x) / dx = sigmoid(-x) for the gate.
#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int kBlk = 16;       // tokens per checkpoint block
constexpr unsigned kRawQK = 1u, kRawBeta = 2u, kRawGate = 4u;   // prologue flags

__device__ __forceinline__ float sigm(float x) { return 1.0f / (1.0f + expf(-x)); }
// the staging's sigmoid: approximate exponential and reciprocal (relative
// error a few 1e-7, far below the gradients' tolerance; 1 / inf = 0)
__device__ __forceinline__ float sigm_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
constexpr int kColsWide = 32, kColsNarrow = 8;   // value columns per CTA

// Sum over the warp of 32 per-lane vectors of N values (N a power of two,
// at most 32): halving exchanges over offsets N/2 .. 1 (a lane keeps the
// half of its values selected by its lane bit and adds the partner's copy of
// that half), then plain exchanges over offsets N .. 16; lane l returns the
// warp sum of value l % N.
template <int N>
__device__ __forceinline__ float warp_transpose_sum(float* v, int lane) {
#pragma unroll
  for (int off = N / 2; off >= 1; off >>= 1) {
    const bool up = lane & off;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float keep = up ? v[j + off] : v[j];
      const float send = up ? v[j] : v[j + off];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float x = v[0];
#pragma unroll
  for (int off = N; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ void red_add(float* p, float x) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(x) : "memory");
}

// kPro: the inputs are raw projections (flags); without it the kernel is
// the plain reverse sweep on ready inputs.
template <typename TIn, int DK, int DV, int kCols, bool kPro>
__global__ void __launch_bounds__(DK, kCols == kColsNarrow ? 1024 / DK : 2)
backward_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                const float* __restrict__ log_alpha, const float* __restrict__ beta,
                const float* __restrict__ init_state, const int32_t* __restrict__ cu_seqlens,
                const TIn* __restrict__ d_o, const float* __restrict__ d_final, int T, int H,
                int gate, unsigned flags, const float* __restrict__ inv_norm,
                float* __restrict__ dq, float* __restrict__ dk,
                float* __restrict__ dv, float* __restrict__ dla, float* __restrict__ dbeta,
                float* __restrict__ d_init, float* __restrict__ ckpt, float* __restrict__ scratch) {
  constexpr int kSlices = DV / kCols;
  constexpr int kWarps = DK / 32;
  const int slice = blockIdx.x % kSlices;
  const int head = (blockIdx.x / kSlices) % H;
  const int seq = blockIdx.x / (kSlices * H);
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const int col0 = slice * kCols;

  long long t_begin, t_end;
  seq_bounds(cu_seqlens, seq, T, &t_begin, &t_end);
  const long long len = t_end - t_begin;
  const int n_blk = (int)((len + kBlk - 1) / kBlk);
  // This sequence's checkpoint blocks start at floor(t_begin / kBlk) + seq,
  // which leaves room for ceil(len / kBlk) blocks before the next sequence's.
  const long long blk0 = t_begin / kBlk + seq;
  auto ckpt_row = [&](int b) {
    return ckpt + ((((size_t)(blk0 + b) * H + head) * kSlices + slice) * DK + i) * kCols;
  };
  float* scr = scratch + (size_t)blockIdx.x * kBlk * DK * kCols + (size_t)i * kCols;

  // One block's inputs, staged once per block: key-row vectors (k, q, decay)
  // and this slice's columns of v and d_o, beta per token.
  __shared__ float s_k[kBlk][DK], s_q[kBlk][DK], s_a[kBlk][DK];
  __shared__ float s_v[kBlk][kCols], s_do[kBlk][kCols];
  __shared__ float s_beta[kBlk];
  __shared__ float s_part[kWarps][kCols];
  __shared__ float s_d[kBlk][kCols], s_vr[kBlk][kCols];   // d_j and v_j - r_j per token
  const bool raw_qk = kPro && (flags & kRawQK);

  auto stage = [&](long long tb, int nb, bool with_q) {
    __syncthreads();   // the previous block's values are no longer read
    for (int s = 0; s < nb; ++s) {
      const size_t tok = (size_t)(tb + s) * H + head;
      if constexpr (kPro) {
        // raw q, k: SiLU(x) / max(|SiLU(x)|, 1e-12), the row's scale from the
        // first kernel (inv_norm[2 row] for q, [2 row + 1] for k)
        const float kx = Io<TIn>::load(k + tok * DK + i);
        s_k[s][i] = raw_qk ? kx * sigm_fast(kx) * __ldg(inv_norm + 2 * tok + 1) : kx;
        if (with_q) {
          const float qx = Io<TIn>::load(q + tok * DK + i);
          s_q[s][i] = raw_qk ? qx * sigm_fast(qx) * __ldg(inv_norm + 2 * tok) : qx;
        }
        float a = 1.f;
        if (gate != 2) {
          const float x = gate == 0 ? __ldg(log_alpha + tok * DK + i) : __ldg(log_alpha + tok);
          a = (flags & kRawGate) ? sigm_fast(x) : expf(x);   // exp(log sigmoid(x)) = sigmoid(x)
        }
        s_a[s][i] = a;
      } else {
        s_k[s][i] = Io<TIn>::load(k + tok * DK + i);
        if (with_q) s_q[s][i] = Io<TIn>::load(q + tok * DK + i);
        s_a[s][i] = gate == 0 ? expf(__ldg(log_alpha + tok * DK + i))
                  : gate == 1 ? expf(__ldg(log_alpha + tok)) : 1.f;
      }
    }
    for (int e = i; e < nb * kCols; e += DK) {
      const int s = e / kCols, j = e - (e / kCols) * kCols;
      const size_t tok = (size_t)(tb + s) * H + head;
      s_v[s][j] = Io<TIn>::load(v + tok * DV + col0 + j);
      if (with_q) s_do[s][j] = Io<TIn>::load(d_o + tok * DV + col0 + j);
    }
    if (i < nb) {
      const float b = __ldg(beta + (size_t)(tb + i) * H + head);
      s_beta[i] = (kPro && (flags & kRawBeta)) ? sigm_fast(b) : b;
    }
    __syncthreads();
  };

  const size_t state_off = ((size_t)seq * H + head) * DK * DV + (size_t)i * DV + col0;
  float S[kCols];
#pragma unroll
  for (int j = 0; j < kCols; j += 4) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init_state) x = *reinterpret_cast<const float4*>(init_state + state_off + j);
    S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
  }

  // One forward step of token slot s on S (row i, this slice's columns);
  // leaves d_j and v_j - r_j in s_d[s], s_vr[s].
  auto forward_step = [&](int s) {
    const float a = s_a[s][i], ki = s_k[s][i];
    float part[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) {
      S[j] *= a;
      part[j] = S[j] * ki;
    }
    const float rl = warp_transpose_sum<kCols>(part, lane);
    if (lane < kCols) s_part[warp][lane] = rl;
    __syncthreads();
    if (warp == 0 && lane < kCols) {
      float r = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) r += s_part[w][lane];
      const float vr = s_v[s][lane] - r;
      s_vr[s][lane] = vr;
      s_d[s][lane] = s_beta[s] * vr;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kCols; ++j) S[j] = fmaf(ki, s_d[s][j], S[j]);
  };

  // Pass 1: forward over the sequence, checkpointing S at every block start.
  for (int b = 0; b < n_blk; ++b) {
    float* cp = ckpt_row(b);
#pragma unroll
    for (int j = 0; j < kCols; j += 4)
      __stcg(reinterpret_cast<float4*>(cp + j), make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
    if (b + 1 == n_blk) break;
    const long long tb = t_begin + (long long)b * kBlk;
    stage(tb, kBlk, false);
    for (int s = 0; s < kBlk; ++s) forward_step(s);
  }

  // Pass 2: blocks from the last; G = dL/dS.
  float G[kCols];
#pragma unroll
  for (int j = 0; j < kCols; j += 4) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (d_final) x = *reinterpret_cast<const float4*>(d_final + state_off + j);
    G[j] = x.x; G[j + 1] = x.y; G[j + 2] = x.z; G[j + 3] = x.w;
  }
  for (int b = n_blk - 1; b >= 0; --b) {
    const long long tb = t_begin + (long long)b * kBlk;
    const int nb = (int)((t_end - tb) < kBlk ? (t_end - tb) : kBlk);
    stage(tb, nb, true);
    const float* cp = ckpt_row(b);
#pragma unroll
    for (int j = 0; j < kCols; j += 4) {
      const float4 x = __ldcg(reinterpret_cast<const float4*>(cp + j));
      S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    // recompute the block, keeping S_t per token in the scratch
    for (int s = 0; s < nb; ++s) {
      forward_step(s);
      float* dst = scr + (size_t)s * DK * kCols;
#pragma unroll
      for (int j = 0; j < kCols; j += 4)
        __stcg(reinterpret_cast<float4*>(dst + j), make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
    }
    // reverse sweep; S_t of the next token (s - 1) is loaded while this one
    // is processed
    float Sn[kCols];
    {
      const float* src = scr + (size_t)(nb - 1) * DK * kCols;
#pragma unroll
      for (int j = 0; j < kCols; j += 4) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(src + j));
        Sn[j] = x.x; Sn[j + 1] = x.y; Sn[j + 2] = x.z; Sn[j + 3] = x.w;
      }
    }
    for (int s = nb - 1; s >= 0; --s) {
#pragma unroll
      for (int j = 0; j < kCols; ++j) S[j] = Sn[j];   // S_t
      if (s > 0) {
        const float* src = scr + (size_t)(s - 1) * DK * kCols;
#pragma unroll
        for (int j = 0; j < kCols; j += 4) {
          const float4 x = __ldcg(reinterpret_cast<const float4*>(src + j));
          Sn[j] = x.x; Sn[j + 1] = x.y; Sn[j + 2] = x.z; Sn[j + 3] = x.w;
        }
      }
      const size_t tok = (size_t)(tb + s) * H + head;
      const float ki = s_k[s][i], qi = s_q[s][i], a = s_a[s][i], bt = s_beta[s];
      // o_t = S_t^T q: G += q do^T; dq_i = sum_j S_t,ij do_j
      float dqi = 0.f;
      float part[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) {
        const float doj = s_do[s][j];
        dqi = fmaf(S[j], doj, dqi);
        G[j] = fmaf(qi, doj, G[j]);
        part[j] = G[j] * ki;
      }
      // dd_j = sum_i G_ij k_i
      const float ddl = warp_transpose_sum<kCols>(part, lane);
      if (lane < kCols) s_part[warp][lane] = ddl;
      __syncthreads();
      // S_t = S' + k d^T; d = beta (v - r); r = S'^T k
      float dki = 0.f, dlai = 0.f, dbt = 0.f;
#pragma unroll
      for (int j = 0; j < kCols; ++j) {
        float ddj = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) ddj += s_part[w][j];
        const float dj = s_d[s][j];
        const float sp = fmaf(-ki, dj, S[j]);          // S'_ij
        const float dr = -bt * ddj;
        dki = fmaf(G[j], dj, dki);                     // G d
        dki = fmaf(sp, dr, dki);                       // S' dr
        dbt = fmaf(ddj, s_vr[s][j], dbt);
        G[j] = fmaf(ki, dr, G[j]);                     // G'
        dlai = fmaf(sp, G[j], dlai);
        G[j] *= a;
      }
      red_add(dq + tok * DK + i, dqi);
      red_add(dk + tok * DK + i, dki);
      if (gate == 0) red_add(dla + tok * DK + i, dlai);
      if (i == 0) red_add(dbeta + tok, dbt);
      if (warp == 0 && lane < kCols) {
        float x = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) x += s_part[w][lane];
        dv[tok * DV + col0 + lane] = bt * x;
      }
      if (gate == 1) {
        // one decay per token: sum over the key rows of the CTA
        float x = dlai;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (lane == 0) red_add(dla + tok, x);
      }
      __syncthreads();   // s_part is reused by the next token
    }
  }
  if (d_init) {
#pragma unroll
    for (int j = 0; j < kCols; j += 4)
      *reinterpret_cast<float4*>(d_init + state_off + j) = make_float4(G[j], G[j + 1], G[j + 2], G[j + 3]);
  }
}

// 1 / max(|SiLU(x)|, 1e-12) of every (token, head) row of raw q and k (one
// warp per row), into inv_norm[2 row] (q) and inv_norm[2 row + 1] (k).
template <typename TIn, int DK>
__global__ void __launch_bounds__(256)
prologue_norms_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, long long rows,
                      float* __restrict__ inv_norm) {
  constexpr int NJ = DK / 32;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;   // the whole warp leaves together
  float nq = 0.f, nk = 0.f;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const size_t idx = (size_t)row * DK + lane + 32 * j;
    const float xq = Io<TIn>::load(q + idx), xk = Io<TIn>::load(k + idx);
    const float uq = xq * sigm(xq), uk = xk * sigm(xk);
    nq = fmaf(uq, uq, nq);
    nk = fmaf(uk, uk, nk);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    nq += __shfl_xor_sync(0xffffffffu, nq, off);
    nk += __shfl_xor_sync(0xffffffffu, nk, off);
  }
  if (lane == 0)
    *reinterpret_cast<float2*>(inv_norm + 2 * row) =
        make_float2(1.f / fmaxf(sqrtf(nq), 1e-12f), 1.f / fmaxf(sqrtf(nk), 1e-12f));
}

// The prologue's reverse mode, after the token steps: one warp per (token,
// head) row. The gradients with respect to the transformed inputs (in dq, dk,
// dbeta, dlog_alpha) become those with respect to the raw inputs, in place.
template <typename TIn, int DK>
__global__ void __launch_bounds__(256)
prologue_vjp_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                    const float* __restrict__ log_alpha, const float* __restrict__ beta,
                    long long rows, int gate, unsigned flags, float* __restrict__ dq,
                    float* __restrict__ dk, float* __restrict__ dla,
                    float* __restrict__ dbeta) {
  constexpr int NJ = DK / 32;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // token * H + head
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;   // the whole warp leaves together
  if (flags & kRawQK) {
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      const TIn* x = which ? k : q;
      float* g = which ? dk : dq;
      float xv[NJ], sv[NJ], uv[NJ], gv[NJ], uu = 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const size_t idx = (size_t)row * DK + lane + 32 * j;
        xv[j] = Io<TIn>::load(x + idx);
        sv[j] = sigm(xv[j]);
        uv[j] = xv[j] * sv[j];
        gv[j] = g[idx];
        uu = fmaf(uv[j], uv[j], uu);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) uu += __shfl_xor_sync(0xffffffffu, uu, off);
      uu = __shfl_sync(0xffffffffu, uu, 0);
      const float r = sqrtf(uu), inv = 1.f / fmaxf(r, 1e-12f);
      // n . g with n = u / max(|u|, 1e-12)
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) dot = fmaf(uv[j] * inv, gv[j], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      dot = __shfl_sync(0xffffffffu, dot, 0);
      const bool proj = r > 1e-12f;   // below it the map is u / 1e-12, a plain scale
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float du = (proj ? fmaf(-uv[j] * inv, dot, gv[j]) : gv[j]) * inv;
        g[(size_t)row * DK + lane + 32 * j] = du * sv[j] * fmaf(xv[j], 1.f - sv[j], 1.f);
      }
    }
  }
  if ((flags & kRawBeta) && lane == 0) {
    const float sb = sigm(__ldg(beta + row));
    dbeta[row] *= sb * (1.f - sb);
  }
  if (flags & kRawGate) {
    if (gate == 0) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const size_t idx = (size_t)row * DK + lane + 32 * j;
        dla[idx] *= sigm(-__ldg(log_alpha + idx));
      }
    } else if (gate == 1 && lane == 0) {
      dla[row] *= sigm(-__ldg(log_alpha + row));
    }
  }
}

}  // namespace bwd

// Workspace: checkpoints (floor(tokens / 16) + n_seq + 1 blocks per head, each
// dk x dv fp32), one 16 x dk x kCols fp32 scratch per CTA (16 x dk x dv per
// head whatever the slice width) and, for raw q and k, two fp32 scales per
// (token, head) row; each region 256-byte aligned.
static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t backward_workspace_bytes(int n_seq, long long tokens, int H, int dk, int dv) {
  if (n_seq <= 0 || H <= 0) return 0;
  const size_t blocks = (size_t)(tokens / bwd::kBlk) + (size_t)n_seq + 1;
  const size_t ck = blocks * (size_t)H * dk * dv * sizeof(float);
  const size_t scr = (size_t)n_seq * H * bwd::kBlk * dk * dv * sizeof(float);
  const size_t nrm = (size_t)tokens * H * 2 * sizeof(float);
  return align256(ck) + align256(scr) + align256(nrm);
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_bwd_t(const void* q, const void* k, const void* v, const float* la,
                                const float* beta, const float* s0, const int32_t* cu,
                                const void* d_o, const float* d_final, int n_seq, int T, int H,
                                int gate, unsigned flags, long long tokens, float* dq, float* dk,
                                float* dv, float* dla, float* dbeta, float* d_init, float* ckpt,
                                float* scratch, float* inv_norm, cudaStream_t stream) {
  const long long rows = tokens * H;
  if ((flags & bwd::kRawQK) && rows > 0) {
    bwd::prologue_norms_kernel<TIn, DK><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
        (const TIn*)q, (const TIn*)k, rows, inv_norm);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // Few chains: narrow slices, so that enough CTAs run to hide the per-token
  // latency of each chain (2 x 148 CTAs of the wide slices fill a B200).
  const long long chains = (long long)n_seq * H;
  const bool narrow = chains * (DV / bwd::kColsWide) < 2 * 148;
#define KDA_BWD_LAUNCH(kC, kPro)                                                               \
  bwd::backward_kernel<TIn, DK, DV, kC, kPro><<<(unsigned)(chains * (DV / kC)), DK, 0, stream>>>( \
      (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, s0, cu, (const TIn*)d_o, d_final,   \
      T, H, gate, flags, inv_norm, dq, dk, dv, dla, dbeta, d_init, ckpt, scratch)
  if (narrow) {
    if (flags) KDA_BWD_LAUNCH(bwd::kColsNarrow, true);
    else KDA_BWD_LAUNCH(bwd::kColsNarrow, false);
  } else {
    if (flags) KDA_BWD_LAUNCH(bwd::kColsWide, true);
    else KDA_BWD_LAUNCH(bwd::kColsWide, false);
  }
#undef KDA_BWD_LAUNCH
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || flags == 0u || tokens == 0) return e;
  bwd::prologue_vjp_kernel<TIn, DK><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
      (const TIn*)q, (const TIn*)k, la, beta, rows, gate, flags, dq, dk, dla, dbeta);
  return cudaGetLastError();
}

// Zeroes the accumulated outputs, then runs the backward kernel.
cudaError_t launch_backward(const void* q, const void* k, const void* v, const float* la,
                            const float* beta, const float* s0, const int32_t* cu,
                            const void* d_o, const float* d_final, int n_seq, int T, int H,
                            int dk, int dv, bool bf16, int gate, unsigned flags, long long tokens,
                            float* dq,
                            float* dkk, float* dvv, float* dla, float* dbeta, float* d_init,
                            void* workspace, cudaStream_t stream) {
  if (n_seq == 0) return cudaSuccess;
  cudaError_t e;
  if (tokens > 0) {
    if ((e = cudaMemsetAsync(dq, 0, sizeof(float) * tokens * H * dk, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dkk, 0, sizeof(float) * tokens * H * dk, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dbeta, 0, sizeof(float) * tokens * H, stream)) != cudaSuccess) return e;
    if (gate != 2) {
      const size_t n = gate == 0 ? (size_t)tokens * H * dk : (size_t)tokens * H;
      if ((e = cudaMemsetAsync(dla, 0, sizeof(float) * n, stream)) != cudaSuccess) return e;
    }
  }
  const size_t blocks = (size_t)(tokens / bwd::kBlk) + (size_t)n_seq + 1;
  const size_t ck = blocks * (size_t)H * dk * dv * sizeof(float);
  const size_t scr = (size_t)n_seq * H * bwd::kBlk * dk * dv * sizeof(float);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* ckpt = reinterpret_cast<float*>(ws);
  float* scratch = reinterpret_cast<float*>(ws + align256(ck));
  float* inv_norm = reinterpret_cast<float*>(ws + align256(ck) + align256(scr));
#define KDA_BWD_ARGS q, k, v, la, beta, s0, cu, d_o, d_final, n_seq, T, H, gate, flags, tokens, dq, \
                     dkk, dvv, dla, dbeta, d_init, ckpt, scratch, inv_norm, stream
  if (bf16) {
    if (dk == 128 && dv == 128) return launch_bwd_t<__nv_bfloat16, 128, 128>(KDA_BWD_ARGS);
    if (dk == 128 && dv == 64) return launch_bwd_t<__nv_bfloat16, 128, 64>(KDA_BWD_ARGS);
    if (dk == 64 && dv == 128) return launch_bwd_t<__nv_bfloat16, 64, 128>(KDA_BWD_ARGS);
    return launch_bwd_t<__nv_bfloat16, 64, 64>(KDA_BWD_ARGS);
  }
  if (dk == 128 && dv == 128) return launch_bwd_t<float, 128, 128>(KDA_BWD_ARGS);
  if (dk == 128 && dv == 64) return launch_bwd_t<float, 128, 64>(KDA_BWD_ARGS);
  if (dk == 64 && dv == 128) return launch_bwd_t<float, 64, 128>(KDA_BWD_ARGS);
  return launch_bwd_t<float, 64, 64>(KDA_BWD_ARGS);
#undef KDA_BWD_ARGS
}

}  // namespace kda
