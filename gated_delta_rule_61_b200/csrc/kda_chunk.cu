// kda_chunk.cu -- chunked KDA prefill on sm_100a tensor cores (tcgen05 MMAs,
// tensor-memory accumulators), chunk C = 64, dk = dv = 128, bf16 inputs.
//
// Method. Pages: "22580: from GPT-2 to Kimi K3, explained", section "DeltaNet,
// or Parallelizing Linear Transformers with Delta Rule" (cut the sequence into
// chunks of C tokens; inside a chunk the deltas come from a unit lower-
// triangular system built from the keys (the UT/WY form of the Householder
// products), across chunks the state carries everything; C is 64 or 128 to
// match tensor-core instruction granularity, UMMA being one example), with the
// per-channel decay of "Gated Delta Net" (cumulative decay is a multiplicative
// prefix sum) and "KDA / Kimi Linear"; the ai-flip.ru KDA explainer
// (channel-wise diagonal gate; chunked computation on tensor cores). Derived
// for the KDA step S_t = (I - b k k^T) Diag(a_t) S_{t-1} + b k v^T, with g the
// within-chunk cumulative sum of log_alpha per key channel and S0 the state
// entering the chunk:
//   M_kk[r,j] = sum_c k_rc k_jc e^{g_rc - g_jc} (j < r)
//   M_qk[r,j] = sum_c q_rc k_jc e^{g_rc - g_jc} (j <= r)
//   X = (I + diag(beta) M_kk)^-1,  T = X diag(beta)
//   W = T (K * e^g),  U = T V,  D = U - W S0
//   O = (Q * e^g) S0 + M_qk D
//   S1 = Diag(e^{g_last}) S0 + (K * e^{g_last - g})^T D
//
// Gram products. e^{g_r - g_j} is split as (x_r e^{g_r - m_a})(k_j e^{m_a - g_j})
// with m_a the midpoint of the cumulative gate over the row's 16-token
// sub-chunk a: for j in the same sub-chunk both factors are at most
// e^{(15/2) * 10} (log_alpha is clamped to >= -10 here), and for j in an
// earlier sub-chunk the right factor is at most 1. One 128 x 160 x 128 bf16
// MMA computes all of it: A = [k rows; q rows] scaled by e^{g - m_a}, B = [E;
// R1; R2; R3] with E_j = k_j e^{m_(sub(j)) - g_j} (diagonal blocks) and
// R_a rows = k_j e^{m_a - g_j} for j < 16 a (off-diagonal blocks of rows in
// sub-chunk a). Entries outside the blocks each row needs are ignored.
//
// Precision. Gram, T, W, U and the products with the state S0 use bf16
// operands with fp32 accumulation; the state update (K~^T D) and the
// output's correction (M_qk D) read D straight from tensor memory as tf32,
// and the state itself stays fp32 in tensor memory for the whole sequence.
//
// Layout. One CTA (512 threads = 16 warps) per (sequence, head) chain,
// walking its chunks in order; or, when chains are few, a cluster of R = 2 or
// 4 CTAs per chain that take chunks round-robin: each CTA prepares its own
// chunks (the state-independent work, most of the time) in parallel with the
// others, and the fp32 state moves to the next CTA through the chain's
// hand-over slot (L2) after each chunk's state update. Warp w reaches
// tensor-memory lanes [32 (w % 4), +32); the four warps sharing a lane
// quadrant split the columns.
// Tensor memory (512 columns, lanes = dv index m for the state-sized
// accumulators):
//   [0,128)   S^T (fp32 state, lane m, column c)
//   [128,192) U^T, then D^T = U^T - (W S0)^T   (lane m, column = position)
//   [192,256) O^T                              (lane m, column = position)
//   [256,416) Gram result (lanes 0..63 k rows, 64..127 q rows); later W^T
// Per chunk n: (P1) operand tiles from the chunk's gates and inputs; (P2)
// Gram MMA, during which the next own chunk's inputs are loaded into
// registers; (P3) rows of M_kk and M_qk; (P4) block inverse for X in warps
// 0-7 while warps 8-15 move the previous own chunk's output to HBM and enter
// the chunk's state (S0 to a bf16 tile, the fp32 state decayed in place;
// with a ring, from the previous CTA's hand-over once it has arrived); (P5)
// W^T and U^T MMAs; -W to shared memory; with a ring whose state arrived
// after P4, the state is received here; (P7) D and the first part of O, during which the next
// own chunk's gates (cumulative sums, sub-chunk ends, decay) are formed
// (with four CTAs per chain, where P7 is on the ring's critical path, at
// the start of that chunk's P1 instead); (P8) tf32 state update and output
// correction; with a ring, the state is handed to the next CTA.
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace chunk64 {

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 512;
constexpr float kLogAlphaMin = -10.0f;
constexpr uint64_t kMaxWaitNs = 1000000000ull;  // 1 s per bounded wait

// Shared memory (byte offsets from a 1024-aligned base).
constexpr uint32_t OFF_SB = 0;         // S0 bf16, K-major [m][c] (also O staging)  32768
constexpr uint32_t OFF_QT = 32768;     // Q*e^g bf16, K-major [r][c]                 16384
constexpr uint32_t OFF_KT = 49152;     // K*e^(glast-g) fp32, K-major [c][j]         32768
constexpr uint32_t OFF_BK = 81920;     // K*e^g bf16, MN-major [j][c]                16384
constexpr uint32_t OFF_VV = 98304;     // V bf16, MN-major [j][m]                    16384
constexpr uint32_t OFF_AG = 114688;    // Gram A bf16 K-major [128][c]               32768
constexpr uint32_t OFF_MQK = OFF_AG;           // after the Gram MMA: M_qk fp32 K-major [r][j]
constexpr uint32_t OFF_TM = OFF_AG + 16384;    // T bf16 K-major [r][j]
constexpr uint32_t OFF_BG = 147456;    // Gram B bf16 K-major [160][c]               40960
constexpr int kLd = 68;                        // row stride (floats) of the solve's matrices
constexpr uint32_t OFF_NMAT = OFF_BG;          // after the Gram MMA: diag(beta) M_kk [64][68]
constexpr uint32_t OFF_XMAT = OFF_BG + 17408;  // X, fp32 [64][68]
constexpr uint32_t OFF_ZBUF = OFF_BG + 34816;  // block products, fp32 [32][34]
constexpr uint32_t OFF_NW = OFF_BG;            // after the solve: -W^T bf16 MN-major [c][r]
constexpr uint32_t OFF_MISC = 188416;
constexpr uint32_t MISC_GAMMA = 0, MISC_BETA = 512, MISC_PAIR = 1280,
                   MISC_GF = 17664, MISC_GL = 19712, MISC_MBAR = 21760, MISC_FULL = 21776,
                   MISC_TMEM = 21784, MISC_TOT4 = 21792,
                   MISC_NORM = 23840,   // raw q/k: per-warp partial squared norms [16][16]
                   MISC_BARA = 24864,   // mbarrier of the k/v tensor-map copies
                   MISC_FLAG = 24872;   // P4: the ring's entering state was already handed over
constexpr uint32_t kSmemBytes = OFF_MISC + 24880 + 1024;
// The next own chunk's raw k and v land by tensor-map copies (128B-swizzled
// [row][channel] tiles, the operand tiles' layout): k in the K e^g tile (P1
// rewrites it in place) and v directly in its MMA operand tile.
// State hand-over between the CTAs of a chain's cluster goes through the
// chain's hand-over slot in global memory (64 KiB, L2-resident; a workspace
// region, or the chain's own final_state): it is
// written and read strictly in turn (CTA r writes S_n+1 after reading S_n;
// CTA r+1 reads it before writing S_n+2), so one arrive on the reader's
// mbarrier per hand-over is the only synchronisation needed. While it
// carries a hand-over the slot holds S^T in 16-byte chunks ordered
// (column group c / 4, row m), so each warp moves 512 contiguous bytes per
// access; the owner of the last chunk writes the final state in its own
// [dk][dv] layout.
__device__ __forceinline__ size_t xfer_chunk(int m, int c4) { return (size_t)c4 * 128 + m; }

// Tensor-memory columns.
constexpr uint32_t TM_S = 0, TM_D = 128, TM_O = 192, TM_G = 256, TM_W = 256;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// 1/x for normal positive x: the hardware approximate reciprocal (a single
// special-function instruction, error a few ulp), ample for operands that
// are rounded to bf16 or tf32 next.
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Read-once inputs: non-coherent loads that do not allocate in L1.
__device__ __forceinline__ float2 ld_stream_f2(const float* p) {
  float2 r;
  asm("ld.global.nc.L1::no_allocate.v2.f32 {%0, %1}, [%2];"
               : "=f"(r.x), "=f"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const __nv_bfloat16* p) {
  uint32_t r;
  asm("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// SiLU from the hardware tanh approximation (one special-function
// instruction): x * sigmoid(x) = x * (1/2 + tanh(x/2)/2). Its absolute error
// (about 2.5e-4 |x|) is far below the bf16 rounding the tensor-core operands
// receive next.
__device__ __forceinline__ float silu_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return x * fmaf(0.5f, t, 0.5f);
}

// log(sigmoid(x)) = min(x, 0) - log(1 + e^-|x|); absolute error a few 1e-8
// (the rounding of 1 + e^-|x|), far below the gate clamp's effect.
__device__ __forceinline__ float log_sigmoid_fast(float x) {
  return fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x)));
}

__device__ __forceinline__ float sigmoid_fast(float x) { return 1.f / (1.f + __expf(-x)); }

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// Warp-level 16x8x8 tf32 MMA (fp32 accumulate), used for the off-diagonal
// block products of the triangular inverse.
__device__ __forceinline__ void mma_16x8x8_tf32(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Thread 0 spins (bounded) on the MMA barrier phase; the outcome is shared
// through the CTA barrier.
__device__ __forceinline__ bool cta_wait(uint32_t mbar, uint32_t parity, int code) {
  int fail = 0;
  if (threadIdx.x == 0) fail = !tc::mbar_wait_bounded(mbar, parity, kMaxWaitNs) ? 1 : 0;
  fail = __syncthreads_or(fail);
  tc::fence_after_sync();
  if (fail && threadIdx.x == 0) report_timeout(code);
  return fail == 0;
}

// Same, for two barriers: the MMA barrier and, when need2, the input-copy
// barrier of the next own chunk (waited here so that chunk's P1 needs no
// barrier of its own). Returns 0, or 1 / 2 for the wait that gave up.
__device__ __forceinline__ int cta_wait2(uint32_t mbar, uint32_t parity, uint32_t mbar2,
                                         uint32_t parity2, bool need2, int code) {
  int fail = 0;
  if (threadIdx.x == 0) {
    fail = tc::mbar_wait_bounded(mbar, parity, kMaxWaitNs) ? 0 : 1;
    if (!fail && need2) fail = tc::mbar_wait_bounded(mbar2, parity2, kMaxWaitNs) ? 0 : 2;
  }
  const int any = __syncthreads_or(fail);
  tc::fence_after_sync();
  if (!any) return 0;
  // (failure path only: tell every thread which wait gave up)
  const int first = __syncthreads_or(fail == 1);
  if (threadIdx.x == 0) report_timeout(code);
  return first ? 1 : 2;
}

__device__ __forceinline__ void cta_sync_tc() {
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
}

// X = (I + N)^-1 for the strictly lower 64 x 64 matrix N (row stride kLd),
// as a recursive 2 x 2 block inverse: for a unit lower block matrix
// [[A, 0], [C, D]] the inverse is [[A^-1, 0], [-D^-1 C A^-1, D^-1]].
// Level 1 inverts the four 16 x 16 diagonal blocks by forward substitution
// (their entries above the diagonal come out as exact zeros), level 2 fills
// the two 16 x 16 blocks below them, level 3 the 32 x 32 block. Entries above
// the diagonal outside the diagonal blocks are never read.
__device__ __forceinline__ void invert_diag_block(const float* N, float* X, uint8_t* tm,
                                                  const float* s_beta, int t) {
  const int base = (t >> 4) * 16, col = t & 15;
  // Column col of the block's inverse by right-looking substitution: once
  // x[j] is final, every later row subtracts its term N[r][j] x[j], so the
  // dependent chain is one FMA per row while the other updates (and all the
  // loads of N) proceed in parallel.
  float x[16];
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) x[rr] = rr == col ? 1.f : 0.f;
  const float* nb = N + base * kLd + base;
#pragma unroll
  for (int j = 0; j < 15; ++j) {
#pragma unroll
    for (int rr = j + 1; rr < 16; ++rr) x[rr] = fmaf(-nb[rr * kLd + j], x[j], x[rr]);
  }
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) X[(base + rr) * kLd + base + col] = x[rr];
  // T = X diag(beta) in bf16 (entries above the diagonal are exact zeros)
  const float bc = s_beta[base + col];
#pragma unroll
  for (int rr = 0; rr < 16; ++rr)
    *reinterpret_cast<__nv_bfloat16*>(tm + tc::sw128<2>(base + rr, base + col, 64)) =
        __float2bfloat16_rn(x[rr] * bc);
}

// bf16 pair (r, j), (r, j + 1) of T, scaled by beta_j, beta_(j+1), into the
// swizzled K-major T tile [r][j] (j even).
__device__ __forceinline__ void store_t2(uint8_t* tm, const float* s_beta, int r, int j,
                                         float x0, float x1) {
  *reinterpret_cast<uint32_t*>(tm + tc::sw128<2>(r, j, 64)) =
      pack_bf16x2(x0 * s_beta[j], x1 * s_beta[j + 1]);
}

// X = (I + N)^-1 as below, writing T = X diag(beta) (bf16, K-major [r][j],
// the W/U MMA's operand) as each block of X is found: diagonal blocks in
// level 1, the level-2 blocks, the level-3 block (which is not kept in fp32),
// and zeros above the block diagonal (warps 2..7 while levels 1 and 2 run).
// Ends without a CTA barrier: the caller's barrier publishes T.
__device__ __forceinline__ void invert_unit_lower64(const float* N, float* X, float* Z,
                                                    uint8_t* tm, const float* s_beta, int t) {
  // Levels 1 and 2 in warps 0 and 1: warp p inverts the diagonal blocks 2p
  // and 2p + 1, then fills block (2p + 1, 2p) below them with two 16 x 16 x 16
  // tf32 m16n8k8 products (tf32 rounding there is below the bf16 rounding T
  // receives next), so nothing outside the warp is waited for until level 3.
  if (t >= 64 && t < 256) {
    // zeros of T above the block diagonal: rows 0-15 x cols 16-63, rows
    // 16-31 x cols 32-63, rows 32-47 x cols 48-63, in 16-byte chunks
    const int idx = t - 64;
    int r, c;
    if (idx < 96) {
      r = idx / 6;
      c = 16 + (idx % 6) * 8;
    } else if (idx < 160) {
      r = 16 + (idx - 96) / 4;
      c = 32 + ((idx - 96) % 4) * 8;
    } else {
      r = 32 + (idx - 160) / 2;
      c = 48 + ((idx - 160) % 2) * 8;
    }
    *reinterpret_cast<uint4*>(tm + tc::sw128<2>(r, c, 64)) = make_uint4(0u, 0u, 0u, 0u);
  }
  if (t < 64) {
    invert_diag_block(N, X, tm, s_beta, t);
    __syncwarp();
    const int p = t >> 5, lane = t & 31, gid = lane >> 2, tig = lane & 3;
    const int a = 32 * p, b = a + 16;
    float* Zp = Z + p * 16 * 34;
    // Z_p = N_{b a} X_{a a}  (X_{a a} lower triangular; its upper entries are zeros)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        if (kt < nt) continue;   // rows k < 8 nt of X_{a a} vanish in these columns
        const int k0 = 8 * kt + tig, c = 8 * nt + gid;
        const uint32_t av[4] = {to_tf32(N[(b + gid) * kLd + a + k0]),
                                to_tf32(N[(b + gid + 8) * kLd + a + k0]),
                                to_tf32(N[(b + gid) * kLd + a + k0 + 4]),
                                to_tf32(N[(b + gid + 8) * kLd + a + k0 + 4])};
        const uint32_t bv[2] = {to_tf32(X[(a + k0) * kLd + a + c]),
                                to_tf32(X[(a + k0 + 4) * kLd + a + c])};
        mma_16x8x8_tf32(d, av, bv);
      }
      const int zc = 8 * nt + 2 * tig;
      *reinterpret_cast<float2*>(Zp + gid * 34 + zc) = make_float2(d[0], d[1]);
      *reinterpret_cast<float2*>(Zp + (gid + 8) * 34 + zc) = make_float2(d[2], d[3]);
    }
    __syncwarp();
    // X_{b a} = -X_{b b} Z_p
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        const int k0 = 8 * kt + tig, c = 8 * nt + gid;
        const uint32_t av[4] = {to_tf32(X[(b + gid) * kLd + b + k0]),
                                to_tf32(X[(b + gid + 8) * kLd + b + k0]),
                                to_tf32(X[(b + gid) * kLd + b + k0 + 4]),
                                to_tf32(X[(b + gid + 8) * kLd + b + k0 + 4])};
        const uint32_t bv[2] = {to_tf32(Zp[k0 * 34 + c]), to_tf32(Zp[(k0 + 4) * 34 + c])};
        mma_16x8x8_tf32(d, av, bv);
      }
      const int xc = a + 8 * nt + 2 * tig;
      *reinterpret_cast<float2*>(X + (b + gid) * kLd + xc) = make_float2(-d[0], -d[1]);
      *reinterpret_cast<float2*>(X + (b + gid + 8) * kLd + xc) = make_float2(-d[2], -d[3]);
      store_t2(tm, s_beta, b + gid, xc, -d[0], -d[1]);
      store_t2(tm, s_beta, b + gid + 8, xc, -d[2], -d[3]);
    }
  }
  __syncthreads();
  // Level 3: Z = N[32:64, 0:32] X[0:32, 0:32];  X[32:64, 0:32] = -X[32:64, 32:64] Z,
  // as tf32 m16n8k8 MMAs: warps 0..7 each own one 16 x 8 tile of the 32 x 32 result.
  const int warp = t >> 5, lane = t & 31, gid = lane >> 2, tig = lane & 3;
  const int mt = (warp >> 2) & 1, nt = warp & 3;
  if (warp < 8) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      if (kt < nt) continue;  // X[0:32,0:32] is lower triangular: these columns are zero
      const int r0 = 32 + 16 * mt + gid, k0 = 8 * kt + tig;
      const uint32_t a[4] = {to_tf32(N[r0 * kLd + k0]), to_tf32(N[(r0 + 8) * kLd + k0]),
                             to_tf32(N[r0 * kLd + k0 + 4]), to_tf32(N[(r0 + 8) * kLd + k0 + 4])};
      const int c = 8 * nt + gid;
      const float x0 = X[k0 * kLd + c], x1 = X[(k0 + 4) * kLd + c];
      const uint32_t b[2] = {to_tf32(k0 >= c ? x0 : 0.f), to_tf32(k0 + 4 >= c ? x1 : 0.f)};
      mma_16x8x8_tf32(d, a, b);
    }
    const int zr = 16 * mt + gid, zc = 8 * nt + 2 * tig;
    *reinterpret_cast<float2*>(Z + zr * 34 + zc) = make_float2(d[0], d[1]);
    *reinterpret_cast<float2*>(Z + (zr + 8) * 34 + zc) = make_float2(d[2], d[3]);
    // The upper result tile (mt = 0) needs only this warp's own Z tile; the
    // lower one (mt = 1) also needs its partner's (warp nt), which announces
    // it on named barrier 4 + nt without waiting.
    if (mt == 0)
      asm volatile("bar.arrive %0, 64;" ::"r"(4 + nt) : "memory");
    else
      asm volatile("bar.sync %0, 64;" ::"r"(4 + nt) : "memory");
    __syncwarp();
  }
  if (warp < 8) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      if (kt > 2 * mt + 1) continue;  // X[32:64,32:64] is lower triangular
      const int r0 = 16 * mt + gid, k0 = 8 * kt + tig;   // rows/cols within the block
      const float y0 = X[(32 + r0) * kLd + 32 + k0], y1 = X[(40 + r0) * kLd + 32 + k0];
      const float y2 = X[(32 + r0) * kLd + 36 + k0], y3 = X[(40 + r0) * kLd + 36 + k0];
      const uint32_t a[4] = {to_tf32(k0 <= r0 ? y0 : 0.f), to_tf32(k0 <= r0 + 8 ? y1 : 0.f),
                             to_tf32(k0 + 4 <= r0 ? y2 : 0.f),
                             to_tf32(k0 + 4 <= r0 + 8 ? y3 : 0.f)};
      const int c = 8 * nt + gid;
      const uint32_t b[2] = {to_tf32(Z[k0 * 34 + c]), to_tf32(Z[(k0 + 4) * 34 + c])};
      mma_16x8x8_tf32(d, a, b);
    }
    const int xr = 32 + 16 * mt + gid, xc = 8 * nt + 2 * tig;
    store_t2(tm, s_beta, xr, xc, -d[0], -d[1]);
    store_t2(tm, s_beta, xr + 8, xc, -d[2], -d[3]);
  }
}

// O^T (lane m, column r) of one chunk -> bf16 [r][m] in shared memory ->
// coalesced 16-byte stores of the first L rows.
__device__ __forceinline__ void store_output(uint32_t tmem, uint32_t lane_off, int grp, int m,
                                             uint8_t* stage, __nv_bfloat16* o, long long t0,
                                             int L, int H, int head) {
  __nv_bfloat16* otile = reinterpret_cast<__nv_bfloat16*>(stage);
  float ov[16];
  tc::tmem_ld16(tmem + lane_off + TM_O + grp * 16, ov);
#pragma unroll
  for (int i = 0; i < 16; ++i) otile[(grp * 16 + i) * DV + m] = __float2bfloat16_rn(ov[i]);
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int idx = it * kThreads + threadIdx.x;
    const int r = idx >> 4, c8 = idx & 15;
    if (r < L)
      *reinterpret_cast<uint4*>(o + ((size_t)(t0 + r) * H + head) * DV + c8 * 8) =
          *reinterpret_cast<const uint4*>(otile + r * DV + c8 * 8);
  }
}

// Same as store_output, run by warps 8..15 only (two per lane quadrant, 32
// output rows each), synchronised with a named barrier among those 256 threads.
__device__ __forceinline__ void store_output_8w(uint32_t tmem, uint32_t lane_off, int half, int m,
                                                uint8_t* stage, __nv_bfloat16* o, long long t0,
                                                int L, int H, int head) {
  __nv_bfloat16* otile = reinterpret_cast<__nv_bfloat16*>(stage);
  float ov[32];
  tc::tmem_ld32(tmem + lane_off + TM_O + half * 32, ov);
#pragma unroll
  for (int i = 0; i < 32; ++i) otile[(half * 32 + i) * DV + m] = __float2bfloat16_rn(ov[i]);
  asm volatile("bar.sync 1, 256;" ::: "memory");
  const int t = threadIdx.x - 256;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int idx = it * 256 + t;
    const int r = idx >> 4, c8 = idx & 15;
    if (r < L)
      *reinterpret_cast<uint4*>(o + ((size_t)(t0 + r) * H + head) * DV + c8 * 8) =
          *reinterpret_cast<const uint4*>(otile + r * DV + c8 * 8);
  }
}

// 32 columns [cb, cb + 32) of row m of the entering state S0 (fp32, in s):
// bf16 into the S0 tile (swizzled K-major [m][c]), decayed by gamma into
// tensor memory at taddr.
__device__ __forceinline__ void state_tile_and_decay(uint32_t taddr, int m, int cb, uint8_t* smem,
                                                     const float* s_gamma, float* s) {
#pragma unroll
  for (int h8 = 0; h8 < 4; ++h8) {
    uint32_t p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = pack_bf16x2(s[h8 * 8 + 2 * e], s[h8 * 8 + 2 * e + 1]);
    *reinterpret_cast<uint4*>(smem + OFF_SB + tc::sw128<2>(m, cb + h8 * 8, 128)) =
        make_uint4(p[0], p[1], p[2], p[3]);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) s[i] *= s_gamma[cb + i];
  tc::tmem_st16(taddr, s);
  tc::tmem_st16(taddr + 16, s + 16);
}

// The entering state of a chunk, by warps 8-15 (two per lane quadrant, 64
// columns [64 half, +64) each): from tensor memory, or (slot != nullptr)
// from the chain's hand-over slot.
__device__ __forceinline__ void enter_state(uint32_t tmem, uint32_t lane_off, int m, int half,
                                            uint8_t* smem, const float* s_gamma,
                                            const float* slot) {
#pragma unroll 1
  for (int hh = 0; hh < 2; ++hh) {
    const int cb = half * 64 + hh * 32;
    const uint32_t tb = tmem + lane_off + TM_S + cb;
    float s[32];
    if (slot) {
      const float4* sl = reinterpret_cast<const float4*>(slot);
#pragma unroll
      for (int v4 = 0; v4 < 8; ++v4) {
        const float4 x = __ldcg(sl + xfer_chunk(m, cb / 4 + v4));
        s[4 * v4] = x.x; s[4 * v4 + 1] = x.y; s[4 * v4 + 2] = x.z; s[4 * v4 + 3] = x.w;
      }
    } else {
      tc::tmem_ld32(tb, s);
    }
    state_tile_and_decay(tb, m, cb, smem, s_gamma, s);
  }
  tc::tmem_wait_st();
}

// kGate: 0 = one decay per key channel (log_alpha [.., H, dk]), 1 = one per
// token (log_alpha [.., H], the same value on every channel), 2 = none.
// kRawQK: q and k are raw projections; each token's vectors become
// normalize(silu(x)) here (the row norms are reduced while the gates are
// formed). flags: bit 1 = beta holds logits (sigmoid applied), bit 2 = the
// gate holds logits x (log_alpha = log sigmoid(x)).
template <int kRing, int kGate, bool kRawQK>
__global__ void __launch_bounds__(kThreads, 1)
chunk64_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
               const __nv_bfloat16* __restrict__ v, const float* __restrict__ log_alpha,
               const float* __restrict__ beta, const float* init_state,
               const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ order,
               int T, int H, __nv_bfloat16* __restrict__ o, float* final_state, float* xfer,
               unsigned flags, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q,
               const __grid_constant__ CUtensorMap tm_la) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  float* s_gamma = reinterpret_cast<float*>(smem + OFF_MISC + MISC_GAMMA);
  float* s_beta = reinterpret_cast<float*>(smem + OFF_MISC + MISC_BETA);
  float* s_gf = reinterpret_cast<float*>(smem + OFF_MISC + MISC_GF);     // [4][128]
  float* s_gl = reinterpret_cast<float*>(smem + OFF_MISC + MISC_GL);     // [4][128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC + MISC_TMEM);
  const uint32_t mbar = sbase + OFF_MISC + MISC_MBAR;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr bool kPair = kRing > 1;
  const int rank = kPair ? (int)tc::cluster_ctarank() : 0;
  const int step = kRing;
  const int chain = (int)blockIdx.x / kRing;
  const int seq = order ? order[chain / H] : chain / H;
  const int head = chain % H;
  long long t_begin, t_end;
  seq_bounds(cu_seqlens, seq, T, &t_begin, &t_end);

  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  const uint32_t mbar_full = sbase + OFF_MISC + MISC_FULL;     // partner's state is in L2
  const uint32_t bar_a = sbase + OFF_MISC + MISC_BARA;   // k and v landed
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    tc::mbar_init(bar_a, 1);
    if (kPair) tc::mbar_init(mbar_full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  cta_sync_tc();
  if (kPair) tc::cluster_sync();   // partner's barriers exist before any remote arrive
  const uint32_t tmem = *tmem_slot;
  uint32_t phase = 0, full_phase = 0, phase_a = 0;
  // Thread 0 issues the MMAs and the input copies; on a failed wait it lets
  // whatever it issued finish (bounded) before memory is released.
  bool pend_mma = false, pend_a = false;
  bool ok = true;

  const int quad = warp & 3, grp = warp >> 2;
  const int m = quad * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
  const size_t state_off = ((size_t)seq * H + head) * DK * DV;
  const size_t xfer_off = state_off;   // this chain's hand-over slot (rings)

  // Initial state: S^T[m][c] = S0[c][m]; this warp covers columns [32 grp, +32).
  // (In a ring, the other CTAs receive their first state from the previous one.)
  if (rank == 0) {
    float vals[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int c = grp * 32 + i;
      vals[i] = init_state ? init_state[state_off + (size_t)c * DV + m] : 0.f;
    }
    tc::tmem_st16(tmem + lane_off + TM_S + grp * 32, vals);
    tc::tmem_st16(tmem + lane_off + TM_S + grp * 32 + 16, vals + 16);
    tc::tmem_wait_st();
  }
  cta_sync_tc();

  const long long len = t_end - t_begin;
  const int n_chunks = (int)((len + C - 1) / C);
  // P1 mapping: channel pair (c0, c0 + 1); row slot i = 2 a + e holds row
  // 16 a + 2 rg + e, so every thread owns two rows of each 16-row sub-chunk
  // (the per-sub-chunk work of the off-diagonal Gram factors is balanced).
  const int pr = tid & 63, rg = tid >> 6, c0 = 2 * pr;
  float* s_pair = reinterpret_cast<float*>(smem + OFF_MISC + MISC_PAIR);   // [32][128]
  float* s_tot4 = reinterpret_cast<float*>(smem + OFF_MISC + MISC_TOT4);   // [4][128]
  // Inputs of a chunk. k and v arrive by tensor-map copies (one thread,
  // bar_a) into their operand tiles; they are issued once the W/U MMA has
  // read those tiles, a whole D/O + update phase before the next own chunk
  // needs them. log_alpha, q and beta are consumed earlier (the gate scan
  // runs during the D/O MMA) and have no free landing place that early, so
  // they are read into registers one own chunk ahead, during the Gram MMA.
  float2 lr[8];
  uint32_t qr[8];
  float bt[2];   // warp 0 only: beta of rows 2 lane, 2 lane + 1
  float gt[2];   // warp 0 only, one decay per token: log_alpha of the same rows
  auto chunk_len = [&](int nn) {
    const long long tc0 = t_begin + (long long)nn * C;
    return (int)((t_end - tc0) < C ? (t_end - tc0) : C);
  };
  auto issue_kv = [&](int nn) {
    const int z = (int)(t_begin + (long long)nn * C);
    if (tid == 0) {
      tc::mbar_arrive_expect_tx(bar_a, 2 * 16384u);
      pend_a = true;
      tc::tma_load_3d(sbase + OFF_BK, &tm_k, 0, head, z, bar_a);
      tc::tma_load_3d(sbase + OFF_BK + 8192, &tm_k, 64, head, z, bar_a);
      tc::tma_load_3d(sbase + OFF_VV, &tm_v, 0, head, z, bar_a);
      tc::tma_load_3d(sbase + OFF_VV + 8192, &tm_v, 64, head, z, bar_a);
    }
  };
  auto load_rows = [&](int nn) {
    const long long tc0 = t_begin + (long long)nn * C;
    const int Lc = chunk_len(nn);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 16 * (i >> 1) + 2 * rg + (i & 1);
      lr[i] = make_float2(0.f, 0.f);
      qr[i] = 0u;
      if (r < Lc) {
        const size_t tok = (size_t)(tc0 + r) * H + head;
        if constexpr (kGate == 0) lr[i] = ld_stream_f2(log_alpha + tok * DK + c0);
        qr[i] = ld_stream_u32(q + tok * DK + c0);
      }
    }
    bt[0] = bt[1] = 0.f;
    gt[0] = gt[1] = 0.f;
    if (warp == 0) {
      if (2 * lane < Lc) bt[0] = __ldg(beta + (size_t)(tc0 + 2 * lane) * H + head);
      if (2 * lane + 1 < Lc) bt[1] = __ldg(beta + (size_t)(tc0 + 2 * lane + 1) * H + head);
      if constexpr (kGate == 1) {
        if (2 * lane < Lc) gt[0] = __ldg(log_alpha + (size_t)(tc0 + 2 * lane) * H + head);
        if (2 * lane + 1 < Lc) gt[1] = __ldg(log_alpha + (size_t)(tc0 + 2 * lane + 1) * H + head);
      }
    }
  };
  if (rank < n_chunks) {
    issue_kv(rank);
    load_rows(rank);
  }
  // Cumulative gates of a chunk from its log_alpha rows (lr), one decay per
  // key channel: pair sums per (sub-chunk, rg) -> one exclusive scan over the
  // 32 pairs per channel -> each thread adds its own rows. Writes g0/g1
  // (registers), beta, the first and last g of every sub-chunk and the
  // chunk's decay e^{g_last} to shared memory. The other gate forms take the
  // two shorter branches at the top. Runs for the next chunk while the
  // current chunk's D/O MMA is in flight; it touches no operand tile.
  float g0[8], g1[8];
  auto gates = [&](int Lc) -> bool {
    if constexpr (kGate == 2) {
      // No decay: only beta is published (and a unit chunk decay).
      if (warp == 0) {
        float b0 = bt[0], b1 = bt[1];
        if (flags & 2u) {
          b0 = 2 * lane < Lc ? sigmoid_fast(b0) : 0.f;
          b1 = 2 * lane + 1 < Lc ? sigmoid_fast(b1) : 0.f;
        }
        *reinterpret_cast<float2*>(s_beta + 2 * lane) = make_float2(b0, b1);
      }
      if (tid < 128) s_gamma[tid] = 1.f;
      __syncthreads();
      return true;
    }
    if constexpr (kGate == 1) {
      // One decay per token: warp 0 scans the chunk's 64 values (lane l holds
      // rows 2 l and 2 l + 1, i.e. sub-chunk l / 8, pair l % 8) into the
      // cumulative gate per row, summing in the per-channel scan's order (pair
      // sums, exclusive sum over the sub-chunk's pairs, then the sub-chunk
      // totals), so both forms give the same bits for the same decays.
      if (warp == 0) {
        float b0 = bt[0], b1 = bt[1];
        if (flags & 2u) {
          b0 = 2 * lane < Lc ? sigmoid_fast(b0) : 0.f;
          b1 = 2 * lane + 1 < Lc ? sigmoid_fast(b1) : 0.f;
        }
        *reinterpret_cast<float2*>(s_beta + 2 * lane) = make_float2(b0, b1);
        float x0 = gt[0], x1 = gt[1];
        if (flags & 4u) {
          if (2 * lane < Lc) x0 = log_sigmoid_fast(x0);
          if (2 * lane + 1 < Lc) x1 = log_sigmoid_fast(x1);
        }
        x0 = fmaxf(x0, kLogAlphaMin);
        x1 = fmaxf(x1, kLogAlphaMin);
        const float pr = x0 + x1;
        const int grp0 = lane & ~7, pos = lane & 7;
        float run = 0.f, excl = 0.f;
#pragma unroll
        for (int r8 = 0; r8 < 8; ++r8) {
          const float x = __shfl_sync(0xffffffffu, pr, grp0 + r8);
          if (r8 == pos) excl = run;
          run += x;
        }
        const float t0 = __shfl_sync(0xffffffffu, run, 0);
        const float t1 = __shfl_sync(0xffffffffu, run, 8);
        const float t2 = __shfl_sync(0xffffffffu, run, 16);
        const float tb1 = t0, tb2 = tb1 + t1, tb3 = tb2 + t2;
        const int a = lane >> 3;
        const float tb = a == 0 ? 0.f : a == 1 ? tb1 : a == 2 ? tb2 : tb3;
        const float ge = (tb + excl) + x0;
        const float go = ge + x1;
        *reinterpret_cast<float2*>(s_gf + 2 * lane) = make_float2(ge, go);   // per row
        if (lane == 31) {
          const float gam = __expf(go);   // decay over the whole chunk
#pragma unroll
          for (int c = 0; c < 128; c += 4)
            *reinterpret_cast<float4*>(s_gamma + c) = make_float4(gam, gam, gam, gam);
        }
      }
      __syncthreads();
      return true;
    }
    {
      float l0[8], l1[8];
      const bool raw_gate = flags & 4u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 16 * (i >> 1) + 2 * rg + (i & 1);
        float x0 = lr[i].x, x1 = lr[i].y;   // zero past the chunk's end: no decay
        if (raw_gate && r < Lc) {
          x0 = log_sigmoid_fast(x0);
          x1 = log_sigmoid_fast(x1);
        }
        l0[i] = fmaxf(x0, kLogAlphaMin);
        l1[i] = fmaxf(x1, kLogAlphaMin);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        s_pair[(a * 8 + rg) * 128 + c0] = l0[2 * a] + l0[2 * a + 1];
        s_pair[(a * 8 + rg) * 128 + c0 + 1] = l1[2 * a] + l1[2 * a + 1];
      }
      if (warp == 0) {
        float b0 = bt[0], b1 = bt[1];
        if (flags & 2u) {   // logits; rows past the chunk's end keep beta = 0
          b0 = 2 * lane < Lc ? sigmoid_fast(b0) : 0.f;
          b1 = 2 * lane + 1 < Lc ? sigmoid_fast(b1) : 0.f;
        }
        *reinterpret_cast<float2*>(s_beta + 2 * lane) = make_float2(b0, b1);
      }
      __syncthreads();
      {
        // Exclusive scan over rg within each sub-chunk (thread = (a, channel)),
        // sub-chunk totals to s_tot4.
        const int a = tid >> 7, c = tid & 127;
        float run = 0.f;
#pragma unroll
        for (int r8 = 0; r8 < 8; ++r8) {
          const float x = s_pair[(a * 8 + r8) * 128 + c];
          s_pair[(a * 8 + r8) * 128 + c] = run;
          run += x;
        }
        s_tot4[a * 128 + c] = run;
      }
      __syncthreads();
      float tb0[4], tb1[4];   // totals of the sub-chunks before a
      tb0[0] = tb1[0] = 0.f;
#pragma unroll
      for (int a = 1; a < 4; ++a) {
        tb0[a] = tb0[a - 1] + s_tot4[(a - 1) * 128 + c0];
        tb1[a] = tb1[a - 1] + s_tot4[(a - 1) * 128 + c0 + 1];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float b0 = tb0[a] + s_pair[(a * 8 + rg) * 128 + c0];
        const float b1 = tb1[a] + s_pair[(a * 8 + rg) * 128 + c0 + 1];
        g0[2 * a] = b0 + l0[2 * a];
        g0[2 * a + 1] = g0[2 * a] + l0[2 * a + 1];
        g1[2 * a] = b1 + l1[2 * a];
        g1[2 * a + 1] = g1[2 * a] + l1[2 * a + 1];
      }
      if (rg == 0) {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          s_gf[a * 128 + c0] = g0[2 * a];
          s_gf[a * 128 + c0 + 1] = g1[2 * a];
        }
      }
      if (rg == 7) {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          s_gl[a * 128 + c0] = g0[2 * a + 1];
          s_gl[a * 128 + c0 + 1] = g1[2 * a + 1];
        }
        s_gamma[c0] = __expf(g0[7]);       // decay over the whole chunk
        s_gamma[c0 + 1] = __expf(g1[7]);
      }
    }
    __syncthreads();
    return true;
  };
  if (rank < n_chunks) ok = gates(chunk_len(rank));

  for (int n = rank; ok && n < n_chunks; n += step) {
    const long long t0 = t_begin + (long long)n * C;
    const int L = chunk_len(n);
    // This thread's two channels of row slot i of a landed bf16 tile (raw k
    // or q), zero past the chunk's end.
    const uint32_t sw_rbase = (uint32_t)((rg >> 2) * 1024 + (rg & 3) * 256 + (c0 & 7) * 2);
    auto raw_pair = [&](uint32_t tile, int i) -> uint32_t {
      const int a = i >> 1, e = i & 1;
      const int r = 16 * a + 2 * rg + e;
      const uint32_t off = (uint32_t)(c0 >> 6) * 8192u + sw_rbase + (uint32_t)(a * 2048 + e * 128) +
                           ((uint32_t)(((c0 & 63) >> 3) ^ (2 * (rg & 3) + e)) << 4);
      return r < L ? *reinterpret_cast<const uint32_t*>(smem + tile + off) : 0u;
    };

    // ---- P1: operand tiles. The gates were formed during the previous own
    // chunk's D/O MMA, except with four CTAs per chain, where that MMA is on
    // the chain's critical path and the gates are formed here. -----------
    if (kRing > 2 && n != rank) {
      ok = gates(L);
      if (!ok) break;
    }
    if (n == rank) {   // later chunks waited for their k and v at the previous P8
      ok = cta_wait(bar_a, phase_a, 7);
      if (!ok) break;
      phase_a ^= 1;
      pend_a = false;
    }
    if constexpr (kRawQK) {
      // Squared norms of SiLU(k) and SiLU(q) per row: this thread's two
      // channels, reduced over the warp's 32 lanes by halving exchanges
      // (16 values in 16 shuffles: at each level a lane keeps the half of
      // its values selected by its lane bit and adds the partner's copy of
      // that half), so lane l ends with the warp sum of value (l >> 1) & 15;
      // the two warps of a row group are added when the tiles are built.
      float nv[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t kr = raw_pair(OFF_BK, i);
        const float k0 = silu_tanh(__uint_as_float(kr << 16));
        const float k1 = silu_tanh(__uint_as_float(kr & 0xffff0000u));
        const float q0 = silu_tanh(__uint_as_float(qr[i] << 16));
        const float q1 = silu_tanh(__uint_as_float(qr[i] & 0xffff0000u));
        nv[i] = fmaf(k0, k0, k1 * k1);
        nv[8 + i] = fmaf(q0, q0, q1 * q1);
      }
#pragma unroll
      for (int off = 16; off >= 2; off >>= 1) {
        const bool up = lane & off;
#pragma unroll
        for (int j = 0; j < off / 2; ++j) {
          const float keep = up ? nv[j + off / 2] : nv[j];
          const float send = up ? nv[j] : nv[j + off / 2];
          nv[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      nv[0] += __shfl_xor_sync(0xffffffffu, nv[0], 1);
      const int idx = (lane >> 1) & 15;
      float* s_norm = reinterpret_cast<float*>(smem + OFF_MISC + MISC_NORM);
      if ((lane & 1) == 0) s_norm[warp * 16 + idx] = nv[0];
      __syncthreads();
    }
    {
      // Sub-chunk midpoints m_a and the per-channel factors, from five
      // exponentials per channel: e^{m_0}, e^{m_a - m_(a-1)} and e^{g_last - m_3};
      // every other factor is a product of these (all at most 1).
      // Without decay every factor is 1 and no exponential is taken.
      constexpr bool kDecay = kGate != 2;
      auto ex = [](float x) { return kDecay ? __expf(x) : 1.f; };
      float mid0[4], mid1[4];
      float gl0, gl1;
      if constexpr (kGate == 1) {   // the per-row scan, the same on every channel
#pragma unroll
        for (int a = 0; a < 4; ++a) mid0[a] = mid1[a] = 0.5f * (s_gf[16 * a] + s_gf[16 * a + 15]);
        gl0 = gl1 = s_gf[63];
      } else {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          mid0[a] = kDecay ? 0.5f * (s_gf[a * 128 + c0] + s_gl[a * 128 + c0]) : 0.f;
          mid1[a] = kDecay ? 0.5f * (s_gf[a * 128 + c0 + 1] + s_gl[a * 128 + c0 + 1]) : 0.f;
        }
        gl0 = kDecay ? s_gl[3 * 128 + c0] : 0.f;
        gl1 = kDecay ? s_gl[3 * 128 + c0 + 1] : 0.f;
      }
      float dd0[4], dd1[4];   // dd[a] = e^{m_a - m_(a-1)}, a >= 1
      dd0[0] = dd1[0] = 1.f;
#pragma unroll
      for (int a = 1; a < 4; ++a) {
        dd0[a] = ex(mid0[a] - mid0[a - 1]);
        dd1[a] = ex(mid1[a] - mid1[a - 1]);
      }
      float em0[4], em1[4], kt0[4], kt1[4];
      em0[0] = ex(mid0[0]);
      em1[0] = ex(mid1[0]);
      kt0[3] = ex(gl0 - mid0[3]);
      kt1[3] = ex(gl1 - mid1[3]);
#pragma unroll
      for (int a = 1; a < 4; ++a) {
        em0[a] = em0[a - 1] * dd0[a];
        em1[a] = em1[a - 1] * dd1[a];
      }
#pragma unroll
      for (int a = 2; a >= 0; --a) {
        kt0[a] = kt0[a + 1] * dd0[a + 1];
        kt1[a] = kt1[a + 1] * dd1[a + 1];
      }
      // Swizzled row offsets: r = 16 a + 2 rg + e, so (r >> 3) = 2 a + (rg >> 2)
      // and (r & 7) = 2 (rg & 3) + e.
      const int xr = (c0 & 63) >> 3;
      const uint32_t rbase = (uint32_t)((rg >> 2) * 1024 + (rg & 3) * 256);
      const uint32_t xo0 = (uint32_t)(xr ^ (2 * (rg & 3))) << 4;
      const uint32_t xo1 = (uint32_t)(xr ^ (2 * (rg & 3) + 1)) << 4;
      const uint32_t colb = (uint32_t)((c0 & 7) * 2) + rbase;
      const uint32_t sl = (uint32_t)(c0 >> 6);
      uint8_t* const pAGk = smem + OFF_AG + sl * 16384u + colb;
      uint8_t* const pBGe = smem + OFF_BG + sl * 20480u + colb;
      uint8_t* const pQT = smem + OFF_QT + sl * 8192u + colb;
      uint8_t* const pBK = smem + OFF_BK + sl * 8192u + colb;
      // K~ as a K-major tf32 operand [c][j]: positions 16 a + 2 rg, +1 per
      // channel, stored as soon as both rows of a sub-chunk are done. Lanes
      // 4-7 of every 8 store their second channel first: the 8 lanes of a
      // store then write rows c = 0..7 (mod 8), i.e. all eight 16-byte
      // positions of the swizzle (no bank conflicts).
      const int odd = (lane >> 2) & 1;
      float kt_p0 = 0.f, kt_p1 = 0.f;   // the sub-chunk's first row, channels c0, c0 + 1
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int a = i >> 1, e = i & 1;
        const uint32_t ro = (uint32_t)(a * 2048 + e * 128) + (e ? xo1 : xo0);
        // bf16 pairs widen exactly: low half << 16, high half masked. Raw k
        // is read where K e^g is written (zero past the chunk's end).
        const uint32_t kr = 16 * a + 2 * rg + e < L ? *reinterpret_cast<const uint32_t*>(pBK + ro)
                                                    : 0u;
        float k0 = __uint_as_float(kr << 16), k1 = __uint_as_float(kr & 0xffff0000u);
        float q0 = __uint_as_float(qr[i] << 16), q1 = __uint_as_float(qr[i] & 0xffff0000u);
        if constexpr (kRawQK) {
          // normalize(silu(x)): divide by max(|silu(x)|, 1e-12) of the row,
          // whose squared norm is the sum of the row group's two warps.
          const float* s_norm = reinterpret_cast<const float*>(smem + OFF_MISC + MISC_NORM);
          const int w0 = 2 * rg;
          const float nk = s_norm[w0 * 16 + i] + s_norm[(w0 + 1) * 16 + i];
          const float nq = s_norm[w0 * 16 + 8 + i] + s_norm[(w0 + 1) * 16 + 8 + i];
          const float ik = rsqrtf(fmaxf(nk, 1e-24f)), iq = rsqrtf(fmaxf(nq, 1e-24f));
          k0 = silu_tanh(k0) * ik;
          k1 = silu_tanh(k1) * ik;
          q0 = silu_tanh(q0) * iq;
          q1 = silu_tanh(q1) * iq;
        }
        // this row's cumulative gate per channel (per row with one decay per token)
        const float gi0 = kGate == 1 ? s_gf[16 * a + 2 * rg + e] : g0[i];
        const float gi1 = kGate == 1 ? gi0 : g1[i];
        const float f0 = kDecay ? __expf(gi0 - mid0[a]) : 1.f;
        const float f1 = kDecay ? __expf(gi1 - mid1[a]) : 1.f;
        const float fi0 = kDecay ? rcp_approx(f0) : 1.f, fi1 = kDecay ? rcp_approx(f1) : 1.f;
        *reinterpret_cast<uint32_t*>(pAGk + ro) = pack_bf16x2(k0 * f0, k1 * f1);
        *reinterpret_cast<uint32_t*>(pAGk + ro + 8192) = pack_bf16x2(q0 * f0, q1 * f1);
        const float e0 = k0 * fi0, e1 = k1 * fi1;
        *reinterpret_cast<uint32_t*>(pBGe + ro) = pack_bf16x2(e0, e1);
        // R sets: row 64 + r (set 1), 80 + r (set 2), 112 + r (set 3): k_j
        // e^{m_a' - g_j} for the later sub-chunks a' > a. The nearest one is
        // one exponential (at most 1), the farther ones multiply it by dd
        // factors (each at most 1), so no intermediate underflows while the
        // product is still representable (starting from E_j, which can be
        // e^75, lost terms of size e^{g_r - g_j} under strong decay).
        if (a < 3) {
          // e^{m_(a+1) - g_j} = e^{m_(a+1) - m_a} e^{m_a - g_j}: a product of two
          // factors already at hand while the first (at most 1) is a normal
          // float; where it is tiny (decays averaging below about -4 per token)
          // the product could have lost it, and the exponential is taken.
          const int an = a < 3 ? a + 1 : 3;
          float n0 = k0, n1 = k1;
          if constexpr (kDecay) {
            if (dd0[an] > 1e-30f && dd1[an] > 1e-30f) {
              n0 = k0 * (fi0 * dd0[an]);
              n1 = k1 * (fi1 * dd1[an]);
            } else {
              n0 = k0 * __expf(mid0[an] - gi0);
              n1 = k1 * __expf(mid1[an] - gi1);
            }
          }
          const uint32_t set_off = a == 0 ? 8192u : a == 1 ? 10240u : 14336u;
          *reinterpret_cast<uint32_t*>(pBGe + ro + set_off) = pack_bf16x2(n0, n1);
          if (a < 2) {
            n0 *= dd0[a + 2 < 4 ? a + 2 : 3];
            n1 *= dd1[a + 2 < 4 ? a + 2 : 3];
            *reinterpret_cast<uint32_t*>(pBGe + ro + (a == 0 ? 10240u : 14336u)) =
                pack_bf16x2(n0, n1);
          }
          if (a < 1) {
            n0 *= dd0[3];
            n1 *= dd1[3];
            *reinterpret_cast<uint32_t*>(pBGe + ro + 14336u) = pack_bf16x2(n0, n1);
          }
        }
        const float eg0 = f0 * em0[a], eg1 = f1 * em1[a];
        *reinterpret_cast<uint32_t*>(pQT + ro) = pack_bf16x2(q0 * eg0, q1 * eg1);
        *reinterpret_cast<uint32_t*>(pBK + ro) = pack_bf16x2(k0 * eg0, k1 * eg1);
        const float kt_e0 = e0 * kt0[a], kt_e1 = e1 * kt1[a];
        if (e == 0) {
          kt_p0 = kt_e0;
          kt_p1 = kt_e1;
        } else {
          const int j = 16 * a + 2 * rg;
          const float2 v0 = make_float2(kt_p0, kt_e0);
          const float2 v1 = make_float2(kt_p1, kt_e1);
          *reinterpret_cast<float2*>(smem + OFF_KT + tc::sw128<4>(c0 + odd, j, 128)) =
              odd ? v1 : v0;
          *reinterpret_cast<float2*>(smem + OFF_KT + tc::sw128<4>(c0 + 1 - odd, j, 128)) =
              odd ? v0 : v1;
        }
      }
    }
    tc::fence_async_smem();
    cta_sync_tc();

    // ---- P2: Gram MMA (M=128, N=160, K=128) --------------------------------
    if (tid == 0) {
      constexpr uint32_t idesc = tc::make_idesc(1, 0, 0, 128, 160);
      // base descriptors once; the k-steps add constant byte offsets (>> 4)
      const uint64_t da0 = tc::make_desc(sbase + OFF_AG, 16, 1024);
      const uint64_t db0 = tc::make_desc(sbase + OFF_BG, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t da = da0 + (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        const uint64_t db = db0 + (uint64_t)(((ks >> 2) * 20480 + (ks & 3) * 32) >> 4);
        tc::mma_bf16_ss(tmem + TM_G, da, db, idesc, ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(mbar);
      pend_mma = true;
    }
    // While the Gram MMA runs: read the next own chunk's log_alpha, q and beta
    // into registers (this chunk's were consumed by the gate scan and the
    // tiles) and warm L2 with the inputs of the own chunk after it.
    if (n + step < n_chunks) load_rows(n + step);
    if (n + 2 * step < n_chunks) {
      // q, k, v and the per-channel gates by tensor-map prefetches (one
      // thread, a few box requests); beta and a per-token gate row by row.
      const long long t1 = t0 + (long long)(2 * step) * C;
      const int z1 = (int)t1;
      if (tid == 32) {
#pragma unroll
        for (int x = 0; x < 128; x += 64) {
          tc::prefetch_box_3d(&tm_q, x, head, z1);
          tc::prefetch_box_3d(&tm_k, x, head, z1);
          tc::prefetch_box_3d(&tm_v, x, head, z1);
        }
        if constexpr (kGate == 0) {
#pragma unroll
          for (int x = 0; x < 128; x += 32) tc::prefetch_box_3d(&tm_la, x, head, z1);
        }
      }
      const int row = tid - 64;
      if (row >= 0 && row < C && t1 + row < t_end) {
        const size_t tok = (size_t)(t1 + row) * H + head;
        tc::prefetch_l2(beta + tok);
        if (kGate == 1) tc::prefetch_l2(log_alpha + tok);
      }
    }
    ok = cta_wait(mbar, phase, 1);
    if (!ok) break;
    pend_mma = false;
    phase ^= 1;

    // ---- P3: rows of M_kk (lanes 0..63) and M_qk (lanes 64..127) ---------
    // Warp (quad, grp) assembles columns j in [16 grp, 16 grp + 16) for its 32
    // rows, which fall in two sub-chunks: a_lo (lanes 0-15) and a_lo + 1.
    // Column block jg of a row in sub-chunk a comes from the R_a set (jg < a),
    // from the diagonal set under the causal mask (jg == a), or is zero, so a
    // warp needs at most two 16-column loads, chosen warp-uniformly.
    {
      const int row = m;
      const bool is_q = row >= 64;
      const int r = row & 63;
      const int jg = grp, a_lo = 2 * (quad & 1), a_hi = a_lo + 1;
      const bool hi = lane >= 16;
      const uint32_t tb = tmem + lane_off + TM_G;
      auto r_col = [&](int a) { return (uint32_t)((a == 1 ? 64 : a == 2 ? 80 : 112) + 16 * jg); };
      float vv[32];
      if (jg < a_lo) {
        tc::tmem_ld16x2(tb + r_col(a_lo), tb + r_col(a_hi), vv);
      } else if (jg == a_lo) {
        tc::tmem_ld16x2(tb + 16 * jg, tb + r_col(a_hi), vv);
      } else if (jg == a_hi) {
        tc::tmem_ld16x2(tb + 16 * jg, tb + 16 * jg, vv);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) vv[i] = 0.f;
      }
      // vv[0..15]: block for the a_lo rows (or the diagonal set), vv[16..31]:
      // block for the a_hi rows. Diagonal entries keep j < r (k rows) or
      // j <= r (q rows).
      // Two equivalent selections; the one that fits each kernel variant's
      // register budget without spills.
      float out[16];
      if constexpr (kRing <= 2) {
        // Per lane: the source half (vv[16..31] only for a_hi rows off the
        // diagonal) and how many of the 16 columns survive: all of an R block,
        // the causal part of the diagonal block (j < r, or j <= r for q rows),
        // none above it.
        const int a_row = hi ? a_hi : a_lo;
        const bool hi_src = hi && jg < a_hi;
        const int keep = jg < a_row ? 16 : jg == a_row ? (is_q ? r + 1 : r) - 16 * jg : 0;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const float x = hi_src ? vv[16 + jj] : vv[jj];
          out[jj] = jj < keep ? x : 0.f;
        }
      } else {
        const int lim = is_q ? r + 1 : r;
        const bool lo_diag = jg == a_lo, hi_diag = jg == a_hi;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const bool causal = jg * 16 + jj < lim;
          const float lo = lo_diag ? (causal ? vv[jj] : 0.f) : (jg < a_lo ? vv[jj] : 0.f);
          const float hv = hi_diag ? (causal ? vv[jj] : 0.f) : (jg < a_hi ? vv[16 + jj] : 0.f);
          out[jj] = hi ? hv : lo;
        }
      }
      if (!is_q) {
        const float br = s_beta[r];
        float* nmat = reinterpret_cast<float*>(smem + OFF_NMAT);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<float4*>(nmat + r * kLd + jg * 16 + q4 * 4) =
              make_float4(br * out[q4 * 4], br * out[q4 * 4 + 1], br * out[q4 * 4 + 2],
                          br * out[q4 * 4 + 3]);
      } else {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<float4*>(smem + OFF_MQK + tc::sw128<4>(r, jg * 16 + q4 * 4, 64)) =
              make_float4(out[q4 * 4], out[q4 * 4 + 1], out[q4 * 4 + 2], out[q4 * 4 + 3]);
      }
    }
    tc::fence_async_smem();
    cta_sync_tc();

    // ---- P4: X = (I + N)^-1; T = X diag(beta) -> bf16 -------------------
    // Warps 0-7 run the solve. Meanwhile warps 8-15 move the previous own
    // chunk's output to HBM (staged in the gate-scan scratch, idle until the
    // next gate scan), then prepare this chunk's entering state: the S0 bf16
    // tile for the D/O MMA and the decayed fp32 state in tensor memory, from
    // tensor memory (one CTA per chain, or a ring's first chunk), or from the
    // chain's hand-over slot when the previous CTA of the ring has already
    // handed it over (otherwise every warp receives it after the W/U MMA).
    bool received = false;
    {
      const float* N = reinterpret_cast<const float*>(smem + OFF_NMAT);
      float* X = reinterpret_cast<float*>(smem + OFF_XMAT);
      int* s_flag = reinterpret_cast<int*>(smem + OFF_MISC + MISC_FLAG);
      if (warp >= 8) {
        const int half = (warp >> 2) & 1;
        if (n >= step)
          store_output_8w(tmem, lane_off, half, m, smem + OFF_MISC + MISC_PAIR, o,
                          t0 - (long long)step * C, C, H, head);
        bool from_slot = false;
        if (kPair && n > 0) {
          if (tid == 256) *s_flag = tc::mbar_test_wait_cluster(mbar_full, full_phase) ? 1 : 0;
          asm volatile("bar.sync 2, 256;" ::: "memory");
          from_slot = *s_flag != 0;
        }
        if (!(kPair && n > 0) || from_slot)
          enter_state(tmem, lane_off, m, half, smem, s_gamma,
                      from_slot ? xfer + xfer_off : nullptr);
      }
      invert_unit_lower64(N, X, reinterpret_cast<float*>(smem + OFF_ZBUF), smem + OFF_TM,
                          s_beta, tid);
      tc::fence_async_smem();
      cta_sync_tc();
      if (kPair && n > 0) received = *s_flag != 0;
      if (received) full_phase ^= 1;
    }

    // ---- P5: W^T = (K e^g)^T T^T and U^T = V^T T^T (M=128, N=64, K=64);
    // then -W^T to shared memory and, in a ring whose state was not yet
    // handed over in P4, the entering state from the hand-over slot --------
    if (tid == 0) {
      constexpr uint32_t idesc = tc::make_idesc(1, 1, 0, 128, 64);
      const uint64_t dw0 = tc::make_desc(sbase + OFF_BK, 8192, 1024);
      const uint64_t du0 = tc::make_desc(sbase + OFF_VV, 8192, 1024);
      const uint64_t dt0 = tc::make_desc(sbase + OFF_TM, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t dw = dw0 + (uint64_t)((ks * 2048) >> 4);
        const uint64_t du = du0 + (uint64_t)((ks * 2048) >> 4);
        const uint64_t dt = dt0 + (uint64_t)((ks * 32) >> 4);
        tc::mma_bf16_ss(tmem + TM_W, dw, dt, idesc, ks > 0 ? 1u : 0u);
        tc::mma_bf16_ss(tmem + TM_D, du, dt, idesc, ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(mbar);
      pend_mma = true;
    }
    const bool receive = kPair && n > 0 && !received;
    ok = cta_wait(mbar, phase, 2);
    if (!ok) break;
    pend_mma = false;
    phase ^= 1;
    // The W/U MMA has read K e^g and V: bring in the next own chunk's k and v.
    if (n + step < n_chunks) issue_kv(n + step);
    {
      // -W^T to shared memory: lane c holds W^T[c][r]; this warp takes r in [16 grp, +16).
      float w[16];
      tc::tmem_ld16(tmem + lane_off + TM_W + grp * 16, w);
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8) {
        uint32_t p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          p[e] = pack_bf16x2(-w[h8 * 8 + 2 * e], -w[h8 * 8 + 2 * e + 1]);
        *reinterpret_cast<uint4*>(smem + OFF_NW + tc::sw128<2>(m, grp * 16 + h8 * 8, 128)) =
            make_uint4(p[0], p[1], p[2], p[3]);
      }
    }
    if (receive) {
      // The partner wrote this chunk's entering state to the hand-over slot.
      int fail = tc::mbar_wait_cluster_bounded(mbar_full, full_phase, kMaxWaitNs) ? 0 : 1;
      full_phase ^= 1;
      fail = __syncthreads_or(fail);
      if (fail) {
        if (tid == 0) report_timeout(5);
        ok = false;
        break;
      }
      float s[32];
      const int cb = grp * 32;
      const float4* slot = reinterpret_cast<const float4*>(xfer + xfer_off);
#pragma unroll
      for (int v4 = 0; v4 < 8; ++v4) {
        const float4 x = __ldcg(slot + xfer_chunk(m, cb / 4 + v4));
        s[4 * v4] = x.x; s[4 * v4 + 1] = x.y; s[4 * v4 + 2] = x.z; s[4 * v4 + 3] = x.w;
      }
      state_tile_and_decay(tmem + lane_off + TM_S + grp * 32, m, grp * 32, smem, s_gamma, s);
      tc::tmem_wait_st();
    }
    tc::fence_async_smem();
    cta_sync_tc();

    // ---- P7: D^T += S0b^T (-W^T);  O^T = S0b^T (Q e^g)^T (K = 128) --------
    if (tid == 0) {
      constexpr uint32_t id_d = tc::make_idesc(1, 0, 1, 128, 64);
      constexpr uint32_t id_o = tc::make_idesc(1, 0, 0, 128, 64);
      const uint64_t da0 = tc::make_desc(sbase + OFF_SB, 16, 1024);
      const uint64_t dn0 = tc::make_desc(sbase + OFF_NW, 16384, 1024);
      const uint64_t dq0 = tc::make_desc(sbase + OFF_QT, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t da = da0 + (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        const uint64_t dn = dn0 + (uint64_t)((ks * 2048) >> 4);
        const uint64_t dq = dq0 + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4);
        tc::mma_bf16_ss(tmem + TM_D, da, dn, id_d, 1u);
        tc::mma_bf16_ss(tmem + TM_O, da, dq, id_o, ks > 0 ? 1u : 0u);
      }
      tc::mma_commit(mbar);
      pend_mma = true;
    }
    // ---- P8: S^T += D^T K~ (tf32, A from TMEM, B K-major); O^T += D^T M_qk^T
    auto issue_update = [&]() {
      constexpr uint32_t id_s = tc::make_idesc(2, 0, 0, 128, 128);
      constexpr uint32_t id_o = tc::make_idesc(2, 0, 0, 128, 64);
      const uint64_t dk0 = tc::make_desc(sbase + OFF_KT, 16, 1024);
      const uint64_t dm0 = tc::make_desc(sbase + OFF_MQK, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a_t = tmem + TM_D + ks * 8;
        const uint64_t dk_ = dk0 + (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        const uint64_t dm = dm0 + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4);
        tc::mma_tf32_ts(tmem + TM_S, a_t, dk_, id_s, 1u);
        tc::mma_tf32_ts(tmem + TM_O, a_t, dm, id_o, 1u);
      }
      tc::mma_commit(mbar);
    };
    if constexpr (kRing > 2) {
      // On the ring's critical path: only the issuing thread needs the D/O
      // results before the update's MMAs, so it waits for them alone and
      // issues the update at once; one CTA barrier afterwards shares the
      // outcome. (With one or two CTAs per chain the gate scan runs here and
      // its barriers wait for the issuing warp anyway.)
      int fail7 = 0;
      if (tid == 0) {
        if (tc::mbar_wait_bounded(mbar, phase, kMaxWaitNs)) {
          tc::fence_after_sync();
          issue_update();
        } else {
          fail7 = 1;
        }
      }
      fail7 = __syncthreads_or(fail7);
      if (fail7) {   // the D/O MMAs are still pending (phase unchanged)
        if (tid == 0) report_timeout(3);
        ok = false;
        break;
      }
      phase ^= 1;   // the D/O MMAs completed; the update's commit is the next phase
    } else {
      if (n + step < n_chunks)   // next own chunk, while the MMAs run
        gates(chunk_len(n + step));
      ok = cta_wait(mbar, phase, 3);
      if (!ok) break;
      phase ^= 1;
      if (tid == 0) issue_update();
    }
    {
      const bool next = n + step < n_chunks;   // its k and v were issued at P5
      const int f = cta_wait2(mbar, phase, bar_a, phase_a, next, 4);
      if (f != 1) {
        pend_mma = false;
        phase ^= 1;
      }
      if (f == 0 && next) {
        pend_a = false;
        phase_a ^= 1;
      }
      ok = f == 0;
      if (!ok) break;
    }

    if (kPair && n + 1 < n_chunks) {
      // Hand the state to the next CTA of the ring, which takes chunk n + 1.
      float s[32];
      tc::tmem_ld32(tmem + lane_off + TM_S + grp * 32, s);
      float4* slot = reinterpret_cast<float4*>(xfer + xfer_off);
#pragma unroll
      for (int v4 = 0; v4 < 8; ++v4)
        __stcg(slot + xfer_chunk(m, grp * 8 + v4),
               make_float4(s[4 * v4], s[4 * v4 + 1], s[4 * v4 + 2], s[4 * v4 + 3]));
      // Announce it: after a CTA barrier that orders every thread's stores
      // before it, thread 0 arrives on the next CTA's barrier with release
      // semantics at cluster scope (cumulative over the stores the barrier
      // ordered); the receiver's acquire wait pairs with it.
      __syncthreads();
      if (tid == 0)
        tc::mbar_remote_arrive(tc::mapa_shared(mbar_full, (uint32_t)((rank + 1) % kRing)));
    }
  }

  __syncthreads();
  if (ok && n_chunks > rank) {
    const int n_mine = rank + step * ((n_chunks - 1 - rank) / step);   // this CTA's last chunk
    const long long t_last = t_begin + (long long)n_mine * C;
    const int L_last = (int)((t_end - t_last) < C ? (t_end - t_last) : C);
    store_output(tmem, lane_off, grp, m, smem + OFF_MISC + MISC_PAIR, o, t_last, L_last, H,
                 head);
  }
  const bool owns_final = n_chunks > 0 ? ((n_chunks - 1) % step == rank) : rank == 0;
  if (ok && final_state && owns_final) {
    float s[32];
    tc::tmem_ld32(tmem + lane_off + TM_S + grp * 32, s);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int c = grp * 32 + i;
      final_state[state_off + (size_t)c * DV + m] = s[i];
    }
  }
  if (!ok && tid == 0) {
    // A wait gave up: give outstanding MMAs and input copies one more bounded
    // chance to land before the tensor and shared memory they write is
    // released.
    if (pend_mma) tc::mbar_wait_bounded(mbar, phase, kMaxWaitNs);
    if (pend_a) tc::mbar_wait_bounded(bar_a, phase_a, kMaxWaitNs);
  }
  cta_sync_tc();
  if (kPair) tc::cluster_sync();   // no remote traffic targets this CTA past this point
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// Longest-first order of the packed sequences (ties by index), so the long
// chains start first and the short ones fill in behind them.
__global__ void order_by_length_kernel(const int32_t* __restrict__ cu, int n_seq,
                                       int32_t* __restrict__ order) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_seq; i += gridDim.x * blockDim.x) {
    const int li = cu[i + 1] - cu[i];
    int rank = 0;
    for (int j = 0; j < n_seq; ++j) {
      const int lj = cu[j + 1] - cu[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
}

__global__ void identity_order_kernel(int n_seq, int32_t* __restrict__ order) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_seq; i += gridDim.x * blockDim.x)
    order[i] = i;
}

// Per-device launch state: the dynamic shared-memory attribute must be set on
// every device the kernels run on, and the ring choice needs that device's SM
// count. Set up once per device, under a lock (first calls from several host
// threads may race).
struct LaunchState {
  bool ready;
  int n_sm;
};
constexpr int kMaxDevices = 64;
static std::mutex g_launch_mutex;
static LaunchState g_launch[kMaxDevices];

template <int kGate, bool kRaw>
static cudaError_t set_smem_attrs() {
  cudaError_t e = cudaFuncSetAttribute(chunk64_kernel<1, kGate, kRaw>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(chunk64_kernel<2, kGate, kRaw>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(chunk64_kernel<4, kGate, kRaw>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
}

static cudaError_t launch_state_for_current_device(int* n_sm) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_launch_mutex);
  LaunchState& st = g_launch[dev];
  if (!st.ready) {
    if ((e = set_smem_attrs<0, false>()) != cudaSuccess) return e;
    if ((e = set_smem_attrs<1, false>()) != cudaSuccess) return e;
    if ((e = set_smem_attrs<2, false>()) != cudaSuccess) return e;
    if ((e = set_smem_attrs<0, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attrs<1, true>()) != cudaSuccess) return e;
    if ((e = set_smem_attrs<2, true>()) != cudaSuccess) return e;
    int count = 0;
    e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    st.n_sm = count;
    st.ready = true;
  }
  *n_sm = st.n_sm;
  return cudaSuccess;
}

struct ChunkArgs {
  const __nv_bfloat16 *q, *k, *v;
  const float *la, *beta, *s0;
  const int32_t *cu, *order;
  int T, H;
  __nv_bfloat16* o;
  float *sT, *xfer;
  unsigned flags;
  CUtensorMap tm_k, tm_v, tm_q, tm_la;   // tm_q, tm_la: L2 prefetch only
};

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point
// (the library does not link the driver library directly). Looked up once.
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static cudaError_t tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  *fn = g_encode;
  return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// A [tokens][H][128] tensor of bf16 (box 64 channels) or fp32 (box 32
// channels) as a 3-D tiled map: innermost the channels, then the head, then
// the token; one box = 64 tokens x 1 head x 128 bytes, 128B-swizzled (the
// operand tiles' layout); rows past the last token read as zeros.
static cudaError_t encode_rows(PFN_cuTensorMapEncodeTiled_v12000 fn, CUtensorMap* map,
                               const void* base, bool bf16, long long tokens, int H) {
  const cuuint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {128 * es, (cuuint64_t)H * 128 * es};
  cuuint32_t box[3] = {bf16 ? 64u : 32u, 1u, 64u};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int kGate, bool kRaw>
static cudaError_t launch_variant(const ChunkArgs& a, long long chains, int ring,
                                  cudaStream_t stream) {
  if (ring > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ring * chains));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ring;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (ring == 4)
      return cudaLaunchKernelEx(&cfg, chunk64_kernel<4, kGate, kRaw>, a.q, a.k, a.v, a.la,
                                a.beta, a.s0, a.cu, a.order, a.T, a.H, a.o, a.sT, a.xfer,
                                a.flags, a.tm_k, a.tm_v, a.tm_q, a.tm_la);
    return cudaLaunchKernelEx(&cfg, chunk64_kernel<2, kGate, kRaw>, a.q, a.k, a.v, a.la,
                              a.beta, a.s0, a.cu, a.order, a.T, a.H, a.o, a.sT, a.xfer,
                              a.flags, a.tm_k, a.tm_v, a.tm_q, a.tm_la);
  }
  chunk64_kernel<1, kGate, kRaw><<<(unsigned)chains, kThreads, kSmemBytes, stream>>>(
      a.q, a.k, a.v, a.la, a.beta, a.s0, a.cu, a.order, a.T, a.H, a.o, a.sT, nullptr, a.flags,
      a.tm_k, a.tm_v, a.tm_q, a.tm_la);
  return cudaGetLastError();
}

}  // namespace chunk64

// xfer: a 16-byte aligned buffer of n_seq x H x dk x dv fp32 (laid out like
// the states) that the CTAs of a ring pass the state through: the caller's
// workspace, or its final_state (each chain's slot is then its own final
// state, written last by the owner of the last chunk); NULL runs one CTA per
// chain. gate: 0 per key channel, 1 scalar per token, 2 none; flags: bit 0
// raw q/k, bit 1 raw beta, bit 2 raw gate.
cudaError_t launch_chunk64(const void* q, const void* k, const void* v, const float* la,
                           const float* beta, const float* s0, const int32_t* cu, int n_seq,
                           int T, int H, void* o, float* sT, float* xfer, int32_t* order,
                           int gate, unsigned flags, cudaStream_t stream) {
  using namespace chunk64;
  const long long chains = (long long)n_seq * H;
  int n_sm = 0;
  cudaError_t e0 = launch_state_for_current_device(&n_sm);
  if (e0 != cudaSuccess) return e0;
  if (cu && order) {
    const int blocks = (n_seq + 255) / 256;
    if (n_seq <= 8192)
      order_by_length_kernel<<<blocks, 256, 0, stream>>>(cu, n_seq, order);
    else
      identity_order_kernel<<<blocks, 256, 0, stream>>>(n_seq, order);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  ChunkArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.k = (const __nv_bfloat16*)k;
  a.v = (const __nv_bfloat16*)v;
  a.la = la;
  a.beta = beta;
  a.s0 = s0;
  a.cu = cu;
  a.order = cu ? order : nullptr;
  a.T = T;
  a.H = H;
  a.o = (__nv_bfloat16*)o;
  a.sT = sT;
  a.xfer = xfer;
  a.flags = flags;
  // Tensor maps of k and v over every token of the call (packed: T; dense
  // batch: n_seq x T).
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e1 = tensor_map_encoder(&enc);
  if (e1 != cudaSuccess) return e1;
  const long long tokens = cu ? (long long)T : (long long)n_seq * T;
  if (tokens == 0) {
    memset(&a.tm_k, 0, sizeof(CUtensorMap));   // no chunk to load: never read
    a.tm_v = a.tm_q = a.tm_la = a.tm_k;
    return launch_variant<2, false>(a, chains, 1, stream);   // initial -> final states
  }
  if ((e1 = encode_rows(enc, &a.tm_k, k, true, tokens, H)) != cudaSuccess) return e1;
  if ((e1 = encode_rows(enc, &a.tm_v, v, true, tokens, H)) != cudaSuccess) return e1;
  if ((e1 = encode_rows(enc, &a.tm_q, q, true, tokens, H)) != cudaSuccess) return e1;
  if (gate == 0) {
    if ((e1 = encode_rows(enc, &a.tm_la, la, false, tokens, H)) != cudaSuccess) return e1;
  } else {
    a.tm_la = a.tm_q;   // no per-channel gate tensor: never read
  }
  // Few chains: R = 4 or 2 CTAs per chain (chunks round-robin), all in one
  // wave; the state passes between them through the chain's xfer slot.
  const int ring = (xfer && 2 * chains <= n_sm) ? (4 * chains <= n_sm ? 4 : 2) : 1;
  const bool raw = flags & 1u;
  switch (gate) {
    case 0: return raw ? launch_variant<0, true>(a, chains, ring, stream)
                       : launch_variant<0, false>(a, chains, ring, stream);
    case 1: return raw ? launch_variant<1, true>(a, chains, ring, stream)
                       : launch_variant<1, false>(a, chains, ring, stream);
    default: return raw ? launch_variant<2, true>(a, chains, ring, stream)
                        : launch_variant<2, false>(a, chains, ring, stream);
  }
}

}  // namespace kda
