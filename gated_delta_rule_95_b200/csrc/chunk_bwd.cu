// Backward pass of the chunkwise forward: gradients of o and S_T with respect to q, k, v,
// log alpha, b, w and S0, by reverse mode of the chunk form (Gated DeltaNet-2 guide,
// "Chunkwise Parallel Algorithm for GPU Training"; WY form with the cumulative decay folded
// into the factors, snilld.dk, "Hvad betyder det for traening og inferens").  Per chunk,
// with entering state S, rows = the chunk's tokens, Kb = K*B*Gamma, Qh = Q*Gamma,
// Kn = K/Gamma, Vw = W*V, A = strictly lower part of Kb Kn^T, P = lower part of Qh Kn^T,
// T = (I + A)^-1, R = Vw - Kb S, U = T R, O = Qh S + P U, St = S + Kn^T U and
// S_next = Diag(Gamma_C) St; given dO and dS_next:
//
//     dSt = Diag(Gamma_C) dS_next,   dGamma_C = rowsum(dS_next * St)
//     dU  = P^T dO + Kn dSt,   dR = T^T dU (= dVw),   dP = lower(dO U^T)
//     dA  = strictly lower part of -T^T (dU R^T) T^T
//     dKb = -dR S^T + dA Kn,   dKn = U dSt^T + dA^T Kb + dP^T Qh,   dQh = dO S^T + dP Kn
//     dS  = Qh^T dO + dSt - Kb^T dR
//
// and, elementwise, dK = dKb*B*Gamma + dKn/Gamma, dB = dKb*K*Gamma, dQ = dQh*Gamma,
// dW = dVw*V, dV = dVw*W, dg = dKb*Kb + dQh*Qh - dKn*Kn (+ dGamma_C*Gamma_C on the last
// row), dlog alpha = reverse cumsum of dg over the chunk.
//
// Kernels: chunk_bwd_kernel, one CTA per (batch, head, 32 value columns) — 16 warps for
// bf16 inputs, 8 for fp32 — (value columns never mix in the recurrence, so dS, U, R and
// the per-column gradients split by columns; the key-side gradients dKb, dKn, dQh,
// dGamma_C are sums over the column slices and are accumulated with atomics).  The state
// entering each chunk comes first: for bf16 inputs with d_k = d_v from the tensor-core
// forward's checkpoint pass (a separate launch), otherwise from a forward sweep of this
// kernel over the chunks (its column slice, into the workspace); then the chunks are swept
// in reverse.  chunk_bwd_finish_kernel turns the summed dKb, dKn, dQh into dq, dk, db and
// dlog alpha.  Operands live in shared memory; the products run as tf32 warp-level MMAs
// (fp32 accumulation) for bf16 inputs and as fp32 FFMA on the CUDA cores for fp32 inputs
// (their 1e-4 accuracy bar); everything else is fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int BC = 64;        // chunk size
constexpr int BJ = 32;        // value columns per CTA
constexpr int BT = 256;       // threads per CTA of the CUDA-core path
constexpr int MW = 16;        // warps per CTA of the tensor-core path
// Row padding of the shared-memory tiles: 1 float for the CUDA-core products (whose
// column-wise reads then meet 32 banks), 4 floats for the tensor-core fragments (the 8 x 4
// element groups of an mma fragment then meet 32 banks)
template <bool TC>
__host__ __device__ constexpr int pad() { return TC ? 4 : 1; }

// four consecutive elements (8- or 16-byte aligned) as fp32
__device__ __forceinline__ float4 ld4f(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 ld4f(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

// C[M][N] = sum_k fa(m, k) fb(k, n), spread over the 256 threads: thread (tm, tn) owns rows
// tm*TM .. +TM and columns tn, tn + N/TN, ... (consecutive threads take consecutive
// columns), handing each result to epi(m, n, value).
template <int M, int N, int TM, int TN, class FA, class FB, class FE>
__device__ __forceinline__ void gemm(int K, FA fa, FB fb, FE epi) {
  constexpr int NC = N / TN;
  static_assert((M / TM) * NC == BT, "thread tiling must cover the output");
  const int tn = threadIdx.x % NC, tm = threadIdx.x / NC;
  float acc[TM][TN];
#pragma unroll
  for (int x = 0; x < TM; ++x)
#pragma unroll
    for (int y = 0; y < TN; ++y) acc[x][y] = 0.f;
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float av[TM], bv[TN];
#pragma unroll
    for (int x = 0; x < TM; ++x) av[x] = fa(tm * TM + x, k);
#pragma unroll
    for (int y = 0; y < TN; ++y) bv[y] = fb(k, tn + y * NC);
#pragma unroll
    for (int x = 0; x < TM; ++x)
#pragma unroll
      for (int y = 0; y < TN; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
  }
#pragma unroll
  for (int x = 0; x < TM; ++x)
#pragma unroll
    for (int y = 0; y < TN; ++y) epi(tm * TM + x, tn + y * NC, acc[x][y]);
}

// The same products on the tensor cores (bf16 inputs): mma.sync m16n8k8 with operands
// rounded to tf32 (nearest), fp32 accumulation.  The 16 x 8 output tiles go to the MW warps
// in row-major order, TPW consecutive tiles per warp sharing one 16-row block, so that a
// warp loads each A fragment once per k step.  d holds the warp's tiles' accumulators.
__device__ __forceinline__ uint32_t tf32r(float x) { return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u; }

template <int M, int N>
struct MT {
  static constexpr int NT = N / 8, TPW = (M / 16) * NT / MW;
  static_assert(TPW >= 1 && NT % TPW == 0, "a warp's tiles must share a row block");
};
template <int M, int N>
__device__ __forceinline__ void mzero(float (&d)[MT<M, N>::TPW][4]) {
#pragma unroll
  for (int q = 0; q < MT<M, N>::TPW; ++q) d[q][0] = d[q][1] = d[q][2] = d[q][3] = 0.f;
}
template <int M, int N, class FA, class FB>
__device__ __forceinline__ void mmac(float (&d)[MT<M, N>::TPW][4], int K, FA fa, FB fb) {
  constexpr int NT = MT<M, N>::NT, TPW = MT<M, N>::TPW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int m0 = (warp * TPW / NT) * 16, nb = (warp * TPW) % NT;
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    const uint32_t a[4] = {tf32r(fa(m0 + g, k0 + t)), tf32r(fa(m0 + g + 8, k0 + t)), tf32r(fa(m0 + g, k0 + t + 4)),
                           tf32r(fa(m0 + g + 8, k0 + t + 4))};
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      const int n0 = 8 * (nb + q);
      const uint32_t b[2] = {tf32r(fb(k0 + t, n0 + g)), tf32r(fb(k0 + t + 4, n0 + g))};
      mma_16x8x8_tf32(d[q], a, b);
    }
  }
}
// two products sharing their B operand: d1 (+)= A1 B and d2 (+)= A2 B, each B fragment
// loaded once for both
template <int M, int N, class FA1, class FA2, class FB>
__device__ __forceinline__ void mmac2(float (&d1)[MT<M, N>::TPW][4], float (&d2)[MT<M, N>::TPW][4], int K, FA1 fa1,
                                      FA2 fa2, FB fb) {
  constexpr int NT = MT<M, N>::NT, TPW = MT<M, N>::TPW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int m0 = (warp * TPW / NT) * 16, nb = (warp * TPW) % NT;
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    const uint32_t a1[4] = {tf32r(fa1(m0 + g, k0 + t)), tf32r(fa1(m0 + g + 8, k0 + t)),
                            tf32r(fa1(m0 + g, k0 + t + 4)), tf32r(fa1(m0 + g + 8, k0 + t + 4))};
    const uint32_t a2[4] = {tf32r(fa2(m0 + g, k0 + t)), tf32r(fa2(m0 + g + 8, k0 + t)),
                            tf32r(fa2(m0 + g, k0 + t + 4)), tf32r(fa2(m0 + g + 8, k0 + t + 4))};
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      const int n0 = 8 * (nb + q);
      const uint32_t b[2] = {tf32r(fb(k0 + t, n0 + g)), tf32r(fb(k0 + t + 4, n0 + g))};
      mma_16x8x8_tf32(d1[q], a1, b);
      mma_16x8x8_tf32(d2[q], a2, b);
    }
  }
}
// epi(m, n, value) for every element of the warp's tiles
template <int M, int N, class FE>
__device__ __forceinline__ void mepi(const float (&d)[MT<M, N>::TPW][4], FE epi) {
  constexpr int NT = MT<M, N>::NT, TPW = MT<M, N>::TPW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int m0 = (warp * TPW / NT) * 16, nb = (warp * TPW) % NT;
#pragma unroll
  for (int q = 0; q < TPW; ++q) {
    const int n0 = 8 * (nb + q);
    epi(m0 + g, n0 + 2 * t, d[q][0]);
    epi(m0 + g, n0 + 2 * t + 1, d[q][1]);
    epi(m0 + g + 8, n0 + 2 * t, d[q][2]);
    epi(m0 + g + 8, n0 + 2 * t + 1, d[q][3]);
  }
}
template <int M, int N, class FA, class FB, class FE>
__device__ __forceinline__ void mgemm(int K, FA fa, FB fb, FE epi) {
  float d[MT<M, N>::TPW][4];
  mzero<M, N>(d);
  mmac<M, N>(d, K, fa, fb);
  mepi<M, N>(d, epi);
}
// the products of the kernel: tensor cores for bf16 inputs, CUDA-core fp32 for fp32 inputs
template <bool TC, int M, int N, int TM, int TN, class FA, class FB, class FE>
__device__ __forceinline__ void prod(int K, FA fa, FB fb, FE epi) {
  if constexpr (TC)
    mgemm<M, N>(K, fa, fb, epi);
  else
    gemm<M, N, TM, TN>(K, fa, fb, epi);
}

template <typename E>
struct BwdParams {
  const E *q, *k, *v, *b, *w;
  const float* la;
  const float* S0;
  const float* dO;
  const float* dST;
  float *dq, *dk, *db;  // on entry zero; receive the summed dQh, dKb, dKn
  float *dv, *dw, *dS0;
  float* states;        // [B H][nch][DK][DV]: each chunk's entering state
  float* dgc;           // [B H][nch][DK]: dGamma_C, zero on entry
  int T, H, nch;
  int states_given;     // the entering states are already in `states`
  unsigned long long* stamps = nullptr;  // instrumented build only: per-chunk clock stamps
};

#ifdef GDN2_STAMPS
// Instrumented build (GDN2_STAMPS): clock64 at fixed points of the reverse sweep, for the
// first CTA (batch 0, head 0, value columns 0-31), into [chunk][slot] of a 64 x 32 array;
// thread 0 writes.
#define BWD_STAMP(cc, slot)                                                                    \
  do {                                                                                         \
    if (p.stamps && blockIdx.x == 0 && threadIdx.x == 0 && (cc) >= 0 && (cc) < 64)             \
      p.stamps[(size_t)(cc) * 32 + (slot)] = (unsigned long long)clock64();                    \
  } while (0)
#else
#define BWD_STAMP(cc, slot) \
  do {                      \
  } while (0)
#endif

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(std::is_same<T, __nv_bfloat16>::value ? 32 * MW : BT, 1)
    chunk_bwd_kernel(const BwdParams<T> p) {
  constexpr bool TC = std::is_same<T, __nv_bfloat16>::value;  // products on the tensor cores
  constexpr int NTH = TC ? 32 * MW : BT;                       // threads of the CTA
  constexpr int LK = DK + pad<TC>();  // padded rows: [BC][DK] tiles
  constexpr int LJ = BJ + pad<TC>();  //              [.][BJ] tiles
  constexpr int LC = BC + pad<TC>();  //              [BC][BC] tiles
  constexpr int NS = DV / BJ;
  extern __shared__ float sm[];
  float* Kb = sm;
  float* Qh = Kb + BC * LK;
  float* Kn = Qh + BC * LK;
  float* Sj = Kn + BC * LK;      // [DK][LJ]  entering state, this CTA's columns
  float* dS = Sj + DK * LJ;      // [DK][LJ]  gradient of the state after the chunk (then before it)
  float* Tm = dS + DK * LJ;      // [BC][LC]  T
  float* Pm = Tm + BC * LC;      // [BC][LC]  P, then Y = dT T^T, then dP
  float* X1 = Pm + BC * LC;      // [BC][LC]  A, then dT, then dA
  float* Rm = X1 + BC * LC;      // [BC][LJ]  R, then dR
  float* dU = Rm + BC * LJ;      // [BC][LJ]  dGamma_C (first DK floats), then dU
  float* Um = dU + BC * LJ;      // [BC][LJ]  U
  float* dOj = Um + BC * LJ;     // [BC][LJ]  dO
  float* gC = dOj + BC * LJ;     // [DK]      Gamma_C
  float* dgC = dU;               // [DK]      dGamma_C, this CTA's part
  float* Ym = Pm;
  float* dR = Rm;

  const int tid = threadIdx.x;
  const int sl = blockIdx.x % NS, bh = blockIdx.x / NS;
  const int h = bh % p.H, bb = bh / p.H;
  const int j0 = sl * BJ;
  const size_t rowstride = (size_t)p.H;  // tokens are [B][T][H][D]
  auto tok = [&](int t) { return ((size_t)bb * p.T + t) * rowstride + h; };  // (token, head) index

  // Kb, Kn (and Qh) of chunk c, Gamma_C; rows past the sequence are zero.  The raw inputs
  // are loaded by all threads (log alpha into the free T, P, A tiles), then thread i < DK
  // walks the rows of key channel i, summing log alpha, and folds the decay in place.
  auto build = [&](int c, bool with_q) {
    const int t0 = c * BC;
    float* raw_la = Pm;  // [BC][DK] over P, A and R (free at this point; T keeps its zeros)
    // four consecutive key channels per load, every load of the thread in flight at once
    constexpr int Q4 = BC * DK / 4 / NTH;
    float4 la4[Q4], k4[Q4], b4[Q4], q4[Q4];
#pragma unroll
    for (int m = 0; m < Q4; ++m) {
      const int e4 = tid + NTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4)), tt = t0 + t;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      la4[m] = k4[m] = b4[m] = q4[m] = z;
      if (tt < p.T) {
        const size_t x = tok(tt) * DK + i;
        la4[m] = ld4f(p.la + x);
        k4[m] = ld4f(p.k + x);
        b4[m] = ld4f(p.b + x);
        if (with_q) q4[m] = ld4f(p.q + x);
      }
    }
#pragma unroll
    for (int m = 0; m < Q4; ++m) {
      const int e4 = tid + NTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
      *reinterpret_cast<float4*>(raw_la + t * DK + i) = la4[m];
      if constexpr (LK % 4 == 0) {  // 16-byte aligned rows: one vector store each
        *reinterpret_cast<float4*>(Kn + t * LK + i) = k4[m];
        *reinterpret_cast<float4*>(Kb + t * LK + i) = b4[m];
        if (with_q) *reinterpret_cast<float4*>(Qh + t * LK + i) = q4[m];
      } else {
        const float kk[4] = {k4[m].x, k4[m].y, k4[m].z, k4[m].w}, bg[4] = {b4[m].x, b4[m].y, b4[m].z, b4[m].w};
        const float qq[4] = {q4[m].x, q4[m].y, q4[m].z, q4[m].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          Kn[t * LK + i + u] = kk[u];
          Kb[t * LK + i + u] = bg[u];
          if (with_q) Qh[t * LK + i + u] = qq[u];
        }
      }
    }
    __syncthreads();
    // the cumulative log decay, RS threads per key channel each over BC / RS rows: segment
    // sums first, then each segment's scan from the sum of the segments before it
    constexpr int RS = NTH / DK, RL = BC / RS;
    float* part = raw_la + BC * DK;  // [RS][DK], past the raw log alpha (2 BC LC + BC LJ >= BC DK + NTH)
    const int i = tid % DK, sgm = tid / DK;
    {
      float sum = 0.f;
#pragma unroll 8
      for (int t = sgm * RL; t < sgm * RL + RL; ++t) sum += raw_la[t * DK + i];
      part[sgm * DK + i] = sum;
    }
    __syncthreads();
    float g = 0.f;
    for (int r = 0; r < sgm; ++r) g += part[r * DK + i];
#pragma unroll 4
    for (int t = sgm * RL; t < sgm * RL + RL; ++t) {
      g += raw_la[t * DK + i];
      const float G = __expf(g), kk = Kn[t * LK + i];
      Kb[t * LK + i] *= kk * G;
      Kn[t * LK + i] = kk * __expf(-g);
      if (with_q) Qh[t * LK + i] *= G;
    }
    if (sgm == RS - 1) gC[i] = __expf(g);
  };
  // the inputs of chunk c into L2 while the current chunk computes (q and dO only for the
  // reverse sweep): one 128-byte line per thread and row segment
  auto prefetch = [&](int c, bool rev) {
    if (c < 0 || c >= p.nch) return;
    const int t0 = c * BC;
    constexpr int KL = DK * (int)sizeof(T) / 128, VL = DV * (int)sizeof(T) / 128;  // lines per row
    constexpr int LL = DK * 4 / 128, OL = DV * 4 / 128;
    const int nseg = 2 * KL + LL + 2 * VL + (rev ? KL + OL : 0);
    for (int e = tid; e < BC * nseg; e += NTH) {
      const int t = e % BC, r = e / BC, tt = t0 + t;
      if (tt >= p.T) continue;
      const char* a;
      int m = r;
      if (m < KL) a = reinterpret_cast<const char*>(p.k + tok(tt) * DK) + 128 * m;
      else if ((m -= KL) < KL) a = reinterpret_cast<const char*>(p.b + tok(tt) * DK) + 128 * m;
      else if ((m -= KL) < LL) a = reinterpret_cast<const char*>(p.la + tok(tt) * DK) + 128 * m;
      else if ((m -= LL) < VL) a = reinterpret_cast<const char*>(p.v + tok(tt) * DV) + 128 * m;
      else if ((m -= VL) < VL) a = reinterpret_cast<const char*>(p.w + tok(tt) * DV) + 128 * m;
      else if ((m -= VL) < KL) a = reinterpret_cast<const char*>(p.q + tok(tt) * DK) + 128 * m;
      else a = reinterpret_cast<const char*>(p.dO + tok(tt) * DV) + 128 * (m - KL);
      asm volatile("prefetch.global.L2 [%0];" :: "l"(a));
    }
    if (rev)  // the chunk's entering state, this CTA's columns: one line per key channel
      for (int i = tid; i < DK; i += NTH) {
        const float* a = p.states + (((size_t)bh * p.nch + c) * DK + i) * DV + j0;
        asm volatile("prefetch.global.L2 [%0];" :: "l"(a));
      }
  };
  // T = (I + A)^-1 from A (strictly lower, in X1), by blocks: the 16 x 16 diagonal blocks by
  // forward substitution (one warp per block, a column per lane, in registers), then the
  // 2 x 2 block merges T21 = -T22 (A21 T11) at 32 and 64 (products staged in the R tile,
  // free at this point).
  auto solve = [&]() {  // (every entry above the diagonal of T is zero from the start; the
                        // first 128 or 256 threads work, the rest only meet the barriers)
    if (tid < 128) {
      // warp w: diagonal block w (rows 16 w ..); lane j < 16 forms column j of its inverse in
      // registers by forward substitution (x[s] = 0 for s < j, so each row sums over s < r)
      const int base = 16 * (tid >> 5), j = tid & 15;
      const float* Ab = X1 + base * LC + base;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float ar[16];
        if constexpr (LC % 4 == 0) {  // 16-byte aligned rows: vector loads
#pragma unroll
          for (int q4 = 0; q4 < (r + 3) / 4; ++q4) {
            const float4 a = *reinterpret_cast<const float4*>(Ab + r * LC + 4 * q4);
            ar[4 * q4] = a.x;
            ar[4 * q4 + 1] = a.y;
            ar[4 * q4 + 2] = a.z;
            ar[4 * q4 + 3] = a.w;
          }
        } else {
#pragma unroll
          for (int s2 = 0; s2 < r; ++s2) ar[s2] = Ab[r * LC + s2];
        }
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int s2 = 0; s2 + 1 < r; s2 += 2) {
          acc0 = fmaf(ar[s2], x[s2], acc0);
          acc1 = fmaf(ar[s2 + 1], x[s2 + 1], acc1);
        }
        if (r & 1) acc0 = fmaf(ar[r - 1], x[r - 1], acc0);
        x[r] = r == j ? 1.f : (r > j ? -(acc0 + acc1) : 0.f);
      }
      if ((tid & 31) < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[(base + r) * LC + base + j] = x[r];
      }
    }
    __syncthreads();
    float* Xs = Rm;  // [32][LJ]
    {
      // 32: blocks q = 0, 1 at offset 32 q; thread: row r of the block, columns c, c + 1
      const int q = (tid >> 7) & 1, r = (tid >> 3) & 15, c = 2 * (tid & 7), o = 32 * q;
      if (tid < 256) {
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float a = X1[(o + 16 + r) * LC + o + m];
          x0 = fmaf(a, Tm[(o + m) * LC + o + c], x0);
          x1 = fmaf(a, Tm[(o + m) * LC + o + c + 1], x1);
        }
        Xs[(16 * q + r) * LJ + c] = x0;
        Xs[(16 * q + r) * LJ + c + 1] = x1;
      }
      __syncthreads();
      if (tid < 256) {
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float t22 = Tm[(o + 16 + r) * LC + o + 16 + m];
          y0 = fmaf(t22, Xs[(16 * q + m) * LJ + c], y0);
          y1 = fmaf(t22, Xs[(16 * q + m) * LJ + c + 1], y1);
        }
        Tm[(o + 16 + r) * LC + o + c] = -y0;
        Tm[(o + 16 + r) * LC + o + c + 1] = -y1;
      }
    }
    __syncthreads();
    {
      // 64: thread: row r of the lower half, columns [4 c4, 4 c4 + 4)
      const int r = (tid >> 3) & 31, c4 = 4 * (tid & 7);
      if (tid < 256) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int m = 0; m < 32; ++m) {
          const float a = X1[(32 + r) * LC + m];
#pragma unroll
          for (int y = 0; y < 4; ++y) x[y] = fmaf(a, Tm[m * LC + c4 + y], x[y]);
        }
#pragma unroll
        for (int y = 0; y < 4; ++y) Xs[r * LJ + c4 + y] = x[y];
      }
      __syncthreads();
      if (tid < 256) {
        float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int m = 0; m < 32; ++m) {
          const float t22 = Tm[(32 + r) * LC + 32 + m];
#pragma unroll
          for (int y = 0; y < 4; ++y) z[y] = fmaf(t22, Xs[m * LJ + c4 + y], z[y]);
        }
#pragma unroll
        for (int y = 0; y < 4; ++y) Tm[(32 + r) * LC + c4 + y] = -z[y];
      }
    }
  };
  // R = Vw - Kb S and U = T R for chunk c
  auto r_and_u = [&](int c) {
    const int t0 = c * BC;
    prod<TC, BC, BJ, 2, 4>(DK, [&](int t, int i) { return Kb[t * LK + i]; }, [&](int i, int j) { return Sj[i * LJ + j]; },
                       [&](int t, int j, float acc) {
                         const int tt = t0 + t;
                         float vw = 0.f;
                         if (tt < p.T) {
                           const size_t x = tok(tt) * DV + j0 + j;
                           vw = ldf(p.w + x) * ldf(p.v + x);
                         }
                         Rm[t * LJ + j] = vw - acc;
                       });
    __syncthreads();
    prod<TC, BC, BJ, 2, 4>(BC, [&](int t, int s) { return Tm[t * LC + s]; }, [&](int s, int j) { return Rm[s * LJ + j]; },
                       [&](int t, int j, float acc) { Um[t * LJ + j] = acc; });
  };
  auto strict_lower_kk = [&](float* dst, const float* Lhs, bool incl_diag) {
    prod<TC, BC, BC, 4, 4>(DK, [&](int t, int i) { return Lhs[t * LK + i]; }, [&](int i, int s) { return Kn[s * LK + i]; },
                       [&](int t, int s, float acc) { dst[t * LC + s] = (s < t || (incl_diag && s == t)) ? acc : 0.f; });
  };

  for (int e = tid; e < BC * LC; e += NTH) Tm[e] = 0.f;  // T: zero above the diagonal for good
  // ---- forward sweep: every chunk's entering state (unless given) ---------------------------
  for (int e = tid; e < DK * BJ && !p.states_given; e += NTH) {
    const int i = e / BJ, j = e % BJ;
    Sj[i * LJ + j] = p.S0 ? p.S0[((size_t)bh * DK + i) * DV + j0 + j] : 0.f;
  }
  __syncthreads();
  for (int c = 0; c < p.nch && !p.states_given; ++c) {
    prefetch(c + 1, false);
    float* st = p.states + ((size_t)bh * p.nch + c) * DK * DV;
    for (int e = tid; e < DK * BJ; e += NTH) {
      const int i = e / BJ, j = e % BJ;
      st[(size_t)i * DV + j0 + j] = Sj[i * LJ + j];
    }
    build(c, false);
    __syncthreads();
    strict_lower_kk(X1, Kb, false);
    __syncthreads();
    solve();
    __syncthreads();
    r_and_u(c);
    __syncthreads();
    // S <- Diag(Gamma_C) (S + Kn^T U)
    prod<TC, DK, BJ, DK / 32, 4>(BC, [&](int i, int s) { return Kn[s * LK + i]; },
                             [&](int s, int j) { return Um[s * LJ + j]; },
                             [&](int i, int j, float acc) { Sj[i * LJ + j] = gC[i] * (Sj[i * LJ + j] + acc); });
    __syncthreads();
  }

  // ---- reverse sweep -------------------------------------------------------------------------
  for (int e = tid; e < DK * BJ; e += NTH) {
    const int i = e / BJ, j = e % BJ;
    dS[i * LJ + j] = p.dST ? p.dST[((size_t)bh * DK + i) * DV + j0 + j] : 0.f;
  }
  __syncthreads();
  for (int c = p.nch - 1; c >= 0; --c) {
    const int t0 = c * BC;
    prefetch(c - 1, true);
    const float* st = p.states + ((size_t)bh * p.nch + c) * DK * DV;
    {
      constexpr int NSQ = DK * BJ / 4 / NTH, NOQ = BC * BJ / 4 / NTH;
      float4 sv[NSQ], ov[NOQ];
#pragma unroll
      for (int m = 0; m < NSQ; ++m) {
        const int e4 = tid + NTH * m, i = e4 / (BJ / 4), j = 4 * (e4 % (BJ / 4));
        sv[m] = ld4f(st + (size_t)i * DV + j0 + j);
      }
#pragma unroll
      for (int m = 0; m < NOQ; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (BJ / 4), j = 4 * (e4 % (BJ / 4)), tt = t0 + t;
        ov[m] = tt < p.T ? ld4f(p.dO + tok(tt) * DV + j0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int m = 0; m < NSQ; ++m) {
        const int e4 = tid + NTH * m, i = e4 / (BJ / 4), j = 4 * (e4 % (BJ / 4));
        Sj[i * LJ + j] = sv[m].x;
        Sj[i * LJ + j + 1] = sv[m].y;
        Sj[i * LJ + j + 2] = sv[m].z;
        Sj[i * LJ + j + 3] = sv[m].w;
      }
#pragma unroll
      for (int m = 0; m < NOQ; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (BJ / 4), j = 4 * (e4 % (BJ / 4));
        dOj[t * LJ + j] = ov[m].x;
        dOj[t * LJ + j + 1] = ov[m].y;
        dOj[t * LJ + j + 2] = ov[m].z;
        dOj[t * LJ + j + 3] = ov[m].w;
      }
    }
    BWD_STAMP(c, 0);
    if (tid < DK) dgC[tid] = 0.f;
    build(c, true);
    __syncthreads();
    BWD_STAMP(c, 1);
    strict_lower_kk(X1, Kb, false);  // A
    strict_lower_kk(Pm, Qh, true);   // P
    __syncthreads();
    BWD_STAMP(c, 2);
    solve();
    __syncthreads();
    BWD_STAMP(c, 3);
    r_and_u(c);
    __syncthreads();
    BWD_STAMP(c, 4);
    // dGamma_C = rowsum(dS_next * (S + Kn^T U)), this CTA's columns: thread (row group,
    // column group) sums its products, then the 8 threads of a row group add theirs
    if constexpr (TC) {
      float d[MT<DK, BJ>::TPW][4];
      mzero<DK, BJ>(d);
      mmac<DK, BJ>(d, BC, [&](int i, int s) { return Kn[s * LK + i]; }, [&](int s, int j) { return Um[s * LJ + j]; });
      float rs[2] = {0.f, 0.f};  // rows g and g + 8 of the warp's row block
      int rows[2] = {0, 0};
      mepi<DK, BJ>(d, [&](int i, int j, float acc) {
        const int h8 = ((i & 15) >= 8);
        rows[h8] = i;
        rs[h8] = fmaf(dS[i * LJ + j], Sj[i * LJ + j] + acc, rs[h8]);
      });
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float r = rs[u];
        r += __shfl_xor_sync(0xffffffffu, r, 1);
        r += __shfl_xor_sync(0xffffffffu, r, 2);
        if ((tid & 3) == 0) atomicAdd(&dgC[rows[u]], r);
      }
    } else {
      constexpr int TM = DK / 32;
      const int tn = tid % 8, tm = tid / 8;
      float acc[TM][4];
#pragma unroll
      for (int x = 0; x < TM; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 4
      for (int t = 0; t < BC; ++t) {
        float kv[TM], uv[4];
#pragma unroll
        for (int x = 0; x < TM; ++x) kv[x] = Kn[t * LK + tm * TM + x];
#pragma unroll
        for (int y = 0; y < 4; ++y) uv[y] = Um[t * LJ + tn + 8 * y];
#pragma unroll
        for (int x = 0; x < TM; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(kv[x], uv[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < TM; ++x) {
        const int i = tm * TM + x;
        float r = 0.f;
#pragma unroll
        for (int y = 0; y < 4; ++y) r = fmaf(dS[i * LJ + tn + 8 * y], Sj[i * LJ + tn + 8 * y] + acc[x][y], r);
        r += __shfl_xor_sync(0xffffffffu, r, 1);
        r += __shfl_xor_sync(0xffffffffu, r, 2);
        r += __shfl_xor_sync(0xffffffffu, r, 4);
        if (tn == 0) dgC[i] = r;
      }
    }
    __syncthreads();
    if (tid < DK) atomicAdd(p.dgc + ((size_t)bh * p.nch + c) * DK + tid, dgC[tid]);
    // dSt = Diag(Gamma_C) dS_next, in place
    for (int e = tid; e < DK * BJ; e += NTH) {
      const int i = e / BJ, j = e % BJ;
      dS[i * LJ + j] *= gC[i];
    }
    __syncthreads();
    BWD_STAMP(c, 5);
    // dU = P^T dO + Kn dSt
    prod<TC, BC, BJ, 2, 4>(BC, [&](int t, int s) { return Pm[s * LC + t]; }, [&](int s, int j) { return dOj[s * LJ + j]; },
                       [&](int t, int j, float acc) { dU[t * LJ + j] = acc; });
    prod<TC, BC, BJ, 2, 4>(DK, [&](int t, int i) { return Kn[t * LK + i]; }, [&](int i, int j) { return dS[i * LJ + j]; },
                       [&](int t, int j, float acc) { dU[t * LJ + j] += acc; });
    __syncthreads();
    // dT = dU R^T over A
    prod<TC, BC, BC, 4, 4>(BJ, [&](int t, int j) { return dU[t * LJ + j]; }, [&](int j, int s) { return Rm[s * LJ + j]; },
                           [&](int t, int s, float acc) { X1[t * LC + s] = acc; });
    __syncthreads();
    // dR = T^T dU (= dVw) over R: dW = dVw * V, dV = dVw * W; Y = dT T^T over P
    prod<TC, BC, BJ, 2, 4>(BC, [&](int t, int s) { return Tm[s * LC + t]; }, [&](int s, int j) { return dU[s * LJ + j]; },
                           [&](int t, int j, float acc) {
                             dR[t * LJ + j] = acc;
                             const int tt = t0 + t;
                             if (tt < p.T) {
                               const size_t x = tok(tt) * DV + j0 + j;
                               p.dw[x] = acc * ldf(p.v + x);
                               p.dv[x] = acc * ldf(p.w + x);
                             }
                           });
    prod<TC, BC, BC, 4, 4>(BC, [&](int t, int r) { return X1[t * LC + r]; }, [&](int r, int s) { return Tm[s * LC + r]; },
                           [&](int t, int s, float acc) { Ym[t * LC + s] = acc; });
    __syncthreads();
    BWD_STAMP(c, 6);
    // dA = strictly lower part of -T^T Y over dT
    prod<TC, BC, BC, 4, 4>(BC, [&](int t, int r) { return Tm[r * LC + t]; }, [&](int r, int s) { return Ym[r * LC + s]; },
                           [&](int t, int s, float acc) { X1[t * LC + s] = s < t ? -acc : 0.f; });
    __syncthreads();
    // dP = lower(dO U^T) over Y
    prod<TC, BC, BC, 4, 4>(BJ, [&](int t, int j) { return dOj[t * LJ + j]; }, [&](int j, int s) { return Um[s * LJ + j]; },
                           [&](int t, int s, float acc) { Pm[t * LC + s] = s <= t ? acc : 0.f; });
    __syncthreads();
    BWD_STAMP(c, 7);
    // key-side gradients of this CTA's columns, summed over the slices in global memory:
    //   dKb = -dR S^T + dA Kn,  dKn = U dSt^T + dA^T Kb + dP^T Qh,  dQh = dO S^T + dP Kn
    if constexpr (TC) {
      float d[MT<BC, DK>::TPW][4], d2[MT<BC, DK>::TPW][4];
      auto out = [&](float* dst, const float (&d)[MT<BC, DK>::TPW][4]) {  // 8-byte atomics
        constexpr int NT = MT<BC, DK>::NT, TPW = MT<BC, DK>::TPW;
        const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
        const int m0 = (warp * TPW / NT) * 16, nb = (warp * TPW) % NT;
#pragma unroll
        for (int q = 0; q < TPW; ++q) {
          const int i = 8 * (nb + q) + 2 * tq;
          const int ta = t0 + m0 + g, tb = ta + 8;
          if (ta < p.T) atomicAdd(reinterpret_cast<float2*>(dst + tok(ta) * DK + i), make_float2(d[q][0], d[q][1]));
          if (tb < p.T) atomicAdd(reinterpret_cast<float2*>(dst + tok(tb) * DK + i), make_float2(d[q][2], d[q][3]));
        }
      };
      // dKb and dQh share their B operands (S, then Kn)
      mzero<BC, DK>(d);
      mzero<BC, DK>(d2);
      mmac2<BC, DK>(d, d2, BJ, [&](int t, int j) { return -dR[t * LJ + j]; }, [&](int t, int j) { return dOj[t * LJ + j]; },
                    [&](int j, int i) { return Sj[i * LJ + j]; });
      mmac2<BC, DK>(d, d2, BC, [&](int t, int s) { return X1[t * LC + s]; }, [&](int t, int s) { return Pm[t * LC + s]; },
                    [&](int s, int i) { return Kn[s * LK + i]; });
      out(p.dk, d);
      out(p.dq, d2);
      mzero<BC, DK>(d);
      mmac<BC, DK>(d, BJ, [&](int t, int j) { return Um[t * LJ + j]; }, [&](int j, int i) { return dS[i * LJ + j]; });
      mmac<BC, DK>(d, BC, [&](int t, int s) { return X1[s * LC + t]; }, [&](int s, int i) { return Kb[s * LK + i]; });
      mmac<BC, DK>(d, BC, [&](int t, int s) { return Pm[s * LC + t]; }, [&](int s, int i) { return Qh[s * LK + i]; });
      out(p.db, d);
    } else {
      // 64 x DK outputs: thread (tm, tn) takes rows 4 tm .. +4 and the key channels
      // 4 tn + 64 g + u (u < 4), so that its sums leave as 16-byte vector atomics
      constexpr int TN = DK / 16, NC = 16;
      const int tn = tid % NC, tm = tid / NC;
      auto col = [&](int y) { return 4 * tn + 64 * (y >> 2) + (y & 3); };
      float akb[4][TN], akn[4][TN], aqh[4][TN];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < TN; ++y) akb[x][y] = akn[x][y] = aqh[x][y] = 0.f;
#pragma unroll 2
      for (int j = 0; j < BJ; ++j) {
        float sv[TN], dsv[TN];
#pragma unroll
        for (int y = 0; y < TN; ++y) {
          sv[y] = Sj[col(y) * LJ + j];
          dsv[y] = dS[col(y) * LJ + j];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int t = tm * 4 + x;
          const float r = dR[t * LJ + j], u = Um[t * LJ + j], o = dOj[t * LJ + j];
#pragma unroll
          for (int y = 0; y < TN; ++y) {
            akb[x][y] = fmaf(-r, sv[y], akb[x][y]);
            akn[x][y] = fmaf(u, dsv[y], akn[x][y]);
            aqh[x][y] = fmaf(o, sv[y], aqh[x][y]);
          }
        }
      }
#pragma unroll 2
      for (int s = 0; s < BC; ++s) {
        float knv[TN], kbv[TN], qhv[TN];
#pragma unroll
        for (int y = 0; y < TN; ++y) {
          const int i = col(y);
          knv[y] = Kn[s * LK + i];
          kbv[y] = Kb[s * LK + i];
          qhv[y] = Qh[s * LK + i];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int t = tm * 4 + x;
          const float da = X1[t * LC + s], daT = X1[s * LC + t], dp = Pm[t * LC + s], dpT = Pm[s * LC + t];
#pragma unroll
          for (int y = 0; y < TN; ++y) {
            akb[x][y] = fmaf(da, knv[y], akb[x][y]);
            akn[x][y] = fmaf(daT, kbv[y], fmaf(dpT, qhv[y], akn[x][y]));
            aqh[x][y] = fmaf(dp, knv[y], aqh[x][y]);
          }
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int tt = t0 + tm * 4 + x;
        if (tt >= p.T) continue;
#pragma unroll
        for (int y = 0; y < TN; y += 4) {
          const size_t xi = tok(tt) * DK + col(y);  // 16-byte aligned
          atomicAdd(reinterpret_cast<float4*>(p.dk + xi), make_float4(akb[x][y], akb[x][y + 1], akb[x][y + 2], akb[x][y + 3]));
          atomicAdd(reinterpret_cast<float4*>(p.db + xi), make_float4(akn[x][y], akn[x][y + 1], akn[x][y + 2], akn[x][y + 3]));
          atomicAdd(reinterpret_cast<float4*>(p.dq + xi), make_float4(aqh[x][y], aqh[x][y + 1], aqh[x][y + 2], aqh[x][y + 3]));
        }
      }
    }
    BWD_STAMP(c, 8);
    // dS (before the chunk) = Qh^T dO + dSt - Kb^T dR
    if constexpr (TC) {
      float d[MT<DK, BJ>::TPW][4];
      mzero<DK, BJ>(d);
      mmac<DK, BJ>(d, BC, [&](int i, int t) { return Qh[t * LK + i]; }, [&](int t, int j) { return dOj[t * LJ + j]; });
      mmac<DK, BJ>(d, BC, [&](int i, int t) { return -Kb[t * LK + i]; }, [&](int t, int j) { return dR[t * LJ + j]; });
      float acc[MT<DK, BJ>::TPW][4];
      int e = 0;
      mepi<DK, BJ>(d, [&](int i, int j, float v) {
        acc[e >> 2][e & 3] = v + dS[i * LJ + j];
        ++e;
      });
      __syncthreads();  // every read of dSt is done
      e = 0;
      mepi<DK, BJ>(d, [&](int i, int j, float v) {
        static_cast<void>(v);
        dS[i * LJ + j] = acc[e >> 2][e & 3];
        ++e;
      });
    } else {
      constexpr int TM = DK / 32;
      const int tn = tid % 8, tm = tid / 8;
      float acc[TM][4];
#pragma unroll
      for (int x = 0; x < TM; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = dS[(tm * TM + x) * LJ + tn + 8 * y];
#pragma unroll 4
      for (int t = 0; t < BC; ++t) {
        float qv[TM], kv[TM], ov[4], rv[4];
#pragma unroll
        for (int x = 0; x < TM; ++x) {
          qv[x] = Qh[t * LK + tm * TM + x];
          kv[x] = Kb[t * LK + tm * TM + x];
        }
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          ov[y] = dOj[t * LJ + tn + 8 * y];
          rv[y] = dR[t * LJ + tn + 8 * y];
        }
#pragma unroll
        for (int x = 0; x < TM; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(qv[x], ov[y], fmaf(-kv[x], rv[y], acc[x][y]));
      }
      __syncthreads();  // every read of dSt is done
#pragma unroll
      for (int x = 0; x < TM; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) dS[(tm * TM + x) * LJ + tn + 8 * y] = acc[x][y];
    }
    __syncthreads();
    BWD_STAMP(c, 9);
  }
  if (p.dS0)
    for (int e = tid; e < DK * BJ; e += NTH) {
      const int i = e / BJ, j = e % BJ;
      p.dS0[((size_t)bh * DK + i) * DV + j0 + j] = dS[i * LJ + j];
    }
}

// dq, dk, db and dlog alpha from the summed dQh, dKb, dKn (held in dq, dk, db): thread i of
// CTA (batch, head, chunk) walks the chunk's rows of key channel i.
template <typename T, int DK>
__global__ void __launch_bounds__(DK) chunk_bwd_finish_kernel(const BwdParams<T> p, float* dla) {
  const int i = threadIdx.x;
  const int c = blockIdx.x % p.nch, bh = blockIdx.x / p.nch;
  const int h = bh % p.H, bb = bh / p.H;
  const int t0 = c * BC, n = min(BC, p.T - t0);
  float G[BC];  // Gamma of each row
  float g = 0.f;
#pragma unroll
  for (int t = 0; t < BC; ++t) {
    if (t < n) g += __ldg(p.la + (((size_t)bb * p.T + t0 + t) * p.H + h) * DK + i);
    G[t] = __expf(g);
  }
  // the last row of the chunk carries dGamma_C (rows past the sequence decay no further)
  float run = p.dgc[((size_t)bh * p.nch + c) * DK + i] * G[BC - 1];
#pragma unroll
  for (int t = BC - 1; t >= 0; --t) {
    if (t >= n) continue;
    const size_t x = (((size_t)bb * p.T + t0 + t) * p.H + h) * DK + i;
    const float kk = ldf(p.k + x), bg = ldf(p.b + x), qq = ldf(p.q + x);
    const float dkb = p.dk[x], dkn = p.db[x], dqh = p.dq[x];
    const float Gt = G[t];
    run += dkb * kk * bg * Gt + dqh * qq * Gt - dkn * kk / Gt;
    dla[x] = run;
    p.dk[x] = dkb * bg * Gt + dkn / Gt;
    p.db[x] = dkb * kk * Gt;
    p.dq[x] = dqh * Gt;
  }
}

template <int DK, bool TC>
constexpr size_t bwd_smem_bytes() {
  constexpr size_t P = pad<TC>(), LK = DK + P, LJ = BJ + P, LC = BC + P;
  return sizeof(float) * (3 * BC * LK + 2 * (size_t)DK * LJ + 3 * BC * LC + 4 * BC * LJ + DK);
}

template <typename T, int DK, int DV>
cudaError_t launch_bwd_t(const ChunkBwdArgs& a, cudaStream_t st) {
  BwdParams<T> p;
  p.q = static_cast<const T*>(a.q);
  p.k = static_cast<const T*>(a.k);
  p.v = static_cast<const T*>(a.v);
  p.b = static_cast<const T*>(a.b);
  p.w = static_cast<const T*>(a.w);
  p.la = a.log_alpha;
  p.S0 = a.S0;
  p.dO = a.dO;
  p.dST = a.dS_T;
  p.dq = a.dq;
  p.dk = a.dk;
  p.db = a.db;
  p.dv = a.dv;
  p.dw = a.dw;
  p.dS0 = a.dS0;
  p.T = a.T;
  p.H = a.H;
  p.nch = (a.T + BC - 1) / BC;
  p.stamps = stamp_buffer();
  const size_t BH = (size_t)a.B * a.H;
  p.states = a.workspace;
  p.dgc = a.workspace + BH * p.nch * DK * DV;
  const size_t tok = (size_t)a.B * a.T * a.H * DK;
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.dq, 0, tok * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dk, 0, tok * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.db, 0, tok * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.dgc, 0, BH * p.nch * DK * sizeof(float), st)) != cudaSuccess) return e;
  // bf16 with d_k = d_v: the entering states from the tensor-core forward's checkpoint phase
  p.states_given = 0;
  if (a.bf16 && DK == DV) {
    ChunkArgs f{a.q, a.k, a.v, a.b, a.w, a.log_alpha, a.S0, nullptr, nullptr, a.B, a.T, a.H, DK, DV, true};
    if ((e = launch_chunk_states_tc(f, p.states, st)) != cudaSuccess) return e;
    p.states_given = 1;
  }
  constexpr size_t smem = bwd_smem_bytes<DK, std::is_same<T, __nv_bfloat16>::value>();
  static_assert(smem <= 227 * 1024, "shared memory of the backward CTA");
  static std::atomic<unsigned long long> attr_done{0};
  if ((e = smem_limit_once(chunk_bwd_kernel<T, DK, DV>, (int)smem, attr_done)) != cudaSuccess) return e;
  constexpr int nth = std::is_same<T, __nv_bfloat16>::value ? 32 * MW : BT;
  chunk_bwd_kernel<T, DK, DV><<<(unsigned)(BH * (DV / BJ)), nth, smem, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  chunk_bwd_finish_kernel<T, DK><<<(unsigned)(BH * p.nch), DK, 0, st>>>(p, a.dlog_alpha);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_dims(const ChunkBwdArgs& a, cudaStream_t st) {
  if (a.dk_ == 128 && a.dv_ == 128) return launch_bwd_t<T, 128, 128>(a, st);
  if (a.dk_ == 128 && a.dv_ == 64) return launch_bwd_t<T, 128, 64>(a, st);
  if (a.dk_ == 64 && a.dv_ == 128) return launch_bwd_t<T, 64, 128>(a, st);
  return launch_bwd_t<T, 64, 64>(a, st);
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
  const size_t nch = (size_t)(T + BC - 1) / BC, BH = (size_t)B * H;
  const size_t warp_mma = sizeof(float) * BH * nch * ((size_t)dk * dv + dk);
  // (the size does not depend on the dtype: d_k = d_v = 128 gets the tensor-core path's)
  if (dk == 128 && dv == 128) {
    const size_t tc = chunk_bwd_tc_workspace_bytes(B, T, H);
    return tc > warp_mma ? tc : warp_mma;
  }
  return warp_mma;
}

cudaError_t launch_chunk_bwd(const ChunkBwdArgs& a, cudaStream_t st) {
  if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
  if (a.bf16 && a.dk_ == 128 && a.dv_ == 128) return launch_chunk_bwd_tc(a, st);
  return a.bf16 ? launch_bwd_dims<__nv_bfloat16>(a, st) : launch_bwd_dims<float>(a, st);
}

}  // namespace gdn2
