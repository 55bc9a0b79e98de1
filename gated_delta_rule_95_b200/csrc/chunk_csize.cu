// Chunkwise prefill forward at a chosen chunk size C = 32, 64 or 128 (bf16 inputs), for
// the chunk-size trade-off study (snilld.dk, "POC-matrix der daekker de haarde hjoerner":
// latency, throughput and peak memory at C = 64 and also 32 and 128).  One kernel
// template covers the three sizes, so they are compared on the same code.
//
// Algorithm: the chunkwise WY form of the Gated DeltaNet-2 guide ("Chunkwise Parallel
// Algorithm for GPU Training") with the cumulative channel-wise decay folded into the
// factors at the chunk start (snilld.dk, "Hvad betyder det for traening og inferens").
// Per chunk of C tokens, entering state S (d_k x d_v), g = in-chunk cumsum of log alpha,
// Gamma = exp(g), rows = tokens:
//     Kb = K*B*Gamma   Kn = K/Gamma   Qh = Q*Gamma   Vw = W*V
//     A  = strictly lower (Kb Kn^T)        P = lower incl. diagonal (Qh Kn^T)
//     U  = (I + A)^-1 (Vw - Kb S)          (block forward substitution, 16-row blocks)
//     O  = Qh S + P U
//     S  = Diag(Gamma_C) (S + Kn^T U)
//
// One CTA of 8 warps (16 at C = 128) owns one (batch, head) and 32 value columns (value
// columns never mix in the recurrence) and walks the chunks in order.  Products run on warp-level tensor-core
// MMAs (m16n8k8, tf32 operands rounded to nearest, fp32 accumulation); the state lives in
// the registers of its owning warps as an fp32 accumulator across chunks, with a tf32 copy
// in shared memory as the operand of the next chunk's products.  The inverse of each 16 x 16
// diagonal block of (I + A) is formed in fp32 by one warp; the off-diagonal substitution
// steps are MMAs.  All tiles are fp32 in shared memory, unpadded, with an XOR swizzle of
// the column (see swz) that keeps every fragment read free of bank conflicts (row-major
// operands are read with ldmatrix); the C x C tile and the two C x d_k tiles set the
// footprint, 231 KB at C = 128, d_k = 128.  Per chunk, log alpha is copied in with 16-byte
// asynchronous copies, its cumsum formed in place, and the bf16 inputs folded in by one
// vectorised pass; Qh is built the same way by the warps that do not run the substitution.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int NV = 32;        // value columns per CTA

// Warps per CTA: 8, or 16 at C = 128, where the shared memory leaves one CTA per SM
template <int C>
struct CsWarps {
  static constexpr int NW = C == 128 ? 16 : 8;
  static constexpr int NTH = 32 * NW;
};

// Element (r, c) of a tile with rows of L floats (L a multiple of 32).  The column is
// XOR-ed with f(r) = 8 (r mod 4) + 4 ((r mod 8) >= 4): the fragment reads of an MMA touch
// either 8 rows x 4 columns (row-major operands) or 4 rows x 8 columns (transposed
// operands), and f maps both patterns onto the 32 banks once each.
template <int L>
__device__ __forceinline__ int swz(int r, int c) {
  return r * L + (c ^ (((r & 3) << 3) | (r & 4)));
}

// four consecutive bf16 (8-byte aligned) as raw bits, and their fp32 values
__device__ __forceinline__ uint2 ld_bf4(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
__device__ __forceinline__ float4 bf4f(uint2 u) {
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}

// Fragment loads for the MMAs, with g = lane / 4 and t = lane % 4 (layout of
// mma_16x8x8_tf32).  A row-major swizzled tile gives an 8 x 4 block of tf32 per 16-byte row
// segment, which is what ldmatrix reads (8 rows of 16 bytes per matrix; lane l receives
// word l % 4 of row l / 4), so a whole A fragment, or the B fragments of two 8-column tiles
// stored as rows (B = X^T), take one ldmatrix.x4 each.  Operands stored the other way round
// ([k][m] or [k][n]) are read as single words; since k advances by 8 and the swizzle only
// depends on the row mod 8, each lane's offsets are fixed and only k * L moves.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const float* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p))
               : "memory");
}
// swizzle term of a row (the row mod 8 decides it)
__device__ __forceinline__ int swf(int r) { return ((r & 3) << 3) | (r & 4); }

// A operand: rows m0 .. m0 + 15 of a row-major tile with rows of L floats, columns k .. k + 7
template <int L>
struct ARow {
  const float* p;  // this lane's ldmatrix row, column 0
  int cx;          // its column offset (0 or 4), to be XOR-ed with the row's swizzle
  int f;
  __device__ __forceinline__ ARow(const float* tile, int m0) {
    const int lane = threadIdx.x & 31, j = lane >> 3, r = m0 + (lane & 7) + 8 * (j & 1);
    p = tile + r * L;
    cx = 4 * (j >> 1);
    f = swf(r);
  }
  __device__ __forceinline__ void load(uint32_t (&a)[4], int k) const { ldsm_x4(a, p + ((k + cx) ^ f)); }
};
// B operand of two 8-column tiles q, q + 1 stored as rows X[n][k] (B = X^T), rows n0 .. n0 + 15
template <int L>
struct BRows {
  const float* p;
  int cx, f;
  __device__ __forceinline__ BRows(const float* tile, int n0) {
    const int lane = threadIdx.x & 31, j = lane >> 3, r = n0 + (lane & 7) + 8 * (j >> 1);
    p = tile + r * L;
    cx = 4 * (j & 1);
    f = swf(r);
  }
  // b0 = {tile q: k + t, k + t + 4}, b1 = the same for tile q + 1
  __device__ __forceinline__ void load(uint32_t (&b0)[2], uint32_t (&b1)[2], int k) const {
    uint32_t r[4];
    ldsm_x4(r, p + ((k + cx) ^ f));
    b0[0] = r[0];
    b0[1] = r[1];
    b1[0] = r[2];
    b1[1] = r[3];
  }
};
// an operand stored [k][c] with rows of L floats, read at (k + t, c0 + g) and (k + t + 4, c0 + g)
// for the 8-column groups c0 = base + 8 q: as a B operand (c = n) or, twice, as a transposed
// A operand (c = m, m + 8)
template <int L, int NQ>
struct KRow {
  const float* p;
  int o0[NQ], o1[NQ];
  __device__ __forceinline__ KRow(const float* tile, int base) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    p = tile + t * L;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      o0[q] = (base + 8 * q + g) ^ swf(t);
      o1[q] = 4 * L + ((base + 8 * q + g) ^ swf(t + 4));
    }
  }
  __device__ __forceinline__ void load(uint32_t (&b)[2], int q, int k) const {
    b[0] = __float_as_uint(p[k * L + o0[q]]);
    b[1] = __float_as_uint(p[k * L + o1[q]]);
  }
};

__device__ __forceinline__ void neg4(uint32_t (&a)[4]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) a[e] ^= 0x80000000u;
}

// d[q] (+)= A B over k in [k0, k1) for the 8-column tiles q < NQ, with A from ARow (negated
// when NEG) and B from KRow
template <int NQ, bool NEG, int LA, int LB>
__device__ __forceinline__ void mma_ak(float (&d)[NQ][4], const ARow<LA>& A, const KRow<LB, NQ>& Bk, int k0, int k1) {
#pragma unroll 2
  for (int k = k0; k < k1; k += 8) {
    uint32_t a[4];
    A.load(a, k);
    if (NEG) neg4(a);
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      uint32_t b[2];
      Bk.load(b, q, k);
      mma_16x8x8_tf32(d[q], a, b);
    }
  }
}
// d[0..1] (+)= A X^T over k in [0, K): a 16 x 16 block, A from ARow, X from BRows
template <int K, int LA, int LB>
__device__ __forceinline__ void mma_ab(float (&d)[2][4], const ARow<LA>& A, const BRows<LB>& X) {
#pragma unroll 4
  for (int k = 0; k < K; k += 8) {
    uint32_t a[4], b0[2], b1[2];
    A.load(a, k);
    X.load(b0, b1, k);
    mma_16x8x8_tf32(d[0], a, b0);
    mma_16x8x8_tf32(d[1], a, b1);
  }
}
// d[q] += A B with A = Y^T read from a [k][m] tile (rows m0 .. m0 + 15) and B from KRow
template <int NQ, int LA, int LB>
__device__ __forceinline__ void mma_kk(float (&d)[NQ][4], const KRow<LA, 2>& At, const KRow<LB, NQ>& Bk, int k0,
                                       int k1) {
#pragma unroll 2
  for (int k = k0; k < k1; k += 8) {
    uint32_t lo[2], hi[2];
    At.load(lo, 0, k);  // (k + t, m0 + g), (k + t + 4, m0 + g)
    At.load(hi, 1, k);  // rows m0 + g + 8
    const uint32_t a[4] = {lo[0], hi[0], lo[1], hi[1]};
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      uint32_t b[2];
      Bk.load(b, q, k);
      mma_16x8x8_tf32(d[q], a, b);
    }
  }
}
// f(row, col, d[q][e]) for every accumulator element of 16 x 8 tiles at (m0, n0 + 8q)
template <int NQ, class F>
__device__ __forceinline__ void for_frag(float (&d)[NQ][4], int m0, int n0, F f) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int q = 0; q < NQ; ++q)
#pragma unroll
    for (int e = 0; e < 4; ++e) f(m0 + g + 8 * (e >> 1), n0 + 8 * q + 2 * t + (e & 1), d[q][e]);
}

struct CsParams {
  const __nv_bfloat16 *q, *k, *v, *b, *w;
  const float* la;
  const float* S0;
  float* o;
  float* S_T;
  int T, H, dv;
};

// shared-memory map, in floats
template <int C, int DK>
struct CsLayout {
  static constexpr int KN = 0;                // Kn [C][DK]
  static constexpr int KQ = KN + C * DK;      // Kb, then Qh [C][DK]
  static constexpr int AP = KQ + C * DK;      // A with (I + A_II)^-1 on its diagonal blocks, then P [C][C]
  static constexpr int UM = AP + C * C;       // Vw, then R, then U [C][NV]
  static constexpr int SM = UM + C * NV;      // state, tf32 copy [DK][NV]
  static constexpr int GC = SM + DK * NV;     // Gamma_C [DK]
  static constexpr int TOT = GC + DK;         // cumsum partials [token range][DK]
  static constexpr int FLOATS = TOT + CsWarps<C>::NTH;
  static constexpr size_t BYTES = FLOATS * sizeof(float);
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

// CTAs per SM that the shared memory admits (d_k = 128), passed to the register allocator
template <int C>
constexpr int csize_min_blocks() { return C == 32 ? 3 : C == 64 ? 2 : 1; }

template <int C, int DK>
__global__ void __launch_bounds__(CsWarps<C>::NTH, csize_min_blocks<C>()) chunk_fwd_csize_kernel(const CsParams p) {
  using Lay = CsLayout<C, DK>;
  constexpr int NW = CsWarps<C>::NW, NTH = CsWarps<C>::NTH;
  constexpr int NB = C / 16;                    // 16-row blocks of a chunk
  constexpr int NBLK = NB * (NB + 1) / 2;       // 16 x 16 blocks on and below the diagonal
  constexpr int SQ = (DK / 16) * (NV / 8) / NW; // state tiles per warp (one row block)
  constexpr int RQ = (C / 16) * (NV / 8) / NW;  // output tiles per warp (C >= 32: >= 1)
  constexpr int PT = NTH / DK, TP = C / PT;     // operand build: threads per key channel, tokens each
  constexpr int QTH = NTH - 32 * (NV / 8) < 2 * DK ? NTH - 32 * (NV / 8) : 2 * DK;  // Qh build: warps
                                                // not in the substitution, at most two per channel
  constexpr int QPT = QTH / DK, QTP = C / QPT;
  constexpr int Q4K = C * DK / 4 / NTH, Q4V = C * NV / 4 / NTH, Q4Q = C * DK / 4 / QTH;  // 4-element groups per thread
  static_assert(Q4K * 4 * NTH == C * DK && Q4V * 4 * NTH == C * NV && Q4Q * 4 * QTH == C * DK, "copy split");
  static_assert((DK / 16) * (NV / 8) % NW == 0 && SQ >= 1 && SQ <= NV / 8, "state tiles: one row block per warp");
  static_assert((C / 16) * (NV / 8) % NW == 0 && RQ >= 1 && RQ <= NV / 8, "output tiles: one row block per warp");
  static_assert(QPT >= 1 && QTH % DK == 0 && QTH % 32 == 0 && C % QPT == 0, "Qh build threads");
  static_assert(NB <= NW, "one warp per diagonal block");

  extern __shared__ __align__(16) float sm[];
  float* Kn = sm + Lay::KN;
  float* KQ = sm + Lay::KQ;
  float* AP = sm + Lay::AP;
  float* Um = sm + Lay::UM;
  float* Sm = sm + Lay::SM;
  float* gC = sm + Lay::GC;
  float* tot = sm + Lay::TOT;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nsl = p.dv / NV;
  const int bh = blockIdx.x / nsl, j0 = (blockIdx.x % nsl) * NV;
  const int h = bh % p.H, bb = bh / p.H;
  auto tok = [&](int t) { return ((size_t)bb * p.T + t) * p.H + h; };  // (token, head) row

  // this warp's state tiles (fp32 accumulators for the whole sequence) and output tiles
  const int s_m0 = 16 * (warp * SQ / (NV / 8)), s_n0 = 8 * (warp * SQ % (NV / 8));
  const int r_m0 = 16 * (warp * RQ / (NV / 8)), r_n0 = 8 * (warp * RQ % (NV / 8));
  float Sacc[SQ][4];
  for_frag<SQ>(Sacc, s_m0, s_n0, [&](int i, int j, float& x) {
    x = p.S0 ? __ldg(p.S0 + ((size_t)bh * DK + i) * p.dv + j0 + j) : 0.f;
  });

  const int ci = tid % DK, part = tid / DK;  // operand build: key channel, token range
  const int nch = (p.T + C - 1) / C;
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * C, n = min(C, p.T - t0);
    // (0) tf32 copy of the state (nobody reads it until the next barrier)
    for_frag<SQ>(Sacc, s_m0, s_n0, [&](int i, int j, float& x) { Sm[swz<NV>(i, j)] = to_tf32(x); });
    // (1) log alpha of the chunk into the Kn tile (16-byte asynchronous copies, rows past the
    // sequence zero-filled); Vw into the U tile; four channels per thread and copy
    {
#pragma unroll
      for (int m = 0; m < Q4K; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
        cp_async16(Kn + swz<DK>(t, i), p.la + (t < n ? tok(t0 + t) * DK + i : 0), t < n);
      }
      uint2 w4[Q4V], v4[Q4V];
#pragma unroll
      for (int m = 0; m < Q4V; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (NV / 4), j = 4 * (e4 % (NV / 4));
        w4[m] = v4[m] = make_uint2(0u, 0u);
        if (t < n) {
          const size_t off = tok(t0 + t) * p.dv + j0 + j;
          w4[m] = ld_bf4(p.w + off);
          v4[m] = ld_bf4(p.v + off);
        }
      }
#pragma unroll
      for (int m = 0; m < Q4V; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (NV / 4), j = 4 * (e4 % (NV / 4));
        const float4 a = bf4f(w4[m]), b = bf4f(v4[m]);
        *reinterpret_cast<float4*>(Um + swz<NV>(t, j)) = make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
      }
      cp_async_wait_all();
    }
    __syncthreads();
    // (2) g = in-chunk cumsum of log alpha, in place: partial sums per (channel, token
    // range), then the running sums; Gamma_C
    {
      float s = 0.f;
#pragma unroll 8
      for (int t = part * TP; t < (part + 1) * TP; ++t) s += Kn[swz<DK>(t, ci)];
      tot[part * DK + ci] = s;
    }
    __syncthreads();
    {
      float gg = 0.f;
      for (int q = 0; q < part; ++q) gg += tot[q * DK + ci];
#pragma unroll 8
      for (int t = part * TP; t < (part + 1) * TP; ++t) {
        gg += Kn[swz<DK>(t, ci)];
        Kn[swz<DK>(t, ci)] = gg;
      }
      if (part == PT - 1) gC[ci] = __expf(gg);
    }
    __syncthreads();
    // Kb = K*B*Gamma into KQ and Kn = K/Gamma over g (rows past the sequence: k = 0)
    {
      uint2 k4[Q4K], b4[Q4K];
#pragma unroll
      for (int m = 0; m < Q4K; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
        k4[m] = b4[m] = make_uint2(0u, 0u);
        if (t < n) {
          const size_t off = tok(t0 + t) * DK + i;
          k4[m] = ld_bf4(p.k + off);
          b4[m] = ld_bf4(p.b + off);
        }
      }
#pragma unroll
      for (int m = 0; m < Q4K; ++m) {
        const int e4 = tid + NTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
        float4* gp = reinterpret_cast<float4*>(Kn + swz<DK>(t, i));
        const float4 gv = *gp, kk = bf4f(k4[m]), bb4 = bf4f(b4[m]);
        *gp = make_float4(to_tf32(kk.x * __expf(-gv.x)), to_tf32(kk.y * __expf(-gv.y)),
                          to_tf32(kk.z * __expf(-gv.z)), to_tf32(kk.w * __expf(-gv.w)));
        *reinterpret_cast<float4*>(KQ + swz<DK>(t, i)) =
            make_float4(to_tf32(kk.x * bb4.x * __expf(gv.x)), to_tf32(kk.y * bb4.y * __expf(gv.y)),
                        to_tf32(kk.z * bb4.z * __expf(gv.z)), to_tf32(kk.w * bb4.w * __expf(gv.w)));
      }
    }
    __syncthreads();
    // (3) A (blocks on and below the diagonal; the diagonal blocks kept in fp32 for the
    // inversion) and R = Vw - Kb S
    for (int blk = warp; blk < NBLK; blk += NW) {
      int mb = 0;
      while ((mb + 1) * (mb + 2) / 2 <= blk) ++mb;
      const int jb = blk - mb * (mb + 1) / 2;
      float d[2][4] = {};
      mma_ab<DK>(d, ARow<DK>(KQ, 16 * mb), BRows<DK>(Kn, 16 * jb));
      for_frag<2>(d, 16 * mb, 16 * jb, [&](int m, int s, float& x) {
        AP[swz<C>(m, s)] = s < m ? (jb == mb ? x : to_tf32(x)) : 0.f;
      });
    }
    {
      float d[RQ][4];
      for_frag<RQ>(d, r_m0, r_n0, [&](int t, int j, float& x) { x = Um[swz<NV>(t, j)]; });
      mma_ak<RQ, true>(d, ARow<DK>(KQ, r_m0), KRow<NV, RQ>(Sm, r_n0), 0, DK);
      for_frag<RQ>(d, r_m0, r_n0, [&](int t, int j, float& x) { Um[swz<NV>(t, j)] = x; });
    }
    __syncthreads();
    // (4a) T_II = (I + A_II)^-1 for every diagonal block, one warp each: lane j (and j + 16)
    // forms column j by forward substitution in fp32
    if (warp < NB) {
      const int base = 16 * warp, j = lane & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = r == j ? 1.f : 0.f;
#pragma unroll
        for (int s = 0; s < r; ++s) acc = fmaf(-AP[swz<C>(base + r, base + s)], x[s], acc);
        x[r] = acc;
      }
      __syncwarp();
      if (lane < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) AP[swz<C>(base + r, base + j)] = to_tf32(x[r]);
      }
    }
    __syncthreads();
    // (4b) U = (I + A)^-1 R by 16-row blocks: X_I = R_I - sum_{J<I} A_IJ U_J, U_I = T_II X_I.
    // Warp w < NV/8 owns value columns 8w .. 8w + 7 throughout; the other warps build Qh.
    if (warp < NV / 8) {
      const int n0 = 8 * warp;
      for (int mb = 0; mb < NB; ++mb) {
        const int m0 = 16 * mb;
        float d[1][4];
        for_frag<1>(d, m0, n0, [&](int t, int j, float& x) { x = Um[swz<NV>(t, j)]; });
        mma_ak<1, true>(d, ARow<C>(AP, m0), KRow<NV, 1>(Um, n0), 0, m0);
        for_frag<1>(d, m0, n0, [&](int t, int j, float& x) { Um[swz<NV>(t, j)] = to_tf32(x); });
        __syncwarp();
        float e[1][4] = {};
        mma_ak<1, false>(e, ARow<C>(AP, m0), KRow<NV, 1>(Um, n0), m0, m0 + 16);
        __syncwarp();
        for_frag<1>(e, m0, n0, [&](int t, int j, float& x) { Um[swz<NV>(t, j)] = to_tf32(x); });
        __syncwarp();
      }
    } else if (tid - 32 * (NV / 8) < QTH) {
      // Qh = Q*Gamma into KQ (free since the A and R products): log alpha copied in, its
      // cumsum formed in place, then multiplied out; barrier 1 spans these warps only
      const int qt = tid - 32 * (NV / 8), qi = qt % DK, qp = qt / DK;
#pragma unroll
      for (int m = 0; m < Q4Q; ++m) {
        const int e4 = qt + QTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
        cp_async16(KQ + swz<DK>(t, i), p.la + (t < n ? tok(t0 + t) * DK + i : 0), t < n);
      }
      uint2 q4[Q4Q];
#pragma unroll
      for (int m = 0; m < Q4Q; ++m) {
        const int e4 = qt + QTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
        q4[m] = t < n ? ld_bf4(p.q + tok(t0 + t) * DK + i) : make_uint2(0u, 0u);
      }
      cp_async_wait_all();
      named_bar_sync(1, QTH);
      float gg = 0.f;
      if constexpr (QPT > 1) {
        float s = 0.f;
        for (int t = qp * QTP; t < (qp + 1) * QTP; ++t) s += KQ[swz<DK>(t, qi)];
        tot[qp * DK + qi] = s;
        named_bar_sync(1, QTH);
        for (int q = 0; q < qp; ++q) gg += tot[q * DK + qi];
      }
#pragma unroll 8
      for (int t = qp * QTP; t < (qp + 1) * QTP; ++t) {
        gg += KQ[swz<DK>(t, qi)];
        KQ[swz<DK>(t, qi)] = gg;
      }
      named_bar_sync(1, QTH);
#pragma unroll
      for (int m = 0; m < Q4Q; ++m) {
        const int e4 = qt + QTH * m, t = e4 / (DK / 4), i = 4 * (e4 % (DK / 4));
        float4* gp = reinterpret_cast<float4*>(KQ + swz<DK>(t, i));
        const float4 gv = *gp, qq = bf4f(q4[m]);
        *gp = make_float4(to_tf32(qq.x * __expf(gv.x)), to_tf32(qq.y * __expf(gv.y)), to_tf32(qq.z * __expf(gv.z)),
                          to_tf32(qq.w * __expf(gv.w)));
      }
    }
    __syncthreads();
    // (5) P over the A tile; the inter-chunk part of the output, Qh S, into registers
    for (int blk = warp; blk < NBLK; blk += NW) {
      int mb = 0;
      while ((mb + 1) * (mb + 2) / 2 <= blk) ++mb;
      const int jb = blk - mb * (mb + 1) / 2;
      float d[2][4] = {};
      mma_ab<DK>(d, ARow<DK>(KQ, 16 * mb), BRows<DK>(Kn, 16 * jb));
      for_frag<2>(d, 16 * mb, 16 * jb, [&](int m, int s, float& x) { AP[swz<C>(m, s)] = s <= m ? to_tf32(x) : 0.f; });
    }
    float Oacc[RQ][4] = {};
    mma_ak<RQ, false>(Oacc, ARow<DK>(KQ, r_m0), KRow<NV, RQ>(Sm, r_n0), 0, DK);
    __syncthreads();
    // (6) O += P U and store; S = Diag(Gamma_C) (S + Kn^T U)
    mma_ak<RQ, false>(Oacc, ARow<C>(AP, r_m0), KRow<NV, RQ>(Um, r_n0), 0, r_m0 + 16);
#pragma unroll
    for (int q = 0; q < RQ; ++q)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int g = lane >> 2, t4 = lane & 3, t = r_m0 + g + 8 * hf;
        if (t < n)
          *reinterpret_cast<float2*>(p.o + tok(t0 + t) * p.dv + j0 + r_n0 + 8 * q + 2 * t4) =
              make_float2(Oacc[q][2 * hf], Oacc[q][2 * hf + 1]);
      }
    mma_kk<SQ>(Sacc, KRow<DK, 2>(Kn, s_m0), KRow<NV, SQ>(Um, s_n0), 0, C);
    for_frag<SQ>(Sacc, s_m0, s_n0, [&](int i, int, float& x) { x *= gC[i]; });
    __syncthreads();
  }
  if (p.S_T) {
    for_frag<SQ>(Sacc, s_m0, s_n0, [&](int i, int j, float& x) {
      p.S_T[((size_t)bh * DK + i) * p.dv + j0 + j] = x;
    });
  }
}

template <int C, int DK>
cudaError_t launch_c(const ChunkArgs& a, cudaStream_t st) {
  const size_t smem = CsLayout<C, DK>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(chunk_fwd_csize_kernel<C, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  CsParams p{static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
             static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.b),
             static_cast<const __nv_bfloat16*>(a.w), a.log_alpha, a.S0, a.o, a.S_T, a.T, a.H, a.dv};
  const long long grid = (long long)a.B * a.H * (a.dv / NV);
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  chunk_fwd_csize_kernel<C, DK><<<(unsigned)grid, CsWarps<C>::NTH, smem, st>>>(p);
  return cudaGetLastError();
}

template <int C>
cudaError_t launch_dk(const ChunkArgs& a, cudaStream_t st) {
  return a.dk == 128 ? launch_c<C, 128>(a, st) : launch_c<C, 64>(a, st);
}

}  // namespace

// The chunk-size study's entry: C = 32 and C = 64 on the tcgen05 kernels (chunk_tc32.cu and
// the production chunk_tc.cu), C = 128 on this warp-MMA kernel (its tiles exceed one SM's
// shared and tensor memory on tcgen05).
size_t chunk_fwd_csize_smem_bytes(int chunk, int dk) {
  if (dk != 64 && dk != 128) return 0;
  switch (chunk) {
    case 32: return chunk_fwd_tc32_smem_bytes();
    case 64: return chunk_fwd_tc_smem_bytes();
    case 128: return dk == 128 ? CsLayout<128, 128>::BYTES : CsLayout<128, 64>::BYTES;
    default: return 0;
  }
}

cudaError_t launch_chunk_fwd_csize(const ChunkArgs& a, int chunk, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  switch (chunk) {
    case 32: return launch_chunk_fwd_tc32(a, st);
    case 64: return launch_chunk_fwd_tc(a, st);
    case 128: return launch_dk<128>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gdn2
