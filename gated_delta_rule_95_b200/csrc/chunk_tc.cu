// Chunkwise prefill forward for bf16 inputs on the 5th-generation tensor cores
// (tcgen05.mma kind::tf32, accumulators and the running state in tensor memory).
//
// Algorithm (Gated DeltaNet-2 guide, "Chunkwise Parallel Algorithm for GPU
// Training"; WY form with the cumulative channel-wise decay folded into the
// factors of each rank-one erase, snilld.dk, "Hvad betyder det for traening og
// inferens").  Per (batch, head), chunks of C = 64 tokens in order, entering
// state S (d_k x d_v, fp32).  With g = in-chunk cumsum of log alpha and
// Gamma = exp(g) (chunk-start reference):
//
//     Kb = K*B*Gamma    Qh = Q*Gamma    Kn = K/Gamma    Vw = W*V
//     [A; P]  = [Kb; Qh] Kn^T           A strictly lower, P lower incl. diagonal
//     T       = (I + A)^-1              blocked triangular inverse, fp32
//     U^T     = Vw^T T^T                W^T = Kb^T T^T
//     U~^T    = U^T - S^T W^T           (= (U - W S)^T, the erase-corrected writes)
//     O^T     = S^T Qh^T + U~^T P^T
//     S^T    <- (S^T + U~^T Kn) Diag(Gamma_C)
//
// All products run as kind::tf32 MMAs with M = 128 (tokens of [Kb; Qh], or the
// d_k / d_v axis of the transposed products), every operand K-major.  The state
// is kept transposed, S^T (rows = value channels), as an fp32 accumulator in
// tensor memory and fed straight back as the A operand of the next chunk's
// products; so is U~^T.  Kb^T and Vw^T, the A operands of the products over
// tokens, are written into tensor memory by a thread-per-channel pass that runs
// while the first product is on the tensor cores; Kn^T is its shared-memory twin.
// Shared-memory and written tensor-memory operands are rounded to tf32 (nearest);
// the accumulators S^T and U~^T are read by the tensor core at tf32 precision.
//
// One CTA (256 threads, 8 warps) owns one (batch, head) and walks its chunks.
// Thread 0 issues TMA and MMAs; all warps do the elementwise work.  The raw bf16
// inputs of chunk c+1 are prefetched into L2 while chunk c runs, and its
// log-alpha tile is loaded by TMA into shared memory.
// d_k or d_v = 64 run the same code with the upper half of each operand zero.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 64;
constexpr int NT = 256;
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait

// ---- shared memory map (byte offsets from a 1024-byte aligned base) ----------------
// fp32 operand tiles with the 128B swizzle, in panels of 32 columns (128 B rows).
constexpr uint32_t R64 = 64 * 128;    // a panel of 64 rows  (8 KB)
constexpr uint32_t R128 = 128 * 128;  // a panel of 128 rows (16 KB)
constexpr uint32_t OFF_KQ = 0;                  // [Kb; Qh] [t][i]: 4 panels x 128 rows
constexpr uint32_t OFF_KN = OFF_KQ + 4 * R128;  // Kn [s][i]: 4 panels x 64 rows; later W [t][i]
constexpr uint32_t OFF_KNT = OFF_KN + 4 * R64;  // Kn^T [i][s]: 2 panels x 128 rows
constexpr uint32_t OFF_T = OFF_KNT + 2 * R128;  // T [t][s]: 2 panels x 64 rows (first: Vw [t][j], 32 KB over T and P)
constexpr uint32_t OFF_P = OFF_T + 2 * R64;     // P [t][s]: 2 panels x 64 rows
constexpr uint32_t OFF_LA = OFF_P + 2 * R64;    // log alpha [64][d_k] fp32 (TMA), cumsum in place
constexpr uint32_t OFF_SCR = OFF_LA + 32768;    // solve scratch: fp32 64 x LDM, then 16 x 48
constexpr uint32_t TILES = OFF_SCR + 20480;     // 212 KB

struct Misc {
  uint64_t bar_la, bar_mma;
  uint32_t tmem_base;
  int abort;
  float gC[128];     // Gamma at the chunk end, per key channel
  float half0[128];  // sum of log alpha over the first 32 tokens, per key channel
};
constexpr uint32_t SMEM_BYTES = TILES + 1024 + sizeof(Misc);

// ---- tensor memory columns (fp32, 128 lanes) -------------------------------------------
constexpr uint32_t TM_AP = 0;     // [A; P], later W^T   lanes: tokens of Kb | Qh (key channel for W^T)
constexpr uint32_t TM_W = 0;
constexpr uint32_t TM_U = 64;     // U^T, then U~^T      lanes: value channel, columns: s
constexpr uint32_t TM_O = 128;    // O^T                 lanes: value channel, columns: t
constexpr uint32_t TM_S = 192;    // S^T (the state)     lanes: value channel, columns: key channel
constexpr uint32_t TM_KBT = 320;  // Kb^T                lanes: key channel,   columns: s
constexpr uint32_t TM_VWT = 384;  // Vw^T                lanes: value channel, columns: s
constexpr uint32_t TM_COLS = 512;

// instruction descriptors (M = 128, both operands K-major)
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);
constexpr uint32_t ID_64NEG = idesc_tf32(128, 64, 0, 0, 0, 1);  // B negated
constexpr uint32_t ID_128 = idesc_tf32(128, 128, 0, 0, 0, 0);

// fp32 scratch of the triangular solve: a 64 x 64 matrix with rows padded to 68
// floats (16-byte aligned rows that start 4 banks apart).  It first holds A
// (strictly lower, zero elsewhere) and is overwritten block-row by block-row
// with T = (I + A)^-1 (unit lower triangular, explicit zeros above).
constexpr int LDM = 68;

struct TcParams {
  const __nv_bfloat16 *q, *k, *v, *b, *w;
  const float* S0;
  float* S_T;
  float* o;
  int T, H, dk, dv, nchunks;
  unsigned* err;
};

__device__ __forceinline__ void st4_tf32(unsigned char* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(to_tf32(f[0]), to_tf32(f[1]), to_tf32(f[2]), to_tf32(f[3]));
}

__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmLA,
                        const TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  // 128B-swizzled tiles need 1024-byte aligned shared addresses
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Misc& ms = *reinterpret_cast<Misc*>(sm + TILES);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;  // TMEM lane quadrant, column half
  const int unit = blockIdx.x, bb = unit / p.H, h = unit % p.H;
  const int dk = p.dk, dv = p.dv;

  if (tid == 0) {
    mbar_init(&ms.bar_la, 1);
    mbar_init(&ms.bar_mma, 1);
    fence_mbar_init();
    ms.abort = 0;
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmB); tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmLA);
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  const uint32_t tlane = tmem + ((uint32_t)(32 * qd) << 16);

  // ---- async copies (thread 0) ---------------------------------------------------------
  int pend_la = 0, pend_mma = 0;
  auto prefetch_raw = [&](int c) {  // raw bf16 inputs of chunk c into L2
    for (int pn = 0; pn < (dk >> 6); ++pn) {
      tma_prefetch_l2_4d(&tmQ, 64 * pn, h, C * c, bb);
      tma_prefetch_l2_4d(&tmK, 64 * pn, h, C * c, bb);
      tma_prefetch_l2_4d(&tmB, 64 * pn, h, C * c, bb);
    }
    for (int pn = 0; pn < (dv >> 6); ++pn) {
      tma_prefetch_l2_4d(&tmV, 64 * pn, h, C * c, bb);
      tma_prefetch_l2_4d(&tmW, 64 * pn, h, C * c, bb);
    }
  };
  auto issue_la = [&](int c) {
    mbar_arrive_expect_tx(&ms.bar_la, (uint32_t)(C * dk * 4));
    tma_load_4d(sm + OFF_LA, &tmLA, &ms.bar_la, 0, h, C * c, bb);
    pend_la = 1;
  };
  if (tid == 0 && p.nchunks > 0) {
    prefetch_raw(0);
    issue_la(0);
  }

  // ---- entering state S0 -> S^T in tensor memory -----------------------------------------
  // Thread (qd, hf, lane) owns lane j = 32 qd + lane (a value channel) and the key-channel
  // columns [64 hf, 64 hf + 64) of S^T.
  const int jrow = 32 * qd + lane;
  {
    const bool ok = p.S0 && jrow < dv;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int i = 64 * hf + 32 * half + x;
        v[x] = (ok && i < dk) ? p.S0[((size_t)unit * dk + i) * dv + jrow] : 0.f;
      }
      tmem_st32(tlane + TM_S + 64 * hf + 32 * half, v);
    }
    tmem_st_wait();
  }

  uint32_t ph_la = 0, ph_mma = 0;
  float* Msc = reinterpret_cast<float*>(sm + OFF_SCR);                  // solve matrix, 64 x LDM fp32
  float* Xsc = reinterpret_cast<float*>(sm + OFF_SCR + 64 * LDM * 4);   // block-row product, 16 x 48 fp32
  float* la = reinterpret_cast<float*>(sm + OFF_LA);

  auto wait_on = [&](uint64_t* bar, uint32_t& ph, int& pend) -> bool {
    const bool ok = mbar_wait_bounded(bar, ph, &ms.abort, p.err, WAIT_LIMIT);
    if (ok) {
      ph ^= 1;
      if (tid == 0) pend = 0;
    }
    return ok;
  };
  auto wait_mma = [&]() -> bool { return wait_on(&ms.bar_mma, ph_mma, pend_mma); };
  auto commit_mma = [&]() {
    umma_commit(&ms.bar_mma);
    pend_mma = 1;
  };
  tc_fence_before();
  __syncthreads();

  for (int c = 0; c < p.nchunks; ++c) {
    const int t0 = C * c, n = min(C, p.T - t0);
    if (tid == 0 && c + 1 < p.nchunks) prefetch_raw(c + 1);
    // ===== raw inputs of this chunk: issue the global loads first ==========================
    // Thread (cg, tg): channels [8 cg, 8 cg + 8) (16 bytes of bf16), tokens tg + 16 r.
    const int cg = tid & 15, tg = tid >> 4, c0 = 8 * cg;
    const bool kval = c0 < dk, vval = c0 < dv;
    uint4 rq[4], rk[4], rb[4], rv[4], rw[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = tg + 16 * r;
      const bool in = t < n;
      const size_t tok = ((size_t)bb * p.T + t0 + t) * p.H + h;
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      rq[r] = (in && kval) ? __ldg(reinterpret_cast<const uint4*>(p.q + tok * dk + c0)) : z;
      rk[r] = (in && kval) ? __ldg(reinterpret_cast<const uint4*>(p.k + tok * dk + c0)) : z;
      rb[r] = (in && kval) ? __ldg(reinterpret_cast<const uint4*>(p.b + tok * dk + c0)) : z;
      rv[r] = (in && vval) ? __ldg(reinterpret_cast<const uint4*>(p.v + tok * dv + c0)) : z;
      rw[r] = (in && vval) ? __ldg(reinterpret_cast<const uint4*>(p.w + tok * dv + c0)) : z;
    }
    // ===== decay cumsum, in place in the log-alpha tile ======================================
    {
      const bool ok = wait_on(&ms.bar_la, ph_la, pend_la);
      if (__syncthreads_or(!ok)) break;
    }
    {
      // thread (ch, half) owns key channel ch and tokens [32 half, 32 half + 32)
      const int ch = tid & 127, half = tid >> 7;
      if (ch < dk && half == 0) {
        float tot = 0.f;
#pragma unroll 8
        for (int t = 0; t < 32; ++t) tot += la[t * dk + ch];
        ms.half0[ch] = tot;
      }
      __syncthreads();
      float g = 0.f;
      if (ch < dk) {
        g = half ? ms.half0[ch] : 0.f;
#pragma unroll 8
        for (int tt = 0; tt < 32; ++tt) {
          const int idx = (32 * half + tt) * dk + ch;
          g += la[idx];
          la[idx] = g;
        }
      }
      if (half == 1) ms.gC[ch] = ch < dk ? __expf(g) : 0.f;
    }
    __syncthreads();
    // ===== folded operands: Kb, Qh, Kn, Vw (fp32, rounded to tf32) ===========================
    {
      float gv[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = tg + 16 * r;
        if (kval) {
          const float4 a = *reinterpret_cast<const float4*>(la + t * dk + c0);
          const float4 e = *reinterpret_cast<const float4*>(la + t * dk + c0 + 4);
          gv[r][0] = a.x; gv[r][1] = a.y; gv[r][2] = a.z; gv[r][3] = a.w;
          gv[r][4] = e.x; gv[r][5] = e.y; gv[r][6] = e.z; gv[r][7] = e.w;
        } else {
#pragma unroll
          for (int m = 0; m < 8; ++m) gv[r][m] = 0.f;
        }
      }
      fence_proxy_async_smem();
      __syncthreads();  // the log-alpha tile is free: load the next chunk's
      if (tid == 0 && c + 1 < p.nchunks) issue_la(c + 1);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = tg + 16 * r;
        float kb[8], qh[8], kn[8], vw[8];
        {
          float kk[8], bgt[8], qq[8], vv[8], ww[8];
          unpack_bf16x8(rk[r], kk);
          unpack_bf16x8(rb[r], bgt);
          unpack_bf16x8(rq[r], qq);
          unpack_bf16x8(rv[r], vv);
          unpack_bf16x8(rw[r], ww);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float G = __expf(gv[r][m]), Gi = __expf(-gv[r][m]);
            kb[m] = kk[m] * bgt[m] * G;
            qh[m] = qq[m] * G;
            kn[m] = kk[m] * Gi;
            vw[m] = ww[m] * vv[m];
          }
        }
        st4_tf32(sm + OFF_KQ + f32_off(t, c0, R128), kb);
        st4_tf32(sm + OFF_KQ + f32_off(t, c0 + 4, R128), kb + 4);
        st4_tf32(sm + OFF_KQ + f32_off(64 + t, c0, R128), qh);
        st4_tf32(sm + OFF_KQ + f32_off(64 + t, c0 + 4, R128), qh + 4);
        st4_tf32(sm + OFF_KN + f32_off(t, c0, R64), kn);
        st4_tf32(sm + OFF_KN + f32_off(t, c0 + 4, R64), kn + 4);
        st4_tf32(sm + OFF_T + f32_off(t, c0, R64), vw);
        st4_tf32(sm + OFF_T + f32_off(t, c0 + 4, R64), vw + 4);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // [A; P] = [Kb; Qh] Kn^T : M=128 (tokens of both halves), N=64 (s), K=128 (key channels)
      // O^T    = S^T Qh^T      : A = S^T from tensor memory, B = Qh rows of the KQ tile
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t ko = (uint32_t)((ks & 3) * 32);
        const uint64_t aKQ = sdesc_sw128(sbase + OFF_KQ + (ks >> 2) * R128 + ko, 16, 1024);
        const uint64_t bKN = sdesc_sw128(sbase + OFF_KN + (ks >> 2) * R64 + ko, 16, 1024);
        umma_tf32_ss(tmem + TM_AP, aKQ, bKN, ID_64, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t ko = (uint32_t)((ks & 3) * 32);
        const uint64_t bQH = sdesc_sw128(sbase + OFF_KQ + (ks >> 2) * R128 + R64 + ko, 16, 1024);
        umma_tf32_ts(tmem + TM_O, tmem + TM_S + 8 * ks, bQH, ID_64, ks > 0);
      }
      commit_mma();
    }
    // ===== transposed operands while the tensor cores run: Kb^T, Vw^T into tensor
    // memory (lane = channel), Kn^T into shared memory (row = key channel) ============
    {
      const int ch = tid & 127;  // also this thread's tensor-memory lane (warp quadrant)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float v[32];
        if (tid < 128) {
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = *reinterpret_cast<const float*>(sm + OFF_KQ + f32_off(32 * hh + x, ch, R128));
          tmem_st32(tlane + TM_KBT + 32 * hh, v);
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = *reinterpret_cast<const float*>(sm + OFF_KN + f32_off(32 * hh + x, ch, R64));
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(sm + OFF_KNT + f32_off(ch, 32 * hh + x, R128)) =
                make_float4(v[x], v[x + 1], v[x + 2], v[x + 3]);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = *reinterpret_cast<const float*>(sm + OFF_T + f32_off(32 * hh + x, ch, R64));
          tmem_st32(tlane + TM_VWT + 32 * hh, v);
        }
      }
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    // ===== A to the solve scratch, P to its operand tile =====================================
    {
      float v[32];
      tmem_ld32(tlane + TM_AP + 32 * hf, v);
      tmem_ld_wait();
      if (qd < 2) {
        const int t = 32 * qd + lane;
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const int s = 32 * hf + x;
          float4 f;
          f.x = (s + 0 < t) ? v[x + 0] : 0.f;
          f.y = (s + 1 < t) ? v[x + 1] : 0.f;
          f.z = (s + 2 < t) ? v[x + 2] : 0.f;
          f.w = (s + 3 < t) ? v[x + 3] : 0.f;
          *reinterpret_cast<float4*>(Msc + t * LDM + s) = f;
        }
      } else {
        const int t = 32 * (qd - 2) + lane;  // P row, causal incl. diagonal
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          float f[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) f[m] = (32 * hf + x + m <= t) ? v[x + m] : 0.f;
          st4_tf32(sm + OFF_P + f32_off(t, 32 * hf + x, R64), f);
        }
      }
    }
    __syncthreads();
    // ===== T = (I + A)^-1 by 16-row blocks ==============================================
    // Diagonal blocks T_II = (I + A_II)^-1 by forward substitution, one column per thread.
    {
      float x[16];
      const int I = tid >> 4, cc = tid & 15;
      if (tid < 64) {
        const float* Ab = Msc + 16 * I * LDM + 16 * I;
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
          float acc = 0.f;
#pragma unroll
          for (int s4 = 0; s4 < r; s4 += 4) {
            const float4 a = *reinterpret_cast<const float4*>(Ab + r * LDM + s4);
            acc = fmaf(a.x, x[s4], acc);
            if (s4 + 1 < r) acc = fmaf(a.y, x[s4 + 1], acc);
            if (s4 + 2 < r) acc = fmaf(a.z, x[s4 + 2], acc);
            if (s4 + 3 < r) acc = fmaf(a.w, x[s4 + 3], acc);
          }
          x[r] = (r > cc) ? -acc : x[r];
        }
      }
      __syncthreads();
      if (tid < 64) {
        float* Tb = Msc + 16 * I * LDM + 16 * I;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * LDM + cc] = x[r];
      }
      __syncthreads();
    }
    // Block rows I = 1..3:  T_I,<I = -T_II (A_I,<I T_<I,<I); every entry above the
    // diagonal is an explicit zero, so the products run over full ranges.  Thread
    // (r, c4) computes four adjacent columns of a row.
#pragma unroll
    for (int I = 1; I < 4; ++I) {
      const int nq = 4 * I;  // float4 columns in the block row
      for (int e = tid; e < 16 * nq; e += NT) {
        const int r = e / nq, c4 = e % nq;
        const float* Arow = Msc + (16 * I + r) * LDM;
        float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int k4 = 0; k4 < 16 * I; k4 += 4) {
          const float4 a = *reinterpret_cast<const float4*>(Arow + k4);
          const float4 t0v = *reinterpret_cast<const float4*>(Msc + (k4 + 0) * LDM + 4 * c4);
          const float4 t1v = *reinterpret_cast<const float4*>(Msc + (k4 + 1) * LDM + 4 * c4);
          const float4 t2v = *reinterpret_cast<const float4*>(Msc + (k4 + 2) * LDM + 4 * c4);
          const float4 t3v = *reinterpret_cast<const float4*>(Msc + (k4 + 3) * LDM + 4 * c4);
          z.x = fmaf(a.x, t0v.x, fmaf(a.y, t1v.x, fmaf(a.z, t2v.x, fmaf(a.w, t3v.x, z.x))));
          z.y = fmaf(a.x, t0v.y, fmaf(a.y, t1v.y, fmaf(a.z, t2v.y, fmaf(a.w, t3v.y, z.y))));
          z.z = fmaf(a.x, t0v.z, fmaf(a.y, t1v.z, fmaf(a.z, t2v.z, fmaf(a.w, t3v.z, z.z))));
          z.w = fmaf(a.x, t0v.w, fmaf(a.y, t1v.w, fmaf(a.z, t2v.w, fmaf(a.w, t3v.w, z.w))));
        }
        *reinterpret_cast<float4*>(Xsc + r * 48 + 4 * c4) = z;
      }
      __syncthreads();
      for (int e = tid; e < 16 * nq; e += NT) {
        const int r = e / nq, c4 = e % nq;
        const float* Trow = Msc + (16 * I + r) * LDM + 16 * I;
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int s4 = 0; s4 < 16; s4 += 4) {
          const float4 tr = *reinterpret_cast<const float4*>(Trow + s4);
          const float4 x0 = *reinterpret_cast<const float4*>(Xsc + (s4 + 0) * 48 + 4 * c4);
          const float4 x1 = *reinterpret_cast<const float4*>(Xsc + (s4 + 1) * 48 + 4 * c4);
          const float4 x2 = *reinterpret_cast<const float4*>(Xsc + (s4 + 2) * 48 + 4 * c4);
          const float4 x3 = *reinterpret_cast<const float4*>(Xsc + (s4 + 3) * 48 + 4 * c4);
          y.x = fmaf(tr.x, x0.x, fmaf(tr.y, x1.x, fmaf(tr.z, x2.x, fmaf(tr.w, x3.x, y.x))));
          y.y = fmaf(tr.x, x0.y, fmaf(tr.y, x1.y, fmaf(tr.z, x2.y, fmaf(tr.w, x3.y, y.y))));
          y.z = fmaf(tr.x, x0.z, fmaf(tr.y, x1.z, fmaf(tr.z, x2.z, fmaf(tr.w, x3.z, y.z))));
          y.w = fmaf(tr.x, x0.w, fmaf(tr.y, x1.w, fmaf(tr.z, x2.w, fmaf(tr.w, x3.w, y.w))));
        }
        *reinterpret_cast<float4*>(Msc + (16 * I + r) * LDM + 4 * c4) = make_float4(-y.x, -y.y, -y.z, -y.w);
      }
      __syncthreads();
    }
    // T as a tf32 K-major operand [t][s]
    for (int e = tid; e < 64 * 16; e += NT) {
      const int t = e >> 4, s4 = e & 15;
      const float4 a = *reinterpret_cast<const float4*>(Msc + t * LDM + 4 * s4);
      const float f[4] = {a.x, a.y, a.z, a.w};
      st4_tf32(sm + OFF_T + f32_off(t, 4 * s4, R64), f);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // U^T = Vw^T T^T : A = Vw^T (tensor memory), B = T (N = t), K = s
      // W^T = Kb^T T^T : A = Kb^T (tensor memory)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t bT = sdesc_sw128(sbase + OFF_T + (ks >> 2) * R64 + (ks & 3) * 32, 16, 1024);
        umma_tf32_ts(tmem + TM_U, tmem + TM_VWT + 8 * ks, bT, ID_64, ks > 0);
        umma_tf32_ts(tmem + TM_W, tmem + TM_KBT + 8 * ks, bT, ID_64, ks > 0);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    // ===== W (token rows) to shared memory: thread = key channel i, one column ==========
    {
      float v[32];
      tmem_ld32(tlane + TM_W + 32 * hf, v);
      tmem_ld_wait();
      const int i = 32 * qd + lane;
#pragma unroll
      for (int x = 0; x < 32; ++x)
        *reinterpret_cast<float*>(sm + OFF_KN + f32_off(32 * hf + x, i, R64)) = to_tf32(v[x]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // U~^T = U^T - S^T W^T : A = S^T from tensor memory, B = -W (N = t), K = key channels
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint64_t bW = sdesc_sw128(sbase + OFF_KN + (ks >> 2) * R64 + (ks & 3) * 32, 16, 1024);
        umma_tf32_ts(tmem + TM_U, tmem + TM_S + 8 * ks, bW, ID_64NEG, 1);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    if (tid == 0) {
      // O^T += U~^T P^T : A = U~^T from tensor memory, B = P (N = t), K = s
      // S^T += U~^T Kn  : B = Kn^T rows (N = key channels)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t bP = sdesc_sw128(sbase + OFF_P + (ks >> 2) * R64 + (ks & 3) * 32, 16, 1024);
        const uint64_t bK = sdesc_sw128(sbase + OFF_KNT + (ks >> 2) * R128 + (ks & 3) * 32, 16, 1024);
        umma_tf32_ts(tmem + TM_O, tmem + TM_U + 8 * ks, bP, ID_64, 1);
        umma_tf32_ts(tmem + TM_S, tmem + TM_U + 8 * ks, bK, ID_128, 1);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    // ===== outputs of the chunk, and the state decay ======================================
    {
      float v[32];
      tmem_ld32(tlane + TM_O + 32 * hf, v);  // O^T: lane = value channel j, columns = tokens
      tmem_ld_wait();
      if (jrow < dv) {
        float* op = p.o + (((size_t)bb * p.T + t0 + 32 * hf) * p.H + h) * dv + jrow;
        const size_t tstride = (size_t)p.H * dv;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (32 * hf + x < n) op[x * tstride] = v[x];
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int i0 = 64 * hf + 32 * half;
        tmem_ld32(tlane + TM_S + i0, v);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] *= ms.gC[i0 + x];
        tmem_st32(tlane + TM_S + i0, v);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
  }

  // ---- final state ----------------------------------------------------------------------
  tc_fence_after();
  if (!ms.abort && p.S_T && jrow < dv) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[32];
      const int i0 = 64 * hf + 32 * half;
      tmem_ld32(tlane + TM_S + i0, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x)
        if (i0 + x < dk) p.S_T[((size_t)unit * dk + i0 + x) * dv + jrow] = v[x];
    }
  }
  // ---- teardown: after a give-up, let outstanding async work drain (bounded) ------------
  if (tid == 0 && ms.abort) {
    volatile int never = 0;
    if (pend_la) mbar_wait_bounded(&ms.bar_la, ph_la, &never, nullptr, WAIT_LIMIT);
    if (pend_mma) mbar_wait_bounded(&ms.bar_mma, ph_mma, &never, nullptr, WAIT_LIMIT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// ---- host side ------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [B, T, H, D] tensor; one box = 64 tokens x box_d channels of one (b, h).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int B, int T, int H, int D,
              int box_d, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize, (cuuint64_t)T * H * D * esize};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)C, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_fwd_tc(const ChunkArgs& a, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mb, mw, mla;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = make_map(&mq, a.q, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mk, a.k, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mb, a.b, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mv, a.v, BF, 2, a.B, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mw, a.w, BF, 2, a.B, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, a.dk, a.dk,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  TcParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.b = static_cast<const __nv_bfloat16*>(a.b);
  p.w = static_cast<const __nv_bfloat16*>(a.w);
  p.S0 = a.S0;
  p.S_T = a.S_T;
  p.o = a.o;
  p.T = a.T;
  p.H = a.H;
  p.dk = a.dk;
  p.dv = a.dv;
  p.nchunks = (a.T + C - 1) / C;
  p.err = device_error_word();
  chunk_fwd_tc_kernel<<<a.B * a.H, NT, SMEM_BYTES, st>>>(mq, mk, mv, mb, mw, mla, p);
  return cudaGetLastError();
}

}  // namespace gdn2
