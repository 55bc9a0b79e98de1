// Chunkwise prefill forward for fp32 inputs with d_k = d_v = 64 on the 5th-generation tensor
// cores.  Every product runs as three tcgen05.mma kind::tf32 products, hi*hi + hi*lo + lo*hi,
// with each fp32 operand x split as hi = tf32(x) and lo = tf32(x - hi): the dropped lo*lo
// term and the rounding of lo are below 2^-21 of the product, so the result keeps the fp32
// accuracy the 1e-4 bar of fp32 inputs needs.  Accumulation is fp32 in tensor memory.
//
// Same chunk form as the bf16 kernel (Gated DeltaNet-2 guide, "Chunkwise Parallel Algorithm
// for GPU Training"; decay folded into the WY factors, snilld.dk, "Hvad betyder det for
// traening og inferens").  Per chunk of C = 64 tokens, entering state S, g = in-chunk cumsum
// of log alpha, Gamma = exp(g):
//
//     Kb = K*B*Gamma    Qh = Q*Gamma    Kn = K/Gamma    Vw = W*V
//     [-A; P]  = [-Kb; Qh] Kn^T         (A strictly lower, P lower incl. the diagonal)
//     T        = (I + A)^-1             forward substitution in fp32 on the CUDA cores
//     [X^T | O^T] = S^T [-Kb; Qh]^T     R^T = Vw^T + X^T
//     U^T      = R^T T^T
//     [O^T | S^T] += U^T [P; Kn^T]^T    S^T <- S^T Diag(Gamma_C)
//
// One CTA of 8 warps per (batch, head) walks its chunks; the phases are separated by block
// barriers (a latency-bound kernel for short fp32 sequences, not a streaming one).  The
// state is kept transposed (S^T, lanes = value channels 0-63, lanes 64-127 zero) in tensor
// memory; its hi and lo parts, then those of R^T and of U^T, take turns in one pair of
// tensor-memory regions as the A operands.  Shared-memory operands are K-major with the
// 128-byte swizzle, each in a hi and a lo tile.
#include <cuda_runtime.h>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 64, D = 64;
constexpr int NT = 256;  // 8 warps: thread t owns tensor-memory lane t mod 128, column half t / 128
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait
constexpr uint32_t R64 = 64 * 128, R128 = 128 * 128;
// shared memory: hi and lo tiles of each operand (fp32 panels of 32 columns)
constexpr uint32_t F_KQH = 0, F_KQL = F_KQH + 2 * R128;  // [-Kb; Qh] [t'][i]: 2 panels x 128 rows
constexpr uint32_t F_KNH = F_KQL + 2 * R128, F_KNL = F_KNH + 2 * R64;  // Kn [s][i]: 2 panels x 64 rows
constexpr uint32_t F_PKH = F_KNL + 2 * R64, F_PKL = F_PKH + 2 * R128;  // [P; Kn^T] [t | i][s]: 2 x 128
constexpr uint32_t F_TH = F_PKL + 2 * R128, F_TL = F_TH + 2 * R64;     // T [t][s]: 2 panels x 64 rows
constexpr uint32_t F_A = F_TL + 2 * R64;                                // A [t][s], fp32, rows of LDA
constexpr int LDA = 68;
constexpr uint32_t F_TILES = F_A + C * LDA * 4;
struct F32Misc {
  uint64_t bar_mma, bar_drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[D];
  alignas(16) float seg[4][D];
};
constexpr uint32_t F_SMEM = F_TILES + 1024 + sizeof(F32Misc);
// tensor memory columns
constexpr uint32_t M_AP = 0;    // [-A; P]   lanes: tokens of Kb | Qh, columns: s
constexpr uint32_t M_X = 64;    // X^T       lanes: value channel, columns: t   } one N = 128 product
constexpr uint32_t M_O = 128;   // O^T       lanes: value channel, columns: t   } } one N = 128
constexpr uint32_t M_S = 192;   // S^T       lanes: value channel, columns: i     } product
constexpr uint32_t M_U = 256;   // U~^T      lanes: value channel, columns: s
constexpr uint32_t M_H = 320;   // hi part of the current A operand (S^T, R^T or U~^T)
constexpr uint32_t M_L = 384;   // lo part
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);
constexpr uint32_t ID_128 = idesc_tf32(128, 128, 0, 0, 0, 0);

__device__ __forceinline__ float hi_of(float x) { return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u); }
__device__ __forceinline__ uint64_t kd(uint32_t base, uint32_t panel, int ks) {
  return sdesc_sw128(base + (uint32_t)(ks >> 2) * panel + (uint32_t)(ks & 3) * 32, 16, 1024);
}
// x into the hi and lo tiles at byte offset o
__device__ __forceinline__ void put_split(unsigned char* sm, uint32_t hi_base, uint32_t lo_base, uint32_t o, float x) {
  const float h = hi_of(x);
  *reinterpret_cast<float*>(sm + hi_base + o) = h;
  *reinterpret_cast<float*>(sm + lo_base + o) = hi_of(x - h);
}

struct F32Params {
  const float *q, *k, *v, *la, *b, *w;
  const float* S0;
  float *o, *S_T;
  int T, H;
  unsigned* err;
};

__global__ void __launch_bounds__(NT, 1) chunk_fwd_f32_tc_kernel(const F32Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  F32Misc& ms = *reinterpret_cast<F32Misc*>(sm + F_TILES);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, ln = tid & 127, hf = tid >> 7;
  const int unit = blockIdx.x, h = unit % p.H, bb = unit / p.H;
  const int nch = (p.T + C - 1) / C;
  float* A = reinterpret_cast<float*>(sm + F_A);
  auto tok = [&](int t) -> size_t { return (((size_t)bb * p.T + t) * p.H + h) * D; };

  if (tid == 0) {
    mbar_init(&ms.bar_mma, 1);
    mbar_init(&ms.bar_drain, 1);
    fence_mbar_init();
    ms.abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  uint32_t ph = 0;
  auto sync_ok = [&](bool ok) -> bool {
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    const bool bad = __syncthreads_or(!ok);
    tc_fence_after();
    return !bad;
  };
  // the issued products' completion: warp 0 polls, the block follows
  auto wait_mma = [&]() -> bool {
    bool ok = true;
    if (warp == 0) ok = mbar_wait_spin(&ms.bar_mma, ph, &ms.abort, p.err, WAIT_LIMIT);
    ph ^= 1;
    const bool bad = __syncthreads_or(!ok);
    tc_fence_after();
    return !bad;
  };
  // columns [32 hf, +32) of the accumulator at `col` split into the hi / lo regions
  auto split_to_hl = [&](uint32_t col) {
    float v[32], hv[32];
    tmem_ld32(tl + col + 32 * hf, v);
    tmem_ld_wait();
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      hv[x] = hi_of(v[x]);
      v[x] = hi_of(v[x] - hv[x]);
    }
    tmem_st32(tl + M_H + 32 * hf, hv);
    tmem_st32(tl + M_L + 32 * hf, v);
  };

  // entering state: S^T (lane j, key columns [32 hf, +32)), and its hi / lo parts
  {
    float v[32];
#pragma unroll
    for (int x = 0; x < 32; ++x)
      v[x] = (p.S0 && ln < D) ? p.S0[((size_t)unit * D + 32 * hf + x) * D + ln] : 0.f;
    tmem_st32(tl + M_S + 32 * hf, v);
    tmem_st_wait();
    split_to_hl(M_S);
  }
  bool dead = !sync_ok(true);

  for (int c = 0; c < nch && !dead; ++c) {
    const int t0 = C * c, n = min(C, p.T - t0);
    // ===== operands: thread (i = tid mod 64, tokens [16 tg, 16 tg + 16)) ====================
    {
      const int i = tid & 63, tg = tid >> 6;
      float g[16], kq[16], qq[16], bq[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int t = 16 * tg + r;
        const bool val = t < n;
        const size_t x = tok(t0 + min(t, n - 1)) + i;
        g[r] = val ? __ldg(p.la + x) : 0.f;
        kq[r] = val ? __ldg(p.k + x) : 0.f;
        qq[r] = val ? __ldg(p.q + x) : 0.f;
        bq[r] = val ? __ldg(p.b + x) : 0.f;
      }
#pragma unroll
      for (int r = 1; r < 16; ++r) g[r] += g[r - 1];
      ms.seg[tg][i] = g[15];
      __syncthreads();
      float off = 0.f, tot = 0.f;
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {
        const float sv = ms.seg[s4][i];
        if (s4 < tg) off += sv;
        tot += sv;
      }
      if (tg == 0) ms.gC[i] = expf(tot);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int t = 16 * tg + r;
        const float G = expf(off + g[r]), Gi = expf(-(off + g[r]));
        put_split(sm, F_KQH, F_KQL, f32_off(t, i, R128), -(kq[r] * bq[r] * G));
        put_split(sm, F_KQH, F_KQL, f32_off(C + t, i, R128), qq[r] * G);
        const float kn = kq[r] * Gi;
        put_split(sm, F_KNH, F_KNL, f32_off(t, i, R64), kn);
        put_split(sm, F_PKH, F_PKL, f32_off(C + i, t, R128), kn);  // Kn^T
      }
    }
    if (!sync_ok(true)) { dead = true; break; }
    // ===== [-A; P] = [-Kb; Qh] Kn^T and [X^T | O^T] = S^T [-Kb; Qh]^T, each as hi*hi + hi*lo +
    // lo*hi ===================================================================================
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ss(tmem + M_AP, kd(sbase + F_KQH, R128, ks), kd(sbase + F_KNH, R64, ks), ID_64, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ss(tmem + M_AP, kd(sbase + F_KQH, R128, ks), kd(sbase + F_KNL, R64, ks), ID_64, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ss(tmem + M_AP, kd(sbase + F_KQL, R128, ks), kd(sbase + F_KNH, R64, ks), ID_64, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_X, tmem + M_H + 8 * ks, kd(sbase + F_KQH, R128, ks), ID_128, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_X, tmem + M_H + 8 * ks, kd(sbase + F_KQL, R128, ks), ID_128, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_X, tmem + M_L + 8 * ks, kd(sbase + F_KQH, R128, ks), ID_128, 1);
      umma_commit(&ms.bar_mma);
    }
    if (!wait_mma()) { dead = true; break; }
    // ===== A to the solve matrix, P to its operand tiles; R^T = Vw^T + X^T to the hi / lo
    // regions (its reads of S^T's parts are done) =============================================
    {
      float v[32];
      tmem_ld32(tl + M_AP + 32 * hf, v);
      tmem_ld_wait();
      if (ln < C) {
        const int t = ln;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int s = 32 * hf + x;
          A[t * LDA + s] = (s < t) ? -v[x] : 0.f;
        }
      } else {
        const int t = ln - C;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int s = 32 * hf + x;
          put_split(sm, F_PKH, F_PKL, f32_off(t, s, R128), (s <= t) ? v[x] : 0.f);
        }
      }
      float xv[32], hv[32];
      tmem_ld32(tl + M_X + 32 * hf, xv);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int t = 32 * hf + x;
        float vw = 0.f;
        if (ln < D && t < n) {
          const size_t e = tok(t0 + t) + ln;
          vw = __ldg(p.v + e) * __ldg(p.w + e);
        }
        const float r = xv[x] + vw;
        hv[x] = hi_of(r);
        xv[x] = hi_of(r - hv[x]);
      }
      tmem_st32(tl + M_H + 32 * hf, hv);
      tmem_st32(tl + M_L + 32 * hf, xv);
    }
    __syncthreads();  // the solve matrix
    // ===== T = (I + A)^-1 by forward substitution in fp32: thread s < 64 owns column s ========
    if (tid < C) {
      const int s = tid;
      float x[C];
#pragma unroll
      for (int r = 0; r < C; ++r) x[r] = (r == s) ? 1.f : 0.f;
#pragma unroll
      for (int t = 1; t < C; ++t) {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < t; ++r) acc = fmaf(A[t * LDA + r], x[r], acc);
        if (t > s) x[t] = -acc;
      }
#pragma unroll
      for (int r = 0; r < C; ++r) put_split(sm, F_TH, F_TL, f32_off(r, s, R64), x[r]);
    }
    if (!sync_ok(true)) { dead = true; break; }
    // ===== U~^T = R^T T^T ======================================================================
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_U, tmem + M_H + 8 * ks, kd(sbase + F_TH, R64, ks), ID_64, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_U, tmem + M_H + 8 * ks, kd(sbase + F_TL, R64, ks), ID_64, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_U, tmem + M_L + 8 * ks, kd(sbase + F_TH, R64, ks), ID_64, 1);
      umma_commit(&ms.bar_mma);
    }
    if (!wait_mma()) { dead = true; break; }
    split_to_hl(M_U);
    if (!sync_ok(true)) { dead = true; break; }
    // ===== [O^T | S^T] += U~^T [P; Kn^T]^T ======================================================
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_O, tmem + M_H + 8 * ks, kd(sbase + F_PKH, R128, ks), ID_128, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_O, tmem + M_H + 8 * ks, kd(sbase + F_PKL, R128, ks), ID_128, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + M_O, tmem + M_L + 8 * ks, kd(sbase + F_PKH, R128, ks), ID_128, 1);
      umma_commit(&ms.bar_mma);
    }
    if (!wait_mma()) { dead = true; break; }
    // ===== the output rows; S^T <- S^T Diag(Gamma_C) and its hi / lo parts ====================
    {
      float v[32];
      tmem_ld32(tl + M_O + 32 * hf, v);
      tmem_ld_wait();
      if (ln < D) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (32 * hf + x < n) p.o[tok(t0 + 32 * hf + x) + ln] = v[x];
      }
      float sv[32], hv[32];
      tmem_ld32(tl + M_S + 32 * hf, sv);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        sv[x] *= ms.gC[32 * hf + x];
        hv[x] = hi_of(sv[x]);
        v[x] = hi_of(sv[x] - hv[x]);
      }
      tmem_st32(tl + M_S + 32 * hf, sv);
      tmem_st32(tl + M_H + 32 * hf, hv);
      tmem_st32(tl + M_L + 32 * hf, v);
    }
    if (!sync_ok(true)) { dead = true; break; }
  }
  // the final state
  if (!dead && p.S_T && ln < D) {
    float v[32];
    tmem_ld32(tl + M_S + 32 * hf, v);
    tmem_ld_wait();
#pragma unroll
    for (int x = 0; x < 32; ++x) p.S_T[((size_t)unit * D + 32 * hf + x) * D + ln] = v[x];
  }
  if (tid == 0 && ms.abort) {  // every MMA issued lands before the block releases its memory
    volatile int never = 0;
    umma_commit(&ms.bar_drain);
    mbar_wait_bounded(&ms.bar_drain, 0, &never, nullptr, WAIT_LIMIT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool chunk_fwd_f32_tc_supported(const ChunkArgs& a) { return !a.bf16 && a.dk == D && a.dv == D && !a.cu_seqlens; }

cudaError_t launch_chunk_fwd_f32_tc(const ChunkArgs& a, cudaStream_t st) {
  if (!chunk_fwd_f32_tc_supported(a)) return cudaErrorInvalidValue;
  if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
  F32Params p;
  p.q = static_cast<const float*>(a.q);
  p.k = static_cast<const float*>(a.k);
  p.v = static_cast<const float*>(a.v);
  p.b = static_cast<const float*>(a.b);
  p.w = static_cast<const float*>(a.w);
  p.la = a.log_alpha;
  p.S0 = a.S0;
  p.o = a.o;
  p.S_T = a.S_T;
  p.T = a.T;
  p.H = a.H;
  p.err = device_error_word();
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = smem_limit_once(chunk_fwd_f32_tc_kernel, (int)F_SMEM, attr_done);
  if (e != cudaSuccess) return e;
  chunk_fwd_f32_tc_kernel<<<a.B * a.H, NT, F_SMEM, st>>>(p);
  return cudaGetLastError();
}

}  // namespace gdn2
