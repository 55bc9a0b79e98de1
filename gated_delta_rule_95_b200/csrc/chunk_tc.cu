// Chunkwise prefill forward for bf16 inputs on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory), operands staged by TMA.
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
//     S      <- Diag(Gamma_C) (S + Kn^T U~)
//
// Every product is written so that its M side is 128 rows (tokens of [A;P], or
// the d_k / d_v axis of the transposed products), which keeps all accumulators
// in the simple M = 128 tensor-memory layout (row r = lane r).
//
// One CTA (256 threads, 8 warps) owns one (batch, head) and walks its chunks.
// Thread 0 issues TMA loads and MMAs; all warps do the elementwise work.  The
// raw inputs of chunk c+1 are loaded by TMA while chunk c is on the tensor cores.
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
// Raw inputs arrive by TMA in 128B-swizzled bf16 tiles of 64-channel panels and are
// turned into tensor-core operands in place; the fp32 -> bf16 rounding of the
// decay-folded operands is compensated by a second "lo" bf16 tile (x = hi + lo).
constexpr uint32_t P64 = 64 * 128;    // a panel of 64 rows x 128 B  (8 KB)
constexpr uint32_t P128 = 128 * 128;  // a panel of 128 rows x 128 B (16 KB)
// b (rows 0-63) and q (rows 64-127) of each key panel -> [Kb; Qh] hi tile;
// later U~^T hi (first 16 KB) and lo (second 16 KB)
constexpr uint32_t OFF_H = 0;
constexpr uint32_t OFF_KN = OFF_H + 2 * P128;   // k -> Kn hi       (2 x 64 rows)
constexpr uint32_t OFF_V = OFF_KN + 2 * P64;    // v -> Vw hi -> W^T (128 rows)
constexpr uint32_t OFF_W = OFF_V + 2 * P64;     // w -> Vw lo
constexpr uint32_t OFF_LA = OFF_W + 2 * P64;    // 2 x 32 KB: log-alpha of a chunk, then its [Kb; Qh] lo tile
constexpr uint32_t OFF_KNLO = OFF_LA + 2 * 32768;  // Kn lo (2 x 64 rows)
constexpr uint32_t OFF_S = OFF_KNLO + 2 * P64;  // S bf16: 2 panels (value channels) x 128 rows (key channels)
constexpr uint32_t OFF_SCR = OFF_S + 2 * P128;  // solve scratch (fp32 64x68 + 16x48), then P hi / P lo
constexpr uint32_t OFF_T = OFF_SCR + 20480;     // T bf16 [t][s]
constexpr uint32_t TILES = OFF_T + P64;         // 220 KB

struct Misc {
  uint64_t bar_qkb, bar_v, bar_w, bar_mma;
  uint64_t bar_la[2];
  uint32_t tmem_base;
  int abort;
  float gC[128];     // Gamma at the chunk end, per key channel
  float half0[128];  // sum of log alpha over the first 32 tokens, per key channel
};
constexpr uint32_t SMEM_BYTES = TILES + 1024 + sizeof(Misc);

// ---- tensor memory columns (fp32 accumulators, 128 lanes) ----------------------------
constexpr uint32_t TM_AP = 0;     // [A; P]  64 columns
constexpr uint32_t TM_U = 64;     // U^T, then U~^T  (lanes = value channel)
constexpr uint32_t TM_W = 128;    // W^T  (lanes = key channel)
constexpr uint32_t TM_O = 192;    // O^T  (lanes = value channel)
constexpr uint32_t TM_D = 256;    // Kn^T U~  128 columns (lanes = key channel)
constexpr uint32_t TM_COLS = 512;

// instruction descriptors
constexpr uint32_t ID_AP = idesc_bf16(128, 64, 0, 0, 0);   // [Kb;Qh] (K-major) x Kn (K-major)
constexpr uint32_t ID_UW = idesc_bf16(128, 64, 1, 0, 0);   // Vw^T / Kb^T (MN-major) x T (K-major)
constexpr uint32_t ID_SW = idesc_bf16(128, 64, 1, 1, 1);   // -(S^T) (MN-major) x W^T (MN-major)
constexpr uint32_t ID_SQ = idesc_bf16(128, 64, 1, 0, 0);   // S^T (MN-major) x Qh (K-major)
constexpr uint32_t ID_UP = idesc_bf16(128, 64, 0, 0, 0);   // U~^T (K-major) x P (K-major)
constexpr uint32_t ID_KU = idesc_bf16(128, 128, 1, 0, 0);  // Kn^T (MN-major) x U~^T (K-major)

// 8 fp32 values -> hi and lo bf16 16-byte chunks.
__device__ __forceinline__ void split8(const float* f, uint4& hi, uint4& lo) {
  uint32_t* h = &hi.x;
  uint32_t* l = &lo.x;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const __nv_bfloat16 a = __float2bfloat16_rn(f[2 * m]), b = __float2bfloat16_rn(f[2 * m + 1]);
    h[m] = pack_bf16(__bfloat162float(a), __bfloat162float(b));
    l[m] = pack_bf16(f[2 * m] - __bfloat162float(a), f[2 * m + 1] - __bfloat162float(b));
  }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  u.x = pack_bf16(f[0], f[1]);
  u.y = pack_bf16(f[2], f[3]);
  u.z = pack_bf16(f[4], f[5]);
  u.w = pack_bf16(f[6], f[7]);
  return u;
}

// fp32 scratch of the triangular solve: a 64 x 64 matrix with rows padded to 68
// floats (16-byte aligned rows that start 4 banks apart).  It first holds A
// (strictly lower, zero elsewhere) and is overwritten block-row by block-row
// with T = (I + A)^-1 (unit lower triangular, explicit zeros above).
constexpr int LDM = 68;

struct TcParams {
  const float* S0;
  float* S_T;
  float* o;
  int T, H, dk, dv, nchunks;
  unsigned* err;
};

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
    mbar_init(&ms.bar_qkb, 1);
    mbar_init(&ms.bar_v, 1);
    mbar_init(&ms.bar_w, 1);
    mbar_init(&ms.bar_mma, 1);
    mbar_init(&ms.bar_la[0], 1);
    mbar_init(&ms.bar_la[1], 1);
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

  // ---- TMA issue (thread 0) and the bookkeeping of what is in flight ----------------
  int pend_qkb = 0, pend_v = 0, pend_w = 0, pend_mma = 0, pend_la0 = 0, pend_la1 = 0;
  auto issue_qkb = [&](int c) {
    mbar_arrive_expect_tx(&ms.bar_qkb, (uint32_t)(3 * (dk >> 6)) * P64);
    for (int pn = 0; pn < (dk >> 6); ++pn) {
      tma_load_4d(sm + OFF_H + pn * P128, &tmB, &ms.bar_qkb, 64 * pn, h, C * c, bb);
      tma_load_4d(sm + OFF_H + pn * P128 + P64, &tmQ, &ms.bar_qkb, 64 * pn, h, C * c, bb);
      tma_load_4d(sm + OFF_KN + pn * P64, &tmK, &ms.bar_qkb, 64 * pn, h, C * c, bb);
    }
    pend_qkb = 1;
  };
  auto issue_v = [&](int c) {
    mbar_arrive_expect_tx(&ms.bar_v, (uint32_t)(dv >> 6) * P64);
    for (int pn = 0; pn < (dv >> 6); ++pn) tma_load_4d(sm + OFF_V + pn * P64, &tmV, &ms.bar_v, 64 * pn, h, C * c, bb);
    pend_v = 1;
  };
  auto issue_w = [&](int c) {
    mbar_arrive_expect_tx(&ms.bar_w, (uint32_t)(dv >> 6) * P64);
    for (int pn = 0; pn < (dv >> 6); ++pn) tma_load_4d(sm + OFF_W + pn * P64, &tmW, &ms.bar_w, 64 * pn, h, C * c, bb);
    pend_w = 1;
  };
  auto issue_la = [&](int c) {
    const int buf = c & 1;
    mbar_arrive_expect_tx(&ms.bar_la[buf], (uint32_t)(C * dk * 4));
    tma_load_4d(sm + OFF_LA + buf * 32768, &tmLA, &ms.bar_la[buf], 0, h, C * c, bb);
    if (buf) pend_la1 = 1; else pend_la0 = 1;
  };
  if (tid == 0 && p.nchunks > 0) {
    issue_qkb(0);
    issue_v(0);
    issue_w(0);
    issue_la(0);
    if (p.nchunks > 1) issue_la(1);
  }

  // ---- entering state: fp32 rows in registers, bf16 copy as an MMA operand ---------
  // Thread (qd, hf, lane) owns key row i = 32 qd + lane, value columns [64 hf, 64 hf + 64).
  const int srow = 32 * qd + lane;
  float Sr[64];
  {
    const float* src = p.S0 ? p.S0 + ((size_t)unit * dk + srow) * dv + 64 * hf : nullptr;
    const bool ok = src && srow < dk && 64 * hf < dv;
#pragma unroll
    for (int x = 0; x < 64; x += 4) {
      float4 f = ok ? *reinterpret_cast<const float4*>(src + x) : make_float4(0.f, 0.f, 0.f, 0.f);
      Sr[x] = f.x; Sr[x + 1] = f.y; Sr[x + 2] = f.z; Sr[x + 3] = f.w;
    }
  }
  auto store_S_bf16 = [&]() {
    unsigned char* dst = sm + OFF_S + hf * P128;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(dst + sw128_off(srow, ch)) = pack8(&Sr[8 * ch]);
  };
  store_S_bf16();

  uint32_t ph_qkb = 0, ph_v = 0, ph_w = 0, ph_mma = 0, ph_la0 = 0, ph_la1 = 0;
  float* Msc = reinterpret_cast<float*>(sm + OFF_SCR);                  // solve matrix, 64 x LDM fp32
  float* Xsc = reinterpret_cast<float*>(sm + OFF_SCR + 64 * LDM * 4);   // block-row product, 16 x 48 fp32

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

  for (int c = 0; c < p.nchunks; ++c) {
    const int t0 = C * c, n = min(C, p.T - t0);
    const int lb = c & 1;
    unsigned char* LO = sm + OFF_LA + lb * 32768;  // this chunk's log-alpha, then its lo tile
    const uint32_t LO_s = sbase + OFF_LA + lb * 32768;
    if (tid == 0 && c >= 1 && c + 1 < p.nchunks) issue_la(c + 1);  // buffer of chunk c-1 is free
    {
      bool ok = wait_on(&ms.bar_qkb, ph_qkb, pend_qkb);
      ok = ok && wait_on(&ms.bar_v, ph_v, pend_v);
      ok = ok && wait_on(&ms.bar_w, ph_w, pend_w);
      ok = ok && (lb ? wait_on(&ms.bar_la[1], ph_la1, pend_la1) : wait_on(&ms.bar_la[0], ph_la0, pend_la0));
      if (__syncthreads_or(!ok)) break;
    }
    // ===== prep: decay cumsum and the folded operands, in place ========================
    float* la = reinterpret_cast<float*>(LO);
    {
      // in-chunk cumsum of log alpha, in place in the fp32 staging [t][d_k]:
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
    {
      // thread (cg, tg): channels [8 cg, 8 cg + 8) (one 16-byte chunk), tokens tg + 16 r
      const int cg = tid & 15, tg = tid >> 4, c0 = 8 * cg;
      const bool kval = c0 < dk, vval = c0 < dv;
      const uint32_t pn = (uint32_t)(cg >> 3);
      const int chk = cg & 7;
      float gv[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (kval) {
          const float4 a = *reinterpret_cast<const float4*>(la + (tg + 16 * r) * dk + c0);
          const float4 b = *reinterpret_cast<const float4*>(la + (tg + 16 * r) * dk + c0 + 4);
          gv[r][0] = a.x; gv[r][1] = a.y; gv[r][2] = a.z; gv[r][3] = a.w;
          gv[r][4] = b.x; gv[r][5] = b.y; gv[r][6] = b.z; gv[r][7] = b.w;
        }
      }
      __syncthreads();  // every cumsum value is read before the buffer becomes the lo tile
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = tg + 16 * r;
        const uint32_t o64 = pn * P64 + sw128_off(t, chk);
        const uint32_t oKb = pn * P128 + sw128_off(t, chk);
        const uint32_t oQh = pn * P128 + sw128_off(64 + t, chk);
        float kb[8], qh[8], kn[8], vw[8];
        if (kval) {
          float kk[8], bg[8], qq[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + OFF_KN + o64), kk);
          unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + OFF_H + oKb), bg);
          unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + OFF_H + oQh), qq);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float G = __expf(gv[r][m]), Gi = __expf(-gv[r][m]);
            kb[m] = kk[m] * bg[m] * G;
            qh[m] = qq[m] * G;
            kn[m] = kk[m] * Gi;
          }
        } else {
#pragma unroll
          for (int m = 0; m < 8; ++m) kb[m] = qh[m] = kn[m] = 0.f;
        }
        if (vval) {
          float vv[8], ww[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + OFF_V + o64), vv);
          unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + OFF_W + o64), ww);
#pragma unroll
          for (int m = 0; m < 8; ++m) vw[m] = ww[m] * vv[m];
        } else {
#pragma unroll
          for (int m = 0; m < 8; ++m) vw[m] = 0.f;
        }
        uint4 hi, lo;
        split8(kb, hi, lo);
        *reinterpret_cast<uint4*>(sm + OFF_H + oKb) = hi;
        *reinterpret_cast<uint4*>(LO + oKb) = lo;
        split8(qh, hi, lo);
        *reinterpret_cast<uint4*>(sm + OFF_H + oQh) = hi;
        *reinterpret_cast<uint4*>(LO + oQh) = lo;
        split8(kn, hi, lo);
        *reinterpret_cast<uint4*>(sm + OFF_KN + o64) = hi;
        *reinterpret_cast<uint4*>(sm + OFF_KNLO + o64) = lo;
        split8(vw, hi, lo);
        *reinterpret_cast<uint4*>(sm + OFF_V + o64) = hi;
        *reinterpret_cast<uint4*>(sm + OFF_W + o64) = lo;
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      // [A; P] = [Kb; Qh] Kn^T : M=128 (tokens of both halves), N=64, K=128 (key channels)
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t ko = (uint32_t)((ks & 3) * 32);
        const uint64_t aH = sdesc_sw128(sbase + OFF_H + (ks >> 2) * P128 + ko, 16, 1024);
        const uint64_t aL = sdesc_sw128(LO_s + (ks >> 2) * P128 + ko, 16, 1024);
        const uint64_t bH = sdesc_sw128(sbase + OFF_KN + (ks >> 2) * P64 + ko, 16, 1024);
        const uint64_t bL = sdesc_sw128(sbase + OFF_KNLO + (ks >> 2) * P64 + ko, 16, 1024);
        umma_bf16(tmem + TM_AP, aH, bH, ID_AP, ks > 0);
        umma_bf16(tmem + TM_AP, aH, bL, ID_AP, 1);
        umma_bf16(tmem + TM_AP, aL, bH, ID_AP, 1);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    // ===== A out of tensor memory (P stays there until the solve is done) ==============
    if (qd < 2) {
      float v[32];
      tmem_ld32(tlane + TM_AP + 32 * hf, v);
      tmem_ld_wait();
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
    // diagonal is an explicit zero, so the products run over full ranges.
#pragma unroll
    for (int I = 1; I < 4; ++I) {
      const int r = tid >> 4, c = tid & 15;
      const float* Arow = Msc + (16 * I + r) * LDM;
      float z[3] = {0.f, 0.f, 0.f};
#pragma unroll
      for (int k4 = 0; k4 < 16 * I; k4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(Arow + k4);
#pragma unroll
        for (int u = 0; u < I; ++u) {
          const float* Tc = Msc + k4 * LDM + c + 16 * u;
          z[u] = fmaf(a.x, Tc[0], z[u]);
          z[u] = fmaf(a.y, Tc[LDM], z[u]);
          z[u] = fmaf(a.z, Tc[2 * LDM], z[u]);
          z[u] = fmaf(a.w, Tc[3 * LDM], z[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < I; ++u) Xsc[r * 48 + c + 16 * u] = z[u];
      __syncthreads();
      const float* Trow = Msc + (16 * I + r) * LDM + 16 * I;
      float y[3] = {0.f, 0.f, 0.f};
#pragma unroll
      for (int s4 = 0; s4 < 16; s4 += 4) {
        const float4 tr = *reinterpret_cast<const float4*>(Trow + s4);
#pragma unroll
        for (int u = 0; u < I; ++u) {
          const float* Xc = Xsc + s4 * 48 + c + 16 * u;
          y[u] = fmaf(tr.x, Xc[0], y[u]);
          y[u] = fmaf(tr.y, Xc[48], y[u]);
          y[u] = fmaf(tr.z, Xc[96], y[u]);
          y[u] = fmaf(tr.w, Xc[144], y[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < I; ++u) Msc[(16 * I + r) * LDM + c + 16 * u] = -y[u];
      __syncthreads();
    }
    // T as a bf16 K-major operand [t][s]
    for (int e = tid; e < 512; e += NT) {
      const int t = e >> 3, q8 = e & 7;
      const float4 a = *reinterpret_cast<const float4*>(Msc + t * LDM + 8 * q8);
      const float4 b = *reinterpret_cast<const float4*>(Msc + t * LDM + 8 * q8 + 4);
      const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      *reinterpret_cast<uint4*>(sm + OFF_T + sw128_off(t, q8)) = pack8(f);
    }
    __syncthreads();  // the scratch is free: P hi / lo go there
    if (qd >= 2) {
      float v[32];
      tmem_ld32(tlane + TM_AP + 32 * hf, v);
      tmem_ld_wait();
      const int t = 32 * (qd - 2) + lane;  // P row, causal incl. diagonal
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float f[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) f[m] = (32 * hf + 8 * q4 + m <= t) ? v[8 * q4 + m] : 0.f;
        uint4 hi, lo;
        split8(f, hi, lo);
        *reinterpret_cast<uint4*>(sm + OFF_SCR + sw128_off(t, 4 * hf + q4)) = hi;
        *reinterpret_cast<uint4*>(sm + OFF_SCR + P64 + sw128_off(t, 4 * hf + q4)) = lo;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // U^T = Vw^T T^T : A = Vw hi/lo (MN-major, M = value channels), B = T (K-major, N = t), K = s
      // W^T = Kb^T T^T : A = Kb hi rows of the H tile (MN-major, M = key channels)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bT = sdesc_sw128(sbase + OFF_T + ks * 32, 16, 1024);
        const uint64_t aVh = sdesc_sw128(sbase + OFF_V + ks * 2048, P64, 1024);
        const uint64_t aVl = sdesc_sw128(sbase + OFF_W + ks * 2048, P64, 1024);
        const uint64_t aK = sdesc_sw128(sbase + OFF_H + ks * 2048, P128, 1024);
        umma_bf16(tmem + TM_U, aVh, bT, ID_UW, ks > 0);
        umma_bf16(tmem + TM_U, aVl, bT, ID_UW, 1);
        umma_bf16(tmem + TM_W, aK, bT, ID_UW, ks > 0);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    if (tid == 0 && c + 1 < p.nchunks) issue_w(c + 1);  // Vw lo consumed
    // ===== W^T to shared memory as an MN-major operand: row = key channel, col = t ======
    {
      float v[32];
      tmem_ld32(tlane + TM_W + 32 * hf, v);
      tmem_ld_wait();
      const int i = 32 * qd + lane;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint4*>(sm + OFF_V + sw128_off(i, 4 * hf + q4)) = pack8(&v[8 * q4]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // U~^T = U^T - S^T W^T : A = S (MN-major, M = value channels), B = W^T (MN-major, N = t), K = key channels
      // O^T  = S^T Qh^T      : B = Qh hi / lo rows of the H / lo tiles (K-major, N = t)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t qo = (ks >> 2) * P128 + P64 + (ks & 3) * 32;
        const uint64_t aS = sdesc_sw128(sbase + OFF_S + ks * 2048, P128, 1024);
        const uint64_t bW = sdesc_sw128(sbase + OFF_V + ks * 2048, P64, 1024);
        const uint64_t bQh = sdesc_sw128(sbase + OFF_H + qo, 16, 1024);
        const uint64_t bQl = sdesc_sw128(LO_s + qo, 16, 1024);
        umma_bf16(tmem + TM_U, aS, bW, ID_SW, 1);
        umma_bf16(tmem + TM_O, aS, bQh, ID_SQ, ks > 0);
        umma_bf16(tmem + TM_O, aS, bQl, ID_SQ, 1);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    if (tid == 0 && c + 1 < p.nchunks) issue_v(c + 1);  // W^T consumed
    // ===== U~^T hi / lo to shared memory as K-major operands: row = value channel, col = s
    {
      float v[32];
      tmem_ld32(tlane + TM_U + 32 * hf, v);
      tmem_ld_wait();
      const int j = 32 * qd + lane;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint4 hi, lo;
        split8(&v[8 * q4], hi, lo);
        *reinterpret_cast<uint4*>(sm + OFF_H + sw128_off(j, 4 * hf + q4)) = hi;
        *reinterpret_cast<uint4*>(sm + OFF_H + P128 + sw128_off(j, 4 * hf + q4)) = lo;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // O^T += U~^T P^T : A = U~^T hi/lo (K-major, M = value channels), B = P hi/lo (K-major, N = t), K = s
      // D    = Kn^T U~  : A = Kn hi/lo (MN-major, M = key channels), B = U~^T hi/lo (K-major, N = value ch.)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t aUh = sdesc_sw128(sbase + OFF_H + ks * 32, 16, 1024);
        const uint64_t aUl = sdesc_sw128(sbase + OFF_H + P128 + ks * 32, 16, 1024);
        const uint64_t bPh = sdesc_sw128(sbase + OFF_SCR + ks * 32, 16, 1024);
        const uint64_t bPl = sdesc_sw128(sbase + OFF_SCR + P64 + ks * 32, 16, 1024);
        const uint64_t aKh = sdesc_sw128(sbase + OFF_KN + ks * 2048, P64, 1024);
        const uint64_t aKl = sdesc_sw128(sbase + OFF_KNLO + ks * 2048, P64, 1024);
        umma_bf16(tmem + TM_O, aUh, bPh, ID_UP, 1);
        umma_bf16(tmem + TM_O, aUh, bPl, ID_UP, 1);
        umma_bf16(tmem + TM_O, aUl, bPh, ID_UP, 1);
        umma_bf16(tmem + TM_D, aKh, aUh, ID_KU, ks > 0);
        umma_bf16(tmem + TM_D, aKh, aUl, ID_KU, 1);
        umma_bf16(tmem + TM_D, aKl, aUh, ID_KU, 1);
      }
      commit_mma();
    }
    if (__syncthreads_or(!wait_mma())) break;
    tc_fence_after();
    if (tid == 0 && c + 1 < p.nchunks) issue_qkb(c + 1);  // H and Kn tiles consumed
    // ===== outputs of the chunk, and the state hand-over ================================
    {
      float v[32];
      tmem_ld32(tlane + TM_O + 32 * hf, v);  // O^T: lane = value channel j, columns = tokens
      tmem_ld_wait();
      const int j = 32 * qd + lane;
      if (j < dv) {
        float* op = p.o + (((size_t)bb * p.T + t0 + 32 * hf) * p.H + h) * dv + j;
        const size_t tstride = (size_t)p.H * dv;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (32 * hf + x < n) op[x * tstride] = v[x];
      }
      const float gc = ms.gC[srow];
      tmem_ld32(tlane + TM_D + 64 * hf, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x) Sr[x] = gc * (Sr[x] + v[x]);
      tmem_ld32(tlane + TM_D + 64 * hf + 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x) Sr[32 + x] = gc * (Sr[32 + x] + v[x]);
      store_S_bf16();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  // ---- final state ----------------------------------------------------------------------
  if (!ms.abort && p.S_T && srow < dk && 64 * hf < dv) {
    float* dst = p.S_T + ((size_t)unit * dk + srow) * dv + 64 * hf;
#pragma unroll
    for (int x = 0; x < 64; x += 4) *reinterpret_cast<float4*>(dst + x) = make_float4(Sr[x], Sr[x + 1], Sr[x + 2], Sr[x + 3]);
  }
  // ---- teardown: after a give-up, let outstanding async work drain (bounded) ------------
  if (tid == 0 && ms.abort) {
    volatile int never = 0;
    if (pend_qkb) mbar_wait_bounded(&ms.bar_qkb, ph_qkb, &never, nullptr, WAIT_LIMIT);
    if (pend_v) mbar_wait_bounded(&ms.bar_v, ph_v, &never, nullptr, WAIT_LIMIT);
    if (pend_w) mbar_wait_bounded(&ms.bar_w, ph_w, &never, nullptr, WAIT_LIMIT);
    if (pend_la0) mbar_wait_bounded(&ms.bar_la[0], ph_la0, &never, nullptr, WAIT_LIMIT);
    if (pend_la1) mbar_wait_bounded(&ms.bar_la[1], ph_la1, &never, nullptr, WAIT_LIMIT);
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
