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
//     T       = (I + A)^-1              recursive 2x2 block inverse (fp32 diagonal blocks)
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
// One CTA (512 threads, 16 warps) owns one (batch, head) and walks its chunks.
// Thread 0 issues TMA and MMAs; all warps do the elementwise work.  Latency is
// hidden across chunks: the raw bf16 inputs of chunk c+1 are prefetched into L2
// while chunk c starts and copied by TMA into tiles that chunk c no longer needs
// once its second product is done; the log-alpha tile of chunk c+1 is loaded by
// TMA while chunk c runs; and the output store and state decay of chunk c-1 run
// while chunk c's first product is on the tensor cores (the output accumulator
// is double-buffered in tensor memory).
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
constexpr int NT = 512;
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait

// ---- shared memory map (byte offsets from a 1024-byte aligned base) ----------------
// fp32 operand tiles with the 128B swizzle, in panels of 32 columns (128 B rows).
constexpr uint32_t R64 = 64 * 128;    // a panel of 64 rows  (8 KB)
constexpr uint32_t R128 = 128 * 128;  // a panel of 128 rows (16 KB)
constexpr uint32_t OFF_KQ = 0;                  // [Kb; Qh] [t][i]: 4 panels x 128 rows (first: raw q, k, b, v)
constexpr uint32_t OFF_KN = OFF_KQ + 4 * R128;  // Kn [s][i]: 4 panels x 64 rows; later W [t][i]
constexpr uint32_t OFF_KNT = OFF_KN + 4 * R64;  // Kn^T [i][s]: 2 panels x 128 rows
constexpr uint32_t OFF_T = OFF_KNT + 2 * R128;  // T [t][s]: 2 panels x 64 rows (first: Vw [t][j], 32 KB over T and P)
constexpr uint32_t OFF_P = OFF_T + 2 * R64;     // P [t][s]: 2 panels x 64 rows
constexpr uint32_t OFF_LA = OFF_P + 2 * R64;    // log alpha [t][i] fp32 (TMA, 128B swizzle): 4 panels x 64 rows;
                                                // between uses: the output tile [t][j] fp32 of a TMA store
constexpr uint32_t OFF_SCR = OFF_LA + 4 * R64;  // solve scratch: fp32 64 x LDM, then 32 x LDX (first: raw w)
// raw bf16 staging (TMA, 128B swizzle): a [64 tokens][128 channels] tile = 2 panels of
// 64 channels x 64 rows
constexpr uint32_t B16 = 2 * R64;
constexpr uint32_t RAW_Q = OFF_KQ, RAW_K = OFF_KQ + B16, RAW_B = OFF_KQ + 2 * B16, RAW_V = OFF_KQ + 3 * B16;
constexpr uint32_t RAW_W = OFF_SCR;
constexpr int LDM = 68;                         // padded row (floats) of the 64 x 64 solve matrix
constexpr int LDX = 36;                         // padded row of the 32 x 32 block product
constexpr uint32_t TILES = OFF_SCR + 22528;     // 214 KB

struct Misc {
  uint64_t bar_la, bar_mma, bar_raw;
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[2][128];  // Gamma at the chunk end, per key channel (chunk parity)
};
constexpr uint32_t SMEM_BYTES = TILES + 1024 + sizeof(Misc);

// ---- tensor memory columns (fp32, 128 lanes) -------------------------------------------
constexpr uint32_t TM_AP = 0;     // [A; P], later W^T   lanes: tokens of Kb | Qh (key channel for W^T)
constexpr uint32_t TM_W = 0;
constexpr uint32_t TM_U = 64;     // U^T, then U~^T      lanes: value channel, columns: s
constexpr uint32_t TM_O = 128;    // O^T, two buffers    lanes: value channel, columns: t
constexpr uint32_t TM_S = 256;    // S^T (the state)     lanes: value channel, columns: key channel
constexpr uint32_t TM_KBT = 384;  // Kb^T                lanes: key channel,   columns: s
constexpr uint32_t TM_VWT = 448;  // Vw^T                lanes: value channel, columns: s
constexpr uint32_t TM_COLS = 512;

// instruction descriptors (M = 128, both operands K-major)
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);
constexpr uint32_t ID_64NEG = idesc_tf32(128, 64, 0, 0, 0, 1);  // B negated
constexpr uint32_t ID_128 = idesc_tf32(128, 128, 0, 0, 0, 0);

struct TcParams {
  const __nv_bfloat16 *q, *k, *v, *b, *w;
  const float* S0;
  float* S_T;
  float* o;
  int T, H, dk, dv, nchunks;
  unsigned* err;
};

// fp32 -> tf32, round to nearest with ties away from zero on the magnitude (add half an
// ulp of the 10-bit mantissa, clear the 13 dropped bits); two integer instructions.
__device__ __forceinline__ float rna_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ void st4_tf32(unsigned char* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(rna_tf32(f[0]), rna_tf32(f[1]), rna_tf32(f[2]), rna_tf32(f[3]));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmLA,
                        const __grid_constant__ CUtensorMap tmO, const TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  // 128B-swizzled tiles need 1024-byte aligned shared addresses
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Misc& ms = *reinterpret_cast<Misc*>(sm + TILES);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, cq = warp >> 2;  // TMEM lane quadrant, column quarter
  const int unit = blockIdx.x, bb = unit / p.H, h = unit % p.H;
  const int dk = p.dk, dv = p.dv;
  const int jrow = 32 * qd + lane;  // this thread's TMEM lane
  const int c0 = 8 * warp;          // prep: this warp's 8 channels

  if (tid == 0) {
    mbar_init(&ms.bar_la, 1);
    mbar_init(&ms.bar_mma, 1);
    mbar_init(&ms.bar_raw, 1);
    fence_mbar_init();
    ms.abort = 0;
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmB); tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmLA);
    tma_prefetch_desc(&tmO);
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

  // ---- async copies (issued by thread TMA_TID, so that thread 0 only issues MMAs) ----------
  constexpr int TMA_TID = 32;
  int pend_la = 0, pend_mma = 0, pend_raw = 0;
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
  auto issue_la = [&](int c) {  // log alpha of chunk c: dk/32 boxes of 32 channels x 64 tokens
    mbar_arrive_expect_tx(&ms.bar_la, (uint32_t)(C * dk * 4));
    for (int pn = 0; pn < (dk >> 5); ++pn)
      tma_load_4d(sm + OFF_LA + pn * R64, &tmLA, &ms.bar_la, 32 * pn, h, C * c, bb);
    pend_la = 1;
  };
  auto issue_raw = [&](int c) {  // raw bf16 inputs of chunk c into the staging tiles
    mbar_arrive_expect_tx(&ms.bar_raw, (uint32_t)(3 * (dk >> 6) + 2 * (dv >> 6)) * R64);
    for (int pn = 0; pn < (dk >> 6); ++pn) {
      tma_load_4d(sm + RAW_Q + pn * R64, &tmQ, &ms.bar_raw, 64 * pn, h, C * c, bb);
      tma_load_4d(sm + RAW_K + pn * R64, &tmK, &ms.bar_raw, 64 * pn, h, C * c, bb);
      tma_load_4d(sm + RAW_B + pn * R64, &tmB, &ms.bar_raw, 64 * pn, h, C * c, bb);
    }
    for (int pn = 0; pn < (dv >> 6); ++pn) {
      tma_load_4d(sm + RAW_V + pn * R64, &tmV, &ms.bar_raw, 64 * pn, h, C * c, bb);
      tma_load_4d(sm + RAW_W + pn * R64, &tmW, &ms.bar_raw, 64 * pn, h, C * c, bb);
    }
    pend_raw = 1;
  };
  if (tid == TMA_TID && p.nchunks > 0) {
    issue_raw(0);
    issue_la(0);
    if (p.nchunks > 1) prefetch_raw(1);
  }

  // ---- entering state S0 -> S^T in tensor memory -----------------------------------------
  // Thread (qd, cq, lane) owns lane j = 32 qd + lane (a value channel) and the key-channel
  // columns [32 cq, 32 cq + 32) of S^T.
  {
    float v[32];
    const bool ok = p.S0 && jrow < dv;
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      const int i = 32 * cq + x;
      v[x] = (ok && i < dk) ? p.S0[((size_t)unit * dk + i) * dv + jrow] : 0.f;
    }
    tmem_st32(tlane + TM_S + 32 * cq, v);
    tmem_st_wait();
  }

  uint32_t ph_la = 0, ph_mma = 0, ph_raw = 0;
  float* Msc = reinterpret_cast<float*>(sm + OFF_SCR);                  // solve matrix, 64 x LDM fp32
  float* Xsc = reinterpret_cast<float*>(sm + OFF_SCR + 64 * LDM * 4);   // block product, 32 x LDX fp32
  const float* la = reinterpret_cast<const float*>(sm + OFF_LA);

  auto wait_on = [&](uint64_t* bar, uint32_t& ph, int& pend) -> bool {
    const bool ok = mbar_wait_bounded(bar, ph, &ms.abort, p.err, WAIT_LIMIT);
    if (ok) {
      ph ^= 1;
      pend = 0;
    }
    return ok;
  };
  auto wait_mma = [&]() -> bool { return wait_on(&ms.bar_mma, ph_mma, pend_mma); };
  auto commit_mma = [&]() {
    umma_commit(&ms.bar_mma);
    pend_mma = 1;
  };
  // Output of chunk cc (O^T in tensor-memory buffer cc & 1) into the shared-memory
  // tile [t][j] (rows of d_v floats) that a TMA store then writes out.
  auto stage_o = [&](int cc) {
    float v[16];
    tmem_ld16(tlane + TM_O + 64 * (cc & 1) + 16 * cq, v);
    tmem_ld_wait();
    if (jrow < dv) {
      float* st = reinterpret_cast<float*>(sm + OFF_LA) + jrow;
#pragma unroll
      for (int x = 0; x < 16; ++x) st[(16 * cq + x) * dv] = v[x];
    }
  };
  auto store_o = [&](int cc) {  // thread TMA_TID, after the staging is visible
    tma_store_4d(&tmO, sm + OFF_LA, 0, h, C * cc, bb);
    bulk_commit();
  };
  // S^T <- S^T Diag(Gamma_C of the chunk with parity gb), in tensor memory.
  auto decay_state = [&](int gb) {
    float v[32];
    tmem_ld32(tlane + TM_S + 32 * cq, v);
    tmem_ld_wait();
#pragma unroll
    for (int x = 0; x < 32; x += 4) {
      const float4 gq = *reinterpret_cast<const float4*>(&ms.gC[gb][32 * cq + x]);
      v[x] *= gq.x;
      v[x + 1] *= gq.y;
      v[x + 2] *= gq.z;
      v[x + 3] *= gq.w;
    }
    tmem_st32(tlane + TM_S + 32 * cq, v);
  };
  tc_fence_before();
  __syncthreads();

  bool dead = false;
  for (int c = 0; c < p.nchunks; ++c) {
    const int ob = c & 1;
    if (tid == TMA_TID && c + 2 < p.nchunks) prefetch_raw(c + 2);
    // ===== decay cumsum by warp scan, then the folded operands in registers ============
    // Warp w owns channels [8 w, 8 w + 8); lane l owns tokens l and l + 32 (rows that
    // differ in their low bits, so the swizzled tile accesses are conflict-free).
    {
      bool ok = wait_on(&ms.bar_la, ph_la, pend_la);
      ok = ok && wait_on(&ms.bar_raw, ph_raw, pend_raw);
      if (__syncthreads_or(!ok)) { dead = true; break; }
    }
    const bool kval = c0 < dk;
    float kb[2][8], qh[2][8], kn[2][8], vw[2][8];
    {
      float a[2][8];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (kval) {
          const float* row = la;  // element (t, i) at f32_off(t, i, R64)
          const float4 x0 = ld4(reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(row) +
                                                               f32_off(lane + 32 * m, c0, R64)));
          const float4 x1 = ld4(reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(row) +
                                                               f32_off(lane + 32 * m, c0 + 4, R64)));
          a[m][0] = x0.x; a[m][1] = x0.y; a[m][2] = x0.z; a[m][3] = x0.w;
          a[m][4] = x1.x; a[m][5] = x1.y; a[m][6] = x1.z; a[m][7] = x1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) a[m][e] = 0.f;
        }
      }
      float gtot[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float i0 = a[0][e], i1 = a[1][e];  // inclusive scans over tokens 0..31 and 32..63
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, i0, off);
          const float y1 = __shfl_up_sync(0xffffffffu, i1, off);
          if (lane >= off) {
            i0 += y0;
            i1 += y1;
          }
        }
        const float half = __shfl_sync(0xffffffffu, i0, 31);
        a[0][e] = i0;         // g at token l
        a[1][e] = i1 + half;  // g at token l + 32
        gtot[e] = __shfl_sync(0xffffffffu, a[1][e], 31);
      }
      if (lane == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) ms.gC[ob][c0 + e] = kval ? __expf(gtot[e]) : 0.f;
      }
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint32_t ro = (uint32_t)(c0 >> 6) * R64 + sw128_off(lane + 32 * m, (c0 & 63) >> 3);
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        const bool vval = c0 < dv;
        float kk[8], bgt[8], qq[8], vv[8], ww[8];
        unpack_bf16x8(kval ? *reinterpret_cast<const uint4*>(sm + RAW_K + ro) : z4, kk);
        unpack_bf16x8(kval ? *reinterpret_cast<const uint4*>(sm + RAW_B + ro) : z4, bgt);
        unpack_bf16x8(kval ? *reinterpret_cast<const uint4*>(sm + RAW_Q + ro) : z4, qq);
        unpack_bf16x8(vval ? *reinterpret_cast<const uint4*>(sm + RAW_V + ro) : z4, vv);
        unpack_bf16x8(vval ? *reinterpret_cast<const uint4*>(sm + RAW_W + ro) : z4, ww);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float G = __expf(a[m][e]), Gi = __expf(-a[m][e]);
          kb[m][e] = kk[e] * bgt[e] * G;
          qh[m][e] = qq[e] * G;
          kn[m][e] = kk[e] * Gi;
          vw[m][e] = ww[e] * vv[e];
        }
      }
    }
    // the previous chunk's last products must be done before its tiles are overwritten
    {
      bool ok = true;
      if (c > 0) ok = wait_mma();
      fence_proxy_async_smem();
      if (__syncthreads_or(!ok)) { dead = true; break; }
    }
    tc_fence_after();
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int t = lane + 32 * m;
      st4_tf32(sm + OFF_KQ + f32_off(t, c0, R128), kb[m]);
      st4_tf32(sm + OFF_KQ + f32_off(t, c0 + 4, R128), kb[m] + 4);
      st4_tf32(sm + OFF_KQ + f32_off(64 + t, c0, R128), qh[m]);
      st4_tf32(sm + OFF_KQ + f32_off(64 + t, c0 + 4, R128), qh[m] + 4);
      st4_tf32(sm + OFF_KN + f32_off(t, c0, R64), kn[m]);
      st4_tf32(sm + OFF_KN + f32_off(t, c0 + 4, R64), kn[m] + 4);
      st4_tf32(sm + OFF_T + f32_off(t, c0, R64), vw[m]);
      st4_tf32(sm + OFF_T + f32_off(t, c0 + 4, R64), vw[m] + 4);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // [A; P] = [Kb; Qh] Kn^T : M=128 (tokens of both halves), N=64 (s), K=128 (key channels)
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t ko = (uint32_t)((ks & 3) * 32);
        const uint64_t aKQ = sdesc_sw128(sbase + OFF_KQ + (ks >> 2) * R128 + ko, 16, 1024);
        const uint64_t bKN = sdesc_sw128(sbase + OFF_KN + (ks >> 2) * R64 + ko, 16, 1024);
        umma_tf32_ss(tmem + TM_AP, aKQ, bKN, ID_64, ks > 0);
      }
      commit_mma();
    }
    // ===== while the tensor cores run: transposed operands, the next chunk's raw inputs,
    // and the output store and state decay of the previous chunk ==========================
    {
      const int ch = tid & 127, part = tid >> 7;  // ch is also this thread's TMEM lane
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (part == 0) {  // Kb^T -> tensor memory
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = *reinterpret_cast<const float*>(sm + OFF_KQ + f32_off(32 * hh + x, ch, R128));
          tmem_st32(tlane + TM_KBT + 32 * hh, v);
        } else if (part == 1) {  // Vw^T -> tensor memory
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = *reinterpret_cast<const float*>(sm + OFF_T + f32_off(32 * hh + x, ch, R64));
          tmem_st32(tlane + TM_VWT + 32 * hh, v);
        } else if (part - 2 == hh) {  // Kn^T rows, tokens [32 hh, 32 hh + 32)
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = *reinterpret_cast<const float*>(sm + OFF_KN + f32_off(32 * hh + x, ch, R64));
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(sm + OFF_KNT + f32_off(ch, 32 * hh + x, R128)) =
                make_float4(v[x], v[x + 1], v[x + 2], v[x + 3]);
        }
      }
    }
    if (c > 0) {
      stage_o(c - 1);  // the log-alpha tile is free until the next chunk's copy
      decay_state(ob ^ 1);
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == TMA_TID && c > 0) store_o(c - 1);
    if (tid == 0) {
      tc_fence_after();
      // O^T = S^T Qh^T : A = S^T from tensor memory, B = Qh rows of the KQ tile
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t ko = (uint32_t)((ks & 3) * 32);
        const uint64_t bQH = sdesc_sw128(sbase + OFF_KQ + (ks >> 2) * R128 + R64 + ko, 16, 1024);
        umma_tf32_ts(tmem + TM_O + 64 * ob, tmem + TM_S + 8 * ks, bQH, ID_64, ks > 0);
      }
    }
    // the other threads read A and P out while thread 0 is still issuing
    const bool ok_ap = wait_mma();
    tc_fence_after();
    // ===== A to the solve scratch, P to its operand tile =====================================
    {
      float v[16];
      tmem_ld16(tlane + TM_AP + 16 * cq, v);
      tmem_ld_wait();
      if (qd < 2) {
        const int t = 32 * qd + lane;
#pragma unroll
        for (int x = 0; x < 16; x += 4) {
          const int s = 16 * cq + x;
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
        for (int x = 0; x < 16; x += 4) {
          float f[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) f[m] = (16 * cq + x + m <= t) ? v[x + m] : 0.f;
          st4_tf32(sm + OFF_P + f32_off(t, 16 * cq + x, R64), f);
        }
      }
    }
    if (__syncthreads_or(!ok_ap)) { dead = true; break; }
    // ===== T = (I + A)^-1: 16x16 diagonal blocks, then 32x32, then 64x64 ===================
    // Every entry above the diagonal is an explicit zero, so block products run dense.
    {
      float x[16];
      const int I = tid >> 4, cc = tid & 15;
      if (tid < 64) {
        const float* Ab = Msc + 16 * I * LDM + 16 * I;
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
          float acc0 = 0.f, acc1 = 0.f;  // two chains: even and odd columns
#pragma unroll
          for (int s4 = 0; s4 < r; s4 += 4) {
            const float4 a = ld4(Ab + r * LDM + s4);
            acc0 = fmaf(a.x, x[s4], acc0);
            if (s4 + 1 < r) acc1 = fmaf(a.y, x[s4 + 1], acc1);
            if (s4 + 2 < r) acc0 = fmaf(a.z, x[s4 + 2], acc0);
            if (s4 + 3 < r) acc1 = fmaf(a.w, x[s4 + 3], acc1);
          }
          x[r] = (r > cc) ? -(acc0 + acc1) : x[r];
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
    // The block products of the next two levels run as warp-level tf32 MMAs
    // (m16n8k8) on fragments read straight from the scratch matrices.
    {
      // 32x32 blocks: T_{2p+1,2p} = -T_{2p+1,2p+1} (A_{2p+1,2p} T_{2p,2p}), p = 0, 1;
      // warp 2 p + nt computes the 16 x 8 output columns [8 nt, 8 nt + 8) of block p.
      const int g = lane >> 2, t = lane & 3;
      const int pp = warp >> 1, nt = warp & 1;
      const int I = 2 * pp + 1, J = 2 * pp;
      float* Xp = Xsc + 16 * pp * LDX;
      if (warp < 4) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const float* Ar = Msc + (16 * I + g) * LDM + 16 * J + 8 * ks + t;
          const float* Bc = Msc + (16 * J + 8 * ks + t) * LDM + 16 * J + 8 * nt + g;
          const uint32_t a[4] = {__float_as_uint(rna_tf32(Ar[0])), __float_as_uint(rna_tf32(Ar[8 * LDM])),
                                 __float_as_uint(rna_tf32(Ar[4])), __float_as_uint(rna_tf32(Ar[8 * LDM + 4]))};
          const uint32_t b[2] = {__float_as_uint(rna_tf32(Bc[0])), __float_as_uint(rna_tf32(Bc[4 * LDM]))};
          mma_16x8x8_tf32(d, a, b);
        }
        *reinterpret_cast<float2*>(Xp + g * LDX + 8 * nt + 2 * t) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(Xp + (g + 8) * LDX + 8 * nt + 2 * t) = make_float2(d[2], d[3]);
      }
      __syncthreads();
      if (warp < 4) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const float* Ar = Msc + (16 * I + g) * LDM + 16 * I + 8 * ks + t;
          const float* Bc = Xp + (8 * ks + t) * LDX + 8 * nt + g;
          const uint32_t a[4] = {__float_as_uint(rna_tf32(Ar[0])), __float_as_uint(rna_tf32(Ar[8 * LDM])),
                                 __float_as_uint(rna_tf32(Ar[4])), __float_as_uint(rna_tf32(Ar[8 * LDM + 4]))};
          const uint32_t b[2] = {__float_as_uint(rna_tf32(Bc[0])), __float_as_uint(rna_tf32(Bc[4 * LDX]))};
          mma_16x8x8_tf32(d, a, b);
        }
        float* Tr = Msc + (16 * I + g) * LDM + 16 * J + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(Tr) = make_float2(-d[0], -d[1]);
        *reinterpret_cast<float2*>(Tr + 8 * LDM) = make_float2(-d[2], -d[3]);
      }
      __syncthreads();
    }
    {
      // 64x64: T_21 = -T_22 (A_21 T_11) with 32x32 blocks; warp 4 mt + nt (8 warps)
      // computes the 16 x 8 output tile (rows [16 mt, +16), columns [8 nt, +8)).
      const int g = lane >> 2, t = lane & 3;
      const int mt = (warp >> 2) & 1, nt = warp & 3;
      if (warp < 8) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const float* Ar = Msc + (32 + 16 * mt + g) * LDM + 8 * ks + t;
          const float* Bc = Msc + (8 * ks + t) * LDM + 8 * nt + g;
          const uint32_t a[4] = {__float_as_uint(rna_tf32(Ar[0])), __float_as_uint(rna_tf32(Ar[8 * LDM])),
                                 __float_as_uint(rna_tf32(Ar[4])), __float_as_uint(rna_tf32(Ar[8 * LDM + 4]))};
          const uint32_t b[2] = {__float_as_uint(rna_tf32(Bc[0])), __float_as_uint(rna_tf32(Bc[4 * LDM]))};
          mma_16x8x8_tf32(d, a, b);
        }
        *reinterpret_cast<float2*>(Xsc + (16 * mt + g) * LDX + 8 * nt + 2 * t) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(Xsc + (16 * mt + g + 8) * LDX + 8 * nt + 2 * t) = make_float2(d[2], d[3]);
      }
      __syncthreads();
      if (warp < 8) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const float* Ar = Msc + (32 + 16 * mt + g) * LDM + 32 + 8 * ks + t;
          const float* Bc = Xsc + (8 * ks + t) * LDX + 8 * nt + g;
          const uint32_t a[4] = {__float_as_uint(rna_tf32(Ar[0])), __float_as_uint(rna_tf32(Ar[8 * LDM])),
                                 __float_as_uint(rna_tf32(Ar[4])), __float_as_uint(rna_tf32(Ar[8 * LDM + 4]))};
          const uint32_t b[2] = {__float_as_uint(rna_tf32(Bc[0])), __float_as_uint(rna_tf32(Bc[4 * LDX]))};
          mma_16x8x8_tf32(d, a, b);
        }
        float* Tr = Msc + (32 + 16 * mt + g) * LDM + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(Tr) = make_float2(-d[0], -d[1]);
        *reinterpret_cast<float2*>(Tr + 8 * LDM) = make_float2(-d[2], -d[3]);
      }
      __syncthreads();
    }
    // T as a tf32 K-major operand [t][s]
    for (int e = tid; e < 64 * 16; e += NT) {
      const int t = e >> 4, s4 = e & 15;
      const float4 a = ld4(Msc + t * LDM + 4 * s4);
      const float f[4] = {a.x, a.y, a.z, a.w};
      st4_tf32(sm + OFF_T + f32_off(t, 4 * s4, R64), f);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == TMA_TID && c + 1 < p.nchunks) {
      bulk_wait_read_all();  // the output staging has been read
      issue_la(c + 1);
    }
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
    if (__syncthreads_or(!wait_mma())) { dead = true; break; }
    tc_fence_after();
    if (tid == TMA_TID && c + 1 < p.nchunks) issue_raw(c + 1);  // the KQ tile and the scratch are free
    // ===== W (token rows) to shared memory: thread = key channel i, one column ==========
    {
      float v[16];
      tmem_ld16(tlane + TM_W + 16 * cq, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 16; ++x)
        *reinterpret_cast<float*>(sm + OFF_KN + f32_off(16 * cq + x, jrow, R64)) = rna_tf32(v[x]);
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
    if (__syncthreads_or(!wait_mma())) { dead = true; break; }
    tc_fence_after();
    if (tid == 0) {
      // O^T += U~^T P^T : A = U~^T from tensor memory, B = P (N = t), K = s
      // S^T += U~^T Kn  : B = Kn^T rows (N = key channels)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t bP = sdesc_sw128(sbase + OFF_P + (ks >> 2) * R64 + (ks & 3) * 32, 16, 1024);
        const uint64_t bK = sdesc_sw128(sbase + OFF_KNT + (ks >> 2) * R128 + (ks & 3) * 32, 16, 1024);
        umma_tf32_ts(tmem + TM_O + 64 * ob, tmem + TM_U + 8 * ks, bP, ID_64, 1);
        umma_tf32_ts(tmem + TM_S, tmem + TM_U + 8 * ks, bK, ID_128, 1);
      }
      commit_mma();  // waited on at the start of the next chunk (or below)
    }
  }

  // ---- last chunk's output and decay, then the final state -------------------------------
  if (!dead && p.nchunks > 0) {
    if (tid == TMA_TID) bulk_wait_read_all();  // the staging tile is about to be rewritten
    if (__syncthreads_or(!wait_mma())) dead = true;
  }
  if (!dead && p.nchunks > 0) {
    tc_fence_after();
    stage_o(p.nchunks - 1);
    decay_state((p.nchunks - 1) & 1);
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == TMA_TID) store_o(p.nchunks - 1);
    if (p.S_T && jrow < dv) {
      float v[32];
      tmem_ld32(tlane + TM_S + 32 * cq, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x)
        if (32 * cq + x < dk) p.S_T[((size_t)unit * dk + 32 * cq + x) * dv + jrow] = v[x];
    }
  }
  // ---- teardown: after a give-up, let outstanding async work drain (bounded) ------------
  if ((tid == 0 || tid == TMA_TID) && ms.abort) {
    volatile int never = 0;
    if (pend_la) mbar_wait_bounded(&ms.bar_la, ph_la, &never, nullptr, WAIT_LIMIT);
    if (pend_mma) mbar_wait_bounded(&ms.bar_mma, ph_mma, &never, nullptr, WAIT_LIMIT);
    if (pend_raw) mbar_wait_bounded(&ms.bar_raw, ph_raw, &never, nullptr, WAIT_LIMIT);
  }
  if (tid == TMA_TID) bulk_wait_all();  // output stores complete before the block exits
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
  CUtensorMap mq, mk, mv, mb, mw, mla, mo;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = make_map(&mq, a.q, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mk, a.k, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mb, a.b, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mv, a.v, BF, 2, a.B, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mw, a.w, BF, 2, a.B, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, a.dk, 32, SW) &&
            make_map(&mo, a.o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, a.dv, a.dv,
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
  chunk_fwd_tc_kernel<<<a.B * a.H, NT, SMEM_BYTES, st>>>(mq, mk, mv, mb, mw, mla, mo, p);
  return cudaGetLastError();
}

}  // namespace gdn2
