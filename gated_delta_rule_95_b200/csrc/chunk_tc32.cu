// Chunkwise prefill forward at chunk size C = 32 for bf16 inputs on the 5th-generation tensor
// cores: the tcgen05 kernel's design (chunk_tc.cu) with 32-token chunks, for the chunk-size
// trade-off (snilld.dk, "POC-matrix der daekker de haarde hjoerner": latency, throughput and
// memory at C = 32, 64 and 128).  Same algorithm and notation as chunk_tc.cu (Gated
// DeltaNet-2 guide, "Chunkwise Parallel Algorithm for GPU Training"; WY form with the
// cumulative decay folded into the factors, snilld.dk, "Hvad betyder det for traening og
// inferens"):
//
//     [A; P]  = [Kb; Qh] Kn^T        T = (I + A)^-1
//     [X^T | O^T] = S^T [-Kb; Qh]^T  R^T = Vw^T + X^T      U~^T = R^T T^T
//     [O^T | S^T] += U~^T [P; Kn^T]^T                      S^T <- S^T Diag(Gamma_C)
//
// What changes with C = 32: the stacked [-Kb; Qh] tile has 64 meaningful rows; it keeps
// 128-row panels so that [A; P] is the same M = 128 product (rows 64-127 hold staging bytes,
// and the accumulator lanes they produce are never read).  The products shrink: [A; P] N = 32,
// [X^T | O^T] N = 64, U~^T N = 32 over K = 32, [O^T | S^T] N = 32 + d_k over K = 32.  The
// solve is 32 x 32 (8x8 diagonal blocks, 16-level merges, one 32-level merge) on warps 0-1,
// and U~ is issued whole once T is complete.  Tensor memory: 320 of 512 columns.  Warp
// roles, the barrier protocol and the copy schedule are those of chunk_tc.cu.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 32;
constexpr int NCOMP = 512;                      // warps 0-15: elementwise work
constexpr int NT = NCOMP + 64;                  // + the control warp and the store warp
constexpr int CTL = NCOMP;                      // the thread that issues MMAs and the input copies
constexpr int STW = NCOMP + 32;                 // the thread that issues output stores and log-alpha copies
constexpr int NSOLVE = 256;                     // warps 0-7: A read-out share, the solve (warps 0-1), U~ rounding
constexpr int BAR_COMP = 1, BAR_AUX = 3, BAR_SOLVE = 4;  // named barriers: compute warps; 8-15; 0-1
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait
constexpr float LOG2E = 1.4426950408889634f;
constexpr float G2_MIN = -115.4f;  // in-chunk cumulative log2 decay below which 2^-g leaves fp32
constexpr int PF_AHEAD = 2;        // chunks of input prefetched into L2 ahead of use

// ---- shared memory map (byte offsets from a 1024-byte aligned base) ----------------
constexpr uint32_t R32 = 32 * 128;    // a panel of 32 rows
constexpr uint32_t R128 = 128 * 128;  // a panel of 128 rows
constexpr uint32_t R160 = 160 * 128;  // a panel of 160 rows
constexpr uint32_t OFF_KQ = 0;                   // [-Kb; Qh] [t][i]: 4 panels x 128 rows (rows 0-63 used)
constexpr uint32_t OFF_KN = OFF_KQ + 4 * R128;   // Kn [s][i]: 4 panels x 32 rows (first: raw v, w)
constexpr uint32_t OFF_PK = OFF_KN + 4 * R32;    // [P; Kn^T] [t | i][s]: 1 panel x 160 rows
constexpr uint32_t OFF_T = OFF_PK + R160;        // T [t][s]: 1 panel x 32 rows
constexpr uint32_t OFF_LA = OFF_T + R32;         // log alpha [t][i] fp32 (TMA): 4 panels x 32 rows, in
                                                 // place the cumulative log2 decay; between uses the
                                                 // output tile [t][j] of a TMA store
constexpr uint32_t OFF_SCR = OFF_LA + 4 * R32;   // solve scratch: fp32 32 x LDM, then 2 x 32 x LDW
constexpr int LDM = 36;
constexpr int LDW = 8;
constexpr uint32_t TILES = OFF_SCR + (32 * LDM + 2 * 32 * LDW) * 4;
// raw bf16 staging (TMA, 128B swizzle): [32 tokens][128 channels] = 2 panels of 64 channels
constexpr uint32_t B16 = 2 * R32;
constexpr uint32_t RAW_Q = OFF_KQ, RAW_K = OFF_KQ + B16, RAW_B = OFF_KQ + 2 * B16;
constexpr uint32_t RAW_V = OFF_KN, RAW_W = OFF_KN + B16;

struct Misc {
  uint64_t bar_la, bar_raw, bar_vw;                   // TMA loads landed
  uint64_t bar_mma, bar_s, bar_drain;                 // tensor-core products done
  uint64_t bar_ops, bar_stage, bar_tdiag, bar_uround;  // compute warps -> control warp
  uint64_t bar_lastread;                              // store warp -> compute warps
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[2][128];    // Gamma at the chunk end, per key channel (chunk parity)
  alignas(16) float segtot[2][128];
};
constexpr uint32_t SMEM_BYTES = TILES + 1024 + sizeof(Misc);

// ---- tensor memory columns (fp32, 128 lanes) -------------------------------------------
constexpr uint32_t TM_AP = 0;    // [-A; P]  lanes: tokens of Kb | Qh (0-63), columns: s
constexpr uint32_t TM_U = 32;    // U~^T     lanes: value channel, columns: s
constexpr uint32_t TM_R = 64;    // R^T      } [X^T | O^T]: one N = 64 product
constexpr uint32_t TM_O = 96;    // O^T      } } [O^T | S^T]: one N = 32 + d_k product
constexpr uint32_t TM_S = 128;   // S^T        }
constexpr uint32_t TM_VW = 256;  // Vw^T, two buffers (chunk parity)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_32 = idesc_tf32(128, 32, 0, 0, 0, 0);
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);
constexpr uint32_t ID_160 = idesc_tf32(128, 160, 0, 0, 0, 0);
constexpr uint32_t ID_96 = idesc_tf32(128, 96, 0, 0, 0, 0);

struct Tc32Params {
  const __nv_bfloat16 *q, *k, *v, *b, *w;
  const float* S0;
  float* S_T;
  int T, H;
  unsigned* err;
};

__device__ __forceinline__ float rna_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ void st4_tf32(unsigned char* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(rna_tf32(f[0]), rna_tf32(f[1]), rna_tf32(f[2]), rna_tf32(f[3]));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ uint32_t tfu(float x) { return __float_as_uint(rna_tf32(x)); }
__device__ __forceinline__ float bf16_at(const unsigned char* p) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(p)) << 16);
}
__device__ __forceinline__ float2 bf16x2_at(const unsigned char* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ void st2_tf32(unsigned char* p, const float2& f) {
  *reinterpret_cast<float2*>(p) = make_float2(rna_tf32(f.x), rna_tf32(f.y));
}
__device__ __forceinline__ uint64_t kdesc(uint32_t base, uint32_t panel, int ks) {
  return sdesc_sw128(base + (uint32_t)(ks >> 2) * panel + (uint32_t)(ks & 3) * 32, 16, 1024);
}

// DK, DV: key and value head dimensions (64 or 128); d = 64 runs with the upper half of each
// operand zero, as in chunk_tc.cu.
template <int DK, int DV>
__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmLA,
                          const __grid_constant__ CUtensorMap tmO, const Tc32Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Misc& ms = *reinterpret_cast<Misc*>(sm + TILES);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int ch = tid & 127;  // channel (key i and value j) and tensor-memory lane
  const int sg = tid >> 7;   // column group of tensor-memory accesses
  const int unit = blockIdx.x, h = unit % p.H, bb = unit / p.H;
  const int len = p.T, nch = (len + C - 1) / C;
  const size_t st_sz = (size_t)DK * DV;
  constexpr int dk = DK, dv = DV;
  const bool kval = ch < dk, vval = ch < dv;

  if (tid == 0) {
    mbar_init(&ms.bar_la, 1);
    mbar_init(&ms.bar_mma, 1);
    mbar_init(&ms.bar_raw, 1);
    mbar_init(&ms.bar_vw, 1);
    mbar_init(&ms.bar_s, 1);
    mbar_init(&ms.bar_drain, 1);
    mbar_init(&ms.bar_ops, NCOMP / 32);
    mbar_init(&ms.bar_stage, NCOMP / 32);
    mbar_init(&ms.bar_tdiag, NCOMP / 32);    // R^T rounded and T complete
    mbar_init(&ms.bar_uround, NSOLVE / 32);
    mbar_init(&ms.bar_lastread, 1);
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
  const uint32_t tlane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);

  auto wait_on = [&](uint64_t* bar, uint32_t& ph) -> bool {
    const bool ok = mbar_wait_bounded(bar, ph, &ms.abort, p.err, WAIT_LIMIT);
    if (ok) ph ^= 1;
    return ok;
  };
  auto warp_arrive = [&](uint64_t* bar) {
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(bar);
  };

  if (warp == NCOMP / 32) {
    // ========================= control warp: MMAs and TMA copies =========================
    if (tid == CTL) {
      int n_raw = 0, n_vw = 0;
      auto prefetch_raw = [&](int c) {
        for (int pn = 0; pn < (dk >> 5); ++pn) tma_prefetch_l2_4d(&tmLA, 32 * pn, h, C * c, bb);
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
      auto issue_qkb = [&](int c) {
        mbar_arrive_expect_tx(&ms.bar_raw, (uint32_t)(3 * (dk >> 6)) * R32);
        for (int pn = 0; pn < (dk >> 6); ++pn) {
          tma_load_4d(sm + RAW_Q + pn * R32, &tmQ, &ms.bar_raw, 64 * pn, h, C * c, bb);
          tma_load_4d(sm + RAW_K + pn * R32, &tmK, &ms.bar_raw, 64 * pn, h, C * c, bb);
          tma_load_4d(sm + RAW_B + pn * R32, &tmB, &ms.bar_raw, 64 * pn, h, C * c, bb);
        }
        ++n_raw;
      };
      auto issue_vw = [&](int c) {
        mbar_arrive_expect_tx(&ms.bar_vw, (uint32_t)(2 * (dv >> 6)) * R32);
        for (int pn = 0; pn < (dv >> 6); ++pn) {
          tma_load_4d(sm + RAW_V + pn * R32, &tmV, &ms.bar_vw, 64 * pn, h, C * c, bb);
          tma_load_4d(sm + RAW_W + pn * R32, &tmW, &ms.bar_vw, 64 * pn, h, C * c, bb);
        }
        ++n_vw;
      };
      uint32_t ph_ops = 0, ph_stage = 0, ph_tdiag = 0, ph_uround = 0, ph_s = 0;
      bool alive = true;
      if (nch > 0) {
        issue_qkb(0);
        issue_vw(0);
        for (int cc = 1; cc <= PF_AHEAD && cc < nch; ++cc) prefetch_raw(cc);
      }
      for (int c = 0; c < nch; ++c) {
        if (c + PF_AHEAD < nch) prefetch_raw(c + PF_AHEAD);
        // [-A; P] = [-Kb; Qh] Kn^T : M = 128 (rows 0-63 the stacked tokens), N = 32, K = d_k
        if (!(alive = wait_on(&ms.bar_ops, ph_ops))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          umma_tf32_ss(tmem + TM_AP, kdesc(sbase + OFF_KQ, R128, ks), kdesc(sbase + OFF_KN, R32, ks), ID_32, ks > 0);
        umma_commit(&ms.bar_mma);
        // [X^T | O^T] = S^T [-Kb; Qh]^T : A = S^T (tensor memory), B = rows 0-63 of the KQ tile
        if (!(alive = wait_on(&ms.bar_stage, ph_stage))) break;
        tc_fence_after();
        // [A; P] has read the Kn tile: the next chunk's v, w
        if (!(alive = mbar_wait_bounded(&ms.bar_mma, (uint32_t)((3 * c) & 1), &ms.abort, p.err, WAIT_LIMIT))) break;
        if (c + 1 < nch) issue_vw(c + 1);
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          umma_tf32_ts(tmem + TM_R, tmem + TM_S + 8 * ks, kdesc(sbase + OFF_KQ, R128, ks), ID_64, ks > 0);
        umma_commit(&ms.bar_s);
        // the state product has read the KQ tile: the next chunk's q, k, b
        if (!(alive = wait_on(&ms.bar_s, ph_s))) break;
        if (c + 1 < nch) issue_qkb(c + 1);
        // U~^T = R^T T^T : A = R^T (tensor memory), B = T (N = s), K = t, once T is complete
        if (!(alive = wait_on(&ms.bar_tdiag, ph_tdiag))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_tf32_ts(tmem + TM_U, tmem + TM_R + 8 * ks, kdesc(sbase + OFF_T, R32, ks), ID_32, ks > 0);
        umma_commit(&ms.bar_mma);
        // [O^T | S^T] += U~^T [P; Kn^T]^T : one N = 32 + d_k product
        if (!(alive = wait_on(&ms.bar_uround, ph_uround))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_tf32_ts(tmem + TM_O, tmem + TM_U + 8 * ks, kdesc(sbase + OFF_PK, R160, ks), DK == 128 ? ID_160 : ID_96, 1);
        umma_commit(&ms.bar_mma);
      }
      if (ms.abort) {  // every MMA and copy issued lands before the block releases its memory
        volatile int never = 0;
        umma_commit(&ms.bar_drain);
        mbar_wait_bounded(&ms.bar_drain, 0, &never, nullptr, WAIT_LIMIT);
        if (n_raw > 0) mbar_wait_bounded(&ms.bar_raw, (uint32_t)((n_raw - 1) & 1), &never, nullptr, WAIT_LIMIT);
        if (n_vw > 0) mbar_wait_bounded(&ms.bar_vw, (uint32_t)((n_vw - 1) & 1), &never, nullptr, WAIT_LIMIT);
      }
      static_cast<void>(alive);
    }
    __syncwarp();
  } else if (warp == NCOMP / 32 + 1) {
    // ========================= store warp: output stores and log-alpha copies ===============
    if (tid == STW) {
      int n_la = 0;
      auto issue_la = [&](int c) {
        mbar_arrive_expect_tx(&ms.bar_la, (uint32_t)(C * dk * 4));
        for (int pn = 0; pn < (dk >> 5); ++pn)
          tma_load_4d(sm + OFF_LA + pn * R32, &tmLA, &ms.bar_la, 32 * pn, h, C * c, bb);
        ++n_la;
      };
      auto store_o = [&](int cc) {
        tma_store_4d(&tmO, sm + OFF_LA, 0, h, C * cc, bb);
        bulk_commit();
      };
      uint32_t ph_stage = 0;
      bool alive = true;
      if (nch > 0) issue_la(0);
      for (int c = 0; c < nch; ++c) {
        if (!(alive = wait_on(&ms.bar_stage, ph_stage))) break;
        if (c > 0) {
          store_o(c - 1);
          bulk_wait_read_all();
        }
        if (c + 1 < nch) issue_la(c + 1);
        else mbar_arrive(&ms.bar_lastread);
      }
      if (alive && nch > 0 && wait_on(&ms.bar_stage, ph_stage)) store_o(nch - 1);
      if (ms.abort && n_la > 0) {
        volatile int never = 0;
        mbar_wait_bounded(&ms.bar_la, (uint32_t)((n_la - 1) & 1), &never, nullptr, WAIT_LIMIT);
      }
      bulk_wait_all();
    }
    __syncwarp();
  } else {
    // ========================= compute warps 0-15 =========================================
    {  // entering state S0 -> S^T (lane j = ch, key-channel columns [32 sg, 32 sg + 32))
      const float* S0u = p.S0 ? p.S0 + (size_t)unit * st_sz : nullptr;
      float v[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int i = 32 * sg + x;
        v[x] = (S0u && vval && i < dk) ? S0u[(size_t)i * dv + ch] : 0.f;
      }
      tmem_st32(tlane + TM_S + 32 * sg, v);
      tmem_st_wait();
    }
    // the T operand tile: blocks above the 8x8 block diagonal stay zero for good
    for (int e = tid; e < (int)R32 / 16; e += NCOMP)
      *reinterpret_cast<float4*>(sm + OFF_T + 16 * e) = make_float4(0.f, 0.f, 0.f, 0.f);
    uint32_t ph_mma = 0, ph_s = 0;
    float* Msc = reinterpret_cast<float*>(sm + OFF_SCR);                 // solve matrix, 32 x LDM fp32
    float* Xsc = reinterpret_cast<float*>(sm + OFF_SCR + 32 * LDM * 4);  // block products, 2 x 32 x LDW
    const int lane = tid & 31;
    auto wait_mma = [&]() -> bool { return wait_on(&ms.bar_mma, ph_mma); };
    auto decay_state = [&](int gb) {  // S^T <- S^T Diag(Gamma_C of the chunk with parity gb)
      float v[32];
      tmem_ld32(tlane + TM_S + 32 * sg, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        const float4 gq = *reinterpret_cast<const float4*>(&ms.gC[gb][32 * sg + x]);
        v[x] *= gq.x;
        v[x + 1] *= gq.y;
        v[x + 2] *= gq.z;
        v[x + 3] *= gq.w;
      }
      tmem_st32(tlane + TM_S + 32 * sg, v);
    };
    // the last finished chunk's output (O^T) into the staging tile [t][j] over the decay tile
    auto stage_o = [&]() {
      float v[8];
      tmem_ld8(tlane + TM_O + 8 * sg, v);
      tmem_ld_wait();
      if (vval) {
        float* st = reinterpret_cast<float*>(sm + OFF_LA) + ch;
#pragma unroll
        for (int x = 0; x < 8; ++x) st[(8 * sg + x) * dv] = v[x];
      }
    };
    // Warps 8-15, one chunk ahead (chunk cc): thread (ch, hf) owns tokens [16 hf, 16 hf + 16).
    uint32_t ph_la = 0, ph_raw = 0, ph_vw = 0;
    auto vw_ahead = [&](int cc, bool ok) -> bool {
      const int hf = sg - 2;
      ok = ok && wait_on(&ms.bar_vw, ph_vw);
      float vw[16];
      const uint32_t pnl = (uint32_t)(ch >> 6) * R32;
      const int chk = (ch & 63) >> 3, byt = (ch & 7) * 2;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const uint32_t ro = pnl + sw128_off(16 * hf + r, chk) + byt;
        vw[r] = vval ? bf16_at(sm + RAW_V + ro) * bf16_at(sm + RAW_W + ro) : 0.f;
      }
      tmem_st16(tlane + TM_VW + 32 * (cc & 1) + 16 * hf, vw);
      tmem_st_wait();
      return ok;
    };
    auto decay_ahead = [&](int cc, bool ok) -> bool {
      const int hf = sg - 2;
      unsigned char* la_w = sm + OFF_LA;
      ok = ok && wait_on(&ms.bar_la, ph_la);
      float x[16];
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r)
        x[r] = kval ? *reinterpret_cast<const float*>(la_w + f32_off(16 * hf + r, ch, R32)) : 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        acc = fmaf(x[r], LOG2E, acc);
        x[r] = acc;
      }
      ms.segtot[hf][ch] = acc;
      named_bar_sync(BAR_AUX, NCOMP - NSOLVE);
      const float off = hf ? ms.segtot[0][ch] : 0.f;
      if (kval) {
#pragma unroll
        for (int r = 0; r < 16; ++r)
          *reinterpret_cast<float*>(la_w + f32_off(16 * hf + r, ch, R32)) = ex2_approx(x[r] + off);
      }
      if (hf == 1) {
        ms.gC[cc & 1][ch] = kval ? ex2_approx(off + acc) : 0.f;
        if (kval && off + acc < G2_MIN && p.err) atomicOr(p.err, kErrDecayRange);
      }
      return ok;
    };

    bool dead = false;
    bool ok_prev = true;
    if (nch > 0 && warp >= NSOLVE / 32) ok_prev = decay_ahead(0, vw_ahead(0, true));
    tc_fence_before();
    if (named_bar_or(BAR_COMP, NCOMP, !ok_prev)) dead = true;
    tc_fence_after();
    for (int c = 0; c < nch && !dead; ++c) {
      const int ob = c & 1;
      // ===== folded operands: thread (channel pair (2 cp, 2 cp + 1), tokens [4 ts, 4 ts + 4))
      const int cp = tid & 63, ts = tid >> 6, c2 = 2 * cp;
      const bool kv2 = c2 < dk;
      float2 nkb[4], qh[4], kn[4];
      bool ok_raw = wait_on(&ms.bar_raw, ph_raw);
      {
        const unsigned char* la_t = sm + OFF_LA;
        const uint32_t pnl = (uint32_t)(c2 >> 6) * R32;
        const int chk = (c2 & 63) >> 3, byt = (c2 & 7) * 2;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = 4 * ts + r;
          const uint32_t ro = pnl + sw128_off(t, chk) + byt;
          float2 G = make_float2(1.f, 1.f), kk = make_float2(0.f, 0.f), bg = kk, qq = kk;
          if (kv2) {
            G = *reinterpret_cast<const float2*>(la_t + f32_off(t, c2, R32));
            kk = bf16x2_at(sm + RAW_K + ro);
            bg = bf16x2_at(sm + RAW_B + ro);
            qq = bf16x2_at(sm + RAW_Q + ro);
          }
          const float2 Gi = make_float2(rcp_approx(G.x), rcp_approx(G.y));
          nkb[r] = make_float2(-(kk.x * bg.x) * G.x, -(kk.y * bg.y) * G.y);
          qh[r] = make_float2(qq.x * G.x, qq.y * G.y);
          kn[r] = make_float2(kk.x * Gi.x, kk.y * Gi.y);
        }
      }
      // every raw read must be done before the operand tiles overwrite the staging
      if (named_bar_or(BAR_COMP, NCOMP, !ok_raw)) { dead = true; break; }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = 4 * ts + r;
        st2_tf32(sm + OFF_KQ + f32_off(t, c2, R128), nkb[r]);
        st2_tf32(sm + OFF_KQ + f32_off(C + t, c2, R128), qh[r]);
        st2_tf32(sm + OFF_KN + f32_off(t, c2, R32), kn[r]);
      }
      // the previous chunk's output/state product must be done before Kn^T, O and S are touched
      const bool ok_op = (c == 0) || wait_mma();
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&ms.bar_ops);
      tc_fence_after();
      {
        // Kn^T rows 2 cp and 2 cp + 1 (rows C + i of the [P; Kn^T] panel), tokens [4 ts, +4)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float f[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) f[r] = e ? kn[r].y : kn[r].x;
          st4_tf32(sm + OFF_PK + f32_off(C + c2 + e, 4 * ts, R160), f);
        }
      }
      // ===== while [A; P] is on the tensor cores: the previous chunk's output and state decay
      if (c > 0) {
        stage_o();
        decay_state(ob ^ 1);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&ms.bar_stage);
      // ===== A (sign restored) to the solve scratch, P to its operand tile ==================
      {
        const bool ok_ap = wait_mma();
        tc_fence_after();
        float v[8];
        tmem_ld8(tlane + TM_AP + 8 * sg, v);
        tmem_ld_wait();
        if (ch < C) {
          const int t = ch;
#pragma unroll
          for (int x = 0; x < 8; x += 4) {
            const int s = 8 * sg + x;
            float4 f;
            f.x = (s + 0 < t) ? -v[x + 0] : 0.f;
            f.y = (s + 1 < t) ? -v[x + 1] : 0.f;
            f.z = (s + 2 < t) ? -v[x + 2] : 0.f;
            f.w = (s + 3 < t) ? -v[x + 3] : 0.f;
            *reinterpret_cast<float4*>(Msc + t * LDM + s) = f;
          }
        } else if (ch < 2 * C) {
          const int t = ch - C;  // P row, causal incl. the diagonal
#pragma unroll
          for (int x = 0; x < 8; x += 4) {
            float f[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) f[m] = (8 * sg + x + m <= t) ? v[x + m] : 0.f;
            st4_tf32(sm + OFF_PK + f32_off(t, 8 * sg + x, R160), f);
          }
        }
        if (named_bar_or(BAR_COMP, NCOMP, !(ok_ap && ok_op))) { dead = true; break; }
      }
      // ===== T = (I + A)^-1 on warps 0-1 (warp k: the 16-row block k by 8x8 substitution and
      // its 16-level merge; then the 32-level merge on warp-level tf32 MMAs).  Warps 8-15
      // meanwhile round R^T once the state product is done.
      bool ok_s = true;
      if (warp < 8) {
        auto put_t = [&](int row, int col, float x) {
          *reinterpret_cast<float*>(sm + OFF_T + f32_off(row, col, R32)) = rna_tf32(x);
        };
        auto put_t2 = [&](int row, int col, float x0, float x1) {
          *reinterpret_cast<float2*>(sm + OFF_T + f32_off(row, col, R32)) = make_float2(rna_tf32(x0), rna_tf32(x1));
        };
        if (warp < 2) {
          const int k = warp, g4 = lane >> 2, t4 = lane & 3;
          float* Xw = Xsc + warp * 32 * LDW;
          {
            // 8x8 diagonal blocks 2k (lanes 0-7) and 2k + 1 (lanes 8-15); lane = column
            const int r0 = 8 * (2 * k + ((lane >> 3) & 1)), col = lane & 7;
            float x[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) x[r] = (r == col) ? 1.f : 0.f;
#pragma unroll
            for (int r = 1; r < 8; ++r) {
              const float4 a0 = ld4(Msc + (r0 + r) * LDM + r0), a1 = ld4(Msc + (r0 + r) * LDM + r0 + 4);
              const float ar[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
              float acc = 0.f;
#pragma unroll
              for (int s2 = 0; s2 < r; ++s2) acc = fmaf(ar[s2], x[s2], acc);
              if (r > col) x[r] = -acc;
            }
            __syncwarp();
            if (lane < 16) {
#pragma unroll
              for (int r = 0; r < 8; ++r) {
                Msc[(r0 + r) * LDM + r0 + col] = x[r];
                put_t(r0 + r, r0 + col, x[r]);
              }
            }
            __syncwarp();
          }
          {
            // 16-level: T_{2k+1,2k} = -T_{2k+1,2k+1} (A_{2k+1,2k} T_{2k,2k})
            const int I = 16 * k + 8, J = 16 * k, row = lane >> 2, c0 = 2 * (lane & 3);
            float z0 = 0.f, z1 = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
              const float a = Msc[(I + row) * LDM + J + s2];
              const float2 tb = *reinterpret_cast<const float2*>(Msc + (J + s2) * LDM + J + c0);
              z0 = fmaf(a, tb.x, z0);
              z1 = fmaf(a, tb.y, z1);
            }
            *reinterpret_cast<float2*>(Xw + row * LDW + c0) = make_float2(z0, z1);
            __syncwarp();
            float y0 = 0.f, y1 = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
              const float tt = Msc[(I + row) * LDM + I + s2];
              const float2 xb = *reinterpret_cast<const float2*>(Xw + s2 * LDW + c0);
              y0 = fmaf(tt, xb.x, y0);
              y1 = fmaf(tt, xb.y, y1);
            }
            *reinterpret_cast<float2*>(Msc + (I + row) * LDM + J + c0) = make_float2(-y0, -y1);
            put_t2(I + row, J + c0, -y0, -y1);
          }
          // ---- 32-level merge: T_10 = -T_11 (A_10 T_00) in 16 x 16 blocks; warp n computes
          // output columns [8 n, 8 n + 8)
          named_bar_sync(BAR_SOLVE, 64);
          {
            const int n = warp;
            const int I = 16, J = 0;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const float* Ar = Msc + (I + g4) * LDM + J + 8 * ks + t4;
              const float* Bc = Msc + (J + 8 * ks + t4) * LDM + J + 8 * n + g4;
              const uint32_t a[4] = {tfu(Ar[0]), tfu(Ar[8 * LDM]), tfu(Ar[4]), tfu(Ar[8 * LDM + 4])};
              const uint32_t b2[2] = {tfu(Bc[0]), tfu(Bc[4 * LDM])};
              mma_16x8x8_tf32(d, a, b2);
            }
            __syncwarp();
            *reinterpret_cast<float2*>(Xw + g4 * LDW + 2 * t4) = make_float2(d[0], d[1]);
            *reinterpret_cast<float2*>(Xw + (g4 + 8) * LDW + 2 * t4) = make_float2(d[2], d[3]);
            __syncwarp();
            d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const float* Ar = Msc + (I + g4) * LDM + I + 8 * ks + t4;
              const float* Bc = Xw + (8 * ks + t4) * LDW + g4;
              const uint32_t a[4] = {tfu(Ar[0]), tfu(Ar[8 * LDM]), tfu(Ar[4]), tfu(Ar[8 * LDM + 4])};
              const uint32_t b2[2] = {tfu(Bc[0]), tfu(Bc[4 * LDW])};
              mma_16x8x8_tf32(d, a, b2);
            }
            const int row = I + g4, colo = J + 8 * n + 2 * t4;
            put_t2(row, colo, -d[0], -d[1]);
            put_t2(row + 8, colo, -d[2], -d[3]);
          }
          fence_proxy_async_smem();  // the T operand tile
          tc_fence_before();
          warp_arrive(&ms.bar_tdiag);
        } else {
          tc_fence_before();
          warp_arrive(&ms.bar_tdiag);
        }
        // ===== U~^T rounded to tf32 in place: the A operand of the chunk's last product ======
        const bool ok_u = wait_mma();
        tc_fence_after();
        float v[16];
        tmem_ld16(tlane + TM_U + 16 * sg, v);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = rna_tf32(v[x]);
        tmem_st16(tlane + TM_U + 16 * sg, v);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(&ms.bar_uround);
        ok_prev = ok_u;
      } else {
        // ===== R^T = Vw^T + X^T rounded to tf32 in place once the state product is done ======
        ok_s = ok_s && wait_on(&ms.bar_s, ph_s);
        tc_fence_after();
        {
          float v[16], w[16];
          tmem_ld16(tlane + TM_R + 16 * (sg - 2), v);
          tmem_ld16(tlane + TM_VW + 32 * (c & 1) + 16 * (sg - 2), w);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 16; ++x) v[x] = rna_tf32(v[x] + w[x]);
          tmem_st16(tlane + TM_R + 16 * (sg - 2), v);
          tmem_st_wait();
        }
        fence_proxy_async_smem();  // this warp's rows of the P operand tile
        tc_fence_before();
        warp_arrive(&ms.bar_tdiag);
        // ===== then one chunk ahead: Vw^T and the cumulative decay of the next chunk =========
        if (c + 1 < nch) ok_s = decay_ahead(c + 1, vw_ahead(c + 1, ok_s));
        // these warps step their phase bit past the U~ product without waiting (its barrier's
        // next phase needs them, so the parity cannot be overtaken)
        ph_mma ^= 1;
        ok_prev = ok_s;
        tc_fence_before();
      }
      if (named_bar_or(BAR_COMP, NCOMP, !ok_prev)) { dead = true; break; }
      tc_fence_after();
    }

    // ---- last chunk's output and decay, then the final state -----------------------------
    if (!dead && nch > 0) {
      uint32_t ph_lr = 0;
      const bool ok = ok_prev && wait_mma() && wait_on(&ms.bar_lastread, ph_lr);
      if (named_bar_or(BAR_COMP, NCOMP, !ok)) dead = true;
    }
    if (!dead && nch > 0) {
      tc_fence_after();
      stage_o();
      decay_state((nch - 1) & 1);
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&ms.bar_stage);
    }
    float* STu = p.S_T ? p.S_T + (size_t)unit * st_sz : nullptr;
    if (!dead && STu && vval) {
      tc_fence_after();
      float v[32];
      tmem_ld32(tlane + TM_S + 32 * sg, v);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x)
        if (32 * sg + x < dk) STu[(size_t)(32 * sg + x) * dv + ch] = v[x];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// ---- host side ------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode32() {
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
// [B, T, H, D] tensor; one box = C tokens x box_d channels of one (b, h)
bool map32(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int B, int T, int H, int D,
           int box_d, CUtensorMapSwizzle swz) {
  auto fn = encode32();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize, (cuuint64_t)T * H * D * esize};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)C, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
cudaError_t launch32(const ChunkArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mb, mw, mla, mo;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!map32(&mq, a.q, BF, 2, a.B, a.T, a.H, DK, 64, SW) || !map32(&mk, a.k, BF, 2, a.B, a.T, a.H, DK, 64, SW) ||
      !map32(&mb, a.b, BF, 2, a.B, a.T, a.H, DK, 64, SW) || !map32(&mv, a.v, BF, 2, a.B, a.T, a.H, DV, 64, SW) ||
      !map32(&mw, a.w, BF, 2, a.B, a.T, a.H, DV, 64, SW) ||
      !map32(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, DK, 32, SW) ||
      !map32(&mo, a.o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, DV, DV, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  Tc32Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.b = static_cast<const __nv_bfloat16*>(a.b);
  p.w = static_cast<const __nv_bfloat16*>(a.w);
  p.S0 = a.S0;
  p.S_T = a.S_T;
  p.T = a.T;
  p.H = a.H;
  p.err = device_error_word();
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = smem_limit_once(chunk_fwd_tc32_kernel<DK, DV>, (int)SMEM_BYTES, attr_done);
  if (e != cudaSuccess) return e;
  chunk_fwd_tc32_kernel<DK, DV><<<a.B * a.H, NT, SMEM_BYTES, st>>>(mq, mk, mv, mb, mw, mla, mo, p);
  return cudaGetLastError();
}

}  // namespace

size_t chunk_fwd_tc32_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_chunk_fwd_tc32(const ChunkArgs& a, cudaStream_t st) {
  if (!a.bf16 || a.cu_seqlens) return cudaErrorInvalidValue;
  if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
  if (a.dk == 128 && a.dv == 128) return launch32<128, 128>(a, st);
  if (a.dk == 128 && a.dv == 64) return launch32<128, 64>(a, st);
  if (a.dk == 64 && a.dv == 128) return launch32<64, 128>(a, st);
  if (a.dk == 64 && a.dv == 64) return launch32<64, 64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace gdn2
