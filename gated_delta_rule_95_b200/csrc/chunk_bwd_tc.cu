// Backward pass of the chunkwise forward on the 5th-generation tensor cores (tcgen05.mma
// kind::tf32, accumulators in tensor memory), bf16 inputs, d_k = d_v = 128, C = 64.
//
// Reverse mode of the chunk form (Gated DeltaNet-2 guide, "Chunkwise Parallel Algorithm for
// GPU Training"; WY form with the cumulative decay folded into the factors, snilld.dk, "Hvad
// betyder det for traening og inferens").  Per chunk, with entering state S and Kb = K*B*Gamma,
// Qh = Q*Gamma, Kn = K/Gamma, A, P, T = (I + A)^-1, R = Vw - Kb S, U = T R as in the forward,
// and the gradient dSn of the state leaving the chunk:
//
//     dSt = Diag(Gamma_C) dSn        dU = P^T dO + Kn dSt        dR = T^T dU (= dVw)
//     dS  = dSt + Qh^T dO - Kb^T dR  (the gradient of the state entering the chunk)
//     dP  = lower(dO U^T)            dA = strictly lower(-dR U^T)
//     dQh = dO S^T + dP Kn           dKb = -dR S^T + dA Kn
//     dKn = U dSt^T + dA^T Kb + dP^T Qh
//     dGamma_C = rowsum(dSn * (S + Kn^T U))
//
// and elementwise dq = dQh*Gamma, dk = dKb*B*Gamma + dKn/Gamma, db = dKb*K*Gamma,
// dv = dVw*W, dw = dVw*V, dlog alpha = reverse in-chunk cumsum of
// dKb*Kb + dQh*Qh - dKn*Kn plus dGamma_C*Gamma_C.
//
// Three launches.  (1) The forward's checkpoint pass (tensor-core chunk kernel): the state
// entering every chunk, and per chunk U, T^T and P^T.  (2) bwd_chain_kernel, one CTA per
// (batch, head) sweeping the chunks in reverse: the only sequential part, dS, carried
// transposed (dS^T, lanes = value channels) as an fp32 accumulator in tensor memory; per chunk
// three products (dU^T, dR^T and the dS^T update) whose A operands (dO^T, dSt^T, dU^T, -dR^T)
// live in tensor memory and whose B operands (P^T, Kn, T^T, [Qh; Kb]^T) are shared-memory
// tiles; it writes dSn and -dR of every chunk and dv, dw.  Its inputs arrive by TMA as
// panel-major tiles, each as soon as its staging is free, and its outputs leave by TMA stores.
// (3) bwd_grad_kernel, persistent (one CTA per SM) over the (batch, head, chunk) units, all
// independent: [dP; dA] = [dO; -dR] U^T, then the key-side gradients transposed (lanes = key
// channels), [dQh^T | dKb^T] = S [dO; -dR]^T + Kn^T [dP; dA]^T, dKn^T = dSt U^T +
// [Qh; Kb]^T [dP; dA], and the elementwise finish (a thread per key channel walks the chunk's
// tokens, so the reverse cumsum of dlog alpha needs no exchange beyond four segment totals);
// the next unit's copies are issued as their tiles free up, the gradients leave by TMA stores.
// Operands are rounded to tf32 (nearest) except dO, which the tensor core reads straight from
// its TMA tile; accumulation is fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 64;     // chunk size
constexpr int D = 128;    // d_k = d_v
constexpr int NTH = 512;  // 16 warps: thread t owns tensor-memory lane (channel) t mod 128 and
                          // column group t / 128 of its accesses
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait
constexpr uint32_t R64 = 64 * 128;              // an fp32 panel of 64 rows x 32 columns (8 KB)
constexpr uint32_t R128 = 128 * 128;            // an fp32 panel of 128 rows x 32 columns (16 KB)
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);
constexpr uint32_t ID_128 = idesc_tf32(128, 128, 0, 0, 0, 0);

__device__ __forceinline__ float rna(float x) {  // fp32 -> tf32, nearest (ties away), as fp32
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ void st4r(unsigned char* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(rna(a), rna(b), rna(c), rna(d));
}
// K-major operand descriptor of k-step ks (8 tf32) in a tile of 32-column panels
__device__ __forceinline__ uint64_t kdesc(uint32_t base, uint32_t panel, int ks) {
  return sdesc_sw128(base + (uint32_t)(ks >> 2) * panel + (uint32_t)(ks & 3) * 32, 16, 1024);
}

#ifdef GDN2_STAMPS
// Instrumented build (GDN2_STAMPS): clock64 at fixed points, written by thread 0 into
// [row][slot] of a 64 x 32 array: the dS sweep of the first CTA by chunk (slots 0-12), the
// per-chunk pass by CTA (the second unit of the first 64 CTAs, slots 16-22).
#define TC_STAMP(on, row, slot)                                                               \
  do {                                                                                        \
    if (p.stamps && (on) && threadIdx.x == 0 && (row) >= 0 && (row) < 64)                     \
      p.stamps[(size_t)(row) * 32 + (slot)] = (unsigned long long)clock64();                  \
  } while (0)
#else
#define TC_STAMP(on, row, slot) \
  do {                          \
  } while (0)
#endif

// ============================== (2) the dS sweep ==========================================
struct ChainParams {
  const float* dS_T;  // [B H][d_k][d_v] or NULL
  float* dS0;         // [B H][d_k][d_v] or NULL
  float* dsn;         // [B H][chunk][d_k][d_v]: gradient of the state leaving each chunk
  int T, H, nch;
  unsigned* err;
  unsigned long long* stamps;  // instrumented build only
};
struct ChainMaps {  // panel-major token tiles (q, k, b, v, w bf16; log alpha, dO fp32), T^T, P^T;
                    // the stores of dv, dw (fp32 tokens) and -dR
  CUtensorMap q, k, b, v, w, la, dO, tt, pt, dv, dw, nr;
};

// shared memory (byte offsets from a 1024-byte aligned base)
constexpr uint32_t K1_KN = 0;                 // Kn [t][i]: 4 panels x 64 rows
constexpr uint32_t K1_KQT = K1_KN + 4 * R64;  // [Qh; Kb]^T [i][t']: 4 panels x 128 rows
constexpr uint32_t K1_Y = K1_KQT + 4 * R128;  // dO [t][j] (fp32, 4 panels), v, w (bf16, 2 panels each)
constexpr uint32_t K1_TP = K1_Y + 8 * R64;    // T^T [s][t] and P^T [t][s]: 2 + 2 panels x 64 rows
constexpr uint32_t K1_TILES = K1_TP + 4 * R64;
// staging of the raw log alpha, k, q, b over the Kn and [Qh; Kb]^T tiles they become
constexpr uint32_t K1_RLA = 0, K1_RK = 4 * R64, K1_RQ = 6 * R64, K1_RB = 8 * R64;
constexpr uint32_t K1_DO = K1_Y, K1_RV = K1_Y + 4 * R64, K1_RW = K1_Y + 6 * R64;
// output staging (fp32 [t][j], 4 panels each) for TMA stores: dv over dO, dw over v and w,
// -dR over T^T and P^T (each read before it is overwritten)
constexpr uint32_t K1_ODV = K1_DO, K1_ODW = K1_RV, K1_ONR = K1_TP;
struct ChainMisc {
  uint64_t bar_xa, bar_xq, bar_xb, bar_y, bar_tp, bar_mma, bar_dsa, bar_drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[D];
  alignas(16) float seg[4][D];
};
constexpr uint32_t K1_SMEM = K1_TILES + 1024 + sizeof(ChainMisc);
// tensor memory columns (lanes = value channels j)
constexpr uint32_t K1_TDS = 0;     // dS^T fp32 accumulator [j][i]
constexpr uint32_t K1_TDSR = 128;  // dSt^T rounded [j][i]
constexpr uint32_t K1_TDO = 256;   // dO^T rounded [j][t]
constexpr uint32_t K1_TDU = 320;   // dU^T [j][t]
constexpr uint32_t K1_TDR = 384;   // dR^T [j][s], then -dR^T rounded

__global__ void __launch_bounds__(NTH, 1) bwd_chain_kernel(const __grid_constant__ ChainMaps mp, const ChainParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  ChainMisc& ms = *reinterpret_cast<ChainMisc*>(sm + K1_TILES);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, ln = tid & 127, cg = tid >> 7, lane = tid & 31;
  const int bh = blockIdx.x, h = bh % p.H, bb = bh / p.H, nch = p.nch;
  const bool st0 = blockIdx.x == 0;
  static_cast<void>(st0);

  // The copies of chunk cc, one per lane of warp 0 (lane 0 posts the byte count first):
  // X = raw log alpha, k, q, b; Y = dO, v, w; TP = T^T, P^T.
  // X in three parts, each as soon as its staging is free: log alpha over the Kn tile (read
  // by the dU product), k and q over the Qh half of [Qh; Kb]^T (read by the first part of the
  // dS update), b over the Kb half (read by its last part)
  auto issue_xa = [&](int cc) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&ms.bar_xa, 4 * R64);
      tma_load_5d(sm + K1_RLA, &mp.la, &ms.bar_xa, 0, C * cc, 0, h, bb);
    }
    __syncwarp();
  };
  auto issue_xq = [&](int cc) {
    if (lane == 0) mbar_arrive_expect_tx(&ms.bar_xq, 2 * 2 * R64);
    __syncwarp();
    if (lane == 0) tma_load_5d(sm + K1_RK, &mp.k, &ms.bar_xq, 0, C * cc, 0, h, bb);
    else if (lane == 1) tma_load_5d(sm + K1_RQ, &mp.q, &ms.bar_xq, 0, C * cc, 0, h, bb);
    __syncwarp();
  };
  auto issue_xb = [&](int cc) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&ms.bar_xb, 2 * R64);
      tma_load_5d(sm + K1_RB, &mp.b, &ms.bar_xb, 0, C * cc, 0, h, bb);
    }
    __syncwarp();
  };
  auto issue_y = [&](int cc) {
    if (lane == 0) mbar_arrive_expect_tx(&ms.bar_y, 4 * R64 + 2 * 2 * R64);
    __syncwarp();
    if (lane == 0) tma_load_5d(sm + K1_DO, &mp.dO, &ms.bar_y, 0, C * cc, 0, h, bb);
    else if (lane == 1) tma_load_5d(sm + K1_RV, &mp.v, &ms.bar_y, 0, C * cc, 0, h, bb);
    else if (lane == 2) tma_load_5d(sm + K1_RW, &mp.w, &ms.bar_y, 0, C * cc, 0, h, bb);
  };
  auto issue_tp = [&](int cc) {
    const int row = (bh * nch + cc) * C;
    if (lane == 0) mbar_arrive_expect_tx(&ms.bar_tp, 4 * R64);
    __syncwarp();
    if (lane == 0) tma_load_3d(sm + K1_TP, &mp.tt, &ms.bar_tp, 0, row, 0);
    else if (lane == 1) tma_load_3d(sm + K1_TP + 2 * R64, &mp.pt, &ms.bar_tp, 0, row, 0);
  };
  auto prefetch = [&](int cc) {  // every input of chunk cc into L2, one lane per tensor
    const int row = (bh * nch + cc) * C;
    switch (lane) {
      case 0: tma_prefetch_l2_5d(&mp.la, 0, C * cc, 0, h, bb); break;
      case 1: tma_prefetch_l2_5d(&mp.k, 0, C * cc, 0, h, bb); break;
      case 2: tma_prefetch_l2_5d(&mp.q, 0, C * cc, 0, h, bb); break;
      case 3: tma_prefetch_l2_5d(&mp.b, 0, C * cc, 0, h, bb); break;
      case 4: tma_prefetch_l2_5d(&mp.dO, 0, C * cc, 0, h, bb); break;
      case 5: tma_prefetch_l2_5d(&mp.v, 0, C * cc, 0, h, bb); break;
      case 6: tma_prefetch_l2_5d(&mp.w, 0, C * cc, 0, h, bb); break;
      case 7: tma_prefetch_l2_3d(&mp.tt, 0, row, 0); break;
      case 8: tma_prefetch_l2_3d(&mp.pt, 0, row, 0); break;
      default: break;
    }
  };

  if (tid == 0) {
    mbar_init(&ms.bar_xa, 1);
    mbar_init(&ms.bar_xq, 1);
    mbar_init(&ms.bar_xb, 1);
    mbar_init(&ms.bar_dsa, 1);
    mbar_init(&ms.bar_y, 1);
    mbar_init(&ms.bar_tp, 1);
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
  // copies issued (warp 0): their count per barrier, for the drain after a give-up
  int n_xa = 0, n_xq = 0, n_xb = 0, n_y = 0, n_tp = 0;
  uint32_t ph_xa = 0, ph_xq = 0, ph_xb = 0, ph_y = 0, ph_tp = 0, ph_mma = 0, ph_dsa = 0;
  if (warp == 0 && nch > 0) {
    issue_xa(nch - 1);
    issue_xq(nch - 1);
    issue_xb(nch - 1);
    issue_y(nch - 1);
    issue_tp(nch - 1);
    ++n_xa, ++n_xq, ++n_xb, ++n_y, ++n_tp;
    if (nch > 1) prefetch(nch - 2);
  }
  // completion of a barrier phase: warp 0 polls (a suspended wait wakes too late for this
  // chain of short steps), the block follows through a hardware barrier; true for every
  // thread unless the wait gave up
  auto wait_all = [&](uint64_t* bar, uint32_t& ph) -> bool {
    bool ok = true;
    if (warp == 0) ok = mbar_wait_spin(bar, ph, &ms.abort, p.err, WAIT_LIMIT);
    ph ^= 1;
    return !__syncthreads_or(!ok);
  };
  // every thread's tensor-memory and shared-memory writes visible to the next MMA; false
  // if any thread's wait gave up
  auto sync_ok = [&](bool ok) -> bool {
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    const bool bad = __syncthreads_or(!ok);
    tc_fence_after();
    return !bad;
  };

  // dS^T of the last chunk's end: dS_T^T (lane j, key columns [32 cg, 32 cg + 32))
  {
    float v[32];
#pragma unroll
    for (int x = 0; x < 32; ++x)
      v[x] = p.dS_T ? __ldg(p.dS_T + ((size_t)bh * D + 32 * cg + x) * D + ln) : 0.f;
    tmem_st32(tl + K1_TDS + 32 * cg, v);
  }
  bool dead = !sync_ok(true);
  const uint32_t rb = (uint32_t)(ln >> 6) * R64 + (uint32_t)(ln & 7) * 2;  // bf16 staging: channel ln
  const int chk = (ln & 63) >> 3;
  auto bf_at = [&](uint32_t base, int t) -> float {
    return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(sm + base + rb + sw128_off(t, chk)))
                           << 16);
  };

  for (int c = nch - 1; c >= 0 && !dead; --c) {
    const int n = min(C, p.T - C * c);  // tokens of this chunk inside the sequence
    TC_STAMP(st0, c, 0);
    if (warp == 0) {
      // the previous chunk's stores have read their staging (over T^T, P^T and dO, v, w):
      // this chunk's copies of those
      if (c < nch - 1) {
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        issue_tp(c);
        issue_y(c);
        ++n_tp, ++n_y;
      }
      if (c >= 2) prefetch(c - 2);
    }
    // ===== build: thread (i = ln, cg) over the tokens [16 cg, 16 cg + 16) ===================
    if (!wait_all(&ms.bar_xa, ph_xa) || !wait_all(&ms.bar_xq, ph_xq) || !wait_all(&ms.bar_xb, ph_xb)) {
      dead = true;
      break;
    }
    TC_STAMP(st0, c, 1);
    float g[16], kq[16], qq[16], bq[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int t = 16 * cg + r;
      g[r] = *reinterpret_cast<const float*>(sm + K1_RLA + f32_off(t, ln, R64));
      kq[r] = bf_at(K1_RK, t);
      qq[r] = bf_at(K1_RQ, t);
      bq[r] = bf_at(K1_RB, t);
    }
#pragma unroll
    for (int r = 1; r < 16; ++r) g[r] += g[r - 1];
    ms.seg[cg][ln] = g[15];
    __syncthreads();  // (also: every read of the raw staging is done)
    TC_STAMP(st0, c, 2);
    float off = 0.f, tot = 0.f;
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4) {
      const float sv = ms.seg[s4][ln];
      if (s4 < cg) off += sv;
      tot += sv;
    }
    if (cg == 0) ms.gC[ln] = __expf(tot);
    if (!wait_all(&ms.bar_y, ph_y)) { dead = true; break; }
    {
      // dO^T rounded into tensor memory (lane j = ln); rows past the sequence read zero
      float dv16[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) dv16[r] = rna(*reinterpret_cast<const float*>(sm + K1_DO + f32_off(16 * cg + r, ln, R64)));
      tmem_st16(tl + K1_TDO + 16 * cg, dv16);
    }
    {
      float qh[16], kb[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float G = __expf(off + g[r]), Gi = __expf(-(off + g[r]));
        qh[r] = qq[r] * G;
        kb[r] = kq[r] * bq[r] * G;
        *reinterpret_cast<float*>(sm + K1_KN + f32_off(16 * cg + r, ln, R64)) = rna(kq[r] * Gi);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        st4r(sm + K1_KQT + f32_off(ln, 16 * cg + 4 * m, R128), qh[4 * m], qh[4 * m + 1], qh[4 * m + 2],
             qh[4 * m + 3]);
        st4r(sm + K1_KQT + f32_off(ln, C + 16 * cg + 4 * m, R128), kb[4 * m], kb[4 * m + 1], kb[4 * m + 2],
             kb[4 * m + 3]);
      }
    }
    __syncthreads();  // gC
    TC_STAMP(st0, c, 3);
    // the first part of dU^T, dO^T P, goes as soon as the dO^T columns and P^T are in place
    if (!sync_ok(true)) { dead = true; break; }
    if (warp == 0) {
      const bool ok = mbar_wait_spin(&ms.bar_tp, ph_tp, &ms.abort, p.err, WAIT_LIMIT);
      ph_tp ^= 1;
      if (ok && lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_tf32_ts(tmem + K1_TDU, tmem + K1_TDO + 8 * ks, kdesc(sbase + K1_TP + 2 * R64, R64, ks), ID_64, ks > 0);
      }
      __syncwarp();
    }
    // ===== dSn (the state gradient leaving this chunk) out; dSt^T = dS^T Diag(Gamma_C) ======
    {
      float v[32], r32[32];
      tmem_ld32(tl + K1_TDS + 32 * cg, v);
      tmem_ld_wait();
      float* dst = p.dsn + ((size_t)bh * nch + c) * D * D + ln;
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int i = 32 * cg + x;
        dst[(size_t)i * D] = v[x];
        v[x] *= ms.gC[i];
        r32[x] = rna(v[x]);
      }
      tmem_st32(tl + K1_TDS + 32 * cg, v);
      tmem_st32(tl + K1_TDSR + 32 * cg, r32);
    }
    TC_STAMP(st0, c, 4);
    if (!sync_ok(true)) { dead = true; break; }
    // ===== dU^T += dSt^T Kn^T =================================================================
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        umma_tf32_ts(tmem + K1_TDU, tmem + K1_TDSR + 8 * ks, kdesc(sbase + K1_KN, R64, ks), ID_64, 1);
      umma_commit(&ms.bar_mma);
    }
    TC_STAMP(st0, c, 5);
    if (!wait_all(&ms.bar_mma, ph_mma)) { dead = true; break; }
    tc_fence_after();
    TC_STAMP(st0, c, 6);
    // the Kn tile is read: the next chunk's log alpha over it
    if (warp == 0 && c >= 1) {
      issue_xa(c - 1);
      ++n_xa;
    }
    {
      float v[16];
      tmem_ld16(tl + K1_TDU + 16 * cg, v);
      tmem_ld_wait();
#pragma unroll
      for (int r = 0; r < 16; ++r) v[r] = rna(v[r]);
      tmem_st16(tl + K1_TDU + 16 * cg, v);
    }
    if (!sync_ok(true)) { dead = true; break; }
    // ===== dR^T = dU^T T =======================================================================
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + K1_TDR, tmem + K1_TDU + 8 * ks, kdesc(sbase + K1_TP, R64, ks), ID_64, ks > 0);
      umma_commit(&ms.bar_mma);
      // the first part of the dS^T update, dS^T += dO^T Qh, runs behind it (tracked by the
      // next commit)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ts(tmem + K1_TDS, tmem + K1_TDO + 8 * ks, kdesc(sbase + K1_KQT, R128, ks), ID_128, 1);
      umma_commit(&ms.bar_dsa);
    }
    TC_STAMP(st0, c, 7);
    if (!wait_all(&ms.bar_mma, ph_mma)) { dead = true; break; }
    tc_fence_after();
    TC_STAMP(st0, c, 8);
    // ===== -dR^T rounded in place (the A operand of the update); dv = dR w, dw = dR v and -dR
    // staged for TMA stores (v and w are read before their staging is overwritten)
    {
      float v[16], nv[16], wv[16], vv[16];
      tmem_ld16(tl + K1_TDR + 16 * cg, v);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        wv[r] = bf_at(K1_RW, 16 * cg + r);
        vv[r] = bf_at(K1_RV, 16 * cg + r);
      }
      tmem_ld_wait();
#pragma unroll
      for (int r = 0; r < 16; ++r) nv[r] = rna(-v[r]);
      tmem_st16(tl + K1_TDR + 16 * cg, nv);
      __syncthreads();  // every read of v and w is done
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const uint32_t o = f32_off(16 * cg + r, ln, R64);
        *reinterpret_cast<float*>(sm + K1_ODV + o) = v[r] * wv[r];
        *reinterpret_cast<float*>(sm + K1_ODW + o) = v[r] * vv[r];
        *reinterpret_cast<float*>(sm + K1_ONR + o) = nv[r];
      }
    }
    if (!sync_ok(true)) { dead = true; break; }
    // the first part of the update has read the Qh half of [Qh; Kb]^T: the next chunk's k, q
    if (warp == 0) {
      const bool ok = mbar_wait_spin(&ms.bar_dsa, ph_dsa, &ms.abort, p.err, WAIT_LIMIT);
      ph_dsa ^= 1;
      if (ok && c >= 1) {
        issue_xq(c - 1);
        ++n_xq;
      }
    }
    // ===== dS^T += -dR^T Kb: the update completes ==============================================
    if (tid == 0) {
#pragma unroll
      for (int ks = 8; ks < 16; ++ks)
        umma_tf32_ts(tmem + K1_TDS, tmem + K1_TDR + 8 * (ks - 8), kdesc(sbase + K1_KQT, R128, ks), ID_128, 1);
      umma_commit(&ms.bar_mma);
    }
    // the stores (rows past the sequence are clipped); the next chunk copies T^T, P^T and
    // dO, v, w over their staging once they have read it
    if (tid == 0) {
      tma_store_5d(&mp.dv, sm + K1_ODV, 0, C * c, 0, h, bb);
      tma_store_5d(&mp.dw, sm + K1_ODW, 0, C * c, 0, h, bb);
      tma_store_3d(&mp.nr, sm + K1_ONR, 0, (bh * nch + c) * C, 0);
      bulk_commit();
    }
    TC_STAMP(st0, c, 9);
    if (!wait_all(&ms.bar_mma, ph_mma)) { dead = true; break; }
    // the Kb half of [Qh; Kb]^T is read: the next chunk's b over it
    if (warp == 0 && c >= 1) {
      issue_xb(c - 1);
      ++n_xb;
    }
    TC_STAMP(st0, c, 10);
    tc_fence_after();
  }
  // the gradient of the entering state
  if (!dead && p.dS0) {
    float v[32];
    tmem_ld32(tl + K1_TDS + 32 * cg, v);
    tmem_ld_wait();
#pragma unroll
    for (int x = 0; x < 32; ++x) p.dS0[((size_t)bh * D + 32 * cg + x) * D + ln] = v[x];
  }
  if (tid == 0) bulk_wait_all();  // the stores complete before the block exits
  // after a give-up: every MMA and copy issued lands before the block releases its memory
  if (tid == 0 && ms.abort) {
    volatile int never = 0;
    umma_commit(&ms.bar_drain);
    mbar_wait_bounded(&ms.bar_drain, 0, &never, nullptr, WAIT_LIMIT);
    if (n_xa > 0) mbar_wait_bounded(&ms.bar_xa, (uint32_t)((n_xa - 1) & 1), &never, nullptr, WAIT_LIMIT);
    if (n_xq > 0) mbar_wait_bounded(&ms.bar_xq, (uint32_t)((n_xq - 1) & 1), &never, nullptr, WAIT_LIMIT);
    if (n_xb > 0) mbar_wait_bounded(&ms.bar_xb, (uint32_t)((n_xb - 1) & 1), &never, nullptr, WAIT_LIMIT);
    if (n_y > 0) mbar_wait_bounded(&ms.bar_y, (uint32_t)((n_y - 1) & 1), &never, nullptr, WAIT_LIMIT);
    if (n_tp > 0) mbar_wait_bounded(&ms.bar_tp, (uint32_t)((n_tp - 1) & 1), &never, nullptr, WAIT_LIMIT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ============================== (3) the gradients, per chunk ==============================
struct GradParams {
  const float* S;    // [B H][chunk][d_k][d_v]: entering states
  const float* dsn;  // [B H][chunk][d_k][d_v]
  int T, H, nch, units;
  unsigned* err;
  unsigned long long* stamps;  // instrumented build only
};

// shared memory: the operand tiles, and the staging of one unit's raw inputs (TMA, 128B
// swizzle) over the two [dP; dA] tiles, which are written only after the inputs are read
constexpr uint32_t K2_DR = 0;                   // [dO; -dR] [t'][j]: 4 panels x 128 rows
constexpr uint32_t K2_U = K2_DR + 4 * R128;     // U [s][j]: 4 panels x 64 rows
constexpr uint32_t K2_KNT = K2_U + 4 * R64;     // Kn^T [i][s]: 2 panels x 128 rows
constexpr uint32_t K2_PA = K2_KNT + 2 * R128;   // [dP; dA] [t'][s]: 2 panels x 128 rows
constexpr uint32_t K2_PAT = K2_PA + 2 * R128;   // [dP; dA]^T [s][t']: 4 panels x 64 rows
constexpr uint32_t K2_RB = K2_PAT + 4 * R64;    // raw b staging (bf16 [t][i], 2 panels of 64 channels)
constexpr uint32_t K2_TILES = K2_RB + 2 * R64;
constexpr uint32_t K2_RLA = K2_PA;              // raw log alpha staging (fp32 [t][i], 4 panels of 32)
constexpr uint32_t K2_RK = K2_PAT, K2_RQ = K2_PAT + 2 * R64;  // raw k, q staging (bf16)
constexpr uint32_t K2_TX = 12 * R64 + 4 * R64 + 3 * 2 * R64;  // bytes of one unit's TMA loads
// output staging of dq, dk, db, dlog alpha (fp32 [t][i], 4 panels of 32 channels each), over
// the tiles the finished products have read
constexpr uint32_t K2_ODQ = K2_U, K2_ODK = K2_KNT, K2_ODB = K2_PA, K2_ODLA = K2_PAT;
constexpr uint32_t K2_TX_DR = 8 * R64;                  // bytes of one unit's dO and -dR copies
constexpr uint32_t K2_TX_REST = K2_TX - K2_TX_DR;       // U and the raw inputs
struct GradMisc {
  uint64_t bar_ld, bar_dr, bar_mma, bar_drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[D];
  alignas(16) float seg[4][D];
  alignas(16) float dot1[4][D];  // sum_j dSn S, per column group
  alignas(16) float dotx[4][D];  // sum_s Kn (dSt U^T), per column group
  alignas(16) float tot[4][D];   // segment totals of the dlog alpha terms
};
constexpr uint32_t K2_SMEM = K2_TILES + 1024 + sizeof(GradMisc);
// tensor memory columns
constexpr uint32_t K2_SX = 0;    // S [i][j] rounded, then dSt [i][j] rounded (lanes: key channel)
constexpr uint32_t K2_KQ = 128;  // [Qh^T | Kb^T] [i][t'] rounded
constexpr uint32_t K2_PX = 256;  // [dP; dA] [t'][s] (lanes: stacked tokens), then X = dSt U^T [i][s]
constexpr uint32_t K2_QK = 320;  // [dQh^T | dKb^T] [i][t']
constexpr uint32_t K2_Y = 448;   // [Qh; Kb]^T [dP; dA] [i][s]

// Persistent: CTA r takes the units (batch, head, chunk) r, r + grid, ...; the next unit's
// dO and -dR are copied once the current unit's first products are done, its U and raw
// inputs once the current outputs have left their staging, and its states are prefetched
// into L2 meanwhile.
__global__ void __launch_bounds__(NTH, 1)
    bwd_grad_kernel(const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmNR,
                    const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ CUtensorMap tmDQ,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDB,
                    const __grid_constant__ CUtensorMap tmDLA, const GradParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  GradMisc& ms = *reinterpret_cast<GradMisc*>(sm + K2_TILES);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, ln = tid & 127, cg = tid >> 7, lane = tid & 31;
  const int stride = gridDim.x;

  // The copies of unit u, one per lane of warp 0 (lane 0 posts the byte count first), on two
  // barriers: dO (rows past the sequence read zero) and -dR by panel into the stacked tile,
  // issued as soon as the previous unit's first products have read that tile; U and the raw
  // q, k, b, log alpha as whole panel-major tiles, once the previous unit's outputs have
  // left their staging.
  auto issue_dr = [&](int u) {
    const int c = u % p.nch, bh = u / p.nch, h = bh % p.H, bb = bh / p.H, l = tid & 31;
    if (l == 0) mbar_arrive_expect_tx(&ms.bar_dr, K2_TX_DR);
    __syncwarp();
    if (l < 4) tma_load_4d(sm + K2_DR + l * R128, &tmDO, &ms.bar_dr, 32 * l, h, C * c, bb);
    else if (l < 8) tma_load_2d(sm + K2_DR + (l - 4) * R128 + R64, &tmNR, &ms.bar_dr, 32 * (l - 4), u * C);
  };
  auto issue_rest = [&](int u) {
    const int c = u % p.nch, bh = u / p.nch, h = bh % p.H, bb = bh / p.H, l = tid & 31;
    if (l == 0) mbar_arrive_expect_tx(&ms.bar_ld, K2_TX_REST);
    __syncwarp();
    if (l == 0) tma_load_3d(sm + K2_U, &tmU, &ms.bar_ld, 0, u * C, 0);
    else if (l == 1) tma_load_5d(sm + K2_RLA, &tmLA, &ms.bar_ld, 0, C * c, 0, h, bb);
    else if (l == 2) tma_load_5d(sm + K2_RK, &tmK, &ms.bar_ld, 0, C * c, 0, h, bb);
    else if (l == 3) tma_load_5d(sm + K2_RQ, &tmQ, &ms.bar_ld, 0, C * c, 0, h, bb);
    else if (l == 4) tma_load_5d(sm + K2_RB, &tmB, &ms.bar_ld, 0, C * c, 0, h, bb);
  };
  // the entering state and state gradient of unit u into L2 (4 + 4 bulk prefetches of 16 KB)
  auto prefetch_states = [&](int u) {
    if (tid < 8) {
      const float* src = (tid < 4 ? p.S : p.dsn) + (size_t)u * D * D + (size_t)(tid & 3) * (D * D / 4);
      bulk_prefetch_l2(src, D * D);
    }
  };

  if (tid == 0) {
    mbar_init(&ms.bar_ld, 1);
    mbar_init(&ms.bar_dr, 1);
    mbar_init(&ms.bar_mma, 1);
    mbar_init(&ms.bar_drain, 1);
    fence_mbar_init();
    ms.abort = 0;
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmNR);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmLA);
    tma_prefetch_desc(&tmDQ);
    tma_prefetch_desc(&tmDK);
    tma_prefetch_desc(&tmDB);
    tma_prefetch_desc(&tmDLA);
  }
  __syncthreads();  // the barrier initialised before the copies use it
  if (warp == 0 && (int)blockIdx.x < p.units) {
    issue_dr(blockIdx.x);
    issue_rest(blockIdx.x);
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
  uint32_t ph_mma = 0, ph_ld = 0, ph_dr = 0;
  // copies issued / waited on each barrier (thread 0), for the drain after a give-up
  int n_ld = (int)blockIdx.x < p.units ? 1 : 0, n_ld_done = 0, n_dr = n_ld, n_dr_done = 0;
  auto sync_ok = [&](bool ok) -> bool {
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    const bool bad = __syncthreads_or(!ok);
    tc_fence_after();
    return !bad;
  };
  // completion of a barrier phase: warp 0 polls (a suspended wait wakes too late for these
  // short steps), the block follows through a hardware barrier
  auto wait_all = [&](uint64_t* bar, uint32_t& ph) -> bool {
    bool ok = true;
    if (warp == 0) ok = mbar_wait_spin(bar, ph, &ms.abort, p.err, WAIT_LIMIT);
    ph ^= 1;
    return !__syncthreads_or(!ok);
  };
  bool dead = false;
  int it = 0;
  for (int u = blockIdx.x; u < p.units && !dead; u += stride, ++it) {
    const int c = u % p.nch, bh = u / p.nch, h = bh % p.H, bb = bh / p.H;
    const int n = min(C, p.T - C * c);
    const int srow = it == 1 ? (int)blockIdx.x : 64;  // stamps: the second unit of the first CTAs
    static_cast<void>(srow);
    TC_STAMP(true, srow, 16);
    // S and dSn rows of this unit (L2), in flight during the wait for the copies
    float4 s4[8], d4[8];
    {
      const float4* Sr = reinterpret_cast<const float4*>(p.S + ((size_t)u * D + ln) * D + 32 * cg);
      const float4* Dr = reinterpret_cast<const float4*>(p.dsn + ((size_t)u * D + ln) * D + 32 * cg);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        s4[m] = __ldg(Sr + m);
        d4[m] = __ldg(Dr + m);
      }
    }
    if (!wait_all(&ms.bar_ld, ph_ld)) { dead = true; break; }
    if (tid == 0) ++n_ld_done;
    TC_STAMP(true, srow, 17);
    // S (rounded) into tensor memory; the dGamma_C term sum_j dSn S
    {
      float sv[32], d1 = 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float se[4] = {s4[m].x, s4[m].y, s4[m].z, s4[m].w}, de[4] = {d4[m].x, d4[m].y, d4[m].z, d4[m].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sv[4 * m + e] = rna(se[e]);
          d1 = fmaf(de[e], se[e], d1);
        }
      }
      ms.dot1[cg][ln] = d1;
      tmem_st32(tl + K2_SX + 32 * cg, sv);
    }
    // ===== operands: thread (i = ln, cg) over the tokens [16 cg, 16 cg + 16) =================
    float G[16];  // Gamma of this thread's tokens (key channel ln)
    {
      float kq[16], qq[16], bq[16];
      const uint32_t rb = (uint32_t)(ln >> 6) * R64 + (uint32_t)(ln & 7) * 2;
      const int chk = (ln & 63) >> 3;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int t = 16 * cg + r;
        G[r] = *reinterpret_cast<const float*>(sm + K2_RLA + f32_off(t, ln, R64));
        const uint32_t o = rb + sw128_off(t, chk);
        kq[r] = __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(sm + K2_RK + o)) << 16);
        qq[r] = __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(sm + K2_RQ + o)) << 16);
        bq[r] = __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(sm + K2_RB + o)) << 16);
      }
#pragma unroll
      for (int r = 1; r < 16; ++r) G[r] += G[r - 1];
      ms.seg[cg][ln] = G[15];
      __syncthreads();
      float off = 0.f, tot = 0.f;
#pragma unroll
      for (int s4i = 0; s4i < 4; ++s4i) {
        const float sv = ms.seg[s4i][ln];
        if (s4i < cg) off += sv;
        tot += sv;
      }
      float qh[16], kb[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float Gi = __expf(-(off + G[r]));
        G[r] = __expf(off + G[r]);
        qh[r] = rna(qq[r] * G[r]);
        kb[r] = rna(kq[r] * bq[r] * G[r]);
        kq[r] *= Gi;  // Kn
      }
      tmem_st16(tl + K2_KQ + 16 * cg, qh);
      tmem_st16(tl + K2_KQ + C + 16 * cg, kb);
#pragma unroll
      for (int m = 0; m < 4; ++m)
        st4r(sm + K2_KNT + f32_off(ln, 16 * cg + 4 * m, R128), kq[4 * m], kq[4 * m + 1], kq[4 * m + 2],
             kq[4 * m + 3]);
      if (cg == 0) ms.gC[ln] = __expf(tot);
    }
    TC_STAMP(true, srow, 18);
    // (every raw read is done before the [dP; dA] tiles overwrite the staging: the barriers below)
    if (!sync_ok(true)) { dead = true; break; }
    // ===== [dP; dA] = [dO; -dR] U^T and [dQh^T | dKb^T] = S [dO; -dR]^T ======================
    bool ok_dr = true;
    if (tid == 0) {
      ok_dr = mbar_wait_spin(&ms.bar_dr, ph_dr, &ms.abort, p.err, WAIT_LIMIT);
      ph_dr ^= 1;
      if (ok_dr) ++n_dr_done;
    }
    if (tid == 0 && ok_dr) {
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        umma_tf32_ss(tmem + K2_PX, kdesc(sbase + K2_DR, R128, ks), kdesc(sbase + K2_U, R64, ks), ID_64, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        umma_tf32_ts(tmem + K2_QK, tmem + K2_SX + 8 * ks, kdesc(sbase + K2_DR, R128, ks), ID_128, ks > 0);
      umma_commit(&ms.bar_mma);
    }
    // dSn again (L2), for dSt = Gamma_C dSn once the product that reads S is done
    {
      const float4* Dr = reinterpret_cast<const float4*>(p.dsn + ((size_t)u * D + ln) * D + 32 * cg);
#pragma unroll
      for (int m = 0; m < 8; ++m) d4[m] = __ldg(Dr + m);
    }
    if (!wait_all(&ms.bar_mma, ph_mma)) { dead = true; break; }
    tc_fence_after();
    TC_STAMP(true, srow, 19);
    // the stacked [dO; -dR] tile has been read (the second products do not use it): the next
    // unit's dO and -dR
    if (warp == 0 && u + stride < p.units) {
      issue_dr(u + stride);
      ++n_dr;
    }
    if (u + stride < p.units) prefetch_states(u + stride);  // (its states into L2, after this unit's loads)
    // read-out of [dP; dA], masked (dP: s <= t, dA: s < t), to both operand tiles
    {
      float v[16];
      tmem_ld16(tl + K2_PX + 16 * cg, v);
      tmem_ld_wait();
      const int t = ln & 63;
      const bool isA = ln >= 64;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int s = 16 * cg + r;
        const bool keep = isA ? (s < t) : (s <= t);
        v[r] = keep ? rna(v[r]) : 0.f;
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<float4*>(sm + K2_PA + f32_off(ln, 16 * cg + 4 * m, R128)) =
            make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
#pragma unroll
      for (int r = 0; r < 16; ++r) *reinterpret_cast<float*>(sm + K2_PAT + f32_off(16 * cg + r, ln, R64)) = v[r];
    }
    // the product that read S is done: dSt takes its place
    {
      const float gc = ms.gC[ln];
      float dv32[32];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        dv32[4 * m] = rna(gc * d4[m].x);
        dv32[4 * m + 1] = rna(gc * d4[m].y);
        dv32[4 * m + 2] = rna(gc * d4[m].z);
        dv32[4 * m + 3] = rna(gc * d4[m].w);
      }
      tmem_st32(tl + K2_SX + 32 * cg, dv32);
    }
    if (!sync_ok(true)) { dead = true; break; }
    TC_STAMP(true, srow, 20);
    // ===== [dQh^T | dKb^T] += Kn^T [dP; dA]^T,  Y = [Qh; Kb]^T [dP; dA],  X = dSt U^T ========
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_tf32_ss(tmem + K2_QK, kdesc(sbase + K2_KNT, R128, ks), kdesc(sbase + K2_PA, R128, ks), ID_128, 1);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        umma_tf32_ts(tmem + K2_Y, tmem + K2_KQ + 8 * ks, kdesc(sbase + K2_PAT, R64, ks), ID_64, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        umma_tf32_ts(tmem + K2_PX, tmem + K2_SX + 8 * ks, kdesc(sbase + K2_U, R64, ks), ID_64, ks > 0);
      umma_commit(&ms.bar_mma);
    }
    if (!wait_all(&ms.bar_mma, ph_mma)) { dead = true; break; }
    tc_fence_after();
    TC_STAMP(true, srow, 21);
    // ===== the elementwise finish, in two halves of 8 tokens (the later half first, for the
    // reverse cumsum), from on-chip copies: dQh, dKb, X, Y, Qh, Kb (tensor memory), Kn (its
    // tile, read first: dk is staged over it), b (its staging), Gamma (registers).
    // dg = dKb Kb + dQh Qh - dKn Kn per token; dq, dk, db and the in-segment suffix sums of dg
    // go to output staging tiles over U, Kn^T and the [dP; dA] tiles (read by the finished
    // products), stored by TMA once complete.
    float kn16[16];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float4 k4 = *reinterpret_cast<const float4*>(sm + K2_KNT + f32_off(ln, 16 * cg + 4 * m, R128));
      kn16[4 * m] = k4.x;
      kn16[4 * m + 1] = k4.y;
      kn16[4 * m + 2] = k4.z;
      kn16[4 * m + 3] = k4.w;
    }
    __syncthreads();  // every read of the Kn^T tile is done
    float dx = 0.f, run = 0.f;
    {
      const uint32_t rbo = (uint32_t)(ln >> 6) * R64 + (uint32_t)(ln & 7) * 2;
      const int chk = (ln & 63) >> 3;
#pragma unroll
      for (int hf = 1; hf >= 0; --hf) {
        float a8[8], b8[8], x8[8], y8[8], qh8[8], kb8[8];
        tmem_ld8(tl + K2_QK + 16 * cg + 8 * hf, a8);
        tmem_ld8(tl + K2_QK + C + 16 * cg + 8 * hf, b8);
        tmem_ld8(tl + K2_PX + 16 * cg + 8 * hf, x8);
        tmem_ld8(tl + K2_Y + 16 * cg + 8 * hf, y8);
        tmem_ld8(tl + K2_KQ + 16 * cg + 8 * hf, qh8);
        tmem_ld8(tl + K2_KQ + C + 16 * cg + 8 * hf, kb8);
        const float* kn8 = kn16 + 8 * hf;
        tmem_ld_wait();
#pragma unroll
        for (int r = 7; r >= 0; --r) {
          const int e = 8 * hf + r, t = 16 * cg + e;
          const float Gt = G[e], Gi = 1.f / Gt, kn = kn8[r];
          const float bt = __uint_as_float(
              (uint32_t)(*reinterpret_cast<const unsigned short*>(sm + K2_RB + rbo + sw128_off(t, chk))) << 16);
          const float dkn = x8[r] + y8[r];
          dx = fmaf(kn, x8[r], dx);
          run += b8[r] * kb8[r] + a8[r] * qh8[r] - dkn * kn;
          const uint32_t o = f32_off(t, ln, R64);
          *reinterpret_cast<float*>(sm + K2_ODQ + o) = a8[r] * Gt;
          *reinterpret_cast<float*>(sm + K2_ODK + o) = b8[r] * bt * Gt + dkn * Gi;
          *reinterpret_cast<float*>(sm + K2_ODB + o) = b8[r] * kn * Gt * Gt;
          *reinterpret_cast<float*>(sm + K2_ODLA + o) = run;  // suffix sum within the segment
        }
      }
    }
    ms.dotx[cg][ln] = dx;
    ms.tot[cg][ln] = run;
    __syncthreads();
    {
      const float gc = ms.gC[ln];
      float d1 = 0.f, dxs = 0.f, later = 0.f;
#pragma unroll
      for (int s4i = 0; s4i < 4; ++s4i) {
        d1 += ms.dot1[s4i][ln];
        dxs += ms.dotx[s4i][ln];
        if (s4i > cg) later += ms.tot[s4i][ln];
      }
      // dGamma_C = sum_j dSn (S + Kn^T U) = sum_j dSn S + (1 / Gamma_C) sum_s Kn (dSt U^T)
      const float carry = (d1 + dxs / gc) * gc + later;
#pragma unroll
      for (int r = 0; r < 16; ++r) *reinterpret_cast<float*>(sm + K2_ODLA + f32_off(16 * cg + r, ln, R64)) += carry;
    }
    fence_proxy_async_smem();
    __syncthreads();
    // the four outputs (rows past the sequence are clipped), then the next unit's copies once
    // the stores have read the staging
    if (warp == 0) {
      if (lane == 0) {
        tma_store_5d(&tmDQ, sm + K2_ODQ, 0, C * c, 0, h, bb);
        tma_store_5d(&tmDK, sm + K2_ODK, 0, C * c, 0, h, bb);
        tma_store_5d(&tmDB, sm + K2_ODB, 0, C * c, 0, h, bb);
        tma_store_5d(&tmDLA, sm + K2_ODLA, 0, C * c, 0, h, bb);
        bulk_commit();
        bulk_wait_read_all();
      }
      __syncwarp();
      if (u + stride < p.units) {
        issue_rest(u + stride);
        ++n_ld;
      }
    }
    TC_STAMP(true, srow, 22);
    // the next unit's read of gC, seg and the tensor memory follows this unit's reads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (tid == 0) bulk_wait_all();  // the output stores complete before the block exits
  if (tid == 0 && ms.abort) {
    volatile int never = 0;
    umma_commit(&ms.bar_drain);
    mbar_wait_bounded(&ms.bar_drain, 0, &never, nullptr, WAIT_LIMIT);
    if (n_ld > n_ld_done) mbar_wait_bounded(&ms.bar_ld, (uint32_t)((n_ld - 1) & 1), &never, nullptr, WAIT_LIMIT);
    if (n_dr > n_dr_done) mbar_wait_bounded(&ms.bar_dr, (uint32_t)((n_dr - 1) & 1), &never, nullptr, WAIT_LIMIT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---- host side ------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode() {
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
// fp32 [rows][cols] row-major; boxes of 64 rows x 32 columns, 128B swizzle
bool map_rows(CUtensorMap* m, const float* base, size_t rows, int cols) {
  auto fn = encode();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)C};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// [B][T][H][D] tokens of esize bytes; boxes of 64 tokens x box_d channels of one (batch,
// head), 128B swizzle (rows past T read zero)
bool map_tokens(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int box_d, int B, int T,
                int H) {
  auto fn = encode();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize, (cuuint64_t)T * H * D * esize};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)C, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// The same tokens as whole panel-major tiles: one box = 64 tokens x all D channels of one
// (batch, head), laid out in shared memory as [panel][token][128 bytes] (dimensions:
// channel within a 128-byte panel, token, panel, head, batch), 128B swizzle.
bool map_token_panels(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int B, int T, int H) {
  auto fn = encode();
  if (!fn) return false;
  const int pw = 128 / esize;  // channels per panel
  cuuint64_t dims[5] = {(cuuint64_t)pw, (cuuint64_t)T, (cuuint64_t)(D / pw), (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)H * D * esize, 128, (cuuint64_t)D * esize, (cuuint64_t)T * H * D * esize};
  cuuint32_t box[5] = {(cuuint32_t)pw, (cuuint32_t)C, (cuuint32_t)(D / pw), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, dt, 5, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// fp32 [rows][cols] row-major as whole panel-major tiles of 64 rows: [panel][row][32]
bool map_row_panels(CUtensorMap* m, const float* base, size_t rows, int cols) {
  auto fn = encode();
  if (!fn) return false;
  cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(cols / 32)};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 4, 128};
  cuuint32_t box[3] = {32, (cuuint32_t)C, (cuuint32_t)(cols / 32)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// workspace carve-up, per (batch, head, chunk): S, dSn (D x D), U, -dR (C x D), T^T, P^T (C x C)
struct BwdWs {
  float *S, *dsn, *U, *nr, *tt, *pt;
};
BwdWs carve(float* ws, size_t units) {
  BwdWs w;
  w.S = ws;
  w.dsn = w.S + units * D * D;
  w.U = w.dsn + units * D * D;
  w.nr = w.U + units * C * D;
  w.tt = w.nr + units * C * D;
  w.pt = w.tt + units * C * C;
  return w;
}

}  // namespace

size_t chunk_bwd_tc_workspace_bytes(int B, int T, int H) {
  const size_t units = (size_t)B * H * ((T + C - 1) / C);
  return sizeof(float) * units * (2 * (size_t)D * D + 2 * (size_t)C * D + 2 * (size_t)C * C);
}

cudaError_t launch_chunk_bwd_tc(const ChunkBwdArgs& a, cudaStream_t st) {
  if (!a.bf16 || a.dk_ != D || a.dv_ != D) return cudaErrorInvalidValue;
  if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
  const int BH = a.B * a.H, nch = (a.T + C - 1) / C;
  const size_t units = (size_t)BH * nch;
  if (units * C > 0x7fffffffull) return cudaErrorInvalidValue;  // TMA row coordinates
  const BwdWs w = carve(a.workspace, units);
  cudaError_t e;
  ChunkArgs f{a.q, a.k, a.v, a.b, a.w, a.log_alpha, a.S0, nullptr, nullptr, a.B, a.T, a.H, D, D, true};
  if ((e = launch_chunk_states_tc(f, w.S, st, w.U, w.tt, w.pt)) != cudaSuccess) return e;
  CUtensorMap mnr, mu, mdo, mq, mk, mb, mla;
  const auto F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32, BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!map_rows(&mnr, w.nr, units * C, D) || !map_row_panels(&mu, w.U, units * C, D) ||
      !map_tokens(&mdo, a.dO, F32, 4, 32, a.B, a.T, a.H) || !map_token_panels(&mq, a.q, BF, 2, a.B, a.T, a.H) ||
      !map_token_panels(&mk, a.k, BF, 2, a.B, a.T, a.H) || !map_token_panels(&mb, a.b, BF, 2, a.B, a.T, a.H) ||
      !map_token_panels(&mla, a.log_alpha, F32, 4, a.B, a.T, a.H))
    return cudaErrorInvalidValue;
  CUtensorMap mdq, mdk, mdb, mdla;
  if (!map_token_panels(&mdq, a.dq, F32, 4, a.B, a.T, a.H) || !map_token_panels(&mdk, a.dk, F32, 4, a.B, a.T, a.H) ||
      !map_token_panels(&mdb, a.db, F32, 4, a.B, a.T, a.H) ||
      !map_token_panels(&mdla, a.dlog_alpha, F32, 4, a.B, a.T, a.H))
    return cudaErrorInvalidValue;
  ChainMaps cm;
  if (!map_token_panels(&cm.q, a.q, BF, 2, a.B, a.T, a.H) || !map_token_panels(&cm.k, a.k, BF, 2, a.B, a.T, a.H) ||
      !map_token_panels(&cm.b, a.b, BF, 2, a.B, a.T, a.H) || !map_token_panels(&cm.v, a.v, BF, 2, a.B, a.T, a.H) ||
      !map_token_panels(&cm.w, a.w, BF, 2, a.B, a.T, a.H) ||
      !map_token_panels(&cm.la, a.log_alpha, F32, 4, a.B, a.T, a.H) ||
      !map_token_panels(&cm.dO, a.dO, F32, 4, a.B, a.T, a.H) || !map_row_panels(&cm.tt, w.tt, units * C, C) ||
      !map_row_panels(&cm.pt, w.pt, units * C, C) || !map_token_panels(&cm.dv, a.dv, F32, 4, a.B, a.T, a.H) ||
      !map_token_panels(&cm.dw, a.dw, F32, 4, a.B, a.T, a.H) || !map_row_panels(&cm.nr, w.nr, units * C, D))
    return cudaErrorInvalidValue;
  ChainParams cp;
  cp.dS_T = a.dS_T;
  cp.dS0 = a.dS0;
  cp.dsn = w.dsn;
  cp.T = a.T;
  cp.H = a.H;
  cp.nch = nch;
  cp.err = device_error_word();
  cp.stamps = stamp_buffer();
  {
    static std::atomic<unsigned long long> attr_done{0};
    if ((e = smem_limit_once(bwd_chain_kernel, (int)K1_SMEM, attr_done)) != cudaSuccess) return e;
  }
  bwd_chain_kernel<<<BH, NTH, K1_SMEM, st>>>(cm, cp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  GradParams gp;
  gp.S = w.S;
  gp.dsn = w.dsn;
  gp.T = a.T;
  gp.H = a.H;
  gp.nch = nch;
  gp.units = (int)units;
  gp.err = cp.err;
  gp.stamps = cp.stamps;
  {
    static std::atomic<unsigned long long> attr_done{0};
    if ((e = smem_limit_once(bwd_grad_kernel, (int)K2_SMEM, attr_done)) != cudaSuccess) return e;
  }
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = (int)(units < (size_t)sms ? units : (size_t)sms);
  bwd_grad_kernel<<<grid, NTH, K2_SMEM, st>>>(mdo, mnr, mu, mq, mk, mb, mla, mdq, mdk, mdb, mdla, gp);
  return cudaGetLastError();
}

}  // namespace gdn2
