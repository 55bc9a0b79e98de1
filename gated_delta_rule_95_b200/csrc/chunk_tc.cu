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
//     X^T     = -S^T Kb^T               O^T = S^T Qh^T        (one product over [-Kb; Qh])
//     R^T     = Vw^T + X^T
//     U~^T    = R^T T^T                 (= ((I + A)^-1 (Vw - Kb S))^T, the erase-corrected writes)
//     O^T    += U~^T P^T
//     S^T    <- (S^T + U~^T Kn) Diag(Gamma_C)
//
// U~ = T (Vw - Kb S) is the WY form U - W S with U = T Vw and W = T Kb multiplied
// out, so the W factor never has to be formed.  All products run as kind::tf32 MMAs
// with M = 128, every operand K-major.  The state is kept transposed, S^T (rows =
// value channels), as an fp32 accumulator in tensor memory and fed straight back as
// the A operand of the next products; so are R^T and U~^T, which are rounded to tf32
// in place first.  Shared-memory operands are rounded to tf32 (nearest).
//
// One CTA owns one (batch, head) and walks its chunks.  Warps 0-15 (512 threads) do the
// elementwise work: thread t owns channel ch = t mod 128 (a key channel and a value
// channel, and the tensor-memory lane of the same index) over the 16 tokens
// [16 sg, 16 sg + 16), sg = t / 128; for the operand build it owns the key-channel pair
// (2 (t mod 64), +1) over the 8 tokens [8 (t / 64), +8).  Warp 16 is the control warp:
// its first thread issues every MMA and the input copies, so that an issue that stalls on a
// full tensor-core queue never holds up the elementwise warps; the first thread of warp 17
// issues the output stores and the log-alpha copies.  The sides hand over through
// mbarriers only (every wait bounded).  Per chunk: the operand tiles are built,
// [A; P] runs while the previous chunk's output is staged for a TMA store and its state
// decay applied; then warps 0-7 read A out and invert (I + A) while the state product
// runs and warps 8-15 round R^T and prepare the next chunk (its Vw^T, and its cumulative
// decay Gamma written in place over the log-alpha tile); the U~ product is issued in two
// parts so that only its T21 term waits for the last level of the solve.  The next
// chunk's v, w are copied once [A; P] has read the Kn tile, q, k, b once the state
// product has read the KQ tile, log alpha once the output staging has been read; every
// input is prefetched into L2 two chunks ahead.
// d_k or d_v = 64 run the same code with the upper half of each operand zero.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 64;
constexpr int NCOMP = 512;                      // warps 0-15: elementwise work
constexpr int NT = NCOMP + 64;                  // + the control warp and the store warp
constexpr int CTL = NCOMP;                      // the thread that issues MMAs and the input copies
constexpr int STW = NCOMP + 32;                 // the thread that issues output stores and log-alpha copies
constexpr int NSOLVE = 256;                     // warps 0-7: A read-out, the solve (warps 0-3), U~ rounding
constexpr int BAR_COMP = 1, BAR_SOLVE = 2, BAR_AUX = 3;  // named barriers: compute warps; warps 0-3; 8-15
constexpr int BAR_PAIR = 4;                     // named barriers 4, 5: warp pairs (0, 1) and (2, 3)
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait
constexpr float LOG2E = 1.4426950408889634f;
// in-chunk cumulative log2 decay below which 2^-g leaves the fp32 range (natural log -80)
constexpr float G2_MIN = -115.4f;
constexpr int PF_AHEAD = 2;                     // chunks of input prefetched into L2 ahead of use
constexpr int LPT_MAX_SEQ = 1024;               // packed batches up to this many sequences start longest first

// ---- shared memory map (byte offsets from a 1024-byte aligned base) ----------------
// fp32 operand tiles with the 128B swizzle, in panels of 32 columns (128 B rows).
constexpr uint32_t R64 = 64 * 128;    // a panel of 64 rows  (8 KB)
constexpr uint32_t R128 = 128 * 128;  // a panel of 128 rows (16 KB)
constexpr uint32_t R192 = 192 * 128;  // a panel of 192 rows (24 KB)
constexpr uint32_t OFF_KQ = 0;                  // [-Kb; Qh] [t][i]: 4 panels x 128 rows (first: raw q, k, b, v)
constexpr uint32_t OFF_KN = OFF_KQ + 4 * R128;  // Kn [s][i]: 4 panels x 64 rows (first: raw w)
constexpr uint32_t OFF_PK = OFF_KN + 4 * R64;   // [P; Kn^T] [t | i][s]: 2 panels x 192 rows
constexpr uint32_t OFF_T = OFF_PK + 2 * R192;   // T [t][s]: 2 panels x 64 rows
constexpr uint32_t OFF_LA = OFF_T + 2 * R64;    // log alpha [t][i] fp32 (TMA, 128B swizzle): 4 panels x 64 rows,
                                                // turned in place into the in-chunk cumulative log2 decay;
                                                // between uses: the output tile [t][j] fp32 of a TMA store
constexpr uint32_t OFF_SCR = OFF_LA + 4 * R64;  // solve scratch: fp32 64 x LDM, then 4 x 32 x LDW
// raw bf16 staging (TMA, 128B swizzle): a [64 tokens][128 channels] tile = 2 panels of
// 64 channels x 64 rows
constexpr uint32_t B16 = 2 * R64;
constexpr uint32_t RAW_Q = OFF_KQ, RAW_K = OFF_KQ + B16, RAW_B = OFF_KQ + 2 * B16;  // free once the
constexpr uint32_t RAW_V = OFF_KN, RAW_W = OFF_KN + B16;  // state product (KQ) / [A; P] (Kn) has read them
constexpr int LDM = 68;                         // padded row (floats) of the 64 x 64 solve matrix
constexpr int LDW = 8;                          // row of a solve warp's block-product scratch (32 x 8)
constexpr uint32_t TILES = OFF_SCR + 22528;     // 214 KB

struct Misc {
  uint64_t bar_la, bar_raw, bar_vw;                    // TMA loads landed: log alpha; q, k, b; v, w
  uint64_t bar_mma, bar_s, bar_drain;                  // tensor-core products done
  uint64_t bar_ops, bar_stage, bar_tdiag, bar_solved, bar_uround;  // compute warps -> control warp
  uint64_t bar_lastread;  // store warp -> compute warps: the last staging tile may be rewritten
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[2][128];    // Gamma at the chunk end, per key channel (chunk parity)
  alignas(16) float segtot[2][128];  // per half chunk: sum of log2 alpha, per key channel
  alignas(16) float rn[128];       // raw projections: 1 / |q_t| (t < 64) and 1 / |k_t| (64 + t)
};
constexpr uint32_t SMEM_BYTES = TILES + 1024 + sizeof(Misc);

// ---- tensor memory columns (fp32, 128 lanes) -------------------------------------------
constexpr uint32_t TM_AP = 0;    // [-A; P]      lanes: tokens of Kb | Qh, columns: s
constexpr uint32_t TM_U = 64;    // U~^T         lanes: value channel, columns: s
constexpr uint32_t TM_R = 128;   // R^T          lanes: value channel, columns: t
constexpr uint32_t TM_O = 192;   // O^T          lanes: value channel, columns: t (after R^T, before S^T)
constexpr uint32_t TM_S = 256;   // S^T (state)  lanes: value channel, columns: key channel
constexpr uint32_t TM_VW = 384;  // Vw^T, two buffers (chunk parity)   lanes: value channel, columns: t
constexpr uint32_t TM_COLS = 512;

// instruction descriptors (M = 128, both operands K-major)
constexpr uint32_t ID_32 = idesc_tf32(128, 32, 0, 0, 0, 0);
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);
constexpr uint32_t ID_128 = idesc_tf32(128, 128, 0, 0, 0, 0);
constexpr uint32_t ID_192 = idesc_tf32(128, 192, 0, 0, 0, 0);

struct TcParams {
  const __nv_bfloat16 *q, *k, *v, *b, *w;
  const float* S0;
  float* S_T;
  float* o;
  int T, H, dk, dv;
  const int* cu_seqlens;  // packed sequences: [N + 1] token offsets (device); NULL = fixed length T
  int nseq;               // packed sequences: N
  const float* dscale;    // raw projections: per-head decay scale s_h (NULL = 1)
  // Sequence split (fixed-length batches): 0 = off; 1 = first pass (segment 0 from S0, and
  // for every later segment its transition M and offset N); 3 = last pass (segments >= 1
  // from their start states).  split_L: tokens per segment (a multiple of C); split_P:
  // segments; ws: workspace [3][B H][P][d_k d_v] fp32 (M, N, start states).
  int split_phase = 0, split_P = 0, split_L = 0;
  float* ws = nullptr;
  // checkpoint phase, for the tensor-core backward (NULL: not written): per (sequence, head,
  // chunk) U~ [s][j], T^T [s][t] and P^T [t][s], fp32 with the tf32 rounding the products used
  float *ck_u = nullptr, *ck_tt = nullptr, *ck_pt = nullptr;
  unsigned* err;
  unsigned long long* stamps = nullptr;  // instrumented build only: per-chunk clock stamps
};

#ifdef GDN2_STAMPS
// Instrumented build (GDN2_STAMPS): clock64 of the SM at fixed points of the per-chunk
// schedule, for the first STAMP_CHUNKS chunks of the launch's first CTA, written by the one
// thread named at each point into [chunk][slot].
constexpr int STAMP_CHUNKS = 64, STAMP_SLOTS = 32;
#define STAMP(cc, slot)                                                                      \
  do {                                                                                       \
    if (p.stamps && blockIdx.x == 0 && (cc) >= 0 && (cc) < STAMP_CHUNKS)                     \
      p.stamps[(size_t)(cc) * STAMP_SLOTS + (slot)] = (unsigned long long)clock64();         \
  } while (0)
#else
#define STAMP(cc, slot) \
  do {                  \
  } while (0)
#endif

// Gate activations of the raw-projection variant, from their definitions, on the
// special-function unit.  sigmoid(x) = (1 + tanh(x / 2)) / 2, one special-function
// operation (tanh.approx, absolute error below 2.5e-4 on the gate); softplus in base-2
// units, softplus(a) log2 e = max(a, 0) log2 e + log2(1 + 2^(-|a| log2 e)), which never
// overflows.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_fast(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }
__device__ __forceinline__ float softplus_log2(float a) {
  return fmaxf(a, 0.f) * LOG2E + lg2_approx(1.f + ex2_approx(-LOG2E * fabsf(a)));
}

// fp32 -> tf32, round to nearest with ties away from zero on the magnitude (add half an
// ulp of the 10-bit mantissa, clear the 13 dropped bits); two integer instructions.
__device__ __forceinline__ float rna_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ void st4_tf32(unsigned char* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(rna_tf32(f[0]), rna_tf32(f[1]), rna_tf32(f[2]), rna_tf32(f[3]));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
// tf32 operand of a warp-level MMA (fp32 bit pattern, low 13 bits cleared)
__device__ __forceinline__ uint32_t tfu(float x) { return __float_as_uint(rna_tf32(x)); }
// one bf16 element of shared memory as fp32
__device__ __forceinline__ float bf16_at(const unsigned char* p) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(p)) << 16);
}
// two adjacent bf16 elements (4-byte aligned) of shared memory as fp32
__device__ __forceinline__ float2 bf16x2_at(const unsigned char* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ void st2_tf32(unsigned char* p, const float2& f) {
  *reinterpret_cast<float2*>(p) = make_float2(rna_tf32(f.x), rna_tf32(f.y));
}

// DK, DV: key and value head dimensions (64 or 128), fixed at compile time so that each
// launch runs straight-line code for its own shape.  VARLEN: the batch is a packed set of
// sequences (a CTA per (sequence, head), token range from cu_seqlens); otherwise B
// sequences of T tokens.  PREP: the inputs are the raw projections, and the kernel applies
// the layer's input activations itself: q and k L2-normalised per token, b = sigmoid(b),
// w = sigmoid(w), log alpha = -s_h softplus(a) (Gated DeltaNet-2 guide, "Decoupled Erase and
// Write Gates" and "Normalization and Short Convolutions").  SPLIT: one pass of the sequence
// split (fixed-length batches, d_k = d_v), below.
template <int DK, int DV, bool VARLEN, bool PREP, bool SPLIT>
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

  const int tid = threadIdx.x, warp = tid >> 5;
  const int ch = tid & 127;  // channel (key i and value j) and tensor-memory lane
  const int sg = tid >> 7;   // token segment [16 sg, 16 sg + 16); column group of TMEM accesses
  const int unit = blockIdx.x;
  int h = unit % p.H;
  // this CTA's sequence: batch coordinate bb, first token t0, length len, chunk count nch,
  // and su, the (sequence, head) index of its entering and final state
  int bb = unit / p.H, t0 = 0, len = p.T, su = unit;
  const size_t st_sz = (size_t)DK * DV;
  // Sequence split of a long sequence (SPLIT): segment s covers tokens [s L, s L + L).  By
  // the recurrence's linearity in (S, v), the state after segment s is M_s S + N_s, with
  // M_s the state reached from S = I with v = 0 (d_k = d_v) and N_s the one reached from
  // S = 0; the host chains them between the passes.  First pass (phase 1): r = 0 runs
  // segment 0 from S0, r in [1, P - 1) gives N_r, r in [P - 1, 2P - 3) gives M_{r-P+2} (the
  // last segment needs neither: it starts from its chained state); last pass
  // (phase 3): segment r + 1 from its start state.  The same instantiation also runs the
  // whole sequence writing the state entering every chunk to the workspace [B H][chunk]
  // [d_k][d_v] and no outputs (phase 5, the checkpoints of the backward pass).
  int sp_r = 0, sp_seg = 0;
  if constexpr (SPLIT) {
    const int BH = p.nseq;
    const int bh = unit % BH;
    sp_r = unit / BH;
    h = bh % p.H;
    bb = bh / p.H;
    su = bh;
    sp_seg = p.split_phase == 1 ? (sp_r < p.split_P - 1 ? sp_r : sp_r - p.split_P + 2) : sp_r + 1;
    t0 = sp_seg * p.split_L;
    len = min(p.split_L, p.T - t0);
    if (p.split_phase == 5) {
      sp_seg = 0;
      t0 = 0;
      len = p.T;
    }
  }
  const bool sp_first = SPLIT && p.split_phase == 1;
  const bool sp_ckpt = SPLIT && p.split_phase == 5;
  const bool write_o = !SPLIT || (sp_first ? sp_r == 0 : !sp_ckpt);  // outputs written
  const bool sp_trans = SPLIT && sp_first && sp_r >= p.split_P - 1;  // M_s: from I, no write term
  if constexpr (VARLEN) {
    int n = unit / p.H;
    if (p.nseq <= LPT_MAX_SEQ) {
      // Launch order by length, longest first (ties by index), so that the longest
      // sequences of an uneven batch do not start last: this CTA takes the sequence of
      // rank unit / H.  The lengths are ranked in the (still unused) solve scratch.
      __shared__ int picked;
      int* lens = reinterpret_cast<int*>(sm + OFF_SCR);
      for (int i = threadIdx.x; i < p.nseq; i += NT) lens[i] = p.cu_seqlens[i + 1] - p.cu_seqlens[i];
      __syncthreads();
      for (int i = threadIdx.x; i < p.nseq; i += NT) {
        const int li = lens[i];
        int rank = 0;
        for (int m = 0; m < p.nseq; ++m) rank += (lens[m] > li) | (lens[m] == li && m < i);
        if (rank == n) picked = i;
      }
      __syncthreads();
      n = picked;
    }
    su = n * p.H + h;
    bb = 0;
    t0 = p.cu_seqlens[n];
    len = p.cu_seqlens[n + 1] - t0;
    if (t0 < 0 || len < 0 || t0 + len > p.T) {  // offsets out of order or out of range
      if (threadIdx.x == 0 && p.err) atomicOr(p.err, kErrBadSeqlens);
      return;
    }
  }
  const int nch = (len + C - 1) / C;
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
    mbar_init(&ms.bar_tdiag, NCOMP / 32);   // R^T rounded, diagonal 32x32 blocks of T written
    mbar_init(&ms.bar_solved, NSOLVE / 32);  // the T_21 block written
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
  const uint32_t tlane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // lanes [32 (warp mod 4), +32)


  auto wait_on = [&](uint64_t* bar, uint32_t& ph) -> bool {
    const bool ok = mbar_wait_bounded(bar, ph, &ms.abort, p.err, WAIT_LIMIT);
    if (ok) ph ^= 1;
    return ok;
  };
  auto warp_arrive = [&](uint64_t* bar) {  // one arrival per warp, after all its lanes
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(bar);
  };

  if (warp == NCOMP / 32) {
    // ========================= control warp: MMAs and TMA copies =========================
    if (tid == CTL) {
      int n_raw = 0, n_vw = 0;
      auto prefetch_raw = [&](int c) {  // every input tile of chunk c into L2
        for (int pn = 0; pn < (dk >> 5); ++pn) tma_prefetch_l2_4d(&tmLA, 32 * pn, h, t0 + C * c, bb);
        for (int pn = 0; pn < (dk >> 6); ++pn) {
          tma_prefetch_l2_4d(&tmQ, 64 * pn, h, t0 + C * c, bb);
          tma_prefetch_l2_4d(&tmK, 64 * pn, h, t0 + C * c, bb);
          tma_prefetch_l2_4d(&tmB, 64 * pn, h, t0 + C * c, bb);
        }
        for (int pn = 0; pn < (dv >> 6); ++pn) {
          tma_prefetch_l2_4d(&tmV, 64 * pn, h, t0 + C * c, bb);
          tma_prefetch_l2_4d(&tmW, 64 * pn, h, t0 + C * c, bb);
        }
      };
      auto issue_qkb = [&](int c) {  // raw q, k, b of chunk c into the KQ tile
        mbar_arrive_expect_tx(&ms.bar_raw, (uint32_t)(3 * (dk >> 6)) * R64);
        for (int pn = 0; pn < (dk >> 6); ++pn) {
          tma_load_4d(sm + RAW_Q + pn * R64, &tmQ, &ms.bar_raw, 64 * pn, h, t0 + C * c, bb);
          tma_load_4d(sm + RAW_K + pn * R64, &tmK, &ms.bar_raw, 64 * pn, h, t0 + C * c, bb);
          tma_load_4d(sm + RAW_B + pn * R64, &tmB, &ms.bar_raw, 64 * pn, h, t0 + C * c, bb);
        }
        ++n_raw;
      };
      auto issue_vw = [&](int c) {  // raw v, w of chunk c into the Kn tile
        mbar_arrive_expect_tx(&ms.bar_vw, (uint32_t)(2 * (dv >> 6)) * R64);
        for (int pn = 0; pn < (dv >> 6); ++pn) {
          tma_load_4d(sm + RAW_V + pn * R64, &tmV, &ms.bar_vw, 64 * pn, h, t0 + C * c, bb);
          tma_load_4d(sm + RAW_W + pn * R64, &tmW, &ms.bar_vw, 64 * pn, h, t0 + C * c, bb);
        }
        ++n_vw;
      };
      uint32_t ph_ops = 0, ph_stage = 0, ph_tdiag = 0, ph_solved = 0, ph_uround = 0, ph_s = 0;
      bool alive = true;
      if (nch > 0) {
        issue_qkb(0);
        issue_vw(0);
        for (int cc = 1; cc <= PF_AHEAD && cc < nch; ++cc) prefetch_raw(cc);
      }
      for (int c = 0; c < nch; ++c) {
        if (c + PF_AHEAD < nch) prefetch_raw(c + PF_AHEAD);
        // [-A; P] = [-Kb; Qh] Kn^T : M=128 (tokens of both halves), N=64 (s), K=128 (key channels)
        if (!(alive = wait_on(&ms.bar_ops, ph_ops))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
          const uint32_t ko = (uint32_t)((ks & 3) * 32);
          const uint64_t aKQ = sdesc_sw128(sbase + OFF_KQ + (ks >> 2) * R128 + ko, 16, 1024);
          const uint64_t bKN = sdesc_sw128(sbase + OFF_KN + (ks >> 2) * R64 + ko, 16, 1024);
          umma_tf32_ss(tmem + TM_AP, aKQ, bKN, ID_64, ks > 0);
        }
        umma_commit(&ms.bar_mma);
        STAMP(c, 0);
        // [X^T | O^T] = S^T [-Kb; Qh]^T : A = S^T (tensor memory), B = the KQ tile (N = 128);
        // X^T = -S^T Kb^T becomes R^T = Vw^T + X^T when warps 8-15 round it
        if (!(alive = wait_on(&ms.bar_stage, ph_stage))) break;
        tc_fence_after();
        // [A; P] has read the Kn tile: the next chunk's v, w.  (Its completion is this
        // barrier's phase 3c; no later phase can complete before this thread issues again.)
        if (!(alive = mbar_wait_bounded(&ms.bar_mma, (uint32_t)((3 * c) & 1), &ms.abort, p.err, WAIT_LIMIT))) break;
        if (c + 1 < nch) issue_vw(c + 1);
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
          const uint64_t bKQ = sdesc_sw128(sbase + OFF_KQ + (ks >> 2) * R128 + (ks & 3) * 32, 16, 1024);
          umma_tf32_ts(tmem + TM_R, tmem + TM_S + 8 * ks, bKQ, ID_128, ks > 0);
        }
        umma_commit(&ms.bar_s);
        STAMP(c, 1);
        // the state product has read the KQ tile: the next chunk's q, k, b
        if (!(alive = wait_on(&ms.bar_s, ph_s))) break;
        if (c + 1 < nch) issue_qkb(c + 1);
        // U~^T = R^T T^T : A = R^T (tensor memory), B = T (N = s), K = t, in 32-column halves
        // of s.  With T = [T11 0; T21 T22] (32 x 32 blocks): U~^T[:, :32] = R1^T T11^T and
        // U~^T[:, 32:] = R2^T T22^T + R1^T T21^T; everything but the T21 term is issued as soon
        // as the diagonal blocks exist, overlapping the last level of the solve.
        if (!(alive = wait_on(&ms.bar_tdiag, ph_tdiag))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {  // s in [0, 32), t in [0, 32)
          const uint64_t bT = sdesc_sw128(sbase + OFF_T + ks * 32, 16, 1024);
          umma_tf32_ts(tmem + TM_U, tmem + TM_R + 8 * ks, bT, ID_32, ks > 0);
        }
#pragma unroll
        for (int ks = 4; ks < 8; ++ks) {  // s in [32, 64), t in [32, 64)
          const uint64_t bT = sdesc_sw128(sbase + OFF_T + R64 + 32 * 128 + (ks & 3) * 32, 16, 1024);
          umma_tf32_ts(tmem + TM_U + 32, tmem + TM_R + 8 * ks, bT, ID_32, ks > 4);
        }
        STAMP(c, 2);
        if (!(alive = wait_on(&ms.bar_solved, ph_solved))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {  // s in [32, 64), t in [0, 32): the T21 block
          const uint64_t bT = sdesc_sw128(sbase + OFF_T + 32 * 128 + ks * 32, 16, 1024);
          umma_tf32_ts(tmem + TM_U + 32, tmem + TM_R + 8 * ks, bT, ID_32, 1);
        }
        umma_commit(&ms.bar_mma);
        STAMP(c, 3);
        // [O^T | S^T] += U~^T [P; Kn^T]^T : O^T += U~^T P^T and S^T += U~^T Kn in one N = 192 product
        if (!(alive = wait_on(&ms.bar_uround, ph_uround))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bPK = sdesc_sw128(sbase + OFF_PK + (ks >> 2) * R192 + (ks & 3) * 32, 16, 1024);
          umma_tf32_ts(tmem + TM_O, tmem + TM_U + 8 * ks, bPK, ID_192, 1);
        }
        umma_commit(&ms.bar_mma);
        STAMP(c, 4);
      }
      // after a give-up: every MMA issued so far (a fresh commit tracks all of them) and
      // the last copies must land before the block releases its memory
      if (ms.abort) {
        volatile int never = 0;
        umma_commit(&ms.bar_drain);
        mbar_wait_bounded(&ms.bar_drain, 0, &never, nullptr, WAIT_LIMIT);
        if (n_raw > 0) mbar_wait_bounded(&ms.bar_raw, (uint32_t)((n_raw - 1) & 1), &never, nullptr, WAIT_LIMIT);
        if (n_vw > 0) mbar_wait_bounded(&ms.bar_vw, (uint32_t)((n_vw - 1) & 1), &never, nullptr, WAIT_LIMIT);
      }
    }
    __syncwarp();  // the warp reconverges before the block-wide barrier
  } else if (warp == NCOMP / 32 + 1) {
    // ========================= store warp: output stores and log-alpha copies ===============
    // The output of chunk c - 1 is staged over the decay tile once the operand build of
    // chunk c has read it; as soon as the store has read the staging, the log alpha of chunk
    // c + 1 is copied over it.  Kept off the control thread, whose MMA issue would otherwise
    // delay that copy, and with it the cumulative decay of the next chunk.
    if (tid == STW) {
      int n_la = 0;
      auto issue_la = [&](int c) {  // log alpha of chunk c: dk/32 boxes of 32 channels x 64 tokens
        mbar_arrive_expect_tx(&ms.bar_la, (uint32_t)(C * dk * 4));
        for (int pn = 0; pn < (dk >> 5); ++pn)
          tma_load_4d(sm + OFF_LA + pn * R64, &tmLA, &ms.bar_la, 32 * pn, h, t0 + C * c, bb);
        ++n_la;
      };
      auto store_o = [&](int cc) {  // the staged output tile of chunk cc (rows past T are clipped)
        tma_store_4d(&tmO, sm + OFF_LA, 0, h, t0 + C * cc, bb);
        bulk_commit();
      };
      uint32_t ph_stage = 0;
      bool alive = true;
      if (nch > 0) issue_la(0);
      for (int c = 0; c < nch; ++c) {
        if (!(alive = wait_on(&ms.bar_stage, ph_stage))) break;
        if (c > 0 && write_o) {
          store_o(c - 1);
          bulk_wait_read_all();
        }
        STAMP(c, 16);
        if (c + 1 < nch) issue_la(c + 1);
        else mbar_arrive(&ms.bar_lastread);  // the last staging may overwrite the tile
      }
      // the last chunk's output, staged by the compute warps (a packed sequence's partial last
      // chunk is written by the compute warps themselves: its box would spill into the next
      // sequence's rows)
      if (alive && nch > 0 && wait_on(&ms.bar_stage, ph_stage) && !(VARLEN && len % C) && write_o) store_o(nch - 1);
      if (ms.abort && n_la > 0) {  // the last copy lands before the block releases its memory
        volatile int never = 0;
        mbar_wait_bounded(&ms.bar_la, (uint32_t)((n_la - 1) & 1), &never, nullptr, WAIT_LIMIT);
      }
      bulk_wait_all();  // output stores complete before the block exits
    }
    __syncwarp();  // the warp reconverges before the block-wide barrier
  } else {
    // ========================= compute warps 0-15 =========================================
    // entering state S0 -> S^T in tensor memory: lane j = ch (a value channel), key-channel
    // columns [32 sg, 32 sg + 32)
    {
      // (split: segment 0 from S0, N_s from zero, M_s from I, the last pass from the start
      // states of the workspace)
      const float* S0u = p.S0 ? p.S0 + (size_t)su * st_sz : nullptr;
      if (SPLIT && !sp_ckpt && (sp_first ? sp_r > 0 : true))
        S0u = sp_first ? nullptr : p.ws + (2 * (size_t)p.nseq * p.split_P + (size_t)su * p.split_P + sp_seg) * st_sz;
      float v[32];
      const bool ok = S0u && vval;
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int i = 32 * sg + x;
        v[x] = (ok && i < dk) ? S0u[(size_t)i * dv + ch] : 0.f;
        if (sp_trans) v[x] = (i == ch && vval) ? 1.f : 0.f;
      }
      if (sp_ckpt && vval && nch > 0) {  // the state entering chunk 0
        float* ck = p.ws + (size_t)su * nch * st_sz + ch;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (32 * sg + x < dk) ck[(size_t)(32 * sg + x) * dv] = v[x];
      }
      tmem_st32(tlane + TM_S + 32 * sg, v);
      tmem_st_wait();
    }
    // the T operand tile: blocks above the 8x8 block diagonal stay zero for good
    for (int e = tid; e < 2 * (int)R64 / 16; e += NCOMP)
      *reinterpret_cast<float4*>(sm + OFF_T + 16 * e) = make_float4(0.f, 0.f, 0.f, 0.f);
    uint32_t ph_mma = 0, ph_s = 0;
    float* Msc = reinterpret_cast<float*>(sm + OFF_SCR);                 // solve matrix, 64 x LDM fp32
    float* Xsc = reinterpret_cast<float*>(sm + OFF_SCR + 64 * LDM * 4);  // block products, 4 x 32 x LDW fp32
    const int lane = tid & 31;
    auto wait_mma = [&]() -> bool { return wait_on(&ms.bar_mma, ph_mma); };
    // S^T <- S^T Diag(Gamma_C of the chunk with parity gb), in tensor memory (checkpoint
    // phase: also written out as the state entering chunk cst, if cst >= 0).
    auto decay_state = [&](int gb, int cst) {
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
      if (sp_ckpt && cst >= 0 && vval) {
        float* ck = p.ws + ((size_t)su * nch + cst) * st_sz + ch;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (32 * sg + x < dk) ck[(size_t)(32 * sg + x) * dv] = v[x];
      }
    };
    // Output of the last finished chunk (O^T in tensor memory) into the shared-memory tile
    // [t][j] (rows of d_v floats, over the log-decay tile, whose reads are done) that the
    // control warp's TMA store writes out.
    auto stage_o = [&]() {
      float v[16];
      tmem_ld16(tlane + TM_O + 16 * sg, v);
      tmem_ld_wait();
      if (vval) {
        float* st = reinterpret_cast<float*>(sm + OFF_LA) + ch;
#pragma unroll
        for (int x = 0; x < 16; ++x) st[(16 * sg + x) * dv] = v[x];
      }
    };

    // Checkpoint phase: T^T and P^T of chunk cc to the backward's workspace (both tiles stay
    // intact until the next chunk's read-out and solve).
    auto ckpt_tp = [&](int cc) {
      const size_t at = ((size_t)su * nch + cc) * C * C;
      for (int e = tid; e < C * C; e += NCOMP) {
        const int r = e >> 6, x = e & 63;
        p.ck_tt[at + e] = *reinterpret_cast<const float*>(sm + OFF_T + f32_off(x, r, R64));    // T[x][r]
        p.ck_pt[at + e] = *reinterpret_cast<const float*>(sm + OFF_PK + f32_off(x, r, R192));  // P[x][r]
      }
    };

    // Warps 8-15, one chunk ahead (chunk cc).  Thread (ch, hf) owns the 32 tokens
    // [32 hf, 32 hf + 32) of channel ch.
    uint32_t ph_la = 0, ph_raw = 0, ph_vw = 0;
    const float dsc = PREP ? (p.dscale ? p.dscale[h] : 1.f) : 0.f;  // decay scale s_h
    // Vw^T = (W * V)^T into the tensor-memory buffer of chunk cc's parity (v and w are copied
    // as soon as [A; P] has read the Kn tile).
    auto vw_ahead = [&](int cc, bool ok) -> bool {
      const int hf = sg - 2;
      ok = ok && wait_on(&ms.bar_vw, ph_vw);
      float vw[32];
      const uint32_t pnl = (uint32_t)(ch >> 6) * R64;
      const int chk = (ch & 63) >> 3, byt = (ch & 7) * 2;
      const int lim = len - (C * cc + 32 * hf);  // rows of this half inside the sequence
      // (packed sequences: the rows past the end, only in a sequence's last chunk, are masked)
      auto fill = [&](auto masked) {
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          const uint32_t ro = pnl + sw128_off(32 * hf + r, chk) + byt;
          const bool tv = !decltype(masked)::value || r < lim;
          float wr = bf16_at(sm + RAW_W + ro);
          if constexpr (PREP) wr = sigmoid_fast(wr);
          vw[r] = (vval && tv) ? bf16_at(sm + RAW_V + ro) * wr : 0.f;
        }
      };
      if (sp_trans) {  // transition runs of the sequence split: no write term
#pragma unroll
        for (int r = 0; r < 32; ++r) vw[r] = 0.f;
      } else if (VARLEN && lim < 32) {
        fill(std::true_type{});
      } else {
        fill(std::false_type{});
      }
      tmem_st32(tlane + TM_VW + 64 * (cc & 1) + 32 * hf, vw);
      tmem_st_wait();
      return ok;
    };
    // The in-chunk cumulative decay Gamma = 2^g (base-2 cumsum of log alpha), written back
    // in place over the log-alpha tile, and the end-of-chunk decay per key channel.
    auto decay_ahead = [&](int cc, bool ok) -> bool {
      const int hf = sg - 2;
      unsigned char* la_w = sm + OFF_LA;
      ok = ok && wait_on(&ms.bar_la, ph_la);
      float x[32];
      float acc = 0.f;
      const int lim = len - (C * cc + 32 * hf);  // rows of this half inside the sequence
      // rows past the sequence add nothing: masked only in its last chunk (packed sequences,
      // whose tile rows there belong to the next sequence; raw projections, whose tail rows
      // read a = 0, and softplus(0) is not 0)
      auto scan = [&](auto masked) {
        constexpr bool M = decltype(masked)::value;
#pragma unroll
        for (int r = 0; r < 32; ++r)
          x[r] = (kval && (!M || r < lim)) ? *reinterpret_cast<const float*>(la_w + f32_off(32 * hf + r, ch, R64))
                                           : 0.f;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          if constexpr (PREP) {  // log2 alpha = -s_h softplus(a) log2 e
            const bool vr = kval && (!M || r < lim);
            acc -= vr ? dsc * softplus_log2(x[r]) : 0.f;
          } else {
            acc = fmaf(x[r], LOG2E, acc);
          }
          x[r] = acc;
        }
      };
      if ((VARLEN || PREP) && lim < 32) scan(std::true_type{});
      else scan(std::false_type{});
      ms.segtot[hf][ch] = acc;
      named_bar_sync(BAR_AUX, NCOMP - NSOLVE);
      const float off = hf ? ms.segtot[0][ch] : 0.f;
      if (kval) {
#pragma unroll
        for (int r = 0; r < 32; ++r)
          *reinterpret_cast<float*>(la_w + f32_off(32 * hf + r, ch, R64)) = ex2_approx(x[r] + off);
      }
      if (hf == 1) {
        ms.gC[cc & 1][ch] = kval ? ex2_approx(off + acc) : 0.f;
        // the chunk-start reference scales keys by 2^-g: beyond a cumulative log decay of -80
        // (log2: G2_MIN) within the chunk that leaves the fp32 range; the result is flagged
        if (kval && off + acc < G2_MIN && p.err) atomicOr(p.err, kErrDecayRange);
      }
      return ok;
    };
    // Raw projections, warps 0-7, one chunk ahead once its q, k, b copies have landed:
    // 1 / |q_t| and 1 / |k_t| (a zero vector stays zero).  Thread a = t mod 256 sums the
    // squares of one 128-byte row: row a / 2 of the stacked [q; k] rows, channel panel a mod 2.
    auto norms_ahead = [&](bool ok) -> bool {
      ok = ok && wait_on(&ms.bar_raw, ph_raw);
      const int a = tid & 255;
      {
        const int row = a >> 1, pn = a & 1, t = row & 63;
        const unsigned char* base = sm + (row < 64 ? RAW_Q : RAW_K) + pn * R64;
        float ss = 0.f;
        if (pn * 64 < dk) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // (the swizzle spreads rows t .. t + 7 over the eight 16-byte bank groups)
            const uint4 u = *reinterpret_cast<const uint4*>(base + sw128_off(t, j));
            const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float lo = __uint_as_float(wd[m] << 16), hi = __uint_as_float(wd[m] & 0xFFFF0000u);
              ss = fmaf(lo, lo, fmaf(hi, hi, ss));
            }
          }
        }
        ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 1);
        if (pn == 0) ms.rn[row] = rsqrtf(fmaxf(ss, 1e-24f));
      }
      return ok;
    };

    bool dead = false;
    bool ok_prev = true;  // failed waits of the previous chunk's tail, voted at the next barrier
    if (nch > 0 && warp >= NSOLVE / 32) ok_prev = decay_ahead(0, vw_ahead(0, true));
    if constexpr (PREP)
      if (nch > 0 && warp < NSOLVE / 32) ok_prev = norms_ahead(true);
    tc_fence_before();
    if (named_bar_or(BAR_COMP, NCOMP, !ok_prev)) dead = true;
    tc_fence_after();
    for (int c = 0; c < nch && !dead; ++c) {
      const int ob = c & 1;
      if (sp_ckpt && p.ck_tt && c > 0) ckpt_tp(c - 1);
      // ===== folded operands.  For this step thread t owns the key-channel pair
      // (2 cp, 2 cp + 1), cp = t mod 64, over the 8 tokens [8 ts, 8 ts + 8), ts = t / 64, so
      // that every raw load and tile store moves both channels at once.  Gamma = 2^g was
      // computed one chunk ahead, in place over the log-alpha tile. ==========================
      const int cp = tid & 63, ts = tid >> 6, c2 = 2 * cp;
      const bool kv2 = c2 < dk;
      float2 nkb[8], qh[8], kn[8];
      // (raw projections: warps 0-7 have seen these copies land already, one chunk ahead)
      bool ok_raw = (PREP && warp < NSOLVE / 32) ? true : wait_on(&ms.bar_raw, ph_raw);
      if (tid == 0) STAMP(c, 5);
      auto build = [&](auto masked) {
        const unsigned char* la_t = sm + OFF_LA;
        const uint32_t pnl = (uint32_t)(c2 >> 6) * R64;  // raw tiles: panels of 64 channels
        const int chk = (c2 & 63) >> 3, byt = (c2 & 7) * 2;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int t = 8 * ts + r;
          const uint32_t ro = pnl + sw128_off(t, chk) + byt;
          float2 G = make_float2(1.f, 1.f), kk = make_float2(0.f, 0.f), bg = kk, qq = kk;
          // (packed sequences: the tile rows past this sequence's end hold the next one's
          // tokens; masked only in its last chunk)
          if (kv2 && (!decltype(masked)::value || C * c + t < len)) {
            G = *reinterpret_cast<const float2*>(la_t + f32_off(t, c2, R64));
            kk = bf16x2_at(sm + RAW_K + ro);
            bg = bf16x2_at(sm + RAW_B + ro);
            qq = bf16x2_at(sm + RAW_Q + ro);
            if constexpr (PREP) {
              const float rq = ms.rn[t], rk = ms.rn[64 + t];
              kk = make_float2(kk.x * rk, kk.y * rk);
              qq = make_float2(qq.x * rq, qq.y * rq);
              bg = make_float2(sigmoid_fast(bg.x), sigmoid_fast(bg.y));
            }
          }
          const float2 Gi = make_float2(rcp_approx(G.x), rcp_approx(G.y));
          nkb[r] = make_float2(-(kk.x * bg.x) * G.x, -(kk.y * bg.y) * G.y);
          qh[r] = make_float2(qq.x * G.x, qq.y * G.y);
          kn[r] = make_float2(kk.x * Gi.x, kk.y * Gi.y);
        }
      };
      if (VARLEN && C * c + C > len) build(std::true_type{});
      else build(std::false_type{});
      // every raw read must be done before the operand tiles overwrite the staging
      if (named_bar_or(BAR_COMP, NCOMP, !ok_raw)) { dead = true; break; }
      // the KQ and Kn tiles were last read by the previous chunk's state product and [A; P]:
      // they are written while the previous chunk's output/state product may still run
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int t = 8 * ts + r;
        st2_tf32(sm + OFF_KQ + f32_off(t, c2, R128), nkb[r]);
        st2_tf32(sm + OFF_KQ + f32_off(64 + t, c2, R128), qh[r]);
        st2_tf32(sm + OFF_KN + f32_off(t, c2, R64), kn[r]);
      }
      // that product must be done before Kn^T, O and S are touched (and before this chunk's
      // [A; P] is issued, so that no wait below trails the MMA barrier by two phases)
      const bool ok_op = (c == 0) || wait_mma();
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&ms.bar_ops);
      if (tid == 0) STAMP(c, 6);
      tc_fence_after();
      {
        // Kn^T rows 2 cp and 2 cp + 1, tokens [8 ts, 8 ts + 8) (read by this chunk's last
        // product only; the staging arrival below publishes them).  The first store of each
        // thread goes to row 2 cp + ((cp >> 2) & 1), so that the 8 threads sharing a
        // 128-byte wavefront hit 8 different swizzle phases.
        const int sw = (cp >> 2) & 1;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int rsel = e ^ sw;  // 0: channel 2 cp, 1: channel 2 cp + 1
          float f[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) f[r] = rsel ? kn[r].y : kn[r].x;
          st4_tf32(sm + OFF_PK + f32_off(64 + c2 + rsel, 8 * ts, R192), f);
          st4_tf32(sm + OFF_PK + f32_off(64 + c2 + rsel, 8 * ts + 4, R192), f + 4);
        }
      }
      // ===== while [A; P] is on the tensor cores: the previous chunk's output and state
      // decay ==================================================================================
      if (c > 0) {
        stage_o();
        decay_state(ob ^ 1, c);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&ms.bar_stage);
      // ===== A (sign restored) to the solve scratch, P to its operand tile =====================
      {
        const bool ok_ap = wait_mma();
        tc_fence_after();
        if (tid == 0) STAMP(c, 7);
        float v[16];
        tmem_ld16(tlane + TM_AP + 16 * sg, v);
        tmem_ld_wait();
        if (ch < 64) {
          const int t = ch;
#pragma unroll
          for (int x = 0; x < 16; x += 4) {
            const int s = 16 * sg + x;
            float4 f;
            f.x = (s + 0 < t) ? -v[x + 0] : 0.f;
            f.y = (s + 1 < t) ? -v[x + 1] : 0.f;
            f.z = (s + 2 < t) ? -v[x + 2] : 0.f;
            f.w = (s + 3 < t) ? -v[x + 3] : 0.f;
            *reinterpret_cast<float4*>(Msc + t * LDM + s) = f;
          }
        } else {
          const int t = ch - 64;  // P row, causal incl. diagonal
#pragma unroll
          for (int x = 0; x < 16; x += 4) {
            float f[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) f[m] = (16 * sg + x + m <= t) ? v[x + m] : 0.f;
            st4_tf32(sm + OFF_PK + f32_off(t, 16 * sg + x, R192), f);
          }
        }
        if (named_bar_or(BAR_COMP, NCOMP, !(ok_ap && ok_op))) { dead = true; break; }
      }
      if (tid == 0) STAMP(c, 8);
      // ===== T = (I + A)^-1 on warps 0-3 (warps 4-7 only round U~ below).  Warp k owns the
      // 16-row block k: its two 8x8 diagonal blocks by forward substitution in fp32, then their
      // 16-level merge T_21 = -T_22 (A_21 T_11), all within the warp; then the 32-level merges
      // (warp pairs) and the 64-level merge (the four warps) on warp-level tf32 MMAs
      // (mma.sync m16n8k8).  Every level writes its blocks to the fp32 scratch (read by the next
      // level) and, rounded, to the T operand tile; entries above the 8x8 block diagonal stay
      // zero.  Warps 8-15 meanwhile round R^T in tensor memory once the state product is done.
      bool ok_s = true;
      if (warp < 8) {
        auto put_t = [&](int row, int col, float x) {  // one element of the T operand tile
          *reinterpret_cast<float*>(sm + OFF_T + f32_off(row, col, R64)) = rna_tf32(x);
        };
        auto put_t2 = [&](int row, int col, float x0, float x1) {  // col even
          *reinterpret_cast<float2*>(sm + OFF_T + f32_off(row, col, R64)) = make_float2(rna_tf32(x0), rna_tf32(x1));
        };
        if (warp < 4) {
          const int k = warp, g4 = lane >> 2, t4 = lane & 3;
          float* Xw = Xsc + warp * 32 * LDW;  // this warp's block-product scratch, 32 x LDW
          {
            // 8x8 diagonal blocks 2k (lanes 0-7) and 2k + 1 (lanes 8-15); a lane holds column
            // lane mod 8 of its block (lanes 16-31 repeat lanes 0-15)
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
            // 16-level: T_{2k+1,2k} (8x8) = -T_{2k+1,2k+1} (A_{2k+1,2k} T_{2k,2k}); lane l
            // computes row l / 4, columns 2 (l mod 4) and + 1 of each product
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
          if (tid == 0) STAMP(c, 9);
          // ---- 32-level merges: T_{2m+1,2m} = -T_{2m+1,2m+1} (A_{2m+1,2m} T_{2m,2m}) in 16 x 16
          // blocks; warp 2m + n computes the 8 output columns [8 n, 8 n + 8)
          named_bar_sync(BAR_PAIR + (warp >> 1), 64);
          {
            const int m = warp >> 1, n = warp & 1;
            const int I = 16 * (2 * m + 1), J = 16 * (2 * m);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const float* Ar = Msc + (I + g4) * LDM + J + 8 * ks + t4;
              const float* Bc = Msc + (J + 8 * ks + t4) * LDM + J + 8 * n + g4;
              const uint32_t a[4] = {tfu(Ar[0]), tfu(Ar[8 * LDM]), tfu(Ar[4]), tfu(Ar[8 * LDM + 4])};
              const uint32_t b[2] = {tfu(Bc[0]), tfu(Bc[4 * LDM])};
              mma_16x8x8_tf32(d, a, b);
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
              const uint32_t b[2] = {tfu(Bc[0]), tfu(Bc[4 * LDW])};
              mma_16x8x8_tf32(d, a, b);
            }
            const int row = I + g4, colo = J + 8 * n + 2 * t4;
            *reinterpret_cast<float2*>(Msc + row * LDM + colo) = make_float2(-d[0], -d[1]);
            *reinterpret_cast<float2*>(Msc + (row + 8) * LDM + colo) = make_float2(-d[2], -d[3]);
            put_t2(row, colo, -d[0], -d[1]);
            put_t2(row + 8, colo, -d[2], -d[3]);
          }
          // the diagonal 32x32 blocks of T are in the operand tile: most of the U~ product can go
          fence_proxy_async_smem();
          tc_fence_before();
          warp_arrive(&ms.bar_tdiag);
          if (tid == 0) STAMP(c, 10);
          named_bar_sync(BAR_SOLVE, 128);
          {
            // ---- 64-level merge: T_21 = -T_22 (A_21 T_11) in 32 x 32 blocks; warp k computes the
            // 8 output columns [8 k, 8 k + 8) (T_11 and T_22 are zero above their diagonals, so
            // those k-steps are skipped)
            float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              if (ks < k) continue;
              const float* Bc = Msc + (8 * ks + t4) * LDM + 8 * k + g4;
              const uint32_t b[2] = {tfu(Bc[0]), tfu(Bc[4 * LDM])};
              const float* A0 = Msc + (32 + g4) * LDM + 8 * ks + t4;
              const float* A1 = A0 + 16 * LDM;
              const uint32_t a0[4] = {tfu(A0[0]), tfu(A0[8 * LDM]), tfu(A0[4]), tfu(A0[8 * LDM + 4])};
              const uint32_t a1[4] = {tfu(A1[0]), tfu(A1[8 * LDM]), tfu(A1[4]), tfu(A1[8 * LDM + 4])};
              mma_16x8x8_tf32(d0, a0, b);
              mma_16x8x8_tf32(d1, a1, b);
            }
            __syncwarp();
            *reinterpret_cast<float2*>(Xw + g4 * LDW + 2 * t4) = make_float2(d0[0], d0[1]);
            *reinterpret_cast<float2*>(Xw + (g4 + 8) * LDW + 2 * t4) = make_float2(d0[2], d0[3]);
            *reinterpret_cast<float2*>(Xw + (g4 + 16) * LDW + 2 * t4) = make_float2(d1[0], d1[1]);
            *reinterpret_cast<float2*>(Xw + (g4 + 24) * LDW + 2 * t4) = make_float2(d1[2], d1[3]);
            __syncwarp();
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int ks = 0; ks < 2 + 2 * mt; ++ks) {
                const float* Ar = Msc + (32 + 16 * mt + g4) * LDM + 32 + 8 * ks + t4;
                const float* Bc = Xw + (8 * ks + t4) * LDW + g4;
                const uint32_t a[4] = {tfu(Ar[0]), tfu(Ar[8 * LDM]), tfu(Ar[4]), tfu(Ar[8 * LDM + 4])};
                const uint32_t b[2] = {tfu(Bc[0]), tfu(Bc[4 * LDW])};
                mma_16x8x8_tf32(d, a, b);
              }
              const int row = 32 + 16 * mt + g4, colo = 8 * k + 2 * t4;
              put_t2(row, colo, -d[0], -d[1]);
              put_t2(row + 8, colo, -d[2], -d[3]);
            }
          }
          fence_proxy_async_smem();  // the T operand tile
          tc_fence_before();
          warp_arrive(&ms.bar_solved);
        } else {
          // warps 4-7 take no part in the solve: their arrivals go first
          tc_fence_before();
          warp_arrive(&ms.bar_tdiag);
          warp_arrive(&ms.bar_solved);
        }
        if (tid == 0) STAMP(c, 11);
        // ===== U~^T rounded to tf32 in place: the A operand of the chunk's last product =======
        const bool ok_u = wait_mma();
        tc_fence_after();
        float v[32];
        tmem_ld32(tlane + TM_U + 32 * sg, v);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = rna_tf32(v[x]);
        tmem_st32(tlane + TM_U + 32 * sg, v);
        if (sp_ckpt && p.ck_u && vval) {  // U~ [s][j] of this chunk, for the backward
          float* du = p.ck_u + ((size_t)su * nch + c) * C * dv + ch;
#pragma unroll
          for (int x = 0; x < 32; ++x) du[(size_t)(32 * sg + x) * dv] = v[x];
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(&ms.bar_uround);
        if (tid == 0) STAMP(c, 12);
        ok_prev = ok_u;
        if constexpr (PREP)
          if (c + 1 < nch) ok_prev = norms_ahead(ok_prev);
      } else {
        // (raw projections: the next chunk's Vw^T first, its sigmoid filling the wait for the
        // state product)
        if constexpr (PREP)
          if (c + 1 < nch) ok_s = vw_ahead(c + 1, ok_s);
        // ===== R^T = Vw^T + X^T rounded to tf32 in place once the state product is done ======
        ok_s = ok_s && wait_on(&ms.bar_s, ph_s);
        tc_fence_after();
        {
          float v[32], w[32];
          tmem_ld32(tlane + TM_R + 32 * (sg - 2), v);
          tmem_ld32(tlane + TM_VW + 64 * (c & 1) + 32 * (sg - 2), w);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = rna_tf32(v[x] + w[x]);
          tmem_st32(tlane + TM_R + 32 * (sg - 2), v);
          tmem_st_wait();
        }
        fence_proxy_async_smem();  // this warp's rows of the P operand tile
        tc_fence_before();
        warp_arrive(&ms.bar_tdiag);
        if (tid == 256) STAMP(c, 13);
        // ===== then one chunk ahead: Vw^T and the cumulative decay of the next chunk =========
        if (c + 1 < nch) ok_s = decay_ahead(c + 1, PREP ? ok_s : vw_ahead(c + 1, ok_s));
        if (tid == 256) STAMP(c, 14);
        // These warps do not use U~; they step their phase bit past its product without
        // waiting (by now the chunk's last product may have completed as well, and a parity
        // wait must never trail its barrier by two phases).  Their next wait, on that last
        // product, cannot be overtaken: the barrier's following phase needs these warps.
        ph_mma ^= 1;
        ok_prev = ok_s;
        tc_fence_before();
      }
      // the next chunk reads what warps 8-15 prepared
      if (named_bar_or(BAR_COMP, NCOMP, !ok_prev)) { dead = true; break; }
      if (tid == 0) STAMP(c, 15);
      tc_fence_after();
    }

    if (!dead && nch > 0 && sp_ckpt && p.ck_tt) ckpt_tp(nch - 1);
    // ---- last chunk's output and decay, then the final state -----------------------------
    if (!dead && nch > 0) {
      uint32_t ph_lr = 0;
      const bool ok = ok_prev && wait_mma() && wait_on(&ms.bar_lastread, ph_lr);
      if (named_bar_or(BAR_COMP, NCOMP, !ok)) dead = true;
    }
    if (!dead && nch > 0) {
      tc_fence_after();
      if (VARLEN && len % C) {
        // partial last chunk of a packed sequence: rows straight to o, masked to the sequence
        float v[16];
        tmem_ld16(tlane + TM_O + 16 * sg, v);
        tmem_ld_wait();
        if (vval) {
          const int tb = C * (nch - 1) + 16 * sg;  // token within the sequence
          float* dst = p.o + ((size_t)(t0 + tb) * p.H + h) * dv + ch;
#pragma unroll
          for (int x = 0; x < 16; ++x)
            if (tb + x < len) dst[(size_t)x * p.H * dv] = v[x];
        }
      } else {
        stage_o();
      }
      decay_state((nch - 1) & 1, -1);
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&ms.bar_stage);
    }
    // the final state (for an empty sequence: the entering one)
    // (split: the end of segment 0 starts segment 1, N_s and M_s go to the workspace, the
    // last pass writes S_T from the last segment only)
    float* STu = p.S_T ? p.S_T + (size_t)su * st_sz : nullptr;
    if constexpr (SPLIT) {
      const size_t blk = (size_t)p.nseq * p.split_P * st_sz, at = ((size_t)su * p.split_P + sp_seg) * st_sz;
      if (sp_ckpt)
        STu = nullptr;
      else if (sp_first)
        STu = sp_r == 0 ? p.ws + 2 * blk + at + st_sz : (sp_trans ? p.ws + at : p.ws + blk + at);
      else if (sp_seg != p.split_P - 1)
        STu = nullptr;
    }
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
  // ---- teardown ---------------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// Between the passes of the sequence split: start states S(s + 1) = M_s S(s) + N_s for
// s = 1 .. P - 2 of every (batch, head), S(1) being the first pass's end of segment 0.  One
// CTA per (batch, head, 16 value columns) walks the segments with the running state's
// column slice in shared memory and M_s staged there row by row (rows padded by one
// float so that the 16 rows a warp reads fall in 16 banks); fp32 throughout.
template <int D>
__global__ void __launch_bounds__(256) split_chain_kernel(float* __restrict__ ws, int BH, int P) {
  constexpr int CPT = D / 16;      // value columns per thread
  constexpr int GROUPS = 16 / CPT;  // threads per row
  extern __shared__ float chain_sm[];
  float* Ms = chain_sm;                // D x (D + 1)
  float* Ss = chain_sm + D * (D + 1);  // D x 16
  const int bh = blockIdx.x / (D / 16), j0 = 16 * (blockIdx.x % (D / 16));
  const size_t st = (size_t)D * D;
  const float* M = ws;
  const float* N = ws + (size_t)BH * P * st;
  float* S = ws + 2 * (size_t)BH * P * st;
  const int tid = threadIdx.x, row = tid / GROUPS, jc = CPT * (tid % GROUPS);
  constexpr int NQ = D * D / 4 / 256;  // float4 of M per thread
  float4 mq[NQ];                       // the next M, in flight while the current one is used
  auto fetch = [&](int sgm) {
    const float4* Mg = reinterpret_cast<const float4*>(M + ((size_t)bh * P + sgm) * st);
#pragma unroll
    for (int m = 0; m < NQ; ++m) mq[m] = __ldg(Mg + tid + 256 * m);
  };
  auto stage = [&]() {
#pragma unroll
    for (int m = 0; m < NQ; ++m) {
      const int e = 4 * (tid + 256 * m), r = e / D, c = e % D;
      Ms[r * (D + 1) + c] = mq[m].x;
      Ms[r * (D + 1) + c + 1] = mq[m].y;
      Ms[r * (D + 1) + c + 2] = mq[m].z;
      Ms[r * (D + 1) + c + 3] = mq[m].w;
    }
  };
  for (int e = tid; e < D * 16; e += 256)
    Ss[e] = S[((size_t)bh * P + 1) * st + (size_t)(e / 16) * D + j0 + e % 16];
  if (P > 2) {
    fetch(1);
    stage();
  }
  __syncthreads();
  for (int sgm = 1; sgm + 1 < P; ++sgm) {
    if (sgm + 2 < P) fetch(sgm + 1);
    const float* Ng = N + ((size_t)bh * P + sgm) * st + (size_t)row * D + j0 + jc;
    float acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = Ng[c];
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float m = Ms[row * (D + 1) + i];
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[c] = fmaf(m, Ss[i * 16 + jc + c], acc[c]);
    }
    __syncthreads();  // every read of the slice and of M_s is done
    float* Sg = S + ((size_t)bh * P + sgm + 1) * st + (size_t)row * D + j0 + jc;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      Ss[row * 16 + jc + c] = acc[c];
      Sg[c] = acc[c];
    }
    if (sgm + 2 < P) stage();
    __syncthreads();
  }
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

// [B, T, H, D] tensor; one box = box_t tokens x box_d channels of one (b, h).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int B, int T, int H, int D,
              int box_d, CUtensorMapSwizzle swz, int box_t = C) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize, (cuuint64_t)T * H * D * esize};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)box_t, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int DK, int DV, bool VARLEN, bool PREP, bool SPLIT = false>
cudaError_t launch_shape(int grid, cudaStream_t st, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mb, const CUtensorMap& mw, const CUtensorMap& mla,
                         const CUtensorMap& mo, const TcParams& p) {
  static std::atomic<unsigned long long> attr_done{0};  // per instantiation, a bit per device
  cudaError_t e = smem_limit_once(chunk_fwd_tc_kernel<DK, DV, VARLEN, PREP, SPLIT>, (int)SMEM_BYTES, attr_done);
  if (e != cudaSuccess) return e;
  chunk_fwd_tc_kernel<DK, DV, VARLEN, PREP, SPLIT><<<grid, NT, SMEM_BYTES, st>>>(mq, mk, mv, mb, mw, mla, mo, p);
  return cudaSuccess;
}

}  // namespace

template <bool VARLEN, bool PREP>
cudaError_t launch_dims(int grid, cudaStream_t st, const CUtensorMap& mq, const CUtensorMap& mk,
                        const CUtensorMap& mv, const CUtensorMap& mb, const CUtensorMap& mw, const CUtensorMap& mla,
                        const CUtensorMap& mo, const TcParams& p) {
  if (p.dk == 128 && p.dv == 128) return launch_shape<128, 128, VARLEN, PREP>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  if (p.dk == 128 && p.dv == 64) return launch_shape<128, 64, VARLEN, PREP>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  if (p.dk == 64 && p.dv == 128) return launch_shape<64, 128, VARLEN, PREP>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  if (p.dk == 64 && p.dv == 64) return launch_shape<64, 64, VARLEN, PREP>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  return cudaErrorInvalidValue;
}

cudaError_t launch_split(const ChunkArgs& a, TcParams p, cudaStream_t st, const CUtensorMap& mq,
                         const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mb, const CUtensorMap& mw,
                         const CUtensorMap& mla, const CUtensorMap& mo) {
  const int nch = (a.T + C - 1) / C;
  const int L = C * ((nch + a.split - 1) / a.split);  // tokens per segment
  const int P = (a.T + L - 1) / L;                      // segments actually used (<= a.split)
  const int BH = a.B * a.H;
  if (P < 2) return launch_dims<false, false>(BH, st, mq, mk, mv, mb, mw, mla, mo, p);
  p.nseq = BH;
  p.split_P = P;
  p.split_L = L;
  p.ws = a.workspace;
  auto pass = [&](int grid) {  // d_k = d_v
    return a.dk == 128 ? launch_shape<128, 128, false, false, true>(grid, st, mq, mk, mv, mb, mw, mla, mo, p)
                       : launch_shape<64, 64, false, false, true>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  };
  p.split_phase = 1;
  // first pass: segment 0, and N_s, M_s for s = 1 .. P - 2 (the chain reads no others)
  cudaError_t e = pass(BH * (2 * P - 3));
  if (e != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (P > 2) {
    const int D = a.dk;
    const size_t smem = (size_t)(D * (D + 1) + D * 16) * sizeof(float);
    if (D == 128) {
      static std::atomic<unsigned long long> attr_done{0};
      if ((e = smem_limit_once(split_chain_kernel<128>, (int)smem, attr_done)) != cudaSuccess) return e;
      split_chain_kernel<128><<<BH * (D / 16), 256, smem, st>>>(a.workspace, BH, P);
    } else {
      split_chain_kernel<64><<<BH * (D / 16), 256, smem, st>>>(a.workspace, BH, P);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  p.split_phase = 3;
  return pass(BH * (P - 1));
}

size_t chunk_fwd_tc_smem_bytes() { return SMEM_BYTES; }

// The state entering every chunk ([B H][chunk][d_k][d_v] fp32 at `states`), for the backward
// pass: the split instantiation's checkpoint phase over whole sequences (bf16, d_k = d_v).
cudaError_t launch_chunk_states_tc(const ChunkArgs& a, float* states, cudaStream_t st, float* ck_u, float* ck_tt,
                                   float* ck_pt) {
  if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
  if (a.dk != a.dv || !a.bf16) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mb, mw, mla, mo;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  // o is never written in this phase: the map only needs a valid, aligned address
  bool ok = make_map(&mq, a.q, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mk, a.k, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mb, a.b, BF, 2, a.B, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mv, a.v, BF, 2, a.B, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mw, a.w, BF, 2, a.B, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, a.dk, 32, SW) &&
            make_map(&mo, states, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, a.dv, a.dv,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  TcParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.b = static_cast<const __nv_bfloat16*>(a.b);
  p.w = static_cast<const __nv_bfloat16*>(a.w);
  p.S0 = a.S0;
  p.S_T = nullptr;
  p.o = nullptr;
  p.T = a.T;
  p.H = a.H;
  p.dk = a.dk;
  p.dv = a.dv;
  p.cu_seqlens = nullptr;
  p.nseq = a.B * a.H;
  p.dscale = nullptr;
  p.err = device_error_word();
  p.stamps = stamp_buffer();
  p.split_phase = 5;
  p.split_P = 1;
  p.split_L = a.T;
  p.ws = states;
  p.ck_u = ck_u;
  p.ck_tt = ck_tt;
  p.ck_pt = ck_pt;
  const int grid = a.B * a.H;
  cudaError_t e = a.dk == 128 ? launch_shape<128, 128, false, false, true>(grid, st, mq, mk, mv, mb, mw, mla, mo, p)
                              : launch_shape<64, 64, false, false, true>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_chunk_fwd_tc(const ChunkArgs& a, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  // packed sequences: one [1, total T, H, D] tensor, sequence n = tokens [cu[n], cu[n+1])
  const bool varlen = a.cu_seqlens != nullptr;
  const int Bm = varlen ? 1 : a.B;
  CUtensorMap mq, mk, mv, mb, mw, mla, mo;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = make_map(&mq, a.q, BF, 2, Bm, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mk, a.k, BF, 2, Bm, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mb, a.b, BF, 2, Bm, a.T, a.H, a.dk, 64, SW) &&
            make_map(&mv, a.v, BF, 2, Bm, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mw, a.w, BF, 2, Bm, a.T, a.H, a.dv, 64, SW) &&
            make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, Bm, a.T, a.H, a.dk, 32, SW) &&
            make_map(&mo, a.o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, Bm, a.T, a.H, a.dv, a.dv,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
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
  p.cu_seqlens = a.cu_seqlens;
  p.nseq = varlen ? a.B : 0;
  p.err = device_error_word();
  p.stamps = stamp_buffer();
  const int grid = a.B * a.H;
  p.dscale = a.decay_scale;
  cudaError_t e;
  if (a.split > 1 && !varlen && !a.raw && a.dk == a.dv) {
    e = launch_split(a, p, st, mq, mk, mv, mb, mw, mla, mo);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (a.raw)
    e = varlen ? launch_dims<true, true>(grid, st, mq, mk, mv, mb, mw, mla, mo, p)
               : launch_dims<false, true>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  else
    e = varlen ? launch_dims<true, false>(grid, st, mq, mk, mv, mb, mw, mla, mo, p)
               : launch_dims<false, false>(grid, st, mq, mk, mv, mb, mw, mla, mo, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace gdn2
