// Chunkwise prefill forward at chunk size C = 128 for bf16 inputs on the 5th-generation tensor
// cores, the largest size of the chunk-size trade-off (snilld.dk, "POC-matrix der daekker de
// haarde hjoerner": latency, throughput and memory at C = 32, 64 and 128).  Same algorithm and
// notation as chunk_tc.cu (Gated DeltaNet-2 guide, "Chunkwise Parallel Algorithm for GPU
// Training"; WY form with the cumulative decay folded into the factors, snilld.dk, "Hvad
// betyder det for traening og inferens"):
//
//     [-A; P] = [-Kb; Qh] Kn^T              T = (I + A)^-1
//     [R^T | X^T] = S^T [-Kb; Qh]^T         R^T <- Vw^T + R^T        U~^T = R^T T^T
//     S^T <- S^T Diag(Gamma_C)              [X^T | S^T] += U~^T [P; (Kn Diag(Gamma_C))^T]^T
//
// X^T becomes O^T.  Why a design of its own: the production kernel keeps every tile of a chunk
// resident and overlaps the next chunk's preparation with the current one; at 128 tokens those
// tiles (the stacked [-Kb; Qh] 128 KB, Kn 64 KB, [P; Kn^T] 128 KB, T 64 KB, all tf32) are far
// over one SM's 227 KB of shared memory, and [-A; P], R^T, X^T, U~^T and S^T need 768 of 512
// tensor-memory columns.  Here the phases of a chunk run one after another, every product's
// completion awaited before the next phase, and the memory is reused inside the chunk:
//   shared region X: the stacked [-Kb; Qh] tile (A operand of [-A; P], B operand of the state
//                    product); once the state product has read it, the [P; Kn Gamma_C ^T] tile
//   shared region Y: Kn (B operand of [-A; P]); then A, inverted into T in place
//   tensor memory:   R^T | X^T (= O^T) | S^T | U~^T; [-A; P] lands in the R^T and U~^T columns
// The solve: 16 x 16 diagonal blocks by forward substitution, then 32-, 64- and 128-level
// block merges T_IJ = -T_II (A_IJ T_JJ) on warp-level tf32 MMAs, in place (a merge reads only
// the off-diagonal block it then overwrites and diagonal blocks already inverted).  One CTA
// of 16 warps per (batch, head); inputs are read with plain coalesced loads from L2, where the
// previous chunk prefetched them (tensor-map box prefetches), every load of a phase issued
// before any is used (clamped token index, values past the sequence end zeroed).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int C = 128;
constexpr int NT = 512;                         // 16 warps
constexpr uint64_t WAIT_LIMIT = 2000000000ull;  // 2 s of wall time per wait
constexpr float LOG2E = 1.4426950408889634f;
constexpr float G2_MIN = -115.4f;  // in-chunk cumulative log2 decay below which 2^-g leaves fp32

// ---- shared memory map (byte offsets from a 1024-byte aligned base) ----------------------
// fp32 operand tiles: 32-column panels of 128-byte rows, 128-byte swizzle (f32_off)
constexpr uint32_t R128 = 128 * 128;        // a panel of 128 rows
constexpr uint32_t R256 = 256 * 128;        // a panel of 256 rows
constexpr uint32_t OFF_X = 0;               // [-Kb; Qh] [t][i], then [P; Kn Gamma_C ^T] [t | i][s]
constexpr uint32_t OFF_Y = OFF_X + 4 * R256;  // Kn [s][i], then A -> T [s][t]
constexpr uint32_t OFF_Z = OFF_Y + 4 * R128;  // solve scratch: the merges' A_IJ T_JJ, 64 x LDZ fp32;
                                              // in the operand build, the decay partials per range
constexpr int LDZ = 72;
constexpr uint32_t TILES = OFF_Z + 64 * LDZ * 4;

struct Misc {
  uint64_t bar_mma, bar_drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float gC[128];      // Gamma at the chunk end, per key channel
};
constexpr uint32_t SMEM_BYTES = TILES + 1024 + sizeof(Misc);

// ---- tensor memory columns (fp32, 128 lanes) ---------------------------------------------
constexpr uint32_t TM_R = 0;    // R^T  lanes: value channel, columns: t   (first -A: lanes t, columns s)
constexpr uint32_t TM_O = 128;  // X^T, then O^T
constexpr uint32_t TM_S = 256;  // S^T  lanes: value channel, columns: key channel
constexpr uint32_t TM_U = 384;  // U~^T lanes: value channel, columns: s   (first P: lanes t, columns s)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_128 = idesc_tf32(128, 128, 0, 0, 0, 0);
constexpr uint32_t ID_64 = idesc_tf32(128, 64, 0, 0, 0, 0);

struct Tc128Params {
  const __nv_bfloat16 *q, *k, *v, *b, *w;
  const float* la;
  const float* S0;
  float* o;
  float* S_T;
  int T, H;
  unsigned* err;
  unsigned long long* stamps;  // instrumented build only
};

#ifdef GDN2_STAMPS
// Instrumented build (GDN2_STAMPS): clock64 at the phase boundaries of the first CTA, written
// by thread 0 into [chunk][slot] of a 64 x 32 array (slots 0-18).
#define TC128_STAMP(c, slot)                                                                  \
  do {                                                                                        \
    if (p.stamps && blockIdx.x == 0 && threadIdx.x == 0 && (c) < 64)                          \
      p.stamps[(size_t)(c) * 32 + (slot)] = (unsigned long long)clock64();                    \
  } while (0)
#else
#define TC128_STAMP(c, slot) \
  do {                       \
  } while (0)
#endif

__device__ __forceinline__ float rna_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}
__device__ __forceinline__ uint32_t tfu(float x) { return __float_as_uint(rna_tf32(x)); }
__device__ __forceinline__ void st4_tf32(unsigned char* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(rna_tf32(f[0]), rna_tf32(f[1]), rna_tf32(f[2]), rna_tf32(f[3]));
}
// the low and high bf16 of a 32-bit word as fp32
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ uint64_t kdesc(uint32_t base, uint32_t panel, int ks) {
  return sdesc_sw128(base + (uint32_t)(ks >> 2) * panel + (uint32_t)(ks & 3) * 32, 16, 1024);
}
// element (r, c) of the 128 x 128 fp32 matrix in region Y
__device__ __forceinline__ float& ye(unsigned char* Y, int r, int c) {
  return *reinterpret_cast<float*>(Y + f32_off(r, c, R128));
}

// One level of the in-place inversion: for every pair of H x H diagonal blocks (J, I = J + H)
// of the 2H-level, T_IJ = -T_II (A_IJ T_JJ).  Output tiles of 16 x 8 are spread over the 16
// warps; the lower-triangular T_JJ and T_II let each product skip the blocks that vanish.
template <int H>
__device__ __forceinline__ void merge_level(unsigned char* Y, float* Zs, int warp, int lane) {
  constexpr int TPM = (H / 16) * (H / 8);  // output tiles per merge
  constexpr int NTILE = TPM * (C / (2 * H));
  const int g4 = lane >> 2, t4 = lane & 3;
  // Z = A_IJ T_JJ
  for (int tile = warp; tile < NTILE; tile += NT / 32) {
    const int m = tile / TPM, r = tile % TPM, rt = r / (H / 8), ct = r % (H / 8);
    const int J = 2 * H * m, I = J + H;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k8 = ct; k8 < H / 8; ++k8) {  // rows of T_JJ above its column block vanish
      const int ar = I + 16 * rt + g4, ac = J + 8 * k8 + t4;
      const uint32_t a[4] = {tfu(ye(Y, ar, ac)), tfu(ye(Y, ar + 8, ac)), tfu(ye(Y, ar, ac + 4)),
                             tfu(ye(Y, ar + 8, ac + 4))};
      const int br = J + 8 * k8 + t4, bc = J + 8 * ct + g4;
      const uint32_t b2[2] = {tfu(ye(Y, br, bc)), tfu(ye(Y, br + 4, bc))};
      mma_16x8x8_tf32(d, a, b2);
    }
    float* z = Zs + (H * m + 16 * rt + g4) * LDZ + 8 * ct + 2 * t4;
    z[0] = d[0];
    z[1] = d[1];
    z[8 * LDZ] = d[2];
    z[8 * LDZ + 1] = d[3];
  }
  __syncthreads();
  // T_IJ = -T_II Z, over the A_IJ block the first product has finished reading
  for (int tile = warp; tile < NTILE; tile += NT / 32) {
    const int m = tile / TPM, r = tile % TPM, rt = r / (H / 8), ct = r % (H / 8);
    const int J = 2 * H * m, I = J + H;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k8 = 0; k8 < 2 * rt + 2; ++k8) {  // columns of T_II past its row block vanish
      const int ar = I + 16 * rt + g4, ac = I + 8 * k8 + t4;
      const uint32_t a[4] = {tfu(ye(Y, ar, ac)), tfu(ye(Y, ar + 8, ac)), tfu(ye(Y, ar, ac + 4)),
                             tfu(ye(Y, ar + 8, ac + 4))};
      const float* zb = Zs + (H * m + 8 * k8 + t4) * LDZ + 8 * ct + g4;
      const uint32_t b2[2] = {tfu(zb[0]), tfu(zb[4 * LDZ])};
      mma_16x8x8_tf32(d, a, b2);
    }
    const int row = I + 16 * rt + g4, col = J + 8 * ct + 2 * t4;
    ye(Y, row, col) = -d[0];
    ye(Y, row, col + 1) = -d[1];
    ye(Y, row + 8, col) = -d[2];
    ye(Y, row + 8, col + 1) = -d[3];
  }
  __syncthreads();
}

// T = (I + A)^-1 in place: region Y holds the strictly lower A (zero on and above the
// diagonal) and ends holding T in fp32 (unit diagonal, zero above it).
__device__ __forceinline__ void solve_in_place(unsigned char* Y, float* Zs, int warp, int lane) {
  if (warp < 4) {
    // 16 x 16 diagonal blocks: half-warp = block, lane = column; T[r][col] = -sum A[r][s] T[s][col]
    const int r0 = 16 * (2 * warp + (lane >> 4)), col = lane & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) x[r] = (r == col) ? 1.f : 0.f;
#pragma unroll
    for (int r = 1; r < 16; ++r) {
      float a[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float4 f = *reinterpret_cast<const float4*>(Y + f32_off(r0 + r, r0 + 4 * q4, R128));
        a[4 * q4] = f.x;
        a[4 * q4 + 1] = f.y;
        a[4 * q4 + 2] = f.z;
        a[4 * q4 + 3] = f.w;
      }
      float acc = 0.f;
#pragma unroll
      for (int s = 0; s < r; ++s) acc = fmaf(a[s], x[s], acc);
      if (r > col) x[r] = -acc;
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r >= col) ye(Y, r0 + r, r0 + col) = x[r];
  }
  __syncthreads();
  merge_level<16>(Y, Zs, warp, lane);
  merge_level<32>(Y, Zs, warp, lane);
  merge_level<64>(Y, Zs, warp, lane);
}

// DK, DV: key and value head dimensions (64 or 128).
template <int DK, int DV>
__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmV,
                           const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmLA,
                           const Tc128Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Misc& ms = *reinterpret_cast<Misc*>(sm + TILES);
  const uint32_t sbase = smem_u32(sm);
  unsigned char* Y = sm + OFF_Y;
  float* Zs = reinterpret_cast<float*>(sm + OFF_Z);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ch = tid & 127;  // tensor-memory lane: token (for [-A; P]) or value channel
  const int sg = tid >> 7;   // column group [32 sg, 32 sg + 32) of tensor-memory accesses
  const int unit = blockIdx.x, h = unit % p.H, bb = unit / p.H;
  const int len = p.T, nch = (len + C - 1) / C;
  constexpr int PARTS = NT / DK, TPP = C / PARTS;     // Kn Gamma_C rows: token ranges per key channel
  constexpr uint32_t KQP = R256;                      // a panel of [-Kb; Qh]
  constexpr uint32_t PKP = (uint32_t)(C + DK) * 128;  // a panel of [P; Kn Gamma_C ^T]
  const int bi = tid % DK, part = tid / DK;           // Kn Gamma_C rows: key channel, token range
  constexpr int QPARTS = NT / (DK / 4), QTP = C / QPARTS;  // operand build: token ranges per channel quad
  const int cq = tid % (DK / 4), qp = tid / (DK / 4);      // operand build: channel quad, token range
  auto tok = [&](int t) -> size_t { return ((size_t)bb * len + t) * p.H + h; };

  if (tid == 0) {
    mbar_init(&ms.bar_mma, 1);
    mbar_init(&ms.bar_drain, 1);
    fence_mbar_init();
    ms.abort = 0;
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

  uint32_t ph = 0;
  // Thread 0 polls the commit barrier of the products it issued; the block learns the outcome
  // (and the products' results become visible to its tensor-memory reads) at the barrier.
  auto mma_done = [&]() -> bool {
    bool ok = true;
    if (tid == 0) ok = mbar_wait_spin(&ms.bar_mma, ph, &ms.abort, p.err, WAIT_LIMIT);
    ph ^= 1;
    tc_fence_before();
    const bool bad = __syncthreads_or(!ok);
    tc_fence_after();
    return !bad;
  };
  // Shared-memory tiles and tensor-memory stores of the block, visible to the products
  // thread 0 issues next.
  auto handoff = [&]() {
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  // chunk cc's input tiles into L2 (thread 0, one box per 128-byte channel panel), one chunk
  // ahead, so that the operand build and the Vw pass read from L2 rather than wait on DRAM
  auto prefetch_chunk = [&](int cc) {
    if (tid != 0) return;
    for (int pn = 0; pn < DK / 32; ++pn) tma_prefetch_l2_4d(&tmLA, 32 * pn, h, C * cc, bb);
    for (int pn = 0; pn < DK / 64; ++pn) {
      tma_prefetch_l2_4d(&tmQ, 64 * pn, h, C * cc, bb);
      tma_prefetch_l2_4d(&tmK, 64 * pn, h, C * cc, bb);
      tma_prefetch_l2_4d(&tmB, 64 * pn, h, C * cc, bb);
    }
    for (int pn = 0; pn < DV / 64; ++pn) {
      tma_prefetch_l2_4d(&tmV, 64 * pn, h, C * cc, bb);
      tma_prefetch_l2_4d(&tmW, 64 * pn, h, C * cc, bb);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmLA);
  }
  if (nch > 0) prefetch_chunk(0);

  if (32 * sg < DK) {  // entering state S0 -> S^T (lane j = ch, key channels [32 sg, 32 sg + 32))
    const float* S0u = p.S0 ? p.S0 + (size_t)unit * DK * DV : nullptr;
    float v[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) v[x] = (S0u && ch < DV) ? S0u[(size_t)(32 * sg + x) * DV + ch] : 0.f;
    tmem_st32(tlane + TM_S + 32 * sg, v);
    tmem_st_wait();
  }
  handoff();

  bool dead = false;
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * C, n = min(C, len - t0);
    TC128_STAMP(c, 0);
    // ===== 1. cumulative decay and the folded operands: thread (key channels [4 cq, 4 cq + 4),
    // tokens [QTP qp, QTP qp + QTP)); a warp's loads cover whole token rows (16-byte log-alpha
    // and 8-byte bf16 groups), issued at clamped tokens before any is used, values past the
    // sequence end zeroed
    {
      float4 g[QTP];
#pragma unroll
      for (int r = 0; r < QTP; ++r) {
        const int t = QTP * qp + r;
        g[r] = *reinterpret_cast<const float4*>(p.la + tok(t0 + min(t, n - 1)) * DK + 4 * cq);
      }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < QTP; ++r) {
        const bool z = QTP * qp + r >= n;
        acc.x = fmaf(z ? 0.f : g[r].x, LOG2E, acc.x);
        acc.y = fmaf(z ? 0.f : g[r].y, LOG2E, acc.y);
        acc.z = fmaf(z ? 0.f : g[r].z, LOG2E, acc.z);
        acc.w = fmaf(z ? 0.f : g[r].w, LOG2E, acc.w);
        g[r] = acc;
      }
      float4* segtot = reinterpret_cast<float4*>(Zs);  // [QPARTS][DK / 4]: the solve scratch, free here
      segtot[qp * (DK / 4) + cq] = acc;
      __syncthreads();
      TC128_STAMP(c, 1);
      float4 off = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < qp; ++q) {
        const float4 f = segtot[q * (DK / 4) + cq];
        off.x += f.x;
        off.y += f.y;
        off.z += f.z;
        off.w += f.w;
      }
      if (qp == QPARTS - 1) {
        const float4 tot = make_float4(off.x + acc.x, off.y + acc.y, off.z + acc.z, off.w + acc.w);
        *reinterpret_cast<float4*>(&ms.gC[4 * cq]) =
            make_float4(ex2_approx(tot.x), ex2_approx(tot.y), ex2_approx(tot.z), ex2_approx(tot.w));
        if (fminf(fminf(tot.x, tot.y), fminf(tot.z, tot.w)) < G2_MIN && p.err) atomicOr(p.err, kErrDecayRange);
      }
      TC128_STAMP(c, 17);
#pragma unroll
      for (int r0 = 0; r0 < QTP; r0 += 2) {  // two tokens' loads in flight at a time
        uint2 kk[2], bg[2], qq[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const size_t e = tok(t0 + min(QTP * qp + r0 + r, n - 1)) * DK + 4 * cq;
          kk[r] = *reinterpret_cast<const uint2*>(p.k + e);
          bg[r] = *reinterpret_cast<const uint2*>(p.b + e);
          qq[r] = *reinterpret_cast<const uint2*>(p.q + e);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int t = QTP * qp + r0 + r;
          const bool z = t >= n;
          const float k4[4] = {bf_lo(kk[r].x), bf_hi(kk[r].x), bf_lo(kk[r].y), bf_hi(kk[r].y)};
          const float b4[4] = {bf_lo(bg[r].x), bf_hi(bg[r].x), bf_lo(bg[r].y), bf_hi(bg[r].y)};
          const float q4[4] = {bf_lo(qq[r].x), bf_hi(qq[r].x), bf_lo(qq[r].y), bf_hi(qq[r].y)};
          const float gl[4] = {g[r0 + r].x + off.x, g[r0 + r].y + off.y, g[r0 + r].z + off.z, g[r0 + r].w + off.w};
          float nkb[4], qh[4], kn[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float G = ex2_approx(gl[m]), Gi = rcp_approx(G);
            const float kv = z ? 0.f : k4[m];
            nkb[m] = -(kv * b4[m]) * G;
            qh[m] = (z ? 0.f : q4[m]) * G;
            kn[m] = kv * Gi;
          }
          st4_tf32(sm + OFF_X + f32_off(t, 4 * cq, KQP), nkb);
          st4_tf32(sm + OFF_X + f32_off(C + t, 4 * cq, KQP), qh);
          st4_tf32(Y + f32_off(t, 4 * cq, R128), kn);
        }
      }
    }
    handoff();
    TC128_STAMP(c, 2);
    // ===== 2. [-A; P] = [-Kb; Qh] Kn^T: two M = 128 products, -A to the R^T columns, P to U~^T's
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < DK / 8; ++ks)
        umma_tf32_ss(tmem + TM_R, kdesc(sbase + OFF_X, KQP, ks), kdesc(sbase + OFF_Y, R128, ks), ID_128, ks > 0);
#pragma unroll
      for (int ks = 0; ks < DK / 8; ++ks)
        umma_tf32_ss(tmem + TM_U, kdesc(sbase + OFF_X + R128, KQP, ks), kdesc(sbase + OFF_Y, R128, ks), ID_128,
                     ks > 0);
      umma_commit(&ms.bar_mma);
    }
    if (!mma_done()) { dead = true; break; }
    TC128_STAMP(c, 3);
    // ===== 3. this thread's Kn values (for the Kn Gamma_C rows), then A (sign restored,
    // strictly lower) over the Kn tile the product has read
    float knr[TPP];
#pragma unroll
    for (int r = 0; r < TPP; ++r) knr[r] = *reinterpret_cast<const float*>(Y + f32_off(TPP * part + r, bi, R128));
    {
      float v[32];
      tmem_ld32(tlane + TM_R + 32 * sg, v);
      tmem_ld_wait();
      __syncthreads();  // every Kn read precedes the A writes
      const int t = ch;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        const int s = 32 * sg + x;
        float4 f;
        f.x = (s + 0 < t) ? -v[x + 0] : 0.f;
        f.y = (s + 1 < t) ? -v[x + 1] : 0.f;
        f.z = (s + 2 < t) ? -v[x + 2] : 0.f;
        f.w = (s + 3 < t) ? -v[x + 3] : 0.f;
        *reinterpret_cast<float4*>(Y + f32_off(t, s, R128)) = f;
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    TC128_STAMP(c, 4);
    // ===== 4. [R^T | X^T] = S^T [-Kb; Qh]^T on the tensor cores while the block solves for T
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < DK / 8; ++ks)
        umma_tf32_ts(tmem + TM_R, tmem + TM_S + 8 * ks, kdesc(sbase + OFF_X, KQP, ks), ID_128, ks > 0);
#pragma unroll
      for (int ks = 0; ks < DK / 8; ++ks)
        umma_tf32_ts(tmem + TM_O, tmem + TM_S + 8 * ks, kdesc(sbase + OFF_X + R128, KQP, ks), ID_128, ks > 0);
      umma_commit(&ms.bar_mma);
    }
    if (c + 1 < nch) prefetch_chunk(c + 1);
    TC128_STAMP(c, 18);
    solve_in_place(Y, Zs, warp, lane);
    TC128_STAMP(c, 5);
    if (!mma_done()) { dead = true; break; }
    TC128_STAMP(c, 6);
    // ===== 5. operands of the chunk's last two products
    {  // P (causal, diagonal included) into rows 0-127 of [P; Kn Gamma_C ^T]: the KQ tile is read
      float v[32];
      tmem_ld32(tlane + TM_U + 32 * sg, v);
      tmem_ld_wait();
      const int t = ch;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        const int s = 32 * sg + x;
        float f[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) f[m] = (s + m <= t) ? v[x + m] : 0.f;
        st4_tf32(sm + OFF_X + f32_off(t, s, PKP), f);
      }
    }
    TC128_STAMP(c, 12);
    {  // rows C + i: Kn Gamma_C, i.e. k_s Gamma_C / Gamma_s
      const float gc = ms.gC[bi];
#pragma unroll
      for (int r = 0; r < TPP; r += 4) {
        const float f[4] = {knr[r] * gc, knr[r + 1] * gc, knr[r + 2] * gc, knr[r + 3] * gc};
        st4_tf32(sm + OFF_X + f32_off(C + bi, TPP * part + r, PKP), f);
      }
    }
    TC128_STAMP(c, 13);
    {  // R^T <- Vw^T + R^T rounded to tf32 in place (lane j = ch, tokens [32 sg, 32 sg + 32), in
       // two halves of 16)
      const int j = ch;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float x[16], vw[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int t = 32 * sg + 16 * hf + r;
          const size_t e = tok(t0 + min(t, n - 1)) * DV + (j < DV ? j : 0);
          vw[r] = __bfloat162float(p.v[e]) * __bfloat162float(p.w[e]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r)
          if (32 * sg + 16 * hf + r >= n || j >= DV) vw[r] = 0.f;
        tmem_ld16(tlane + TM_R + 32 * sg + 16 * hf, x);
        tmem_ld_wait();
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = rna_tf32(x[r] + vw[r]);
        tmem_st16(tlane + TM_R + 32 * sg + 16 * hf, x);
      }
    }
    TC128_STAMP(c, 14);
    if (32 * sg < DK) {  // S^T <- S^T Diag(Gamma_C): the state product has read S^T
      float x[32];
      tmem_ld32(tlane + TM_S + 32 * sg, x);
      tmem_ld_wait();
#pragma unroll
      for (int r = 0; r < 32; r += 4) {
        const float4 gq = *reinterpret_cast<const float4*>(&ms.gC[32 * sg + r]);
        x[r] *= gq.x;
        x[r + 1] *= gq.y;
        x[r + 2] *= gq.z;
        x[r + 3] *= gq.w;
      }
      tmem_st32(tlane + TM_S + 32 * sg, x);
    }
    tmem_st_wait();
    TC128_STAMP(c, 15);
    for (int e = tid; e < C * C / 4; e += NT) {  // T rounded to tf32 in place
      float4* p4 = reinterpret_cast<float4*>(Y) + e;
      const float4 f = *p4;
      *p4 = make_float4(rna_tf32(f.x), rna_tf32(f.y), rna_tf32(f.z), rna_tf32(f.w));
    }
    TC128_STAMP(c, 16);
    handoff();
    TC128_STAMP(c, 7);
    // ===== 6. U~^T = R^T T^T (K = t)
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < C / 8; ++ks)
        umma_tf32_ts(tmem + TM_U, tmem + TM_R + 8 * ks, kdesc(sbase + OFF_Y, R128, ks), ID_128, ks > 0);
      umma_commit(&ms.bar_mma);
    }
    if (!mma_done()) { dead = true; break; }
    TC128_STAMP(c, 8);
    {  // U~^T rounded to tf32 in place: the A operand of the last product
      float x[32];
      tmem_ld32(tlane + TM_U + 32 * sg, x);
      tmem_ld_wait();
#pragma unroll
      for (int r = 0; r < 32; ++r) x[r] = rna_tf32(x[r]);
      tmem_st32(tlane + TM_U + 32 * sg, x);
      tmem_st_wait();
    }
    handoff();
    TC128_STAMP(c, 9);
    // ===== 7. [O^T | S^T] += U~^T [P; Kn Gamma_C ^T]^T (K = s)
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < C / 8; ++ks)
        umma_tf32_ts(tmem + TM_O, tmem + TM_U + 8 * ks, kdesc(sbase + OFF_X, PKP, ks), ID_128, 1);
#pragma unroll
      for (int ks = 0; ks < C / 8; ++ks)
        umma_tf32_ts(tmem + TM_S, tmem + TM_U + 8 * ks, kdesc(sbase + OFF_X + C * 128, PKP, ks),
                     DK == 128 ? ID_128 : ID_64, 1);
      umma_commit(&ms.bar_mma);
    }
    if (!mma_done()) { dead = true; break; }
    TC128_STAMP(c, 10);
    {  // ===== 8. O^T -> o (lane j = ch: a warp stores 32 consecutive value channels of a token)
      float x[32];
      tmem_ld32(tlane + TM_O + 32 * sg, x);
      tmem_ld_wait();
      if (ch < DV) {
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          const int t = 32 * sg + r;
          if (t < n) p.o[tok(t0 + t) * DV + ch] = x[r];
        }
      }
    }
    TC128_STAMP(c, 11);
    tc_fence_before();  // the next chunk's state product overwrites O^T after the next barrier
  }

  if (dead) {
    if (tid == 0) {  // every product issued lands before the block releases its memory
      volatile int never = 0;
      umma_commit(&ms.bar_drain);
      mbar_wait_bounded(&ms.bar_drain, 0, &never, nullptr, WAIT_LIMIT);
    }
  } else if (p.S_T && 32 * sg < DK) {
    float v[32];
    tmem_ld32(tlane + TM_S + 32 * sg, v);
    tmem_ld_wait();
    if (ch < DV) {
      float* STu = p.S_T + (size_t)unit * DK * DV;
#pragma unroll
      for (int x = 0; x < 32; ++x) STu[(size_t)(32 * sg + x) * DV + ch] = v[x];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

PFN_cuTensorMapEncodeTiled_v12000 encode128() {
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
// [B, T, H, D] tensor; one box = 128 bytes of channels x C tokens of one (b, h), for L2 prefetches
bool map128(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int B, int T, int H, int D) {
  auto fn = encode128();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize, (cuuint64_t)T * H * D * esize};
  cuuint32_t box[4] = {(cuuint32_t)(128 / esize), 1, (cuuint32_t)C, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
cudaError_t launch128(const ChunkArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mb, mv, mw, mla;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!map128(&mq, a.q, BF, 2, a.B, a.T, a.H, DK) || !map128(&mk, a.k, BF, 2, a.B, a.T, a.H, DK) ||
      !map128(&mb, a.b, BF, 2, a.B, a.T, a.H, DK) || !map128(&mv, a.v, BF, 2, a.B, a.T, a.H, DV) ||
      !map128(&mw, a.w, BF, 2, a.B, a.T, a.H, DV) ||
      !map128(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.B, a.T, a.H, DK))
    return cudaErrorInvalidValue;
  Tc128Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.b = static_cast<const __nv_bfloat16*>(a.b);
  p.w = static_cast<const __nv_bfloat16*>(a.w);
  p.la = a.log_alpha;
  p.S0 = a.S0;
  p.o = a.o;
  p.S_T = a.S_T;
  p.T = a.T;
  p.H = a.H;
  p.err = device_error_word();
  p.stamps = stamp_buffer();
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = smem_limit_once(chunk_fwd_tc128_kernel<DK, DV>, (int)SMEM_BYTES, attr_done);
  if (e != cudaSuccess) return e;
  chunk_fwd_tc128_kernel<DK, DV><<<a.B * a.H, NT, SMEM_BYTES, st>>>(mq, mk, mb, mv, mw, mla, p);
  return cudaGetLastError();
}

}  // namespace

size_t chunk_fwd_tc128_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_chunk_fwd_tc128(const ChunkArgs& a, cudaStream_t st) {
  if (!a.bf16 || a.cu_seqlens) return cudaErrorInvalidValue;
  if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
  if (a.dk == 128 && a.dv == 128) return launch128<128, 128>(a, st);
  if (a.dk == 128 && a.dv == 64) return launch128<128, 64>(a, st);
  if (a.dk == 64 && a.dv == 128) return launch128<64, 128>(a, st);
  if (a.dk == 64 && a.dv == 64) return launch128<64, 64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace gdn2
