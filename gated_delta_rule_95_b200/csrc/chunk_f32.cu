// Chunkwise prefill forward for fp32 inputs, on CUDA cores in fp32.
//
// Same chunkwise WY algorithm as the tensor-core kernel (Gated DeltaNet-2 guide,
// "Chunkwise Parallel Algorithm for GPU Training"; decay folded into the WY
// factors as on snilld.dk, "Hvad betyder det for traening og inferens"), kept in
// full fp32 so that fp32 inputs get fp32 results.  Per chunk of C = 64 tokens
// with entering state S and g = in-chunk cumsum of log alpha, Gamma = exp(g):
//     Kb = K * B * Gamma,  Kn = K / Gamma,  Qh = Q * Gamma,  Vw = W * V
//     A  = strictly_lower(Kb Kn^T),   P = lower_incl(Qh Kn^T)
//     U~ = (I + A)^-1 (Vw - Kb S)                     (forward substitution)
//     O  = Qh S + P U~
//     S  = Diag(Gamma_C) (S + Kn^T U~)
// One CTA owns one (batch, head) and a slice of NV = 32 value columns; value
// columns never mix, so slices are independent.
#include <cuda_runtime.h>

#include "gdn2_internal.h"

namespace gdn2 {
namespace {

constexpr int C = 64;
constexpr int NV = 32;
constexpr int NT = 256;

template <int DK>
struct F32Smem {
  float Kb[C][DK], Kn[C][DK], Qh[C][DK];
  float A[C][C + 1], P[C][C + 1];
  float R[C][NV], U[C][NV];
  float S[DK][NV];
  float gC[DK];
};

template <int DK>
__global__ void __launch_bounds__(NT) chunk_fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                           const float* __restrict__ v,
                                                           const float* __restrict__ la,
                                                           const float* __restrict__ bg,
                                                           const float* __restrict__ wg,
                                                           const float* __restrict__ S0, float* __restrict__ o,
                                                           float* __restrict__ S_T, int T, int H, int dk, int dv) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  F32Smem<DK>& sm = *reinterpret_cast<F32Smem<DK>*>(smem_raw);
  const int nslice = dv / NV;
  const int unit = blockIdx.x / nslice, slice = blockIdx.x % nslice;
  const int bb = unit / H, h = unit % H, j0 = slice * NV;
  const int tid = threadIdx.x;

  // state slice S[:, j0 : j0 + NV]
  for (int idx = tid; idx < DK * NV; idx += NT) {
    const int i = idx / NV, jj = idx % NV;
    sm.S[i][jj] = (S0 && i < dk) ? S0[((size_t)unit * dk + i) * dv + j0 + jj] : 0.f;
  }

  const int nchunks = (T + C - 1) / C;
  for (int c = 0; c < nchunks; ++c) {
    const int t0 = c * C, n = min(C, T - t0);
    // --- decay cumsum and folded operands; one thread per key channel
    if (tid < DK) {
      const int i = tid;
      float g = 0.f;
      for (int t = 0; t < C; ++t) {
        float kb = 0.f, kn = 0.f, qh = 0.f;
        if (t < n && i < dk) {
          const size_t off = (((size_t)bb * T + t0 + t) * H + h) * dk + i;
          g += la[off];
          const float G = __expf(g), kk = k[off];
          kb = kk * bg[off] * G;
          kn = kk * __expf(-g);
          qh = q[off] * G;
        }
        sm.Kb[t][i] = kb;
        sm.Kn[t][i] = kn;
        sm.Qh[t][i] = qh;
      }
      sm.gC[i] = __expf(g);
    }
    for (int idx = tid; idx < C * NV; idx += NT) {
      const int t = idx / NV, jj = idx % NV;
      float x = 0.f;
      if (t < n) {
        const size_t off = (((size_t)bb * T + t0 + t) * H + h) * dv + j0 + jj;
        x = wg[off] * v[off];
      }
      sm.R[t][jj] = x;
    }
    __syncthreads();
    // --- A, P (C x C) and R = Vw - Kb S
    for (int idx = tid; idx < C * C; idx += NT) {
      const int t = idx / C, s = idx % C;
      float a = 0.f, p = 0.f;
      if (s <= t) {
        for (int i = 0; i < DK; ++i) {
          a = fmaf(sm.Kb[t][i], sm.Kn[s][i], a);
          p = fmaf(sm.Qh[t][i], sm.Kn[s][i], p);
        }
      }
      sm.A[t][s] = (s < t) ? a : 0.f;
      sm.P[t][s] = p;
    }
    for (int idx = tid; idx < C * NV; idx += NT) {
      const int t = idx / NV, jj = idx % NV;
      float acc = sm.R[t][jj];
      for (int i = 0; i < DK; ++i) acc = fmaf(-sm.Kb[t][i], sm.S[i][jj], acc);
      sm.R[t][jj] = acc;
    }
    __syncthreads();
    // --- U~ = (I + A)^-1 R by forward substitution, one thread per value column
    if (tid < NV) {
      const int jj = tid;
      for (int t = 0; t < C; ++t) {
        float acc = sm.R[t][jj];
        for (int s = 0; s < t; ++s) acc = fmaf(-sm.A[t][s], sm.U[s][jj], acc);
        sm.U[t][jj] = acc;
      }
    }
    __syncthreads();
    // --- O = Qh S + P U~
    for (int idx = tid; idx < C * NV; idx += NT) {
      const int t = idx / NV, jj = idx % NV;
      if (t < n) {
        float acc = 0.f;
        for (int i = 0; i < DK; ++i) acc = fmaf(sm.Qh[t][i], sm.S[i][jj], acc);
        for (int s = 0; s <= t; ++s) acc = fmaf(sm.P[t][s], sm.U[s][jj], acc);
        o[(((size_t)bb * T + t0 + t) * H + h) * dv + j0 + jj] = acc;
      }
    }
    __syncthreads();
    // --- S = Diag(Gamma_C) (S + Kn^T U~)
    for (int idx = tid; idx < DK * NV; idx += NT) {
      const int i = idx / NV, jj = idx % NV;
      float acc = sm.S[i][jj];
      for (int s = 0; s < C; ++s) acc = fmaf(sm.Kn[s][i], sm.U[s][jj], acc);
      sm.S[i][jj] = sm.gC[i] * acc;
    }
    __syncthreads();
  }
  if (S_T) {
    for (int idx = tid; idx < DK * NV; idx += NT) {
      const int i = idx / NV, jj = idx % NV;
      if (i < dk) S_T[((size_t)unit * dk + i) * dv + j0 + jj] = sm.S[i][jj];
    }
  }
}

template <int DK>
cudaError_t launch_dk(const ChunkArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(F32Smem<DK>);
  cudaError_t e = cudaFuncSetAttribute(chunk_fwd_f32_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.B * a.H * (a.dv / NV);
  chunk_fwd_f32_kernel<DK><<<grid, NT, smem, st>>>(
      static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.v),
      a.log_alpha, static_cast<const float*>(a.b), static_cast<const float*>(a.w), a.S0,
      a.o, a.S_T, a.T, a.H, a.dk, a.dv);
  return cudaGetLastError();
}

// S_T = S0 (or zeros) for an empty sequence.
__global__ void state_copy_kernel(const float* __restrict__ S0, float* __restrict__ S_T, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    S_T[i] = S0 ? S0[i] : 0.f;
}

}  // namespace

cudaError_t launch_chunk_fwd_f32(const ChunkArgs& a, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  return a.dk == 128 ? launch_dk<128>(a, st) : launch_dk<64>(a, st);
}

cudaError_t launch_state_copy(const ChunkArgs& a, cudaStream_t st) {
  const size_t n = (size_t)a.B * a.H * a.dk * a.dv;
  if (n == 0 || a.S_T == nullptr || a.S_T == a.S0) return cudaSuccess;
  state_copy_kernel<<<296, 256, 0, st>>>(a.S0, a.S_T, n);
  return cudaGetLastError();
}

}  // namespace gdn2
