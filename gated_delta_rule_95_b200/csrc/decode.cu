// Recurrent decode step of the Gated Delta Rule-2 (one token per sequence and
// head), bandwidth-bound: each (sequence, head) state of d_k x d_v fp32 is read
// once and written once.
//
// Expanding the update (snilld.dk, compact update) for one token, with
// x = alpha * b * k and y = alpha * q:
//     e      = S^T x                      (what the erase removes, per value column)
//     delta  = w * v - e
//     S'     = Diag(alpha) S + k delta^T
//     o      = S'^T q = S^T y + (q . k) delta
// so one pass over S (two key-axis reductions per value column) gives o, and a
// second pass over the registers that already hold S writes S'.
//
// Raw projections (PREP): b = sigmoid(b), w = sigmoid(w) and log alpha = -s_h softplus(a)
// (Gated DeltaNet-2 guide, "Normalization and Short Convolutions" and "Decoupled Erase and
// Write Gates") in fp32 while the state loads are in flight, on the fast exp / log / divide
// intrinsics (softplus(a) = max(a, 0) + log(1 + e^-|a|) never overflows, and its absolute
// error of about 1e-7 in log alpha is far inside the fp32 bar); q and k are L2-normalised by
// carrying 1/|q| and 1/|k| as factors (reduced with q . k) into e, S^T y, q . k and the
// rank-one write, which are linear in them.
//
// Work split: one CTA of 256 threads per (sequence, head).  Warp r owns rows
// [r*DK/8, (r+1)*DK/8); lane c owns value columns [c*DV/32, (c+1)*DV/32), so
// every warp-wide load or store of S covers whole contiguous rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "gdn2_internal.h"

namespace gdn2 {
namespace {

template <typename T>
__device__ __forceinline__ float ld_tok(const T* p);
template <>
__device__ __forceinline__ float ld_tok<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_tok<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

template <typename T, int DK, int DV, bool PREP>
__global__ void __launch_bounds__(256) decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v,
                                                          const float* __restrict__ log_alpha,
                                                          const T* __restrict__ bg, const T* __restrict__ wg,
                                                          float* __restrict__ S, float* __restrict__ o, int H,
                                                          const float* __restrict__ dscale) {
  constexpr int ROWS = DK / 8;   // rows per warp
  constexpr int CPL = DV / 32;   // columns per lane (2 or 4)
  using vec_t = typename std::conditional<CPL == 4, float4, float2>::type;

  __shared__ float s_alpha[DK], s_k[DK], s_x[DK], s_y[DK];
  __shared__ float s_wv[DV], s_delta[DV];
  __shared__ float s_red[2][8][DV];
  __shared__ float s_qk, s_rq, s_rk;

  const int unit = blockIdx.x;               // b * H + h
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t tk = (size_t)unit * DK, tv = (size_t)unit * DV;

  // Issue the state loads first: they are the HBM traffic that matters.
  float* Su = S + (size_t)unit * DK * DV;
  float s[ROWS][CPL];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const vec_t x = __ldcs(reinterpret_cast<const vec_t*>(Su + (size_t)(warp * ROWS + r) * DV) + lane);
    const float* xf = reinterpret_cast<const float*>(&x);
#pragma unroll
    for (int c = 0; c < CPL; ++c) s[r][c] = xf[c];
  }

  if (tid < DK) {
    float la = __ldg(log_alpha + tk + tid);
    if constexpr (PREP) {  // log alpha = -s_h softplus(a)
      const float sh = dscale ? __ldg(dscale + unit % H) : 1.f;
      la = -sh * (fmaxf(la, 0.f) + __logf(1.f + __expf(-fabsf(la))));
    }
    const float a = __expf(la);
    const float kk = ld_tok(k + tk + tid), qq = ld_tok(q + tk + tid);
    float bb = ld_tok(bg + tk + tid);
    if constexpr (PREP) {
      bb = sigmoid_f(bb);
      // |q|^2 and |k|^2, reduced like q . k (slots 1 and 2 of the reduction buffer)
      float pq = qq * qq, pk = kk * kk;
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        pq += __shfl_xor_sync(0xffffffffu, pq, off);
        pk += __shfl_xor_sync(0xffffffffu, pk, off);
      }
      if (lane == 0) {
        s_red[0][warp][1] = pq;
        s_red[0][warp][2] = pk;
      }
    }
    s_alpha[tid] = a;
    s_k[tid] = kk;
    s_x[tid] = a * bb * kk;
    s_y[tid] = a * qq;
    // q . k, reduced inside the warps that hold the key channels
    float p = qq * kk;
#pragma unroll
    for (int off = 16; off; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
    if (lane == 0) s_red[0][warp][0] = p;  // reuse of the reduction buffer before it is needed
  }
  if (tid < DV) {
    float ww = ld_tok(wg + tv + tid);
    if constexpr (PREP) ww = sigmoid_f(ww);
    s_wv[tid] = ww * ld_tok(v + tv + tid);
  }
  __syncthreads();
  if (tid == 0) {
    float p = 0.f;
#pragma unroll
    for (int w = 0; w < DK / 32; ++w) p += s_red[0][w][0];
    if constexpr (PREP) {
      float nq = 0.f, nk = 0.f;
#pragma unroll
      for (int w = 0; w < DK / 32; ++w) {
        nq += s_red[0][w][1];
        nk += s_red[0][w][2];
      }
      const float rq = rsqrtf(fmaxf(nq, 1e-24f)), rk = rsqrtf(fmaxf(nk, 1e-24f));  // zero stays zero
      s_rq = rq;
      s_rk = rk;
      p *= rq * rk;
    }
    s_qk = p;
  }

  // Partial key-axis reductions over this warp's rows.
  float e[CPL], r_[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) e[c] = r_[c] = 0.f;
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int i = warp * ROWS + r;
    const float xi = s_x[i], yi = s_y[i];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      e[c] = fmaf(xi, s[r][c], e[c]);
      r_[c] = fmaf(yi, s[r][c], r_[c]);
    }
  }
  __syncthreads();  // s_qk read below; s_red[0] slot reused
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    s_red[0][warp][lane * CPL + c] = e[c];
    s_red[1][warp][lane * CPL + c] = r_[c];
  }
  __syncthreads();
  if (tid < DV) {
    float ee = 0.f, rr = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      ee += s_red[0][w][tid];
      rr += s_red[1][w][tid];
    }
    if constexpr (PREP) {
      ee *= s_rk;
      rr *= s_rq;
    }
    const float d = s_wv[tid] - ee;
    s_delta[tid] = PREP ? d * s_rk : d;  // (the write k delta^T with the raw k)
    o[tv + tid] = fmaf(s_qk, d, rr);
  }
  __syncthreads();

  float dl[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) dl[c] = s_delta[lane * CPL + c];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int i = warp * ROWS + r;
    const float a = s_alpha[i], kk = s_k[i];
    vec_t x;
    float* xf = reinterpret_cast<float*>(&x);
#pragma unroll
    for (int c = 0; c < CPL; ++c) xf[c] = fmaf(a, s[r][c], kk * dl[c]);
    __stcs(reinterpret_cast<vec_t*>(Su + (size_t)i * DV) + lane, x);
  }
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  const T *q = static_cast<const T*>(a.q), *k = static_cast<const T*>(a.k), *v = static_cast<const T*>(a.v);
  const T *b = static_cast<const T*>(a.b), *w = static_cast<const T*>(a.w);
  if (a.raw)
    decode_step_kernel<T, DK, DV, true><<<a.B * a.H, 256, 0, st>>>(q, k, v, a.log_alpha, b, w, a.S, a.o, a.H,
                                                                   a.decay_scale);
  else
    decode_step_kernel<T, DK, DV, false><<<a.B * a.H, 256, 0, st>>>(q, k, v, a.log_alpha, b, w, a.S, a.o, a.H,
                                                                    nullptr);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dims(const DecodeArgs& a, cudaStream_t st) {
  if (a.dk == 128 && a.dv == 128) return launch_t<T, 128, 128>(a, st);
  if (a.dk == 128 && a.dv == 64) return launch_t<T, 128, 64>(a, st);
  if (a.dk == 64 && a.dv == 128) return launch_t<T, 64, 128>(a, st);
  return launch_t<T, 64, 64>(a, st);
}

}  // namespace

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  return a.bf16 ? launch_dims<__nv_bfloat16>(a, st) : launch_dims<float>(a, st);
}

}  // namespace gdn2
