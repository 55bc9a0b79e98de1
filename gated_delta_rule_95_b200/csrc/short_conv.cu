// Short causal depthwise convolution (kernel size 4) over the token axis, applied to
// q, k and v before the recurrence (Gated DeltaNet-2 guide, "Normalization and Short
// Convolutions"; the guide's layer convolves each channel with 4 taps, padded on the
// left so that token t sees tokens t-3 .. t, with a bias):
//
//     y[t, c] = bias[c] + sum_{j=0..3} weight[c, j] * x[t - 3 + j, c]
//
// where the tokens before a sequence's first come from its carried history (the last
// three inputs of the previous call) or are zero.  Bandwidth-bound: every input element is
// read once and every output written once.
//
// Work split: a block of 256 threads takes a strip of tokens by a block of 1024 channels.
// One thread copies the strip's rows (and the three rows before it) into shared memory
// with 1-D bulk copies on one mbarrier, so that a block keeps its whole tile (70 KB for
// bf16) in flight without holding it in registers and three blocks share an SM; then
// thread t walks the strip for the four channels [4 t, 4 t + 4) of the block with a
// three-token window in registers and stores y directly (a warp writes 256 contiguous
// bytes of bf16 per token).  A strip may cross sequence boundaries (packed batches): the
// window is reloaded from the history at each sequence start.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gdn2_internal.h"
#include "ptx.cuh"

namespace gdn2 {
namespace {

constexpr int CONV_THREADS = 256;
// tokens per strip: 32 of bf16 or 16 of fp32 (a tile of at most 35 or 19 rows of 2 or 4 KB)
template <typename T>
__host__ __device__ constexpr int strip_of() { return 64 / (int)sizeof(T); }
template <typename T>
__host__ __device__ constexpr uint32_t conv_smem_bytes() {
  return (uint32_t)(strip_of<T>() + 3) * CONV_THREADS * 4 * (uint32_t)sizeof(T) + 16;
}
constexpr uint64_t CONV_WAIT_LIMIT = 2000000000ull;  // 2 s

// Four adjacent channels of one token: 8 bytes of bf16 or 16 bytes of fp32.
template <typename T>
struct Quad;
template <>
struct Quad<float> {
  using V = float4;
  static __device__ __forceinline__ float4 load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
  static __device__ __forceinline__ void store(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
  static __device__ __forceinline__ float4 f(float4 v) { return v; }
  static __device__ __forceinline__ float4 from(float4 v) { return v; }
  static __device__ __forceinline__ float4 zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};
template <>
struct Quad<__nv_bfloat16> {
  using V = uint2;
  static __device__ __forceinline__ uint2 load(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, uint2 v) { __stcs(reinterpret_cast<uint2*>(p), v); }
  static __device__ __forceinline__ float4 f(uint2 v) {
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xFFFF0000u));
  }
  static __device__ __forceinline__ uint2 from(float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
  static __device__ __forceinline__ uint2 zero() { return make_uint2(0u, 0u); }
};

// Sequence of flat token g: fixed length T per sequence, or the packed offsets cu[0..nseq].
__device__ __forceinline__ int seq_of(int g, const int* cu, int nseq, int T) {
  if (!cu) return g / T;
  int lo = 0, hi = nseq;  // cu[lo] <= g < cu[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

// Packed offsets are checked where they are used: a strip whose sequence lookup is not
// consistent (offsets out of order or out of range) sets kErrBadSeqlens and writes nothing.
// Block b covers channel block b mod ncb of strip b / ncb, so that consecutive blocks read
// consecutive parts of the same token rows.
template <typename T>
__global__ void __launch_bounds__(CONV_THREADS) short_conv_kernel(const T* __restrict__ x, const float* __restrict__ w,
                                                                const float* __restrict__ bias, const int* cu,
                                                                int nseq, const T* hist, T* __restrict__ y,
                                                                int ntok, int T_seq, int C, int ncb, unsigned* err) {
  using Q = Quad<T>;
  constexpr int STRIP = strip_of<T>();
  const int cb = blockIdx.x % ncb, strip = blockIdx.x / ncb;
  const int c = 4 * (cb * CONV_THREADS + threadIdx.x);  // may be >= C in the last channel block
  const int g0 = strip * STRIP;
  if (cu) {
    const int n0 = seq_of(g0, cu, nseq, T_seq);
    const bool bad = cu[0] != 0 || cu[nseq] != ntok || cu[n0] < 0 || cu[n0] > g0 || cu[n0 + 1] <= g0;
    if (bad) {
      if (threadIdx.x == 0 && err) atomicOr(err, kErrBadSeqlens);
      return;
    }
  }
  const int g1 = min(g0 + STRIP, ntok);
  // the tile: rows r0 .. g1 - 1 (the strip and up to three rows before it) of this block's
  // channels [c0, c0 + width), row i at tile + i * width
  extern __shared__ __align__(16) unsigned char conv_smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(conv_smem);
  T* tile = reinterpret_cast<T*>(conv_smem + 16);
  const int c0 = cb * CONV_THREADS * 4;
  const int width = min(CONV_THREADS * 4, C - c0);
  const int r0 = max(g0 - 3, 0);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t row_bytes = (uint32_t)width * sizeof(T);
    mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)(g1 - r0));
    for (int r = r0; r < g1; ++r)
      bulk_load_1d(tile + (size_t)(r - r0) * width, x + (size_t)r * C + c0, row_bytes, bar);
  }
  // taps of the four channels: wt[j] = (w[c][j], w[c+1][j], w[c+2][j], w[c+3][j])
  const bool active = c < C;
  float4 wt[4];
  float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
    const float4 r0w = __ldg(reinterpret_cast<const float4*>(w + 4 * (size_t)c));
    const float4 r1w = __ldg(reinterpret_cast<const float4*>(w + 4 * (size_t)c + 4));
    const float4 r2w = __ldg(reinterpret_cast<const float4*>(w + 4 * (size_t)c + 8));
    const float4 r3w = __ldg(reinterpret_cast<const float4*>(w + 4 * (size_t)c + 12));
    wt[0] = make_float4(r0w.x, r1w.x, r2w.x, r3w.x);
    wt[1] = make_float4(r0w.y, r1w.y, r2w.y, r3w.y);
    wt[2] = make_float4(r0w.z, r1w.z, r2w.z, r3w.z);
    wt[3] = make_float4(r0w.w, r1w.w, r2w.w, r3w.w);
    if (bias) b0 = __ldg(reinterpret_cast<const float4*>(bias + c));
  }
  volatile int never = 0;
  if (!mbar_wait_bounded(bar, 0, &never, err, CONV_WAIT_LIMIT)) {
    // the copies must land before the block's shared memory is released
    mbar_wait_bounded(bar, 0, &never, nullptr, CONV_WAIT_LIMIT);
    return;
  }
  if (!active) return;
  const T* tc = tile + 4 * threadIdx.x;  // this thread's channels in row 0 of the tile
  auto row = [&](int g) { return Q::f(*reinterpret_cast<const typename Q::V*>(tc + (size_t)(g - r0) * width)); };

  int n = seq_of(g0, cu, nseq, T_seq);
  int start = cu ? cu[n] : n * T_seq;
  int next = cu ? cu[n + 1] : start + T_seq;  // first token of the next sequence
  // window h[j] = input at token g - 3 + j (j = 0, 1, 2) for the strip's first token
  float4 h[3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int gj = g0 - 3 + j;  // >= start - 3
    if (gj >= start) {  // (start >= 0, so gj >= r0)
      h[j] = row(gj);
    } else if (hist) {  // history slot 3 - (start - gj) of sequence n, oldest first
      h[j] = Q::f(Q::load(hist + ((size_t)n * 3 + 3 - (start - gj)) * C + c));
    } else {
      h[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int i = 0; i < STRIP; ++i) {
    const int g = g0 + i;
    if (g >= g1) break;
    if (g >= next) {  // a new sequence starts here (skipping empty ones): its own history
      while (g >= next && n + 1 < nseq) {  // (g < cu[nseq] stops it first for valid offsets)
        ++n;
        start = next;
        next = cu ? cu[n + 1] : start + T_seq;
      }
      if (g < start || g >= next) return;  // offsets out of order: nothing more is written
#pragma unroll
      for (int j = 0; j < 3; ++j)  // g == start: slot j of the new sequence's history
        h[j] = hist ? Q::f(Q::load(hist + ((size_t)n * 3 + j) * C + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float4 xi = row(g);
    float4 o;
    o.x = fmaf(wt[0].x, h[0].x, fmaf(wt[1].x, h[1].x, fmaf(wt[2].x, h[2].x, fmaf(wt[3].x, xi.x, b0.x))));
    o.y = fmaf(wt[0].y, h[0].y, fmaf(wt[1].y, h[1].y, fmaf(wt[2].y, h[2].y, fmaf(wt[3].y, xi.y, b0.y))));
    o.z = fmaf(wt[0].z, h[0].z, fmaf(wt[1].z, h[1].z, fmaf(wt[2].z, h[2].z, fmaf(wt[3].z, xi.z, b0.z))));
    o.w = fmaf(wt[0].w, h[0].w, fmaf(wt[1].w, h[1].w, fmaf(wt[2].w, h[2].w, fmaf(wt[3].w, xi.w, b0.w))));
    Q::store(y + (size_t)g * C + c, Q::from(o));
    h[0] = h[1];
    h[1] = h[2];
    h[2] = xi;
  }
}

// The history after the call: the last three inputs of each sequence, counting the carried
// history before it (a sequence shorter than three tokens keeps part of its old history).
// One thread per (sequence, channel pair) reads its three values before writing, so the
// history may be updated in place.
template <typename T>
__global__ void short_conv_history_kernel(const T* __restrict__ x, const int* cu, const T* hist_in, T* hist_out,
                                          int nseq, int ntok, int T_seq, int C, unsigned* err) {
  using Q = Quad<T>;
  const int c = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  const int n = blockIdx.y;
  if (c >= C || n >= nseq) return;
  const int start = cu ? cu[n] : n * T_seq;
  const int len = cu ? cu[n + 1] - start : T_seq;
  if (start < 0 || len < 0 || start + len > ntok) {  // offsets out of order or out of range
    if (c == 0 && err) atomicOr(err, kErrBadSeqlens);
    return;
  }
  typename Q::V v[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int e = len + i;  // position in [history (3) | the sequence's tokens]
    if (e >= 3) {
      v[i] = Q::load(x + (size_t)(start + e - 3) * C + c);
    } else if (hist_in) {
      v[i] = *reinterpret_cast<const typename Q::V*>(hist_in + ((size_t)n * 3 + e) * C + c);
    } else {
      v[i] = Q::zero();
    }
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) *reinterpret_cast<typename Q::V*>(hist_out + ((size_t)n * 3 + i) * C + c) = v[i];
}

template <typename T>
cudaError_t launch_typed(const ShortConvArgs& a, cudaStream_t st) {
  const T* x = static_cast<const T*>(a.x);
  const T* hin = static_cast<const T*>(a.hist_in);
  T* y = static_cast<T*>(a.y);
  T* hout = static_cast<T*>(a.hist_out);
  const int nseq = a.B;
  const int ntok = a.cu_seqlens ? a.T : a.B * a.T;
  const int quads = a.C / 4;
  if (ntok > 0) {
    const int ncb = (quads + CONV_THREADS - 1) / CONV_THREADS;
    constexpr int STRIP = strip_of<T>();
    const long long blocks = (long long)((ntok + STRIP - 1) / STRIP) * ncb;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    static std::atomic<unsigned long long> attr_done{0};  // per element type, a bit per device
    cudaError_t e = smem_limit_once(short_conv_kernel<T>, (int)conv_smem_bytes<T>(), attr_done);
    if (e != cudaSuccess) return e;
    short_conv_kernel<T><<<(unsigned)blocks, CONV_THREADS, conv_smem_bytes<T>(), st>>>(x, a.weight, a.bias, a.cu_seqlens, nseq, hin, y,
                                                                     ntok, a.T, a.C, ncb, device_error_word());
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (hout) {
    dim3 grid((quads + 127) / 128, nseq);
    short_conv_history_kernel<T><<<grid, 128, 0, st>>>(x, a.cu_seqlens, hin, hout, nseq, ntok, a.T, a.C,
                                                        device_error_word());
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_short_conv(const ShortConvArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.C == 0) return cudaSuccess;
  return a.bf16 ? launch_typed<__nv_bfloat16>(a, st) : launch_typed<float>(a, st);
}

}  // namespace gdn2
