// Internal interface between the C ABI (api.cu) and the kernel launchers.
#pragma once
#include <cuda_runtime.h>

#include <atomic>

namespace gdn2 {

struct DecodeArgs {
  const void *q, *k, *v, *b, *w;
  const float* log_alpha;
  float* S;
  float* o;
  int B, H, dk, dv;
  bool bf16;
  // raw projections: q, k un-normalised, b, w gate logits, log_alpha holds the decay
  // pre-activation a (log alpha = -s_h softplus(a)); decay_scale: s_h per head (NULL = 1)
  bool raw = false;
  const float* decay_scale = nullptr;
};

struct ChunkArgs {
  const void *q, *k, *v, *b, *w;
  const float* log_alpha;
  const float* S0;
  float* o;
  float* S_T;
  int B, T, H, dk, dv;  // packed sequences: B = number of sequences, T = total tokens
  bool bf16;
  const int* cu_seqlens;  // packed sequences: [B + 1] device token offsets; NULL otherwise
  // raw projections: q, k un-normalised, b, w gate logits, log_alpha holds the decay
  // pre-activation a (log alpha = -s_h softplus(a)); decay_scale: s_h per head (NULL = 1)
  bool raw = false;
  const float* decay_scale = nullptr;
  // sequence split: segments per sequence (<= 1: off) and the caller's workspace
  // [3][B H][split][d_k d_v] fp32
  int split = 0;
  float* workspace = nullptr;
};

// Device error word of this library: bits set by kernels, read and cleared by
// gdn2_device_status().
enum : unsigned {
  kErrWaitTimeout = 1u,  // a bounded wait gave up
  kErrBadSeqlens = 2u,   // packed-sequence offsets out of order or out of range
  kErrDecayRange = 4u    // an in-chunk cumulative log decay fell below -80
};
unsigned* device_error_word();
// Instrumented builds (GDN2_STAMPS): the device buffer of per-chunk clock stamps of the
// chunk kernel on the current device; NULL in the product build.
unsigned long long* stamp_buffer();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// device (the attribute belongs to each device's context): `done` holds one bit per device
// index below 64 (higher indices set the attribute on every call).  Safe from several host
// threads: a race sets the same value twice.
template <class K>
cudaError_t smem_limit_once(K* kernel, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Backward of the chunkwise forward (gradients fp32; dq, dk, db are zeroed and accumulated).
struct ChunkBwdArgs {
  const void *q, *k, *v, *b, *w;
  const float* log_alpha;
  const float* S0;
  const float* dO;
  const float* dS_T;
  float *dq, *dk, *dv, *dlog_alpha, *db, *dw, *dS0;
  float* workspace;  // chunk_bwd_workspace_bytes
  int B, T, H, dk_, dv_;
  bool bf16;
};
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_chunk_bwd(const ChunkBwdArgs& a, cudaStream_t st);
// bf16, d_k = d_v = 128: the tensor-core backward (checkpoint pass, dS sweep, per-chunk pass)
size_t chunk_bwd_tc_workspace_bytes(int B, int T, int H);
cudaError_t launch_chunk_bwd_tc(const ChunkBwdArgs& a, cudaStream_t st);

// Short causal (4 taps) over [B, T, C] (or packed [T, C] with cu_seqlens).
struct ShortConvArgs {
  const void* x;
  const float* weight;    // [C, 4]
  const float* bias;      // [C] or NULL
  const int* cu_seqlens;  // packed: [B + 1] device offsets; NULL: B sequences of T tokens
  const void* hist_in;    // [B, 3, C] or NULL (zeros)
  void* y;
  void* hist_out;         // [B, 3, C] or NULL; may alias hist_in
  int B, T, C;
  bool bf16;
};
cudaError_t launch_short_conv(const ShortConvArgs& a, cudaStream_t st);

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t st);
// bf16 inputs: tcgen05/TMEM kernel fed by TMA.
cudaError_t launch_chunk_fwd_tc(const ChunkArgs& a, cudaStream_t st);
// bf16, d_k = d_v: the state entering every chunk, [B H][chunk][d_k][d_v] fp32 (no outputs);
// with ck_u, ck_tt, ck_pt also U~ [B H][chunk][64][d_v], T^T and P^T [B H][chunk][64][64] of
// every chunk (the tensor-core backward's inputs).
cudaError_t launch_chunk_states_tc(const ChunkArgs& a, float* states, cudaStream_t st, float* ck_u = nullptr,
                                   float* ck_tt = nullptr, float* ck_pt = nullptr);
// fp32 inputs, d_k = d_v = 64: tcgen05 kernel with split (3 x tf32) products.
bool chunk_fwd_f32_tc_supported(const ChunkArgs& a);
cudaError_t launch_chunk_fwd_f32_tc(const ChunkArgs& a, cudaStream_t st);
// fp32 inputs of the other head sizes: fp32 CUDA-core kernel of the same chunkwise algorithm.
cudaError_t launch_chunk_fwd_f32(const ChunkArgs& a, cudaStream_t st);
// bf16, chunk size 32 (tcgen05 kernel for 32-token chunks), 64 (the production tcgen05
// kernel) or 128 (tcgen05 kernel with the phases of a chunk in sequence); shared memory per
// CTA, 0 for an unsupported (chunk, d_k).
size_t chunk_fwd_tc_smem_bytes();
size_t chunk_fwd_tc32_smem_bytes();
cudaError_t launch_chunk_fwd_tc32(const ChunkArgs& a, cudaStream_t st);
size_t chunk_fwd_tc128_smem_bytes();
cudaError_t launch_chunk_fwd_tc128(const ChunkArgs& a, cudaStream_t st);
size_t chunk_fwd_csize_smem_bytes(int chunk, int dk);
cudaError_t launch_chunk_fwd_csize(const ChunkArgs& a, int chunk, cudaStream_t st);
// T = 0: S_T = S0 (or zeros).
cudaError_t launch_state_copy(const ChunkArgs& a, cudaStream_t st);

}  // namespace gdn2
