// C ABI of the Gated DeltaNet-2 token mixer: argument checks, dispatch, status.
// Every entry point validates before touching CUDA, so argument errors come
// back synchronously and without a device.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gdn2.h"
#include "gdn2_internal.h"

namespace gdn2 {

__device__ unsigned g_error_word = 0;

// Address of the error word on the current device (looked up once per device; several host
// threads may ask at once, so the cache is filled under a lock).
unsigned* device_error_word() {
  constexpr int kMaxDev = 64;
  static unsigned* ptrs[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess) ptrs[dev] = static_cast<unsigned*>(p);
  }
  return ptrs[dev];
}

#ifdef GDN2_STAMPS
// Instrumented build only: per-chunk clock stamps of the chunk kernel's first CTA.
constexpr int kStampWords = 64 * 32;
__device__ unsigned long long g_stamps[kStampWords];
unsigned long long* stamp_buffer() {
  constexpr int kMaxDev = 64;
  static unsigned long long* ptrs[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_stamps) == cudaSuccess) ptrs[dev] = static_cast<unsigned long long*>(p);
  }
  return ptrs[dev];
}
#else
unsigned long long* stamp_buffer() { return nullptr; }
#endif

namespace {

thread_local char g_last_cuda[256] = "";

gdn2_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda, sizeof(g_last_cuda), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return GDN2_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Largest element count of any tensor must fit comfortably in 63 bits and in
// the 32-bit grid/tensor-map limits used by the kernels.
bool sizes_ok(long long B, long long T, long long H, long long dk, long long dv) {
  if (B < 0 || T < 0 || H < 0) return false;
  if (!head_dim_ok((int)dk) || !head_dim_ok((int)dv)) return false;
  if (B * H > 0x7fffffffLL) return false;
  if (T > (1LL << 31) - 64) return false;
  const long long tok = B * T * H;
  return tok <= (1LL << 46) / 128;
}

}  // namespace
}  // namespace gdn2

using namespace gdn2;

extern "C" gdn2_status gdn2_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                                      const void* b, const void* w, const float* S0, float* o, float* S_T, int B,
                                      int T, int H, int d_k, int d_v, gdn2_dtype dt, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (!sizes_ok(B, T, H, d_k, d_v)) return GDN2_ERR_SHAPE;
  const bool tokens = (long long)B * T * H > 0;
  if (tokens && (!q || !k || !v || !log_alpha || !b || !w || !o)) return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S0, o, S_T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if ((long long)B * H == 0) return GDN2_OK;

  ChunkArgs a{q, k, v, b, w, log_alpha, S0, o, S_T, B, T, H, d_k, d_v, dt == GDN2_BF16};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (T == 0)
    e = launch_state_copy(a, st);
  else
    e = a.bf16 ? launch_chunk_fwd_tc(a, st)
               : (chunk_fwd_f32_tc_supported(a) ? launch_chunk_fwd_f32_tc(a, st) : launch_chunk_fwd_f32(a, st));
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" int gdn2_chunk_fwd_split_segments(int B, int T, int H, int sm_count) {
  // waves of one CTA per SM: the first pass runs (2P - 3) B H segment runs, the last
  // (P - 1) B H, each of ceil(chunks / P) chunks; one pass of B H full runs without a split
  if (B <= 0 || T <= 0 || H <= 0 || sm_count <= 0) return 1;
  const long long bh = (long long)B * H, nch = (T + 63) / 64, sms = sm_count;
  auto waves = [&](long long units) { return (units + sms - 1) / sms; };
  long long best = waves(bh) * nch;
  int best_p = 1;
  for (int P = 2; P <= 64 && P <= nch; ++P) {
    const long long len = (nch + P - 1) / P;
    const long long est = (waves(bh * (2 * P - 3)) + waves(bh * (P - 1))) * len + 1;  // + the chaining
    if (est < best) {
      best = est;
      best_p = P;
    }
  }
  return best_p;
}

extern "C" size_t gdn2_chunk_fwd_split_workspace_bytes(int B, int H, int d_k, int d_v, int segments) {
  if (B <= 0 || H <= 0 || segments <= 1 || !head_dim_ok(d_k) || !head_dim_ok(d_v)) return 0;
  return (size_t)3 * B * H * segments * d_k * d_v * sizeof(float);
}

extern "C" gdn2_status gdn2_chunk_fwd_split(const void* q, const void* k, const void* v, const float* log_alpha,
                                            const void* b, const void* w, const float* S0, float* o, float* S_T,
                                            int B, int T, int H, int d_k, int d_v, gdn2_dtype dt, int segments,
                                            void* workspace, size_t workspace_bytes, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (dt != GDN2_BF16) return GDN2_ERR_DTYPE;  // the tensor-core path only
  if (!sizes_ok(B, T, H, d_k, d_v) || d_k != d_v || segments < 1 || segments > 4096) return GDN2_ERR_SHAPE;
  const bool tokens = (long long)B * T * H > 0;
  if (tokens && (!q || !k || !v || !log_alpha || !b || !w || !o)) return GDN2_ERR_NULL;
  if (segments > 1 && !workspace) return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S0, o, S_T, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if (segments > 1 && workspace_bytes < gdn2_chunk_fwd_split_workspace_bytes(B, H, d_k, d_v, segments))
    return GDN2_ERR_SHAPE;
  if ((long long)B * H == 0) return GDN2_OK;

  ChunkArgs a{q, k, v, b, w, log_alpha, S0, o, S_T, B, T, H, d_k, d_v, true};
  a.split = segments;
  a.workspace = static_cast<float*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = (T == 0) ? launch_state_copy(a, st) : launch_chunk_fwd_tc(a, st);
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

namespace gdn2 {
namespace {
// Scratch of gdn2_chunk_fwd_split_static: a fixed array in the module's device memory,
// so that the call allocates nothing.  Its address is looked up once per device.
constexpr size_t kSplitScratchBytes = size_t(16) << 20;  // 16 MiB
__device__ __align__(256) float g_split_scratch[kSplitScratchBytes / sizeof(float)];

cudaError_t split_scratch_address(float** out) {
  constexpr int kMaxDev = 64;
  static float* ptrs[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_split_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev] = static_cast<float*>(p);
  }
  *out = ptrs[dev];
  return cudaSuccess;
}
}  // namespace
}  // namespace gdn2

extern "C" gdn2_status gdn2_chunk_fwd_split_static(const void* q, const void* k, const void* v,
                                                   const float* log_alpha, const void* b, const void* w,
                                                   const float* S0, float* o, float* S_T, int B, int T, int H,
                                                   int d_k, int d_v, gdn2_dtype dt, int segments, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (!sizes_ok(B, T, H, d_k, d_v) || d_k != d_v || segments < 1 || segments > 4096) return GDN2_ERR_SHAPE;
  const size_t need = gdn2_chunk_fwd_split_workspace_bytes(B, H, d_k, d_v, segments);
  if (need > kSplitScratchBytes) return GDN2_ERR_SHAPE;  // beyond the fixed scratch
  const bool tokens = (long long)B * T * H > 0;
  if (tokens && (!q || !k || !v || !log_alpha || !b || !w || !o)) return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S0, o, S_T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if ((long long)B * H == 0) return GDN2_OK;
  float* scratch = nullptr;
  if (need > 0) {
    cudaError_t e = split_scratch_address(&scratch);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return gdn2_chunk_fwd_split(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, d_k, d_v, dt, segments, scratch,
                              kSplitScratchBytes, stream);
}

extern "C" size_t gdn2_chunk_fwd_csize_smem_bytes(int chunk, int d_k) {
  return chunk_fwd_csize_smem_bytes(chunk, d_k);
}

extern "C" gdn2_status gdn2_chunk_fwd_csize(const void* q, const void* k, const void* v, const float* log_alpha,
                                            const void* b, const void* w, const float* S0, float* o, float* S_T,
                                            int B, int T, int H, int d_k, int d_v, gdn2_dtype dt, int chunk,
                                            void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (dt != GDN2_BF16) return GDN2_ERR_DTYPE;  // the tensor-core path only
  if (!sizes_ok(B, T, H, d_k, d_v) || chunk_fwd_csize_smem_bytes(chunk, d_k) == 0) return GDN2_ERR_SHAPE;
  const bool tokens = (long long)B * T * H > 0;
  if (tokens && (!q || !k || !v || !log_alpha || !b || !w || !o)) return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S0, o, S_T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if ((long long)B * H == 0) return GDN2_OK;
  ChunkArgs a{q, k, v, b, w, log_alpha, S0, o, S_T, B, T, H, d_k, d_v, true};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = (T == 0) ? launch_state_copy(a, st) : launch_chunk_fwd_csize(a, chunk, st);
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" size_t gdn2_chunk_bwd_workspace_bytes(int B, int T, int H, int d_k, int d_v) {
  if (!sizes_ok(B, T, H, d_k, d_v)) return 0;
  return chunk_bwd_workspace_bytes(B, T, H, d_k, d_v);
}

extern "C" gdn2_status gdn2_chunk_bwd(const void* q, const void* k, const void* v, const float* log_alpha,
                                      const void* b, const void* w, const float* S0, const float* dO,
                                      const float* dS_T, float* dq, float* dk, float* dv, float* dlog_alpha,
                                      float* db, float* dw, float* dS0, int B, int T, int H, int d_k, int d_v,
                                      gdn2_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (!sizes_ok(B, T, H, d_k, d_v)) return GDN2_ERR_SHAPE;
  const bool tokens = (long long)B * T * H > 0;
  if (tokens && (!q || !k || !v || !log_alpha || !b || !w || !dO || !dq || !dk || !dv || !dlog_alpha || !db ||
                 !dw || !workspace))
    return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk, dv, dlog_alpha, db, dw, dS0, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if (tokens && workspace_bytes < chunk_bwd_workspace_bytes(B, T, H, d_k, d_v)) return GDN2_ERR_SHAPE;
  if ((long long)B * H == 0) return GDN2_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (T == 0) {  // no tokens: the gradient passes straight to the entering state
    if (dS0) {
      const size_t n = (size_t)B * H * d_k * d_v * sizeof(float);
      e = dS_T ? cudaMemcpyAsync(dS0, dS_T, n, cudaMemcpyDeviceToDevice, st) : cudaMemsetAsync(dS0, 0, n, st);
    }
  } else {
    ChunkBwdArgs a{q, k, v, b, w, log_alpha, S0, dO, dS_T, dq, dk, dv, dlog_alpha, db, dw, dS0,
                   static_cast<float*>(workspace), B, T, H, d_k, d_v, dt == GDN2_BF16};
    e = launch_chunk_bwd(a, st);
  }
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" gdn2_status gdn2_chunk_fwd_varlen(const void* q, const void* k, const void* v, const float* log_alpha,
                                             const void* b, const void* w, const int* cu_seqlens, const float* S0,
                                             float* o, float* S_T, int N, int T, int H, int d_k, int d_v,
                                             gdn2_dtype dt, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (dt != GDN2_BF16) return GDN2_ERR_DTYPE;  // packed sequences: bf16 inputs only
  if (!sizes_ok(1, T, H, d_k, d_v) || N < 0 || (long long)N * H > 0x7fffffffLL) return GDN2_ERR_SHAPE;
  if ((long long)N * H == 0) return GDN2_OK;
  if (!cu_seqlens) return GDN2_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !log_alpha || !b || !w || !o)) return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S0, o, S_T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return GDN2_ERR_ALIGN;

  ChunkArgs a{q, k, v, b, w, log_alpha, S0, o, S_T, N, T, H, d_k, d_v, true, cu_seqlens};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // no tokens at all: every sequence is empty and keeps its entering state
  cudaError_t e = (T == 0) ? launch_state_copy(a, st) : launch_chunk_fwd_tc(a, st);
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" gdn2_status gdn2_chunk_fwd_raw(const void* q_raw, const void* k_raw, const void* v, const float* a_raw,
                                          const void* b_raw, const void* w_raw, const float* decay_scale,
                                          const int* cu_seqlens, const float* S0, float* o, float* S_T, int B, int T,
                                          int H, int d_k, int d_v, gdn2_dtype dt, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (dt != GDN2_BF16) return GDN2_ERR_DTYPE;  // raw projections: bf16 inputs only
  const bool packed = cu_seqlens != nullptr;
  if (!sizes_ok(packed ? 1 : B, T, H, d_k, d_v) || B < 0 || (long long)B * H > 0x7fffffffLL) return GDN2_ERR_SHAPE;
  if ((long long)B * H == 0) return GDN2_OK;
  if (T > 0 && (!q_raw || !k_raw || !v || !a_raw || !b_raw || !w_raw || !o)) return GDN2_ERR_NULL;
  const void* ptrs[] = {q_raw, k_raw, v, a_raw, b_raw, w_raw, S0, o, S_T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return GDN2_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(decay_scale) & 3u) != 0) return GDN2_ERR_ALIGN;

  ChunkArgs a{q_raw, k_raw, v, b_raw, w_raw, a_raw, S0, o, S_T, B, T, H, d_k, d_v, true, cu_seqlens};
  a.raw = true;
  a.decay_scale = decay_scale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = (T == 0) ? launch_state_copy(a, st) : launch_chunk_fwd_tc(a, st);
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" gdn2_status gdn2_short_conv(const void* x, const float* weight, const float* bias, const int* cu_seqlens,
                                       const void* hist_in, void* y, void* hist_out, int B, int T, int C,
                                       gdn2_dtype dt, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  const bool packed = cu_seqlens != nullptr;
  if (B < 0 || T < 0 || C < 0 || C % 8 != 0 || C > (1 << 24)) return GDN2_ERR_SHAPE;
  const long long ntok = packed ? (long long)T : (long long)B * T;
  if (ntok > 0x7fffffffLL - 64 || ntok * C > (1LL << 46)) return GDN2_ERR_SHAPE;
  if (B == 0 || C == 0) return GDN2_OK;
  if (ntok > 0 && (!x || !y || !weight)) return GDN2_ERR_NULL;
  if (hist_out && !x && ntok > 0) return GDN2_ERR_NULL;
  const void* ptrs[] = {x, weight, bias, hist_in, y, hist_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN2_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return GDN2_ERR_ALIGN;
  if (x && x == y) return GDN2_ERR_SHAPE;  // the window reads inputs other threads would overwrite
  ShortConvArgs a{x, weight, bias, cu_seqlens, hist_in, y, hist_out, B, T, C, dt == GDN2_BF16};
  cudaError_t e = launch_short_conv(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" gdn2_status gdn2_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                                        const void* b, const void* w, float* S, float* o, int B, int H, int d_k,
                                        int d_v, gdn2_dtype dt, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (!sizes_ok(B, 1, H, d_k, d_v)) return GDN2_ERR_SHAPE;
  if ((long long)B * H == 0) return GDN2_OK;
  if (!q || !k || !v || !log_alpha || !b || !w || !S || !o) return GDN2_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, b, w, S, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN2_ERR_ALIGN;
  DecodeArgs a{q, k, v, b, w, log_alpha, S, o, B, H, d_k, d_v, dt == GDN2_BF16};
  cudaError_t e = launch_decode_step(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" gdn2_status gdn2_decode_step_raw(const void* q_raw, const void* k_raw, const void* v, const float* a_raw,
                                            const void* b_raw, const void* w_raw, const float* decay_scale, float* S,
                                            float* o, int B, int H, int d_k, int d_v, gdn2_dtype dt, void* stream) {
  if (dt != GDN2_F32 && dt != GDN2_BF16) return GDN2_ERR_DTYPE;
  if (!sizes_ok(B, 1, H, d_k, d_v)) return GDN2_ERR_SHAPE;
  if ((long long)B * H == 0) return GDN2_OK;
  if (!q_raw || !k_raw || !v || !a_raw || !b_raw || !w_raw || !S || !o) return GDN2_ERR_NULL;
  const void* ptrs[] = {q_raw, k_raw, v, a_raw, b_raw, w_raw, S, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN2_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(decay_scale) & 3u) != 0) return GDN2_ERR_ALIGN;
  DecodeArgs a{q_raw, k_raw, v, b_raw, w_raw, a_raw, S, o, B, H, d_k, d_v, dt == GDN2_BF16};
  a.raw = true;
  a.decay_scale = decay_scale;
  cudaError_t e = launch_decode_step(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN2_OK : cuda_fail(e);
}

extern "C" gdn2_status gdn2_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e);
  if (word) {
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word & kErrBadSeqlens) return GDN2_ERR_SHAPE;
    if (word & kErrWaitTimeout) return GDN2_ERR_TIMEOUT;
    return GDN2_ERR_RANGE;
  }
  return GDN2_OK;
}

extern "C" const char* gdn2_status_string(int status) {
  switch (status) {
    case GDN2_OK: return "ok";
    case GDN2_ERR_NULL: return "a required pointer is NULL";
    case GDN2_ERR_SHAPE: return "bad shape (negative size, d_k/d_v not 64 or 128, or too large)";
    case GDN2_ERR_DTYPE: return "unknown dtype";
    case GDN2_ERR_ALIGN: return "pointer not 16-byte aligned";
    case GDN2_ERR_CUDA: return "CUDA error";
    case GDN2_ERR_TIMEOUT: return "device-side wait timed out";
    case GDN2_ERR_RANGE: return "decay out of range (cumulative log decay within a chunk below -80)";
    default: return "unknown status";
  }
}

extern "C" const char* gdn2_last_cuda_error(void) { return g_last_cuda; }

extern "C" int gdn2_version(void) { return 200; }

#ifdef GDN2_STAMPS
// Instrumented build only: copies the stamp words ([chunk][slot] clock64 values of the last
// chunk launch's first CTA) to host memory; returns the number of words copied.
extern "C" GDN2_API int gdn2_stamps_read(unsigned long long* host, int n) {
  if (!host || n <= 0) return 0;
  if (n > kStampWords) n = kStampWords;
  if (cudaDeviceSynchronize() != cudaSuccess) return 0;
  if (cudaMemcpyFromSymbol(host, g_stamps, (size_t)n * sizeof(unsigned long long)) != cudaSuccess) return 0;
  return n;
}
#endif
