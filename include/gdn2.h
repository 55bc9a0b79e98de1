/*
 * gdn2.h — C ABI of the Gated DeltaNet-2 token mixer for NVIDIA B200 (sm_100a).
 *
 * The operation (snilld.dk, "Gated DeltaNet-2 fra NVIDIA kan gore dekodning
 * billigere...", section "Hvad Gated DeltaNet-2 aendrer", the compact update),
 * per batch element b and head h, with a d_k x d_v fp32 state S:
 *
 *     S_t = (I - k_t (b_t * k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t * v_t)^T
 *     o_t = S_t^T q_t
 *
 * alpha_t in (0,1]^{d_k} is the channel-wise decay (applied before the edit),
 * b_t in [0,1]^{d_k} the erase gate on the key axis, w_t in [0,1]^{d_v} the write
 * gate on the value axis.  The readout uses the updated state (Gated DeltaNet-2
 * guide, "End-to-End PyTorch Implementation").  There is no query scaling.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no pointer after the call returns.
 *   - Tensors are dense, row-major (C order), and 16-byte aligned.
 *   - The decay gate is passed as log(alpha), fp32, finite and <= 0.  Within one
 *     chunk of 64 tokens the cumulative log decay of a channel must stay above
 *     -80 (the chunk form scales keys by exp(-sum log alpha)); beyond that the
 *     result is undefined, and the chunk kernels flag it: the next
 *     gdn2_device_status() returns GDN2_ERR_RANGE.  This holds for the
 *     raw-projection entry points too, where log alpha = -s_h softplus(a) is
 *     formed inside the kernel (a_raw averaging above about 1.2 over a chunk at
 *     s_h = 1 leaves the range).
 *   - dt selects the type of q, k, v, b and w: GDN2_BF16 or GDN2_F32.  The
 *     output o and the state (S0, S_T, S) are always fp32, and accumulation is
 *     fp32.  (o is stored in fp32 because its values are heavy-tailed: rounding
 *     it to bf16 alone would cost over half of a 2e-2 max-error/RMS budget.)
 *   - d_k and d_v are each 64 or 128.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it.  Argument errors are returned synchronously before any
 *     work is queued; launch failures return GDN2_ERR_CUDA.  A device-side wait
 *     that runs out of time sets a device error word that gdn2_device_status()
 *     reports as GDN2_ERR_TIMEOUT; it never traps or hangs the GPU.
 *   - No exception crosses this boundary.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN2_OK = 0,
  GDN2_ERR_NULL = 1,    /* a required pointer is NULL */
  GDN2_ERR_SHAPE = 2,   /* negative size, or d_k / d_v not 64 or 128, or sizes overflow */
  GDN2_ERR_DTYPE = 3,   /* dt is not a gdn2_dtype value */
  GDN2_ERR_ALIGN = 4,   /* a pointer is not 16-byte aligned */
  GDN2_ERR_CUDA = 5,    /* a CUDA runtime/driver call failed (see gdn2_last_cuda_error) */
  GDN2_ERR_TIMEOUT = 6, /* a bounded device-side wait gave up (device error word set) */
  GDN2_ERR_RANGE = 7    /* the decay left the supported range: some channel's cumulative log
                           decay within one 64-token chunk fell below -80 (outputs undefined;
                           reported by gdn2_device_status) */
} gdn2_status;

typedef enum { GDN2_F32 = 0, GDN2_BF16 = 1 } gdn2_dtype;

/*
 * Chunkwise-parallel prefill forward, chunk size C = 64.
 *
 * Follows the chunkwise decomposition of the Gated DeltaNet-2 guide ("Chunkwise
 * Parallel Algorithm for GPU Training": chunks of C tokens, intra-chunk work as
 * tensor-core products, the state handed across chunks) in the WY form with the
 * cumulative channel-wise decay folded into the factors of each rank-one erase
 * (snilld.dk, "Hvad betyder det for traening og inferens").  The result equals
 * the token-by-token recurrence above up to rounding.  bf16 inputs: tcgen05 tf32
 * products with fp32 accumulation; fp32 inputs with d_k = d_v = 64: tcgen05 split
 * products (hi*hi + hi*lo + lo*hi of tf32 parts, fp32-accurate); fp32 inputs with a head
 * size of 128: fp32 products on the CUDA cores.
 *
 *   q, k, b      : [B, T, H, d_k]  dt
 *   v, w         : [B, T, H, d_v]  dt
 *   log_alpha    : [B, T, H, d_k]  fp32
 *   S0           : [B, H, d_k, d_v] fp32, read only; NULL means a zero state
 *   o            : [B, T, H, d_v]  fp32, written
 *   S_T          : [B, H, d_k, d_v] fp32, the state after token T-1, written;
 *                  NULL means "do not write"; may alias S0
 *   B, T, H      : >= 0; T need not be a multiple of 64 (the last chunk may be
 *                  partial); T = 0 copies S0 (or zeros) to S_T
 */
GDN2_API gdn2_status gdn2_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                           const void* b, const void* w, const float* S0, float* o, float* S_T,
                           int B, int T, int H, int d_k, int d_v, gdn2_dtype dt, void* stream);

/*
 * Chunkwise prefill forward with every sequence split into `segments` consecutive
 * segments that run in parallel: for long sequences with few (batch, head) pairs, which
 * would otherwise occupy one SM each and leave the rest idle.  The result is
 * gdn2_chunk_fwd's, up to rounding.
 *
 * The recurrence is linear in (state, v) (snilld.dk, "Hvad Gated DeltaNet-2 aendrer":
 * S_t = (I - k_t (b_t * k_t)^T) D_t S_{t-1} + k_t (w_t * v_t)^T), so the state after
 * segment s is M_s S + N_s, with M_s = the state reached from S = I with no writes and
 * N_s = the state reached from S = 0.  A first pass computes segment 0 from S0 and
 * (M_s, N_s) for every later segment; a small kernel chains the start states
 * S(s+1) = M_s S(s) + N_s; a last pass recomputes segments 1 .. P-1 from their start
 * states, writing o and, for the last segment, S_T.  This is the exchange step of a
 * sequence-parallel prefill done within one GPU; it costs about 3x the work of the
 * segments it splits, in exchange for P times the parallelism.
 *
 *   q .. S_T, B, T, H, dt : as gdn2_chunk_fwd; d_k = d_v required; dt = GDN2_BF16
 *   segments              : >= 1 (1 = gdn2_chunk_fwd); gdn2_chunk_fwd_split_segments()
 *                           gives the count a simple wave model prefers
 *   workspace             : DEVICE scratch of at least
 *                           gdn2_chunk_fwd_split_workspace_bytes(B, H, d_k, d_v, segments)
 *                           bytes, 16-byte aligned, owned by the caller; overwritten; two
 *                           calls in flight must not share it
 */
GDN2_API int gdn2_chunk_fwd_split_segments(int B, int T, int H, int sm_count);
GDN2_API size_t gdn2_chunk_fwd_split_workspace_bytes(int B, int H, int d_k, int d_v, int segments);
GDN2_API gdn2_status gdn2_chunk_fwd_split(const void* q, const void* k, const void* v, const float* log_alpha,
                                 const void* b, const void* w, const float* S0, float* o, float* S_T, int B,
                                 int T, int H, int d_k, int d_v, gdn2_dtype dt, int segments, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * Backward of gdn2_chunk_fwd: given dO = dL/do and dS_T = dL/dS_T, the gradients of L with
 * respect to q, k, v, log_alpha, b, w and S0 (reverse mode of the chunkwise WY form of
 * the Gated DeltaNet-2 guide's "Chunkwise Parallel Algorithm for GPU Training", the
 * training-time counterpart of the forward).  The forward's inputs are passed again; the
 * chunk states are recomputed (bf16 inputs with d_k = d_v: by the tensor-core forward, tf32
 * products; otherwise in fp32).  bf16 inputs with d_k = d_v = 128 run on the 5th-generation
 * tensor cores (tcgen05, tf32 products, fp32 accumulation): the forward's checkpoint pass, a
 * reverse sweep per (batch, head) carrying the state gradient, and a pass over all chunks in
 * parallel for the other gradients.  Other bf16 shapes use tf32 warp-level MMAs; fp32
 * inputs run fp32 products on the CUDA cores.
 *
 *   q .. w, S0, B, T, H, d_k, d_v, dt : as gdn2_chunk_fwd (the forward's inputs)
 *   dO          : [B, T, H, d_v] fp32
 *   dS_T        : [B, H, d_k, d_v] fp32, or NULL for zero
 *   dq, dk, db, dlog_alpha : [B, T, H, d_k] fp32, written
 *   dv, dw      : [B, T, H, d_v] fp32, written
 *   dS0         : [B, H, d_k, d_v] fp32, written, or NULL for "not needed"
 *   workspace   : DEVICE scratch of gdn2_chunk_bwd_workspace_bytes(B, T, H, d_k, d_v)
 *                 bytes (per chunk: its entering state, and for d_k = d_v = 128 also the
 *                 state gradient leaving it and the chunk's U, -dR, T^T, P^T), 16-byte
 *                 aligned, owned by the caller; two calls in flight must not share it
 * Gradient buffers must not alias the inputs or each other.
 */
GDN2_API size_t gdn2_chunk_bwd_workspace_bytes(int B, int T, int H, int d_k, int d_v);
GDN2_API gdn2_status gdn2_chunk_bwd(const void* q, const void* k, const void* v, const float* log_alpha,
                           const void* b, const void* w, const float* S0, const float* dO, const float* dS_T,
                           float* dq, float* dk, float* dv, float* dlog_alpha, float* db, float* dw,
                           float* dS0, int B, int T, int H, int d_k, int d_v, gdn2_dtype dt, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * gdn2_chunk_fwd_split without a caller workspace, for callers that cannot allocate: the
 * scratch is a fixed 16 MiB array in the library's own device memory, reserved when the
 * library's device module is loaded on a device (with CUDA's lazy module loading, at the
 * first call that touches the module there) and held until the process exits.  The Gated DeltaNet-2 pages describe no counterpart of this
 * entry point; it is an interface convenience over the same kernels.
 *
 *   arguments   : as gdn2_chunk_fwd_split, without workspace and workspace_bytes
 *   limit       : gdn2_chunk_fwd_split_workspace_bytes(B, H, d_k, d_v, segments) must not
 *                 exceed 16 MiB (e.g. 16 heads x 5 segments at d = 128); larger requests
 *                 return GDN2_ERR_SHAPE before any work is queued
 *   first call  : on each device, the first call looks up the scratch's address
 *                 (cudaGetSymbolAddress, with that device current); make that first call
 *                 outside any stream capture.  A failed lookup returns GDN2_ERR_CUDA.
 *   zeroing     : nothing in the scratch needs to start at zero: every value is written
 *                 before it is read within the call
 *   concurrency : the scratch is shared by all calls on a device; two calls in flight at
 *                 the same time (on different streams or host threads) race on it
 */
GDN2_API gdn2_status gdn2_chunk_fwd_split_static(const void* q, const void* k, const void* v, const float* log_alpha,
                                        const void* b, const void* w, const float* S0, float* o, float* S_T,
                                        int B, int T, int H, int d_k, int d_v, gdn2_dtype dt, int segments,
                                        void* stream);

/*
 * Chunkwise prefill forward at a chosen chunk size, for the chunk-size trade-off that the
 * snilld.dk article's proof-of-concept list asks to measure ("POC-matrix der daekker de
 * haarde hjoerner": latency, throughput and peak memory at C = 64 and also at 32 and 128).
 * Same recurrence and result as gdn2_chunk_fwd (the Gated DeltaNet-2 guide's chunkwise WY
 * form, decay folded at the chunk start), each size on a tcgen05 kernel (tf32 operands,
 * fp32 accumulation in tensor memory): C = 64 is gdn2_chunk_fwd's kernel, C = 32 the same
 * design with 32-token chunks, C = 128 the same products with the phases of a chunk run in
 * sequence (its tiles do not fit one SM's memory when held resident).
 *
 *   q .. S_T, B, T, H, d_k, d_v : as gdn2_chunk_fwd
 *   dt          : GDN2_BF16 (fp32 inputs return GDN2_ERR_DTYPE)
 *   chunk       : 32, 64 or 128 tokens per chunk; anything else returns GDN2_ERR_SHAPE
 * The decay limit of the shared conventions holds per chunk of the chosen size: the
 * cumulative log decay of a channel over 128 tokens at chunk = 128 (flagged the same way).
 * gdn2_chunk_fwd_csize_smem_bytes(chunk, d_k) is the shared memory one CTA of the kernel
 * holds (one CTA per (batch, head)), or 0 for an unsupported pair; the call needs no device
 * memory besides its arguments.
 */
GDN2_API size_t gdn2_chunk_fwd_csize_smem_bytes(int chunk, int d_k);
GDN2_API gdn2_status gdn2_chunk_fwd_csize(const void* q, const void* k, const void* v, const float* log_alpha,
                                 const void* b, const void* w, const float* S0, float* o, float* S_T, int B,
                                 int T, int H, int d_k, int d_v, gdn2_dtype dt, int chunk, void* stream);

/*
 * Chunkwise prefill forward over a packed batch of variable-length sequences, each
 * with its own state: the serving case of many independent dialogues or documents
 * whose states are carried between calls (DeltaNet-2 AI architecture guide: the
 * inference endpoint accepts and returns the updated state; Gated DeltaNet-2 guide,
 * "Enterprise Strategy": continuous dialogues and streaming documents).  Sequence n
 * is the token range [cu_seqlens[n], cu_seqlens[n+1]) of the packed tensors; each
 * sequence is computed exactly as gdn2_chunk_fwd computes one batch element.
 *
 *   q, k, b      : [T, H, d_k]  bf16 (T = total tokens of all sequences)
 *   v, w         : [T, H, d_v]  bf16
 *   log_alpha    : [T, H, d_k]  fp32
 *   cu_seqlens   : [N + 1] int32 DEVICE array, cu_seqlens[0] = 0, non-decreasing,
 *                  cu_seqlens[N] = T; a sequence may be empty.  Offsets out of order
 *                  or out of range are detected on the device: that sequence is
 *                  skipped and gdn2_device_status() reports GDN2_ERR_SHAPE.
 *   S0           : [N, H, d_k, d_v] fp32, read only; NULL means zero states
 *   o            : [T, H, d_v]  fp32, written
 *   S_T          : [N, H, d_k, d_v] fp32, each sequence's final state, written;
 *                  NULL means "do not write"; may alias S0
 *   N, T, H      : >= 0
 *   dt           : GDN2_BF16 (fp32 inputs return GDN2_ERR_DTYPE)
 */
GDN2_API gdn2_status gdn2_chunk_fwd_varlen(const void* q, const void* k, const void* v, const float* log_alpha,
                                  const void* b, const void* w, const int* cu_seqlens, const float* S0,
                                  float* o, float* S_T, int N, int T, int H, int d_k, int d_v, gdn2_dtype dt,
                                  void* stream);

/*
 * Chunkwise prefill forward fed with the raw projections, the layer's input
 * activations applied inside the kernel as it loads each chunk (so they cost no
 * extra pass over memory): q and k are L2-normalised per (token, head) (a zero
 * vector stays zero), b = sigmoid(b_raw), w = sigmoid(w_raw) (Gated DeltaNet-2 guide,
 * "Normalization and Short Convolutions" and "Decoupled Erase and Write Gates"), and
 * log alpha = -s_h * softplus(a_raw) with a per-head scale s_h (a channel-wise decay
 * in (0, 1): snilld.dk, "Hvad Gated DeltaNet-2 aendrer").  The result is gdn2_chunk_fwd (or
 * gdn2_chunk_fwd_varlen) on the activated inputs, up to rounding: the activations are
 * computed in fp32 and never rounded back to bf16.
 *
 *   q_raw, k_raw, b_raw : [B, T, H, d_k]  bf16 (packed: [T, H, d_k])
 *   v, w_raw            : [B, T, H, d_v]  bf16 (packed: [T, H, d_v])
 *   a_raw               : [B, T, H, d_k]  fp32, finite (packed: [T, H, d_k])
 *   decay_scale         : [H] fp32 DEVICE array of s_h > 0, 4-byte aligned; NULL means 1
 *   cu_seqlens          : NULL: B sequences of T tokens each.  Otherwise a packed batch
 *                         of B sequences over T tokens in total, exactly as
 *                         gdn2_chunk_fwd_varlen takes it (N = B).
 *   S0, o, S_T          : as gdn2_chunk_fwd (packed: as gdn2_chunk_fwd_varlen)
 *   dt                  : GDN2_BF16 (fp32 inputs return GDN2_ERR_DTYPE)
 */
GDN2_API gdn2_status gdn2_chunk_fwd_raw(const void* q_raw, const void* k_raw, const void* v, const float* a_raw,
                               const void* b_raw, const void* w_raw, const float* decay_scale,
                               const int* cu_seqlens, const float* S0, float* o, float* S_T, int B, int T,
                               int H, int d_k, int d_v, gdn2_dtype dt, void* stream);

/*
 * Short causal depthwise convolution with 4 taps over the token axis, the local mixing
 * the layer applies to q, k and v before the recurrence (Gated DeltaNet-2 guide,
 * "Normalization and Short Convolutions"; the guide's layer pads each channel on the
 * left so that token t sees tokens t-3 .. t, and adds a bias):
 *
 *     y[t, c] = bias[c] + sum_{j=0..3} weight[c, j] * x[t - 3 + j, c]
 *
 * Tokens before a sequence's first are taken from its carried history (the last three
 * inputs of the previous call, oldest first), or are zero.  Accumulation in fp32; y is
 * rounded to dt.  Streaming decode is the case T = 1 with hist_out = hist_in.
 *
 *   x, y       : [B, T, C] dt (packed: [T, C]); y must not alias x
 *   weight     : [C, 4] fp32 (the layout of a depthwise Conv1d weight [C, 1, 4])
 *   bias       : [C] fp32, or NULL for none
 *   cu_seqlens : NULL: B sequences of T tokens.  Otherwise [B + 1] int32 DEVICE offsets of
 *                B packed sequences over T tokens, as gdn2_chunk_fwd_varlen takes them;
 *                offsets out of order or out of range are reported by
 *                gdn2_device_status() as GDN2_ERR_SHAPE (the affected outputs are not
 *                written)
 *   hist_in    : [B, 3, C] dt, read only, or NULL for zeros
 *   hist_out   : [B, 3, C] dt, written with each sequence's last three inputs (for a
 *                sequence shorter than three, the tail of its history first), or NULL;
 *                may alias hist_in
 *   C          : a multiple of 8 (16-byte rows), at most 2^24
 */
GDN2_API gdn2_status gdn2_short_conv(const void* x, const float* weight, const float* bias, const int* cu_seqlens,
                            const void* hist_in, void* y, void* hist_out, int B, int T, int C, gdn2_dtype dt,
                            void* stream);

/*
 * One recurrent decode step: the update above for a single token per
 * (sequence, head), with the state updated in place (Gated DeltaNet-2 guide,
 * "4.5x Higher Decoding Throughput with Zero KV Cache": a fixed-size state
 * streamed once per generated token).
 *
 *   q, k, b      : [B, H, d_k]  dt
 *   v, w         : [B, H, d_v]  dt
 *   log_alpha    : [B, H, d_k]  fp32
 *   S            : [B, H, d_k, d_v] fp32, read and overwritten with S'
 *   o            : [B, H, d_v]  fp32, written
 */
GDN2_API gdn2_status gdn2_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                             const void* b, const void* w, float* S, float* o,
                             int B, int H, int d_k, int d_v, gdn2_dtype dt, void* stream);

/*
 * One decode step on the raw projections: the activations of gdn2_chunk_fwd_raw (q and k
 * L2-normalised per (sequence, head), b = sigmoid(b_raw), w = sigmoid(w_raw), log alpha =
 * -s_h softplus(a_raw)) computed in fp32 inside the step, then gdn2_decode_step.
 *
 *   q_raw, k_raw, b_raw : [B, H, d_k]  dt
 *   v, w_raw            : [B, H, d_v]  dt
 *   a_raw               : [B, H, d_k]  fp32, finite
 *   decay_scale         : [H] fp32 DEVICE array of s_h > 0, 4-byte aligned; NULL means 1
 *   S, o                : as gdn2_decode_step
 */
GDN2_API gdn2_status gdn2_decode_step_raw(const void* q_raw, const void* k_raw, const void* v, const float* a_raw,
                                 const void* b_raw, const void* w_raw, const float* decay_scale, float* S,
                                 float* o, int B, int H, int d_k, int d_v, gdn2_dtype dt, void* stream);

/* Synchronises the current device, then reports and clears the device error
 * word: GDN2_OK, GDN2_ERR_TIMEOUT (a bounded wait gave up), GDN2_ERR_SHAPE (bad
 * cu_seqlens), or GDN2_ERR_CUDA if the sync itself failed. */
GDN2_API gdn2_status gdn2_device_status(void);

/* Static description of a status code. */
GDN2_API const char* gdn2_status_string(int status);

/* Text of the last CUDA error seen by this library on the calling thread. */
GDN2_API const char* gdn2_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
GDN2_API int gdn2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN2_H */
