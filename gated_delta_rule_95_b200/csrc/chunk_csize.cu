// The chunk-size study's entry: the prefill forward at C = 32, 64 or 128 (bf16 inputs), each
// size on a tcgen05 kernel (snilld.dk, "POC-matrix der daekker de haarde hjoerner": latency,
// throughput and peak memory at C = 64, the implementation's size, and also at 32 and 128).
//   C = 32:  chunk_tc32.cu, the production kernel's design with 32-token chunks
//   C = 64:  chunk_tc.cu, the production kernel
//   C = 128: chunk_tc128.cu, the same products with the phases of a chunk run in sequence
//            (its tiles exceed one SM's shared and tensor memory when held resident)
#include <cuda_runtime.h>

#include "gdn2_internal.h"

namespace gdn2 {

size_t chunk_fwd_csize_smem_bytes(int chunk, int dk) {
  if (dk != 64 && dk != 128) return 0;
  switch (chunk) {
    case 32: return chunk_fwd_tc32_smem_bytes();
    case 64: return chunk_fwd_tc_smem_bytes();
    case 128: return chunk_fwd_tc128_smem_bytes();
    default: return 0;
  }
}

cudaError_t launch_chunk_fwd_csize(const ChunkArgs& a, int chunk, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  switch (chunk) {
    case 32: return launch_chunk_fwd_tc32(a, st);
    case 64: return launch_chunk_fwd_tc(a, st);
    case 128: return launch_chunk_fwd_tc128(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gdn2
