// Decode-attention kernels for 4-bit K codes (every V bit width, head_dim
// 128 and 256, every mode and group width); the kernel is in
// tq_decode_kernel.cuh.

#include "tq_decode_kernel.cuh"

namespace tq {

int launch_decode_k4(DecodeParams& p, cudaStream_t stream) { return dec::dispatch_kb<4>(p, stream); }

}  // namespace tq
