// Decode-attention launcher: one translation unit per K bit width holds the
// kernel instantiations (tq_decode_k{2,3,4}.cu, kernel in tq_decode_kernel.cuh);
// this file picks one.

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {

int launch_decode_k2(DecodeParams& p, cudaStream_t stream);
int launch_decode_k3(DecodeParams& p, cudaStream_t stream);
int launch_decode_k4(DecodeParams& p, cudaStream_t stream);

int launch_decode(const DecodeParams& params, cudaStream_t stream) {
  DecodeParams p = params;  // the launcher adds the shared-memory plan
  switch (p.k_bits) {
    case 2: return launch_decode_k2(p, stream);
    case 3: return launch_decode_k3(p, stream);
    case 4: return launch_decode_k4(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
