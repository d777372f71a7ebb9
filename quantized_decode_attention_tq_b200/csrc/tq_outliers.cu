// Calibration of the V v3 outlier channels ("llama-tq" article, V
// sub-families: v3 with outlier-channel separation): for every kv-head, the k
// channels of largest mean square over sample V rows.  One CTA per kv-head,
// one thread per channel; sums in fp64 in a fixed order, so the choice is
// deterministic; a tie goes to the lower channel.

#include <cuda_fp16.h>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kMaxD = kMaxDecodeHeadDim;

__global__ void __launch_bounds__(kMaxD) pick_outliers_kernel(const void* v, int f16, int batch, int kv_heads,
                                                              int rows, int head_dim, int k, int32_t* channels) {
  __shared__ double ms[kMaxD];
  __shared__ int taken[kMaxD];
  const int h = blockIdx.x, c = threadIdx.x;
  if (c < head_dim) {
    double acc = 0.0;
    for (int b = 0; b < batch; ++b) {
      const size_t base = (((size_t)b * kv_heads + h) * rows) * head_dim + c;
      for (int r = 0; r < rows; ++r) {
        const float x = f16 ? __half2float(static_cast<const __half*>(v)[base + (size_t)r * head_dim])
                            : static_cast<const float*>(v)[base + (size_t)r * head_dim];
        acc += (double)x * (double)x;
      }
    }
    ms[c] = acc;
    taken[c] = 0;
  }
  __syncthreads();
  if (c == 0) {
    int sel[kOutlierMax];
    for (int j = 0; j < k; ++j) {  // largest remaining; the first (lowest) on a tie
      int best = -1;
      for (int i = 0; i < head_dim; ++i)
        if (!taken[i] && (best < 0 || ms[i] > ms[best])) best = i;
      taken[best] = 1;
      sel[j] = best;
    }
    for (int a = 1; a < k; ++a) {  // ascending channel order
      const int x = sel[a];
      int b = a - 1;
      while (b >= 0 && sel[b] > x) {
        sel[b + 1] = sel[b];
        --b;
      }
      sel[b + 1] = x;
    }
    for (int j = 0; j < k; ++j) channels[(size_t)h * k + j] = sel[j];
  }
}

}  // namespace

int launch_pick_outliers(const void* v, int f16, int batch, int kv_heads, int rows, int head_dim, int k,
                         int32_t* channels, cudaStream_t stream) {
  if (head_dim > kMaxD || k > kOutlierMax) return TQ_ERR_UNSUPPORTED;
  pick_outliers_kernel<<<kv_heads, kMaxD, 0, stream>>>(v, f16, batch, kv_heads, rows, head_dim, k, channels);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq
