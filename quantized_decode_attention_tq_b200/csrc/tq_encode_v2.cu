// V v2 encoder: trellis-coded quantisation (TCQ) of each 128-coordinate block.
//
// Method: "llama-tq" article (zingnex), V sub-family section: v2 is a group
// Viterbi trellis code, the default V format (V is heavy-tailed; a trellis
// spends its bits where the values are).  The page names the technique only;
// the reading taken here is TCQ (Marcellin and Fischer, IEEE Trans. Commun.
// 38(1), 1990) on the normalised rotated coordinates u = H.(s o x) / ||x||
// that the v1 quantiser uses:
//   * doubled codebook: the 2^(b+1) Lloyd-Max levels of N(0,1), split into
//     four subsets D_k = {levels of index k mod 4};
//   * 4-state trellis: branch bit beta takes state s to ((s & 1) << 1) | beta
//     and carries subset (s & 1) + 2 (beta xor (s >> 1)), i.e.
//       s = 0: D0, D2   s = 1: D1, D3   s = 2: D2, D0   s = 3: D3, D1;
//   * one block per group, from state 0; the Viterbi search minimises the
//     squared error; each branch takes the nearest level of its subset;
//   * ties: the lower predecessor state, the lower final state, the lower
//     level inside a subset;
//   * storage: 64 fields of 2b bits per block, LSB-first; field k holds
//     j_2k, j_2k+1 (b - 1 bits each), then beta_2k, beta_2k+1.
// The block norm and rotation are those of the v1 encoder.
//
// Mapping: a warp takes 32 consecutive blocks (one contiguous input range).
// Eight blocks at a time it loads them (lane l: elements l, l + 32, l + 64,
// l + 96 of each), then block by block flips the signs, runs the unnormalised
// WHT (two in-lane stages, five shuffle stages), reduces the squared norm and
// writes u to shared memory, one row per block (stride 129 floats, so both
// these row writes and the per-lane row reads below are bank-conflict free).
// Then lane i searches block i: per step the nearest level of each subset and
// its squared error, four add-compare-selects (4 decision bits per step, in
// shared memory), then the traceback, which takes each step's level index
// from its subset's decision points and rebuilds the pair fields in
// registers.

#include <cuda_fp16.h>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kV2Warps = 2;
constexpr int kV2Threads = 32 * kV2Warps;
constexpr int kURow = kBlock + 1;  // floats per u row
constexpr int kDecRow = 17;        // decision words per lane (16 + pad)

template <int BITS>
struct Tcq {
  static constexpr int kJ = 1 << (BITS - 1);  // levels per subset
  float lv[4][kJ];                             // level j of subset k
  float mid[4][kJ > 1 ? kJ - 1 : 1];           // decision points between them
  __device__ void load(const float* levels) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int j = 0; j < kJ; ++j) lv[k][j] = levels[4 * j + k];
#pragma unroll
      for (int j = 0; j + 1 < kJ; ++j) mid[k][j] = 0.5f * (lv[k][j] + lv[k][j + 1]);
    }
  }
  // nearest level of subset k (a compile-time index) to u (the lower one at
  // a midpoint)
  __device__ __forceinline__ int nearest(float u, int k, float& level) const {
    int j = 0;
    float l = lv[k][0];
#pragma unroll
    for (int m = 0; m + 1 < kJ; ++m) {
      const bool up = u > mid[k][m];
      j += up ? 1 : 0;
      l = up ? lv[k][m + 1] : l;
    }
    level = l;
    return j;
  }
  __device__ __forceinline__ float err(float u, int k) const {
    float l;
    nearest(u, k, l);
    const float d = u - l;
    return d * d;
  }
};

// Unnormalised WHT of one 128-block held by a warp, lane l holding elements
// l + 32e (e = 0..3): strides 1..16 between lanes l and l ^ stride (the lane
// with the bit clear keeps a + b, the other a - b), strides 32 and 64 in the
// lane.
__device__ __forceinline__ void wht_block(float (&v)[4], int lane) {
  float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2;
  v[1] = a1 + a3;
  v[2] = a0 - a2;
  v[3] = a1 - a3;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
      v[e] = hi ? o - v[e] : v[e] + o;
    }
  }
}

template <int BITS, bool F16>
__global__ void __launch_bounds__(kV2Threads)
encode_v2_kernel(const __grid_constant__ EncodeParams p) {
  constexpr int JW = BITS - 1;          // bits of a subset index
  constexpr int FW = 2 * BITS;          // bits of a pair field
  constexpr int NW = 4 * BITS;          // 32-bit words of a block's codes
  __shared__ float su[kV2Warps][32][kURow];
  __shared__ uint32_t sdec[kV2Warps][32][kDecRow];
  __shared__ __align__(16) float smid[4][4];  // decision points of each subset, for the traceback
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 16) {
    const int k = threadIdx.x >> 2, m = threadIdx.x & 3;
    smid[k][m] = m + 1 < (1 << (BITS - 1)) ? 0.5f * (p.tcq_levels[4 * m + k] + p.tcq_levels[4 * (m + 1) + k])
                                           : INFINITY;
  }
  __syncthreads();
  const int nb = p.head_dim / kBlock;
  const long long n_items = (long long)p.batch * p.kv_heads * p.seq_new * nb;
  const long long first = ((long long)blockIdx.x * kV2Warps + warp) * 32;
  uint32_t sgn = 0;  // bit e: the sign of element lane + 32e
#pragma unroll
  for (int e = 0; e < 4; ++e) sgn |= ((p.sign_mask[e] >> lane) & 1u) << e;
  const void* in = p.in[1];

  // ---- rotation and norm by the whole warp, eight blocks' loads in flight
  // at a time (the warp's 32 blocks are one contiguous input range) ---------
  float my_norm = 0.0f;
  for (int g0 = 0; g0 < 32; g0 += 8) {
    if (first + g0 >= n_items) break;  // warp-uniform
    float v8[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long item = first + g0 + i;
      const size_t off = (size_t)item * kBlock + lane;  // item * 128 = row * D + blk * 128
#pragma unroll
      for (int e = 0; e < 4; ++e)
        v8[i][e] = item >= n_items ? 0.0f
                   : F16 ? __half2float(static_cast<const __half*>(in)[off + 32 * e])
                         : static_cast<const float*>(in)[off + 32 * e];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float (&v)[4] = v8[i];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((sgn >> e) & 1u) v[e] = -v[e];
      float ss = v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3];
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      const float n = sqrtf(ss);
      wht_block(v, lane);
      const float inv = n > 0.0f ? 1.0f / n : 0.0f;  // u = 0 for a zero block
#pragma unroll
      for (int e = 0; e < 4; ++e) su[warp][g0 + i][lane + 32 * e] = v[e] * inv;
      if (lane == g0 + i) my_norm = n;
    }
  }
  __syncwarp();

  const long long item = first + lane;
  if (item >= n_items) return;
  // the host keeps the item count below 2^31: 32-bit splits by multiply-high
  const int lnb = nb == 1 ? 0 : nb == 2 ? 1 : 2;  // nb is 1, 2 or 4
  const uint32_t row = (uint32_t)item >> lnb;
  const int blk = (int)(item & (nb - 1));
  const uint32_t bh = p.div_seq_new.div(row);
  const int t = (int)(row - bh * (uint32_t)p.seq_new);
  const int b = (int)p.div_kv_heads.div(bh);
  int pos = t;
  if (p.start_pos) pos += __ldg(p.start_pos + b);
  if (pos < 0 || pos >= p.seq_cap) {
    if (p.status) atomicOr(p.status, TQ_DEV_POS_RANGE);
    return;
  }

  Tcq<BITS> tc;
  tc.load(p.tcq_levels);
  const float* u = su[warp][lane];
  uint32_t* dec = sdec[warp][lane];

  // ---- Viterbi search: metrics of states 0..3 -----------------------------
  float m0 = 0.0f, m1 = INFINITY, m2 = INFINITY, m3 = INFINITY;
  for (int w = 0; w < 16; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8) {
      const float x = u[8 * w + s8];
      const float e0 = tc.err(x, 0), e1 = tc.err(x, 1), e2 = tc.err(x, 2), e3 = tc.err(x, 3);
      // state 0 <- (0, D0) | (2, D2); 1 <- (0, D2) | (2, D0);
      // state 2 <- (1, D1) | (3, D3); 3 <- (1, D3) | (3, D1)
      const float a0 = m0 + e0, b0 = m2 + e2;
      const float a1 = m0 + e2, b1 = m2 + e0;
      const float a2 = m1 + e1, b2 = m3 + e3;
      const float a3 = m1 + e3, b3 = m3 + e1;
      const bool d0 = b0 < a0, d1 = b1 < a1, d2 = b2 < a2, d3 = b3 < a3;
      m0 = d0 ? b0 : a0;
      m1 = d1 ? b1 : a1;
      m2 = d2 ? b2 : a2;
      m3 = d3 ? b3 : a3;
      word |= ((d0 ? 1u : 0u) | (d1 ? 2u : 0u) | (d2 ? 4u : 0u) | (d3 ? 8u : 0u)) << (4 * s8);
    }
    dec[w] = word;
  }
  int s = 0;
  float best = m0;
  if (m1 < best) { best = m1; s = 1; }
  if (m2 < best) { best = m2; s = 2; }
  if (m3 < best) { best = m3; s = 3; }

  // ---- traceback, pair by pair from the end; fields assembled in place ---
  uint32_t out[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) out[w] = 0u;
#pragma unroll
  for (int k = 63; k >= 0; --k) {
    uint32_t jj[2], bb[2];
#pragma unroll
    for (int q = 1; q >= 0; --q) {
      const int i = 2 * k + q;
      const uint32_t d = (dec[i >> 3] >> (4 * (i & 7) + s)) & 1u;
      const int pred = d ? ((s >> 1) | 2) : (s >> 1);
      const int beta = s & 1;
      const int sub = (pred & 1) + 2 * (beta ^ (pred >> 1));
      // the level index in the subset: #{decision points below u} (the same
      // points the forward search compared with; unused slots are +inf)
      const float4 md = *reinterpret_cast<const float4*>(smid[sub]);
      const float x = u[i];
      jj[q] = (x > md.x ? 1u : 0u) + (x > md.y ? 1u : 0u) + (x > md.z ? 1u : 0u);
      bb[q] = (uint32_t)beta;
      s = pred;
    }
    const uint32_t field = jj[0] | (jj[1] << JW) | (bb[0] << (2 * JW)) | (bb[1] << (2 * JW + 1));
    const int bit = FW * k, wi = bit >> 5, sh = bit & 31;
    out[wi] |= field << sh;
    if (sh + FW > 32) out[wi + 1] |= field >> (32 - sh);
  }

  const size_t dst = ((size_t)bh * p.seq_cap + pos) * nb + blk;
  uint4* cd = reinterpret_cast<uint4*>(p.codes[1] + dst * (16 * BITS));
#pragma unroll
  for (int c = 0; c < NW / 4; ++c) cd[c] = make_uint4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
  const __half hn = __float2half_rn(my_norm);
  if (__hisinf(hn) && p.status) atomicOr(p.status, TQ_DEV_NORM_OVERFLOW);
  p.norms[1][dst] = __half_as_ushort(__hisinf(hn) ? __float2half_rn(65504.0f) : hn);
}

template <int BITS, bool F16>
int launch_v2_typed(const EncodeParams& p, cudaStream_t stream) {
  const long long items = (long long)p.batch * p.kv_heads * p.seq_new * (p.head_dim / kBlock);
  if (items >= (1LL << 31)) return TQ_ERR_UNSUPPORTED;  // 32-bit index splits in the kernel
  const long long ctas = (items + kV2Threads - 1) / kV2Threads;
  encode_v2_kernel<BITS, F16><<<(unsigned)ctas, kV2Threads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace

int launch_encode_v2(const EncodeParams& p, cudaStream_t stream) {
  if (p.seq_new == 0 || p.batch == 0) return TQ_OK;
  switch (p.bits[1] * 2 + (p.f16 ? 1 : 0)) {
    case 4: return launch_v2_typed<2, false>(p, stream);
    case 5: return launch_v2_typed<2, true>(p, stream);
    case 6: return launch_v2_typed<3, false>(p, stream);
    case 7: return launch_v2_typed<3, true>(p, stream);
    default: return TQ_ERR_UNSUPPORTED;
  }
}

}  // namespace tq
