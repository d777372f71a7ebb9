// Encoder kernel: sign flip, fast Walsh-Hadamard transform, fp16 block norm,
// Lloyd-Max quantisation and bit packing of 128-element KV blocks.
//
// Method: "TheTom/llama-cpp-turboquant" README, table "量化类型" (WHT rotation
// then codebook quantisation on 128-element blocks); intelliparadigm
// TurboQuant article §3.2 (H_random from a random +-1 diagonal and the
// Hadamard matrix, fast transform in O(d log d)) and §3.3 (Lloyd-Max).
//
// Mapping: two lanes per 128-block.  The block is 16 chunks of 8 elements;
// lane h holds chunks 2c + h (c = 0..7) as 32 float2 registers, so a lane
// pair reads 32 contiguous bytes per fp16 load.  The butterfly stages commute,
// so the six whose partners share a lane run in registers (five of them on
// packed f32x2 arithmetic) and the stride-8 stage pairs the two lanes through
// one shuffle per element.  Lane 0 stores chunks 0..7 of the packed bitstream
// and lane 1 chunks 8..15 (8*b bytes each, plain vector stores) after the
// pair swaps four chunk words.  For fp16 input the random signs are applied
// to the fp16 sign bits as the elements are converted (one XOR per pair).

#include <cuda_fp16.h>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kEncThreads = 256;

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// Apply the sign of element i: bit i of the 64-bit mask set means s_i = -1.
__device__ __forceinline__ float apply_sign(float x, uint32_t word, int bit) {
  return __uint_as_float(__float_as_uint(x) ^ ((word << (31 - bit)) & 0x80000000u));
}

template <int BITS>
__device__ __forceinline__ void store_codes(uint8_t* dst, const uint32_t (&w)[2 * BITS]) {
  if constexpr (BITS == 4) {
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if constexpr (BITS == 3) {
    uint2* d = reinterpret_cast<uint2*>(dst);
    d[0] = make_uint2(w[0], w[1]);
    d[1] = make_uint2(w[2], w[3]);
    d[2] = make_uint2(w[4], w[5]);
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int BITS, bool F16, int SIDE, bool OUTL>
__device__ __forceinline__ void encode_side(const EncodeParams& p, uint32_t* warp_signs) {
  constexpr int L = 1 << BITS;
  constexpr int NPOS = L / 2 - 1;  // positive decision boundaries
  const void* in = p.in[SIDE];
  const int lane = threadIdx.x & 31;
  const int h = lane & 1;
  const int nb = p.head_dim / kBlock;
  const long long n_blocks = (long long)p.batch * p.kv_heads * p.seq_new * nb;
  const long long blk = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 1;
  const bool valid = blk < n_blocks;

  int b = 0, j = 0, t = 0;
  long long row = 0, bh = 0;
  if (valid) {
    j = (int)(blk % nb);
    row = blk / nb;
    t = (int)(row % p.seq_new);
    bh = row / p.seq_new;
    b = (int)(bh / p.kv_heads);
  }
  int pos = t;
  if (valid && p.start_pos) pos += __ldg(p.start_pos + b);
  const bool ok = valid && pos >= 0 && pos < p.seq_cap;
  if (valid && !ok && h == 0 && p.status) atomicOr(p.status, TQ_DEV_POS_RANGE);

  // ---- load 64 elements (E1), convert to fp32 --------------------------
  float2 x[32];
  if constexpr (F16) {
    // chunk 2c + h of the block (8 elements, 16 B): a lane pair reads 32
    // contiguous bytes per load
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __half*>(in) +
                                                      (row * p.head_dim + j * kBlock)) + h;
    uint4 raw[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) raw[c] = ok ? __ldcs(src + 2 * c) : make_uint4(0, 0, 0, 0);
    // s o x (E1) on the fp16 bits, one mask word per element pair: word m of
    // lane half hh covers elements i, i+1 with i = 16(m/4) + 8hh + 2(m%4),
    // s_i in bit 15 and s_(i+1) in bit 31.  Each warp builds its own copy
    // while its loads are in flight.
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = 16 * (lane >> 2) + 8 * hh + 2 * (lane & 3);
      const uint32_t wd = p.sign_mask[i >> 5];
      const int bit = i & 31;
      warp_signs[hh * 32 + lane] = (((wd >> bit) & 1u) << 15) | (((wd >> (bit + 1)) & 1u) << 31);
    }
    __syncwarp();
    const uint4* sgn = reinterpret_cast<const uint4*>(warp_signs + 32 * h);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = raw[c];
      const uint4 mk = sgn[c];
      const uint32_t wv[4] = {v.x ^ mk.x, v.y ^ mk.y, v.z ^ mk.z, v.w ^ mk.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 hv = *reinterpret_cast<const __half2*>(&wv[e]);
        x[c * 4 + e] = __half22float2(hv);
      }
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(in) +
                                                        (row * p.head_dim + j * kBlock + 8 * h));
#pragma unroll
    for (int c = 0; c < 8; ++c) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float4 v = ok ? __ldcs(src + 4 * c + q) : make_float4(0.f, 0.f, 0.f, 0.f);
        x[4 * c + 2 * q] = make_float2(v.x, v.y);
        x[4 * c + 2 * q + 1] = make_float2(v.z, v.w);
      }
    }
  }

  // ---- V v3: the outlier channels of this block are zeroed before the norm
  // and the transform (their values are stored exactly, below) -------------
  if constexpr (OUTL) {
    const int kvh = (int)(bh % p.kv_heads);
    uint32_t bm[4] = {0u, 0u, 0u, 0u};  // block mask: bit i <=> channel 128 j + i
    for (int t = 0; t < p.vo_k; ++t) {
      const int ch = __ldg(p.vo_channels + (size_t)kvh * p.vo_k + t) - kBlock * j;
      if (ch >= 0 && ch < kBlock) {
        const uint32_t bit = 1u << (ch & 31);
        const int wsel = ch >> 5;
        bm[0] |= wsel == 0 ? bit : 0u;
        bm[1] |= wsel == 1 ? bit : 0u;
        bm[2] |= wsel == 2 ? bit : 0u;
        bm[3] |= wsel == 3 ? bit : 0u;
      }
    }
    // element e of the lane's chunk c is i = 16c + 8h + e: byte 2c + h of bm
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t zb = (bm[c >> 1] >> (16 * (c & 1) + 8 * h)) & 0xFFu;
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        if ((zb >> e) & 1u) x[4 * c + e / 2].x = 0.0f;
        if ((zb >> (e + 1)) & 1u) x[4 * c + e / 2].y = 0.0f;
      }
    }
    // the lane pair of the vector's first block writes the values row:
    // entry t = V[channels[kvh][t]] for t < k, 0 up to the padded width
    if (j == 0 && ok) {
      const size_t row_in = (size_t)row * p.head_dim;
      uint16_t* dst = p.vo_values + ((size_t)bh * p.seq_cap + pos) * p.vo_kp;
      for (int t = h; t < p.vo_kp; t += 2) {
        __half val = __float2half_rn(0.0f);
        if (t < p.vo_k) {
          const int ch = __ldg(p.vo_channels + (size_t)kvh * p.vo_k + t);
          if (ch >= 0 && ch < p.head_dim) {
            val = F16 ? static_cast<const __half*>(in)[row_in + ch]
                      : __float2half_rn(static_cast<const float*>(in)[row_in + ch]);
          } else if (p.status) {
            atomicOr(p.status, TQ_DEV_CHANNEL_RANGE);
          }
        }
        dst[t] = __half_as_ushort(val);
      }
    }
  }

  // ---- norm (E3): 8 partial sums then a tree, then across the lane pair --
  float2 acc[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) acc[a] = __fmul2_rn(x[a], x[a]);
#pragma unroll
  for (int m = 4; m < 32; ++m) acc[m & 3] = __ffma2_rn(x[m], x[m], acc[m & 3]);
  float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
  float2 s = __fadd2_rn(s01, s23);
  float ss = s.x + s.y;
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  const float n = __fsqrt_rn(ss);

  // ---- sign flip (E1): s o x (fp32 input; fp16 input was flipped on load)
  if constexpr (!F16) {
    // element (c, e) of the lane is i = 16c + 8h + e: sign word c/2, bit
    // 16(c%2) + 8h + e
    uint32_t sw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) sw[q] = p.sign_mask[q] >> (8 * h);
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      const int c = m >> 2, bit = 16 * (c & 1) + 2 * (m & 3);
      x[m].x = apply_sign(x[m].x, sw[c >> 1], bit);
      x[m].y = apply_sign(x[m].y, sw[c >> 1], bit + 1);
    }
  }

  // ---- fast WHT (E2): 7 unnormalised butterfly stages ---------------------
#pragma unroll
  for (int m = 0; m < 32; ++m) x[m] = make_float2(x[m].x + x[m].y, x[m].x - x[m].y);
#pragma unroll
  for (int sp = 1; sp < 32; sp <<= 1) {  // element strides 2..32 = float2 strides 1..16
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      if ((m & sp) == 0) {
        const float2 a = x[m], c = x[m + sp];
        x[m] = __fadd2_rn(a, c);
        x[m + sp] = sub2(a, c);
      }
    }
  }
  {  // stride 8: the partner lane holds the other chunks of the block.
    const float sg = h ? -1.0f : 1.0f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      float2 o;
      o.x = __shfl_xor_sync(0xffffffffu, x[m].x, 1);
      o.y = __shfl_xor_sync(0xffffffffu, x[m].y, 1);
      x[m] = __ffma2_rn(sg2, x[m], o);  // h=0: x + o ; h=1: o - x
    }
  }

  // ---- quantise (E4): idx = #{boundaries < y / n} -------------------------
  // With symmetric boundaries {-T_k} U {0} U {T_k}, for y > 0 the count is
  // L/2 + #{T_k < |y|/n}; for y <= 0 it is L/2 - 1 - #{T_k < |y|/n} (an exact
  // tie at a negative boundary is the only case where this differs from the
  // strict count, by one, and only on the boundary itself).  Comparing |y|
  // against T_k * n avoids a division.
  float thr[NPOS > 0 ? NPOS : 1];
#pragma unroll
  for (int k = 0; k < NPOS; ++k) thr[k] = p.pos_bounds[SIDE][k] * n;

  // Codes of the lane's chunk c (8 codes, 8*BITS bits) in g[c]; chunk c of
  // lane h is chunk 2c + h of the block.
  uint32_t g[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) g[c] = 0;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float y = (i & 1) ? x[i >> 1].y : x[i >> 1].x;
    const float a = fabsf(y);
    // m = #{k : T_k < |y|/n}, found by bisection of the ascending T_k
    int m;
    if constexpr (NPOS == 1) {
      m = (a > thr[0]) ? 1 : 0;
    } else if constexpr (NPOS == 3) {
      const int c1 = (a > thr[1]) ? 1 : 0;
      m = 2 * c1 + ((a > (c1 ? thr[2] : thr[0])) ? 1 : 0);
    } else {
      const int c2 = (a > thr[3]) ? 1 : 0;
      const int c1 = (a > (c2 ? thr[5] : thr[1])) ? 1 : 0;
      const float t0 = c2 ? (c1 ? thr[6] : thr[4]) : (c1 ? thr[2] : thr[0]);
      m = 4 * c2 + 2 * c1 + ((a > t0) ? 1 : 0);
    }
    const int lowside = L / 2 - 1 - m;
    const uint32_t idx = (uint32_t)(y > 0.0f ? (lowside ^ (L - 1)) : lowside);
    g[i >> 3] |= idx << (BITS * (i & 7));
  }
  // ---- pack (E5): LSB-first bitstream.  Lane 0 stores chunks 0..7, lane 1
  // chunks 8..15; the pair swaps the four chunk words each needs.
  uint32_t grp[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t r = __shfl_xor_sync(0xffffffffu, h ? g[q] : g[4 + q], 1);
    grp[2 * q] = h ? r : g[q];
    grp[2 * q + 1] = h ? g[4 + q] : r;
  }
  uint32_t w[2 * BITS];
#pragma unroll
  for (int k = 0; k < 2 * BITS; ++k) w[k] = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int bit = 8 * BITS * q;
    const int wi = bit >> 5, sh = bit & 31;
    w[wi] |= grp[q] << sh;
    if (sh + 8 * BITS > 32) w[wi + 1] |= grp[q] >> (32 - sh);
  }

  if (ok) {
    const long long cache_blk = ((bh * p.seq_cap) + pos) * nb + j;
    store_codes<BITS>(p.codes[SIDE] + cache_blk * (16 * BITS) + 8 * BITS * h, w);
    if (h == 0) {
      __half nh = __float2half_rn(n);
      if (__hisinf(nh)) {
        nh = __ushort_as_half((unsigned short)0x7BFF);
        if (p.status) atomicOr(p.status, TQ_DEV_NORM_OVERFLOW);
      }
      p.norms[SIDE][cache_blk] = __half_as_ushort(nh);
    }
  }
}

template <int KB, int VB, bool F16, bool OUTL>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(const __grid_constant__ EncodeParams p) {
  __shared__ __align__(16) uint32_t signs[kEncThreads / 32][64];  // per-warp fp16 sign masks
  uint32_t* ws = signs[threadIdx.x >> 5];
  if (blockIdx.y == 0) {
    if (p.in[0]) encode_side<KB, F16, 0, false>(p, ws);
  } else {
    if (p.in[1]) encode_side<VB, F16, 1, OUTL>(p, ws);
  }
}

template <int KB, int VB>
int launch_kb_vb(const EncodeParams& p, cudaStream_t stream) {
  const long long n_blocks = (long long)p.batch * p.kv_heads * p.seq_new * (p.head_dim / kBlock);
  const long long threads = n_blocks * 2;
  const long long grid_x = (threads + kEncThreads - 1) / kEncThreads;
  if (grid_x > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
  dim3 grid((unsigned)grid_x, 2);
  const bool outl = p.vo_k > 0 && p.in[1] != nullptr;
  if (p.f16) {
    if (outl) encode_kernel<KB, VB, true, true><<<grid, kEncThreads, 0, stream>>>(p);
    else encode_kernel<KB, VB, true, false><<<grid, kEncThreads, 0, stream>>>(p);
  } else {
    if (outl) encode_kernel<KB, VB, false, true><<<grid, kEncThreads, 0, stream>>>(p);
    else encode_kernel<KB, VB, false, false><<<grid, kEncThreads, 0, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int KB>
int launch_kb(const EncodeParams& p, cudaStream_t stream) {
  // A side that is not encoded keeps a valid bit width from the descriptor.
  switch (p.bits[1]) {
    case 2: return launch_kb_vb<KB, 2>(p, stream);
    case 3: return launch_kb_vb<KB, 3>(p, stream);
    case 4: return launch_kb_vb<KB, 4>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace

int launch_encode(const EncodeParams& p, cudaStream_t stream) {
  switch (p.bits[0]) {
    case 2: return launch_kb<2>(p, stream);
    case 3: return launch_kb<3>(p, stream);
    case 4: return launch_kb<4>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
