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
//
// The grid is persistent (as many CTAs as fit, split between K and V); each
// lane pair walks blocks with a grid stride and copies the next block into a
// per-warp staging area with cp.async while it transforms the current one,
// so the loads stay in flight through the arithmetic.

#include <cuda_fp16.h>

#include <algorithm>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kEncThreads = 128;

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

// 16-byte chunks a lane copies per block: fp16 8, fp32 16.  Staging of one
// warp: 2 stages x chunks x 32 lanes x 16 B, chunk c of lane l at (c * 32 + l) * 16.
template <bool F16>
__host__ __device__ constexpr int lane_chunks() { return F16 ? 8 : 16; }
template <bool F16>
__host__ __device__ constexpr uint32_t stage_bytes() { return (uint32_t)lane_chunks<F16>() * 32 * 16; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ uint4 ld_shared16(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// The lane's chunks of block blk into staging `st` (one commit group; an
// empty group past the end keeps the waits counting right).
template <bool F16>
__device__ __forceinline__ void stage_block(const EncodeParams& p, const void* in, uint32_t blk, uint32_t n_blocks,
                                            uint32_t st, int lane) {
  if (blk < n_blocks) {
    const int nb = p.head_dim / kBlock;
    const int lnb = nb == 1 ? 0 : nb == 2 ? 1 : 2;  // nb is 1, 2 or 4
    const size_t base = (size_t)(blk >> lnb) * p.head_dim + (size_t)(blk & (nb - 1)) * kBlock + 8 * (lane & 1);
#pragma unroll
    for (int c = 0; c < lane_chunks<F16>(); ++c) {
      // fp16: chunk c is elements 16c + 8h .. +7; fp32: half c & 1 of that chunk for c / 2
      const void* src = F16 ? static_cast<const void*>(static_cast<const __half*>(in) + base + 16 * c)
                            : static_cast<const void*>(static_cast<const float*>(in) + base + 16 * (c >> 1) + 4 * (c & 1));
      cp_async16(st + (uint32_t)(c * 32 + lane) * 16u, src);
    }
  }
  cp_async_commit();
}

template <int BITS, bool F16, int SIDE, bool OUTL>
__device__ __forceinline__ void encode_block(const EncodeParams& p, const uint32_t* warp_signs, uint32_t blk,
                                             uint32_t n_blocks, uint32_t st) {
  constexpr int L = 1 << BITS;
  constexpr int NPOS = L / 2 - 1;  // positive decision boundaries
  const void* in = p.in[SIDE];
  const int lane = threadIdx.x & 31;
  const int h = lane & 1;
  const int nb = p.head_dim / kBlock;
  // the host keeps the flattened block count below 2^31: 32-bit index math,
  // divisions by multiply-high (a 64-bit division is a long subroutine)
  const bool valid = blk < n_blocks;

  int b = 0, j = 0, t = 0;
  long long row = 0, bh = 0;
  if (valid) {
    const int lnb = nb == 1 ? 0 : nb == 2 ? 1 : 2;  // nb is 1, 2 or 4
    j = (int)(blk & (nb - 1));
    const uint32_t r32 = blk >> lnb;
    const uint32_t bh32 = p.div_seq_new.div(r32);
    t = (int)(r32 - bh32 * (uint32_t)p.seq_new);
    b = (int)p.div_kv_heads.div(bh32);
    row = r32;
    bh = bh32;
  }
  int pos = t;
  if (valid && p.start_pos) pos += __ldg(p.start_pos + b);
  const bool ok = valid && pos >= 0 && pos < p.seq_cap;
  if (valid && !ok && h == 0 && p.status) atomicOr(p.status, TQ_DEV_POS_RANGE);

  // ---- load 64 elements (E1), convert to fp32 --------------------------
  float2 x[32];
  if constexpr (F16) {
    // chunk 2c + h of the block (8 elements, 16 B), staged by this lane
    uint4 raw[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) raw[c] = valid ? ld_shared16(st + (uint32_t)(c * 32 + lane) * 16u) : make_uint4(0, 0, 0, 0);
    // s o x (E1) on the fp16 bits (the per-warp mask words, see encode_kernel)
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
#pragma unroll
    for (int c = 0; c < 8; ++c) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint4 u = valid ? ld_shared16(st + (uint32_t)((2 * c + q) * 32 + lane) * 16u) : make_uint4(0, 0, 0, 0);
        const float4 v = make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                                     __uint_as_float(u.w));
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
  // lane h is chunk 2c + h of the block.  With m = #{T_k < |y|/n}, the code is
  // L/2 - 1 - m = (L/2 - 1) ^ m for y <= 0 and L/2 + m = (L/2 - 1) ^ m ^ (L - 1)
  // for y > 0, so every field starts at L/2 - 1 and each decision bit of the
  // bisection, and the sign, toggles bits of it in place.
  constexpr uint32_t kNeg = (uint32_t)(L / 2 - 1) * (BITS == 2 ? 0x5555u : BITS == 3 ? 0x249249u : 0x11111111u);
  uint32_t g[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) g[c] = kNeg;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float y = (i & 1) ? x[i >> 1].y : x[i >> 1].x;
    const float a = fabsf(y);
    const int sh = BITS * (i & 7);
    uint32_t& gw = g[i >> 3];
    // m = #{k : T_k < |y|/n}, by bisection of the ascending T_k
    if constexpr (NPOS == 1) {
      if (a > thr[0]) gw ^= 1u << sh;
    } else if constexpr (NPOS == 3) {
      const bool c1 = a > thr[1];
      if (c1) gw ^= 2u << sh;
      if (a > (c1 ? thr[2] : thr[0])) gw ^= 1u << sh;
    } else {
      const bool c2 = a > thr[3];
      const bool c1 = a > (c2 ? thr[5] : thr[1]);
      const float t0 = c2 ? (c1 ? thr[6] : thr[4]) : (c1 ? thr[2] : thr[0]);
      if (c2) gw ^= 4u << sh;
      if (c1) gw ^= 2u << sh;
      if (a > t0) gw ^= 1u << sh;
    }
    if (y > 0.0f) gw ^= (uint32_t)(L - 1) << sh;
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

template <int BITS, bool F16, int SIDE, bool OUTL>
__device__ __forceinline__ void encode_side(const EncodeParams& p, const uint32_t* ws, uint32_t st0,
                                            uint32_t n_blocks, uint32_t cta, uint32_t ctas) {
  const int lane = threadIdx.x & 31;
  // lane pairs walk the blocks with a stride of this side's lane pairs; the
  // warp stays together (its pairs are consecutive) so the loop is warp-uniform
  const uint32_t pairs = (ctas * blockDim.x) >> 1;
  const uint32_t warp0 = (cta * blockDim.x + (threadIdx.x & ~31u)) >> 1;
  const uint32_t mine = lane >> 1;
  if (warp0 >= n_blocks) return;
  stage_block<F16>(p, p.in[SIDE], warp0 + mine, n_blocks, st0, lane);
  uint32_t s = 0;
  for (uint32_t base = warp0; base < n_blocks; base += pairs) {
    stage_block<F16>(p, p.in[SIDE], base + pairs + mine, n_blocks, st0 + (s ^ 1u) * stage_bytes<F16>(), lane);
    cp_async_wait1();  // this lane's chunks of the current block have landed
    encode_block<BITS, F16, SIDE, OUTL>(p, ws, base + mine, n_blocks, st0 + s * stage_bytes<F16>());
    s ^= 1u;
  }
}

template <int KB, int VB, bool F16, bool OUTL>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(const __grid_constant__ EncodeParams p) {
  __shared__ __align__(16) uint32_t signs[kEncThreads / 32][64];  // per-warp fp16 sign masks
  extern __shared__ __align__(16) uint8_t stage[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* ws = signs[warp];
  if constexpr (F16) {
    // sign mask words for s o x on the fp16 bits: word m of lane half hh
    // covers elements i, i+1 with i = 16(m/4) + 8hh + 2(m%4), s_i in bit 15
    // and s_(i+1) in bit 31
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = 16 * (lane >> 2) + 8 * hh + 2 * (lane & 3);
      const uint32_t wd = p.sign_mask[i >> 5];
      const int bit = i & 31;
      ws[hh * 32 + lane] = (((wd >> bit) & 1u) << 15) | (((wd >> (bit + 1)) & 1u) << 31);
    }
    __syncwarp();
  }
  const uint32_t st0 = (uint32_t)__cvta_generic_to_shared(stage) + (uint32_t)warp * 2u * stage_bytes<F16>();
  const uint32_t n_blocks = (uint32_t)p.batch * p.kv_heads * p.seq_new * (p.head_dim / kBlock);
  // the first k_ctas CTAs encode K, the rest V (k_ctas = 0: V only; all: K only)
  const uint32_t kc = p.k_ctas;
  if (blockIdx.x < kc) encode_side<KB, F16, 0, false>(p, ws, st0, n_blocks, blockIdx.x, kc);
  else encode_side<VB, F16, 1, OUTL>(p, ws, st0, n_blocks, blockIdx.x - kc, gridDim.x - kc);
}

// Instructions per element by code width, for splitting the CTAs between K
// and V in proportion to their work: the transform, loads and packing (about
// 12) plus the quantiser's compares and bit toggles.
inline int side_cost(int bits) { return 12 + (bits == 2 ? 4 : bits == 3 ? 7 : 11); }

// Persistent launch: as many CTAs as are resident at once, split between the
// sides in proportion to their work, at most one lane pair per block.
template <typename K>
int launch_typed(K kern, uint32_t stage, EncodeParams p, long long n_blocks, cudaStream_t stream) {
  const size_t smem = (size_t)(kEncThreads / 32) * 2 * stage;
  int dev = 0, sms = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kEncThreads, smem) != cudaSuccess) return TQ_ERR_CUDA;
  if (occ < 1) return TQ_ERR_UNSUPPORTED;
  const long long needed = (n_blocks * 2 + kEncThreads - 1) / kEncThreads;  // CTAs one side can use
  const long long resident = (long long)occ * sms;
  long long kc = 0, vc = 0;
  if (p.in[0] && p.in[1]) {
    const int ck = side_cost(p.bits[0]), cv = side_cost(p.bits[1]);
    kc = std::max(1LL, std::min(resident - 1, (resident * ck + (ck + cv) / 2) / (ck + cv)));
    vc = std::max(1LL, resident - kc);
  } else if (p.in[0]) {
    kc = resident;
  } else {
    vc = resident;
  }
  kc = std::min(kc, needed);
  vc = std::min(vc, needed);
  p.k_ctas = (uint32_t)kc;
  kern<<<(unsigned)(kc + vc), kEncThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int KB, int VB>
int launch_kb_vb(const EncodeParams& p, cudaStream_t stream) {
  const long long n_blocks = (long long)p.batch * p.kv_heads * p.seq_new * (p.head_dim / kBlock);
  if (n_blocks >= (1LL << 31)) return TQ_ERR_UNSUPPORTED;  // 32-bit index math in the kernel
  const bool outl = p.vo_k > 0 && p.in[1] != nullptr;
  if (p.f16) {
    if (outl) return launch_typed(encode_kernel<KB, VB, true, true>, stage_bytes<true>(), p, n_blocks, stream);
    return launch_typed(encode_kernel<KB, VB, true, false>, stage_bytes<true>(), p, n_blocks, stream);
  }
  if (outl) return launch_typed(encode_kernel<KB, VB, false, true>, stage_bytes<false>(), p, n_blocks, stream);
  return launch_typed(encode_kernel<KB, VB, false, false>, stage_bytes<false>(), p, n_blocks, stream);
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
