// Decode attention over the packed TurboQuant cache (one query token per
// sequence, GQA, per-sequence lengths, optional exact sparse-V).
//
// Method: "llama-tq" article, K-cache section (Q.K in the Hadamard domain,
// no K dequantisation); "TheTom/llama-cpp-turboquant" README, table "量化类型"
// (WHT + codebook on 128-element blocks) and "压缩策略" (sparse-V dequant);
// "TurboQuant+" section "注意力门控稀疏V解压" (skipped V counts as zero).
//
// Kernel design (sm_100a):
//  * Work = (unit, 16-token tile), unit = (batch, kv-head, group of <= 8
//    q-heads).  All tiles of all units are laid end to end and cut into one
//    range per persistent CTA, one 16-warp CTA per SM.  The cut weighs each
//    tile 1 and each unit start kSwitchTiles more, so CTAs whose range spans
//    two units get fewer tiles (see Split).  A CTA writes one partial
//    (m, l, acc) per unit it touches; the CTA that completes a unit (atomic
//    tile count) merges the partials in a fixed order and applies the inverse
//    rotation, so results do not depend on scheduling.
//  * Each warp streams its own future tiles (packed K and V codes and their
//    fp16 norms) into a private shared-memory ring with 16-byte cp.async
//    (zero-filled past the end of the sequence) and waits for them with
//    cp.async.wait_group, so several tiles per warp are in flight without
//    holding registers, and no warp waits on another.
//  * Scores: S[16 tok x 8 cols] = Kc[16 x 128] . Qhat[128 x 8] with
//    mma.sync m16n8k16 (f16 in, f32 accumulate).  K codes are turned into f16
//    A fragments in registers through a shared-memory table indexed by two
//    codes and replicated per lane (conflict-free).  Contraction order is
//    permuted so each lane's fragment comes from 32 contiguous codes.
//  * Online softmax in the log2 domain with a lazy rescale (only when the
//    running max grows by more than 2^6), exact because the stored max is the
//    one every exponent used.
//  * P.V with up to four q-heads per kv-head (GQ = 4): the 8 MMA columns are
//    (head, dim parity) pairs, so each V A-fragment register is one token's
//    pair of adjacent dims straight from the table.  With more heads (GQ = 8)
//    O^T[128 dims x 8 heads] += Vc^T[dims x 16 tok] . P'^T[16 tok x 8] with V
//    re-paired by token.  P' = p * nV / 128 reaches the B fragment through two
//    movmatrix transposes.  V stays in the rotated domain until the end.
//  * Sparse-V is exact and two-pass: pass 1 stores log2-domain scores and
//    per-partial (m, l); pass 2 forms the log-sum-exp, zeroes the normalised
//    weights below the threshold and accumulates V with the rest.
//  * Decode step: given the new token's K/V rows, the CTA holding a unit's
//    last tile first encodes them into the cache (append_block).

#include <cuda_fp16.h>

#include <type_traits>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

#ifndef TQ_DECODE_WARPS
#define TQ_DECODE_WARPS 16
#endif
#ifndef TQ_DECODE_MIN_CTAS
#define TQ_DECODE_MIN_CTAS 1
#endif
#ifndef TQ_DECODE_MIN_CTAS_WIDE  // head_dim 256 kernels
#define TQ_DECODE_MIN_CTAS_WIDE (TQ_DECODE_MIN_CTAS > 2 ? 2 : TQ_DECODE_MIN_CTAS)
#endif
#ifndef TQ_KCHAINS
#define TQ_KCHAINS 2  // independent accumulator chains of the score MMAs
#endif
#ifndef TQ_SWITCH_TILES
#define TQ_SWITCH_TILES 96  // cost of starting another unit inside a CTA, in tiles
#endif
#ifndef TQ_RING_DEPTH
#define TQ_RING_DEPTH 4
#endif
constexpr int kKChains = TQ_KCHAINS;
constexpr int kCWarps = TQ_DECODE_WARPS;        // warps per CTA
constexpr int kCThreads = 32 * kCWarps;
constexpr int kThreads = kCThreads;
constexpr int kRingDepth = TQ_RING_DEPTH;       // tiles per warp ring (all in flight), at most
constexpr int kMaxSmem = 227 * 1024;            // shared memory of one CTA (static + dynamic)
constexpr float kTau = 6.0f;                    // lazy-rescale threshold (log2 units)
constexpr int kMergeChunk = 64;                 // partials merged per pass of the final merge

enum Mode { kFused = 0, kScores = 1, kSparseV = 2 };

// ----------------------------------------------------------------- helpers --

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  return __byte_perm(a, b, sel);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory loads on 32-bit shared-window addresses (volatile: they are
// ordered with the asynchronous copies and barriers around them).
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
  uint32_t x;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(x) : "r"(a));
  return x;
}
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
  uint2 x;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(x.x), "=r"(x.y) : "r"(a));
  return x;
}
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
  uint4 x;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "r"(a));
  return x;
}

// Table read.  Not volatile: the tables do not change after the prologue, and
// every address depends on code words read (volatile, after the copy waits)
// from the ring, so the compiler may schedule these freely, e.g. ahead of the
// softmax that precedes their use.
__device__ __forceinline__ uint32_t ld_table(uint32_t a) {
  uint32_t x;
  asm("ld.shared.b32 %0, [%1];" : "=r"(x) : "r"(a));
  return x;
}

// Lane-replicated table lookup.  The table holds, for every value of a field
// of `fb` bits (two codes), one 4-byte entry per lane: entry f of lane l sits
// at table + f*128 + l*4, so the 32 lanes always hit 32 different banks.
// `lb` is table + lane*4.  When the table is aligned to its own size the
// field bits can be OR-ed into lb (ALIGNED); otherwise they are added.  The
// field is the one at bit `pos` of the word array w; pos and fb are
// compile-time after unrolling, so exactly one of the forms below is emitted:
// a shift and one three-input logic op (plus an add when not ALIGNED), or a
// funnel shift for a field that crosses a word boundary.
template <bool ALIGNED>
__device__ __forceinline__ uint32_t lut_get(const uint32_t* w, int pos, int fb, uint32_t lb) {
  const int wi = pos >> 5, sh = pos & 31;
  const uint32_t mask = ((1u << fb) - 1u) << 7;
  uint32_t a;
  if (sh + fb > 32) {
    const uint32_t v = __funnelshift_r(w[wi], w[wi + 1], sh) << 7;
    a = ALIGNED ? ((v & mask) | lb) : ((v & mask) + lb);
  } else if (sh >= 7) {
    if (ALIGNED)
      asm("{ .reg .b32 t; shr.b32 t, %1, %2; and.b32 t, t, %3; or.b32 %0, t, %4; }"
          : "=r"(a) : "r"(w[wi]), "r"(sh - 7), "r"(mask), "r"(lb));
    else
      asm("{ .reg .b32 t; shr.b32 t, %1, %2; and.b32 t, t, %3; add.u32 %0, t, %4; }"
          : "=r"(a) : "r"(w[wi]), "r"(sh - 7), "r"(mask), "r"(lb));
  } else {
    if (ALIGNED)
      asm("{ .reg .b32 t; shl.b32 t, %1, %2; and.b32 t, t, %3; or.b32 %0, t, %4; }"
          : "=r"(a) : "r"(w[wi]), "r"(7 - sh), "r"(mask), "r"(lb));
    else
      asm("{ .reg .b32 t; shl.b32 t, %1, %2; and.b32 t, t, %3; add.u32 %0, t, %4; }"
          : "=r"(a) : "r"(w[wi]), "r"(7 - sh), "r"(mask), "r"(lb));
  }
  return ld_table(a);
}

// ---------------------------------------------------------- async copies --

// 16-byte global -> shared copy; src_bytes < 16 zero-fills the rest (0: no read).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

// 4-byte global -> shared copy with the same zero-fill rule.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void consumer_sync() { __syncthreads(); }

template <int B>
struct Fmt {
  static constexpr int kEntries = 1 << (2 * B);
  static constexpr int kLutBytes = kEntries * 128;
  static constexpr int kBlockBytes = 16 * B;
};

// Token order inside a 16-token tile.  MMA row r of the score product holds
// token pi(r): pi(R) = 2R, pi(R + 8) = 2R + 1, so lane (R = lane/4, g = lane%4)
// holds the adjacent tokens 2R and 2R+1 (their norms are one 32-bit word).
// The P.V product then needs, in lane g, tokens pi(2g) = 4g, pi(2g+1) = 4g+2,
// pi(2g+8) = 4g+1 and pi(2g+9) = 4g+3 -- four adjacent tokens.
//
// Per lane and tile:
//   k[rr][blk]  : codes of dims [32g, 32g+32) of token 2R+rr (KB words);
//   v[tt][blk]  : codes of dims [16R, 16R+16) of token vtok(tt) (2 words);
//   kn, vn      : the fp16 norms of tokens 2R and 2R+1 (NB=1: one half2
//                 word; NB=2: one word per token holding both blocks).
template <int KB, int VB, int NB>
struct TileRegs {
  uint32_t k[2][NB][KB > 0 ? KB : 1];
  uint32_t v[4][NB][2];
  uint32_t kn[NB];
  uint32_t vn[NB];
};

// Code words of one tile from a ring slot.  ks / vs are the shared addresses
// of this lane's first K / V word in the slot.
template <int KB, int VB, int NB, bool LOADK, bool LOADV>
__device__ __forceinline__ void read_tile(TileRegs<KB, VB, NB>& r, uint32_t ks, uint32_t vs, int R) {
  if constexpr (LOADK) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const uint32_t s = ks + (rr * NB + blk) * Fmt<KB>::kBlockBytes;
        if constexpr (KB == 4) {
          const uint4 x = ld_s128(s);
          r.k[rr][blk][0] = x.x; r.k[rr][blk][1] = x.y; r.k[rr][blk][2] = x.z; r.k[rr][blk][3] = x.w;
        } else if constexpr (KB == 3) {
          r.k[rr][blk][0] = ld_s32(s); r.k[rr][blk][1] = ld_s32(s + 4); r.k[rr][blk][2] = ld_s32(s + 8);
        } else {
          const uint2 x = ld_s64(s);
          r.k[rr][blk][0] = x.x; r.k[rr][blk][1] = x.y;
        }
      }
  }
  if constexpr (LOADV) {
    const uint32_t vsh = (VB == 3 && (R & 1)) ? 16u : 0u;
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const int toff = ((tt & 1) << 1) + (tt >> 1);  // vtok(g, tt) - 4g
        const uint32_t s = vs + (toff * NB + blk) * Fmt<VB>::kBlockBytes;
        if constexpr (VB == 4) {
          const uint2 x = ld_s64(s);
          r.v[tt][blk][0] = x.x; r.v[tt][blk][1] = x.y;
        } else if constexpr (VB == 3) {
          const uint32_t w0 = ld_s32(s), w1 = ld_s32(s + 4);
          r.v[tt][blk][0] = __funnelshift_r(w0, w1, vsh);
          r.v[tt][blk][1] = w1 >> vsh;
        } else {
          r.v[tt][blk][0] = ld_s32(s);
          r.v[tt][blk][1] = 0u;
        }
      }
  }
}

// Norm words of tokens 2R and 2R+1 from a ring slot (see TileRegs).
template <int NB>
__device__ __forceinline__ void read_norms(uint32_t (&dst)[NB], uint32_t nbase, int R) {
  if constexpr (NB == 1) {
    dst[0] = ld_s32(nbase + 4 * R);
  } else {
    const uint2 x = ld_s64(nbase + 8 * R);
    dst[0] = x.x;
    dst[1] = x.y;
  }
}

// Norms of tokens 2R (x) and 2R+1 (y) for block blk, as fp32.
template <int NB>
__device__ __forceinline__ float2 norm_pair(const uint32_t (&w)[NB], int blk) {
  if constexpr (NB == 1) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w[0]));
  } else {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w[0]));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w[1]));
    return blk == 0 ? make_float2(a.x, b.x) : make_float2(a.y, b.y);
  }
}

// ----------------------------------------------------- shared-memory plan --

template <int KB, int VB, int NB, int MODE>
struct Smem {
  static constexpr int D = NB * kBlock;
  static constexpr bool kHasK = MODE != kSparseV;
  static constexpr bool kHasV = MODE != kScores;
  static constexpr int kLutK = kHasK ? Fmt<KB>::kLutBytes : 0;
  static constexpr int kLutV = kHasV ? Fmt<VB>::kLutBytes : 0;
  // Tables of up to 8 KB live in static shared memory with room to place them
  // at an address aligned to their own size (field bits then OR into the
  // address); a larger table lives unaligned in dynamic shared memory.
  static constexpr bool kAlignK = kLutK <= 8192;
  static constexpr bool kAlignV = kLutV <= 8192;
  // Both aligned tables share one static array: the larger one first, at an
  // address aligned to its size; the smaller follows (still aligned, since
  // the sizes are powers of two).  Slack: the larger size.
  static constexpr int kAK = (kAlignK && kLutK) ? kLutK : 0;
  static constexpr int kAV = (kAlignV && kLutV) ? kLutV : 0;
  static constexpr int kAMax = kAK > kAV ? kAK : kAV;
  static constexpr int kRawLut = (kAK + kAV) ? kAK + kAV + kAMax : 16;
  static constexpr bool kKFirst = kAK >= kAV;
  static constexpr int kDynLut = (kAlignK ? 0 : kLutK) + (kAlignV ? 0 : kLutV);
  // One ring slot holds one tile: K codes, V codes, K norms, V norms.
  static constexpr int kSlotK = kHasK ? kTile * NB * Fmt<KB>::kBlockBytes : 0;
  static constexpr int kSlotV = kHasV ? kTile * NB * Fmt<VB>::kBlockBytes : 0;
  static constexpr int kSlotKN = kHasK ? kTile * NB * 2 : 0;
  static constexpr int kSlotVN = kHasV ? kTile * NB * 2 : 0;
  static constexpr int kOffSlotV = kSlotK;
  static constexpr int kOffSlotKN = kOffSlotV + kSlotV;
  static constexpr int kOffSlotVN = kOffSlotKN + kSlotKN;
  static constexpr int kSlotBytes = (kOffSlotVN + kSlotVN + 127) / 128 * 128;
  static constexpr int kWorkFloats = kCWarps * kMaxGroup * D;    // per-warp partials / qhat
  static constexpr int kResFloats = kMaxGroup * D;               // merged rotated-domain acc
  static constexpr int kOffLutK = 0;                       // dynamic, when not aligned
  static constexpr int kOffLutV = kAlignK ? 0 : kLutK;
  static constexpr int kOffRing = (kDynLut + 127) / 128 * 128;
  // misc: warp m/l [kCWarps][8] x2, merged M/L/lse [8] x3, qexp [8], warp
  // totals [16], flags [4], reduction scratch [kCThreads] x2, merge factors.
  static constexpr int kMiscFloats = 2 * kCWarps * kMaxGroup + 4 * kMaxGroup + 16 + 4 +
                                     2 * kCThreads + 2 * kMergeChunk * kMaxGroup;
  // Ring depth: kRingDepth tiles per warp when they fit next to everything
  // else (the batch prefix counted at its largest), fewer otherwise.
  static constexpr int kFixed = kRawLut + kOffRing + (kResFloats + kMiscFloats) * 4 + (kMaxBatch + 1) * 4;
  static constexpr int kFit = (kMaxSmem - kFixed) / (kCWarps * kSlotBytes);
  static constexpr int kDepth = kFit >= kRingDepth ? kRingDepth : (kFit < 1 ? 1 : kFit);
  // The warp partials and the query scratch reuse the ring: the ring is empty
  // (every copy waited for) whenever they are in use.
  static constexpr int kRingBytes = kCWarps * kDepth * kSlotBytes;
  static constexpr int kRingArea = kRingBytes > kWorkFloats * 4 ? kRingBytes : kWorkFloats * 4;
  static constexpr int kOffWork = kOffRing;
  static constexpr int kOffRes = kOffRing + kRingArea;
  static constexpr int kOffMisc = kOffRes + kResFloats * 4;
  static constexpr int kOffPrefix = kOffMisc + kMiscFloats * 4;
  static size_t bytes(int batch) { return (size_t)kOffPrefix + (size_t)(batch + 1) * 4; }
};

// Unnormalised Walsh-Hadamard transform of each 128-block of one row held by
// a warp: lane l holds elements 4l..4l+3 of every block.  Strides 1 and 2 are
// in-lane, strides 4..64 pair lane l with lane l ^ (stride / 4); the lower
// index of a pair gets u + w, the upper u - w.
template <int NB>
__device__ __forceinline__ void wht_rows(float (&v)[NB][4], int lane) {
#pragma unroll
  for (int blk = 0; blk < NB; ++blk) {
    const float t0 = v[blk][0] + v[blk][1], t1 = v[blk][0] - v[blk][1];
    const float t2 = v[blk][2] + v[blk][3], t3 = v[blk][2] - v[blk][3];
    v[blk][0] = t0 + t2;
    v[blk][2] = t0 - t2;
    v[blk][1] = t1 + t3;
    v[blk][3] = t1 - t3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float o = __shfl_xor_sync(0xffffffffu, v[blk][k], m);
        v[blk][k] = (lane & m) ? o - v[blk][k] : v[blk][k] + o;
      }
    }
  }
}

// Decode step: encode 128-block `blk` of the new token's K (side 0) or V
// (side 1) row `row` of kv_new into cache token `tok`, by one warp (lane l
// holds elements 4l..4l+3).  Same steps as the encoder: fp16 block norm of
// x, signs, unnormalised WHT, idx = #{boundaries < y / n} counted on |y|
// against T_k * n, LSB-first packing ("TheTom/llama-cpp-turboquant" README,
// table "量化类型"; intelliparadigm TurboQuant article §3.2-§3.3).  `stage`
// is 16 words of this warp's shared memory.
__device__ __noinline__ void append_block(const DecodeParams& p, int side, int blk, size_t row,
                                          size_t tok, int lane, uint32_t* stage) {
  const int bits = side ? p.v_bits : p.k_bits;
  const int L = 1 << bits;
  const int nb = p.head_dim / kBlock;
  const size_t e0 = row * p.head_dim + (size_t)blk * kBlock + 4 * lane;
  float v[1][4];
  if (p.kv_new_f16) {
    const uint2 h = *reinterpret_cast<const uint2*>(static_cast<const __half*>(p.kv_new[side]) + e0);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
    v[0][0] = a.x; v[0][1] = a.y; v[0][2] = c.x; v[0][3] = c.y;
  } else {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(p.kv_new[side]) + e0);
    v[0][0] = a.x; v[0][1] = a.y; v[0][2] = a.z; v[0][3] = a.w;
  }
  float ss = v[0][0] * v[0][0];
  ss = fmaf(v[0][1], v[0][1], ss);
  ss = fmaf(v[0][2], v[0][2], ss);
  ss = fmaf(v[0][3], v[0][3], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float n = __fsqrt_rn(ss);
  const uint32_t sgn = p.sign_mask[lane >> 3] >> (4 * (lane & 7));
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if ((sgn >> k) & 1u) v[0][k] = -v[0][k];
  wht_rows<1>(v, lane);
  uint32_t field = 0;  // this lane's 4 codes, bits*4 bits
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float y = v[0][e], a = fabsf(y);
    int m = 0;
    for (int k = 0; k < L / 2 - 1; ++k) m += (a > p.pos_bounds[side][k] * n) ? 1 : 0;
    const int lowside = L / 2 - 1 - m;
    const uint32_t idx = (uint32_t)(y > 0.0f ? (lowside ^ (L - 1)) : lowside);
    field |= idx << (bits * e);
  }
  // lane l's codes are bits [4*bits*l, 4*bits*(l+1)) of the block's stream
  if (lane < 4 * bits) stage[lane] = 0u;
  __syncwarp();
  const int bit = 4 * bits * lane, wi = bit >> 5, sh = bit & 31;
  atomicOr(stage + wi, field << sh);
  if (sh + 4 * bits > 32) atomicOr(stage + wi + 1, field >> (32 - sh));
  __syncwarp();
  uint32_t* dst = reinterpret_cast<uint32_t*>(p.app_codes[side] + (tok * nb + blk) * 16 * bits);
  if (lane < 4 * bits) dst[lane] = stage[lane];
  if (lane == 0) {
    __half nh = __float2half_rn(n);
    if (__hisinf(nh)) {
      nh = __ushort_as_half((unsigned short)0x7BFF);
      if (p.status) atomicOr(p.status, TQ_DEV_NORM_OVERFLOW);
    }
    p.app_norms[side][tok * nb + blk] = __half_as_ushort(nh);
  }
}

// How the flattened (unit, tile) space [0, T) is split over the persistent
// CTAs.  Every unit's tiles cost 1 each and starting a unit costs kSwitchTiles
// more (its query preparation, the drained copy ring, the partial's merge
// and publication), so a CTA whose range spans two units gets fewer tiles:
// CTA c takes the tiles whose cost falls in [c, c+1) * Ctot / P.  The cost
// before batch entry b is UB * (prefix[b] + kSwitchTiles * b).  A cost that
// falls between two units maps to the start of the second, so a cut there
// adds no segment.  Results do not depend on the split (each part is computed
// and merged in a fixed order); it only moves where the CTAs end.
constexpr long long kSwitchTiles = TQ_SWITCH_TILES;

// floor(a / b) for 0 <= a, 0 < b, both below 2^52: the double quotient is
// within one of the exact one, and one integer step corrects it (a 64-bit
// integer division is a long instruction sequence on the GPU).
__device__ __forceinline__ long long fdiv(long long a, long long b) {
  long long q = (long long)((double)a / (double)b);
  if (q * b > a) --q; else if ((q + 1) * b <= a) ++q;
  return q;
}

struct Split {
  const int* prefix;  // [B+1] tiles per batch entry, exclusive prefix (shared memory)
  int B, UB;
  long long P, T, Ctot;
  __device__ Split(const int* pre, int batch, int ub, long long parts)
      : prefix(pre), B(batch), UB(ub), P(parts) {
    T = (long long)pre[batch] * ub;
    Ctot = (long long)ub * ((long long)pre[batch] + kSwitchTiles * batch);
  }
  // first tile of part c (c = P gives T)
  __device__ long long start(long long c) const {
    if (c >= P) return T;
    const long long y = fdiv(c * Ctot, P);
    int bl = 0, bh = B;  // largest b with cost(b) <= y
    while (bh - bl > 1) {
      const int mid = (bl + bh) >> 1;
      if ((long long)UB * (prefix[mid] + kSwitchTiles * mid) <= y) bl = mid; else bh = mid;
    }
    const long long nt = prefix[bl + 1] - prefix[bl];
    const long long rem = y - (long long)UB * (prefix[bl] + kSwitchTiles * bl);
    const long long r = fdiv(rem, nt + kSwitchTiles), t = rem - r * (nt + kSwitchTiles);
    return (long long)UB * prefix[bl] + r * nt + min(t, nt);
  }
  __device__ bool empty(long long c) const { return start(c) == start(c + 1); }
  // The part whose range holds tile x (0 <= x < T): the last c whose cost
  // floor(c * Ctot / P) is at most x's cost F.
  __device__ long long part_of(long long x) const {
    int bl = 0, bh = B;  // largest b with UB * prefix[b] <= x
    while (bh - bl > 1) {
      const int mid = (bl + bh) >> 1;
      if ((long long)UB * prefix[mid] <= x) bl = mid; else bh = mid;
    }
    const long long nt = prefix[bl + 1] - prefix[bl];
    const long long off = x - (long long)UB * prefix[bl];
    const long long r = fdiv(off, nt), t = off - r * nt;
    const long long F = (long long)UB * (prefix[bl] + kSwitchTiles * bl) + r * (nt + kSwitchTiles) + t;
    const long long c = fdiv((F + 1) * P - 1, Ctot);
    return c < P - 1 ? c : P - 1;
  }
};

// (m, l) of partials c0 .. c0+n-1 of one unit into shared memory, every load
// in flight at once; heads >= Gu and CTAs whose range is empty get (-inf, 0).
__device__ __forceinline__ void stage_ml(const float* slot_ml, long long c0, int n, const Split& sp,
                                         long long unit, int Gu, float* sm, float* sl) {
  for (int i = threadIdx.x; i < n * kMaxGroup; i += kCThreads) {
    const long long c = c0 + i / kMaxGroup;
    const int hd = i % kMaxGroup;
    float2 ml = make_float2(-INFINITY, 0.0f);
    if (hd < Gu && !sp.empty(c))
      ml = __ldcg(reinterpret_cast<const float2*>(slot_ml + ((c + unit) * kMaxGroup + hd) * 2));
    sm[i] = ml.x;
    sl[i] = ml.y;
  }
}

// Per-head (M, L) = (max m, sum l * 2^(m - M)) over the partials c_first ..
// c_last of one unit.  Partials are staged kMergeChunk at a time; thread t
// of the first kFold folds head t % 8 of every (kFold/8)-th staged partial,
// then the running pairs of a head are combined, all in a fixed order.  On
// return sm/sl hold the last staged chunk.
__device__ __forceinline__ void unit_stats(const float* slot_ml, long long c_first, long long c_last,
                                           const Split& sp, long long unit, int Gu,
                                           float* sm, float* sl, float* red_m, float* red_l,
                                           float* outM, float* outL) {
  constexpr int kFold = kCThreads < 128 ? kCThreads : 128;  // threads that fold
  constexpr int J = kFold / kMaxGroup;
  const int tid = threadIdx.x, hd = tid % kMaxGroup, j = tid / kMaxGroup;
  float m = -INFINITY, l = 0.0f;
  for (long long c0 = c_first; c0 <= c_last; c0 += kMergeChunk) {
    const int n = (int)min((long long)kMergeChunk, c_last - c0 + 1);
    consumer_sync();  // the previous chunk has been folded
    stage_ml(slot_ml, c0, n, sp, unit, Gu, sm, sl);
    consumer_sync();
    for (int k = j; tid < kFold && k < n; k += J) {
      const float mc = sm[k * kMaxGroup + hd], lc = sl[k * kMaxGroup + hd];
      if (mc == -INFINITY) continue;
      if (mc > m) {
        l = l * ex2(m - mc) + lc;
        m = mc;
      } else {
        l += lc * ex2(mc - m);
      }
    }
  }
  red_m[tid] = m;
  red_l[tid] = l;
  consumer_sync();
  if (tid < Gu) {
    float M = -INFINITY;
    for (int jj = 0; jj < J; ++jj) M = fmaxf(M, red_m[jj * kMaxGroup + tid]);
    float L = 0.0f;
    for (int jj = 0; jj < J; ++jj) {
      const float mj = red_m[jj * kMaxGroup + tid];
      if (mj != -INFINITY) L += red_l[jj * kMaxGroup + tid] * ex2(mj - M);
    }
    outM[tid] = M;
    outL[tid] = L;
  }
  consumer_sync();
}

// Where tile x of the flattened (unit, tile) space lies.
struct Segment {
  int b, r, nt, unit, kvh, hg, h0, Gu, len, seg_lo, seg_hi;
  long long Su;
};

__device__ __forceinline__ Segment locate(long long x, long long hi, const int* prefix, int batch,
                                          int UB, int n_hg, int G, int seq_cap,
                                          const int32_t* seq_lens) {
  Segment s;
  const long long y = x / UB;  // in units of "tiles per batch entry"
  int bl = 0, bh = batch;      // largest b with prefix[b] <= y
  while (bh - bl > 1) {
    const int mid = (bl + bh) >> 1;
    if (prefix[mid] <= y) bl = mid; else bh = mid;
  }
  s.b = bl;
  s.nt = prefix[bl + 1] - prefix[bl];
  const long long TB = (long long)prefix[bl] * UB;
  s.r = (int)((x - TB) / s.nt);
  s.Su = TB + (long long)s.r * s.nt;
  s.seg_lo = (int)(x - s.Su);
  s.seg_hi = (int)(min(hi, s.Su + s.nt) - s.Su);
  s.unit = bl * UB + s.r;
  s.kvh = s.r / n_hg;
  s.hg = s.r % n_hg;
  s.h0 = s.kvh * G + s.hg * kMaxGroup;  // first (virtual) head of the unit
  s.Gu = min(kMaxGroup, G - s.hg * kMaxGroup);
  s.len = min(max(__ldg(seq_lens + bl), 0), seq_cap);
  return s;
}

// --------------------------------------------------------------- the kernel --

template <int KB, int VB, int NB, int MODE, int GQ>
__global__ void __launch_bounds__(kThreads, NB == 1 ? TQ_DECODE_MIN_CTAS : TQ_DECODE_MIN_CTAS_WIDE)
decode_kernel(const __grid_constant__ DecodeParams p, int p1_ctas) {
  using SM = Smem<KB, VB, NB, MODE>;
  constexpr int D = SM::D;
  constexpr bool HASK = SM::kHasK, HASV = SM::kHasV;
  constexpr int KBB = Fmt<KB>::kBlockBytes, VBB = Fmt<VB>::kBlockBytes;
  constexpr int kDepth = SM::kDepth;
  // GQ == 4 (at most four query heads per unit): score columns 4..7 repeat
  // heads 0..3, and the V products use the eight MMA columns as (head, dim
  // parity) pairs, so V fragments come straight from the table.  GQ == 8:
  // one column per head, V fragments re-paired by token.
  static_assert(GQ == 4 || GQ == 8, "GQ");
  static_assert(kCWarps >= 2 * NB, "the decode step appends one block per warp");
  constexpr bool kDup = GQ == 4;
  constexpr int kMT = kDup ? 4 : 8;  // V accumulator tiles per 128-block
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(128) uint8_t rawLut[SM::kRawLut];
  // shared-window addresses of the two tables
  uint32_t lutK_s, lutV_s;
  {
    const uint32_t a = SM::kAMax ? (uint32_t)SM::kAMax : 16u;
    const uint32_t first = (smem_addr(rawLut) + a - 1) & ~(a - 1);
    const uint32_t second = first + (uint32_t)(SM::kKFirst ? SM::kAK : SM::kAV);
    lutK_s = SM::kAlignK ? (SM::kKFirst ? first : second) : smem_addr(smem + SM::kOffLutK);
    lutV_s = SM::kAlignV ? (SM::kKFirst ? second : first) : smem_addr(smem + SM::kOffLutV);
  }
  uint8_t* ring = smem + SM::kOffRing;
  float* work = reinterpret_cast<float*>(smem + SM::kOffWork);
  float* res = reinterpret_cast<float*>(smem + SM::kOffRes);
  float* misc = reinterpret_cast<float*>(smem + SM::kOffMisc);
  float* w_m = misc;                                  // [kCWarps][8]
  float* w_l = misc + kCWarps * kMaxGroup;            // [kCWarps][8]
  float* u_M = misc + 2 * kCWarps * kMaxGroup;        // [8]
  float* u_L = u_M + kMaxGroup;                       // [8]
  float* u_lse = u_L + kMaxGroup;                     // [8]
  int* qexp = reinterpret_cast<int*>(u_lse + kMaxGroup);  // [8]
  int* wtot = qexp + kMaxGroup;                       // [16]
  int* flag = wtot + 16;                              // [4]
  float* red_m = reinterpret_cast<float*>(flag + 4);  // [kCThreads]
  float* red_l = red_m + kCThreads;                   // [kCThreads]
  float* fac = red_l + kCThreads;                     // [kMergeChunk][8] staged m, then weights
  float* stl = fac + kMergeChunk * kMaxGroup;         // [kMergeChunk][8] staged l
  int* prefix = reinterpret_cast<int*>(smem + SM::kOffPrefix);  // [B+1] tiles per batch, prefix

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = lane >> 2, g = lane & 3;
  const uint32_t lane4 = (uint32_t)lane * 4u;
  const uint32_t lbK = lutK_s + lane4, lbV = lutV_s + lane4;
  // kDup B fragments: a token's weight in the low half (s' = 0, R < 4) or
  // the high half (s' = 1) of the register, zero in the other
  const uint32_t selLo = R < 4 ? 0x4410u : 0x1044u, selHi = R < 4 ? 0x4432u : 0x3244u;
  // Heads of a unit are "virtual heads" (query token j, q-head h of the
  // kv-head's group), vl = j * G + h, so n_q query tokens per sequence share
  // the K/V fragments of each tile.  Virtual head vh = kvh * Gv + vl of batch
  // entry b reads q and writes out row (b * n_q + j) * q_heads + kvh * G + h.
  const int G = p.q_heads / p.kv_heads;
  const int Gv = G * p.n_q;
  const int n_hg = (Gv + kMaxGroup - 1) / kMaxGroup;
  const int UB = p.kv_heads * n_hg;  // units per batch entry
  auto vrow = [&](int b, int vh) -> size_t {
    const int kvh = vh / Gv, vl = vh % Gv;
    return ((size_t)b * p.n_q + vl / G) * p.q_heads + kvh * G + vl % G;
  };

  // ---- tables: code pair -> half2 codewords, replicated for every lane ----
  if constexpr (HASK) {
    for (int e = tid; e < Fmt<KB>::kEntries * 32; e += kThreads) {
      const int ent = e >> 5;
      const float lo = p.kcent[ent & ((1 << KB) - 1)], hi = p.kcent[ent >> KB];
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(lutK_s + 4u * e), "r"(pack_half2(lo, hi)) : "memory");
    }
  }
  if constexpr (HASV) {
    for (int e = tid; e < Fmt<VB>::kEntries * 32; e += kThreads) {
      const int ent = e >> 5;
      const float lo = p.vcent[ent & ((1 << VB) - 1)], hi = p.vcent[ent >> VB];
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(lutV_s + 4u * e), "r"(pack_half2(lo, hi)) : "memory");
    }
  }

  // ---- lengths: clamp, tiles per batch entry, exclusive prefix ------------
  {
    const int B = p.batch;
    const int per = (B + kThreads - 1) / kThreads;
    int local = 0;
    const int b_lo = tid * per;
    for (int b = b_lo; b < min(B, b_lo + per); ++b) {
      int len = __ldg(p.seq_lens + b);
      if (len < 0 || len > p.seq_cap) {
        if (blockIdx.x == 0 && p.status) atomicOr(p.status, TQ_DEV_LEN_RANGE);
        len = min(max(len, 0), p.seq_cap);
      }
      local += (len + kTile - 1) / kTile;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    int warp_off = 0;
    for (int w = 0; w < warp; ++w) warp_off += wtot[w];
    int run = warp_off + incl - local;
    for (int b = b_lo; b < min(B, b_lo + per); ++b) {
      prefix[b] = run;
      int len = min(max(__ldg(p.seq_lens + b), 0), p.seq_cap);
      run += (len + kTile - 1) / kTile;
    }
    if (tid == kThreads - 1) prefix[B] = run;
    __syncthreads();
  }
  const Split sp(prefix, p.batch, UB, gridDim.x);  // this launch's split
  const long long T = sp.T;

  // ---- zero rows of empty sequences (only the V-producing passes) ---------
  if constexpr (MODE != kScores) {
    const long long rows = (long long)p.batch * p.n_q * p.q_heads;
    for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
      const int b = (int)(row / ((long long)p.n_q * p.q_heads));
      if (prefix[b + 1] == prefix[b]) {
        for (int d = tid; d < D; d += kThreads) p.out[row * D + d] = 0.0f;
      }
    }
  }
  if (T == 0) return;

  const long long lo = sp.start(blockIdx.x), hi = sp.start(blockIdx.x + 1);
  const int cw = warp;
  uint8_t* wring = ring + (size_t)cw * kDepth * SM::kSlotBytes;  // this warp's ring
  const uint32_t wring_s = smem_addr(wring);
  // ---- query preparation: qhat = H.(s o q) (D1), as this lane's fp16 MMA
  // B fragments plus the per-column score multipliers.  One warp per head
  // row: lane l holds dims 4l..4l+3 of every 128-block, the butterflies of
  // stride 1 and 2 are in-lane, strides 4..64 cross lanes.  Uses res as
  // scratch.
  auto prep_q = [&](int b, int h0, int Gu, uint32_t (&qf)[NB][8][2], float (&qmul)[2]) {
    constexpr int kQRows = kDup ? 4 : kMaxGroup;
    float* qs = res;  // [kQRows][D] scaled qhat
    for (int j = cw; j < kQRows; j += kCWarps) {
      float v[NB][4];
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const size_t qi = vrow(b, h0 + j) * D + blk * kBlock + 4 * lane;
        if (j >= Gu) {
          v[blk][0] = v[blk][1] = v[blk][2] = v[blk][3] = 0.0f;
        } else if (p.q_f16) {
          const uint2 h = *reinterpret_cast<const uint2*>(reinterpret_cast<const __half*>(p.q) + qi);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
          const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
          v[blk][0] = a.x; v[blk][1] = a.y; v[blk][2] = c.x; v[blk][3] = c.y;
        } else {
          const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.q) + qi);
          v[blk][0] = a.x; v[blk][1] = a.y; v[blk][2] = a.z; v[blk][3] = a.w;
        }
        const uint32_t sgn = p.sign_mask[lane >> 3] >> (4 * (lane & 7));  // signs of dims 4l..4l+3
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if ((sgn >> k) & 1u) v[blk][k] = -v[blk][k];
      }
      wht_rows<NB>(v, lane);
      // power-of-two scale per head so fp16 fragments neither overflow nor
      // fall into subnormals
      float mx = 0.0f;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int k = 0; k < 4; ++k) mx = fmaxf(mx, fabsf(v[blk][k]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const int qe = (mx > 0.0f) ? (ilogbf(mx) - 13) : 0;
      if (lane == 0) qexp[j] = qe;
      const float sc = ldexpf(1.0f, -qe);
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
        *reinterpret_cast<float4*>(qs + j * D + blk * kBlock + 4 * lane) =
            make_float4(v[blk][0] * sc, v[blk][1] * sc, v[blk][2] * sc, v[blk][3] * sc);
    }
    consumer_sync();
    const int hr = kDup ? (R & 3) : R;  // this lane's score column's head
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float* q4 = qs + hr * D + blk * kBlock + 32 * g + 4 * j;
        qf[blk][j][0] = pack_half2(q4[0], q4[1]);
        qf[blk][j][1] = pack_half2(q4[2], q4[3]);
      }
    }
    qmul[0] = p.score_mult * ldexpf(1.0f, qexp[kDup ? (2 * g) & 3 : 2 * g]);
    qmul[1] = p.score_mult * ldexpf(1.0f, qexp[kDup ? (2 * g + 1) & 3 : 2 * g + 1]);
    consumer_sync();  // res and qexp are reused after this
  };

  // ---- D7/D8: a unit's output from res, one inverse rotation per head,
  // o = s o (H.acc) / L ---------------------------------------------------------
  auto emit = [&](const Segment& sg) {
    const int Gu = sg.Gu, b = sg.b, h0 = sg.h0;
    const uint32_t sgn = p.sign_mask[lane >> 3] >> (4 * (lane & 7));  // signs of dims 4l..4l+3
    for (int hd = cw; hd < Gu; hd += kCWarps) {  // one warp per head row
      float v[NB][4];
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const float4 a = *reinterpret_cast<const float4*>(res + hd * D + blk * kBlock + 4 * lane);
        v[blk][0] = a.x; v[blk][1] = a.y; v[blk][2] = a.z; v[blk][3] = a.w;
      }
      wht_rows<NB>(v, lane);
      const float L = (MODE == kFused) ? u_L[hd] : 1.0f;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if constexpr (MODE == kFused) v[blk][k] = L > 0.0f ? v[blk][k] / L : 0.0f;  // L = 0: no position seen
          if ((sgn >> k) & 1u) v[blk][k] = -v[blk][k];
        }
        *reinterpret_cast<float4*>(p.out + vrow(b, h0 + hd) * D + blk * kBlock + 4 * lane) =
            make_float4(v[blk][0], v[blk][1], v[blk][2], v[blk][3]);
      }
    }
  };

  // ---- every partial of a unit merged into res (and u_M, u_L) in a fixed
  // order; the unit's ticket is cleared for the next launch -------------------
  auto merge_unit = [&](const Segment& sg) {
    const int Gu = sg.Gu, unit = sg.unit, nt = sg.nt;
    const long long Su = sg.Su;
    __threadfence();
    const long long c_first = sp.part_of(Su), c_last = sp.part_of(Su + nt - 1);
    if constexpr (HASK) unit_stats(p.slot_ml, c_first, c_last, sp, unit, Gu, fac, stl, red_m, red_l, u_M, u_L);
    for (int i = tid; i < Gu * D; i += kCThreads) res[i] = 0.0f;
    const bool one_chunk = c_last - c_first < kMergeChunk;
    for (long long c0 = c_first; c0 <= c_last; c0 += kMergeChunk) {
      const int n = (int)min((long long)kMergeChunk, c_last - c0 + 1);
      // weights 2^(m_c - M) of this chunk's partials (0 for empty ranges;
      // without scores, 1 for every non-empty range)
      if constexpr (HASK) {
        if (!one_chunk) {  // else unit_stats left this chunk staged
          consumer_sync();
          stage_ml(p.slot_ml, c0, n, sp, unit, Gu, fac, stl);
          consumer_sync();
        }
        for (int i = tid; i < n * kMaxGroup; i += kCThreads) {
          const float mc = fac[i];
          fac[i] = (mc == -INFINITY) ? 0.0f : ex2(mc - u_M[i % kMaxGroup]);
        }
      } else {
        consumer_sync();
        for (int i = tid; i < n * kMaxGroup; i += kCThreads) {
          const long long c = c0 + i / kMaxGroup;
          fac[i] = (i % kMaxGroup < Gu && !sp.empty(c)) ? 1.0f : 0.0f;
        }
      }
      consumer_sync();
      // four consecutive dims per thread, many partials in flight (the
      // merge is on the critical path of the whole launch)
      for (int i = tid; i < Gu * D / 4; i += kCThreads) {
        const int hd = (4 * i) / D, d = (4 * i) % D;
        const float4* src =
            reinterpret_cast<const float4*>(p.slot_acc + ((c0 + unit) * kMaxGroup + hd) * D + d);
        float4 sacc = reinterpret_cast<const float4*>(res)[i];
#pragma unroll 16
        for (int cc = 0; cc < n; ++cc) {
          const float f = fac[cc * kMaxGroup + hd];
          const float4 a = __ldcg(src + (size_t)cc * kMaxGroup * D / 4);
          if (f != 0.0f) {  // a partial that was never written may hold anything
            sacc.x = fmaf(a.x, f, sacc.x);
            sacc.y = fmaf(a.y, f, sacc.y);
            sacc.z = fmaf(a.z, f, sacc.z);
            sacc.w = fmaf(a.w, f, sacc.w);
          }
        }
        reinterpret_cast<float4*>(res)[i] = sacc;
      }
    }
    consumer_sync();
    if (tid == 0) p.tickets[unit] = 0u;
    consumer_sync();
  };

  // ---- add a segment's tiles to its unit's count: true for the CTA that
  // completes it ------------------------------------------------------------------
  auto count_tiles = [&](const Segment& sg) -> bool {
    __threadfence();
    consumer_sync();
    if (tid == 0) {
      const unsigned add = (unsigned)(sg.seg_hi - sg.seg_lo);
      const unsigned old = atomicAdd(p.tickets + sg.unit, add);
      flag[0] = (old + add == (unsigned)sg.nt) ? 1 : 0;
    }
    consumer_sync();
    return flag[0] != 0;
  };

  for (long long x = lo; x < hi;) {
    const Segment sg = locate(x, hi, prefix, p.batch, UB, n_hg, Gv, p.seq_cap, p.seq_lens);
    const int b = sg.b, nt = sg.nt, unit = sg.unit, h0 = sg.h0, Gu = sg.Gu, len = sg.len;
    const int seg_lo = sg.seg_lo, seg_hi = sg.seg_hi;
    const long long Su = sg.Su;
    const size_t cache_row = (size_t)(b * p.kv_heads + sg.kvh) * p.seq_cap;
    const uint8_t* kcp = p.k_codes + cache_row * NB * KBB;
    const uint8_t* vcp = p.v_codes + cache_row * NB * VBB;
    const uint16_t* knp = p.k_norms + cache_row * NB;
    const uint16_t* vnp = p.v_norms + cache_row * NB;

    // Copy tile `tile` of this unit into ring slot `slot` (all lanes; one
    // commit group).  Bytes past the end of the sequence are zero-filled.
    auto issue = [&](int tile, int slot) {
      const int t0 = tile * kTile;
      const int nval = min(kTile, len - t0);  // >= 1
      const bool full = nval == kTile;
      const uint32_t sb = wring_s + (uint32_t)(slot * SM::kSlotBytes);
      if constexpr (HASK) {
        constexpr int kChunks = kTile * NB * KB;  // 16-byte chunks (KBB = 16 * KB)
        constexpr int kPerTok = NB * KB;
        const uint8_t* src = kcp + (size_t)t0 * NB * KBB;
#pragma unroll
        for (int c0 = 0; c0 < kChunks; c0 += 32) {
          const int c = c0 + lane;
          if (c < kChunks) {
            const bool ok = full || c / kPerTok < nval;
            cp_async16(sb + 16u * c, src + (ok ? 16 * c : 0), ok ? 16u : 0u);
          }
        }
        if (lane < 8 * NB) {  // norms: 4-byte pieces of the tile's 16*NB halves
          const int e = 2 * lane;  // first half of the piece
          const int valid = full ? 2 : max(0, min(2, nval * NB - e));
          cp_async4(sb + SM::kOffSlotKN + 4u * lane, knp + (size_t)t0 * NB + (valid ? e : 0),
                    2u * (uint32_t)valid);
        }
      }
      if constexpr (HASV) {
        constexpr int kChunks = kTile * NB * VB;
        constexpr int kPerTok = NB * VB;
        const uint8_t* src = vcp + (size_t)t0 * NB * VBB;
#pragma unroll
        for (int c0 = 0; c0 < kChunks; c0 += 32) {
          const int c = c0 + lane;
          if (c < kChunks) {
            const bool ok = full || c / kPerTok < nval;
            cp_async16(sb + SM::kOffSlotV + 16u * c, src + (ok ? 16 * c : 0), ok ? 16u : 0u);
          }
        }
        if (lane < 8 * NB) {
          const int e = 2 * lane;
          const int valid = full ? 2 : max(0, min(2, nval * NB - e));
          cp_async4(sb + SM::kOffSlotVN + 4u * lane, vnp + (size_t)t0 * NB + (valid ? e : 0),
                    2u * (uint32_t)valid);
        }
      }
    };

    // This lane's first K / V word inside a slot.
    const int vlane = VB == 4 ? 8 * R : (VB == 3 ? 4 * ((3 * R) >> 1) : 4 * R);
    const uint32_t koff = (uint32_t)((2 * R) * NB * KBB + g * KB * 4);
    const uint32_t voff = (uint32_t)(SM::kOffSlotV + (4 * g) * NB * VBB + vlane);
    // ---- decode step: the CTA that holds a unit's last tile first writes the
    // sequence's new token (position len - 1) into the cache, K and V, one
    // warp per 128-block, so that its own copies read it.  Other head groups
    // of the same kv-head write the same bytes.  A length outside
    // [1, seq_cap] appends nothing: clamping it would overwrite a cached
    // token (the range error is reported by the length scan).
    if (MODE != kSparseV && p.kv_new[0] != nullptr && seg_hi == nt && len > 0 &&
        __ldg(p.seq_lens + b) == len) {
      if (cw < 2 * NB) {
        append_block(p, cw / NB, cw % NB, (size_t)b * p.kv_heads + sg.kvh, cache_row + (len - 1), lane,
                     reinterpret_cast<uint32_t*>(res) + 16 * cw);
      }
      __threadfence();
      consumer_sync();
    }
    // Warp cw takes tiles seg_lo + cw, seg_lo + cw + kCWarps, ...: tile i of
    // the warp (i = 0, 1, ...) lives in slot i % kDepth.  The first kDepth
    // copies are issued before the query preparation, which they overlap.
    const int first = seg_lo + cw;
    const int n_mine = first < seg_hi ? (seg_hi - first + kCWarps - 1) / kCWarps : 0;
#pragma unroll
    for (int i = 0; i < kDepth; ++i) {
      if (i < n_mine) issue(first + i * kCWarps, i);
      cp_async_commit();
    }
    // ---- per-unit query preparation ----------------------------------------
    uint32_t qf[NB][8][2];
    float qmul[2] = {0.0f, 0.0f};
    float lse2[2] = {0.0f, 0.0f};
    if constexpr (HASK) prep_q(b, h0, Gu, qf, qmul);
    if constexpr (MODE == kSparseV) {
      // log-sum-exp (log2 domain) of every head of this unit, from the
      // partials that pass 1 (p1_ctas CTAs) wrote
      const Split sp1(prefix, p.batch, UB, p1_ctas);
      unit_stats(p.slot_ml, sp1.part_of(Su), sp1.part_of(Su + nt - 1), sp1, unit, Gu, fac, stl, red_m, red_l,
                 u_M, u_L);
      if (tid < Gu) u_lse[tid] = u_M[tid] + __log2f(u_L[tid]);
      consumer_sync();
      const int hd0 = kDup ? (2 * g) & 3 : 2 * g, hd1 = kDup ? (2 * g + 1) & 3 : 2 * g + 1;
      lse2[0] = (hd0 < Gu) ? u_lse[hd0] : 0.0f;
      lse2[1] = (hd1 < Gu) ? u_lse[hd1] : 0.0f;
    }
    const float log2_thr = (MODE == kSparseV) ? __log2f(p.sparse_thr) : 0.0f;

    // ---- warp loop over this segment's stages -----------------------------
    float acc[NB][kMT][4];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk)
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[blk][mt][e] = 0.0f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};

    // Phase 1 of a tile: raw Hadamard-domain score sums per block (D2/D3),
    // straight from the codes, in kKChains independent accumulator chains.
    struct Raw { float c[NB][4]; };
    auto scores = [&](const TileRegs<KB, VB, NB>& tr) {
      Raw r{};
      if constexpr (HASK) {
        float ca[kKChains][NB][4];
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
          for (int c = 0; c < kKChains; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) ca[c][blk][e] = 0.0f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t a0 = lut_get<SM::kAlignK>(tr.k[0][blk], 2 * KB * (2 * j), 2 * KB, lbK);
            const uint32_t a1 = lut_get<SM::kAlignK>(tr.k[1][blk], 2 * KB * (2 * j), 2 * KB, lbK);
            const uint32_t a2 = lut_get<SM::kAlignK>(tr.k[0][blk], 2 * KB * (2 * j + 1), 2 * KB, lbK);
            const uint32_t a3 = lut_get<SM::kAlignK>(tr.k[1][blk], 2 * KB * (2 * j + 1), 2 * KB, lbK);
            mma16816(ca[j % kKChains][blk], a0, a1, a2, a3, qf[blk][j][0], qf[blk][j][1]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float t = ca[0][blk][e];
#pragma unroll
            for (int c = 1; c < kKChains; ++c) t += ca[c][blk][e];
            r.c[blk][e] = t;
          }
        }
      }
      return r;
    };

    // Phase 2 of a tile: scale and mask the scores, online softmax (D4) or the
    // sparse-V gate (D5), then the V sum in the rotated domain (D6).
    // Positions each of this lane's two score columns may see: query token j
    // of the sequence sits at len - n_q + j and sees the positions up to its
    // own.  Padding columns (head >= Gu) see the whole sequence.
    int lim[2];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int hd = kDup ? (2 * g + cc) & 3 : 2 * g + cc;
      const int tok = (sg.hg * kMaxGroup + hd) / G;
      lim[cc] = hd < Gu ? min(len, len - p.n_q + tok + 1) : len;
    }
    const int len_full = len - p.n_q + 1;  // tiles ending here see no mask at all

    auto finish = [&](const TileRegs<KB, VB, NB>& tr, int tile, const Raw& raw, auto full_tag) {
      constexpr bool FULL = decltype(full_tag)::value;
      const int t0 = tile * kTile;
      // rows R and R+8 of the score tile are tokens 2R and 2R+1
      bool okR[2], okR8[2];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        okR[cc] = FULL || t0 + 2 * R < lim[cc];
        okR8[cc] = FULL || t0 + 2 * R + 1 < lim[cc];
      }
      float pR[2], pR8[2];
      if constexpr (HASK) {
        float sR[2], sR8[2];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float a = 0.0f, bb = 0.0f;
#pragma unroll
          for (int blk = 0; blk < NB; ++blk) {
            const float2 kn = norm_pair<NB>(tr.kn, blk);
            a = fmaf(raw.c[blk][cc], kn.x, a);
            bb = fmaf(raw.c[blk][2 + cc], kn.y, bb);
          }
          sR[cc] = okR[cc] ? a * qmul[cc] : -INFINITY;
          sR8[cc] = okR8[cc] ? bb * qmul[cc] : -INFINITY;
        }
        if constexpr (MODE == kScores) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int hd = 2 * g + cc;  // columns 4..7 repeat heads 0..3 when kDup
            if (hd < Gu && (!kDup || g < 2)) {
              float* srow = p.scores + ((size_t)b * p.kv_heads * Gv + h0 + hd) * p.seq_cap + t0 + 2 * R;
              if (okR8[cc]) {
                *reinterpret_cast<float2*>(srow) = make_float2(sR[cc], sR8[cc]);
              } else if (okR[cc]) {
                srow[0] = sR[cc];
              }
            }
          }
        }
        // D4: online softmax.  The per-head maximum is only reduced across the
        // warp when some lane's scores exceed the reference by more than 2^kTau.
        const float lm0 = fmaxf(sR[0], sR8[0]), lm1 = fmaxf(sR[1], sR8[1]);
        const bool need = (lm0 > m_run[0] + kTau) || (lm1 > m_run[1] + kTau);
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float tmax = cc ? lm1 : lm0;
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
            if (tmax > m_run[cc] + kTau) {
              const float alpha = ex2(m_run[cc] - tmax);
              l_run[cc] *= alpha;
              if constexpr (MODE == kFused) {
#pragma unroll
                for (int blk = 0; blk < NB; ++blk)
#pragma unroll
                  for (int mt = 0; mt < kMT; ++mt) {
                    acc[blk][mt][cc] *= alpha;
                    acc[blk][mt][2 + cc] *= alpha;
                  }
              }
              m_run[cc] = tmax;
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          // a column that has seen no position yet (a later query token's
          // causal limit) keeps m = -inf: its weights are 0, not NaN
          const float mref = m_run[cc] == -INFINITY ? 0.0f : m_run[cc];
          pR[cc] = ex2(sR[cc] - mref);
          pR8[cc] = ex2(sR8[cc] - mref);
          l_run[cc] += pR[cc] + pR8[cc];
        }
      } else {
        // pass 2 of sparse-V: normalised weights from the stored scores (D5)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int hd = kDup ? (2 * g + cc) & 3 : 2 * g + cc;
          float wR = 0.0f, wR8 = 0.0f;
          if (hd < Gu) {
            const float* srow = p.scores + ((size_t)b * p.kv_heads * Gv + h0 + hd) * p.seq_cap + t0 + 2 * R;
            float s0 = -INFINITY, s1 = -INFINITY;
            if (okR8[cc]) {
              const float2 sv = __ldcs(reinterpret_cast<const float2*>(srow));
              s0 = sv.x;
              s1 = sv.y;
            } else if (okR[cc]) {
              s0 = __ldcs(srow);
            }
            const float d0 = s0 - lse2[cc], d1 = s1 - lse2[cc];
            wR = d0 >= log2_thr ? ex2(d0) : 0.0f;
            wR8 = d1 >= log2_thr ? ex2(d1) : 0.0f;
          }
          pR[cc] = wR;
          pR8[cc] = wR8;
        }
      }
      if constexpr (HASV) {
        bool any = true;
        if constexpr (MODE == kSparseV)
          any = __any_sync(0xffffffffu, (pR[0] + pR[1] + pR8[0] + pR8[1]) > 0.0f);
        if (any) {
          // D6: V accumulated in the rotated domain
#pragma unroll
          for (int blk = 0; blk < NB; ++blk) {
            const float2 vn = norm_pair<NB>(tr.vn, blk);
            const float sv0 = vn.x * (1.0f / kBlock), sv1 = vn.y * (1.0f / kBlock);
            // P^T fragments: lane (R, g) gets tokens 4g, 4g+2 (b0) and
            // 4g+1, 4g+3 (b1) of score column R
            const uint32_t b0 = movtrans(pack_half2(pR[0] * sv0, pR[1] * sv0));
            const uint32_t b1 = movtrans(pack_half2(pR8[0] * sv1, pR8[1] * sv1));
            if constexpr (kDup) {
              // k = 2*tau + s, column n = h + 4*s': the product pairs the
              // weight of token tau with dim 2*pair + s only when s == s', so
              // each A register is one token's pair of adjacent dims.  Rows R,
              // R+8 of tile q are dim pairs 8R+2q, 8R+2q+1.
              const uint32_t pa0 = prmt(b0, 0u, selLo), pa1 = prmt(b0, 0u, selHi);
              const uint32_t pb0 = prmt(b1, 0u, selLo), pb1 = prmt(b1, 0u, selHi);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int f0 = 2 * VB * (2 * q), f1 = 2 * VB * (2 * q + 1);
                mma16816(acc[blk][q], lut_get<SM::kAlignV>(tr.v[0][blk], f0, 2 * VB, lbV),
                         lut_get<SM::kAlignV>(tr.v[0][blk], f1, 2 * VB, lbV),
                         lut_get<SM::kAlignV>(tr.v[1][blk], f0, 2 * VB, lbV),
                         lut_get<SM::kAlignV>(tr.v[1][blk], f1, 2 * VB, lbV), pa0, pa1);
                mma16816(acc[blk][q], lut_get<SM::kAlignV>(tr.v[2][blk], f0, 2 * VB, lbV),
                         lut_get<SM::kAlignV>(tr.v[2][blk], f1, 2 * VB, lbV),
                         lut_get<SM::kAlignV>(tr.v[3][blk], f0, 2 * VB, lbV),
                         lut_get<SM::kAlignV>(tr.v[3][blk], f1, 2 * VB, lbV), pb0, pb1);
              }
            } else {
#pragma unroll
              for (int mt = 0; mt < 8; ++mt) {
                const uint32_t x0 = lut_get<SM::kAlignV>(tr.v[0][blk], 2 * VB * mt, 2 * VB, lbV);
                const uint32_t x1 = lut_get<SM::kAlignV>(tr.v[1][blk], 2 * VB * mt, 2 * VB, lbV);
                const uint32_t x2 = lut_get<SM::kAlignV>(tr.v[2][blk], 2 * VB * mt, 2 * VB, lbV);
                const uint32_t x3 = lut_get<SM::kAlignV>(tr.v[3][blk], 2 * VB * mt, 2 * VB, lbV);
                mma16816(acc[blk][mt], prmt(x0, x1, 0x5410), prmt(x0, x1, 0x7632),
                         prmt(x2, x3, 0x5410), prmt(x2, x3, 0x7632), b0, b1);
              }
            }
          }
        }
      }
    };

    {
      // Tile i of the warp sits in slot i % kDepth.  Once both halves of a
      // tile are in registers, its slot is handed to tile i + kDepth, so the
      // copy runs under the tile's arithmetic.
      for (int i = 0; i < n_mine; ++i) {
        TileRegs<KB, VB, NB> tr;
        const uint32_t sl = wring_s + (uint32_t)((i % kDepth) * SM::kSlotBytes);
        cp_async_wait<kDepth - 1>();  // tile i has landed
        __syncwarp();
        read_tile<KB, VB, NB, HASK, HASV>(tr, sl + koff, sl + voff, R);
        if constexpr (HASK) read_norms<NB>(tr.kn, sl + SM::kOffSlotKN, R);
        if constexpr (HASV) read_norms<NB>(tr.vn, sl + SM::kOffSlotVN, R);
        __syncwarp();  // no lane reads the slot any more
        if (i + kDepth < n_mine) issue(first + (i + kDepth) * kCWarps, i % kDepth);
        cp_async_commit();
        const int tile = first + i * kCWarps;
        const Raw raw = scores(tr);
        if (tile * kTile + kTile <= len_full)
          finish(tr, tile, raw, std::true_type{});
        else
          finish(tr, tile, raw, std::false_type{});
      }
      cp_async_wait<0>();
      __syncwarp();
    }

    // ---- warp partials to shared memory -----------------------------------
    consumer_sync();  // every warp is done with its ring, which holds the partials
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float l = l_run[cc];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      if (R == 0 && (!kDup || g < 2)) {
        w_m[cw * kMaxGroup + 2 * g + cc] = m_run[cc];
        w_l[cw * kMaxGroup + 2 * g + cc] = l;
      }
    }
    if constexpr (HASV) {
      if constexpr (kDup) {
        // element e of tile q: column 2g + (e & 1) = head h + 4 s' (s' = g >> 1),
        // row R + 8 (e >> 1) = dim pair 8R + 2q + (e >> 1), dim 2 pair + s'
#pragma unroll
        for (int blk = 0; blk < NB; ++blk)
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int h = (2 * g + (e & 1)) & 3;
              const int d = blk * kBlock + 16 * R + 4 * q + 2 * (e >> 1) + (g >> 1);
              work[(cw * kMaxGroup + h) * D + d] = acc[blk][q][e];
            }
      } else {
#pragma unroll
        for (int blk = 0; blk < NB; ++blk)
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const int d0 = blk * kBlock + 16 * R + 2 * mt;
            float* w0 = work + (cw * kMaxGroup + 2 * g) * D + d0;
            float* w1 = work + (cw * kMaxGroup + 2 * g + 1) * D + d0;
            *reinterpret_cast<float2*>(w0) = make_float2(acc[blk][mt][0], acc[blk][mt][2]);
            *reinterpret_cast<float2*>(w1) = make_float2(acc[blk][mt][1], acc[blk][mt][3]);
          }
      }
    }
    consumer_sync();

    // ---- merge the warps in a fixed order ----------------------------------
    if constexpr (HASK) {
      if (tid < Gu) {
        float M = -INFINITY;
        for (int w = 0; w < kCWarps; ++w) M = fmaxf(M, w_m[w * kMaxGroup + tid]);
        float L = 0.0f;
        for (int w = 0; w < kCWarps; ++w) {
          const float mw = w_m[w * kMaxGroup + tid];
          if (mw != -INFINITY) L += w_l[w * kMaxGroup + tid] * ex2(mw - M);
        }
        u_M[tid] = M;
        u_L[tid] = L;
      }
    }
    if constexpr (HASV) {
      for (int i = tid; i < Gu * D; i += kCThreads) {
        const int hd = i / D, d = i % D;
        float M = 0.0f;
        if constexpr (HASK) {
          M = -INFINITY;
          for (int w = 0; w < kCWarps; ++w) M = fmaxf(M, w_m[w * kMaxGroup + hd]);
        }
        float s = 0.0f;
        for (int w = 0; w < kCWarps; ++w) {
          float f = 1.0f;
          if constexpr (HASK) {
            const float mw = w_m[w * kMaxGroup + hd];
            f = (mw == -INFINITY) ? 0.0f : ex2(mw - M);
          }
          s = fmaf(work[(w * kMaxGroup + hd) * D + d], f, s);
        }
        res[i] = s;
      }
    }
    consumer_sync();

    const bool whole = (seg_lo == 0 && seg_hi == nt);
    if (whole && MODE != kScores) {
      emit(sg);  // this CTA saw the entire unit: no partial needed
    } else {
      // ---- publish the partial ---------------------------------------------
      const long long slot = blockIdx.x + unit;
      if constexpr (HASK) {
        if (tid < Gu) {
          p.slot_ml[(slot * kMaxGroup + tid) * 2] = u_M[tid];
          p.slot_ml[(slot * kMaxGroup + tid) * 2 + 1] = u_L[tid];
        }
      }
      if constexpr (HASV) {
        for (int i = tid; i < Gu * D; i += kCThreads)
          p.slot_acc[(slot * kMaxGroup + i / D) * D + i % D] = res[i];
      }
      if constexpr (MODE != kScores) {
        if (count_tiles(sg)) {  // the last CTA of the unit merges its partials
          merge_unit(sg);
          emit(sg);
        }
      }
    }
    consumer_sync();
    x = Su + seg_hi;
  }

}

// --------------------------------------------------------------- launching --

template <int KB, int VB, int NB, int MODE, int GQ>
int run(const DecodeParams& p, cudaStream_t stream, int p1_ctas, int* ctas_out) {
  using SM = Smem<KB, VB, NB, MODE>;
  const size_t smem = SM::bytes(p.batch);
  auto kern = decode_kernel<KB, VB, NB, MODE, GQ>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  static int cached_sms[64] = {0};
  static int cached_occ[64] = {0};
  static size_t cached_smem[64] = {0};
  if (dev >= 64) return TQ_ERR_UNSUPPORTED;
  if (cached_sms[dev] == 0 || cached_smem[dev] != smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return TQ_ERR_CUDA;
    int sms = 0, occ = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem) != cudaSuccess)
      return TQ_ERR_CUDA;
    if (occ < 1) return TQ_ERR_UNSUPPORTED;
    cached_occ[dev] = occ;
    cached_smem[dev] = smem;
    cached_sms[dev] = sms;
  }
  const int ctas = min(kMaxCtas, cached_sms[dev] * cached_occ[dev]);
  kern<<<ctas, kThreads, smem, stream>>>(p, p1_ctas);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  if (ctas_out) *ctas_out = ctas;
  return TQ_OK;
}

template <int KB, int VB, int NB, int GQ>
int dispatch_modes(const DecodeParams& p, cudaStream_t stream) {
  if (p.sparse_thr > 0.0f) {
    int p1 = 0;
    int st = run<KB, 2, NB, kScores, GQ>(p, stream, 0, &p1);
    if (st != TQ_OK) return st;
    return run<2, VB, NB, kSparseV, GQ>(p, stream, p1, nullptr);
  }
  return run<KB, VB, NB, kFused, GQ>(p, stream, 0, nullptr);
}

template <int KB, int VB, int NB>
int dispatch_gq(const DecodeParams& p, cudaStream_t stream) {
  if (p.q_heads / p.kv_heads * p.n_q <= 4) return dispatch_modes<KB, VB, NB, 4>(p, stream);
  return dispatch_modes<KB, VB, NB, 8>(p, stream);
}

template <int KB, int VB>
int dispatch_nb(const DecodeParams& p, cudaStream_t stream) {
  switch (p.head_dim / kBlock) {
    case 1: return dispatch_gq<KB, VB, 1>(p, stream);
    case 2: return dispatch_gq<KB, VB, 2>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

template <int KB>
int dispatch_vb(const DecodeParams& p, cudaStream_t stream) {
  switch (p.v_bits) {
    case 2: return dispatch_nb<KB, 2>(p, stream);
    case 3: return dispatch_nb<KB, 3>(p, stream);
    case 4: return dispatch_nb<KB, 4>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode(const DecodeParams& p, cudaStream_t stream) {
  switch (p.k_bits) {
    case 2: return dispatch_vb<2>(p, stream);
    case 3: return dispatch_vb<3>(p, stream);
    case 4: return dispatch_vb<4>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
