// Decode attention over the packed TurboQuant cache (single- or multi-token
// queries, GQA, per-sequence lengths, optional exact sparse-V, optional
// in-launch append of the newest token).  Included by one translation unit per
// K bit width (tq_decode_k{2,3,4}.cu).
//
// Method: "llama-tq" article, K-cache section (Q.K in the Hadamard domain,
// no K dequantisation); "TheTom/llama-cpp-turboquant" README, table "量化类型"
// (WHT + codebook on 128-element blocks) and "压缩策略" (sparse-V dequant);
// "TurboQuant+" section "注意力门控稀疏V解压" (skipped V counts as zero).
//
// Kernel design (sm_100a):
//  * Work = (unit, 16-token tile), unit = (batch, kv-head, group of <= 8
//    query heads).  All tiles of all units are laid end to end and cut into
//    one range per persistent CTA, one 16-warp CTA per SM.  The cut weighs each
//    tile 1 and each unit boundary more (see Split).  A CTA writes
//    one partial (m, l, acc) per unit it touches; the CTA that completes a unit
//    (atomic tile count) merges the partials in a fixed order, so results do
//    not depend on scheduling.
//  * Each warp streams its own future tiles into a private ring of slots in
//    shared memory with 16-byte cp.async (4-byte for the fp16 norms), one copy
//    group per tile, zero-filled past the end of the sequence.  Each run of
//    four tokens is placed with a small gap so that the lanes' reads of a slot
//    are free of bank conflicts.  (A ring filled by bulk copies, one lane per
//    run, with a per-slot mbarrier was measured: its waits, fences and
//    branches cost more instructions per tile than the per-lane copies.)
//  * Scores: S[16 tok x 8 cols] = Kc[16 x 128] . Qhat[128 x 8] with
//    mma.sync m16n8k16 (f16 in, f32 accumulate).  Codes become f16 A fragments
//    through shared-memory tables replicated per lane (every lane hits its own
//    bank): a 3-bit code pair indexes a 64-entry table whose address is a
//    shift and one three-input logic op; 4-bit code pairs and 2-bit code quads
//    are whole bytes, so one byte permute builds the address, and a 2-bit quad
//    returns two fragment registers in one 64-bit load.
//  * Online softmax in the log2 domain with a lazy rescale (only when the
//    running max grows by more than 2^kTau); weights carry 2^-7, the 1/128 of
//    the block norm, so the P fragments are p * nV directly.
//  * P.V with up to four heads per kv-head (GQ = 4): the 8 MMA columns are
//    (head, dim parity) pairs, so each V A-fragment register is one token's
//    pair of adjacent dims straight from the table.  With more heads (GQ = 8)
//    V is re-paired by token.  V stays in the rotated domain until the end.
//  * Sparse-V is exact and two-pass: pass 1 stores log2-domain scores and
//    per-partial (m, l); pass 2 forms each head's maximum M and log-sum-exp,
//    drops the positions whose normalised weight 2^(s - LSE) is below the
//    threshold and accumulates V with weights 2^(s - M - 7), as the fused
//    pass does, dividing by the head's sum at the end.
//  * V v3 (VO): each tile also carries its 16 tokens' outlier-channel values
//    (fp16); one more MMA per tile sums them with the plain weights, and the
//    emit overwrites those channels of the output.
//  * V v2 (V2): the V codes are trellis pair fields; a pair's two levels are
//    indexed by the stream bits that end with its field (the two branch bits
//    before it included), so V fragments come from pair tables as in v1.
//  * The tail has no block-wide merge stage: warp h merges the 16 warps'
//    partials of head h and either emits the head (inverse rotation in
//    registers) or publishes the CTA's partial; the completing CTA's warp h
//    merges every partial of head h in one pass of loads and emits it.
#pragma once

#include <cuda_fp16.h>

#include <type_traits>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace dec {
namespace {  // every including translation unit keeps its own copy

#ifndef TQ_SWITCH_TILES
#define TQ_SWITCH_TILES 96  // cost of starting another unit inside a CTA, in tiles
#endif
#ifndef TQ_APPEND_TILES
#define TQ_APPEND_TILES 64  // extra cost of a unit end whose CTA appends the new token, in tiles
#endif
#ifndef TQ_KCHAINS
#define TQ_KCHAINS 2  // independent accumulator chains of the score MMAs
#endif
constexpr int kKChains = TQ_KCHAINS;
constexpr int kCWarps = kDecodeWarps;   // warps per CTA
constexpr int kThreads = 32 * kCWarps;
constexpr int kMaxDepth = 4;            // tiles per warp ring, at most (the planner may choose fewer)
constexpr uint32_t kSmemBase = 1024;    // shared-window address of dynamic shared memory
constexpr uint32_t kMaxDyn = 227 * 1024;
constexpr float kTau = 6.0f;            // lazy-rescale threshold (log2 units)
constexpr float kPShift = 7.0f;         // weights carry 2^-7 = 1/128
constexpr long long kSwitchTiles = TQ_SWITCH_TILES;
constexpr long long kAppendTiles = TQ_APPEND_TILES;
constexpr long long kMinCtaTiles = 32;  // a CTA per this many tiles at most (two per warp)

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
__device__ __forceinline__ float4 ld_s128f(uint32_t a) {
  float4 x;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w) : "r"(a));
  return x;
}
__device__ __forceinline__ void st_s32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void st_s64(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}

// Table reads.  Not volatile: the tables do not change after the prologue,
// and every address depends on code words read (volatile, after the copy
// waits) from the ring, so the compiler may schedule these freely.
__device__ __forceinline__ uint32_t ld_table(uint32_t a) {
  uint32_t x;
  asm("ld.shared.b32 %0, [%1];" : "=r"(x) : "r"(a));
  return x;
}
__device__ __forceinline__ uint2 ld_table2(uint32_t a) {
  uint2 x;
  asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(x.x), "=r"(x.y) : "r"(a));
  return x;
}

// ------------------------------------------------------- code -> address --
//
// Table layouts (entry f of lane l):
//  * 3-bit pair table ("OR table"): 64 entries x 128 B, f = two codes (low
//    code in bits 0..2); half2(c[lo], c[hi]) at T + f*128 + l*4.  T is
//    aligned to 8 KiB, so the address is (field << 7) OR (T + l*4).
//  * byte tables: 256 entries x 256 B inside a 64 KiB-aligned region R, one
//    side in each 128-byte half (K at +0, V at +128).  A 4-bit pair byte f
//    holds half2(c[f & 15], c[f >> 4]) at R + f*256 + half + l*4; a 2-bit quad
//    byte holds half2(c0, c1), half2(c2, c3) (c_i = code i of the byte) at
//    R + f*256 + half + (l % 16)*8.  The address is the byte of the code word
//    put in bits 8..15 of this lane's base word by one byte permute.

// Address of the 3-bit pair whose field starts at bit `pos` of the word array
// w: the field shifted to bit 7 (one funnel shift by pos - 7 when it continues
// in the next word: such a field starts at bit 27 or later), then the mask and
// the lane base in one three-input logic op.
__device__ __forceinline__ uint32_t addr3(const uint32_t* w, int pos, uint32_t lb) {
  const int wi = pos >> 5, sh = pos & 31;
  uint32_t x;
  if (sh + 6 > 32) x = __funnelshift_r(w[wi], w[wi + 1], sh - 7);
  else x = sh >= 7 ? w[wi] >> (sh - 7) : w[wi] << (7 - sh);
  return (x & (63u << 7)) | lb;
}

// V v2 (trellis codes) pair tables: the index of pair p of a lane's window is
// the W = 2b + 2 stream bits that end with the pair's field (the two branch
// bits before the pair, then the field: j_a, j_b, beta_a, beta_b); entry f
// holds half2(level a, level b) at T + (f << S) + l*4, S = 7 for a table of
// its own (T aligned to 2^(W+7)) or S = 8 in the free V half of a byte-table
// region (T = region + 128, the region 64 KiB-aligned).
template <int W, int S>
__device__ __forceinline__ uint32_t addr_field(const uint32_t* w, int pos, uint32_t lb) {
  const int wi = pos >> 5, sh = pos & 31;
  uint32_t x;
  if (sh + W > 32) x = __funnelshift_r(w[wi], w[wi + 1], sh) << S;
  else x = sh >= S ? w[wi] >> (sh - S) : w[wi] << (S - sh);
  return (x & (((1u << W) - 1u) << S)) | lb;
}
template <int B, int S>
__device__ __forceinline__ uint2 pair2_frag_v2(const uint32_t* w, int r, uint32_t lb) {
  static_assert(B == 2 || B == 3, "v2 rates");
  return make_uint2(ld_table(addr_field<2 * B + 2, S>(w, 2 * B * (2 * r), lb)),
                    ld_table(addr_field<2 * B + 2, S>(w, 2 * B * (2 * r + 1), lb)));
}

// Address of the byte-table entry indexed by the byte at bit `pos` (a
// multiple of 8) of w, for the lane base word lbw.
__device__ __forceinline__ uint32_t addr_byte(const uint32_t* w, int pos, uint32_t lbw) {
  const uint32_t k = (uint32_t)((pos >> 3) & 3);
  return prmt(w[pos >> 5], lbw, 0x7604u | (k << 4));
}

// Fragment registers of code pairs: pair q (codes 2q, 2q+1) of the window w
// of a B-bit code stream.  Pair2 returns pairs 2r and 2r+1 together.
template <int B>
__device__ __forceinline__ uint32_t pair_frag(const uint32_t* w, int q, uint32_t lb) {
  static_assert(B == 3 || B == 4, "pair tables");
  if constexpr (B == 3)
    return ld_table(addr3(w, 6 * q, lb));
  else
    return ld_table(addr_byte(w, 8 * q, lb));
}
template <int B>
__device__ __forceinline__ uint2 pair2_frag(const uint32_t* w, int r, uint32_t lb) {
  if constexpr (B == 2) {
    return ld_table2(addr_byte(w, 8 * r, lb));
  } else {
    return make_uint2(pair_frag<B>(w, 2 * r, lb), pair_frag<B>(w, 2 * r + 1, lb));
  }
}

// ---------------------------------------------------------- async copies --

// 4-byte global -> shared copy; src_bytes < 4 zero-fills the rest (0: no read).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// 16-byte global -> shared copy with the same zero-fill rule.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Wait until at most depth - 1 of this thread's copy groups are pending.
__device__ __forceinline__ void cp_async_wait_depth(uint32_t depth) {
  if (depth >= 4) cp_async_wait<3>();
  else if (depth == 3) cp_async_wait<2>();
  else cp_async_wait<1>();
}

// Predicated forms (one instruction, no branch): `on` selects the lanes.
__device__ __forceinline__ void cp_async16_if(bool on, uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile(
      "{ .reg .pred q; setp.ne.b32 q, %3, 0;\n"
      "@q cp.async.cg.shared.global [%0], [%1], 16, %2; }" ::"r"(dst),
      "l"(src), "r"(src_bytes), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void cp_async4_if(bool on, uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile(
      "{ .reg .pred q; setp.ne.b32 q, %3, 0;\n"
      "@q cp.async.ca.shared.global [%0], [%1], 4, %2; }" ::"r"(dst),
      "l"(src), "r"(src_bytes), "r"((uint32_t)on)
      : "memory");
}

__device__ __forceinline__ void consumer_sync() { __syncthreads(); }

// Programmatic dependent launch.  A launch made with programmatic stream
// serialisation may start while the kernel before it in the stream is still
// running, once every CTA of that kernel has triggered (or exited).
// pdl_wait() returns when the earlier kernel has completed and its writes are
// visible; without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <int B>
struct Fmt {
  static constexpr int kBlockBytes = 16 * B;
};

// ------------------------------------------------------ slot layout (host) --
//
// A ring slot holds one 16-token tile: K codes, V codes (each as four runs of
// four tokens, runs placed with the gaps below), K norms and V norms.  The
// gaps make the lanes' reads of the slot bank-conflict free (found by
// exhaustive search over 16-byte gaps for every bit width and block count).
inline void run_gaps(bool is_k, int bits, int nb, uint32_t (&g)[4]) {
  static const uint32_t k_tab[3][2][4] = {{{0, 32, 32, 64}, {0, 32, 32, 64}},    // 2-bit
                                          {{0, 0, 16, 16}, {0, 16, 32, 48}},     // 3-bit
                                          {{0, 0, 0, 0}, {0, 0, 0, 0}}};         // 4-bit
  static const uint32_t v_tab[3][2][4] = {{{0, 32, 64, 96}, {0, 32, 64, 96}},
                                          {{0, 0, 0, 0}, {0, 0, 48, 48}},
                                          {{0, 32, 64, 96}, {0, 32, 64, 96}}};
  const uint32_t(&t)[4] = (is_k ? k_tab : v_tab)[bits - 2][nb - 1];
  for (int j = 0; j < 4; ++j) g[j] = t[j];
}

// ------------------------------------------------------------------ WHT --

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
// is the shared address of 16 words of this warp's scratch.
__device__ __noinline__ void append_block(const DecodeParams& p, int side, int blk, size_t row,
                                          size_t tok, int lane, uint32_t stage) {
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
  if (lane < 4 * bits) st_s32(stage + 4u * lane, 0u);
  __syncwarp();
  const int bit = 4 * bits * lane, wi = bit >> 5, sh = bit & 31;
  uint32_t* st = static_cast<uint32_t*>(__cvta_shared_to_generic(stage));
  atomicOr(st + wi, field << sh);
  if (sh + 4 * bits > 32) atomicOr(st + wi + 1, field >> (32 - sh));
  __syncwarp();
  uint32_t* dst = reinterpret_cast<uint32_t*>(p.app_codes[side] + (tok * nb + blk) * 16 * bits);
  if (lane < 4 * bits) dst[lane] = ld_s32(stage + 4u * lane);
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
// CTAs.  Every unit's tiles cost 1 each and each unit boundary costs sw more
// (kSwitchTiles: the query preparation, the drained copy ring, the partial's
// merge and publication; plus kAppendTiles in a decode step, whose CTA that
// holds a unit's last tile first appends the new token), so a CTA whose range
// spans a boundary gets fewer tiles: CTA c takes the tiles whose cost falls in
// [c, c+1) * Ctot / P.  The cost before batch entry b is
// UB * (prefix[b] + sw * b).  A cost that
// falls between two units maps to the start of the second, so a cut there
// adds no segment.  Results do not depend on the split (each part is computed
// and merged in a fixed order); it only moves where the CTAs end.

// floor(a / b) for 0 <= a, 0 < b, both below 2^52, from the reciprocal
// inv_b ~= 1 / b: the double estimate is within one of the exact quotient and
// integer steps correct it (a 64-bit integer division, or a double division,
// is a long instruction sequence on the GPU).
__device__ __forceinline__ long long qdiv(long long a, long long b, double inv_b) {
  long long q = (long long)((double)a * inv_b);
  while (q > 0 && q * b > a) --q;
  while ((q + 1) * b <= a) ++q;
  return q;
}
// floor(a / b) when the quotient is below 2^20: a single-precision estimate
// from the hardware reciprocal, then exact integer steps.
__device__ __forceinline__ long long qdiv_small(long long a, long long b) {
  long long q = (long long)((float)a * __frcp_rn((float)b));
  if (q < 0) q = 0;
  while (q > 0 && q * b > a) --q;
  while ((q + 1) * b <= a) ++q;
  return q;
}

struct Split {
  const int* prefix;  // [B+1] tiles per batch entry, exclusive prefix (shared memory)
  int B, UB;
  long long P, T, Ctot, sw;
  double invP, invCtot, invUB;
  __device__ Split(const int* pre, int batch, int ub, long long parts, long long switch_cost)
      : prefix(pre), B(batch), UB(ub), P(parts), sw(switch_cost) {
    T = (long long)pre[batch] * ub;
    Ctot = (long long)ub * ((long long)pre[batch] + sw * batch);
    invP = 1.0 / (double)P;
    invCtot = Ctot > 0 ? 1.0 / (double)Ctot : 0.0;
    invUB = 1.0 / (double)ub;
  }
  // first tile of part c (c = P gives T)
  __device__ long long start(long long c) const {
    if (c >= P) return T;
    const long long y = qdiv(c * Ctot, P, invP);
    int bl = 0, bh = B;  // largest b with cost(b) <= y
    while (bh - bl > 1) {
      const int mid = (bl + bh) >> 1;
      if ((long long)UB * (prefix[mid] + sw * mid) <= y) bl = mid; else bh = mid;
    }
    const long long nt = prefix[bl + 1] - prefix[bl];
    const long long rem = y - (long long)UB * (prefix[bl] + sw * bl);
    const long long r = qdiv_small(rem, nt + sw), t = rem - r * (nt + sw);
    return (long long)UB * prefix[bl] + r * nt + min(t, nt);
  }
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
    const long long r = qdiv_small(off, nt), t = off - r * nt;
    const long long F = (long long)UB * (prefix[bl] + sw * bl) + r * (nt + sw) + t;
    const long long c = qdiv((F + 1) * P - 1, Ctot, invCtot);
    return c < P - 1 ? c : P - 1;
  }
};

// Bits of the parts c0 .. c0+31 (of parts c_first .. c_last, plus the part
// after, for the end test) whose tile range is empty, by one warp: bit j of
// the result is part c0 + j.  Every lane returns the same word.
__device__ __forceinline__ uint32_t empty_bits(const Split& sp, long long c0, long long c_last, int lane) {
  const long long c = c0 + lane;
  const long long s0 = c <= c_last + 1 ? sp.start(c) : 0;  // start(c_last + 1) ends the last part
  long long s1 = __shfl_down_sync(0xffffffffu, s0, 1);
  if (lane == 31 && c <= c_last) s1 = sp.start(c + 1);
  return __ballot_sync(0xffffffffu, c <= c_last && s0 == s1);
}

// Per-head (M, L) = (max m, sum l * 2^(m - M)) over the partials c_first ..
// c_last of one unit, by one warp: lanes split the partials, then a warp
// reduction in a fixed order.  Partials with an empty range are skipped.
__device__ __forceinline__ float2 unit_ml_warp(const float* slot_ml, long long c_first, long long c_last,
                                               const Split& sp, long long unit, int hd, int lane) {
  float m = -INFINITY, l = 0.0f;
  for (long long c0 = c_first; c0 <= c_last; c0 += 32) {
    const uint32_t emp = empty_bits(sp, c0, c_last, lane);
    const long long c = c0 + lane;
    if (c <= c_last && !((emp >> lane) & 1u)) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(slot_ml + ((c + unit) * kMaxGroup + hd) * 2));
      if (ml.x != -INFINITY) {
        if (ml.x > m) {
          l = l * ex2(m - ml.x) + ml.y;
          m = ml.x;
        } else {
          l += ml.y * ex2(ml.x - m);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o), lo = __shfl_xor_sync(0xffffffffu, l, o);
    const float M = fmaxf(m, mo);
    l = (M == -INFINITY) ? 0.0f : l * ex2(m - M) + lo * ex2(mo - M);
    m = M;
  }
  return make_float2(m, l);
}

// Where tile x of the flattened (unit, tile) space lies.
struct Segment {
  int b, r, nt, unit, kvh, hg, h0, Gu, len, seg_lo, seg_hi;
  long long Su;
};

__device__ __forceinline__ Segment locate(long long x, long long hi, const int* prefix, int batch,
                                          int UB, double invUB, int n_hg, int G, int seq_cap,
                                          const int32_t* seq_lens) {
  Segment s;
  const long long y = qdiv(x, UB, invUB);  // in units of "tiles per batch entry"
  int bl = 0, bh = batch;      // largest b with prefix[b] <= y
  while (bh - bl > 1) {
    const int mid = (bl + bh) >> 1;
    if (prefix[mid] <= y) bl = mid; else bh = mid;
  }
  s.b = bl;
  s.nt = prefix[bl + 1] - prefix[bl];
  const long long TB = (long long)prefix[bl] * UB;
  s.r = (int)qdiv_small(x - TB, s.nt);
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

// Per-lane tile registers.  MMA row r of the score product holds token pi(r):
// pi(R) = 2R, pi(R + 8) = 2R + 1, so lane (R = lane/4, g = lane%4) holds the
// adjacent tokens 2R and 2R+1 (their norms are one 32-bit word).  The P.V
// product then needs, in lane g, tokens 4g, 4g+2, 4g+1 and 4g+3.
//   k[rr][blk]  : codes of dims [32g, 32g+32) of token 2R+rr (KB words);
//   v[tt][blk]  : codes of dims [16R, 16R+16) of token 4g + toff(tt) (2 words);
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
template <int KB, int VB, int NB, bool LOADK, bool LOADV, bool V2 = false>
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
    (void)vsh;
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const int toff = ((tt & 1) << 1) + (tt >> 1);  // vtok(g, tt) - 4g
        const uint32_t s = vs + (toff * NB + blk) * Fmt<VB>::kBlockBytes;
        if constexpr (V2) {
          // v2: the lane's fields (bits [16b R, 16b R + 16b) of the block's
          // stream) and the two bits before them (zero before the block)
          if constexpr (VB == 3) {
            const uint32_t w0 = ld_s32(s), w1 = ld_s32(s + 4);
            if (R & 1) {  // the window starts at bit 14 of w0
              r.v[tt][blk][0] = __funnelshift_r(w0, w1, 14);
              r.v[tt][blk][1] = w1 >> 14;
            } else {
              const uint32_t pw = R > 0 ? ld_s32(s - 4) : 0u;
              r.v[tt][blk][0] = __funnelshift_r(pw, w0, 30);
              r.v[tt][blk][1] = __funnelshift_r(w0, w1, 30);
            }
          } else {
            const uint32_t w0 = ld_s32(s);
            const uint32_t pw = R > 0 ? ld_s32(s - 4) : 0u;
            r.v[tt][blk][0] = __funnelshift_r(pw, w0, 30);
            r.v[tt][blk][1] = w0 >> 30;
          }
        } else if constexpr (VB == 4) {
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

// Query scratch layout: row hr of qhat, dims [32g + 4j, 32g + 4j + 4) of block
// blk at float hr * qrow + blk * 144 + g * 36 + 4 j.  The 16-byte groups of
// one row land 9 groups apart per g and a row stride of qrow / 4 = 4 (mod 8)
// groups, so the eight lanes of each 16-byte read phase hit eight distinct
// bank groups.
template <int NB>
struct QScratch {
  static constexpr int kRow = NB == 1 ? 144 : 304;  // floats per row
  static __device__ __forceinline__ int at(int hr, int blk, int g, int j) {
    return hr * kRow + blk * 144 + g * 36 + 4 * j;
  }
};

// Misc shared area (floats / ints), offsets in 4-byte words.
struct Misc {
  static constexpr int kWm = 0;                              // warp m [kCWarps][8]
  static constexpr int kWl = kWm + kCWarps * kMaxGroup;      // warp l [kCWarps][8]
  static constexpr int kQexp = kWl + kCWarps * kMaxGroup;    // [8]
  static constexpr int kLse = kQexp + kMaxGroup;             // [8]
  static constexpr int kUm = kLse + kMaxGroup;               // [8]
  static constexpr int kUl = kUm + kMaxGroup;                // [8]
  static constexpr int kWtot = kUl + kMaxGroup;              // [kCWarps]
  static constexpr int kWords = kWtot + kCWarps;
};

// --------------------------------------------------------------- the kernel --

template <int KB, int VB, int NB, int MODE, int GQ, bool VO, bool V2>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ DecodeParams p, int p1_ctas) {
  constexpr int D = NB * kBlock;
  // floats per head of a published partial: acc, then (v3) the outlier sums
  constexpr int PD = VO ? acc_stride(D) : D;
  constexpr bool HASK = MODE != kSparseV, HASV = MODE != kScores;
  static_assert(!VO || HASV, "v3 outliers ride with the V pass");
  static_assert(!V2 || (HASV && !VO && (VB == 2 || VB == 3)), "v2 trellis V: rates 2 and 3");
  // a v2 table shares the byte-table region of a 2- or 4-bit K side
  constexpr int V2S = (V2 && HASK && (KB == 2 || KB == 4)) ? 8 : 7;
  constexpr int KBB = Fmt<KB>::kBlockBytes, VBB = Fmt<VB>::kBlockBytes;
  // GQ == 4 (at most four query heads per unit): score columns 4..7 repeat
  // heads 0..3, and the V products use the eight MMA columns as (head, dim
  // parity) pairs, so V fragments come straight from the table.  GQ == 8:
  // one column per head, V fragments re-paired by token.
  static_assert(GQ == 4 || GQ == 8, "GQ");
  static_assert(kCWarps >= 2 * NB && kCWarps >= kMaxGroup, "warp roles");
  constexpr bool kDup = GQ == 4;
  constexpr int kMT = kDup ? 4 : 8;  // V accumulator tiles per 128-block
  extern __shared__ __align__(1024) uint8_t smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = lane >> 2, g = lane & 3;
  const SmemPlan& sm = p.sm;

  // The next launch in the stream may start its prologue on any SM this
  // launch leaves; everything it reads or writes that this launch touches
  // comes after its pdl_wait().
  pdl_trigger();

  // The plan's addresses assume where dynamic shared memory starts; a
  // mismatch (another driver's layout) is reported, never used.
  {
    uint32_t dyn;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    if (smem_addr(smem) != sm.base || dyn < sm.bytes) {
      if (tid == 0 && p.status) atomicOr(p.status, TQ_DEV_INTERNAL);
      return;
    }
  }
  auto gptr = [&](uint32_t a) { return smem + (a - sm.base); };
  float* res = reinterpret_cast<float*>(gptr(sm.res));
  float* misc = reinterpret_cast<float*>(gptr(sm.misc));
  float* w_m = misc + Misc::kWm;
  float* w_l = misc + Misc::kWl;
  int* qexp = reinterpret_cast<int*>(misc + Misc::kQexp);
  float* u_lse = misc + Misc::kLse;  // sparse-V pass 2, per head of the unit: log2 sum_t 2^s_t,
  float* u_m = misc + Misc::kUm;      // the maximum score M
  float* u_l = misc + Misc::kUl;      // and 2^-7 sum_t 2^(s_t - M)
  int* wtot = reinterpret_cast<int*>(misc + Misc::kWtot);
  int* prefix = reinterpret_cast<int*>(gptr(sm.prefix));  // [B+1] tiles per batch, prefix
  const uint32_t depth = sm.depth;

  // Lane base words of the code tables.
  uint32_t lbK = 0, lbV = 0;
  if constexpr (KB == 3) lbK = sm.lut_k + 4u * lane;
  if constexpr (KB == 4) lbK = sm.lut_k + 4u * lane;
  if constexpr (KB == 2) lbK = sm.lut_k + 8u * (lane & 15);
  if constexpr (VB == 3 || V2) lbV = sm.lut_v + 4u * lane;
  if constexpr (VB == 4) lbV = sm.lut_v + 4u * lane;
  if constexpr (VB == 2 && !V2) lbV = sm.lut_v + 8u * (lane & 15);

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

  // ---- code tables, filled by the threads [t_first, t_first + t_count) ------
  auto fill_table = [&](int bits, const float* cent, uint32_t base, uint32_t half, int t_first, int t_count) {
    const int t = tid - t_first;
    if (bits == 3) {  // 64 pairs x 32 lanes
      for (int e = t; e < 64 * 32; e += t_count) {
        const int f = e >> 5;
        *reinterpret_cast<uint32_t*>(gptr(base + 4u * e)) = pack_half2(cent[f & 7], cent[f >> 3]);
      }
    } else if (bits == 4) {  // 256 pairs x 32 lanes
      for (int e = t; e < 256 * 32; e += t_count) {
        const int f = e >> 5, l = e & 31;
        *reinterpret_cast<uint32_t*>(gptr(base + 256u * f + half + 4u * l)) = pack_half2(cent[f & 15], cent[f >> 4]);
      }
    } else {  // 2 bits: 256 quads x 16 lanes
      for (int e = t; e < 256 * 16; e += t_count) {
        const int f = e >> 4, l = e & 15;
        *reinterpret_cast<uint2*>(gptr(base + 256u * f + half + 8u * l)) =
            make_uint2(pack_half2(cent[f & 3], cent[(f >> 2) & 3]), pack_half2(cent[(f >> 4) & 3], cent[f >> 6]));
      }
    }
  };
  // v2 pair table: entry f = (beta_{-2}, beta_{-1}, j_a, j_b, beta_a, beta_b)
  // from bit 0 up; level index 4 j + subset, subset = beta_{i-1} + 2 (beta_i
  // xor beta_{i-2}) (the trellis of the v2 encoder); cent = doubled codebook
  auto fill_table_v2 = [&](int bits, const float* cent, uint32_t base, int t_first, int t_count) {
    const int t = tid - t_first;
    const int jw = bits - 1, n = 1 << (2 * bits + 2);
    for (int e = t; e < n * 32; e += t_count) {
      const int f = e >> 5, l = e & 31;
      const int w0 = f & 1, w1 = (f >> 1) & 1;
      const int ja = (f >> 2) & ((1 << jw) - 1), jb = (f >> (2 + jw)) & ((1 << jw) - 1);
      const int ba = (f >> (2 + 2 * jw)) & 1, bb = (f >> (3 + 2 * jw)) & 1;
      const int sa = w1 + 2 * (ba ^ w0), sb = ba + 2 * (bb ^ w1);
      *reinterpret_cast<uint32_t*>(gptr(base + ((uint32_t)f << V2S) + 4u * l)) =
          pack_half2(cent[4 * ja + sa], cent[4 * jb + sb]);
    }
  };
  auto fill_tables = [&](int t_first, int t_count) {
    if (tid < t_first || tid >= t_first + t_count) return;
    if constexpr (HASK)
      fill_table(KB, p.kcent, KB == 3 ? sm.lut_k : sm.lut_k & ~255u, KB == 3 ? 0u : (sm.lut_k & 128u), t_first, t_count);
    if constexpr (HASV && V2) fill_table_v2(VB, p.vcent, sm.lut_v, t_first, t_count);
    if constexpr (HASV && !V2)
      fill_table(VB, p.vcent, VB == 3 ? sm.lut_v : sm.lut_v & ~255u, VB == 3 ? 0u : (sm.lut_v & 128u), t_first, t_count);
  };

  // ---- lengths: clamp, tiles per batch entry, exclusive prefix ------------
  // (the code tables are filled while this thread's length loads are in
  // flight; the barrier below publishes them)
  {
    const int B = p.batch;
    const int per = (B + kThreads - 1) / kThreads;  // at most kMaxBatch / kThreads = 4
    int local = 0;
    const int b_lo = tid * per;
    int lens_r[kMaxBatch / kThreads];
#pragma unroll
    for (int i = 0; i < kMaxBatch / kThreads; ++i)
      lens_r[i] = (i < per && b_lo + i < B) ? __ldg(p.seq_lens + b_lo + i) : 0;
    fill_tables(0, kThreads);
#pragma unroll
    for (int i = 0; i < kMaxBatch / kThreads; ++i) {
      if (i >= per || b_lo + i >= B) break;
      int len = lens_r[i];
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
    __syncthreads();  // also publishes the tables and the barrier initialisation
  }
  // the cost of a unit boundary: a decode step (new rows given) appends there
  const long long sw = kSwitchTiles + (p.kv_new[0] != nullptr ? kAppendTiles : 0);
  const Split sp(prefix, p.batch, UB, gridDim.x, sw);  // this launch's split
  const long long T = sp.T;

  const long long lo = T > 0 ? sp.start(blockIdx.x) : 0, hi = T > 0 ? sp.start(blockIdx.x + 1) : 0;
  const int cw = warp;
  const uint32_t wring_s = sm.ring[cw];  // this warp's ring
  const uint32_t slot_bytes = sm.slot_bytes;

  // This lane's first K / V word inside a slot (tokens 2R, 2R+1 sit in K run
  // R / 2; tokens 4g..4g+3 are V run g).
  uint32_t koff = 0, voff = 0;
  if constexpr (HASK) {
    const uint32_t kr = (R >> 1) == 0 ? sm.kc_off[0] : (R >> 1) == 1 ? sm.kc_off[1] : (R >> 1) == 2 ? sm.kc_off[2] : sm.kc_off[3];
    koff = kr + (uint32_t)(((2 * R) & 3) * NB * KBB + g * KB * 4);
  }
  if constexpr (HASV) {
    const int vlane = VB == 4 ? 8 * R : (VB == 3 ? 4 * ((3 * R) >> 1) : 4 * R);
    const uint32_t vr = g == 0 ? sm.vc_off[0] : g == 1 ? sm.vc_off[1] : g == 2 ? sm.vc_off[2] : sm.vc_off[3];
    voff = vr + (uint32_t)vlane;
  }
  // Copy plan of this lane: a tile's codes are 16-byte chunks, contiguous in
  // the cache row; lane l copies chunks l, l + 32, ... of K and of V.  Chunk c
  // of token t lands at the token's place in its 4-token run of the slot.
  constexpr int kCPTK = NB * KB, kCPTV = NB * VB;  // chunks per token
  constexpr int kCK = HASK ? kTile * kCPTK : 0, kCV = HASV ? kTile * kCPTV : 0;
  constexpr int kRK = (kCK + 31) / 32, kRV = (kCV + 31) / 32;  // copy rounds
  uint32_t kdst[kRK > 0 ? kRK : 1], vdst[kRV > 0 ? kRV : 1];
  auto run_off = [&](const uint32_t(&offs)[4], int t) {
    const int j = t >> 2;
    return j == 0 ? offs[0] : j == 1 ? offs[1] : j == 2 ? offs[2] : offs[3];
  };
#pragma unroll
  for (int r = 0; r < kRK; ++r) {
    const int c = min(lane + 32 * r, kCK - 1), t = c / kCPTK;
    kdst[r] = run_off(sm.kc_off, t) + (uint32_t)((t & 3) * NB * KBB + 16 * (c % kCPTK));
  }
#pragma unroll
  for (int r = 0; r < kRV; ++r) {
    const int c = min(lane + 32 * r, kCV - 1), t = c / kCPTV;
    vdst[r] = run_off(sm.vc_off, t) + (uint32_t)((t & 3) * NB * VBB + 16 * (c % kCPTV));
  }
  // Norm copies: lanes 0..8NB-1 copy K norms, the next 8NB lanes V norms
  // (4 bytes each = two fp16 norms).
  constexpr int kNL = 8 * NB;
  const bool kn_lane = HASK && lane < kNL;
  const bool vn_lane = HASV && (HASK ? (lane >= kNL && lane < 2 * kNL) : lane < kNL);
  const bool norm_lane = kn_lane || vn_lane;
  const int nidx = lane % kNL;
  const uint32_t ndst = (kn_lane ? sm.kn_off : sm.vn_off) + 4u * (uint32_t)nidx;
  // V v3 outlier values: a tile's run is 16 tokens x kp fp16 (kp = 8 or 16),
  // copied as 16-byte chunks (lane l takes chunk l).  Inside each 128-byte
  // line of the slot the chunk index is XOR-ed with the line's low two bits,
  // so that the fragment loads (8 tokens of one parity x 4 channel pairs)
  // fall into 32 distinct banks.
  auto vo_swz = [](int c) { return (uint32_t)((c >> 3) * 128 + 16 * ((c & 7) ^ ((c >> 3) & 3))); };
  const int vo_kp = VO ? p.vo_kp : 8;
  const bool vo_lane = VO && lane < 2 * vo_kp;
  const uint32_t vo_dst = VO ? sm.vo_off + vo_swz(lane) : 0u;
  const int vo_tok = (lane * 8) / vo_kp;  // the token of chunk `lane`
  // A fragment words (token parity, channel half): lane (R, g) reads channels
  // 8 half + 2g, +1 of token 2R + parity; transposed, they become the MMA's
  // rows (channels) by its k (tokens, in the P^T order of the V products)
  uint32_t vo_a[4] = {0u, 0u, 0u, 0u};
  if constexpr (VO) {
#pragma unroll
    for (int par = 0; par < 2; ++par)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        if (hf == 0 || vo_kp == 16)
          vo_a[2 * par + hf] = sm.vo_off + vo_swz((2 * R + par) * vo_kp / 8 + hf) + 4u * g;
  }

  // The warp's ring is used in order across all its segments: consumed tile
  // n sits in slot n % depth, kept incrementally (cslot for consumption,
  // islot for issue).  Each tile owns one cp.async group.
  uint32_t cslot = 0, islot = 0;

  // ---- query preparation: qhat = H.(s o q) (D1), as this lane's fp16 MMA
  // B fragments plus the per-column score multipliers.  One warp per head
  // row: lane l holds dims 4l..4l+3 of every 128-block.  Uses res as scratch.
  // The raw query row of this warp (row j = cw of the unit, warps below the
  // row count), loaded at the segment start ahead of the tile copies so that
  // its latency overlaps them.
  constexpr int kQRows = kDup ? 4 : kMaxGroup;
  auto load_q_row = [&](int b, int h0, int Gu, float (&v)[NB][4]) {
    const int j = cw;
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      v[blk][0] = v[blk][1] = v[blk][2] = v[blk][3] = 0.0f;
      if (j < kQRows && j < Gu) {
        const size_t qi = vrow(b, h0 + j) * D + blk * kBlock + 4 * lane;
        if (p.q_f16) {
          const uint2 h = *reinterpret_cast<const uint2*>(reinterpret_cast<const __half*>(p.q) + qi);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
          const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
          v[blk][0] = a.x; v[blk][1] = a.y; v[blk][2] = c.x; v[blk][3] = c.y;
        } else {
          const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.q) + qi);
          v[blk][0] = a.x; v[blk][1] = a.y; v[blk][2] = a.z; v[blk][3] = a.w;
        }
      }
    }
  };
  auto prep_q = [&](const float (&qrow)[NB][4], uint32_t (&qf)[NB][8][2], float (&qmul)[2]) {
    float* qs = res;  // [kQRows] rows of scaled qhat (QScratch layout)
    if (cw < kQRows) {
      const int j = cw;
      float v[NB][4];
      const uint32_t sgn = p.sign_mask[lane >> 3] >> (4 * (lane & 7));  // signs of dims 4l..4l+3
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int k = 0; k < 4; ++k) v[blk][k] = ((sgn >> k) & 1u) ? -qrow[blk][k] : qrow[blk][k];
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
      for (int blk = 0; blk < NB; ++blk)  // dims 4l..4l+3: g = l / 8, j = l % 8
        *reinterpret_cast<float4*>(qs + QScratch<NB>::at(j, blk, lane >> 3, lane & 7)) =
            make_float4(v[blk][0] * sc, v[blk][1] * sc, v[blk][2] * sc, v[blk][3] * sc);
    }
    consumer_sync();
    const int hr = kDup ? (R & 3) : R;  // this lane's score column's head
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 q4 = *reinterpret_cast<const float4*>(qs + QScratch<NB>::at(hr, blk, g, j));
        qf[blk][j][0] = pack_half2(q4.x, q4.y);
        qf[blk][j][1] = pack_half2(q4.z, q4.w);
      }
    }
    qmul[0] = p.score_mult * ldexpf(1.0f, qexp[kDup ? (2 * g) & 3 : 2 * g]);
    qmul[1] = p.score_mult * ldexpf(1.0f, qexp[kDup ? (2 * g + 1) & 3 : 2 * g + 1]);
    consumer_sync();  // res and qexp are reused after this
  };

  // ---- D8: o = s o (H.acc) / L for one head row held by a warp (lane l
  // holds dims 4l..4l+3 of each block) ------------------------------------------
  auto emit_row = [&](float (&v)[NB][4], const float (&ov)[4], float div, int b, int vh) {
    wht_rows<NB>(v, lane);
    const uint32_t sgn = p.sign_mask[lane >> 3] >> (4 * (lane & 7));  // signs of dims 4l..4l+3
    const float inv = div > 0.0f ? 1.0f / div : 0.0f;  // div = 0: no position seen
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[blk][k] *= inv;
        if ((sgn >> k) & 1u) v[blk][k] = -v[blk][k];
      }
    }
    if constexpr (VO) {
      // v3: each outlier channel of the row is the weighted sum of its stored
      // values (original domain; the weights carry 2^-7, the divisor 128 more
      // than the plain sum of weights)
      const int32_t* chs = p.vo_channels + (size_t)(vh / Gv) * p.vo_k;
      const float oinv = 128.0f * inv;
#pragma unroll
      for (int t = 0; t < kOutlierMax; ++t) {
        if (t < p.vo_k) {
          const float val = __shfl_sync(0xffffffffu, ov[t & 3], t >> 2) * oinv;
          const int ch = __ldg(chs + t);
          if ((ch < 0 || ch >= D) && lane == 0 && p.status) atomicOr(p.status, TQ_DEV_CHANNEL_RANGE);
          const bool own = ch >= 0 && ch < D && lane == ((ch & (kBlock - 1)) >> 2);
#pragma unroll
          for (int blk = 0; blk < NB; ++blk)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (own && (ch >> 7) == blk && (ch & 3) == k) v[blk][k] = val;
        }
      }
    }
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      *reinterpret_cast<float4*>(p.out + vrow(b, vh) * D + blk * kBlock + 4 * lane) =
          make_float4(v[blk][0], v[blk][1], v[blk][2], v[blk][3]);
    }
  };

  // Up to here only the lengths, the parameters and shared memory were read.
  // The cache, the query, the workspace and the output may belong to the
  // launch before this one in the stream: wait for it to complete.
  pdl_wait();

  for (long long x = lo; x < hi;) {
    const Segment sg = locate(x, hi, prefix, p.batch, UB, sp.invUB, n_hg, Gv, p.seq_cap, p.seq_lens);
    const int b = sg.b, nt = sg.nt, unit = sg.unit, h0 = sg.h0, Gu = sg.Gu, len = sg.len;
    const int seg_lo = sg.seg_lo, seg_hi = sg.seg_hi;
    const long long Su = sg.Su;
    const size_t cache_row = (size_t)(b * p.kv_heads + sg.kvh) * p.seq_cap;
    const uint8_t* kcp = p.k_codes + cache_row * NB * KBB;
    const uint8_t* vcp = p.v_codes + cache_row * NB * VBB;
    const uint16_t* knp = p.k_norms + cache_row * NB;
    const uint16_t* vnp = p.v_norms + cache_row * NB;
    const uint8_t* ksrc = kcp + 16 * lane;  // chunk `lane` of tile 0
    const uint8_t* vsrc = vcp + 16 * lane;
    const uint16_t* nsrc = (kn_lane ? knp : vnp) + 2 * nidx;  // this lane's first norm of a tile
    const uint16_t* vop = VO ? p.vo_values + cache_row * vo_kp : nullptr;

    // Copy tile `tile` of this unit into this warp's next slot (one cp.async
    // group).
    auto issue = [&](int tile) {
      const uint32_t sb = wring_s + islot * slot_bytes;
      const int t0 = tile * kTile;
      const int nval = min(kTile, len - t0);  // >= 1
      const size_t kt = (size_t)t0 * kCPTK * 16, vt = (size_t)t0 * kCPTV * 16;
      if (nval == kTile) {
#pragma unroll
        for (int r = 0; r < kRK; ++r)
          cp_async16_if(32 * r + 32 <= kCK || lane + 32 * r < kCK, sb + kdst[r], ksrc + kt + 512 * r, 16u);
#pragma unroll
        for (int r = 0; r < kRV; ++r)
          cp_async16_if(32 * r + 32 <= kCV || lane + 32 * r < kCV, sb + vdst[r], vsrc + vt + 512 * r, 16u);
        cp_async4_if(norm_lane, sb + ndst, nsrc + (size_t)t0 * NB, 4u);
        if constexpr (VO) cp_async16_if(vo_lane, sb + vo_dst, vop + (size_t)t0 * vo_kp + 8 * lane, 16u);
      } else {
        // the last tile of a sequence: chunks and norms past the end are
        // zero-filled (a zero code and a zero norm contribute nothing)
#pragma unroll
        for (int r = 0; r < kRK; ++r) {
          const int c = lane + 32 * r;
          const bool ok = c / kCPTK < nval;
          cp_async16_if(c < kCK, sb + kdst[r], ok ? ksrc + kt + 512 * r : kcp, ok ? 16u : 0u);
        }
#pragma unroll
        for (int r = 0; r < kRV; ++r) {
          const int c = lane + 32 * r;
          const bool ok = c / kCPTV < nval;
          cp_async16_if(c < kCV, sb + vdst[r], ok ? vsrc + vt + 512 * r : vcp, ok ? 16u : 0u);
        }
        const int valid = max(0, min(2, nval * NB - 2 * nidx));  // fp16 norms of this piece
        cp_async4_if(norm_lane, sb + ndst, valid ? nsrc + (size_t)t0 * NB : knp, 2u * (uint32_t)valid);
        if constexpr (VO) {
          const bool ok = vo_tok < nval;
          cp_async16_if(vo_lane, sb + vo_dst, ok ? vop + (size_t)t0 * vo_kp + 8 * lane : vop, ok ? 16u : 0u);
        }
      }
      cp_async_commit();
      if (++islot == depth) islot = 0;
    };

    // this warp's query row, loaded now: its latency overlaps the append and
    // the first copies
    float qrow[NB][4];
    if constexpr (HASK) load_q_row(b, h0, Gu, qrow);

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
                     sm.res + 64u * cw);
      }
      __threadfence();
      consumer_sync();
    }
    // Warp cw takes tiles seg_lo + cw, seg_lo + cw + kCWarps, ...  The first
    // `depth` copies are issued before the query preparation, which they
    // overlap.
    const int first = seg_lo + cw;
    const int n_mine = first < seg_hi ? (seg_hi - first + kCWarps - 1) / kCWarps : 0;
    for (int i = 0; i < (int)depth; ++i) {
      if (i < n_mine) issue(first + i * kCWarps);
      else cp_async_commit();  // one group per tile slot, so the waits count right
    }
    // ---- per-unit query preparation ----------------------------------------
    uint32_t qf[NB][8][2];
    float qmul[2] = {0.0f, 0.0f};
    float lse2[2] = {0.0f, 0.0f}, moff2[2] = {0.0f, 0.0f};
    if constexpr (HASK) prep_q(qrow, qf, qmul);
    if constexpr (MODE == kSparseV) {
      // log-sum-exp (log2 domain) of every head of this unit, from the
      // partials that pass 1 (p1_ctas CTAs) wrote; warp hd takes head hd
      const Split sp1(prefix, p.batch, UB, p1_ctas, sw);  // pass 1 had the same parameters
      if (cw < Gu) {
        const float2 ML = unit_ml_warp(p.slot_ml, sp1.part_of(Su), sp1.part_of(Su + nt - 1), sp1, unit, cw, lane);
        if (lane == 0) {
          const bool seen = ML.x != -INFINITY && ML.y > 0.0f;  // no position visible: weights 0
          u_lse[cw] = seen ? ML.x + __log2f(ML.y) + kPShift : INFINITY;  // pass-1 l carries 2^-7
          u_m[cw] = seen ? ML.x : 0.0f;
          u_l[cw] = seen ? ML.y : 0.0f;
        }
      }
      consumer_sync();
      const int hd0 = kDup ? (2 * g) & 3 : 2 * g, hd1 = kDup ? (2 * g + 1) & 3 : 2 * g + 1;
      // the gate compares s - LSE with log2(thr); the kept weights are
      // 2^(s - M - 7), as in the fused path (normal fp16 range for the
      // largest ones), and the output is divided by 128 * u_l at the end
      lse2[0] = (hd0 < Gu) ? u_lse[hd0] : INFINITY;
      lse2[1] = (hd1 < Gu) ? u_lse[hd1] : INFINITY;
      moff2[0] = ((hd0 < Gu) ? u_m[hd0] : 0.0f) + kPShift;
      moff2[1] = ((hd1 < Gu) ? u_m[hd1] : 0.0f) + kPShift;
    }
    const float log2_thr = (MODE == kSparseV) ? __log2f(p.sparse_thr) : 0.0f;

    // ---- warp loop over this segment's tiles ----------------------------------
    float acc[NB][kMT][4];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk)
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[blk][mt][e] = 0.0f;
    // v3: outlier sums, rows = channel slots R / R + 8, columns = score columns
    float acc_o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    uint32_t oa[4] = {0u, 0u, 0u, 0u};  // this tile's outlier A fragments
    // Online softmax state per score column, in the unscaled domain of
    // s' = raw * nK (the score is s = s' * qmul): m_run is the running max of
    // s, moff = m_ref + kPShift the exponent offset (m_ref = 0 while no
    // position has been seen), thr the value of s' above which the max must be
    // refreshed (m_run + kTau) / qmul.
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    float moff[2] = {kPShift, kPShift};
    float thr[2] = {-INFINITY, -INFINITY};

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
            // a0/a1: pair 2j of tokens 2R / 2R+1; a2/a3: pair 2j+1
            const uint2 t0 = pair2_frag<KB>(tr.k[0][blk], j, lbK);
            const uint2 t1 = pair2_frag<KB>(tr.k[1][blk], j, lbK);
            mma16816(ca[j % kKChains][blk], t0.x, t1.x, t0.y, t1.y, qf[blk][j][0], qf[blk][j][1]);
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

    auto vfrag2 = [&](const uint32_t* w, int r) -> uint2 {
      if constexpr (V2) return pair2_frag_v2<VB, V2S>(w, r, lbV);
      else return pair2_frag<VB>(w, r, lbV);
    };
    auto finish = [&](TileRegs<KB, VB, NB>& tr, int tile, const Raw& raw, auto full_tag) {
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
        float sR[2], sR8[2];  // s' = raw * nK (masked: -inf)
        {
          float a[2] = {0.0f, 0.0f}, bb[2] = {0.0f, 0.0f};
#pragma unroll
          for (int blk = 0; blk < NB; ++blk) {
            const float2 kn = norm_pair<NB>(tr.kn, blk);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              a[cc] = fmaf(raw.c[blk][cc], kn.x, a[cc]);
              bb[cc] = fmaf(raw.c[blk][2 + cc], kn.y, bb[cc]);
            }
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            sR[cc] = okR[cc] ? a[cc] : -INFINITY;
            sR8[cc] = okR8[cc] ? bb[cc] : -INFINITY;
          }
        }
        if constexpr (MODE == kScores) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int hd = 2 * g + cc;  // columns 4..7 repeat heads 0..3 when kDup
            if (hd < Gu && (!kDup || g < 2)) {
              float* srow = p.scores + ((size_t)b * p.kv_heads * Gv + h0 + hd) * p.seq_cap + t0 + 2 * R;
              if (okR8[cc]) {
                *reinterpret_cast<float2*>(srow) = make_float2(sR[cc] * qmul[cc], sR8[cc] * qmul[cc]);
              } else if (okR[cc]) {
                srow[0] = sR[cc] * qmul[cc];
              }
            }
          }
        }
        // D4: online softmax.  The per-head maximum is only reduced across the
        // warp when some lane's scores exceed the reference by more than 2^kTau.
        const float lm0 = fmaxf(sR[0], sR8[0]), lm1 = fmaxf(sR[1], sR8[1]);
        const bool need = (lm0 > thr[0]) || (lm1 > thr[1]);
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float tmax = (cc ? lm1 : lm0) * qmul[cc];
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
                if constexpr (VO) {
                  acc_o[cc] *= alpha;
                  acc_o[2 + cc] *= alpha;
                }
              }
              m_run[cc] = tmax;
              moff[cc] = tmax + kPShift;
              thr[cc] = (tmax + kTau) / qmul[cc];
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          // p' = 2^(s - m_ref - 7); a column that has seen no position yet (a
          // later query token's causal limit) has s' = -inf: weight 0
          pR[cc] = ex2(fmaf(sR[cc], qmul[cc], -moff[cc]));
          pR8[cc] = ex2(fmaf(sR8[cc], qmul[cc], -moff[cc]));
          l_run[cc] += pR[cc] + pR8[cc];
        }
      } else {
        // pass 2 of sparse-V: the gate on the normalised weight 2^(s - LSE)
        // (D5), the kept positions weighted 2^(s - M - 7)
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
            wR = s0 - lse2[cc] >= log2_thr ? ex2(s0 - moff2[cc]) : 0.0f;
            wR8 = s1 - lse2[cc] >= log2_thr ? ex2(s1 - moff2[cc]) : 0.0f;
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
            // P^T fragments: lane (R, g) gets tokens 4g, 4g+2 (b0) and
            // 4g+1, 4g+3 (b1) of score column R
            const uint32_t b0 = movtrans(pack_half2(pR[0] * vn.x, pR[1] * vn.x));
            const uint32_t b1 = movtrans(pack_half2(pR8[0] * vn.y, pR8[1] * vn.y));
            if constexpr (kDup) {
              // k = 2*tau + s, column n = h + 4*s': the product pairs the
              // weight of token tau with dim 2*pair + s only when s == s', so
              // each A register is one token's pair of adjacent dims.  Rows R,
              // R+8 of tile q are dim pairs 8R+2q, 8R+2q+1.
              const uint32_t pa0 = prmt(b0, 0u, selLo), pa1 = prmt(b0, 0u, selHi);
              const uint32_t pb0 = prmt(b1, 0u, selLo), pb1 = prmt(b1, 0u, selHi);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint2 v0 = vfrag2(tr.v[0][blk], q);
                const uint2 v1 = vfrag2(tr.v[1][blk], q);
                mma16816(acc[blk][q], v0.x, v0.y, v1.x, v1.y, pa0, pa1);
                const uint2 v2 = vfrag2(tr.v[2][blk], q);
                const uint2 v3 = vfrag2(tr.v[3][blk], q);
                mma16816(acc[blk][q], v2.x, v2.y, v3.x, v3.y, pb0, pb1);
              }
            } else {
#pragma unroll
              for (int m2 = 0; m2 < 4; ++m2) {
                const uint2 x0 = vfrag2(tr.v[0][blk], m2);
                const uint2 x1 = vfrag2(tr.v[1][blk], m2);
                const uint2 x2 = vfrag2(tr.v[2][blk], m2);
                const uint2 x3 = vfrag2(tr.v[3][blk], m2);
                mma16816(acc[blk][2 * m2], prmt(x0.x, x1.x, 0x5410), prmt(x0.x, x1.x, 0x7632),
                         prmt(x2.x, x3.x, 0x5410), prmt(x2.x, x3.x, 0x7632), b0, b1);
                mma16816(acc[blk][2 * m2 + 1], prmt(x0.y, x1.y, 0x5410), prmt(x0.y, x1.y, 0x7632),
                         prmt(x2.y, x3.y, 0x5410), prmt(x2.y, x3.y, 0x7632), b0, b1);
              }
            }
          }
          if constexpr (VO) {
            // outlier channels: sum_t w_t val_t, the plain weights (no norm)
            const uint32_t ob0 = movtrans(pack_half2(pR[0], pR[1]));
            const uint32_t ob1 = movtrans(pack_half2(pR8[0], pR8[1]));
            mma16816(acc_o, oa[0], oa[1], oa[2], oa[3], ob0, ob1);
          }
        }
      }
    };

    {
      // Tile i of the warp sits in slot cslot.  Its slot is handed to tile
      // i + depth once the tile's registers have been used (end of the
      // iteration): every read of the slot has completed before the copy that
      // overwrites it is issued.
      for (int i = 0; i < n_mine; ++i) {
        TileRegs<KB, VB, NB> tr;
        const uint32_t sl = wring_s + cslot * slot_bytes;
        cp_async_wait_depth(depth);  // this lane's copies of tile i have landed
        __syncwarp();                // and every other lane's
        read_tile<KB, VB, NB, HASK, HASV, V2>(tr, sl + koff, sl + voff, R);
        if constexpr (HASK) read_norms<NB>(tr.kn, sl + sm.kn_off, R);
        if constexpr (HASV) read_norms<NB>(tr.vn, sl + sm.vn_off, R);
        if constexpr (VO) {
          oa[0] = movtrans(ld_s32(sl + vo_a[0]));
          oa[2] = movtrans(ld_s32(sl + vo_a[2]));
          if (vo_kp == 16) {
            oa[1] = movtrans(ld_s32(sl + vo_a[1]));
            oa[3] = movtrans(ld_s32(sl + vo_a[3]));
          }
        }
        if (++cslot == depth) cslot = 0;
        const int tile = first + i * kCWarps;
        const Raw raw = scores(tr);
        if (tile * kTile + kTile <= len_full)
          finish(tr, tile, raw, std::true_type{});
        else
          finish(tr, tile, raw, std::false_type{});
        __syncwarp();
        if (i + (int)depth < n_mine) issue(first + (i + (int)depth) * kCWarps);
        else cp_async_commit();
      }
      cp_async_wait<0>();
      __syncwarp();
    }

    // ---- warp partials: this warp's ring holds its acc [head][D] -----------
    consumer_sync();  // every warp is done with its ring
    const uint32_t wpart = wring_s;
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
              st_s32(wpart + 4u * (h * D + d), __float_as_uint(acc[blk][q][e]));
            }
      } else {
#pragma unroll
        for (int blk = 0; blk < NB; ++blk)
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const int d0 = blk * kBlock + 16 * R + 2 * mt;
            st_s64(wpart + 4u * ((2 * g) * D + d0), __float_as_uint(acc[blk][mt][0]),
                   __float_as_uint(acc[blk][mt][2]));
            st_s64(wpart + 4u * ((2 * g + 1) * D + d0), __float_as_uint(acc[blk][mt][1]),
                   __float_as_uint(acc[blk][mt][3]));
          }
      }
      if constexpr (VO) {  // outlier sums in res: [warp][head][slot]
        if (!kDup || g < 2) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const uint32_t o = sm.res + 4u * ((cw * GQ + 2 * g + cc) * kOutlierMax + R);
            st_s32(o, __float_as_uint(acc_o[cc]));
            st_s32(o + 32u, __float_as_uint(acc_o[2 + cc]));
          }
        }
      }
    }
    consumer_sync();

    // ---- warp hd merges the 16 warps' partials of head hd in a fixed order,
    // then emits the head (the CTA saw the whole unit) or publishes the CTA's
    // partial and adds the segment's tiles to the (unit, head) count; the
    // warp that completes the count merges every partial of head hd.  No
    // other warp takes part, so there is no block-wide step. ---------------------
    const bool whole = (seg_lo == 0 && seg_hi == nt);
    const long long slot = blockIdx.x + unit;
    if (cw < Gu) {
      const int hd = cw;
      float M = 0.0f, L = 0.0f;
      float fw[kCWarps];
      if constexpr (HASK) {
        M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kCWarps; ++w) M = fmaxf(M, w_m[w * kMaxGroup + hd]);
#pragma unroll
        for (int w = 0; w < kCWarps; ++w) {
          const float mw = w_m[w * kMaxGroup + hd];
          fw[w] = (mw == -INFINITY) ? 0.0f : ex2(mw - M);
          L = fmaf(w_l[w * kMaxGroup + hd], fw[w], L);
        }
      } else {
#pragma unroll
        for (int w = 0; w < kCWarps; ++w) fw[w] = 1.0f;
      }
      float v[NB][4];
#pragma unroll
      for (int blk = 0; blk < NB; ++blk)
#pragma unroll
        for (int k = 0; k < 4; ++k) v[blk][k] = 0.0f;
      if constexpr (HASV) {
#pragma unroll
        for (int w = 0; w < kCWarps; ++w) {
#pragma unroll
          for (int blk = 0; blk < NB; ++blk) {
            const float4 a = ld_s128f(sm.ring[w] + 4u * (hd * D + blk * kBlock + 4 * lane));
            if (fw[w] != 0.0f) {  // a warp that saw nothing may hold stale values
              v[blk][0] = fmaf(a.x, fw[w], v[blk][0]);
              v[blk][1] = fmaf(a.y, fw[w], v[blk][1]);
              v[blk][2] = fmaf(a.z, fw[w], v[blk][2]);
              v[blk][3] = fmaf(a.w, fw[w], v[blk][3]);
            }
          }
        }
      }
      float ov[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // v3: lane i < 4 holds outlier slots 4i..4i+3
      if constexpr (VO) {
        if (lane < 4) {
#pragma unroll
          for (int w = 0; w < kCWarps; ++w) {
            const float4 a = ld_s128f(sm.res + 4u * ((w * GQ + hd) * kOutlierMax + 4 * lane));
            if (fw[w] != 0.0f) {
              ov[0] = fmaf(a.x, fw[w], ov[0]);
              ov[1] = fmaf(a.y, fw[w], ov[1]);
              ov[2] = fmaf(a.z, fw[w], ov[2]);
              ov[3] = fmaf(a.w, fw[w], ov[3]);
            }
          }
        }
      }
      if (whole && MODE != kScores) {
        // this CTA saw the entire unit: no partial needed
        emit_row(v, ov, (MODE == kFused ? L : u_l[hd]) * 128.0f, b, h0 + hd);
      } else {
        // (m, l) of the partial: the fused merge weighs by it and pass 2 of
        // sparse-V reads pass 1's.  Pass 2 itself writes none: its CTAs read
        // pass 1's (m, l) at each segment start, and a write to the same slot
        // could land before another CTA's read.
        if (lane == 0 && MODE != kSparseV)
          *reinterpret_cast<float2*>(p.slot_ml + (slot * kMaxGroup + hd) * 2) = make_float2(M, L);
        if constexpr (HASV) {
#pragma unroll
          for (int blk = 0; blk < NB; ++blk)
            *reinterpret_cast<float4*>(p.slot_acc + (slot * kMaxGroup + hd) * PD + blk * kBlock + 4 * lane) =
                make_float4(v[blk][0], v[blk][1], v[blk][2], v[blk][3]);
          if (VO && lane < 4)
            *reinterpret_cast<float4*>(p.slot_acc + (slot * kMaxGroup + hd) * PD + D + 4 * lane) =
                make_float4(ov[0], ov[1], ov[2], ov[3]);
        }
        if constexpr (MODE != kScores) {
          __threadfence();  // this lane's partial before the count
          __syncwarp();
          unsigned last = 0;
          if (lane == 0) {
            const unsigned add = (unsigned)(seg_hi - seg_lo);
            const unsigned old = atomicAdd(p.tickets + (size_t)unit * kMaxGroup + hd, add);
            last = (old + add == (unsigned)nt) ? 1u : 0u;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence();  // every other partial of head hd is visible
            const long long c_first = sp.part_of(Su), c_last = sp.part_of(Su + nt - 1);
            const float* ml_base = p.slot_ml + ((long long)unit * kMaxGroup + hd) * 2;
            const float* acc_base = p.slot_acc + ((long long)unit * kMaxGroup + hd) * PD + 4 * lane;
            const long long ml_stride = kMaxGroup * 2, part_stride = (long long)kMaxGroup * PD;
            // One pass over the partials in chunks of 32 (lane j holds part
            // c0 + j): the chunk's (m, l) give its maximum; a chunk whose
            // maximum exceeds the running one rescales what came before (no
            // rescale with a single chunk, the common case); then every
            // partial's acc is added in part order with the loads in flight.
            float Mx = -INFINITY, Lx = 0.0f;
            float u[NB][4];
#pragma unroll
            for (int blk = 0; blk < NB; ++blk)
#pragma unroll
              for (int k = 0; k < 4; ++k) u[blk][k] = 0.0f;
            float uo[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (long long c0 = c_first; c0 <= c_last; c0 += 32) {
              const uint32_t emp = empty_bits(sp, c0, c_last, lane);
              const long long c = c0 + lane;
              const bool live = c <= c_last && !((emp >> lane) & 1u);
              float wgt = live ? 1.0f : 0.0f;
              if constexpr (MODE == kFused) {
                const float2 ml = live ? __ldcg(reinterpret_cast<const float2*>(ml_base + c * ml_stride))
                                       : make_float2(-INFINITY, 0.0f);
                float cm = ml.x;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
                if (cm > Mx) {  // warp-uniform
                  const float sc = (Mx == -INFINITY) ? 0.0f : ex2(Mx - cm);
                  Lx *= sc;
#pragma unroll
                  for (int blk = 0; blk < NB; ++blk)
#pragma unroll
                    for (int k = 0; k < 4; ++k) u[blk][k] *= sc;
#pragma unroll
                  for (int k = 0; k < 4; ++k) uo[k] *= sc;
                  Mx = cm;
                }
                wgt = (ml.x == -INFINITY) ? 0.0f : ex2(ml.x - Mx);
                float lw = wgt != 0.0f ? ml.y * wgt : 0.0f;  // L: fixed-order reduction over the chunk
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
                Lx += lw;
              }
              const int n = (int)min((long long)32, c_last - c0 + 1);
#pragma unroll 8
              for (int j = 0; j < n; ++j) {
                const float wj = __shfl_sync(0xffffffffu, wgt, j);
                float4 a[NB];
#pragma unroll
                for (int blk = 0; blk < NB; ++blk)
                  a[blk] = __ldcg(reinterpret_cast<const float4*>(acc_base + (c0 + j) * part_stride + blk * kBlock));
#pragma unroll
                for (int blk = 0; blk < NB; ++blk) {  // skipped parts may hold anything: select, not multiply
                  u[blk][0] += wj != 0.0f ? a[blk].x * wj : 0.0f;
                  u[blk][1] += wj != 0.0f ? a[blk].y * wj : 0.0f;
                  u[blk][2] += wj != 0.0f ? a[blk].z * wj : 0.0f;
                  u[blk][3] += wj != 0.0f ? a[blk].w * wj : 0.0f;
                }
                if (VO && lane < 4) {
                  const float4 a4 = __ldcg(reinterpret_cast<const float4*>(acc_base + (c0 + j) * part_stride + D));
                  uo[0] += wj != 0.0f ? a4.x * wj : 0.0f;
                  uo[1] += wj != 0.0f ? a4.y * wj : 0.0f;
                  uo[2] += wj != 0.0f ? a4.z * wj : 0.0f;
                  uo[3] += wj != 0.0f ? a4.w * wj : 0.0f;
                }
              }
            }
            emit_row(u, uo, (MODE == kFused ? Lx : u_l[hd]) * 128.0f, b, h0 + hd);
            if (lane == 0) p.tickets[(size_t)unit * kMaxGroup + hd] = 0u;  // ready for the next launch
          }
        }
      }
    }
    consumer_sync();  // misc, res and the rings are reused by the next segment
    x = Su + seg_hi;
  }


  // ---- zero rows of empty sequences (only the V-producing passes; off the
  // critical path, after the tiles) ---------------------------------------------
  if constexpr (MODE != kScores) {
    const long long rows = (long long)p.batch * p.n_q * p.q_heads;
    for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
      const int b = (int)(row / ((long long)p.n_q * p.q_heads));
      if (prefix[b + 1] == prefix[b]) {
        for (int d = tid; d < D; d += kThreads) p.out[row * D + d] = 0.0f;
      }
    }
  }
}

// --------------------------------------------------------------- launching --

// Shared-memory plan for one instantiation (host).  Tables first (the byte
// tables in a 64 KiB-aligned region, 3-bit tables 8 KiB-aligned), then the
// other areas first-fit into the gaps, then the rings, as deep as fits.
struct Planner {
  uint32_t lo[8], hi[8];
  int n = 0;
  explicit Planner(uint32_t a, uint32_t b) { lo[0] = a; hi[0] = b; n = 1; }
  // first-fit allocation of `size` bytes at alignment `al`; 0 if none fits
  uint32_t take(uint32_t size, uint32_t al) {
    for (int i = 0; i < n; ++i) {
      const uint32_t a = (lo[i] + al - 1) / al * al;
      if (a + size <= hi[i]) {
        // split [lo, hi) into [lo, a) and [a + size, hi)
        const uint32_t l0 = lo[i], h0 = hi[i];
        lo[i] = a + size;
        hi[i] = h0;
        if (a > l0 && n < 8) {
          for (int j = n; j > i; --j) { lo[j] = lo[j - 1]; hi[j] = hi[j - 1]; }
          lo[i] = l0; hi[i] = a;
          lo[i + 1] = a + size; hi[i + 1] = h0;
          ++n;
        }
        return a;
      }
    }
    return 0;
  }
};

template <int KB, int VB, int NB, int MODE, int GQ, bool VO, bool V2>
bool plan_smem(int batch, SmemPlan& s) {
  constexpr bool HASK = MODE != kSparseV, HASV = MODE != kScores;
  constexpr int D = NB * kBlock;
  const int kb = HASK ? KB : 0, vb = HASV ? VB : 0;
  // the query scratch of one unit: GQ == 4 ? 4 : 8 padded rows
  // (v3: also the warps' outlier sums [warp][GQ heads][kOutlierMax] at the merge)
  uint32_t res_bytes = (uint32_t)((GQ == 4 ? 4 : kMaxGroup) * QScratch<NB>::kRow * 4);
  if (VO && res_bytes < (uint32_t)(kCWarps * GQ * kOutlierMax * 4)) res_bytes = kCWarps * GQ * kOutlierMax * 4;
  (void)D;
  for (int depth = kMaxDepth; depth >= 2; --depth) {
    s = SmemPlan{};
    s.base = kSmemBase;
    Planner pl(kSmemBase, kSmemBase + kMaxDyn);
    // tables
    const bool byte_k = kb == 2 || kb == 4, byte_v = !V2 && (vb == 2 || vb == 4);
    if (byte_k || byte_v) {
      const uint32_t region = pl.take(65536, 65536);
      if (!region) continue;
      if (byte_k) s.lut_k = region;
      if (byte_v) s.lut_v = region + 128;
    }
    if (kb == 3 && !(s.lut_k = pl.take(8192, 8192))) continue;
    if (!V2 && vb == 3 && !(s.lut_v = pl.take(8192, 8192))) continue;
    // v2: in the V half of the byte-table region, or a table of its own
    // (2^(2b+2) entries x 128 B)
    const uint32_t v2_tab = (V2 && !byte_k) ? (uint32_t)(128u << (2 * vb + 2)) : 0u;
    if (V2 && byte_k) s.lut_v = s.lut_k + 128;
    if (v2_tab && !(s.lut_v = pl.take(v2_tab, v2_tab))) continue;
    // slot: K runs, V runs (with gaps), K norms, V norms
    uint32_t off = 0, gk[4] = {0, 0, 0, 0}, gv[4] = {0, 0, 0, 0};
    if (HASK) {
      run_gaps(true, KB, NB, gk);
      for (int j = 0; j < 4; ++j) s.kc_off[j] = off + gk[j] + (uint32_t)(4 * j * NB * Fmt<KB>::kBlockBytes);
      off = s.kc_off[3] + 4 * NB * Fmt<KB>::kBlockBytes;
    }
    if (HASV) {
      off = (off + 127) / 128 * 128;
      run_gaps(false, VB, NB, gv);
      for (int j = 0; j < 4; ++j) s.vc_off[j] = off + gv[j] + (uint32_t)(4 * j * NB * Fmt<VB>::kBlockBytes);
      off = s.vc_off[3] + 4 * NB * Fmt<VB>::kBlockBytes;
    }
    off = (off + 15) / 16 * 16;
    if (VO) {  // v3 outlier values: 16 tokens x 16 fp16 (x 8 when k <= 8)
      s.vo_off = off;
      off += kTile * kOutlierMax * 2;
    }
    s.kn_off = off;
    if (HASK) off += kTile * NB * 2;
    s.vn_off = off;
    if (HASV) off += kTile * NB * 2;
    s.slot_bytes = (off + 127) / 128 * 128;
    s.depth = (uint32_t)depth;
    // a warp's ring also holds its partial acc [GQ heads][D] between tiles
    uint32_t ring_bytes = s.slot_bytes * depth;
    const uint32_t part_bytes = (uint32_t)(GQ * D * 4);
    if (ring_bytes < part_bytes) ring_bytes = part_bytes;
    bool ok = true;
    for (int w = 0; w < kCWarps && ok; ++w) ok = (s.ring[w] = pl.take(ring_bytes, 128)) != 0;
    if (!ok) continue;
    if (!(s.res = pl.take(res_bytes, 16))) continue;
    if (!(s.misc = pl.take((uint32_t)(Misc::kWords * 4), 16))) continue;
    if (!(s.prefix = pl.take((uint32_t)((batch + 1) * 4), 16))) continue;
    uint32_t end = 0;
    // the highest byte used: tables, rings and the small areas
    auto upd = [&](uint32_t a, uint32_t n) { if (a && a + n > end) end = a + n; };
    if (byte_k || byte_v) upd(byte_k ? s.lut_k : s.lut_v - 128, 65536);
    if (kb == 3) upd(s.lut_k, 8192);
    if (!V2 && vb == 3) upd(s.lut_v, 8192);
    if (v2_tab) upd(s.lut_v, v2_tab);
    for (int w = 0; w < kCWarps; ++w) upd(s.ring[w], ring_bytes);
    upd(s.res, res_bytes);
    upd(s.misc, Misc::kWords * 4);
    upd(s.prefix, (uint32_t)(batch + 1) * 4);
    s.bytes = end - kSmemBase;
    return true;
  }
  return false;
}

template <int KB, int VB, int NB, int MODE, int GQ, bool VO, bool V2 = false>
int run(DecodeParams& p, cudaStream_t stream, int p1_ctas, int* ctas_out, bool pdl = true) {
  if (!plan_smem<KB, VB, NB, MODE, GQ, VO, V2>(p.batch, p.sm)) return TQ_ERR_UNSUPPORTED;
  const size_t smem = p.sm.bytes;
  auto kern = decode_kernel<KB, VB, NB, MODE, GQ, VO, V2>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  static int cached_sms[64] = {0};
  static size_t cached_smem[64] = {0};
  if (dev >= 64) return TQ_ERR_UNSUPPORTED;
  if (cached_sms[dev] == 0 || cached_smem[dev] < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDyn) != cudaSuccess)
      return TQ_ERR_CUDA;
    int sms = 0, occ = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem) != cudaSuccess)
      return TQ_ERR_CUDA;
    if (occ < 1) return TQ_ERR_UNSUPPORTED;
    cached_smem[dev] = kMaxDyn;
    cached_sms[dev] = sms;
  }
  // one CTA per SM, but no more than one per kMinCtaTiles tiles of the
  // largest launch these sizes allow (a short cache is done by fewer CTAs,
  // with fewer partials to merge)
  const long long n_hg = (p.q_heads / p.kv_heads * p.n_q + kMaxGroup - 1) / kMaxGroup;
  const long long tiles_max = (long long)p.batch * p.kv_heads * n_hg * ((p.seq_cap + kTile - 1) / kTile);
  int ctas = min(kMaxCtas, cached_sms[dev]);
  if ((tiles_max + kMinCtaTiles - 1) / kMinCtaTiles < ctas)
    ctas = (int)max(1LL, (tiles_max + kMinCtaTiles - 1) / kMinCtaTiles);
  // Programmatic stream serialisation: the launch may begin while the
  // kernel before it finishes (see pdl_wait in the kernel).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, p, p1_ctas) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  if (ctas_out) *ctas_out = ctas;
  return TQ_OK;
}

template <int KB, int VB, int NB, int GQ, bool VO, bool V2 = false>
int dispatch_modes(DecodeParams& p, cudaStream_t stream) {
  if (p.sparse_thr > 0.0f) {
    // The two passes launch without programmatic serialisation: on either
    // launch it made a graph of sparse-V steps 2-4 % slower (measured), while
    // a single fused launch gains from it.
    int p1 = 0;
    int st = run<KB, 2, NB, kScores, GQ, false>(p, stream, 0, &p1, false);
    if (st != TQ_OK) return st;
    return run<2, VB, NB, kSparseV, GQ, VO, V2>(p, stream, p1, nullptr, false);
  }
  return run<KB, VB, NB, kFused, GQ, VO, V2>(p, stream, 0, nullptr);
}

template <int KB, int VB, int NB, int GQ>
int dispatch_vo(DecodeParams& p, cudaStream_t stream) {
  if (p.v2) {
    if constexpr (VB == 2 || VB == 3) return dispatch_modes<KB, VB, NB, GQ, false, true>(p, stream);
    else return TQ_ERR_UNSUPPORTED;
  }
  if (p.vo_k > 0) return dispatch_modes<KB, VB, NB, GQ, true>(p, stream);
  return dispatch_modes<KB, VB, NB, GQ, false>(p, stream);
}

template <int KB, int VB, int NB>
int dispatch_gq(DecodeParams& p, cudaStream_t stream) {
  if (p.q_heads / p.kv_heads * p.n_q <= 4) return dispatch_vo<KB, VB, NB, 4>(p, stream);
  return dispatch_vo<KB, VB, NB, 8>(p, stream);
}

template <int KB, int VB>
int dispatch_nb(DecodeParams& p, cudaStream_t stream) {
  switch (p.head_dim / kBlock) {
    case 1: return dispatch_gq<KB, VB, 1>(p, stream);
    case 2: return dispatch_gq<KB, VB, 2>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

template <int KB>
int dispatch_kb(DecodeParams& p, cudaStream_t stream) {
  switch (p.v_bits) {
    case 2: return dispatch_nb<KB, 2>(p, stream);
    case 3: return dispatch_nb<KB, 3>(p, stream);
    case 4: return dispatch_nb<KB, 4>(p, stream);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace dec
}  // namespace tq
