// Internal interface between the C-ABI host layer (tq_host.cpp) and the
// sm_100a kernels (tq_encode.cu, tq_decode.cu).  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/tq.h"

namespace tq {

constexpr int kBlock = 128;        // elements per rotated/quantised block
constexpr int kTile = 16;          // tokens per decode MMA tile
constexpr int kMaxGroup = 8;       // q-heads handled together per kv-head (MMA N = 8)
constexpr int kMaxCtas = 1024;     // upper bound on persistent decode CTAs
constexpr int kMaxBatch = 2048;    // decode batch limit (the tile prefix lives in shared memory)
constexpr int kMaxHeadDim = 512;   // encoder: up to 4 blocks per vector
constexpr int kMaxDecodeHeadDim = 256;  // decode kernels are built for 1 or 2 blocks

// Division of 32-bit unsigned n by a fixed d >= 1 without a divide: with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1, t = mulhi(m, n)
// gives n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0) for every n
// below 2^32 (Granlund and Montgomery, PLDI 1994, figure 4.1).
struct FastDiv {
  uint32_t d, m, s1, s2;
  static FastDiv make(uint32_t div) {
    FastDiv f{};
    f.d = div;
    int l = 0;
    while ((1ull << l) < div) ++l;
    f.m = (uint32_t)((((1ull << l) - div) << 32) / div + 1);
    f.s1 = l > 0 ? 1u : 0u;
    f.s2 = l > 1 ? (uint32_t)(l - 1) : 0u;
    return f;
  }
#ifdef __CUDACC__
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    const uint32_t t = __umulhi(m, n);
    return (t + ((n - t) >> s1)) >> s2;
  }
#endif
};

// Encoder launch parameters (one launch writes K and V).
struct EncodeParams {
  const void* in[2];          // K, V inputs [B, Hkv, seq_new, D] (either may be null)
  uint8_t* codes[2];
  uint16_t* norms[2];
  int bits[2];
  float pos_bounds[2][7];     // positive decision boundaries, ascending
  const int32_t* start_pos;   // device [B] or null
  uint32_t* status;           // device status word or null
  uint32_t sign_mask[4];      // bit i set <=> s_i = -1
  int f16;                    // input dtype: 1 = fp16, 0 = fp32
  int batch, kv_heads, head_dim, seq_cap, seq_new;
  FastDiv div_seq_new, div_kv_heads;  // index splits of the flattened rows (below 2^31)
  uint32_t k_ctas;                    // CTAs of the launch that encode K (set by launch_encode)
  // V v3 (vo_k > 0): channels [kv_heads, vo_k] of V are zeroed before the
  // encoding and their values written to vo_values [.., seq_cap, vo_kp]
  const int32_t* vo_channels;
  uint16_t* vo_values;
  int vo_k, vo_kp;
  // V v2: the doubled codebook's 2^(bits + 1) levels (launch_encode_v2)
  float tcq_levels[16];
};

int launch_pick_outliers(const void* v, int f16, int batch, int kv_heads, int rows, int head_dim, int k,
                         int32_t* channels, cudaStream_t stream);

int launch_encode(const EncodeParams& p, cudaStream_t stream);
// V side only, in the v2 trellis format (p.in[1], p.codes[1], p.norms[1], p.bits[1] in {2, 3})
int launch_encode_v2(const EncodeParams& p, cudaStream_t stream);

constexpr int kDecodeWarps = 16;   // warps of one persistent decode CTA (one CTA per SM)

// Shared-memory plan of a decode launch, computed on the host.  Every
// address is an absolute shared-window address; the kernel checks that its
// dynamic shared memory starts at `base` before using any of them.
struct SmemPlan {
  uint32_t base;                  // shared-window address of dynamic shared memory
  uint32_t bytes;                 // dynamic shared memory requested
  uint32_t lut_k, lut_v;          // code tables (byte tables: 64 KiB region + 0 / + 128)
  uint32_t ring[kDecodeWarps];    // each warp's ring of tile slots (also its partial)
  uint32_t res, misc, prefix;
  uint32_t depth, slot_bytes;     // slots per ring, bytes per slot
  uint32_t kc_off[4], vc_off[4];  // K / V codes of tokens 4j..4j+3 within a slot
  uint32_t kn_off, vn_off;        // K / V norms within a slot
  uint32_t vo_off;                // v3 outlier values within a slot
};

// Decode launch parameters.
struct DecodeParams {
  const void* q;
  int q_f16;
  const uint8_t* k_codes;
  const uint16_t* k_norms;
  const uint8_t* v_codes;
  const uint16_t* v_norms;
  const int32_t* seq_lens;
  float* out;
  uint32_t* status;
  // workspace views
  uint32_t* tickets;   // [units][kMaxGroup] tiles counted per (unit, head)
  float* slot_ml;      // [(kMaxCtas + units) * kMaxGroup * 2]
  float* slot_acc;     // [(kMaxCtas + units) * kMaxGroup * acc_stride(head_dim)]
  float* scores;       // sparse only: [B, Hq, seq_cap] (log2-domain scores)
  float kcent[16], vcent[16];
  uint32_t sign_mask[4];
  int k_bits, v_bits;
  int batch, kv_heads, q_heads, head_dim, seq_cap;
  float score_mult;    // scale * log2(e) / 128
  float sparse_thr;    // > 0: two-pass exact sparse-V
  int n_q;             // query tokens per sequence (the last n_q positions, causal)
  // Decode step only (kv_new[0] != null): the new token of sequence b,
  // rows [B, Hkv, D] of K and V, is encoded into the cache at position
  // seq_lens[b] - 1 before attention reads it.
  const void* kv_new[2];
  int kv_new_f16;
  uint8_t* app_codes[2];
  uint16_t* app_norms[2];
  float pos_bounds[2][7];  // positive decision boundaries of K and V, ascending
  // V v3 (vo_k > 0): outlier channels [kv_heads, vo_k] and their values
  // [B, Hkv, seq_cap, vo_kp] fp16
  const int32_t* vo_channels;
  const uint16_t* vo_values;
  int vo_k, vo_kp;
  // V v2 (v2 != 0): V codes are trellis pair fields, vcent the doubled
  // codebook (2^(v_bits + 1) levels)
  int v2;
  SmemPlan sm;        // filled by the launcher
};

constexpr int kOutlierMax = 16;   // outlier channels per kv-head, at most
// floats per head of a partial: the rotated-domain acc, then the v3 outlier sums
__host__ __device__ constexpr int acc_stride(int head_dim) { return head_dim + kOutlierMax; }

// Workspace layout shared by the size query and the launcher.
struct DecodeWorkspace {
  size_t tickets_off, ml_off, acc_off, scores_off, total;
};
DecodeWorkspace decode_workspace_layout(int batch, int kv_heads, int q_heads, int head_dim,
                                        int seq_cap, bool sparse);

int launch_decode(const DecodeParams& p, cudaStream_t stream);

// Host-side argument checks shared by every decode entry point (no CUDA call;
// the workspace is checked separately by the entry points that take one).
int validate_decode(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                    int q_heads, int n_q, const void* q, int q_dtype, const uint8_t* k_codes,
                    const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_norms,
                    const int32_t* seq_lens, float scale, float sparse_thr, const float* out,
                    const uint32_t* dev_status, int v_fmt = 1);

}  // namespace tq
