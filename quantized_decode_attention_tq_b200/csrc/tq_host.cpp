// C-ABI host layer: argument validation, the rotation's sign vector, the
// Lloyd-Max codebook, workspace layout, and dispatch to the sm_100a kernels.
// Validation never touches the GPU, so every error path runs without one.

#include <cmath>
#include <cstring>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014): Weyl-sequence state plus two
// xor-shift-multiply mixing rounds.
struct SplitMix64 {
  uint64_t state;
  uint64_t next() {
    state += kGolden;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

// Sign bit mask of the random diagonal: bit i set <=> s_i = -1.
void sign_mask(uint64_t seed, uint32_t mask[4]) {
  SplitMix64 g{seed};
  mask[0] = mask[1] = mask[2] = mask[3] = 0;
  for (int i = 0; i < tq::kBlock; ++i)
    if (g.next() >> 63) mask[i >> 5] |= 1u << (i & 31);
}

// Standard normal density and the probability mass of [a, b] for 0 <= a <= b.
double npdf(double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) * 0.3989422804014327; }
double nmass_pos(double a, double b) {
  const double r = 0.7071067811865476;
  double ea = std::erfc(a * r), eb = std::isinf(b) ? 0.0 : std::erfc(b * r);
  return 0.5 * (ea - eb);
}

// Lloyd-Max on the N(0,1) density, using its symmetry: iterate the positive
// half only (cells [t_{k-1}, t_k] with t_{-1} = 0 and the last cell open),
// so the codebook is exactly symmetric and the middle boundary is exactly 0.
// Start from an even spread; the density is log-concave, so the fixed point
// is unique and the start only affects the number of iterations.
void lloyd_max_positive(int levels, double* c) {
  const int half = levels / 2;
  for (int k = 0; k < half; ++k) c[k] = (k + 0.5) * 4.0 / levels;
  for (int it = 0; it < 2000000; ++it) {
    double delta = 0.0;
    double lo = 0.0;
    double nc[8];
    for (int k = 0; k < half; ++k) {
      double hi = (k + 1 < half) ? 0.5 * (c[k] + c[k + 1]) : INFINITY;
      nc[k] = (npdf(lo) - npdf(hi)) / nmass_pos(lo, hi);
      lo = hi;
    }
    for (int k = 0; k < half; ++k) {
      delta = std::fmax(delta, std::fabs(nc[k] - c[k]));
      c[k] = nc[k];
    }
    if (delta < 1e-15) break;
  }
}

bool valid_bits(int b) { return b >= 2 && b <= 4; }

int check_desc(const tq_kv_desc* d) {
  if (!d) return TQ_ERR_INVALID_ARG;
  if (d->batch < 1 || d->kv_heads < 1 || d->seq_cap < 1 || d->head_dim < 1)
    return TQ_ERR_INVALID_ARG;
  if (d->head_dim % tq::kBlock != 0 || d->head_dim > tq::kMaxHeadDim) return TQ_ERR_UNSUPPORTED;
  if (!valid_bits(d->k_bits) || !valid_bits(d->v_bits)) return TQ_ERR_UNSUPPORTED;
  return TQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_codebook(const tq_codebook* cb, int bits) {
  if (!cb) return TQ_ERR_INVALID_ARG;
  if (cb->bits != bits) return TQ_ERR_INVALID_ARG;
  const int levels = 1 << bits;
  for (int j = 0; j < levels; ++j)
    if (!std::isfinite(cb->centroids[j])) return TQ_ERR_INVALID_ARG;
  // The kernels rely on ascending, symmetric boundaries with 0 in the middle.
  for (int j = 0; j < levels - 1; ++j) {
    if (!std::isfinite(cb->boundaries[j])) return TQ_ERR_INVALID_ARG;
    if (j > 0 && !(cb->boundaries[j] > cb->boundaries[j - 1])) return TQ_ERR_INVALID_ARG;
    if (cb->boundaries[j] != -cb->boundaries[levels - 2 - j]) return TQ_ERR_INVALID_ARG;
  }
  return TQ_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// fp16 entries per token of a v3 values row: 8 for up to 8 channels, else 16
int outlier_row(int k) { return k <= 8 ? 8 : 16; }

int check_outliers(const tq_v_outliers* vo, int head_dim) {
  if (!vo || vo->k == 0) return TQ_OK;
  if (vo->k < 0 || vo->k > TQ_MAX_OUTLIERS || vo->k > head_dim) return TQ_ERR_INVALID_ARG;
  if (!vo->channels || !vo->values || !aligned(vo->channels, 4) || !aligned(vo->values, 16))
    return TQ_ERR_INVALID_ARG;
  return TQ_OK;
}

}  // namespace

namespace tq {

DecodeWorkspace decode_workspace_layout(int batch, int kv_heads, int q_heads, int head_dim,
                                        int seq_cap, bool sparse) {
  DecodeWorkspace w{};
  const int group = q_heads / kv_heads;
  const size_t n_hg = (group + kMaxGroup - 1) / kMaxGroup;
  const size_t units = (size_t)batch * kv_heads * n_hg;
  const size_t slots = kMaxCtas + units;
  size_t off = 0;
  w.tickets_off = off;  // one count per (unit, head of the unit's group)
  off = align_up(off + units * kMaxGroup * sizeof(uint32_t), 256);
  w.ml_off = off;
  off = align_up(off + slots * kMaxGroup * 2 * sizeof(float), 256);
  w.acc_off = off;
  off = align_up(off + slots * kMaxGroup * (size_t)acc_stride(head_dim) * sizeof(float), 256);
  w.scores_off = off;
  if (sparse) off = align_up(off + (size_t)batch * q_heads * seq_cap * sizeof(float), 256);
  w.total = off;
  return w;
}

}  // namespace tq

namespace {

// New-token rows of a decode step (null for plain decode attention).
struct StepRows {
  const void* k_new;
  const void* v_new;
  int kv_dtype;
  uint8_t* k_codes;
  uint16_t* k_norms;
  uint8_t* v_codes;
  uint16_t* v_norms;
};

}  // namespace

namespace tq {

int validate_decode(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                    int q_heads, int n_q, const void* q, int q_dtype, const uint8_t* k_codes,
                    const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_norms,
                    const int32_t* seq_lens, float scale, float sparse_thr, const float* out,
                    const uint32_t* dev_status, int v_fmt) {
  int st = check_desc(desc);
  if (st != TQ_OK) return st;
  if (desc->batch > tq::kMaxBatch || desc->head_dim > tq::kMaxDecodeHeadDim) return TQ_ERR_UNSUPPORTED;
  if (desc->seq_cap % 2 != 0) return TQ_ERR_UNSUPPORTED;  // norm rows must start 4-byte aligned
  if ((long long)desc->batch * ((desc->seq_cap + tq::kTile - 1) / tq::kTile) >= (1LL << 31))
    return TQ_ERR_UNSUPPORTED;
  if (q_heads < desc->kv_heads || q_heads % desc->kv_heads != 0) return TQ_ERR_INVALID_ARG;
  if (n_q < 1 || n_q > TQ_MAX_QUERY_TOKENS) return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
  if (!q || !k_codes || !k_norms || !v_codes || !v_norms || !seq_lens || !out)
    return TQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_codes, 16) || !aligned(v_codes, 16) || !aligned(k_norms, 4) ||
      !aligned(v_norms, 4) || !aligned(seq_lens, 4) || !aligned(out, 16))
    return TQ_ERR_INVALID_ARG;
  if (dev_status && !aligned(dev_status, 4)) return TQ_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f) || std::isnan(sparse_thr)) return TQ_ERR_INVALID_ARG;
  if ((st = check_codebook(k_cb, desc->k_bits)) != TQ_OK) return st;
  if (v_fmt == 2) {  // v2: the doubled codebook; rates 2 and 3
    if (desc->v_bits != 2 && desc->v_bits != 3) return TQ_ERR_UNSUPPORTED;
    return check_codebook(v_cb, desc->v_bits + 1);
  }
  return check_codebook(v_cb, desc->v_bits);
}

}  // namespace tq

namespace {

int decode_common(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                  int q_heads, int n_q, const void* q, int q_dtype,
                  const uint8_t* k_codes, const uint16_t* k_norms,
                  const uint8_t* v_codes, const uint16_t* v_norms,
                  const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                  void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                  void* stream, const StepRows* step, const tq_v_outliers* vo = nullptr, int v_fmt = 1) {
  int st = tq::validate_decode(desc, k_cb, v_cb, q_heads, n_q, q, q_dtype, k_codes, k_norms, v_codes,
                               v_norms, seq_lens, scale, sparse_thr, out, dev_status, v_fmt);
  if (st != TQ_OK) return st;
  if ((st = check_outliers(vo, desc->head_dim)) != TQ_OK) return st;
  if (vo && vo->k > 0 && desc->head_dim > tq::kBlock && desc->k_bits + desc->v_bits >= 7) return TQ_ERR_UNSUPPORTED;
  if (step) {
    if (step->kv_dtype != TQ_F32 && step->kv_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
    if (!step->k_new || !step->v_new || !aligned(step->k_new, 16) || !aligned(step->v_new, 16))
      return TQ_ERR_INVALID_ARG;
  }
  const bool sparse = sparse_thr > 0.0f;
  tq::DecodeWorkspace w = tq::decode_workspace_layout(desc->batch, desc->kv_heads, q_heads * n_q,
                                                      desc->head_dim, desc->seq_cap, sparse);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.total) return TQ_ERR_WORKSPACE;

  tq::DecodeParams p{};
  p.q = q;
  p.q_f16 = q_dtype == TQ_F16;
  p.k_codes = k_codes;
  p.k_norms = k_norms;
  p.v_codes = v_codes;
  p.v_norms = v_norms;
  p.seq_lens = seq_lens;
  p.out = out;
  p.status = dev_status;
  char* base = static_cast<char*>(workspace);
  p.tickets = reinterpret_cast<uint32_t*>(base + w.tickets_off);
  p.slot_ml = reinterpret_cast<float*>(base + w.ml_off);
  p.slot_acc = reinterpret_cast<float*>(base + w.acc_off);
  p.scores = sparse ? reinterpret_cast<float*>(base + w.scores_off) : nullptr;
  const int v_levels = 1 << (desc->v_bits + (v_fmt == 2 ? 1 : 0));
  for (int j = 0; j < 16; ++j) {
    p.kcent[j] = j < (1 << desc->k_bits) ? k_cb->centroids[j] : 0.0f;
    p.vcent[j] = j < v_levels ? v_cb->centroids[j] : 0.0f;
  }
  p.v2 = v_fmt == 2 ? 1 : 0;
  sign_mask(desc->sign_seed, p.sign_mask);
  p.k_bits = desc->k_bits;
  p.v_bits = desc->v_bits;
  p.batch = desc->batch;
  p.kv_heads = desc->kv_heads;
  p.q_heads = q_heads;
  p.head_dim = desc->head_dim;
  p.seq_cap = desc->seq_cap;
  p.score_mult = (float)((double)scale * 1.4426950408889634 / tq::kBlock);
  p.sparse_thr = sparse ? sparse_thr : 0.0f;
  p.n_q = n_q;
  if (vo && vo->k > 0) {
    p.vo_k = vo->k;
    p.vo_kp = outlier_row(vo->k);
    p.vo_channels = vo->channels;
    p.vo_values = vo->values;
  }
  if (step) {
    p.kv_new[0] = step->k_new;
    p.kv_new[1] = step->v_new;
    p.kv_new_f16 = step->kv_dtype == TQ_F16;
    p.app_codes[0] = step->k_codes;
    p.app_codes[1] = step->v_codes;
    p.app_norms[0] = step->k_norms;
    p.app_norms[1] = step->v_norms;
    const tq_codebook* cbs[2] = {k_cb, v_cb};
    const int bits[2] = {desc->k_bits, desc->v_bits};
    for (int sd = 0; sd < 2; ++sd) {
      const int levels = 1 << bits[sd];
      for (int j = 0; j < levels / 2 - 1; ++j) p.pos_bounds[sd][j] = cbs[sd]->boundaries[levels / 2 + j];
    }
  }
  return tq::launch_decode(p, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int tq_make_codebook(int bits, tq_codebook* out) {
  if (!out) return TQ_ERR_INVALID_ARG;
  if (bits < 1 || bits > 4) return TQ_ERR_UNSUPPORTED;
  std::memset(out, 0, sizeof(*out));
  out->bits = bits;
  const int levels = 1 << bits, half = levels / 2;
  double c[8];
  lloyd_max_positive(levels, c);
  for (int k = 0; k < half; ++k) {
    out->centroids[half + k] = (float)c[k];
    out->centroids[half - 1 - k] = (float)-c[k];
  }
  out->boundaries[half - 1] = 0.0f;
  for (int k = 0; k + 1 < half; ++k) {
    float t = (float)(0.5 * (c[k] + c[k + 1]));
    out->boundaries[half + k] = t;
    out->boundaries[half - 2 - k] = -t;
  }
  return TQ_OK;
}

int tq_sign_vector(uint64_t seed, int8_t* out) {
  if (!out) return TQ_ERR_INVALID_ARG;
  uint32_t m[4];
  sign_mask(seed, m);
  for (int i = 0; i < tq::kBlock; ++i) out[i] = ((m[i >> 5] >> (i & 31)) & 1u) ? -1 : 1;
  return TQ_OK;
}

int tq_encode_kv(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                 const void* k, const void* v, int in_dtype, int seq_new,
                 const int32_t* start_pos, uint8_t* k_codes, uint16_t* k_norms,
                 uint8_t* v_codes, uint16_t* v_norms, uint32_t* dev_status, void* stream) {
  return tq_encode_kv_v3(desc, k_cb, v_cb, k, v, in_dtype, seq_new, start_pos, k_codes, k_norms, v_codes,
                         v_norms, nullptr, dev_status, stream);
}

int tq_encode_kv_v3(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                    const void* k, const void* v, int in_dtype, int seq_new,
                    const int32_t* start_pos, uint8_t* k_codes, uint16_t* k_norms,
                    uint8_t* v_codes, uint16_t* v_norms, const tq_v_outliers* vo,
                    uint32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != TQ_OK) return st;
  if ((st = check_outliers(vo, desc->head_dim)) != TQ_OK) return st;
  if (vo && vo->k > 0 && !v) return TQ_ERR_INVALID_ARG;
  if (in_dtype != TQ_F32 && in_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
  if (seq_new < 0) return TQ_ERR_INVALID_ARG;
  if (!k && !v) return TQ_ERR_INVALID_ARG;
  if (k) {
    if (!k_codes || !k_norms || !aligned(k, 16) || !aligned(k_codes, 16) || !aligned(k_norms, 4))
      return TQ_ERR_INVALID_ARG;
    if ((st = check_codebook(k_cb, desc->k_bits)) != TQ_OK) return st;
  }
  if (v) {
    if (!v_codes || !v_norms || !aligned(v, 16) || !aligned(v_codes, 16) || !aligned(v_norms, 4))
      return TQ_ERR_INVALID_ARG;
    if ((st = check_codebook(v_cb, desc->v_bits)) != TQ_OK) return st;
  }
  if (start_pos && !aligned(start_pos, 4)) return TQ_ERR_INVALID_ARG;
  if (dev_status && !aligned(dev_status, 4)) return TQ_ERR_INVALID_ARG;
  if (seq_new == 0) return TQ_OK;

  tq::EncodeParams p{};
  p.in[0] = k;
  p.in[1] = v;
  p.codes[0] = k_codes;
  p.codes[1] = v_codes;
  p.norms[0] = k_norms;
  p.norms[1] = v_norms;
  p.bits[0] = desc->k_bits;
  p.bits[1] = desc->v_bits;
  const tq_codebook* cbs[2] = {k_cb, v_cb};
  for (int s = 0; s < 2; ++s) {
    if (!p.in[s]) continue;
    const int levels = 1 << p.bits[s];
    for (int j = 0; j < levels / 2 - 1; ++j) p.pos_bounds[s][j] = cbs[s]->boundaries[levels / 2 + j];
  }
  p.start_pos = start_pos;
  p.status = dev_status;
  sign_mask(desc->sign_seed, p.sign_mask);
  p.f16 = in_dtype == TQ_F16;
  p.batch = desc->batch;
  p.kv_heads = desc->kv_heads;
  p.head_dim = desc->head_dim;
  p.seq_cap = desc->seq_cap;
  p.seq_new = seq_new;
  p.div_seq_new = tq::FastDiv::make((uint32_t)seq_new);
  p.div_kv_heads = tq::FastDiv::make((uint32_t)desc->kv_heads);
  if (vo && vo->k > 0) {
    p.vo_k = vo->k;
    p.vo_kp = outlier_row(vo->k);
    p.vo_channels = vo->channels;
    p.vo_values = vo->values;
  }
  return tq::launch_encode(p, static_cast<cudaStream_t>(stream));
}

size_t tq_decode_workspace_size(const tq_kv_desc* desc, int q_heads, float sparse_thr) {
  if (check_desc(desc) != TQ_OK) return 0;
  if (q_heads < desc->kv_heads || q_heads % desc->kv_heads != 0) return 0;
  if (std::isnan(sparse_thr)) return 0;
  return tq::decode_workspace_layout(desc->batch, desc->kv_heads, q_heads, desc->head_dim,
                                     desc->seq_cap, sparse_thr > 0.0f)
      .total;
}

int tq_decode_attention(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                        int q_heads, const void* q, int q_dtype,
                        const uint8_t* k_codes, const uint16_t* k_norms,
                        const uint8_t* v_codes, const uint16_t* v_norms,
                        const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                        void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                        void* stream) {
  return decode_common(desc, k_cb, v_cb, q_heads, 1, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       nullptr);
}

int tq_decode_attention_multi(const tq_kv_desc* desc, const tq_codebook* k_cb,
                              const tq_codebook* v_cb, int q_heads, int n_q, const void* q,
                              int q_dtype, const uint8_t* k_codes, const uint16_t* k_norms,
                              const uint8_t* v_codes, const uint16_t* v_norms,
                              const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                              void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                              void* stream) {
  return decode_common(desc, k_cb, v_cb, q_heads, n_q, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       nullptr);
}

int tq_decode_step(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                   int q_heads, const void* q, int q_dtype, const void* k_new, const void* v_new,
                   int kv_dtype, uint8_t* k_codes, uint16_t* k_norms, uint8_t* v_codes,
                   uint16_t* v_norms, const int32_t* seq_lens, float scale, float sparse_thr,
                   float* out, void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                   void* stream) {
  const StepRows step{k_new, v_new, kv_dtype, k_codes, k_norms, v_codes, v_norms};
  return decode_common(desc, k_cb, v_cb, q_heads, 1, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       &step);
}

int tq_decode_attention_v3(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                           int q_heads, const void* q, int q_dtype, const uint8_t* k_codes,
                           const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_norms,
                           const tq_v_outliers* vo, const int32_t* seq_lens, float scale,
                           float sparse_thr, float* out, void* workspace, size_t workspace_bytes,
                           uint32_t* dev_status, void* stream) {
  return decode_common(desc, k_cb, v_cb, q_heads, 1, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       nullptr, vo);
}

int tq_encode_kv_v2(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_tcq,
                    const void* k, const void* v, int in_dtype, int seq_new, const int32_t* start_pos,
                    uint8_t* k_codes, uint16_t* k_norms, uint8_t* v_codes, uint16_t* v_norms,
                    uint32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != TQ_OK) return st;
  if (desc->v_bits != 2 && desc->v_bits != 3) return TQ_ERR_UNSUPPORTED;
  if (in_dtype != TQ_F32 && in_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
  if (seq_new < 0) return TQ_ERR_INVALID_ARG;
  if (!k && !v) return TQ_ERR_INVALID_ARG;
  if (k) {
    if (!k_codes || !k_norms || !aligned(k, 16) || !aligned(k_codes, 16) || !aligned(k_norms, 4))
      return TQ_ERR_INVALID_ARG;
    if ((st = check_codebook(k_cb, desc->k_bits)) != TQ_OK) return st;
  }
  if (v) {
    if (!v_codes || !v_norms || !aligned(v, 16) || !aligned(v_codes, 16) || !aligned(v_norms, 4))
      return TQ_ERR_INVALID_ARG;
    if ((st = check_codebook(v_tcq, desc->v_bits + 1)) != TQ_OK) return st;
  }
  if (start_pos && !aligned(start_pos, 4)) return TQ_ERR_INVALID_ARG;
  if (dev_status && !aligned(dev_status, 4)) return TQ_ERR_INVALID_ARG;
  if (seq_new == 0) return TQ_OK;
  if (k) {  // the K side is the plain format
    st = tq_encode_kv_v3(desc, k_cb, nullptr, k, nullptr, in_dtype, seq_new, start_pos, k_codes, k_norms,
                         nullptr, nullptr, nullptr, dev_status, stream);
    if (st != TQ_OK || !v) return st;
  }
  tq::EncodeParams p{};
  p.in[1] = v;
  p.codes[1] = v_codes;
  p.norms[1] = v_norms;
  p.bits[1] = desc->v_bits;
  for (int j = 0; j < (2 << desc->v_bits); ++j) p.tcq_levels[j] = v_tcq->centroids[j];
  p.div_seq_new = tq::FastDiv::make((uint32_t)seq_new);
  p.div_kv_heads = tq::FastDiv::make((uint32_t)desc->kv_heads);
  p.start_pos = start_pos;
  p.status = dev_status;
  sign_mask(desc->sign_seed, p.sign_mask);
  p.f16 = in_dtype == TQ_F16;
  p.batch = desc->batch;
  p.kv_heads = desc->kv_heads;
  p.head_dim = desc->head_dim;
  p.seq_cap = desc->seq_cap;
  p.seq_new = seq_new;
  return tq::launch_encode_v2(p, static_cast<cudaStream_t>(stream));
}

int tq_decode_attention_v2(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_tcq,
                           int q_heads, const void* q, int q_dtype, const uint8_t* k_codes,
                           const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_norms,
                           const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                           void* workspace, size_t workspace_bytes, uint32_t* dev_status, void* stream) {
  return decode_common(desc, k_cb, v_tcq, q_heads, 1, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       nullptr, nullptr, 2);
}

int tq_decode_attention_multi_v3(const tq_kv_desc* desc, const tq_codebook* k_cb,
                                 const tq_codebook* v_cb, int q_heads, int n_q, const void* q,
                                 int q_dtype, const uint8_t* k_codes, const uint16_t* k_norms,
                                 const uint8_t* v_codes, const uint16_t* v_norms,
                                 const tq_v_outliers* vo, const int32_t* seq_lens, float scale,
                                 float sparse_thr, float* out, void* workspace,
                                 size_t workspace_bytes, uint32_t* dev_status, void* stream) {
  return decode_common(desc, k_cb, v_cb, q_heads, n_q, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       nullptr, vo);
}

int tq_decode_attention_multi_v2(const tq_kv_desc* desc, const tq_codebook* k_cb,
                                 const tq_codebook* v_tcq, int q_heads, int n_q, const void* q,
                                 int q_dtype, const uint8_t* k_codes, const uint16_t* k_norms,
                                 const uint8_t* v_codes, const uint16_t* v_norms,
                                 const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                                 void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                                 void* stream) {
  return decode_common(desc, k_cb, v_tcq, q_heads, n_q, q, q_dtype, k_codes, k_norms, v_codes, v_norms,
                       seq_lens, scale, sparse_thr, out, workspace, workspace_bytes, dev_status, stream,
                       nullptr, nullptr, 2);
}

int tq_pick_outlier_channels(const tq_kv_desc* desc, const void* v, int v_dtype, int rows, int k,
                             int32_t* channels, void* stream) {
  int st = check_desc(desc);
  if (st != TQ_OK) return st;
  if (desc->head_dim > tq::kMaxDecodeHeadDim) return TQ_ERR_UNSUPPORTED;
  if (v_dtype != TQ_F32 && v_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
  if (rows < 1 || k < 1 || k > TQ_MAX_OUTLIERS || k > desc->head_dim) return TQ_ERR_INVALID_ARG;
  if (!v || !channels || !aligned(v, 16) || !aligned(channels, 4)) return TQ_ERR_INVALID_ARG;
  return tq::launch_pick_outliers(v, v_dtype == TQ_F16, desc->batch, desc->kv_heads, rows, desc->head_dim, k,
                                  channels, static_cast<cudaStream_t>(stream));
}

int tq_read_device_status(const uint32_t* dev_status, uint32_t* bits_out, void* stream) {
  if (!dev_status || !bits_out || !aligned(dev_status, 4)) return TQ_ERR_INVALID_ARG;
  uint32_t bits = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&bits, dev_status, sizeof(bits), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TQ_ERR_CUDA;
  *bits_out = bits;
  return bits ? TQ_ERR_DEVICE_BOUNDS : TQ_OK;
}

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case TQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TQ_ERR_CUDA: return "CUDA runtime error";
    case TQ_ERR_DEVICE_BOUNDS: return "the device status word reports a range error (clamped or skipped rows)";
    case TQ_ERR_SCRATCH_LIMIT: return "request needs more than the built-in no-alloc scratch array";
    default: return "unknown status";
  }
}

}  // extern "C"
