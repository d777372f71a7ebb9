/*
 * tq.h -- C ABI of a TurboQuant-style compressed KV cache for one NVIDIA B200
 * (sm_100a): an encoder that writes packed b-bit codes plus one fp16 norm per
 * 128-element block, and single-token decode attention that reads the packed
 * cache directly.
 *
 * Method (pages cited by title and section):
 *   - "TheTom/llama-cpp-turboquant" README, table "量化类型": every turbo KV
 *     format rotates 128-element blocks with a Walsh-Hadamard transform and
 *     then quantises them with a (polar: radius + direction) codebook.
 *   - intelliparadigm TurboQuant article, §3.2: the rotation is a randomized
 *     Hadamard transform, a Hadamard matrix combined with a random +-1
 *     diagonal, computed with the O(d log d) fast transform; §3.3: the scalar
 *     quantiser is Lloyd-Max.
 *   - "llama-tq" article, section on the K cache: Q.K is evaluated in the
 *     Hadamard domain so the K cache is never dequantised.
 *   - README "压缩策略" and "TurboQuant+" section "注意力门控稀疏V解压": V
 *     positions whose softmax weight is below a threshold are skipped and
 *     count as zero.
 *
 * Conventions that hold for every entry point:
 *   - Ownership: the caller allocates and owns every buffer.  The library
 *     never allocates device memory and keeps no pointer after a call returns.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *     default stream).  Device work is asynchronous on that stream; only
 *     tq_make_codebook and tq_sign_vector are synchronous (host only).
 *   - Launch overlap: the decode entry points without sparse-V launch with
 *     programmatic stream serialisation, so a decode launch may start while
 *     the kernel before it in the stream is still running if that kernel
 *     signals its dependents early (griddepcontrol.launch_dependents /
 *     cudaTriggerProgrammaticLaunchCompletion; of this library's kernels only
 *     the decode kernel does).  The launch reads `seq_lens` before it waits
 *     for that kernel and everything else (query, cache, new rows, workspace,
 *     output) after: a preceding kernel that signals early must not write
 *     `seq_lens` after its signal.  After any other kernel, a copy or an
 *     event wait the launch starts as an ordinary one.
 *   - Errors: every call returns a tq_status code and never throws.  Host-side
 *     validation runs first; when it fails nothing is launched.  Range errors
 *     that only the device can see (a position or a length outside the cache,
 *     an fp16 norm overflow) set bits of the caller's optional device status
 *     word (`dev_status`, one uint32 in device memory, may be NULL); the
 *     offending rows are clamped or skipped and the kernel never traps.
 *   - Block layout: D = head_dim is a multiple of 128; nb = D / 128 blocks
 *     per vector.  For b-bit codes one block stores 16*b bytes of codes
 *     (index i of the block at stream bits [b*i, b*i+b), LSB-first,
 *     little-endian bytes) and one fp16 norm: b + 16/128 bits per value.
 *   - Cache tensors (row-major, contiguous):
 *       codes [batch, kv_heads, seq_cap, nb, 16*b]  uint8
 *       norms [batch, kv_heads, seq_cap, nb]        fp16 (stored as uint16)
 *     K and V are separate tensors, each with its own bit width.  Code
 *     tensors must be 16-byte aligned, norm tensors 4-byte aligned.
 *   - GQA: q-head h reads kv-head h / (q_heads / kv_heads).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_BLOCK 128

/* Return codes. */
typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment           */
  TQ_ERR_UNSUPPORTED = 2,  /* valid but not built: bits, head_dim, group     */
  TQ_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required     */
  TQ_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute) */
  TQ_ERR_DEVICE_BOUNDS = 5,/* tq_read_device_status: a range bit is set      */
  TQ_ERR_SCRATCH_LIMIT = 6 /* needs more than the built-in scratch array      */
} tq_status;

/* Bits of the device status word (sticky; the library only ORs into it). */
#define TQ_DEV_POS_RANGE 1u      /* encode row outside [0, seq_cap): skipped */
#define TQ_DEV_NORM_OVERFLOW 2u  /* block norm above fp16 max: saturated     */
#define TQ_DEV_LEN_RANGE 4u      /* seq_lens[b] outside [0, seq_cap]: clamped */
#define TQ_DEV_INTERNAL 8u       /* internal failure: the decode kernel's
                                    shared-memory plan did not match the device
                                    (nothing was computed; outputs are invalid) */
#define TQ_DEV_CHANNEL_RANGE 16u /* v3 outlier channel outside [0, head_dim):
                                    that entry is stored as 0 and never written
                                    to the output */

typedef enum { TQ_F32 = 0, TQ_F16 = 1 } tq_dtype;

/* Lloyd-Max codebook for N(0,1) with L = 2^bits levels: centroids[0..L-1]
 * ascending and symmetric, boundaries[0..L-2] the midpoints.  Unused tail
 * entries are zero. */
typedef struct {
  int32_t bits;
  float centroids[16];
  float boundaries[15];
} tq_codebook;

/* Shape and format of one layer's compressed KV cache. */
typedef struct {
  int32_t batch;     /* B >= 1                                   */
  int32_t kv_heads;  /* Hkv >= 1                                 */
  int32_t head_dim;  /* D, a multiple of 128: encode <= 512, decode <= 256 */
  int32_t seq_cap;   /* S_cap >= 1: positions per (b, kv-head)   */
  uint64_t sign_seed;/* seed of the +-1 diagonal (SplitMix64)    */
  int32_t k_bits;    /* 2, 3 or 4                                */
  int32_t v_bits;    /* 2, 3 or 4                                */
} tq_kv_desc;

/*
 * tq_make_codebook -- Lloyd-Max quantiser of the standard normal density.
 * Source: intelliparadigm TurboQuant article §3.3 (initialise centres, assign
 * each point to the nearest centre, move each centre to the mean of its
 * points, repeat to convergence), run on the N(0,1) density itself.
 * bits: 1..4.  out: host pointer.  Synchronous, host only, no CUDA calls.
 * Returns TQ_ERR_INVALID_ARG for a null `out`, TQ_ERR_UNSUPPORTED for bits
 * outside 1..4.
 */
int tq_make_codebook(int bits, tq_codebook* out);

/*
 * tq_sign_vector -- the 128 entries (+1 or -1) of the random diagonal D of
 * the rotation H.D (intelliparadigm TurboQuant article §3.2).  Entry i is -1
 * when the top bit of the i-th SplitMix64 output from state `seed` is set.
 * out: host array of 128 int8.  Synchronous, host only.
 */
int tq_sign_vector(uint64_t seed, int8_t* out);

/*
 * tq_encode_kv -- write `seq_new` new positions of K and V into the cache.
 * Per 128-element block ("TheTom/llama-cpp-turboquant" README table
 * "量化类型"; TurboQuant article §3.2-§3.3): x_s = s o x; y = H.x_s (fast
 * WHT, unnormalised); n = ||x||_2 stored as fp16 (round to nearest even);
 * idx_i = #{ j : boundaries[j] < y_i / n }; idx bit-packed as described above.
 *
 * k, v: device, [batch, kv_heads, seq_new, head_dim] contiguous, dtype
 *       in_dtype (TQ_F32 or TQ_F16), 16-byte aligned.  Either may be NULL to
 *       encode only the other side (its codes/norms pointers may then be NULL).
 * start_pos: device int32 [batch] (row t of batch b goes to position
 *       start_pos[b] + t) or NULL (= 0).  Rows that would land outside
 *       [0, seq_cap) are skipped and set TQ_DEV_POS_RANGE.
 * k_cb, v_cb: host codebooks whose bits equal desc->k_bits / desc->v_bits.
 * dev_status: optional device uint32 (see above).
 * seq_new == 0 is a no-op.  Returns TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED
 * on bad arguments (nothing launched), TQ_ERR_CUDA if the launch fails.
 */
int tq_encode_kv(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                 const void* k, const void* v, int in_dtype, int seq_new,
                 const int32_t* start_pos, uint8_t* k_codes, uint16_t* k_norms,
                 uint8_t* v_codes, uint16_t* v_norms, uint32_t* dev_status, void* stream);

/*
 * tq_decode_workspace_size -- bytes of device workspace tq_decode_attention
 * needs for this cache shape, q_heads and sparse setting (sparse_thr > 0 adds
 * an fp32 score buffer of batch * q_heads * seq_cap entries).  Returns 0 for
 * invalid arguments.
 */
size_t tq_decode_workspace_size(const tq_kv_desc* desc, int q_heads, float sparse_thr);

/*
 * tq_decode_attention -- one query token per sequence against the packed
 * cache ("llama-tq" article, K-cache section: Q.K in the Hadamard domain, no
 * K dequantisation; README "压缩策略": sparse-V).
 *   q^ = H.(s o q) per block, once per q-head;
 *   s_t = scale * sum_blk (nK_t,blk / 128) * q^_blk . cK[idx_t,blk];
 *   w = softmax over t < seq_lens[b];
 *   o = sum_t w_t vt_t, computed as s o (H.acc) with
 *       acc = sum_t w_t (nV_t,blk / 128) cV[idx_t,blk] (V summed in the
 *       rotated domain, one inverse rotation per head).
 * Sparse-V (sparse_thr > 0): positions with w_t < sparse_thr (w the
 * normalised weight) contribute zero and the rest are not renormalised.
 *
 * Supported: head_dim 128 or 256, an even seq_cap, batch <= 2048
 * (TQ_ERR_UNSUPPORTED otherwise), and any q_heads / kv_heads ratio (groups
 * above 8 run in slices of 8).
 * q: device [batch, q_heads, head_dim], q_dtype TQ_F32 or TQ_F16.
 *    q_heads must be a multiple of kv_heads.
 * scale: the softmax scale, finite and > 0 (1/sqrt(head_dim) in the usual
 *    attention); other values give TQ_ERR_INVALID_ARG.
 * seq_lens: device int32 [batch]; values are clamped to [0, seq_cap]
 *    (TQ_DEV_LEN_RANGE).  A length of 0 gives an all-zero output row.
 * out: device fp32 [batch, q_heads, head_dim].
 * workspace: device buffer of at least tq_decode_workspace_size() bytes,
 *    256-byte aligned.  It must be all-zero before its first use; every call
 *    that runs to completion leaves it ready for the next call.  Calls that
 *    share one workspace must not overlap in time (use one stream).
 * Returns TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED / TQ_ERR_WORKSPACE on bad
 * arguments (nothing launched), TQ_ERR_CUDA if a launch fails.
 */
int tq_decode_attention(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                        int q_heads, const void* q, int q_dtype,
                        const uint8_t* k_codes, const uint16_t* k_norms,
                        const uint8_t* v_codes, const uint16_t* v_norms,
                        const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                        void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                        void* stream);

/*
 * tq_decode_attention_multi -- n_q query tokens per sequence (a speculative
 * or chunked decode step) against the packed cache.  The README backend table
 * lists CUDA "multi-token" paths without detail; here the n_q tokens are the
 * last n_q positions of each sequence, and query token j (position
 * seq_lens[b] - n_q + j) sees the positions up to its own:
 *   out[b, j, h] = tq_decode_attention output of q[b, j, h] over positions
 *                  [0, seq_lens[b] - n_q + j], zero when that range is empty.
 * All n_q tokens of a sequence are computed from the same K/V fragments of
 * each tile (the codes are turned into MMA operands once per tile).
 *   - n_q: 1..TQ_MAX_QUERY_TOKENS.
 *   - q: device [batch, n_q, q_heads, head_dim]; out: fp32 [batch, n_q,
 *     q_heads, head_dim].
 *   - workspace: tq_decode_workspace_size(desc, q_heads * n_q, sparse_thr)
 *     bytes.
 * Every other argument, limit and error is that of tq_decode_attention
 * (n_q = 1 gives exactly its results).
 */
#define TQ_MAX_QUERY_TOKENS 16
int tq_decode_attention_multi(const tq_kv_desc* desc, const tq_codebook* k_cb,
                              const tq_codebook* v_cb, int q_heads, int n_q, const void* q,
                              int q_dtype, const uint8_t* k_codes, const uint16_t* k_norms,
                              const uint8_t* v_codes, const uint16_t* v_norms,
                              const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                              void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                              void* stream);

/*
 * tq_decode_step -- one decode step in one launch: append every sequence's
 * new token to the cache, then attend over the cache including it.  In a
 * decode step the new token's K/V rows are written into the quantised cache
 * and flash attention then reads it (README backend table: turbo KV rows
 * written by SET_ROWS, read by the flash-attention kernels); here both run in
 * the same kernel.
 *   - seq_lens counts the new token: for sequence b, rows k_new[b, h, :] and
 *     v_new[b, h, :] are encoded exactly as tq_encode_kv would (block norm,
 *     signs, WHT, codebook index, packing) and written at position
 *     seq_lens[b] - 1.  A sequence whose seq_lens[b] is outside [1, seq_cap]
 *     appends nothing, so no cached token is overwritten (values outside
 *     [0, seq_cap] set TQ_DEV_LEN_RANGE and are clamped for the attention).
 *     Then the output is that of tq_decode_attention over positions
 *     [0, seq_lens[b]).
 *   - k_new, v_new: device [batch, kv_heads, head_dim], kv_dtype TQ_F32 or
 *     TQ_F16, 16-byte aligned.  The norms and codes of the appended token
 *     may differ from tq_encode_kv's by one fp16 ulp where the fp32 norm is
 *     at an fp16 rounding midpoint, and by one code where a value is within
 *     rounding of a decision boundary (the norm is summed in another order).
 *   - With sparse_thr > 0 the step is two launches (the append rides in the
 *     first, which scores K).
 * Every other argument, limit and error is that of tq_decode_attention; the
 * cache buffers are written as well as read.
 */
int tq_decode_step(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                   int q_heads, const void* q, int q_dtype, const void* k_new, const void* v_new,
                   int kv_dtype, uint8_t* k_codes, uint16_t* k_norms, uint8_t* v_codes,
                   uint16_t* v_norms, const int32_t* seq_lens, float scale, float sparse_thr,
                   float* out, void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                   void* stream);

/*
 * tq_decode_attention_noalloc -- tq_decode_attention for callers that must
 * not allocate device memory.  The pages have no counterpart: this is a
 * deployment variant of the same decode kernels, not a step of the method.
 *
 * Who needs it: code that receives its device buffers from a host application
 * owning all device memory (a plugin inside a serving engine with its own
 * pool, a component with a fixed memory budget) cannot call cudaMalloc, or
 * cannot afford the device synchronisation an allocation may cause, and so
 * cannot supply a workspace.  This entry point takes the same arguments as
 * tq_decode_attention minus the workspace and allocates nothing: its scratch
 * is a fixed array of TQ_NOALLOC_SCRATCH_BYTES (64 MiB) built into the
 * library, which every GPU that loads the library holds until exit.
 *   - Limit: when tq_decode_workspace_size(desc, q_heads, sparse_thr) exceeds
 *     TQ_NOALLOC_SCRATCH_BYTES it returns TQ_ERR_SCRATCH_LIMIT and launches
 *     nothing.  Other argument errors are those of tq_decode_attention; all
 *     of them are found before any CUDA call is made.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (with that device current); make that first call before any
 *     stream capture.  Later calls do no set-up.  The address is kept for the
 *     life of the process, so this entry point must not be called on a device
 *     after cudaDeviceReset() has destroyed the context it was looked up in.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     last call's contents; each call clears the counters that must start at
 *     zero (one cudaMemsetAsync on `stream`, no allocation).  Calls whose
 *     executions overlap on the GPU (different streams, or concurrent host
 *     threads) race on the array and give wrong results: serialise them.
 */
#define TQ_NOALLOC_SCRATCH_BYTES (64u << 20)
int tq_decode_attention_noalloc(const tq_kv_desc* desc, const tq_codebook* k_cb,
                                const tq_codebook* v_cb, int q_heads, const void* q, int q_dtype,
                                const uint8_t* k_codes, const uint16_t* k_norms,
                                const uint8_t* v_codes, const uint16_t* v_norms,
                                const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                                uint32_t* dev_status, void* stream);

/*
 * tq_read_device_status -- read the device status word that the kernels OR
 * their range errors into (TQ_DEV_* bits above): rows written outside the
 * cache and skipped, lengths clamped, norms saturated.  The kernels never
 * trap on such data; this call is how a caller (or a test) learns of it.
 * dev_status: device pointer, 4-byte aligned, the word passed to the other
 *   calls.  bits_out: host pointer that receives the word.
 * Synchronous: copies the word on `stream` and waits for the stream, so the
 * bits of every call queued before it are included.  The word is not
 * cleared (the caller owns it).  Returns TQ_OK when no bit is set,
 * TQ_ERR_DEVICE_BOUNDS when any is, TQ_ERR_INVALID_ARG for a null or
 * misaligned pointer and TQ_ERR_CUDA if the copy fails.
 */
int tq_read_device_status(const uint32_t* dev_status, uint32_t* bits_out, void* stream);

/*
 * V v3: outlier-channel separation ("llama-tq" article, V sub-families: "v3
 * with outlier-channel separation", the high-quality tier; the pages name the
 * technique only).  Reading taken here: every kv-head has a fixed set of k
 * outlier channels (dimensions of the V vector), chosen by calibration as the
 * k channels of largest mean square; their values are stored exactly as fp16
 * beside the codes, and the V vector with those channels set to zero is
 * encoded as usual (norm of the remainder, signs, WHT, codebook, packing).
 * Decode uses the usual reconstruction of the remainder with the outlier
 * channels replaced by their stored values; k = 0 is the plain format.  K
 * is unchanged.
 *
 *   k:        0..TQ_MAX_OUTLIERS outlier channels per kv-head.
 *   channels: device int32 [kv_heads, k], each row ascending and distinct,
 *             values in [0, head_dim) (an entry outside it sets
 *             TQ_DEV_CHANNEL_RANGE and is ignored).
 *   values:   device fp16 (uint16) [batch, kv_heads, seq_cap, kp], with
 *             kp = 8 when k <= 8 and 16 otherwise (16-byte rows); entry j of a
 *             row holds V[channels[h][j]] and entries k..kp-1 are written 0.
 *             16-byte aligned.
 */
#define TQ_MAX_OUTLIERS 16
typedef struct {
  int32_t k;
  const int32_t* channels;
  uint16_t* values;
} tq_v_outliers;

/*
 * tq_pick_outlier_channels -- calibration of the v3 outlier channels: for
 * every kv-head, the k channels of largest mean square over the rows of v
 * (device [batch, kv_heads, rows, head_dim], v_dtype TQ_F32 or TQ_F16,
 * 16-byte aligned), written ascending to `channels` (device int32
 * [kv_heads, k]); a tie goes to the lower channel.  Asynchronous on `stream`.
 * Returns TQ_ERR_INVALID_ARG for bad pointers or sizes (rows < 1, k outside
 * 1..TQ_MAX_OUTLIERS or above head_dim), TQ_ERR_UNSUPPORTED for a head_dim
 * the decode does not build (above 256), TQ_ERR_CUDA on a launch failure.
 */
int tq_pick_outlier_channels(const tq_kv_desc* desc, const void* v, int v_dtype, int rows, int k,
                             int32_t* channels, void* stream);

/*
 * tq_encode_kv_v3 -- tq_encode_kv with the V side in v3 format: V rows are
 * encoded with the channels of `vo` zeroed and their values written to
 * vo->values (see above).  vo may be NULL or have k = 0 (then this is
 * tq_encode_kv).  Every other argument, limit and error is that of
 * tq_encode_kv; TQ_ERR_INVALID_ARG also for a bad vo (k out of range, null
 * or misaligned channels / values when k > 0, or v NULL with k > 0).
 */
int tq_encode_kv_v3(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                    const void* k, const void* v, int in_dtype, int seq_new,
                    const int32_t* start_pos, uint8_t* k_codes, uint16_t* k_norms,
                    uint8_t* v_codes, uint16_t* v_norms, const tq_v_outliers* vo,
                    uint32_t* dev_status, void* stream);

/*
 * tq_decode_attention_v3 -- tq_decode_attention over a cache whose V side is
 * in v3 format: the output is that of the plain decode with every outlier
 * channel c of each head replaced by sum_t w_t values[t][j] (c =
 * channels[kv-head][j], w the softmax weights, sparse-V gated the same way).
 * vo may be NULL or have k = 0 (then this is tq_decode_attention).  The
 * workspace is tq_decode_workspace_size's.  Every other argument, limit and
 * error is that of tq_decode_attention; in addition, head_dim 256 with
 * k_bits + v_bits >= 7 returns TQ_ERR_UNSUPPORTED (a tile's codes and
 * outlier values no longer fit the kernel's shared-memory rings).
 */
int tq_decode_attention_v3(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_cb,
                           int q_heads, const void* q, int q_dtype, const uint8_t* k_codes,
                           const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_norms,
                           const tq_v_outliers* vo, const int32_t* seq_lens, float scale,
                           float sparse_thr, float* out, void* workspace, size_t workspace_bytes,
                           uint32_t* dev_status, void* stream);

/*
 * V v2: trellis-coded quantisation ("llama-tq" article, V sub-families: "v2
 * based on a group Viterbi trellis", the default V format; the page names
 * the technique only).  Reading taken here: TCQ (Marcellin and Fischer 1990)
 * of the same normalised rotated block coordinates u that the plain format
 * quantises.  The doubled codebook (the 2^(v_bits+1)-level Lloyd-Max
 * quantiser of N(0,1), i.e. tq_make_codebook(v_bits + 1)) is split into four
 * subsets D_k = {levels of index k mod 4}.  A 4-state trellis: branch bit
 * beta moves state s to ((s & 1) << 1) | beta and draws from subset
 * (s & 1) + 2 (beta xor (s >> 1)).  Each 128-coordinate block is one group
 * that starts in state 0; the encoder's Viterbi search picks the path of
 * least squared error (each branch taking the nearest level of its subset;
 * ties to the lower predecessor state, the lower final state and the lower
 * level).  Per coordinate v_bits bits: beta and the level's index j in its
 * subset.  Block layout (16 * v_bits bytes, as the plain format): 64 fields
 * of 2 * v_bits bits, LSB-first; field k = j_2k | j_2k+1 << (b-1) |
 * beta_2k << (2b-2) | beta_2k+1 << (2b-1).  Norms and rotation are the plain
 * format's.  Rates v_bits = 2 and 3; K is the plain format.
 */

/*
 * tq_encode_kv_v2 -- tq_encode_kv with the V side in v2 format.  v_tcq is
 * the doubled codebook (bits = v_bits + 1).  Every other argument, limit and
 * error is that of tq_encode_kv; TQ_ERR_UNSUPPORTED for v_bits outside
 * {2, 3}.  K (when given) is encoded by the plain encoder first.
 */
int tq_encode_kv_v2(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_tcq,
                    const void* k, const void* v, int in_dtype, int seq_new, const int32_t* start_pos,
                    uint8_t* k_codes, uint16_t* k_norms, uint8_t* v_codes, uint16_t* v_norms,
                    uint32_t* dev_status, void* stream);

/*
 * tq_decode_attention_v2 -- tq_decode_attention over a cache whose V side is
 * in v2 format (v_tcq: the doubled codebook).  The V sum runs in the rotated
 * domain on the trellis levels of each coordinate (a level depends on the
 * coordinate's own code and the two branch bits before it).  Every other
 * argument, limit and error is that of tq_decode_attention; TQ_ERR_UNSUPPORTED
 * for v_bits outside {2, 3}.
 */
int tq_decode_attention_v2(const tq_kv_desc* desc, const tq_codebook* k_cb, const tq_codebook* v_tcq,
                           int q_heads, const void* q, int q_dtype, const uint8_t* k_codes,
                           const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_norms,
                           const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                           void* workspace, size_t workspace_bytes, uint32_t* dev_status, void* stream);

/*
 * tq_decode_attention_multi_v3, tq_decode_attention_multi_v2 -- multi-token
 * queries (tq_decode_attention_multi) over a v3 or a v2 V cache: query token
 * j of sequence b sees positions [0, seq_lens[b] - n_q + j], and its output
 * is that of tq_decode_attention_v3 / tq_decode_attention_v2 over that range.
 * q and out are [batch, n_q, q_heads, head_dim]; the workspace is
 * tq_decode_workspace_size(desc, q_heads * n_q, sparse_thr) bytes.  Every
 * other argument, limit and error is that of the single-token entry point of
 * the same format and of tq_decode_attention_multi (n_q = 1 gives exactly
 * the single-token results).
 */
int tq_decode_attention_multi_v3(const tq_kv_desc* desc, const tq_codebook* k_cb,
                                 const tq_codebook* v_cb, int q_heads, int n_q, const void* q,
                                 int q_dtype, const uint8_t* k_codes, const uint16_t* k_norms,
                                 const uint8_t* v_codes, const uint16_t* v_norms,
                                 const tq_v_outliers* vo, const int32_t* seq_lens, float scale,
                                 float sparse_thr, float* out, void* workspace,
                                 size_t workspace_bytes, uint32_t* dev_status, void* stream);
int tq_decode_attention_multi_v2(const tq_kv_desc* desc, const tq_codebook* k_cb,
                                 const tq_codebook* v_tcq, int q_heads, int n_q, const void* q,
                                 int q_dtype, const uint8_t* k_codes, const uint16_t* k_norms,
                                 const uint8_t* v_codes, const uint16_t* v_norms,
                                 const int32_t* seq_lens, float scale, float sparse_thr, float* out,
                                 void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                                 void* stream);

/* Static description of a status code. */
const char* tq_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H_ */
