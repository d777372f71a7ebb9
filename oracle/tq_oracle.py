"""Plain, slow, fp64 CPU oracle for TurboQuant-style KV-cache compression.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, tables or
constants with the CUDA library; every function is written from the pages'
definitions in the most direct form (dense matrices, explicit loops where the
definition is a loop, numpy/BLAS only as a step primitive).

Pages cited (by title and section):
  [llama-tq]      "llama-tq: 让大模型在消费级显卡上跑起10万token长上下文的技术突破",
                  section "KV缓存量化的技术困境与TurboQuant的解决方案" (K cache:
                  randomized Hadamard + Lloyd-Max; Q.K in the Hadamard domain,
                  no K dequantisation; V "v1 codebook" sub-family).
  [tq+ README]    "TheTom/llama-cpp-turboquant" README, table "量化类型"
                  (all turbo formats: WHT rotation then polar codebook
                  quantisation on 128-element blocks) and "压缩策略" (sparse-V
                  dequant: skip V where the softmax weight is below a threshold).
  [TurboQuant+]   "TurboQuant+: 面向生产环境的LLM KV缓存与权重量化技术", sections
                  "Walsh-Hadamard变换" and "注意力门控稀疏V解压" (skipped V is
                  treated as zero).
  [TQ article]    intelliparadigm TurboQuant article, §3.2 "随机哈达玛变换详解"
                  (H_random = D x H, D diagonal random +-1, fast WHT O(d log d)),
                  §3.3 "Lloyd-Max量化算法" (init centres, assign to nearest,
                  centre = mean of its points, repeat), §4.1 table (bits/ratio).

Readings taken where the pages are silent:
  * rotation order H.D (signs first, then the unnormalised Sylvester WHT);
  * sign vector from SplitMix64 (Steele, Lea, Flood 2014), state = seed,
    s_i = -1 when the top bit of the i-th output is set;
  * one sign vector for K, V, every block, head and batch entry;
  * per-block norm = the raw fp64 L2 norm of the input block, stored as fp16
    (round to nearest even); direction u = y / n with the unrounded norm;
  * Lloyd-Max run on the N(0,1) density (not on samples); boundaries are
    midpoints; the fp32-rounded boundaries decide the codes; a value equal to a
    boundary goes to the lower index; a zero block gives index L/2 - 1;
  * codes packed LSB-first into a little-endian bitstream of 16*b bytes;
  * sparse-V weight = normalised softmax weight exp(s - LSE); positions below
    the threshold contribute zero and the rest are not renormalised;
  * V v3 (outlier-channel separation): a fixed set of k channels per kv-head
    (largest mean square on calibration vectors) kept exactly as fp16, the
    rest of the vector encoded as v1 (see encode_v3);
  * V v2 (group-Viterbi trellis): trellis-coded quantisation of the rotated
    block, 4-state trellis, one 128-coordinate block per group (see
    encode_v2).
"""
from __future__ import annotations

import math
from statistics import NormalDist

import numpy as np

BLOCK = 128
_MASK64 = (1 << 64) - 1

# ---------------------------------------------------------------------------
# Rotation: H_random = H . diag(s)   ([TQ article] §3.2; [TurboQuant+] WHT)
# ---------------------------------------------------------------------------


def splitmix64(seed: int, count: int) -> list[int]:
    """The first ``count`` outputs of SplitMix64 started from state ``seed``.

    Published generator (Steele, Lea, Flood, OOPSLA 2014): the state advances
    by the golden-ratio increment and each output is the state passed through
    two xor-shift-multiply rounds and a final xor-shift.
    """
    state = seed & _MASK64
    out = []
    for _ in range(count):
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        z = z ^ (z >> 31)
        out.append(z)
    return out


def sign_vector(seed: int, d: int = BLOCK) -> np.ndarray:
    """The random +-1 diagonal of D ([TQ article] §3.2), as fp64."""
    return np.array([-1.0 if (z >> 63) else 1.0 for z in splitmix64(seed, d)])


def hadamard(d: int = BLOCK) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    h = np.empty((d, d))
    for i in range(d):
        for j in range(d):
            h[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return h


def rotate(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = H . diag(s) . x for every 128-element block along the last axis.

    Dense matrix product, not a butterfly (the oracle must not share the fast
    transform's structure with the kernels).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    assert d % BLOCK == 0
    blocks = x.reshape(*x.shape[:-1], d // BLOCK, BLOCK)
    y = (blocks * signs) @ hadamard(BLOCK).T
    return y.reshape(x.shape)


def unrotate(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """Inverse of :func:`rotate`: x = diag(s) . H . y / d (since H.H^T = d.I)."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    blocks = y.reshape(*y.shape[:-1], d // BLOCK, BLOCK)
    x = (blocks @ hadamard(BLOCK).T) * signs / BLOCK
    return x.reshape(y.shape)


# ---------------------------------------------------------------------------
# Lloyd-Max codebook for N(0,1)   ([TQ article] §3.3; [llama-tq] K cache)
# ---------------------------------------------------------------------------


def _phi(t: float) -> float:
    if math.isinf(t):
        return 0.0
    return math.exp(-0.5 * t * t) / math.sqrt(2.0 * math.pi)


def _Phi(t: float) -> float:
    if t == -math.inf:
        return 0.0
    if t == math.inf:
        return 1.0
    return 0.5 * math.erfc(-t / math.sqrt(2.0))


def lloyd_max_gaussian(bits: int, tol: float = 1e-13, max_iter: int = 200000):
    """Lloyd-Max quantiser of the N(0,1) density, in fp64.

    Follows the four steps of [TQ article] §3.3 with the continuous density in
    place of data points:
      1. initial centres c_j = Phi^-1((j + 1/2) / L);
      2. assignment to the nearest centre = cells bounded by the midpoints
         t_j = (c_j + c_{j+1}) / 2 (t_{-1} = -inf, t_{L-1} = +inf);
      3. each centre becomes the mean of its cell,
         c_j = (phi(t_{j-1}) - phi(t_j)) / (Phi(t_j) - Phi(t_{j-1}));
      4. repeat 2-3 until no centre moves by ``tol`` or more.
    Returns (centroids[L], boundaries[L-1]) in fp64.
    """
    levels = 1 << bits
    nd = NormalDist()
    c = [nd.inv_cdf((j + 0.5) / levels) for j in range(levels)]
    for _ in range(max_iter):
        t = [(c[j] + c[j + 1]) / 2.0 for j in range(levels - 1)]
        edges = [-math.inf] + t + [math.inf]
        new = [(_phi(edges[j]) - _phi(edges[j + 1])) / (_Phi(edges[j + 1]) - _Phi(edges[j]))
               for j in range(levels)]
        delta = max(abs(a - b) for a, b in zip(new, c))
        c = new
        if delta < tol:
            break
    t = [(c[j] + c[j + 1]) / 2.0 for j in range(levels - 1)]
    return np.array(c), np.array(t)


def codebook_f32(bits: int):
    """The codebook as the kernels use it: fp32 centroids and boundaries."""
    c, t = lloyd_max_gaussian(bits)
    return c.astype(np.float32), t.astype(np.float32)


def gaussian_distortion(centroids, boundaries) -> float:
    """E[(X - Q(X))^2] for X ~ N(0,1), from the closed-form cell moments."""
    c = [float(v) for v in centroids]
    edges = [-math.inf] + [float(v) for v in boundaries] + [math.inf]
    total = 0.0
    for j, cj in enumerate(c):
        a, b = edges[j], edges[j + 1]
        p = _Phi(b) - _Phi(a)
        m1 = _phi(a) - _phi(b)                       # integral of x phi(x)
        m2 = p + (a * _phi(a) if not math.isinf(a) else 0.0) \
            - (b * _phi(b) if not math.isinf(b) else 0.0)  # integral of x^2 phi
        total += m2 - 2.0 * cj * m1 + cj * cj * p
    return total


# ---------------------------------------------------------------------------
# Encoder: sign, rotate, norm, quantise, pack ([tq+ README] 量化类型; [llama-tq])
# ---------------------------------------------------------------------------


def quantize(u: np.ndarray, boundaries_f32: np.ndarray) -> np.ndarray:
    """idx = #{ j : t_j < u }, with t_j the fp32 boundaries read as fp64.

    A value equal to a boundary is not counted, so it takes the lower index.
    """
    t = np.asarray(boundaries_f32, dtype=np.float32).astype(np.float64)
    u = np.asarray(u, dtype=np.float64)
    idx = np.zeros(u.shape, dtype=np.int64)
    for tj in t:
        idx += (tj < u)
    return idx


def pack_codes(idx: np.ndarray, bits: int) -> np.ndarray:
    """Bit-pack b-bit indices, LSB-first, into a little-endian bitstream.

    ``idx`` has a last axis of 128; the result has a last axis of 16*bits
    bytes.  Index i occupies stream bits [b*i, b*i + b).
    """
    idx = np.asarray(idx, dtype=np.int64)
    assert idx.shape[-1] == BLOCK
    flat = idx.reshape(-1, BLOCK)
    out = np.zeros((flat.shape[0], 16 * bits), dtype=np.uint8)
    for i in range(BLOCK):
        for k in range(bits):
            bit = (flat[:, i] >> k) & 1
            pos = bits * i + k
            out[:, pos // 8] |= (bit << (pos % 8)).astype(np.uint8)
    return out.reshape(*idx.shape[:-1], 16 * bits)


def unpack_codes(packed: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    packed = np.asarray(packed, dtype=np.uint8)
    assert packed.shape[-1] == 16 * bits
    flat = packed.reshape(-1, 16 * bits).astype(np.int64)
    idx = np.zeros((flat.shape[0], BLOCK), dtype=np.int64)
    for i in range(BLOCK):
        for k in range(bits):
            pos = bits * i + k
            idx[:, i] |= ((flat[:, pos // 8] >> (pos % 8)) & 1) << k
    return idx.reshape(*packed.shape[:-1], BLOCK)


def encode(x: np.ndarray, signs: np.ndarray, bits: int, boundaries_f32: np.ndarray):
    """Encode vectors ``x[..., D]`` (D a multiple of 128).

    Per 128-element block: n = ||x||_2 in fp64; y = H.(s o x); u = y / n
    (u = 0 for a zero block); idx = quantize(u); codes = pack(idx).
    Returns (codes[..., D/128, 16*bits] uint8, norms[..., D/128] fp16,
    u[..., D/128, 128] fp64) -- u is returned so tests can measure distances
    to decision boundaries.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    nb = d // BLOCK
    blocks = x.reshape(*x.shape[:-1], nb, BLOCK)
    n = np.sqrt(np.sum(blocks * blocks, axis=-1))
    y = rotate(blocks, signs)
    with np.errstate(invalid="ignore", divide="ignore"):
        u = np.where(n[..., None] > 0, y / n[..., None], 0.0)
    idx = quantize(u, boundaries_f32)
    return pack_codes(idx, bits), n.astype(np.float16), u


def dequantize(codes: np.ndarray, norms_f16: np.ndarray, bits: int,
               centroids_f32: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """x~ = (n^ / d) . diag(s) . H . c[idx] per block, n^ the stored fp16 norm."""
    idx = unpack_codes(codes, bits)                      # [..., nb, 128]
    c = np.asarray(centroids_f32, dtype=np.float32).astype(np.float64)[idx]
    nhat = np.asarray(norms_f16, dtype=np.float16).astype(np.float64)
    xt = unrotate(c, signs) * nhat[..., None]            # unrotate divides by d
    return xt.reshape(*xt.shape[:-2], xt.shape[-2] * BLOCK)


# ---------------------------------------------------------------------------
# Decode attention
# ---------------------------------------------------------------------------


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, seq_lens, scale: float,
              sparse_thr: float = 0.0) -> np.ndarray:
    """Single-token softmax attention in fp64 on dense K/V.

    q: [B, Hq, D]; k, v: [B, Hkv, S, D]; q-head h reads kv-head h // (Hq/Hkv).
    w = softmax(scale . q.k_t) over t < seq_lens[b] (max-subtracted, fp64).
    Sparse-V ([tq+ README] 压缩策略; [TurboQuant+] 注意力门控稀疏V解压): with
    sparse_thr > 0, positions whose normalised weight w_t is below the
    threshold contribute zero and the kept weights are not renormalised.
    A sequence of length 0 gives a zero output.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    bsz, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    out = np.zeros((bsz, hq, d))
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        for h in range(hq):
            kv = h // group
            s = scale * (k[b, kv, :n] @ q[b, h])
            w = np.exp(s - s.max())
            w = w / w.sum()
            if sparse_thr > 0:
                w = np.where(w < sparse_thr, 0.0, w)
            out[b, h] = w @ v[b, kv, :n]
    return out


def attention_weights(q: np.ndarray, k: np.ndarray, seq_lens, scale: float):
    """Normalised softmax weights w_t = exp(s_t - LSE), s_t = scale . q.k_t, in
    fp64, as a dict {(b, h): w[seq_lens[b]]} (same GQA mapping as attention)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    group = q.shape[1] // k.shape[1]
    out = {}
    for b in range(q.shape[0]):
        n = int(seq_lens[b])
        for h in range(q.shape[1]):
            s = scale * (k[b, h // group, :n] @ q[b, h])
            w = np.exp(s - s.max()) if n else s
            out[(b, h)] = w / w.sum() if n else w
    return out


def decode_dequant(q, k_codes, k_norms, v_codes, v_norms, seq_lens, scale,
                   k_bits, v_bits, k_centroids, v_centroids, signs, sparse_thr=0.0):
    """Formulation A: dequantise the whole cache, then plain attention."""
    kt = dequantize(k_codes, k_norms, k_bits, k_centroids, signs)
    vt = dequantize(v_codes, v_norms, v_bits, v_centroids, signs)
    return attention(q, kt, vt, seq_lens, scale, sparse_thr)


def decode_rotated(q, k_codes, k_norms, v_codes, v_norms, seq_lens, scale,
                   k_bits, v_bits, k_centroids, v_centroids, signs, sparse_thr=0.0):
    """Formulation B: the Hadamard-domain steps, in fp64.

    q^ = H.(s o q) per block (Q rotated once, [llama-tq] K cache);
    s_t = scale . sum_blk (nK_t,blk / d) . q^_blk . cK[idx_t,blk] (no K
    dequantisation); w = softmax(s); V summed in the rotated domain,
    acc = sum_t w_t (nV_t,blk / d) cV[idx_t,blk]; one inverse rotation per
    head, o = s o (H.acc) per block.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, hq, d = q.shape
    hkv = k_codes.shape[1]
    group = hq // hkv
    nb = d // BLOCK
    qhat = rotate(q, signs).reshape(bsz, hq, nb, BLOCK)
    ck = np.asarray(k_centroids, dtype=np.float32).astype(np.float64)[unpack_codes(k_codes, k_bits)]
    cv = np.asarray(v_centroids, dtype=np.float32).astype(np.float64)[unpack_codes(v_codes, v_bits)]
    nk = np.asarray(k_norms, dtype=np.float16).astype(np.float64) / BLOCK
    nv = np.asarray(v_norms, dtype=np.float16).astype(np.float64) / BLOCK
    h_mat = hadamard(BLOCK)
    out = np.zeros((bsz, hq, d))
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        for h in range(hq):
            kv = h // group
            # [n, nb] block dot products, weighted by the block norms.
            dots = np.einsum("tbi,bi->tb", ck[b, kv, :n], qhat[b, h])
            s = scale * np.sum(nk[b, kv, :n] * dots, axis=1)
            w = np.exp(s - s.max())
            w = w / w.sum()
            if sparse_thr > 0:
                w = np.where(w < sparse_thr, 0.0, w)
            acc = np.einsum("t,tb,tbi->bi", w, nv[b, kv, :n], cv[b, kv, :n])
            o = (acc @ h_mat.T) * signs
            out[b, h] = o.reshape(d)
    return out


def attention_multi(q: np.ndarray, k: np.ndarray, v: np.ndarray, seq_lens, scale: float,
                    sparse_thr: float = 0.0) -> np.ndarray:
    """Multi-token queries in fp64 on dense K/V (the CUDA backend's
    "multi-token" path of the [tq+ README] backend table; the pages give no
    detail, so: n_q query tokens per sequence are its last n_q positions, as in
    a speculative or chunked decode step).

    q: [B, n_q, Hq, D]; k, v: [B, Hkv, S, D].  Query token j of sequence b sits
    at position p_j = seq_lens[b] - n_q + j and sees positions t <= p_j: the
    scores form one [n, n_q] matrix with the causal mask t <= p_j applied
    column by column, then softmax per column.  Sparse-V as in attention().
    A token with p_j < 0 gives a zero row.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    bsz, n_q, hq, d = q.shape
    group = hq // k.shape[1]
    out = np.zeros((bsz, n_q, hq, d))
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        t = np.arange(n)[:, None]
        p = n - n_q + np.arange(n_q)[None, :]
        visible = t <= p                                      # [n, n_q]
        for h in range(hq):
            kv = h // group
            s = scale * (k[b, kv, :n] @ q[b, :, h].T)         # [n, n_q]
            s = np.where(visible, s, -np.inf)
            for j in range(n_q):
                if p[0, j] < 0:
                    continue
                w = np.exp(s[:, j] - s[:, j].max())
                w = w / w.sum()
                if sparse_thr > 0:
                    w = np.where(w < sparse_thr, 0.0, w)
                out[b, j, h] = w @ v[b, kv, :n]
    return out


# ---------------------------------------------------------------------------
# V sub-family v3: outlier-channel separation ([llama-tq], K-cache and V
# sub-family sections: "v3 with outlier-channel separation", the high-quality
# tier).  The pages name the technique only.  Reading taken: every kv-head
# has a fixed set of k outlier channels (dimensions of the head vector),
# chosen by calibration as the k channels of largest mean square over sample
# vectors; their values are stored exactly as fp16 beside the codes, and the
# vector with those channels set to zero is encoded as v1 (norm of the
# remainder, rotation, quantisation, packing).  Reconstruction is the v1
# reconstruction of the remainder with the outlier channels replaced by
# their stored values, so k = 0 is v1 and k = D keeps the whole vector.
# ---------------------------------------------------------------------------


def outlier_channels(x: np.ndarray, k: int) -> np.ndarray:
    """The k channels of largest mean square over the sample vectors
    x[..., D] of one kv-head, in ascending channel order (a tie goes to the
    lower channel index)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ms = np.mean(x.reshape(-1, d) ** 2, axis=0)
    order = sorted(range(d), key=lambda c: (-ms[c], c))
    return np.array(sorted(order[:k]), dtype=np.int64)


def encode_v3(x: np.ndarray, signs: np.ndarray, bits: int, boundaries_f32: np.ndarray,
              channels: np.ndarray):
    """v3 encoding of the vectors x[..., D] (one kv-head) with outlier
    channels `channels` [k].  Returns (codes, norms, values fp16 [..., k], u)."""
    x = np.asarray(x, dtype=np.float64)
    ch = np.asarray(channels, dtype=np.int64)
    vals = x[..., ch].astype(np.float16)
    rest = x.copy()
    rest[..., ch] = 0.0
    codes, norms, u = encode(rest, signs, bits, boundaries_f32)
    return codes, norms, vals, u


def dequantize_v3(codes, norms_f16, bits, centroids_f32, signs, values_f16, channels):
    """v1 reconstruction of the remainder, outlier channels replaced by their
    stored fp16 values."""
    xt = dequantize(codes, norms_f16, bits, centroids_f32, signs)
    ch = np.asarray(channels, dtype=np.int64)
    xt[..., ch] = np.asarray(values_f16, dtype=np.float16).astype(np.float64)
    return xt


def decode_v3_dequant(q, k_codes, k_norms, v_codes, v_norms, v_values, v_channels, seq_lens, scale,
                      k_bits, v_bits, k_centroids, v_centroids, signs, sparse_thr=0.0):
    """Formulation A for a v3 V cache: dequantise, then plain attention.
    v_values [B, Hkv, S, k] fp16; v_channels [Hkv, k]."""
    kt = dequantize(k_codes, k_norms, k_bits, k_centroids, signs)
    vt = np.stack([dequantize_v3(v_codes[:, h], v_norms[:, h], v_bits, v_centroids, signs,
                                 v_values[:, h], v_channels[h]) for h in range(v_codes.shape[1])], axis=1)
    return attention(q, kt, vt, seq_lens, scale, sparse_thr)


def decode_v3_rotated(q, k_codes, k_norms, v_codes, v_norms, v_values, v_channels, seq_lens, scale,
                      k_bits, v_bits, k_centroids, v_centroids, signs, sparse_thr=0.0):
    """Formulation B for a v3 V cache: the rotated-domain decode of the
    remainders (decode_rotated), then each outlier channel of the output
    replaced by the weighted sum of its stored values, sum_t w_t val_t."""
    out = decode_rotated(q, k_codes, k_norms, v_codes, v_norms, seq_lens, scale, k_bits, v_bits,
                         k_centroids, v_centroids, signs, sparse_thr)
    kt = dequantize(k_codes, k_norms, k_bits, k_centroids, signs)
    ws = attention_weights(q, kt, seq_lens, scale)
    group = q.shape[1] // k_codes.shape[1]
    vv = np.asarray(v_values, dtype=np.float16).astype(np.float64)
    for (b, h), w in ws.items():
        n = int(seq_lens[b])
        if n == 0:
            continue
        if sparse_thr > 0:
            w = np.where(w < sparse_thr, 0.0, w)
        kv = h // group
        out[b, h, np.asarray(v_channels[kv], dtype=np.int64)] = w @ vv[b, kv, :n]
    return out


def sparse_skip_fraction(q, k, seq_lens, scale, thr, group):
    """Fraction of (q-head, position) pairs whose normalised weight is < thr."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    skipped = total = 0
    for b in range(q.shape[0]):
        n = int(seq_lens[b])
        for h in range(q.shape[1]):
            s = scale * (k[b, h // group, :n] @ q[b, h])
            w = np.exp(s - s.max())
            w /= w.sum()
            skipped += int(np.sum(w < thr))
            total += n
    return skipped / max(total, 1)


# ---------------------------------------------------------------------------
# V sub-family v2: group-Viterbi trellis coding ([llama-tq], V sub-family
# section: "v2 based on a group-Viterbi trellis", the default V format; V is
# heavy-tailed and a trellis spends its bits where the values are).  The pages
# name the technique only.  Reading taken: trellis-coded quantisation (TCQ,
# Marcellin and Fischer, IEEE Trans. Commun. 38(1), 1990) of the same
# normalised rotated coordinates u that v1 quantises, with
#   * the doubled codebook: the 2^(b+1)-level Lloyd-Max quantiser of N(0,1)
#     (fp32 levels), partitioned into four subsets D_k = {levels whose index
#     is k mod 4}, each ascending with 2^(b-1) levels;
#   * the 4-state trellis of Ungerboeck's amplitude-modulation code that TCQ
#     uses: state s and branch bit beta lead to state ((s & 1) << 1) | beta,
#     and the branch carries subset TCQ_SUBSET[s][beta]; even states draw
#     from D0 u D2, odd states from D1 u D3;
#   * a group = one 128-coordinate block, starting in state 0, no tail
#     condition; the encoder is the Viterbi search for the path of least
#     squared error sum_i (u_i - level_i)^2, where each branch takes the
#     nearest level of its subset;
#   * per coordinate b bits: the branch bit beta_i and the index j_i of the
#     level inside its subset (level index 4 j_i + subset);
#   * storage per block (16 b bytes, as v1): 64 fields of 2b bits, one per
#     coordinate pair (2k, 2k+1), LSB-first in a little-endian bitstream;
#     field k = j_2k | j_2k+1 << (b-1) | beta_2k << (2b-2) | beta_2k+1 << (2b-1),
#     so the 2b + 2 stream bits that end with field k hold everything the
#     levels of the pair depend on (the pair's own bits and the two branch
#     bits before it);
#   * ties: a smaller path metric wins, then the lower predecessor state, then
#     the lower final state; inside a subset the lower level wins.
# Norms and rotation are those of v1; the reconstruction is the v1 one with
# the trellis levels in place of the centroids.
# ---------------------------------------------------------------------------

TCQ_NEXT = ((0, 1), (2, 3), (0, 1), (2, 3))     # [state][branch bit] -> state
TCQ_SUBSET = ((0, 2), (1, 3), (2, 0), (3, 1))   # [state][branch bit] -> subset k


def tcq_levels_f32(bits: int) -> np.ndarray:
    """The doubled codebook of a b-bit v2 code: 2^(b+1) fp32 levels."""
    return codebook_f32(bits + 1)[0]


def _nearest_in_subset(u: float, levels: np.ndarray, k: int):
    """(j, squared error) of the level of subset D_k nearest to u (the lower
    level on a tie)."""
    best_j, best_e = 0, math.inf
    for j in range(len(levels) // 4):
        e = (u - float(levels[4 * j + k])) ** 2
        if e < best_e:
            best_j, best_e = j, e
    return best_j, best_e


def tcq_viterbi(u: np.ndarray, levels: np.ndarray):
    """Viterbi search over the 4-state trellis for one group of coordinates
    u[n], from state 0.  Returns (beta[n], j[n], squared error of the path)."""
    u = [float(v) for v in np.asarray(u, dtype=np.float64).ravel()]
    n = len(u)
    metric = [0.0, math.inf, math.inf, math.inf]
    back = []  # per step and state: (predecessor, branch bit, j)
    for i in range(n):
        new = [math.inf] * 4
        step = [None] * 4
        for s_next in range(4):
            beta = s_next & 1
            for pred in (s_next >> 1, (s_next >> 1) | 2):   # lower predecessor first
                assert TCQ_NEXT[pred][beta] == s_next
                if metric[pred] == math.inf:
                    continue
                j, e = _nearest_in_subset(u[i], levels, TCQ_SUBSET[pred][beta])
                cost = metric[pred] + e
                if cost < new[s_next]:
                    new[s_next], step[s_next] = cost, (pred, beta, j)
        metric = new
        back.append(step)
    state = min(range(4), key=lambda s: (metric[s], s))
    total = metric[state]
    beta = np.zeros(n, dtype=np.int64)
    jj = np.zeros(n, dtype=np.int64)
    for i in range(n - 1, -1, -1):
        pred, beta[i], jj[i] = back[i][state]
        state = pred
    return beta, jj, total


def tcq_reconstruct(beta: np.ndarray, j: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """Levels of a path: walk the trellis from state 0 along the branch bits."""
    out = np.zeros(len(beta))
    state = 0
    for i in range(len(beta)):
        b = int(beta[i])
        out[i] = float(levels[4 * int(j[i]) + TCQ_SUBSET[state][b]])
        state = TCQ_NEXT[state][b]
    return out


def pack_v2(beta: np.ndarray, j: np.ndarray, bits: int) -> np.ndarray:
    """The v2 block layout: one 2b-bit field per coordinate pair, written
    LSB-first into a little-endian bitstream of 16 b bytes; field k holds
    j_2k, j_2k+1 (b - 1 bits each), then beta_2k, beta_2k+1.  Last axes
    [..., 128] -> [..., 16 b]."""
    beta = np.asarray(beta, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    assert beta.shape[-1] == BLOCK and j.shape == beta.shape
    fb = beta.reshape(-1, BLOCK)
    fj = j.reshape(-1, BLOCK)
    out = np.zeros((fb.shape[0], 16 * bits), dtype=np.uint8)
    w = bits - 1
    for k in range(BLOCK // 2):
        field = fj[:, 2 * k] | (fj[:, 2 * k + 1] << w) | (fb[:, 2 * k] << (2 * w)) | (fb[:, 2 * k + 1] << (2 * w + 1))
        for t in range(2 * bits):
            pos = 2 * bits * k + t
            out[:, pos // 8] |= (((field >> t) & 1) << (pos % 8)).astype(np.uint8)
    return out.reshape(*beta.shape[:-1], 16 * bits)


def unpack_v2(packed: np.ndarray, bits: int):
    """Inverse of :func:`pack_v2`: (beta[..., 128], j[..., 128])."""
    packed = np.asarray(packed, dtype=np.uint8)
    assert packed.shape[-1] == 16 * bits
    flat = packed.reshape(-1, 16 * bits).astype(np.int64)
    beta = np.zeros((flat.shape[0], BLOCK), dtype=np.int64)
    j = np.zeros((flat.shape[0], BLOCK), dtype=np.int64)
    w = bits - 1
    for k in range(BLOCK // 2):
        field = np.zeros(flat.shape[0], dtype=np.int64)
        for t in range(2 * bits):
            pos = 2 * bits * k + t
            field |= ((flat[:, pos // 8] >> (pos % 8)) & 1) << t
        j[:, 2 * k] = field & ((1 << w) - 1)
        j[:, 2 * k + 1] = (field >> w) & ((1 << w) - 1)
        beta[:, 2 * k] = (field >> (2 * w)) & 1
        beta[:, 2 * k + 1] = (field >> (2 * w + 1)) & 1
    shape = packed.shape[:-1] + (BLOCK,)
    return beta.reshape(shape), j.reshape(shape)


def encode_v2(x: np.ndarray, signs: np.ndarray, bits: int, levels_f32: np.ndarray):
    """v2 encoding of x[..., D]: the v1 norm and rotation, u = y / n per block,
    then one Viterbi search per block.  Returns (codes [..., D/128, 16 b] in
    the v2 layout, norms fp16, u, per-block squared error of the chosen
    path)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    nb = d // BLOCK
    blocks = x.reshape(*x.shape[:-1], nb, BLOCK)
    n = np.sqrt(np.sum(blocks * blocks, axis=-1))
    y = rotate(blocks, signs)
    with np.errstate(invalid="ignore", divide="ignore"):
        u = np.where(n[..., None] > 0, y / n[..., None], 0.0)
    flat = u.reshape(-1, BLOCK)
    beta = np.zeros(flat.shape, dtype=np.int64)
    jj = np.zeros(flat.shape, dtype=np.int64)
    err = np.zeros(flat.shape[0])
    for r in range(flat.shape[0]):
        beta[r], jj[r], err[r] = tcq_viterbi(flat[r], levels_f32)
    beta = beta.reshape(u.shape)
    jj = jj.reshape(u.shape)
    return pack_v2(beta, jj, bits), n.astype(np.float16), u, err.reshape(u.shape[:-1])


def v2_levels(codes: np.ndarray, bits: int, levels_f32: np.ndarray) -> np.ndarray:
    """Trellis levels of every coordinate of v2-coded blocks [..., 16 b] ->
    [..., 128] (the rotated-domain values before the norm)."""
    beta, jj = unpack_v2(codes, bits)
    fb = beta.reshape(-1, BLOCK)
    fj = jj.reshape(-1, BLOCK)
    out = np.stack([tcq_reconstruct(fb[r], fj[r], levels_f32) for r in range(fb.shape[0])])
    return out.reshape(beta.shape)


def dequantize_v2(codes: np.ndarray, norms_f16: np.ndarray, bits: int, levels_f32: np.ndarray,
                  signs: np.ndarray) -> np.ndarray:
    """x~ = (n^ / d) . diag(s) . H . level[path] per block."""
    lv = v2_levels(codes, bits, levels_f32)
    nhat = np.asarray(norms_f16, dtype=np.float16).astype(np.float64)
    xt = unrotate(lv, signs) * nhat[..., None]
    return xt.reshape(*xt.shape[:-2], xt.shape[-2] * BLOCK)


def decode_v2_dequant(q, k_codes, k_norms, v_codes, v_norms, seq_lens, scale, k_bits, v_bits,
                      k_centroids, v_levels_f32, signs, sparse_thr=0.0):
    """Formulation A for a v2 V cache: dequantise, then plain attention."""
    kt = dequantize(k_codes, k_norms, k_bits, k_centroids, signs)
    vt = dequantize_v2(v_codes, v_norms, v_bits, v_levels_f32, signs)
    return attention(q, kt, vt, seq_lens, scale, sparse_thr)


def decode_v2_rotated(q, k_codes, k_norms, v_codes, v_norms, seq_lens, scale, k_bits, v_bits,
                      k_centroids, v_levels_f32, signs, sparse_thr=0.0):
    """Formulation B for a v2 V cache: scores in the Hadamard domain from the
    K codes; V summed in the rotated domain from the trellis levels,
    acc = sum_t w_t (nV_t,blk / d) level_t,blk; one inverse rotation per head."""
    q = np.asarray(q, dtype=np.float64)
    bsz, hq, d = q.shape
    hkv = k_codes.shape[1]
    group = hq // hkv
    nb = d // BLOCK
    qhat = rotate(q, signs).reshape(bsz, hq, nb, BLOCK)
    ck = np.asarray(k_centroids, dtype=np.float32).astype(np.float64)[unpack_codes(k_codes, k_bits)]
    lv = v2_levels(v_codes, v_bits, v_levels_f32)
    nk = np.asarray(k_norms, dtype=np.float16).astype(np.float64) / BLOCK
    nv = np.asarray(v_norms, dtype=np.float16).astype(np.float64) / BLOCK
    h_mat = hadamard(BLOCK)
    out = np.zeros((bsz, hq, d))
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        for h in range(hq):
            kv = h // group
            dots = np.einsum("tbi,bi->tb", ck[b, kv, :n], qhat[b, h])
            s = scale * np.sum(nk[b, kv, :n] * dots, axis=1)
            w = np.exp(s - s.max())
            w = w / w.sum()
            if sparse_thr > 0:
                w = np.where(w < sparse_thr, 0.0, w)
            acc = np.einsum("t,tb,tbi->bi", w, nv[b, kv, :n], lv[b, kv, :n])
            out[b, h] = ((acc @ h_mat.T) * signs).reshape(d)
    return out
