"""Pins of the CPU oracle to facts fixed outside it (CPU only).

Each test checks one oracle function against something other than itself: a
closed form, an invariant of the mathematics, a published table, a library
routine, or brute force.  A plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import tq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_max():
    table = {}
    with open(os.path.join(GOLDEN, "max1960_gaussian.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            lv, kind, vals = [p.strip() for p in line.split("|")]
            table[(int(lv), kind)] = [float(v) for v in vals.split()]
    return table


def _fwht(x):
    """Independent in-place butterfly Walsh-Hadamard transform (unnormalised)."""
    x = np.array(x, dtype=np.float64)
    h = 1
    while h < x.shape[-1]:
        for i in range(0, x.shape[-1], 2 * h):
            a = x[..., i:i + h].copy()
            b = x[..., i + h:i + 2 * h].copy()
            x[..., i:i + h] = a + b
            x[..., i + h:i + 2 * h] = a - b
        h *= 2
    return x


# --------------------------------------------------------------- rotation ---

def test_hadamard_orthogonal_exact():
    h = O.hadamard(128)
    assert np.array_equal(h @ h.T, 128.0 * np.eye(128))
    assert np.array_equal(h, h.T)
    assert set(np.unique(h)) == {-1.0, 1.0}


def test_dense_rotation_equals_butterfly():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 256))
    s = O.sign_vector(5)
    dense = O.rotate(x, s)
    fast = np.concatenate([_fwht(s * x[:, :128]), _fwht(s * x[:, 128:])], axis=1)
    assert np.max(np.abs(dense - fast)) <= 1e-12 * np.max(np.abs(fast))


def test_rotation_preserves_geometry_up_to_d():
    rng = np.random.default_rng(2)
    x, y = rng.standard_normal((2, 128))
    s = O.sign_vector(0)
    rx, ry = O.rotate(x, s), O.rotate(y, s)
    assert math.isclose(rx @ ry, 128.0 * (x @ y), rel_tol=1e-12, abs_tol=1e-9)
    assert math.isclose(np.linalg.norm(rx), math.sqrt(128) * np.linalg.norm(x), rel_tol=1e-12)
    assert np.allclose(O.unrotate(rx, s), x, atol=1e-12)


def test_splitmix64_published_check_values():
    with open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) as f:
        want = [int(l) for l in f if l.strip() and not l.startswith("#")]
    assert O.splitmix64(1234567, 5) == want


def test_sign_vector_is_top_bit_of_splitmix64():
    s = O.sign_vector(1234567, 5)
    with open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) as f:
        want = [int(l) for l in f if l.strip() and not l.startswith("#")]
    assert list(s) == [-1.0 if w >= 2**63 else 1.0 for w in want]
    s0 = O.sign_vector(0)
    assert s0.shape == (128,) and set(np.unique(s0)) == {-1.0, 1.0}
    assert 40 < np.sum(s0 > 0) < 88


# --------------------------------------------------------------- codebook ---

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_max_1960(bits):
    table = _golden_max()
    levels = 1 << bits
    c, t = O.lloyd_max_gaussian(bits)
    half = c[levels // 2:]
    np.testing.assert_allclose(half, table[(levels, "centroids")], rtol=6e-4, atol=6e-4)
    if (levels, "boundaries") in table:
        np.testing.assert_allclose(t[levels // 2:], table[(levels, "boundaries")], rtol=6e-4, atol=6e-4)
    dist = O.gaussian_distortion(c, t)
    assert math.isclose(dist, table[(levels, "distortion")][0], rel_tol=2e-3)


def test_codebook_one_bit_closed_form():
    c, t = O.lloyd_max_gaussian(1)
    assert math.isclose(c[1], math.sqrt(2 / math.pi), rel_tol=1e-12)
    assert c[0] == -c[1] and t[0] == 0.0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codebook_fixed_point_conditions_by_quadrature(bits):
    """Centroid condition checked with numerical quadrature (independent of the
    closed-form cell moments the oracle iterates); midpoint condition exactly."""
    c, t = O.lloyd_max_gaussian(bits)
    levels = len(c)
    np.testing.assert_allclose(c, -c[::-1], atol=1e-15)
    np.testing.assert_allclose(t, (c[:-1] + c[1:]) / 2, atol=0)
    edges = [-np.inf] + list(t) + [np.inf]
    for j in range(levels):
        mass = integrate.quad(stats.norm.pdf, edges[j], edges[j + 1], epsabs=1e-14)[0]
        mom = integrate.quad(lambda x: x * stats.norm.pdf(x), edges[j], edges[j + 1], epsabs=1e-14)[0]
        assert abs(mom / mass - c[j]) < 1e-9


def test_codebook_unique_fixed_point_from_other_init():
    """N(0,1) is log-concave, so Lloyd-Max has one fixed point: a plain
    sample-free iteration started from a uniform grid reaches the same one."""
    for bits in (2, 3, 4):
        c_ref, _ = O.lloyd_max_gaussian(bits)
        levels = 1 << bits
        c = np.linspace(-2.5, 2.5, levels)
        for _ in range(20000):
            t = (c[:-1] + c[1:]) / 2
            e = np.concatenate([[-np.inf], t, [np.inf]])
            c = (stats.norm.pdf(e[:-1]) - stats.norm.pdf(e[1:])) / (stats.norm.cdf(e[1:]) - stats.norm.cdf(e[:-1]))
        np.testing.assert_allclose(c, c_ref, atol=1e-9)


# -------------------------------------------------------------- quantizer ---

@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantizer_is_nearest_centroid(bits):
    c32, t32 = O.codebook_f32(bits)
    rng = np.random.default_rng(bits)
    u = np.concatenate([rng.standard_normal(200000) * 1.5,
                        np.nextafter(t32.astype(np.float64), np.inf),
                        np.nextafter(t32.astype(np.float64), -np.inf)])
    idx = O.quantize(u, t32)
    brute = np.argmin(np.abs(u[:, None] - c32.astype(np.float64)[None, :]), axis=1)
    # Away from a boundary the nearest centroid is unique and must agree.
    far = np.min(np.abs(u[:, None] - t32.astype(np.float64)[None, :]), axis=1) > 1e-6
    assert np.array_equal(idx[far], brute[far])
    # Exactly on a boundary: lower index.  Zero maps to L/2 - 1.
    assert np.array_equal(O.quantize(t32.astype(np.float64), t32), np.arange(len(t32)))
    assert O.quantize(np.array([0.0]), t32)[0] == (1 << bits) // 2 - 1


# ---------------------------------------------------------------- packing ---

def test_pack_known_patterns():
    idx4 = np.arange(128) % 16
    p4 = O.pack_codes(idx4, 4)
    assert p4.shape == (64,)
    assert list(p4[:3]) == [0x10, 0x32, 0x54]
    idx2 = np.arange(128) % 4
    assert np.all(O.pack_codes(idx2, 2) == 0xE4)
    idx3 = np.arange(128) % 8          # 0..7 repeats: octal 01234567 -> 88 C6 FA
    p3 = O.pack_codes(idx3, 3)
    assert p3.shape == (48,)
    assert list(p3[:6]) == [0x88, 0xC6, 0xFA, 0x88, 0xC6, 0xFA]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip_and_bits_per_value(bits):
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, size=(3, 5, 128))
    packed = O.pack_codes(idx, bits)
    assert np.array_equal(O.unpack_codes(packed, bits), idx)
    # Stored bytes per 128-block: 16*b code bytes + one fp16 norm.
    per_block = packed.shape[-1] + 2
    assert per_block * 8 / 128 == bits + 16 / 128
    assert round(16 / (bits + 0.125), 2) == {2: 7.53, 3: 5.12, 4: 3.88}[bits]


# ---------------------------------------------------------------- encoder ---

def _sphere_coordinate_mse(centroids, boundaries, d=128):
    """E[(u - Q(u))^2] where u/sqrt(d) is one coordinate of a uniform point
    on the unit sphere in R^d: density prop. to (1 - u^2/d)^((d-3)/2)."""
    r = math.sqrt(d)
    dens = lambda u: (1 - u * u / d) ** ((d - 3) / 2)
    z = integrate.quad(dens, -r, r)[0]
    edges = [-r] + [float(b) for b in boundaries] + [r]
    tot = 0.0
    for j, cj in enumerate(centroids):
        tot += integrate.quad(lambda u: (u - float(cj)) ** 2 * dens(u), edges[j], edges[j + 1])[0]
    return tot / z


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_reconstruction_mse_matches_sphere_integral(bits):
    c32, t32 = O.codebook_f32(bits)
    s = O.sign_vector(0)
    rng = np.random.default_rng(10 + bits)
    x = rng.standard_normal((3000, 128)) * rng.lognormal(0, 1, (3000, 1))
    codes, norms, _ = O.encode(x, s, bits, t32)
    xt = O.dequantize(codes, norms, bits, c32, s)
    rel = np.mean(np.sum((x - xt) ** 2, axis=1) / np.sum(x * x, axis=1))
    want = _sphere_coordinate_mse(c32, t32)
    assert abs(rel - want) < 0.02 * want, (rel, want)


def test_encode_norm_and_zero_block():
    s = O.sign_vector(3)
    c32, t32 = O.codebook_f32(3)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((4, 256))
    x[2, :128] = 0.0
    codes, norms, u = O.encode(x, s, 3, t32)
    assert norms.dtype == np.float16 and norms.shape == (4, 2)
    np.testing.assert_array_equal(norms, np.linalg.norm(x.reshape(4, 2, 128), axis=-1).astype(np.float16))
    assert np.all(O.unpack_codes(codes[2, 0], 3) == 3)
    # u has unit second moment per coordinate: |u|^2 = d exactly.
    np.testing.assert_allclose(np.sum(u[0] ** 2, axis=-1), 128.0, rtol=1e-12)


# -------------------------------------------------------------- attention ---

def _random_cache(rng, bsz, hkv, seq, d, kb, vb, seed=0):
    s = O.sign_vector(seed)
    ck, tk = O.codebook_f32(kb)
    cv, tv = O.codebook_f32(vb)
    k = rng.standard_normal((bsz, hkv, seq, d))
    v = rng.standard_normal((bsz, hkv, seq, d))
    kc, kn, _ = O.encode(k, s, kb, tk)
    vc, vn, _ = O.encode(v, s, vb, tv)
    return s, (ck, cv), (k, v), (kc, kn, vc, vn)


def test_two_formulations_agree():
    rng = np.random.default_rng(7)
    s, (ck, cv), _, (kc, kn, vc, vn) = _random_cache(rng, 2, 2, 40, 256, 3, 2)
    q = rng.standard_normal((2, 8, 256))
    lens = [40, 17]
    for thr in (0.0, 2e-2):
        a = O.decode_dequant(q, kc, kn, vc, vn, lens, 1 / 16, 3, 2, ck, cv, s, thr)
        b = O.decode_rotated(q, kc, kn, vc, vn, lens, 1 / 16, 3, 2, ck, cv, s, thr)
        assert np.max(np.abs(a - b)) <= 1e-10 * np.max(np.abs(a))


def test_attention_special_cases():
    rng = np.random.default_rng(8)
    s, (ck, cv), _, (kc, kn, vc, vn) = _random_cache(rng, 1, 1, 6, 128, 4, 4)
    vt = O.dequantize(vc, vn, 4, cv, s)
    kt = O.dequantize(kc, kn, 4, ck, s)
    q = rng.standard_normal((1, 1, 128))
    dec = lambda qq, lens, thr=0.0: O.decode_rotated(qq, kc, kn, vc, vn, lens, 1 / math.sqrt(128), 4, 4, ck, cv, s, thr)
    np.testing.assert_allclose(dec(q, [1])[0, 0], vt[0, 0, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dec(np.zeros_like(q), [6])[0, 0], vt[0, 0].mean(axis=0), atol=1e-12)
    assert np.all(dec(q, [0]) == 0)
    # Two positions, expanded by hand: o = sigmoid(s0 - s1) v0 + sigmoid(s1 - s0) v1.
    sc = (kt[0, 0, :2] @ q[0, 0]) / math.sqrt(128)
    w0 = 1 / (1 + math.exp(sc[1] - sc[0]))
    np.testing.assert_allclose(dec(q, [2])[0, 0], w0 * vt[0, 0, 0] + (1 - w0) * vt[0, 0, 1], atol=1e-12)
    # One dominant score picks its value vector.
    qd = 60.0 * kt[0, 0, 3][None, None, :] / np.linalg.norm(kt[0, 0, 3])
    np.testing.assert_allclose(dec(qd, [6])[0, 0], vt[0, 0, 3], atol=1e-6)
    # A threshold above every weight leaves nothing; a threshold <= 0 is dense.
    assert np.all(dec(q, [6], thr=1.01) == 0)
    np.testing.assert_array_equal(dec(q, [6], thr=-1.0), dec(q, [6]))


def test_dense_attention_matches_torch_sdpa():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, 8, 128))
    k = rng.standard_normal((2, 2, 30, 128))
    v = rng.standard_normal((2, 2, 30, 128))
    lens = [30, 11]
    ours = O.attention(q, k, v, lens, 1 / math.sqrt(128))
    for b in range(2):
        n = lens[b]
        qt = torch.tensor(q[b][:, None, :])                         # [Hq, 1, D]
        kt = torch.tensor(np.repeat(k[b, :, :n], 4, axis=0))       # [Hq, n, D]
        vt = torch.tensor(np.repeat(v[b, :, :n], 4, axis=0))
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=1 / math.sqrt(128))
        np.testing.assert_allclose(ours[b], ref[:, 0].numpy(), rtol=1e-12, atol=1e-12)


def test_sparse_skip_fraction_matches_gaussian_prediction():
    """w_t < thr with w_t = exp(s_t - LSE).  Given q, the scores are
    N(0, sigma^2) with sigma = scale |q|, so LSE ~ log N + sigma^2 / 2 and the
    skipped fraction is Phi((log(thr N) + sigma^2/2) / sigma)."""
    rng = np.random.default_rng(11)
    n, d, heads = 4096, 128, 32
    thr = 1e-6 * 131072 / n
    q = rng.standard_normal((1, heads, d))
    k = rng.standard_normal((1, 1, n, d))
    got = O.sparse_skip_fraction(q, k, [n], 1 / math.sqrt(d), thr, heads)
    sig = np.linalg.norm(q[0], axis=1) / math.sqrt(d)
    pred = np.mean(stats.norm.cdf((np.log(thr * n) + sig ** 2 / 2) / sig))
    assert abs(got - pred) < 0.004, (got, pred)
    assert 0.04 < got < 0.09


def test_attention_weights_match_torch_softmax():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(12)
    q = rng.standard_normal((2, 4, 128))
    k = rng.standard_normal((2, 2, 20, 128))
    ws = O.attention_weights(q, k, [20, 7], 0.1)
    for (b, h), w in ws.items():
        n = [20, 7][b]
        ref = torch.softmax(torch.tensor(k[b, h // 2, :n] @ q[b, h]) * 0.1, dim=0).numpy()
        np.testing.assert_allclose(w, ref, rtol=1e-12, atol=1e-15)


def test_multi_token_attention_single_token_is_decode():
    rng = np.random.default_rng(21)
    q = rng.standard_normal((2, 8, 128))
    k = rng.standard_normal((2, 2, 40, 128))
    v = rng.standard_normal((2, 2, 40, 128))
    lens = [40, 9]
    got = O.attention_multi(q[:, None], k, v, lens, 0.09)[:, 0]
    np.testing.assert_allclose(got, O.attention(q, k, v, lens, 0.09), rtol=1e-12, atol=1e-12)


def test_multi_token_attention_matches_torch_sdpa_with_causal_mask():
    """Query token j of a sequence of length n sits at n - n_q + j and sees
    t <= n - n_q + j: an explicit boolean mask for torch's SDPA."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(22)
    n_q, scale = 5, 1 / math.sqrt(128)
    q = rng.standard_normal((2, n_q, 8, 128))
    k = rng.standard_normal((2, 2, 30, 128))
    v = rng.standard_normal((2, 2, 30, 128))
    lens = [30, 12]
    ours = O.attention_multi(q, k, v, lens, scale)
    for b in range(2):
        n = lens[b]
        qt = torch.tensor(q[b].transpose(1, 0, 2))                  # [Hq, n_q, D]
        kt = torch.tensor(np.repeat(k[b, :, :n], 4, axis=0))       # [Hq, n, D]
        vt = torch.tensor(np.repeat(v[b, :, :n], 4, axis=0))
        mask = torch.tensor(np.arange(n)[None, :] <= (n - n_q + np.arange(n_q))[:, None])  # [n_q, n]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
        np.testing.assert_allclose(ours[b], ref.numpy().transpose(1, 0, 2), rtol=1e-12, atol=1e-12)


def test_multi_token_attention_is_decode_at_each_position():
    """Token j equals single-token attention over the first n - n_q + j + 1
    positions; a token before the sequence start gives zeros; positions past
    seq_lens never matter."""
    rng = np.random.default_rng(23)
    n_q = 4
    q = rng.standard_normal((3, n_q, 4, 128))
    k = rng.standard_normal((3, 1, 20, 128))
    v = rng.standard_normal((3, 1, 20, 128))
    lens = np.array([20, 7, 2])
    got = O.attention_multi(q, k, v, lens, 0.1, sparse_thr=1e-3)
    for j in range(n_q):
        lj = np.maximum(lens - n_q + j + 1, 0)
        want = O.attention(q[:, j], k, v, lj, 0.1, sparse_thr=1e-3)
        np.testing.assert_allclose(got[:, j], want, rtol=1e-12, atol=1e-12)
    assert np.all(got[2, :2] == 0.0)                                # positions -2, -1
    k2, v2 = k.copy(), v.copy()
    k2[1, :, 7:] = 1e6
    v2[1, :, 7:] = np.nan
    np.testing.assert_array_equal(O.attention_multi(q, k2, v2, lens, 0.1)[1],
                                  O.attention_multi(q, k, v, lens, 0.1)[1])


# --------------------------------------------------------- sparse-V gate ---
# README "压缩策略" and "TurboQuant+" section "注意力门控稀疏V解压": V rows whose
# softmax weight is below the threshold are skipped and count as zero.  The
# weight is the normalised softmax weight; the kept weights are not rescaled.
# The reference below is torch.softmax (a library routine) with the mask
# applied to its output, so neither slip of the oracle's gate -- gating on the
# unnormalised exp(s - max), or renormalising the kept weights -- can hide.


def _torch_gated(q, k, v, lens, scale, thr, limits=None):
    """o[b, h] = sum_t [w_t >= thr] w_t v_t with w = torch.softmax(scale q.k)."""
    torch = pytest.importorskip("torch")
    group = q.shape[1] // k.shape[1]
    out = np.zeros(q.shape)
    for b in range(q.shape[0]):
        n = int(lens[b] if limits is None else limits[b])
        if n <= 0:
            continue
        for h in range(q.shape[1]):
            kv = h // group
            s = torch.tensor(k[b, kv, :n] @ q[b, h], dtype=torch.float64) * scale
            w = torch.softmax(s, dim=0)
            w = torch.where(w >= thr, w, torch.zeros_like(w))
            out[b, h] = (w @ torch.tensor(v[b, kv, :n], dtype=torch.float64)).numpy()
    return out


def _slips(q, k, v, lens, scale, thr):
    """The two plausible wrong gates, for checking that a case discriminates."""
    group = q.shape[1] // k.shape[1]
    unnorm = np.zeros(q.shape)
    renorm = np.zeros(q.shape)
    for b in range(q.shape[0]):
        n = int(lens[b])
        for h in range(q.shape[1]):
            kv = h // group
            s = scale * (k[b, kv, :n] @ q[b, h])
            e = np.exp(s - s.max())
            w = e / e.sum()
            keep_u = e >= thr
            unnorm[b, h] = (w * keep_u) @ v[b, kv, :n]
            keep = w >= thr
            renorm[b, h] = (w * keep / max((w * keep).sum(), 1e-300)) @ v[b, kv, :n]
    return unnorm, renorm


def _gate_case(rng, bsz=2, hkv=2, group=3, n=160, d=128):
    q = rng.standard_normal((bsz, hkv * group, d)) * 1.5
    k = rng.standard_normal((bsz, hkv, n, d))
    v = rng.standard_normal((bsz, hkv, n, d))
    return q, k, v


def test_sparse_gate_dense_attention_matches_masked_torch_softmax():
    rng = np.random.default_rng(31)
    q, k, v = _gate_case(rng)
    lens = [160, 97]
    scale = 1 / math.sqrt(128)
    for thr in (0.5 / 160, 1.0 / 160, 3e-3):
        ref = _torch_gated(q, k, v, lens, scale, thr)
        np.testing.assert_allclose(O.attention(q, k, v, lens, scale, thr), ref, rtol=0, atol=1e-12)
        # the case discriminates: both slips move the output by far more
        unnorm, renorm = _slips(q, k, v, lens, scale, thr)
        assert np.max(np.abs(unnorm - ref)) > 1e-2 and np.max(np.abs(renorm - ref)) > 1e-2


def test_sparse_gate_of_both_cache_formulations_matches_masked_torch_softmax():
    rng = np.random.default_rng(32)
    s, (ck, cv), _, (kc, kn, vc, vn) = _random_cache(rng, 2, 2, 120, 256, 3, 2)
    kt = O.dequantize(kc, kn, 3, ck, s)
    vt = O.dequantize(vc, vn, 2, cv, s)
    q = rng.standard_normal((2, 6, 256)) * 1.5
    lens = [120, 45]
    scale = 1 / 16
    # thresholds at the median and the upper quartile of the weights drop a
    # large share of the mass
    w_all = np.concatenate([w for w in O.attention_weights(q, kt, lens, scale).values()])
    for thr in (np.quantile(w_all, 0.5), np.quantile(w_all, 0.75), 1.0 / 120):
        ref = _torch_gated(q, kt, vt, lens, scale, thr)
        a = O.decode_dequant(q, kc, kn, vc, vn, lens, scale, 3, 2, ck, cv, s, thr)
        b = O.decode_rotated(q, kc, kn, vc, vn, lens, scale, 3, 2, ck, cv, s, thr)
        tol = 1e-10 * np.max(np.abs(ref))
        assert np.max(np.abs(a - ref)) <= tol and np.max(np.abs(b - ref)) <= tol
        unnorm, renorm = _slips(q, kt, vt, lens, scale, thr)
        assert np.max(np.abs(unnorm - ref)) > 1e-2 * np.max(np.abs(ref))
        assert np.max(np.abs(renorm - ref)) > 1e-2 * np.max(np.abs(ref))


def test_sparse_gate_of_multi_token_attention_matches_masked_torch_softmax():
    """Query token j sees positions t <= n - n_q + j; its gate uses the
    softmax over exactly those positions."""
    rng = np.random.default_rng(33)
    n_q = 3
    q = rng.standard_normal((2, n_q, 4, 128)) * 1.5
    k = rng.standard_normal((2, 2, 90, 128))
    v = rng.standard_normal((2, 2, 90, 128))
    lens = np.array([90, 40])
    scale = 1 / math.sqrt(128)
    for thr in (0.5 / 90, 1.0 / 60):
        got = O.attention_multi(q, k, v, lens, scale, thr)
        for j in range(n_q):
            lim = lens - n_q + j + 1
            ref = _torch_gated(q[:, j], k, v, lens, scale, thr, limits=lim)
            np.testing.assert_allclose(got[:, j], ref, rtol=0, atol=1e-12)
            unnorm, renorm = _slips(q[:, j], k, v, lim, scale, thr)
            assert np.max(np.abs(unnorm - ref)) > 1e-2 and np.max(np.abs(renorm - ref)) > 1e-2


def test_sparse_gate_keeps_weights_at_the_threshold_and_drops_below():
    """Hand-built scores: n/2 positions at score 1 and n/2 at 0, so the
    normalised weights are e/Z and 1/Z with Z = n/2 (e + 1).  A threshold
    between them keeps only the first half, unrescaled: o = (e/Z) sum of
    their V rows.  A threshold above both drops everything (an unnormalised
    gate would keep every position there)."""
    n, d = 40, 128
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k = np.zeros((1, 1, n, d))
    k[0, 0, : n // 2, 0] = 1.0
    rng = np.random.default_rng(34)
    v = rng.standard_normal((1, 1, n, d))
    z = n / 2 * (math.e + 1)
    hi, lo = math.e / z, 1 / z
    kept = O.attention(q, k, v, [n], 1.0, sparse_thr=(hi + lo) / 2)
    np.testing.assert_allclose(kept[0, 0], hi * v[0, 0, : n // 2].sum(axis=0), rtol=1e-12, atol=1e-13)
    at = O.attention(q, k, v, [n], 1.0, sparse_thr=lo)      # w == thr is kept
    np.testing.assert_allclose(at, O.attention(q, k, v, [n], 1.0), rtol=1e-12, atol=1e-13)
    assert np.all(O.attention(q, k, v, [n], 1.0, sparse_thr=2 * hi) == 0.0)


# ------------------------------------------------- V v3: outlier channels ---

def _outlier_rows(rng, n, d=128, planted=(5, 40, 77), gain=20.0):
    x = rng.standard_normal((n, d))
    x[:, list(planted)] *= gain
    return x


def test_v3_calibration_finds_planted_channels():
    rng = np.random.default_rng(40)
    x = _outlier_rows(rng, 500)
    assert list(O.outlier_channels(x, 3)) == [5, 40, 77]
    # ties go to the lower channel: all-equal mean squares pick 0..k-1
    assert list(O.outlier_channels(np.ones((4, 128)), 2)) == [0, 1]


def test_v3_with_no_channel_is_v1():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((6, 256))
    s = O.sign_vector(3)
    c, t = O.codebook_f32(3)
    codes, norms, vals, _ = O.encode_v3(x, s, 3, t, np.array([], dtype=np.int64))
    c1, n1, _ = O.encode(x, s, 3, t)
    assert np.array_equal(codes, c1) and np.array_equal(norms.view(np.uint16), n1.view(np.uint16))
    assert vals.shape == (6, 0)
    np.testing.assert_array_equal(O.dequantize_v3(codes, norms, 3, c, s, vals, []),
                                  O.dequantize(c1, n1, 3, c, s))


def test_v3_with_every_channel_is_exact_and_kept_channels_are_fp16():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((5, 128)) * 3
    s = O.sign_vector(0)
    c, t = O.codebook_f32(2)
    allc = np.arange(128)
    codes, norms, vals, _ = O.encode_v3(x, s, 2, t, allc)
    assert np.all(norms == 0)  # nothing is left to quantise
    got = O.dequantize_v3(codes, norms, 2, c, s, vals, allc)
    np.testing.assert_array_equal(got, x.astype(np.float16).astype(np.float64))
    ch = np.array([3, 64, 100])
    codes, norms, vals, _ = O.encode_v3(x, s, 2, t, ch)
    got = O.dequantize_v3(codes, norms, 2, c, s, vals, ch)
    np.testing.assert_array_equal(got[:, ch], x[:, ch].astype(np.float16).astype(np.float64))
    # the stored norm is the remainder's
    rest = x.copy()
    rest[:, ch] = 0
    np.testing.assert_array_equal(norms, np.sqrt(np.sum(rest ** 2, axis=1)).astype(np.float16)[:, None])


def test_v3_recovers_the_snr_lost_to_outlier_channels():
    """On vectors with three channels scaled x20, keeping them restores the
    reconstruction SNR of plain Gaussian vectors (the remainder is Gaussian
    again), while v1 loses most of it to the inflated block norm."""
    rng = np.random.default_rng(43)
    x = _outlier_rows(rng, 400)
    s = O.sign_vector(0)
    c, t = O.codebook_f32(3)
    snr = lambda a, b: 10 * np.log10(np.sum(b ** 2) / np.sum((a - b) ** 2))
    ch = O.outlier_channels(x, 3)
    codes, norms, vals, _ = O.encode_v3(x, s, 3, t, ch)
    v3 = O.dequantize_v3(codes, norms, 3, c, s, vals, ch)
    c1, n1, _ = O.encode(x, s, 3, t)
    v1 = O.dequantize(c1, n1, 3, c, s)
    rest = x.copy()
    rest[:, ch] = 0
    assert snr(v3, x) > snr(v1, x) + 10
    # the v3 error is v1's error on the remainder outside the kept channels,
    # and the fp16 rounding of the kept values on them
    cr, nr, _ = O.encode(rest, s, 3, t)
    er = O.dequantize(cr, nr, 3, c, s) - rest
    er[:, ch] = x[:, ch].astype(np.float16).astype(np.float64) - x[:, ch]
    np.testing.assert_allclose(v3 - x, er, rtol=0, atol=1e-12)


def test_v3_decode_formulations_agree():
    rng = np.random.default_rng(44)
    B, H, S, D = 2, 2, 30, 256
    s = O.sign_vector(0)
    ck, tk = O.codebook_f32(3)
    cv, tv = O.codebook_f32(2)
    k = rng.standard_normal((B, H, S, D))
    v = rng.standard_normal((B, H, S, D))
    v[..., [7, 130, 200]] *= 15
    kc, kn, _ = O.encode(k, s, 3, tk)
    chans = np.stack([O.outlier_channels(v[:, h], 4) for h in range(H)])
    enc = [O.encode_v3(v[:, h], s, 2, tv, chans[h]) for h in range(H)]
    vc = np.stack([e[0] for e in enc], axis=1)
    vn = np.stack([e[1] for e in enc], axis=1)
    vv = np.stack([e[2] for e in enc], axis=1)
    q = rng.standard_normal((B, 6, D))
    lens = [30, 11]
    for thr in (0.0, 0.02):
        a = O.decode_v3_dequant(q, kc, kn, vc, vn, vv, chans, lens, 1 / 16, 3, 2, ck, cv, s, thr)
        b = O.decode_v3_rotated(q, kc, kn, vc, vn, vv, chans, lens, 1 / 16, 3, 2, ck, cv, s, thr)
        assert np.max(np.abs(a - b)) <= 1e-10 * np.max(np.abs(a))
    # the outlier channels of the output are the weighted sums of the kept values
    kt = O.dequantize(kc, kn, 3, ck, s)
    w = O.attention_weights(q, kt, lens, 1 / 16)[(1, 5)]
    got = O.decode_v3_rotated(q, kc, kn, vc, vn, vv, chans, lens, 1 / 16, 3, 2, ck, cv, s)[1, 5, chans[1]]
    np.testing.assert_allclose(got, w @ vv[1, 1, :11].astype(np.float64), rtol=1e-12)


# ------------------------------------------------ V v2: trellis (TCQ) coding ---

def _all_paths(n, bits):
    """Every (beta, j) sequence of length n for a b-bit code."""
    nj = 1 << (bits - 1)
    for code in range((2 * nj) ** n):
        beta, jj = [], []
        for _ in range(n):
            beta.append(code & 1)
            code >>= 1
            jj.append(code % nj)
            code //= nj
        yield np.array(beta), np.array(jj)


@pytest.mark.parametrize("bits,n", [(1, 1), (1, 5), (1, 9), (2, 1), (2, 4), (2, 6), (3, 4)])
def test_v2_viterbi_finds_the_least_error_path_by_brute_force(bits, n):
    """Over every code sequence of a short group, the Viterbi path has the
    least squared error, and the error it reports is its path's."""
    rng = np.random.default_rng(100 + 10 * bits + n)
    lv = O.tcq_levels_f32(bits)
    for trial in range(4):
        u = rng.standard_normal(n) * (1.0 + trial)
        beta, jj, err = O.tcq_viterbi(u, lv)
        path = O.tcq_reconstruct(beta, jj, lv)
        assert math.isclose(err, float(np.sum((u - path) ** 2)), rel_tol=1e-12, abs_tol=1e-15)
        best = min(float(np.sum((u - O.tcq_reconstruct(b, j, lv)) ** 2)) for b, j in _all_paths(n, bits))
        assert math.isclose(err, best, rel_tol=1e-12, abs_tol=1e-15)


def test_v2_trellis_has_memory_two_and_ungerboeck_subsets():
    """The structure TCQ requires of its 4-state trellis: the state is fixed
    by the last two branch bits (a shift register, so every state is reached
    from state 0 in two steps); the two branches leaving a state carry the two
    subsets of one union codebook, D0 u D2 from even states and D1 u D3 from
    odd ones; the two branches entering a state carry the two subsets of one
    union codebook too."""
    def walk(bits_seq):
        s = 0
        for b in bits_seq:
            s = O.TCQ_NEXT[s][b]
        return s
    for n in range(2, 7):
        for code in range(1 << n):
            seq = [(code >> i) & 1 for i in range(n)]
            assert walk(seq) == walk(seq[-2:])
    assert sorted(walk([a, b]) for a in (0, 1) for b in (0, 1)) == [0, 1, 2, 3]
    for s in range(4):
        assert sorted(O.TCQ_SUBSET[s]) == ([0, 2] if s % 2 == 0 else [1, 3])
        entering = sorted(O.TCQ_SUBSET[p][b] for p in range(4) for b in (0, 1) if O.TCQ_NEXT[p][b] == s)
        assert entering in ([0, 2], [1, 3])


def test_v2_doubled_codebook_and_subsets():
    # 2^(b+1) Lloyd-Max levels; subset k holds the levels of index k mod 4
    for bits in (1, 2, 3):
        lv = O.tcq_levels_f32(bits)
        assert len(lv) == 1 << (bits + 1) and np.all(np.diff(lv) > 0)
        np.testing.assert_array_equal(lv, O.codebook_f32(bits + 1)[0])
    # rate 1: one level per subset, so the code is the branch bits alone
    lv = O.tcq_levels_f32(1)
    beta = np.array([1, 1, 0, 1, 0, 0])
    path = O.tcq_reconstruct(beta, np.zeros(6, dtype=np.int64), lv)
    assert set(path) <= set(lv.astype(np.float64))


def test_v2_beats_scalar_lloyd_max_and_stays_above_the_rate_distortion_bound():
    """On i.i.d. N(0,1) coordinates the 4-state trellis lowers the squared
    error of the b-bit Lloyd-Max quantiser (Max 1960 distortions 0.3634,
    0.1175, 0.03455 for b = 1, 2, 3) -- by 0.2 dB at rate 1 and 0.7 dB at
    rates 2 and 3, well inside the granular gain of a 4-state trellis -- and
    cannot go below the Gaussian rate-distortion bound 2^(-2b)."""
    rng = np.random.default_rng(7)
    u = rng.standard_normal((60, 128))
    table = _golden_max()
    for bits in (1, 2, 3):
        lv = O.tcq_levels_f32(bits)
        mse = np.mean([O.tcq_viterbi(r, lv)[2] for r in u]) / 128
        scalar = table[(1 << bits, "distortion")][0]
        gain_db = 0.2 if bits == 1 else 0.7
        assert mse < scalar * 10 ** (-gain_db / 10), (bits, mse, scalar)
        assert mse > 2.0 ** (-2 * bits)


def test_v2_pack_layout_known_patterns():
    # b = 3: 6-bit pair fields j_a | j_b << 2 | beta_a << 4 | beta_b << 5
    beta = np.zeros(128, dtype=np.int64)
    jj = np.zeros(128, dtype=np.int64)
    beta[1] = 1          # field 0 bit 5 -> stream bit 5
    jj[2] = 3            # field 1 bits 0-1 -> stream bits 6, 7
    beta[127] = 1        # field 63 bit 5 -> stream bit 383 (last bit)
    jj[126] = 2          # field 63 bit 1 -> stream bit 379
    p = O.pack_v2(beta, jj, 3)
    assert p.shape == (48,)
    assert p[0] == 0xE0 and p[47] == 0x88 and not np.any(p[1:47])
    b2, j2 = O.unpack_v2(p, 3)
    np.testing.assert_array_equal(b2, beta)
    np.testing.assert_array_equal(j2, jj)
    # b = 2: 4-bit fields j_a | j_b << 1 | beta_a << 2 | beta_b << 3
    p = O.pack_v2(beta, np.minimum(jj, 1), 2)
    assert p.shape == (32,)
    assert p[0] == 0x08 | 0x10 and p[31] == 0x80 | 0x10 and not np.any(p[1:31])
    # b = 1: the branch bits alone, two per field
    p = O.pack_v2(beta, jj * 0, 1)
    assert p.shape == (16,) and p[0] == 0x02 and p[15] == 0x80
    # round trip on random paths
    rng = np.random.default_rng(3)
    for bits in (1, 2, 3, 4):
        bb = rng.integers(0, 2, size=(5, 128))
        j = rng.integers(0, 1 << (bits - 1), size=(5, 128))
        b2, j2 = O.unpack_v2(O.pack_v2(bb, j, bits), bits)
        np.testing.assert_array_equal(b2, bb)
        np.testing.assert_array_equal(j2, j)


def test_v2_encode_is_v1_norm_and_rotation_and_zero_block():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((3, 256)) * 2
    x[1, :128] = 0.0
    s = O.sign_vector(5)
    lv = O.tcq_levels_f32(2)
    codes, norms, u, err = O.encode_v2(x, s, 2, lv)
    _, n1, u1 = O.encode(x, s, 2, O.codebook_f32(2)[1])
    np.testing.assert_array_equal(norms.view(np.uint16), n1.view(np.uint16))
    np.testing.assert_array_equal(u, u1)
    xt = O.dequantize_v2(codes, norms, 2, lv, s)
    assert np.all(xt[1, :128] == 0.0)
    # the reported error is the rotated-domain error of the reconstruction
    lvl = O.v2_levels(codes, 2, lv)
    np.testing.assert_allclose(err, np.sum((u - lvl) ** 2, axis=-1), rtol=1e-12)
    # and maps to the input domain through the orthogonal rotation and the norm
    nhat = norms.astype(np.float64)
    rel = np.sum((xt - x).reshape(3, 2, 128) ** 2, axis=-1)
    exp = np.sum((lvl * nhat[..., None] - u * np.sqrt(np.sum(x.reshape(3, 2, 128) ** 2, -1))[..., None]) ** 2,
                 axis=-1) / 128
    np.testing.assert_allclose(rel, exp, rtol=1e-9, atol=1e-12)


def test_v2_decode_formulations_agree():
    rng = np.random.default_rng(9)
    B, H, S, D = 2, 2, 20, 256
    s = O.sign_vector(0)
    ck, tk = O.codebook_f32(3)
    lv = O.tcq_levels_f32(2)
    k = rng.standard_normal((B, H, S, D))
    v = rng.standard_t(4.0, size=(B, H, S, D))
    kc, kn, _ = O.encode(k, s, 3, tk)
    vc, vn, _, _ = O.encode_v2(v, s, 2, lv)
    q = rng.standard_normal((B, 4, D))
    for thr in (0.0, 0.03):
        a = O.decode_v2_dequant(q, kc, kn, vc, vn, [20, 7], 1 / 16, 3, 2, ck, lv, s, thr)
        b = O.decode_v2_rotated(q, kc, kn, vc, vn, [20, 7], 1 / 16, 3, 2, ck, lv, s, thr)
        assert np.max(np.abs(a - b)) <= 1e-10 * np.max(np.abs(a))
