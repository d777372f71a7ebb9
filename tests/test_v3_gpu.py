"""V v3 (outlier-channel separation) through the C ABI, against the oracle.

Calibration: the channels tq_pick_outlier_channels picks equal the oracle's
top-k mean-square channels.  Encoding: the stored values are the fp16 of the
outlier channels (bit-exact, zero padding), the remainder's codes and norms
follow the encoder's acceptance rules against the oracle's v3 encoding, and
the K side is that of the plain encoder.  Decode: the output against the fp64
oracle (rotated-domain decode of the remainders, outlier channels replaced by
sum_t w_t val_t) on the GPU's own cache, the outlier channels and the other
channels each within the decode tolerance of their own scale; k = 0 is the
plain decode bit for bit; and v3 beats the plain format on outlier-channel V.
"""
import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import inputs
from oracle import tq_oracle as O

from ._parity import (DECODE_REL_TOL, SNR_BAND_DB, SPARSE_BAND, check_codes, check_norms, host, snr_db,
                      to_dev, torch_mod)

pytestmark = pytest.mark.gpu


def _desc(w, seq_cap=None):
    return tq.kv_desc(w.batch, w.kv_heads, w.head_dim, seq_cap or w.seq_cap, w.k_bits, w.v_bits, w.sign_seed)


def _oracle_channels(v, k):
    """Oracle calibration per kv-head over every batch entry and row."""
    return np.stack([O.outlier_channels(v[:, h], k) for h in range(v.shape[1])])


def _encode_v3(w, k, channels=None, status=None):
    torch = torch_mod()
    desc = _desc(w)
    kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
    vd = to_dev(w.v)
    ch = tq.pick_outlier_channels(desc, vd, k) if channels is None else to_dev(np.asarray(channels, np.int32))
    vo = tq.alloc_outliers(desc, ch)
    cache = tq.alloc_cache(desc)
    tq.encode_kv_v3(cache, kcb, vcb, vo, to_dev(w.k), vd, status=status)
    torch.cuda.synchronize()
    return cache, kcb, vcb, vo


def _decode_v3(cache, kcb, vcb, vo, q, lens, scale, sparse_thr=0.0, status=None):
    torch = torch_mod()
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, q.shape[1], sparse_thr)
    tq.decode_attention_v3(cache, kcb, vcb, vo, to_dev(q), to_dev(np.asarray(lens, np.int32)), scale, out, ws,
                           sparse_thr=sparse_thr, status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _oracle_v3(w, cache, vo, lens, sparse_thr):
    kc, kn, vc, vn = host(cache)
    vals = vo.values.cpu().numpy().view(np.float16)[..., : vo.k]
    ch = vo.channels.cpu().numpy()
    kcent, _ = O.codebook_f32(w.k_bits)
    vcent, _ = O.codebook_f32(w.v_bits)
    return O.decode_v3_rotated(w.q.astype(np.float64), kc, kn, vc, vn, vals, ch, lens, w.scale, w.k_bits,
                               w.v_bits, kcent, vcent, O.sign_vector(w.sign_seed), sparse_thr)


def _v3_flip_bound(w, cache, vo, lens, thr):
    """The sparse gate's ambiguity bound (see the plain decode's parity tests)
    with the v3 reconstruction of V: a position within SPARSE_BAND of the
    threshold may be kept or dropped; flipping it moves output d of head h by
    at most w_t |v~_t[d]|."""
    kc, kn, vc, vn = host(cache)
    s = O.sign_vector(w.sign_seed)
    kt = O.dequantize(kc, kn, w.k_bits, O.codebook_f32(w.k_bits)[0], s)
    vals = vo.values.cpu().numpy().view(np.float16)[..., : vo.k]
    ch = vo.channels.cpu().numpy()
    vt = np.stack([O.dequantize_v3(vc[:, h], vn[:, h], w.v_bits, O.codebook_f32(w.v_bits)[0], s, vals[:, h], ch[h])
                   for h in range(w.kv_heads)], axis=1)
    ws = O.attention_weights(w.q, kt, lens, w.scale)
    group = w.q_heads // w.kv_heads
    bound = np.zeros(w.q.shape, dtype=np.float64)
    for (b, h), wt in ws.items():
        n = int(lens[b])
        if n == 0:
            continue
        amb = np.abs(np.log(np.maximum(wt, 1e-300) / thr)) < SPARSE_BAND
        bound[b, h] = wt[amb] @ np.abs(vt[b, h // group, :n][amb])
    return bound


def _check_v3_decode(o_gpu, o_ref, ch, group, bound=None):
    """Outlier channels and the other channels, each within DECODE_REL_TOL of
    its own max |o_ref| (plus the sparse bound where given)."""
    B, Hq, D = o_ref.shape
    is_out = np.zeros((Hq, D), dtype=bool)
    for h in range(Hq):
        is_out[h, ch[h // group]] = True
    is_out = np.broadcast_to(is_out, o_ref.shape)
    bnd = np.zeros_like(o_ref) if bound is None else bound
    errs = []
    for sel in (is_out, ~is_out):
        ref, got = o_ref[sel], o_gpu[sel]
        sc = max(np.max(np.abs(ref)), 1e-300)
        excess = np.abs(got - ref) - (DECODE_REL_TOL * sc + bnd[sel])
        assert np.all(excess <= 0), f"decode error {np.max(np.abs(got - ref)) / sc:.3e} beyond bound"
        errs.append(float(np.max(np.maximum(np.abs(got - ref) - bnd[sel], 0)) / sc))
    return errs


# ---- calibration -----------------------------------------------------------

@pytest.mark.parametrize("name,k", [("gqa", 4), ("gqa", 16), ("ragged", 8), ("ragged", 13)])
def test_pick_outlier_channels_matches_oracle(name, k):
    w = inputs.make(name, batch=2, seq=300, dist="outlier_v", with_q=False)
    ch = tq.pick_outlier_channels(_desc(w), to_dev(w.v), k).cpu().numpy()
    assert np.array_equal(ch, _oracle_channels(w.v, k))


def test_pick_outlier_channels_ties_go_to_lower_index():
    torch = torch_mod()
    v = np.ones((1, 2, 5, 128), dtype=np.float16)
    v[0, 1, :, 77] = 2.0   # head 1: channel 77 first, then the lowest of the tied rest
    desc = tq.kv_desc(1, 2, 128, 5, 3, 3)
    ch = tq.pick_outlier_channels(desc, to_dev(v), 4).cpu().numpy()
    torch.cuda.synchronize()
    assert ch.tolist() == [[0, 1, 2, 3], [0, 1, 2, 77]]
    assert np.array_equal(ch, _oracle_channels(v, 4))


# ---- encoding --------------------------------------------------------------

@pytest.mark.parametrize("name,k", [("gqa", 6), ("gqa", 16), ("ragged", 9)])
def test_encode_v3_matches_oracle(name, k):
    w = inputs.make(name, batch=2, seq=160, dist="outlier_v", with_q=False)
    cache, kcb, vcb, vo = _encode_v3(w, k)
    ch = vo.channels.cpu().numpy()
    assert np.array_equal(ch, _oracle_channels(w.v, k))
    kc, kn, vc, vn = host(cache)
    vals = vo.values.cpu().numpy()
    kp = tq.outlier_row(k)
    assert vals.shape == (w.batch, w.kv_heads, w.seq_cap, kp)
    signs = O.sign_vector(w.sign_seed)
    _, t32 = O.codebook_f32(w.v_bits)
    for h in range(w.kv_heads):
        x = w.v[:, h].astype(np.float64)
        _, _, want_vals, _ = O.encode_v3(x, signs, w.v_bits, t32, ch[h])
        # exact fp16 values, zero padding
        assert np.array_equal(vals[:, h, :, :k], want_vals.view(np.int16))
        assert not np.any(vals[:, h, :, k:])
        rest = x.copy()
        rest[..., ch[h]] = 0.0
        check_norms(vn[:, h], rest)
        check_codes(vc[:, h], rest, w.v_bits, signs)
    # the K side is the plain encoder's
    ref = tq.alloc_cache(cache.desc)
    tq.encode_kv(ref, kcb, vcb, to_dev(w.k), to_dev(w.v))
    rk, rkn, _, _ = host(ref)
    assert np.array_equal(kc, rk) and np.array_equal(kn, rkn)


def test_encode_v3_append_at_positions():
    """Rows appended at per-sequence start positions land in the values rows
    of those positions, and only there."""
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=64, dist="outlier_v", with_q=False)
    desc = _desc(w)
    kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
    ch = tq.pick_outlier_channels(desc, to_dev(w.v), 5)
    vo = tq.alloc_outliers(desc, ch)
    cache = tq.alloc_cache(desc)
    start = np.array([10, 40], dtype=np.int32)
    tq.encode_kv_v3(cache, kcb, vcb, vo, to_dev(w.k[:, :, :3]), to_dev(w.v[:, :, :3]), start_pos=to_dev(start))
    torch.cuda.synchronize()
    vals = vo.values.cpu().numpy().view(np.float16)
    chh = ch.cpu().numpy()
    for b in range(2):
        for h in range(w.kv_heads):
            got = vals[b, h, start[b]:start[b] + 3, :5]
            assert np.array_equal(got, w.v[b, h, :3][:, chh[h]])
        keep = np.ones(64, dtype=bool)
        keep[start[b]:start[b] + 3] = False
        assert not np.any(vals[b][:, keep])


# ---- decode ----------------------------------------------------------------

CASES = [
    # name, batch, seq, lens, k, sparse   (GQ 4 / 8 column layouts, NB 1 / 2,
    # whole units and units split across CTAs, ragged tails, kp 8 / 16)
    ("gqa", 3, 300, [300, 171, 17], 4, 0.0),
    ("gqa", 1, 4096, [4096], 12, 0.0),
    ("gqa", 2, 1000, [1000, 333], 16, 1e-4),
    ("ragged", 2, 700, [700, 129], 8, 0.0),
    ("ragged", 1, 3000, [2999], 10, 1e-5),
]


@pytest.mark.parametrize("name,batch,seq,lens,k,thr", CASES)
def test_decode_v3_matches_oracle(name, batch, seq, lens, k, thr):
    w = inputs.make(name, batch=batch, seq=seq, dist="outlier_v")
    cache, kcb, vcb, vo = _encode_v3(w, k)
    o_gpu = _decode_v3(cache, kcb, vcb, vo, w.q, lens, w.scale, thr)
    o_ref = _oracle_v3(w, cache, vo, lens, thr)
    bound = _v3_flip_bound(w, cache, vo, lens, thr) if thr > 0 else None
    _check_v3_decode(o_gpu, o_ref, vo.channels.cpu().numpy(), w.q_heads // w.kv_heads, bound)
    exact = O.attention(w.q, w.k, w.v, lens, w.scale, thr)
    assert abs(snr_db(o_gpu, exact) - snr_db(o_ref, exact)) <= SNR_BAND_DB


def test_decode_v3_group_of_eight():
    # Hq 16 / Hkv 2: eight heads per unit (one score column per head)
    w = inputs.make("gqa", batch=2, seq=500, dist="outlier_v")
    rng = np.random.default_rng(3)
    w.q_heads, w.kv_heads = 16, 2
    w.k, w.v = w.k[:, :2], w.v[:, :2]
    w.q = rng.standard_normal((2, 16, 128)).astype(np.float16)
    lens = [500, 77]
    cache, kcb, vcb, vo = _encode_v3(w, 7)
    o_gpu = _decode_v3(cache, kcb, vcb, vo, w.q, lens, w.scale)
    o_ref = _oracle_v3(w, cache, vo, lens, 0.0)
    _check_v3_decode(o_gpu, o_ref, vo.channels.cpu().numpy(), 8)


def test_decode_v3_with_k0_is_the_plain_decode():
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=256)
    desc = _desc(w)
    kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
    cache = tq.alloc_cache(desc)
    tq.encode_kv(cache, kcb, vcb, to_dev(w.k), to_dev(w.v))
    vo = tq.VOutliers(0, torch.zeros((w.kv_heads, 1), dtype=torch.int32, device="cuda"),
                      torch.zeros((1, 8), dtype=torch.int16, device="cuda"))
    lens = np.array([256, 99], dtype=np.int32)
    a = _decode_v3(cache, kcb, vcb, vo, w.q, lens, w.scale)
    out = torch.empty(w.q.shape, dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(desc, w.q_heads)
    tq.decode_attention(cache, kcb, vcb, to_dev(w.q), to_dev(lens), w.scale, out, ws)
    torch.cuda.synchronize()
    assert np.array_equal(a, out.cpu().numpy().astype(np.float64))


def test_v3_improves_snr_on_outlier_channels():
    """On V with outlier channels, the v3 output is closer to unquantised
    attention than the plain format's, and more so with more channels kept
    (up to the number of outlier channels)."""
    w = inputs.make("gqa", batch=2, seq=512, dist="outlier_v")
    lens = [512, 300]
    exact = O.attention(w.q, w.k, w.v, lens, w.scale)
    snrs = []
    for k in (0, 3, 6):
        if k == 0:  # the plain format, through the same entry point
            torch = torch_mod()
            desc = _desc(w)
            kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
            cache = tq.alloc_cache(desc)
            tq.encode_kv(cache, kcb, vcb, to_dev(w.k), to_dev(w.v))
            vo = tq.VOutliers(0, torch.zeros((w.kv_heads, 1), dtype=torch.int32, device="cuda"),
                              torch.zeros((1, 8), dtype=torch.int16, device="cuda"))
        else:
            cache, kcb, vcb, vo = _encode_v3(w, k)
        snrs.append(snr_db(_decode_v3(cache, kcb, vcb, vo, w.q, lens, w.scale), exact))
    assert snrs[0] < snrs[1] < snrs[2], snrs


def test_v3_channel_out_of_range_sets_status():
    torch = torch_mod()
    w = inputs.make("gqa", batch=1, seq=64, dist="outlier_v")
    ch = np.tile(np.array([3, 50, 130, -1], dtype=np.int32), (w.kv_heads, 1))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache, kcb, vcb, vo = _encode_v3(w, 4, channels=ch, status=status)
    assert status.item() == tq.TQ_DEV_CHANNEL_RANGE
    vals = vo.values.cpu().numpy().view(np.float16)
    assert not np.any(vals[..., 2:4].astype(np.float64))          # ignored entries stored as 0
    status.zero_()
    o_gpu = _decode_v3(cache, kcb, vcb, vo, w.q, [64], w.scale, status=status)
    assert status.item() == tq.TQ_DEV_CHANNEL_RANGE
    # the two valid channels follow the oracle; the others are the remainder's
    valid = np.tile(np.array([3, 50]), (w.kv_heads, 1))
    vo2 = tq.VOutliers(2, to_dev(valid.astype(np.int32)), vo.values[..., :8].contiguous())
    o_ref = _oracle_v3(w, cache, vo2, [64], 0.0)
    _check_v3_decode(o_gpu, o_ref, valid, w.q_heads // w.kv_heads)


def test_decode_v3_edge_lengths():
    # an empty sequence (zero row), a single position, and a full cache
    w = inputs.make("gqa", batch=3, seq=96, dist="outlier_v")
    lens = [0, 1, 96]
    cache, kcb, vcb, vo = _encode_v3(w, 5)
    o_gpu = _decode_v3(cache, kcb, vcb, vo, w.q, lens, w.scale)
    assert np.all(o_gpu[0] == 0.0)
    o_ref = _oracle_v3(w, cache, vo, lens, 0.0)
    _check_v3_decode(o_gpu[1:], o_ref[1:], vo.channels.cpu().numpy(), w.q_heads // w.kv_heads)


def test_decode_v3_full_gqa_sampled():
    """The full GQA workload (B8, S32768) with outlier-channel V, k = 8, in the
    benchmark's launch shape; sampled (batch, kv-head) units against the oracle."""
    w = inputs.make("gqa", dist="outlier_v")
    cache, kcb, vcb, vo = _encode_v3(w, 8)
    o_gpu = _decode_v3(cache, kcb, vcb, vo, w.q, w.seq_lens, w.scale)
    kc, kn, vc, vn = host(cache)
    vals = vo.values.cpu().numpy().view(np.float16)[..., : vo.k]
    ch = vo.channels.cpu().numpy()
    g = w.q_heads // w.kv_heads
    kcent, _ = O.codebook_f32(w.k_bits)
    vcent, _ = O.codebook_f32(w.v_bits)
    for b, h in [(0, 0), (5, 3), (7, 7)]:
        sl = slice(h, h + 1)
        qs = w.q[b:b + 1, h * g:(h + 1) * g].astype(np.float64)
        o_ref = O.decode_v3_rotated(qs, kc[b:b + 1, sl], kn[b:b + 1, sl], vc[b:b + 1, sl], vn[b:b + 1, sl],
                                    vals[b:b + 1, sl], ch[sl], w.seq_lens[b:b + 1], w.scale, w.k_bits, w.v_bits,
                                    kcent, vcent, O.sign_vector(w.sign_seed))
        _check_v3_decode(o_gpu[b:b + 1, h * g:(h + 1) * g], o_ref, ch[sl], g)
