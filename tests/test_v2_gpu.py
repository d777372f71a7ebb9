"""V v2 (trellis-coded V) through the C ABI, against the oracle.

Encoding: fp16 block norms by the encoder's midpoint rule; the Viterbi path
the GPU picks is optimal up to fp32 rounding -- its squared error, measured
by the oracle in fp64 on the oracle's own u, is within a relative 1e-5 of the
oracle's optimum in every block -- and equals the oracle's path in almost
every block (paths may differ only where two paths' errors tie to rounding).
The K side is the plain encoder's.  Decode: the output against the fp64
oracle's rotated-domain v2 decode on the GPU's own cache (element-wise at the
decode tolerance, SNR band against unquantised attention), across group
sizes, head dims, ragged lengths, CTA splits and sparse-V; and v2 beats the
plain format at the same rate.
"""
import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import inputs
from oracle import tq_oracle as O

from ._parity import (SNR_BAND_DB, SPARSE_BAND, check_decode, check_norms, host, snr_db, to_dev, torch_mod)

pytestmark = pytest.mark.gpu

PATH_REL_TOL = 1e-5        # GPU path error vs the optimum, per block
SAME_PATH_MIN = 0.98       # fraction of blocks whose path equals the oracle's


def _encode_v2(w, status=None, start_pos=None, k=None, v=None):
    torch = torch_mod()
    desc = tq.kv_desc(w.batch, w.kv_heads, w.head_dim, w.seq_cap, w.k_bits, w.v_bits, w.sign_seed)
    kcb, vtq = tq.make_codebook(w.k_bits), tq.make_tcq_codebook(w.v_bits)
    cache = tq.alloc_cache(desc)
    sp = None if start_pos is None else to_dev(np.asarray(start_pos, dtype=np.int32))
    tq.encode_kv_v2(cache, kcb, vtq, to_dev(w.k if k is None else k), to_dev(w.v if v is None else v),
                    start_pos=sp, status=status)
    torch.cuda.synchronize()
    return cache, kcb, vtq


def _decode_v2(cache, kcb, vtq, q, lens, scale, sparse_thr=0.0):
    torch = torch_mod()
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, q.shape[1], sparse_thr)
    tq.decode_attention_v2(cache, kcb, vtq, to_dev(q), to_dev(np.asarray(lens, np.int32)), scale, out, ws,
                           sparse_thr=sparse_thr)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _oracle_v2(w, cache, lens, thr):
    kc, kn, vc, vn = host(cache)
    return O.decode_v2_rotated(w.q.astype(np.float64), kc, kn, vc, vn, lens, w.scale, w.k_bits, w.v_bits,
                               O.codebook_f32(w.k_bits)[0], O.tcq_levels_f32(w.v_bits),
                               O.sign_vector(w.sign_seed), thr)


def _v2_flip_bound(w, cache, lens, thr):
    """The sparse gate's ambiguity bound with the v2 reconstruction of V."""
    kc, kn, vc, vn = host(cache)
    s = O.sign_vector(w.sign_seed)
    kt = O.dequantize(kc, kn, w.k_bits, O.codebook_f32(w.k_bits)[0], s)
    vt = O.dequantize_v2(vc, vn, w.v_bits, O.tcq_levels_f32(w.v_bits), s)
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


def _check_v2_codes(w, cache):
    """Norms by the midpoint rule; per block, the GPU path's error within
    PATH_REL_TOL of the optimum; most paths identical to the oracle's."""
    _, _, vc, vn = host(cache)
    lv = O.tcq_levels_f32(w.v_bits)
    s = O.sign_vector(w.sign_seed)
    x = w.v.astype(np.float64)
    codes, _, u, err = O.encode_v2(x, s, w.v_bits, lv)
    check_norms(vn, x)
    got = np.sum((u - O.v2_levels(vc, w.v_bits, lv)) ** 2, axis=-1)
    assert np.all(got <= err * (1 + PATH_REL_TOL) + 1e-9), float(np.max(got / np.maximum(err, 1e-300)))
    same = np.all(vc == codes, axis=-1)
    assert np.mean(same) >= SAME_PATH_MIN, float(np.mean(same))
    return float(np.mean(same))


# ---- encoding --------------------------------------------------------------

@pytest.mark.parametrize("name,dist", [("gqa", "normal"), ("encode", "outlier_t4"), ("ragged", "normal")])
def test_encode_v2_matches_oracle(name, dist):
    w = inputs.make(name, batch=2, seq=96, dist=dist, with_q=False)
    if name == "gqa":
        w.v_bits = 3
    w.k_bits = 3
    cache, kcb, vtq = _encode_v2(w)
    _check_v2_codes(w, cache)
    # the K side is the plain encoder's
    ref = tq.alloc_cache(cache.desc)
    tq.encode_kv(ref, kcb, tq.make_codebook(w.v_bits), to_dev(w.k), to_dev(w.v))
    torch_mod().cuda.synchronize()
    rk, rkn, _, _ = host(ref)
    kc, kn, _, _ = host(cache)
    assert np.array_equal(kc, rk) and np.array_equal(kn, rkn)


def test_encode_v2_fp32_input_and_zero_rows():
    w = inputs.make("toy", batch=1, seq=64, with_q=False)   # fp32 rows
    w.v_bits = 2
    w.v = w.v.copy()
    w.v[0, 0, 5] = 0.0                                         # a zero block
    cache, _, _ = _encode_v2(w)
    _check_v2_codes(w, cache)
    _, _, _, vn = host(cache)
    assert vn[0, 0, 5, 0] == 0


def test_encode_v2_append_at_positions_and_range():
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=64, with_q=False)
    desc = tq.kv_desc(2, w.kv_heads, 128, 64, w.k_bits, w.v_bits, w.sign_seed)
    kcb, vtq = tq.make_codebook(w.k_bits), tq.make_tcq_codebook(w.v_bits)
    cache = tq.alloc_cache(desc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    start = to_dev(np.array([10, 62], dtype=np.int32))   # sequence 1: rows 62, 63 land, row 64 is out
    tq.encode_kv_v2(cache, kcb, vtq, to_dev(w.k[:, :, :3]), to_dev(w.v[:, :, :3]), start_pos=start,
                    status=status)
    torch.cuda.synchronize()
    assert status.item() == tq.TQ_DEV_POS_RANGE
    _, _, vc, vn = host(cache)
    ref = tq.alloc_cache(desc)
    tq.encode_kv_v2(ref, kcb, vtq, to_dev(w.k), to_dev(w.v))
    torch.cuda.synchronize()
    _, _, rc, rn = host(ref)
    np.testing.assert_array_equal(vc[0, :, 10:13], rc[0, :, 0:3])
    np.testing.assert_array_equal(vc[1, :, 62:64], rc[1, :, 0:2])
    keep = np.ones(64, dtype=bool)
    keep[10:13] = False
    assert not np.any(vc[0][:, keep]) and not np.any(vn[0][:, keep])


# ---- decode ----------------------------------------------------------------

CASES = [
    # name, batch, seq, lens, v_bits, sparse  (G 4 and 8 column layouts,
    # D 128 / 256, whole units and units split across CTAs, ragged tails)
    ("gqa", 3, 300, [300, 171, 17], 3, 0.0),
    ("gqa", 1, 4096, [4096], 2, 0.0),
    ("gqa", 2, 1000, [1000, 333], 3, 1e-4),
    ("ragged", 2, 700, [700, 129], 2, 0.0),
    ("ragged", 1, 3000, [2999], 3, 1e-5),
]


@pytest.mark.parametrize("name,batch,seq,lens,vb,thr", CASES)
def test_decode_v2_matches_oracle(name, batch, seq, lens, vb, thr):
    w = inputs.make(name, batch=batch, seq=seq)
    w.v_bits = vb
    cache, kcb, vtq = _encode_v2(w)
    o_gpu = _decode_v2(cache, kcb, vtq, w.q, lens, w.scale, thr)
    o_ref = _oracle_v2(w, cache, lens, thr)
    check_decode(o_gpu, o_ref, _v2_flip_bound(w, cache, lens, thr) if thr > 0 else None)
    exact = O.attention(w.q, w.k, w.v, lens, w.scale, thr)
    assert abs(snr_db(o_gpu, exact) - snr_db(o_ref, exact)) <= SNR_BAND_DB


def test_decode_v2_group_of_eight():
    w = inputs.make("gqa", batch=2, seq=500)
    rng = np.random.default_rng(5)
    w.q_heads, w.kv_heads = 16, 2
    w.k, w.v = w.k[:, :2], w.v[:, :2]
    w.q = rng.standard_normal((2, 16, 128)).astype(np.float16)
    lens = [500, 77]
    cache, kcb, vtq = _encode_v2(w)
    check_decode(_decode_v2(cache, kcb, vtq, w.q, lens, w.scale), _oracle_v2(w, cache, lens, 0.0))


@pytest.mark.parametrize("vb", [2, 3])
def test_v2_beats_the_plain_format_at_the_same_rate(vb):
    """At the same rate, the GPU's v2 V reconstruction is at least 0.5 dB
    closer to V than the plain format's (the trellis gain), and the decode
    output is closer to unquantised attention."""
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=512)
    w.v_bits = vb
    lens = [512, 300]
    exact = O.attention(w.q, w.k, w.v, lens, w.scale)
    cache, kcb, vtq = _encode_v2(w)
    s2 = snr_db(_decode_v2(cache, kcb, vtq, w.q, lens, w.scale), exact)
    desc = cache.desc
    c1 = tq.alloc_cache(desc)
    vcb = tq.make_codebook(vb)
    tq.encode_kv(c1, kcb, vcb, to_dev(w.k), to_dev(w.v))
    out = torch.empty(w.q.shape, dtype=torch.float32, device="cuda")
    tq.decode_attention(c1, kcb, vcb, to_dev(w.q), to_dev(np.asarray(lens, np.int32)), w.scale, out,
                        tq.alloc_workspace(desc, w.q_heads))
    torch.cuda.synchronize()
    s1 = snr_db(out.cpu().numpy().astype(np.float64), exact)
    assert s2 > s1, (s1, s2)
    sg = O.sign_vector(w.sign_seed)
    x = w.v.astype(np.float64)
    _, _, vc2, vn2 = host(cache)
    _, _, vc1, vn1 = host(c1)
    r2 = O.dequantize_v2(vc2, vn2, vb, O.tcq_levels_f32(vb), sg)
    r1 = O.dequantize(vc1, vn1, vb, O.codebook_f32(vb)[0], sg)
    assert snr_db(r2, x) > snr_db(r1, x) + 0.5


def test_decode_v2_edge_lengths():
    # an empty sequence (zero row), a single position (the trellis's first
    # step), and a full cache
    w = inputs.make("gqa", batch=3, seq=96)
    lens = [0, 1, 96]
    cache, kcb, vtq = _encode_v2(w)
    o_gpu = _decode_v2(cache, kcb, vtq, w.q, lens, w.scale)
    assert np.all(o_gpu[0] == 0.0)
    check_decode(o_gpu[1:], _oracle_v2(w, cache, lens, 0.0)[1:])


@pytest.mark.parametrize("name,units", [("gqa", [(0, 0), (6, 2)]), ("ragged", [(0, 1), (3, 3)])])
def test_decode_v2_full_sampled(name, units):
    """Full workloads in the benchmark's launch shape (GQA K3/V3; ragged K3/V2
    D256 with sparse-V); sampled (batch, kv-head) units against the oracle."""
    w = inputs.make(name)
    cache, kcb, vtq = _encode_v2(w)
    o_gpu = _decode_v2(cache, kcb, vtq, w.q, w.seq_lens, w.scale, w.sparse_thr)
    kc, kn, vc, vn = host(cache)
    g = w.q_heads // w.kv_heads
    for b, h in units:
        sl = slice(h, h + 1)
        qs = w.q[b:b + 1, h * g:(h + 1) * g].astype(np.float64)
        o_ref = O.decode_v2_rotated(qs, kc[b:b + 1, sl], kn[b:b + 1, sl], vc[b:b + 1, sl], vn[b:b + 1, sl],
                                    w.seq_lens[b:b + 1], w.scale, w.k_bits, w.v_bits,
                                    O.codebook_f32(w.k_bits)[0], O.tcq_levels_f32(w.v_bits),
                                    O.sign_vector(w.sign_seed), w.sparse_thr)
        bound = None
        if w.sparse_thr > 0:
            kt = O.dequantize(kc[b:b + 1, sl], kn[b:b + 1, sl], w.k_bits, O.codebook_f32(w.k_bits)[0],
                              O.sign_vector(w.sign_seed))
            vt = O.dequantize_v2(vc[b:b + 1, sl], vn[b:b + 1, sl], w.v_bits, O.tcq_levels_f32(w.v_bits),
                                 O.sign_vector(w.sign_seed))
            wts = O.attention_weights(qs, kt, w.seq_lens[b:b + 1], w.scale)
            bound = np.zeros(qs.shape)
            n = int(w.seq_lens[b])
            for (bb, hh), wt in wts.items():
                amb = np.abs(np.log(np.maximum(wt, 1e-300) / w.sparse_thr)) < SPARSE_BAND
                bound[bb, hh] = wt[amb] @ np.abs(vt[bb, 0, :n][amb])
        check_decode(o_gpu[b:b + 1, h * g:(h + 1) * g], o_ref, bound)
