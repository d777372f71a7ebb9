"""Multi-token queries (tq_decode_attention_multi): n_q query tokens per
sequence are its last n_q positions, each seeing the positions up to its own.

Token j of a sequence of length n equals single-token decode attention over
the first n - n_q + j + 1 positions (an identity pinned in the oracle tests),
so each token is checked against the fp64 oracle (formulation B) on the GPU's
own codes with that length, plus the reconstruction-SNR band against the
oracle's dense multi-token attention; n_q = 1 must give tq_decode_attention's
output bit for bit."""
import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import inputs
from oracle import tq_oracle as O

from ._parity import (SNR_BAND_DB, check_decode, gpu_encode, host, oracle_decode, snr_db,
                      sparse_flip_bound, to_dev, torch_mod)

pytestmark = pytest.mark.gpu


def _multi(cache, kcb, vcb, q, lens, scale, sparse_thr=0.0):
    torch = torch_mod()
    B, n_q, hq, D = q.shape
    out = torch.full((B, n_q, hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, hq * n_q, sparse_thr)
    tq.decode_attention_multi(cache, kcb, vcb, to_dev(q), to_dev(np.asarray(lens, dtype=np.int32)), scale,
                              out, ws, sparse_thr=sparse_thr)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _check(w, n_q, lens, sparse_thr=0.0, seed=0):
    rng = np.random.default_rng(seed)
    B, hq, D = w.batch, w.q_heads, w.head_dim
    q = rng.standard_normal((B, n_q, hq, D)).astype(np.float16)
    cache, kcb, vcb = gpu_encode(w)
    o = _multi(cache, kcb, vcb, q, lens, w.scale, sparse_thr)
    kc, kn, vc, vn = host(cache)
    lens = np.asarray(lens)
    for j in range(n_q):
        lj = np.maximum(lens - n_q + j + 1, 0)
        ref = oracle_decode(q[:, j], kc, kn, vc, vn, lj, w.scale, w.k_bits, w.v_bits, sparse_thr)
        bound = None
        if sparse_thr > 0:
            bound, _ = sparse_flip_bound(q[:, j], kc, kn, vc, vn, lj, w.scale, w.k_bits, w.v_bits,
                                         sparse_thr)
        check_decode(o[:, j], ref, bound)
        assert np.all(o[lj == 0, j] == 0.0)
    exact = O.attention_multi(q, w.k, w.v, lens, w.scale, sparse_thr)
    refs = np.stack([oracle_decode(q[:, j], kc, kn, vc, vn, np.maximum(lens - n_q + j + 1, 0), w.scale,
                                   w.k_bits, w.v_bits, sparse_thr) for j in range(n_q)], axis=1)
    assert abs(snr_db(o, exact) - snr_db(refs, exact)) <= SNR_BAND_DB
    return o, q, cache, kcb, vcb


@pytest.mark.parametrize("n_q", [2, 4, 7])
def test_decode_multi_gqa(n_q):
    # group 4: 8, 16 and 28 (token, head) columns per kv-head
    w = inputs.make("gqa", batch=2, seq=300)
    _check(w, n_q, [300, 137], seed=n_q)


def test_decode_multi_single_token_is_decode_bit_for_bit():
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=200)
    o, q, cache, kcb, vcb = _check(w, 1, [200, 77])
    out = torch.empty(2, w.q_heads, 128, dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, w.q_heads)
    tq.decode_attention(cache, kcb, vcb, to_dev(q[:, 0]), to_dev(np.array([200, 77], dtype=np.int32)),
                        w.scale, out, ws)
    torch.cuda.synchronize()
    assert np.array_equal(o[:, 0], out.cpu().numpy().astype(np.float64))


def test_decode_multi_sparse_v():
    w = inputs.make("long", batch=2, seq=1024)
    _check(w, 3, [1024, 500], sparse_thr=1e-4, seed=3)


def test_decode_multi_wide_head():
    w = inputs.make("ragged", batch=2, seq=400)
    _check(w, 2, [400, 161], sparse_thr=0.0, seed=5)


def test_decode_multi_short_sequences():
    # sequences shorter than n_q: the first tokens see nothing and give zeros
    w = inputs.make("gqa", batch=3, seq=64)
    _check(w, 5, [3, 64, 0], seed=7)


def test_decode_multi_sixteen_tokens():
    # the largest n_q the ABI accepts: 64 (token, head) columns per kv-head
    w = inputs.make("gqa", batch=2, seq=256)
    _check(w, tq._lib.TQ_MAX_QUERY_TOKENS, [256, 90], seed=16)


# ---- multi-token queries over v3 and v2 V caches ---------------------------

def _multi_fmt(fn, cache, kcb, vcb, q, lens, scale, *extra):
    torch = torch_mod()
    B, n_q, hq, D = q.shape
    out = torch.full((B, n_q, hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, hq * n_q, 0.0)
    fn(cache, kcb, vcb, *extra, to_dev(q), to_dev(np.asarray(lens, dtype=np.int32)), scale, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("n_q,lens", [(2, [400, 251]), (3, [400, 3])])
def test_decode_multi_v3(n_q, lens):
    """Token j over a v3 cache equals the single-token v3 oracle over the first
    len - n_q + j + 1 positions (outlier channels and the rest each within the
    decode tolerance); n_q = 1 is tq_decode_attention_v3 bit for bit."""
    from .test_v3_gpu import _check_v3_decode, _decode_v3, _encode_v3
    w = inputs.make("gqa", batch=2, seq=400, dist="outlier_v")
    rng = np.random.default_rng(40 + n_q)
    q = rng.standard_normal((2, n_q, w.q_heads, w.head_dim)).astype(np.float16)
    cache, kcb, vcb, vo = _encode_v3(w, 8)
    o = _multi_fmt(tq.decode_attention_multi_v3, cache, kcb, vcb, q, lens, w.scale, vo)
    kc, kn, vc, vn = host(cache)
    vals = vo.values.cpu().numpy().view(np.float16)[..., : vo.k]
    ch = vo.channels.cpu().numpy()
    kcent, vcent = O.codebook_f32(w.k_bits)[0], O.codebook_f32(w.v_bits)[0]
    for j in range(n_q):
        lj = np.maximum(np.asarray(lens) - n_q + j + 1, 0)
        ref = O.decode_v3_rotated(q[:, j].astype(np.float64), kc, kn, vc, vn, vals, ch, lj, w.scale, w.k_bits,
                                  w.v_bits, kcent, vcent, O.sign_vector(w.sign_seed), 0.0)
        _check_v3_decode(o[:, j], ref, ch, w.q_heads // w.kv_heads)
    one = _multi_fmt(tq.decode_attention_multi_v3, cache, kcb, vcb, q[:, :1], lens, w.scale, vo)
    single = _decode_v3(cache, kcb, vcb, vo, q[:, 0], lens, w.scale)
    assert np.array_equal(one[:, 0], single)


@pytest.mark.parametrize("n_q,lens,vb", [(2, [400, 251], 3), (3, [400, 3], 2)])
def test_decode_multi_v2(n_q, lens, vb):
    """Token j over a v2 cache equals the single-token v2 oracle over the first
    len - n_q + j + 1 positions; n_q = 1 is tq_decode_attention_v2 bit for bit."""
    from .test_v2_gpu import _decode_v2, _encode_v2
    w = inputs.make("gqa", batch=2, seq=400)
    w.v_bits = vb
    rng = np.random.default_rng(50 + n_q)
    q = rng.standard_normal((2, n_q, w.q_heads, w.head_dim)).astype(np.float16)
    cache, kcb, vtq = _encode_v2(w)
    o = _multi_fmt(tq.decode_attention_multi_v2, cache, kcb, vtq, q, lens, w.scale)
    kc, kn, vc, vn = host(cache)
    for j in range(n_q):
        lj = np.maximum(np.asarray(lens) - n_q + j + 1, 0)
        ref = O.decode_v2_rotated(q[:, j].astype(np.float64), kc, kn, vc, vn, lj, w.scale, w.k_bits, w.v_bits,
                                  O.codebook_f32(w.k_bits)[0], O.tcq_levels_f32(w.v_bits),
                                  O.sign_vector(w.sign_seed), 0.0)
        check_decode(o[:, j], ref)
    one = _multi_fmt(tq.decode_attention_multi_v2, cache, kcb, vtq, q[:, :1], lens, w.scale)
    single = _decode_v2(cache, kcb, vtq, q[:, 0], lens, w.scale)
    assert np.array_equal(one[:, 0], single)
