"""Decode step (tq_decode_step): the new token of every sequence is encoded
into the cache inside the decode launch, then attention reads it.

Checks: the appended codes and norms by the encoder's acceptance rules
against the oracle's encoding of the new rows; the output against the fp64
oracle run on the GPU's own codes after the step; the reconstruction-SNR band
against unquantised attention; and agreement with the two-call path
(tq_encode_kv append, then tq_decode_attention)."""
import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import inputs
from oracle import tq_oracle as O

from ._parity import (SNR_BAND_DB, check_codes, check_decode, check_norms, host, oracle_decode,
                      rel_err, snr_db, sparse_flip_bound, to_dev, torch_mod)

pytestmark = pytest.mark.gpu


def _step_case(w, lens, sparse_thr=0.0, kv_dtype=np.float16):
    """Cache holding every position except each sequence's last (len - 1),
    which is left as garbage; the step writes it from the true rows."""
    torch = torch_mod()
    lens = np.asarray(lens, dtype=np.int32)
    B, Hkv, S, D = w.k.shape
    rows = np.arange(B)
    pos = np.maximum(lens - 1, 0)
    k_new = np.ascontiguousarray(w.k[rows, :, pos]).astype(kv_dtype)   # [B, Hkv, D]
    v_new = np.ascontiguousarray(w.v[rows, :, pos]).astype(kv_dtype)
    k_old, v_old = w.k.copy(), w.v.copy()
    rng = np.random.default_rng(5)
    for b in range(B):
        if lens[b] > 0:
            k_old[b, :, pos[b]] = rng.standard_normal((Hkv, D)) * 3
            v_old[b, :, pos[b]] = rng.standard_normal((Hkv, D)) * 3
    desc = tq.kv_desc(B, Hkv, D, S, w.k_bits, w.v_bits, w.sign_seed)
    kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
    cache = tq.alloc_cache(desc)
    tq.encode_kv(cache, kcb, vcb, to_dev(k_old), to_dev(v_old))
    q = to_dev(w.q)
    lens_d = to_dev(lens)
    out = torch.full((B, w.q_heads, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(desc, w.q_heads, sparse_thr)
    tq.decode_step(cache, kcb, vcb, q, to_dev(k_new), to_dev(v_new), lens_d, w.scale, out, ws,
                   sparse_thr=sparse_thr)
    torch.cuda.synchronize()
    return cache, kcb, vcb, out.cpu().numpy().astype(np.float64), k_new, v_new, k_old, v_old, lens


def _check_step(w, lens, sparse_thr=0.0, kv_dtype=np.float16):
    cache, kcb, vcb, o_gpu, k_new, v_new, k_old, v_old, lens = _step_case(w, lens, sparse_thr, kv_dtype)
    kc, kn, vc, vn = host(cache)
    signs = O.sign_vector(w.sign_seed)
    # the appended rows, by the encoder's rules
    sel = [(b, int(lens[b]) - 1) for b in range(w.batch) if lens[b] > 0]
    for side, codes, norms, rows, bits in ((0, kc, kn, k_new, w.k_bits), (1, vc, vn, v_new, w.v_bits)):
        x = np.stack([rows[b] for b, _ in sel]).astype(np.float64)            # [n, Hkv, D]
        got_c = np.stack([codes[b, :, t] for b, t in sel])                    # [n, Hkv, nb, 16b]
        got_n = np.stack([norms[b, :, t] for b, t in sel])
        check_norms(got_n, x)
        check_codes(got_c, x, bits, signs)
    # every other position is untouched by the step
    mask = np.ones(kc.shape[:3], dtype=bool)
    for b, t in sel:
        mask[b, :, t] = False
    desc = cache.desc
    ref = tq.alloc_cache(desc)
    tq.encode_kv(ref, kcb, vcb, to_dev(k_old), to_dev(v_old))
    rk, _, rv, _ = host(ref)
    assert np.array_equal(kc[mask], rk[mask]) and np.array_equal(vc[mask], rv[mask])
    # the output, against the oracle on the GPU's codes after the step
    o_ref = oracle_decode(w.q, kc, kn, vc, vn, lens, w.scale, w.k_bits, w.v_bits, sparse_thr)
    bound = None
    if sparse_thr > 0:
        bound, _ = sparse_flip_bound(w.q, kc, kn, vc, vn, lens, w.scale, w.k_bits, w.v_bits, sparse_thr)
    check_decode(o_gpu, o_ref, bound)
    k_true, v_true = k_old.copy(), v_old.copy()
    for b, t in sel:
        k_true[b, :, t] = k_new[b].astype(np.float64)
        v_true[b, :, t] = v_new[b].astype(np.float64)
    exact = O.attention(w.q, k_true, v_true, lens, w.scale, sparse_thr)
    assert abs(snr_db(o_gpu, exact) - snr_db(o_ref, exact)) <= SNR_BAND_DB
    return o_gpu, cache, kcb, vcb, k_new, v_new, lens


def test_decode_step_gqa():
    w = inputs.make("gqa", batch=3, seq=300)
    _check_step(w, [300, 171, 17])


def test_decode_step_sparse_long_shape():
    w = inputs.make("long", batch=2, seq=1024)
    _check_step(w, [1024, 555], sparse_thr=1e-4)


def test_decode_step_wide_head_fp32_rows():
    w = inputs.make("ragged", batch=2, seq=400)
    _check_step(w, [400, 129], sparse_thr=0.0, kv_dtype=np.float32)


@pytest.mark.parametrize("hq,hkv", [(24, 2), (2, 2)])
def test_decode_step_group_sizes(hq, hkv):
    # groups above 8 split into head groups that each write the same token
    w = inputs.make("gqa", batch=2, seq=200)
    rng = np.random.default_rng(hq)
    w.q_heads, w.kv_heads = hq, hkv
    w.k, w.v = w.k[:, :hkv], w.v[:, :hkv]
    w.q = rng.standard_normal((2, hq, 128)).astype(np.float16)
    _check_step(w, [200, 64])


def test_decode_step_edge_lengths():
    # length 1 (only the new token), a full cache, and an empty sequence
    w = inputs.make("gqa", batch=3, seq=96)
    _check_step(w, [1, 96, 0])


def test_decode_step_agrees_with_append_then_decode():
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=256)
    o_step, cache, kcb, vcb, k_new, v_new, lens = _check_step(w, [256, 100])
    # the two-call path on a cache with the same old rows
    _, _, _, _, _, _, k_old, v_old, _ = _step_case(w, lens)
    c2 = tq.alloc_cache(cache.desc)
    tq.encode_kv(c2, kcb, vcb, to_dev(k_old), to_dev(v_old))
    start = to_dev(np.asarray(lens, dtype=np.int32) - 1)
    tq.encode_kv(c2, kcb, vcb, to_dev(k_new[:, :, None, :]), to_dev(v_new[:, :, None, :]), start_pos=start)
    out = torch.empty(o_step.shape, dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, w.q_heads)
    tq.decode_attention(c2, kcb, vcb, to_dev(w.q), to_dev(np.asarray(lens, dtype=np.int32)), w.scale, out, ws)
    torch.cuda.synchronize()
    assert rel_err(o_step, out.cpu().numpy().astype(np.float64)) <= 1e-3


def test_decode_step_length_beyond_cache_appends_nothing():
    """seq_lens[b] = seq_cap + 1 is a range error: the status bit is set, the
    attention runs over the clamped length, and no cached token -- in
    particular the last one, where a clamped append would land -- changes."""
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=64)
    desc = tq.kv_desc(2, w.kv_heads, 128, 64, w.k_bits, w.v_bits, w.sign_seed)
    kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
    cache = tq.alloc_cache(desc)
    tq.encode_kv(cache, kcb, vcb, to_dev(w.k), to_dev(w.v))
    before = host(cache)
    lens = np.array([65, 40], dtype=np.int32)
    rng = np.random.default_rng(9)
    k_new = (rng.standard_normal((2, w.kv_heads, 128)) * 3).astype(np.float16)
    v_new = (rng.standard_normal((2, w.kv_heads, 128)) * 3).astype(np.float16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((2, w.q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(desc, w.q_heads)
    tq.decode_step(cache, kcb, vcb, to_dev(w.q), to_dev(k_new), to_dev(v_new), to_dev(lens), w.scale,
                   out, ws, status=status)
    torch.cuda.synchronize()
    assert status.item() == tq.TQ_DEV_LEN_RANGE
    after = host(cache)
    # sequence 0: nothing written; sequence 1: only position 39 changed
    for a, b in zip(before, after):
        assert np.array_equal(a[0], b[0])
        keep = np.ones(a.shape[2], dtype=bool)
        keep[39] = False
        assert np.array_equal(a[1][:, keep], b[1][:, keep])
    kc, kn, vc, vn = after
    o_ref = oracle_decode(w.q, kc, kn, vc, vn, [64, 40], w.scale, w.k_bits, w.v_bits, 0.0)
    check_decode(out.cpu().numpy().astype(np.float64), o_ref)
