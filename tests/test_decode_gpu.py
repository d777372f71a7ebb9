"""Decode-attention parity: CUDA path (through the C ABI) against the fp64
oracle run on the GPU's own codes, plus the reconstruction-SNR band against
fp64 attention on the unquantised K/V."""
import math

import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import inputs
from oracle import tq_oracle as O

from ._parity import (DECODE_REL_TOL, SNR_BAND_DB, check_decode, gpu_decode, gpu_encode, host,
                      oracle_decode, rel_err, snr_db, sparse_flip_bound, to_dev, torch_mod)

pytestmark = pytest.mark.gpu


def _run(w, sparse_thr=None, check_snr=True):
    thr = w.sparse_thr if sparse_thr is None else sparse_thr
    cache, kcb, vcb = gpu_encode(w)
    o_gpu, _ = gpu_decode(cache, kcb, vcb, w.q, w.seq_lens, w.scale, thr)
    kc, kn, vc, vn = host(cache)
    o_ref = oracle_decode(w.q, kc, kn, vc, vn, w.seq_lens, w.scale, w.k_bits, w.v_bits, thr)
    bound = None
    if thr > 0:
        bound, _ = sparse_flip_bound(w.q, kc, kn, vc, vn, w.seq_lens, w.scale, w.k_bits, w.v_bits, thr)
    err = check_decode(o_gpu, o_ref, bound)
    if check_snr:
        exact = O.attention(w.q, w.k, w.v, w.seq_lens, w.scale, thr)
        s_gpu, s_orc = snr_db(o_gpu, exact), snr_db(o_ref, exact)
        assert abs(s_gpu - s_orc) <= SNR_BAND_DB, (s_gpu, s_orc)
    return o_gpu, o_ref, err


def test_decode_toy():
    _run(inputs.make("toy"))


@pytest.mark.parametrize("sparse", [False, True])
def test_decode_gqa_reduced(sparse):
    w = inputs.make("gqa", batch=2, seq=1000)
    w.seq_lens = np.array([1000, 777], dtype=np.int32)
    _run(w, sparse_thr=3e-4 if sparse else 0.0)


@pytest.mark.parametrize("sparse", [False, True])
def test_decode_long_reduced(sparse):
    w = inputs.make("long", seq=4096)
    # the 131072-token threshold scaled to 4096 tokens skips the same fraction
    _run(w, sparse_thr=(1e-6 * 131072 / 4096) if sparse else 0.0)


@pytest.mark.parametrize("sparse", [False, True])
def test_decode_ragged_wide_head_reduced(sparse):
    w = inputs.make("ragged", seq=1200)
    _run(w, sparse_thr=(1e-5 * 40960 / 700) if sparse else 0.0)


@pytest.mark.parametrize("kb", [2, 3, 4])
@pytest.mark.parametrize("vb", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256])
def test_decode_bit_widths(kb, vb, d):
    rng = np.random.default_rng(100 * kb + 10 * vb + d)
    w = inputs.make("ragged" if d == 256 else "gqa", batch=2, seq=150)
    w.k_bits, w.v_bits = kb, vb
    w.seq_lens = np.array([150, 61], dtype=np.int32)
    w.q = (rng.standard_normal(w.q.shape) * 2).astype(np.float16)
    _run(w)


@pytest.mark.parametrize("kb,vb", [(4, 4), (3, 4), (4, 2)])
@pytest.mark.parametrize("hq", [8, 16])
def test_decode_wide_head_fused_bit_widths(kb, vb, hq):
    # head_dim 256 with sparse-V off: the fused kernel with the largest ring
    # slots (the ring is shortened to fit shared memory); groups of 2 and 4
    w = inputs.make("ragged", batch=2, seq=700)
    rng = np.random.default_rng(7 * kb + vb + hq)
    w.k_bits, w.v_bits, w.q_heads = kb, vb, hq
    w.seq_lens = np.array([700, 333], dtype=np.int32)
    w.q = rng.standard_normal((2, hq, 256)).astype(np.float16)
    _run(w, sparse_thr=0.0)


@pytest.mark.parametrize("hq,hkv", [(2, 2), (6, 2), (16, 2), (24, 2), (20, 4)])
def test_decode_group_sizes(hq, hkv):
    w = inputs.make("gqa", batch=2, seq=200)
    rng = np.random.default_rng(hq)
    w.q_heads, w.kv_heads = hq, hkv
    w.k, w.v = w.k[:, :hkv], w.v[:, :hkv]
    w.q = rng.standard_normal((2, hq, 128)).astype(np.float16)
    w.seq_lens = np.array([200, 133], dtype=np.int32)
    _run(w)
    _run(w, sparse_thr=2e-3)


def test_decode_edge_lengths_and_fp32_query():
    # seq_cap not a multiple of the 16-token tile; lengths 0, 1, 15, 16, 17, cap
    w = inputs.make("gqa", batch=6, seq=70)
    w.seq_lens = np.array([0, 1, 15, 16, 17, 70], dtype=np.int32)
    o_gpu, o_ref, _ = _run(w, check_snr=False)
    assert np.all(o_gpu[0] == 0)
    w.q = w.q.astype(np.float32) * 1.7
    _run(w, check_snr=False)
    _run(w, sparse_thr=1e-2, check_snr=False)


def test_decode_single_token_equals_dequantised_value():
    w = inputs.make("toy", seq=16)
    w.seq_lens = np.array([1], dtype=np.int32)
    cache, kcb, vcb = gpu_encode(w)
    o_gpu, _ = gpu_decode(cache, kcb, vcb, w.q, w.seq_lens, w.scale)
    kc, kn, vc, vn = host(cache)
    v0 = O.dequantize(vc[0, 0, 0], vn[0, 0, 0], 4, O.codebook_f32(4)[0], O.sign_vector(0))
    assert rel_err(o_gpu[0, 0], v0) <= DECODE_REL_TOL


def test_decode_length_clamp_sets_status():
    torch = torch_mod()
    w = inputs.make("gqa", batch=2, seq=64)
    cache, kcb, vcb = gpu_encode(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_gpu, _ = gpu_decode(cache, kcb, vcb, w.q, [100, -5], w.scale, status=status)
    assert status.item() == tq.TQ_DEV_LEN_RANGE
    kc, kn, vc, vn = host(cache)
    o_ref = oracle_decode(w.q, kc, kn, vc, vn, [64, 0], w.scale, w.k_bits, w.v_bits, 0.0)
    assert rel_err(o_gpu, o_ref) <= DECODE_REL_TOL
    assert np.all(o_gpu[1] == 0)


def test_decode_repeatable_and_workspace_reuse():
    """Fixed merge order: repeated calls on one workspace are bit-identical,
    and the workspace is left ready (counters back to zero) after each call."""
    torch = torch_mod()
    w = inputs.make("long", seq=3000)
    cache, kcb, vcb = gpu_encode(w)
    o1, ws = gpu_decode(cache, kcb, vcb, w.q, w.seq_lens, w.scale)
    o2, _ = gpu_decode(cache, kcb, vcb, w.q, w.seq_lens, w.scale, workspace=ws, reps=3)
    assert np.array_equal(o1, o2)
    units = w.batch * w.kv_heads
    assert torch.all(ws[: 4 * units * 8] == 0).item()  # one count per (unit, head slot)


# ---------------------------------------------------------------- full size --

def _full_sampled(w, units, sparse_thr):
    """Decode the full workload on the GPU (the benchmark's launch), then check
    sampled (batch, kv-head) units against the oracle one by one."""
    cache, kcb, vcb = gpu_encode(w)
    o_gpu, _ = gpu_decode(cache, kcb, vcb, w.q, w.seq_lens, w.scale, sparse_thr)
    g = w.q_heads // w.kv_heads
    kc, kn, vc, vn = host(cache)
    for b, h in units:
        sl = slice(h, h + 1)
        qs = w.q[b:b + 1, h * g:(h + 1) * g]
        o_ref = oracle_decode(qs, kc[b:b + 1, sl], kn[b:b + 1, sl], vc[b:b + 1, sl], vn[b:b + 1, sl],
                              w.seq_lens[b:b + 1], w.scale, w.k_bits, w.v_bits, sparse_thr)
        got = o_gpu[b:b + 1, h * g:(h + 1) * g]
        bound = None
        if sparse_thr > 0:
            bound, _ = sparse_flip_bound(qs, kc[b:b + 1, sl], kn[b:b + 1, sl], vc[b:b + 1, sl],
                                         vn[b:b + 1, sl], w.seq_lens[b:b + 1], w.scale, w.k_bits,
                                         w.v_bits, sparse_thr)
        check_decode(got, o_ref, bound)
        exact = O.attention(qs, w.k[b:b + 1, sl], w.v[b:b + 1, sl], w.seq_lens[b:b + 1], w.scale, sparse_thr)
        assert abs(snr_db(got, exact) - snr_db(o_ref, exact)) <= SNR_BAND_DB


def test_decode_full_gqa_sampled():
    _full_sampled(inputs.make("gqa"), [(0, 0), (3, 5), (7, 7)], 0.0)


@pytest.mark.parametrize("sparse", [False, True])
def test_decode_full_long_sampled(sparse):
    w = inputs.make("long")
    _full_sampled(w, [(0, 0), (0, 6)], w.sparse_thr if sparse else 0.0)


def test_decode_full_ragged_sampled():
    w = inputs.make("ragged")
    _full_sampled(w, [(0, 1), (3, 3)], w.sparse_thr)


# ------------------------------------------------- heavy tails and peaks --

@pytest.mark.parametrize("name,seq", [("gqa", 600), ("ragged", 700)])
def test_decode_heavy_tailed_kv(name, seq):
    """The encode-only workload's distributions through decode: K with
    LogNormal per-channel scales and 2 % of channels x20 (block norms up to
    ~100x the Gaussian ones), V ~ Student-t(4), at D128 and D256."""
    w = inputs.make(name, batch=2, seq=seq, dist="outlier_t4")
    w.seq_lens = np.array([seq, seq // 2 + 3], dtype=np.int32)
    _run(w)
    _run(w, sparse_thr=2e-3)


@pytest.mark.parametrize("pos", ["first", "middle", "last"])
@pytest.mark.parametrize("gain", [30.0, 60.0])
def test_decode_peaked_attention(pos, gain):
    """One cached key dominates: q_h = gain * k_j / |k_j| (scores of position j
    about gain, the rest ~N(0, gain^2 / D)).  The running maximum jumps by far
    more than the lazy-rescale threshold inside a tile, and every CTA that
    does not hold position j sees weights that vanish after the merge.  The
    sequences span several CTAs each."""
    w = inputs.make("gqa", batch=2, seq=6000)
    w.seq_lens = np.array([6000, 4321], dtype=np.int32)
    q = np.empty((2, w.q_heads, 128), dtype=np.float64)
    g = w.q_heads // w.kv_heads
    for b in range(2):
        n = int(w.seq_lens[b])
        j = {"first": 3, "middle": n // 2 + 5, "last": n - 1}[pos]
        for h in range(w.q_heads):
            k = w.k[b, h // g, j].astype(np.float64)
            q[b, h] = gain * k / np.linalg.norm(k) * (1.0 if h % 2 == 0 else 0.5)
    w.q = q.astype(np.float16)
    _run(w)
