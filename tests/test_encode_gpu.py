"""Encoder parity: CUDA kernel (through the C ABI) against the fp64 oracle."""
import itertools

import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import inputs
from oracle import tq_oracle as O

from ._parity import check_codes, check_norms, gpu_encode, host, to_dev, torch_mod

pytestmark = pytest.mark.gpu

SIGNS0 = O.sign_vector(0)


def _check_all(w, cache, k=None, v=None, signs=SIGNS0):
    kc, kn, vc, vn = host(cache)
    k = w.k if k is None else k
    v = w.v if v is None else v
    check_norms(kn, k)
    check_norms(vn, v)
    check_codes(kc, k, w.k_bits, signs)
    check_codes(vc, v, w.v_bits, signs)


def test_encode_toy_fp32():
    w = inputs.make("toy")
    cache, _, _ = gpu_encode(w)
    _check_all(w, cache)


def test_encode_outlier_workload_reduced():
    w = inputs.make("encode", batch=2, seq=1024)
    cache, _, _ = gpu_encode(w)
    _check_all(w, cache)


@pytest.mark.parametrize("kb,vb", list(itertools.product([2, 3, 4], repeat=2)))
def test_encode_bit_widths_fp16_d256(kb, vb):
    rng = np.random.default_rng(kb * 10 + vb)
    w = inputs.make("ragged", batch=1, seq=40)
    w.k_bits, w.v_bits = kb, vb
    w.k = (rng.standard_normal(w.k.shape) * 3).astype(np.float16)
    cache, _, _ = gpu_encode(w)
    _check_all(w, cache)


def test_encode_sign_seed_matters():
    w = inputs.make("toy")
    w.sign_seed = 987654321
    cache, _, _ = gpu_encode(w)
    _check_all(w, cache, signs=O.sign_vector(987654321))


def test_encode_start_pos_out_of_range_rows_are_skipped():
    torch = torch_mod()
    w = inputs.make("toy", seq=16)
    w.k = np.concatenate([w.k, w.k + 1], axis=0)
    w.v = np.concatenate([w.v, w.v - 1], axis=0)
    w.batch = 2
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache, _, _ = gpu_encode(w, start_pos=[3, 57], seq_cap=64, status=status)
    kc, kn, vc, vn = host(cache)
    assert status.item() == tq.TQ_DEV_POS_RANGE
    # batch 0: rows land at 3..18; batch 1: rows 0..6 land at 57..63, rows 7.. skipped
    check_norms(kn[0, :, 3:19], w.k[0])
    check_codes(kc[0, :, 3:19], w.k[0], 4, SIGNS0)
    check_codes(vc[1, :, 57:64], w.v[1, :, :7], 4, SIGNS0)
    assert np.all(kc[0, :, :3] == 0) and np.all(kc[0, :, 19:] == 0)
    assert np.all(kc[1, :, :57] == 0)


def test_encode_zero_block_and_norm_overflow():
    torch = torch_mod()
    w = inputs.make("toy", seq=8)
    k = w.k.copy()
    k[0, 0, 2] = 0.0
    k[0, 0, 5] = 1.0e5          # norm ~1.1e6 > fp16 max
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache, _, _ = gpu_encode(w, k=k, status=status)
    kc, kn, _, _ = host(cache)
    assert status.item() == tq.TQ_DEV_NORM_OVERFLOW
    assert kn[0, 0, 2, 0] == 0 and np.all(O.unpack_codes(kc[0, 0, 2, 0], 4) == 7)
    assert kn[0, 0, 5, 0].view(np.uint16) == 0x7BFF
    check_codes(kc, k, 4, SIGNS0)          # codes use the unrounded norm


def test_encode_k_only_leaves_v_untouched():
    torch = torch_mod()
    w = inputs.make("toy", seq=32)
    desc = tq.kv_desc(1, 1, 128, 32, 4, 4)
    cache = tq.alloc_cache(desc)
    tq.encode_kv(cache, tq.make_codebook(4), tq.make_codebook(4), k=to_dev(w.k))
    torch.cuda.synchronize()
    kc, kn, vc, vn = host(cache)
    check_codes(kc, w.k, 4, SIGNS0)
    assert np.all(vc == 0) and np.all(vn.view(np.uint16) == 0)


def test_encode_full_size_outlier_workload_sampled():
    """Full encode workload (B8, Hkv8, S32768, fp16, K3/V2), launched as the
    benchmark launches it; 20000 sampled blocks per side against the oracle."""
    w = inputs.make("encode")
    cache, _, _ = gpu_encode(w)
    kc, kn, vc, vn = host(cache)
    rng = np.random.default_rng(123)
    n = 20000
    bi = rng.integers(0, w.batch, n)
    hi = rng.integers(0, w.kv_heads, n)
    ti = rng.integers(0, w.seq_cap, n)
    for codes, norms, x, bits in ((kc, kn, w.k, w.k_bits), (vc, vn, w.v, w.v_bits)):
        xs = x[bi, hi, ti]
        check_norms(norms[bi, hi, ti], xs)
        check_codes(codes[bi, hi, ti], xs, bits, SIGNS0)
