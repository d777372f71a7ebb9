"""C-ABI host tests (CPU only): the library loads, exports every symbol that
include/tq.h declares, its host-side codebook and sign vector agree with the
oracle, and invalid arguments are rejected before anything is launched."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import _lib
from oracle import tq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _header_functions()
    assert len(names) == 17
    lib = tq.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES)


def test_struct_layouts():
    assert ctypes.sizeof(_lib.Codebook) == 4 + 16 * 4 + 15 * 4
    assert ctypes.sizeof(_lib.KVDesc) == 32
    assert _lib.KVDesc.sign_seed.offset == 16
    assert ctypes.sizeof(_lib.VOutliers) == 24 and _lib.VOutliers.channels.offset == 8


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_oracle(bits):
    cb = tq.make_codebook(bits)
    c, t = tq.codebook_arrays(cb)
    oc, ot = O.codebook_f32(bits)
    assert np.array_equal(c, oc)
    # The oracle's middle boundary carries an fp64 rounding residue (~1e-16);
    # the library's is exactly 0 by symmetry.
    np.testing.assert_allclose(t, ot, rtol=0, atol=1e-15)
    assert t[len(t) // 2] == 0.0
    assert np.array_equal(c, -c[::-1]) and np.array_equal(t, -t[::-1])


@pytest.mark.parametrize("seed", [0, 1, 1234567, 2**64 - 1])
def test_sign_vector_matches_oracle(seed):
    assert np.array_equal(tq.sign_vector(seed), O.sign_vector(seed).astype(np.int8))


def test_codebook_errors():
    lib = tq.lib()
    assert lib.tq_make_codebook(3, None) == _lib.TQ_ERR_INVALID_ARG
    cb = _lib.Codebook()
    assert lib.tq_make_codebook(5, ctypes.byref(cb)) == _lib.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_codebook(0, ctypes.byref(cb)) == _lib.TQ_ERR_UNSUPPORTED
    assert lib.tq_sign_vector(0, None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_status_string(3).decode().startswith("workspace")


def _fake(addr):
    return ctypes.c_void_p(addr)


GOOD = 0x7f0000000000  # aligned fake device addresses: never dereferenced on error paths


def test_encode_rejects_bad_arguments_without_launch():
    lib = tq.lib()
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)

    def call(desc, k=GOOD, v=GOOD, dtype=1, seq_new=4, kcb=cb3, vcb=cb2, kc=GOOD, vn=GOOD, sp=None):
        return lib.tq_encode_kv(ctypes.byref(desc) if desc is not None else None,
                                ctypes.byref(kcb), ctypes.byref(vcb),
                                _fake(k) if k else None, _fake(v) if v else None, dtype, seq_new,
                                _fake(sp) if sp else None, _fake(kc) if kc else None, _fake(GOOD),
                                _fake(GOOD), _fake(vn) if vn else None, None, None)

    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    assert call(None) == _lib.TQ_ERR_INVALID_ARG
    assert call(tq.kv_desc(2, 2, 96, 64, 3, 2)) == _lib.TQ_ERR_UNSUPPORTED
    assert call(tq.kv_desc(2, 2, 128, 64, 5, 2)) == _lib.TQ_ERR_UNSUPPORTED
    assert call(tq.kv_desc(0, 2, 128, 64, 3, 2)) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, dtype=7) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, seq_new=-1) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, k=0, v=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, kc=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, vn=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, k=GOOD + 8) == _lib.TQ_ERR_INVALID_ARG          # misaligned input
    assert call(d, kc=GOOD + 4) == _lib.TQ_ERR_INVALID_ARG         # misaligned codes
    assert call(d, kcb=cb2) == _lib.TQ_ERR_INVALID_ARG             # codebook bits mismatch
    assert call(d, sp=GOOD + 2) == _lib.TQ_ERR_INVALID_ARG
    bad = tq.make_codebook(3)
    bad.boundaries[0] = bad.boundaries[1] + 1.0                    # not ascending
    assert call(d, kcb=bad) == _lib.TQ_ERR_INVALID_ARG
    assert call(d, seq_new=0) == _lib.TQ_OK                        # no-op, nothing launched


def test_decode_rejects_bad_arguments_without_launch():
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)
    need = tq.decode_workspace_size(d, 8)

    def call(desc=d, hq=8, q=GOOD, qd=1, kc=GOOD, lens=GOOD, scale=0.1, thr=0.0, out=GOOD, ws=GOOD,
             wsb=None, kcb=cb3, vcb=cb2):
        return lib.tq_decode_attention(ctypes.byref(desc), ctypes.byref(kcb), ctypes.byref(vcb), hq,
                                       _fake(q) if q else None, qd, _fake(kc) if kc else None,
                                       _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                       _fake(lens) if lens else None, scale, thr,
                                       _fake(out) if out else None, _fake(ws) if ws else None,
                                       need if wsb is None else wsb, None, None)

    assert call(hq=7) == _lib.TQ_ERR_INVALID_ARG
    assert call(hq=1) == _lib.TQ_ERR_INVALID_ARG
    assert call(q=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(qd=3) == _lib.TQ_ERR_INVALID_ARG
    assert call(kc=GOOD + 1) == _lib.TQ_ERR_INVALID_ARG
    assert call(lens=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(out=GOOD + 4) == _lib.TQ_ERR_INVALID_ARG
    assert call(scale=math.inf) == _lib.TQ_ERR_INVALID_ARG
    assert call(thr=math.nan) == _lib.TQ_ERR_INVALID_ARG
    assert call(kcb=cb2) == _lib.TQ_ERR_INVALID_ARG
    assert call(ws=0) == _lib.TQ_ERR_WORKSPACE
    assert call(ws=GOOD + 16) == _lib.TQ_ERR_WORKSPACE
    assert call(wsb=need - 1) == _lib.TQ_ERR_WORKSPACE
    # sparse mode needs the score buffer: the dense size is too small
    assert call(thr=1e-5) == _lib.TQ_ERR_WORKSPACE
    assert call(desc=tq.kv_desc(2, 2, 384, 64, 3, 2)) in (_lib.TQ_ERR_UNSUPPORTED, _lib.TQ_ERR_WORKSPACE)
    assert call(desc=tq.kv_desc(2049, 2, 128, 64, 3, 2)) in (_lib.TQ_ERR_UNSUPPORTED, _lib.TQ_ERR_WORKSPACE)
    odd = tq.kv_desc(2, 2, 128, 63, 3, 2)
    assert lib.tq_decode_attention(ctypes.byref(odd), ctypes.byref(cb3), ctypes.byref(cb2), 8, _fake(GOOD), 1,
                                   _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), 0.1, 0.0,
                                   _fake(GOOD), _fake(GOOD), 1 << 30, None, None) == _lib.TQ_ERR_UNSUPPORTED


def test_decode_step_rejects_bad_arguments_without_launch():
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)
    need = tq.decode_workspace_size(d, 8)

    def call(kn=GOOD, vn=GOOD, kvd=1, q=GOOD, wsb=None):
        return lib.tq_decode_step(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), 8,
                                  _fake(q) if q else None, 1, _fake(kn) if kn else None,
                                  _fake(vn) if vn else None, kvd, _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                  _fake(GOOD), _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD),
                                  need if wsb is None else wsb, None, None)

    assert call(kn=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(vn=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(kn=GOOD + 8) == _lib.TQ_ERR_INVALID_ARG      # misaligned new rows
    assert call(kvd=5) == _lib.TQ_ERR_INVALID_ARG
    assert call(q=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(wsb=need - 1) == _lib.TQ_ERR_WORKSPACE


def test_decode_multi_rejects_bad_token_counts():
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)

    def call(n_q):
        need = tq.decode_workspace_size(d, 8 * max(n_q, 1))
        return lib.tq_decode_attention_multi(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), 8, n_q,
                                             _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                             _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD), need, None, None)

    assert call(0) == _lib.TQ_ERR_INVALID_ARG
    assert call(_lib.TQ_MAX_QUERY_TOKENS + 1) == _lib.TQ_ERR_INVALID_ARG
    # the workspace must be sized for q_heads * n_q
    need1 = tq.decode_workspace_size(d, 8)
    assert lib.tq_decode_attention_multi(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), 8, 4,
                                         _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                         _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD), need1, None,
                                         None) == _lib.TQ_ERR_WORKSPACE


def test_workspace_size_formula():
    d = tq.kv_desc(8, 8, 128, 32768, 3, 3)
    dense = tq.decode_workspace_size(d, 32)
    sparse = tq.decode_workspace_size(d, 32, 1e-6)
    assert dense > 0 and sparse - dense >= 8 * 32 * 32768 * 4
    assert tq.decode_workspace_size(d, 33) == 0
    assert tq.decode_workspace_size(tq.kv_desc(8, 8, 100, 32768, 3, 3), 32) == 0


def test_cache_shapes_give_b_plus_one_eighth_bits():
    for b in (2, 3, 4):
        d = tq.kv_desc(2, 3, 256, 10, b, b)
        s = tq.cache_shapes(d)
        code_bytes = int(np.prod(s["k_codes"]))
        norm_bytes = 2 * int(np.prod(s["k_norms"]))
        values = 2 * 3 * 10 * 256
        assert (code_bytes + norm_bytes) * 8 / values == b + 16 / 128


def test_noalloc_checks_arguments_before_any_cuda_call():
    """Every argument error of the no-alloc entry point is found on the host,
    before the scratch array is looked up: here, with no GPU at all, a bad
    call returns its own status, never TQ_ERR_CUDA."""
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)

    def call(desc=d, hq=8, q=GOOD, qd=1, lens=GOOD, out=GOOD, scale=0.1, thr=0.0, kcb=cb3, status=None):
        return lib.tq_decode_attention_noalloc(ctypes.byref(desc), ctypes.byref(kcb), ctypes.byref(cb2), hq,
                                               _fake(q) if q else None, qd, _fake(GOOD), _fake(GOOD),
                                               _fake(GOOD), _fake(GOOD), _fake(lens) if lens else None,
                                               scale, thr, _fake(out) if out else None,
                                               _fake(status) if status else None, None)

    assert call(q=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(qd=9) == _lib.TQ_ERR_INVALID_ARG
    assert call(hq=7) == _lib.TQ_ERR_INVALID_ARG
    assert call(lens=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(out=GOOD + 4) == _lib.TQ_ERR_INVALID_ARG
    assert call(scale=math.nan) == _lib.TQ_ERR_INVALID_ARG
    assert call(kcb=cb2) == _lib.TQ_ERR_INVALID_ARG
    assert call(status=GOOD + 2) == _lib.TQ_ERR_INVALID_ARG
    assert call(desc=tq.kv_desc(2, 2, 128, 63, 3, 2)) == _lib.TQ_ERR_UNSUPPORTED
    big = tq.kv_desc(64, 8, 256, 65536, 3, 3)
    assert lib.tq_decode_attention_noalloc(ctypes.byref(big), ctypes.byref(cb3), ctypes.byref(cb3), 32,
                                           _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                           _fake(GOOD), _fake(GOOD), 0.1, 1e-5, _fake(GOOD), None,
                                           None) == _lib.TQ_ERR_SCRATCH_LIMIT


def test_read_device_status_argument_errors():
    lib = tq.lib()
    bits = ctypes.c_uint32(0)
    assert lib.tq_read_device_status(None, ctypes.byref(bits), None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_read_device_status(_fake(GOOD), None, None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_read_device_status(_fake(GOOD + 2), ctypes.byref(bits), None) == _lib.TQ_ERR_INVALID_ARG
    assert lib.tq_status_string(_lib.TQ_ERR_DEVICE_BOUNDS).decode().startswith("the device status")
    assert lib.tq_status_string(_lib.TQ_ERR_SCRATCH_LIMIT).decode().startswith("request needs")


def _vo(k=4, ch=GOOD, val=GOOD):
    return _lib.VOutliers(k, _fake(ch) if ch else None, _fake(val) if val else None)


def test_v3_encode_rejects_bad_outliers_without_launch():
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)

    def call(vo, v=GOOD):
        return lib.tq_encode_kv_v3(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), _fake(GOOD),
                                   _fake(v) if v else None, 1, 4, None, _fake(GOOD), _fake(GOOD),
                                   _fake(GOOD) if v else None, _fake(GOOD) if v else None,
                                   ctypes.byref(vo) if vo is not None else None, None, None)

    assert call(_vo(k=17)) == _lib.TQ_ERR_INVALID_ARG               # above TQ_MAX_OUTLIERS
    assert call(_vo(k=-1)) == _lib.TQ_ERR_INVALID_ARG
    assert call(_vo(ch=0)) == _lib.TQ_ERR_INVALID_ARG               # no channel list
    assert call(_vo(val=0)) == _lib.TQ_ERR_INVALID_ARG              # no value buffer
    assert call(_vo(ch=GOOD + 2)) == _lib.TQ_ERR_INVALID_ARG        # misaligned channels
    assert call(_vo(val=GOOD + 8)) == _lib.TQ_ERR_INVALID_ARG       # values rows are 16-byte
    assert call(_vo(), v=0) == _lib.TQ_ERR_INVALID_ARG              # v3 needs the V side
    # k = 0 is the plain format: the checks of tq_encode_kv apply (here a no-op)
    assert lib.tq_encode_kv_v3(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), _fake(GOOD), _fake(GOOD),
                               1, 0, None, _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD),
                               ctypes.byref(_vo(k=0, ch=0, val=0)), None, None) == _lib.TQ_OK


def test_v3_decode_rejects_bad_outliers_without_launch():
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2 = tq.make_codebook(3), tq.make_codebook(2)
    need = tq.decode_workspace_size(d, 8)

    def call(vo, wsb=need, hq=8):
        return lib.tq_decode_attention_v3(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), hq,
                                          _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                          ctypes.byref(vo), _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD),
                                          wsb, None, None)

    assert call(_vo(k=17)) == _lib.TQ_ERR_INVALID_ARG
    assert call(_vo(ch=0)) == _lib.TQ_ERR_INVALID_ARG
    assert call(_vo(val=GOOD + 4)) == _lib.TQ_ERR_INVALID_ARG
    assert call(_vo(), hq=7) == _lib.TQ_ERR_INVALID_ARG             # the plain decode's checks too
    assert call(_vo(), wsb=need - 1) == _lib.TQ_ERR_WORKSPACE
    # head_dim 256 with 7 or 8 bits per K/V pair: no shared-memory plan
    d256 = tq.kv_desc(2, 2, 256, 64, 4, 3)
    assert lib.tq_decode_attention_v3(ctypes.byref(d256), ctypes.byref(tq.make_codebook(4)), ctypes.byref(cb3), 8,
                                      _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                      ctypes.byref(_vo()), _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD),
                                      tq.decode_workspace_size(d256, 8), None, None) == _lib.TQ_ERR_UNSUPPORTED


def test_pick_outlier_channels_rejects_bad_arguments_without_launch():
    lib = tq.lib()

    def call(desc=tq.kv_desc(2, 2, 128, 64, 3, 2), v=GOOD, dt=1, rows=64, k=4, ch=GOOD):
        return lib.tq_pick_outlier_channels(ctypes.byref(desc), _fake(v) if v else None, dt, rows, k,
                                            _fake(ch) if ch else None, None)

    assert call(k=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(k=17) == _lib.TQ_ERR_INVALID_ARG
    assert call(rows=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(dt=4) == _lib.TQ_ERR_INVALID_ARG
    assert call(v=0) == _lib.TQ_ERR_INVALID_ARG
    assert call(v=GOOD + 2) == _lib.TQ_ERR_INVALID_ARG
    assert call(ch=GOOD + 1) == _lib.TQ_ERR_INVALID_ARG
    assert call(desc=tq.kv_desc(2, 2, 384, 64, 3, 2)) == _lib.TQ_ERR_UNSUPPORTED
    assert call(desc=tq.kv_desc(2, 2, 100, 64, 3, 2)) == _lib.TQ_ERR_UNSUPPORTED


def test_outlier_row_width():
    assert [tq.outlier_row(k) for k in (1, 8, 9, 16)] == [8, 8, 16, 16]


def test_v2_entry_points_reject_bad_arguments_without_launch():
    lib = tq.lib()
    cb3 = tq.make_codebook(3)

    def enc(desc, vtq, k=GOOD, v=GOOD, seq_new=4):
        return lib.tq_encode_kv_v2(ctypes.byref(desc), ctypes.byref(cb3), ctypes.byref(vtq),
                                   _fake(k) if k else None, _fake(v) if v else None, 1, seq_new, None,
                                   _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), None, None)

    d3 = tq.kv_desc(2, 2, 128, 64, 3, 3)
    assert enc(d3, tq.make_codebook(3)) == _lib.TQ_ERR_INVALID_ARG       # V needs the doubled codebook
    assert enc(tq.kv_desc(2, 2, 128, 64, 3, 4), tq.make_codebook(4)) == _lib.TQ_ERR_UNSUPPORTED  # rate 4
    assert enc(d3, tq.make_tcq_codebook(3), k=0, v=0) == _lib.TQ_ERR_INVALID_ARG
    assert enc(d3, tq.make_tcq_codebook(3), v=GOOD + 8) == _lib.TQ_ERR_INVALID_ARG
    assert enc(d3, tq.make_tcq_codebook(3), seq_new=0) == _lib.TQ_OK            # no-op

    def dec(desc, vtq, wsb=None):
        need = tq.decode_workspace_size(desc, 8)
        return lib.tq_decode_attention_v2(ctypes.byref(desc), ctypes.byref(cb3), ctypes.byref(vtq), 8,
                                          _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                          _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD),
                                          need if wsb is None else wsb, None, None)

    d2 = tq.kv_desc(2, 2, 128, 64, 3, 2)
    assert dec(d2, tq.make_codebook(2)) == _lib.TQ_ERR_INVALID_ARG
    assert dec(tq.kv_desc(2, 2, 128, 64, 3, 4), tq.make_codebook(4)) == _lib.TQ_ERR_UNSUPPORTED
    assert dec(d2, tq.make_tcq_codebook(2), wsb=16) == _lib.TQ_ERR_WORKSPACE


def test_multi_token_v3_v2_reject_bad_arguments_without_launch():
    lib = tq.lib()
    d = tq.kv_desc(2, 2, 128, 64, 3, 2)
    cb3, cb2, vtq = tq.make_codebook(3), tq.make_codebook(2), tq.make_tcq_codebook(2)

    def v3(n_q, vo, wsb=None):
        need = tq.decode_workspace_size(d, 8 * max(n_q, 1)) if wsb is None else wsb
        return lib.tq_decode_attention_multi_v3(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(cb2), 8, n_q,
                                                _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                                _fake(GOOD), ctypes.byref(vo), _fake(GOOD), 0.1, 0.0, _fake(GOOD),
                                                _fake(GOOD), need, None, None)

    def v2(n_q, vcb, wsb=None):
        need = tq.decode_workspace_size(d, 8 * max(n_q, 1)) if wsb is None else wsb
        return lib.tq_decode_attention_multi_v2(ctypes.byref(d), ctypes.byref(cb3), ctypes.byref(vcb), 8, n_q,
                                                _fake(GOOD), 1, _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                                _fake(GOOD), _fake(GOOD), 0.1, 0.0, _fake(GOOD), _fake(GOOD),
                                                need, None, None)

    for n_q in (0, _lib.TQ_MAX_QUERY_TOKENS + 1):
        assert v3(n_q, _vo()) == _lib.TQ_ERR_INVALID_ARG
        assert v2(n_q, vtq) == _lib.TQ_ERR_INVALID_ARG
    assert v3(4, _vo(k=17)) == _lib.TQ_ERR_INVALID_ARG                       # the v3 checks
    assert v2(4, cb2) == _lib.TQ_ERR_INVALID_ARG                             # V needs the doubled codebook
    # the workspace must be sized for q_heads * n_q
    assert v3(4, _vo(), wsb=tq.decode_workspace_size(d, 8)) == _lib.TQ_ERR_WORKSPACE
    assert v2(4, vtq, wsb=tq.decode_workspace_size(d, 8)) == _lib.TQ_ERR_WORKSPACE

