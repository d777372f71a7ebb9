"""Shared helpers for the GPU parity tests: run the library through its C ABI,
bring the results back, and compare them with the oracle by the acceptance
rules (code match rate and boundary distance, fp16 norm midpoint rule,
decode relative max-abs error and reconstruction-SNR band)."""
from __future__ import annotations

import numpy as np

import quantized_decode_attention_tq_b200 as tq
from oracle import tq_oracle as O

# Acceptance bounds (fixed by the method's specification).
CODE_MATCH_MIN = 0.9999        # fraction of indices equal to the oracle's
BOUNDARY_TOL = 1e-5            # a mismatch must sit this close to a boundary
NORM_MIDPOINT_TOL = 1e-6       # relative distance to an fp16 rounding midpoint
DECODE_REL_TOL = 2e-3          # max|o_gpu - o_oracle| / max|o_oracle|
SNR_BAND_DB = 0.25             # |SNR_gpu - SNR_oracle| vs unquantised attention


def torch_mod():
    import torch
    return torch


def to_dev(a):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_encode(w, k=None, v=None, start_pos=None, seq_cap=None, status=None):
    """Encode workload ``w`` (numpy K/V) with the library; returns the cache."""
    torch = torch_mod()
    desc = tq.kv_desc(w.batch, w.kv_heads, w.head_dim, seq_cap or w.seq_cap, w.k_bits, w.v_bits,
                      w.sign_seed)
    cache = tq.alloc_cache(desc)
    kcb, vcb = tq.make_codebook(w.k_bits), tq.make_codebook(w.v_bits)
    kk = to_dev(w.k if k is None else k)
    vv = to_dev(w.v if v is None else v)
    sp = None if start_pos is None else to_dev(np.asarray(start_pos, dtype=np.int32))
    tq.encode_kv(cache, kcb, vcb, kk, vv, start_pos=sp, status=status)
    torch.cuda.synchronize()
    return cache, kcb, vcb


def host(cache):
    return (cache.k_codes.cpu().numpy(), cache.k_norms.cpu().numpy().view(np.float16),
            cache.v_codes.cpu().numpy(), cache.v_norms.cpu().numpy().view(np.float16))


def fp16_midpoint_distance(n64: np.ndarray) -> np.ndarray:
    """Relative distance of fp64 values to the nearest fp16 rounding midpoint."""
    n64 = np.asarray(n64, dtype=np.float64)
    lo = n64.astype(np.float16)
    lo = np.where(lo.astype(np.float64) > n64, np.nextafter(lo, np.float16(-np.inf)), lo)
    hi = np.nextafter(lo, np.float16(np.inf))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) / 2
    return np.abs(n64 - mid) / np.maximum(np.abs(n64), 1e-300)


def check_norms(gpu_n: np.ndarray, x: np.ndarray):
    """Bit-equal fp16 norms, or 1 ulp apart where the fp64 norm is within
    NORM_MIDPOINT_TOL of an fp16 rounding midpoint."""
    nb = x.shape[-1] // 128
    n64 = np.sqrt(np.sum(x.astype(np.float64).reshape(*x.shape[:-1], nb, 128) ** 2, axis=-1))
    want = n64.astype(np.float16)
    diff = gpu_n.view(np.uint16).astype(np.int64) - want.view(np.uint16).astype(np.int64)
    bad = diff != 0
    if np.any(bad):
        assert np.all(np.abs(diff[bad]) == 1), "norm off by more than one fp16 ulp"
        assert np.all(fp16_midpoint_distance(n64[bad]) <= NORM_MIDPOINT_TOL), "norm mismatch away from a midpoint"
    return int(np.sum(bad))


def check_codes(gpu_codes: np.ndarray, x: np.ndarray, bits: int, signs: np.ndarray):
    """Code match rate >= CODE_MATCH_MIN; every mismatch adjacent and within
    BOUNDARY_TOL of the boundary between the two indices (oracle's u)."""
    _, t32 = O.codebook_f32(bits)
    _, _, u = O.encode(x, signs, bits, t32)
    want = O.quantize(u, t32)
    got = O.unpack_codes(gpu_codes, bits)
    mism = got != want
    n_bad = int(np.sum(mism))
    rate = 1.0 - n_bad / want.size
    assert rate >= CODE_MATCH_MIN, f"code match rate {rate}"
    if n_bad:
        g, w_, uu = got[mism], want[mism], u[mism]
        assert np.all(np.abs(g - w_) == 1), "non-adjacent code mismatch"
        tb = t32.astype(np.float64)[np.minimum(g, w_)]
        assert np.all(np.abs(uu - tb) <= BOUNDARY_TOL), "code mismatch away from a boundary"
    return n_bad, rate


def rel_err(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def snr_db(o, ref):
    return float(10 * np.log10(np.sum(ref ** 2) / max(np.sum((o - ref) ** 2), 1e-300)))


def gpu_decode(cache, kcb, vcb, q, seq_lens, scale, sparse_thr=0.0, status=None, workspace=None,
               reps=1):
    torch = torch_mod()
    qd = to_dev(q)
    lens = to_dev(np.asarray(seq_lens, dtype=np.int32))
    out = torch.full((q.shape[0], q.shape[1], q.shape[2]), float("nan"), dtype=torch.float32,
                     device="cuda")
    ws = workspace if workspace is not None else tq.alloc_workspace(cache.desc, q.shape[1], sparse_thr)
    for _ in range(reps):
        tq.decode_attention(cache, kcb, vcb, qd, lens, scale, out, ws, sparse_thr=sparse_thr,
                            status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), ws


SPARSE_BAND = 1e-2             # |ln(w / thr)| below this: either gate decision is correct


def sparse_flip_bound(q, kc, kn, vc, vn, seq_lens, scale, k_bits, v_bits, thr, seed=0):
    """Per-output bound on what gating decisions near the threshold can move.

    The sparse-V gate is discontinuous: a position whose normalised weight is
    within rounding of the threshold may be kept by one implementation and
    dropped by another, and both outputs are correct.  Positions with
    |ln(w_t / thr)| < SPARSE_BAND (fp64 oracle weights) are such ambiguous
    ones; flipping them changes output element d of head h by at most
    sum_t w_t |v~_t[d]|.  SPARSE_BAND is ~10x the score error of fp16 query
    and codeword rounding on these workloads.
    """
    s = O.sign_vector(seed)
    kt = O.dequantize(kc, kn, k_bits, O.codebook_f32(k_bits)[0], s)
    vt = O.dequantize(vc, vn, v_bits, O.codebook_f32(v_bits)[0], s)
    ws = O.attention_weights(q, kt, seq_lens, scale)
    group = q.shape[1] // kc.shape[1]
    bound = np.zeros(q.shape, dtype=np.float64)
    n_amb = 0
    for (b, h), w in ws.items():
        n = int(seq_lens[b])
        if n == 0 or thr <= 0:
            continue
        amb = np.abs(np.log(np.maximum(w, 1e-300) / thr)) < SPARSE_BAND
        n_amb += int(np.sum(amb))
        bound[b, h] = w[amb] @ np.abs(vt[b, h // group, :n][amb])
    return bound, n_amb


def check_decode(o_gpu, o_ref, bound=None):
    """max|o_gpu - o_ref| <= DECODE_REL_TOL * max|o_ref|, widened elementwise
    by the sparse gate's ambiguity bound when one is given."""
    scale = max(np.max(np.abs(o_ref)), 1e-300)
    allowed = DECODE_REL_TOL * scale + (0.0 if bound is None else bound)
    excess = np.abs(o_gpu - o_ref) - allowed
    assert np.all(excess <= 0), f"decode error {np.max(np.abs(o_gpu - o_ref)) / scale:.3e} beyond bound"
    if bound is None:
        return rel_err(o_gpu, o_ref)
    return float(np.max(np.maximum(np.abs(o_gpu - o_ref) - bound, 0)) / scale)


def oracle_decode(q, kc, kn, vc, vn, seq_lens, scale, k_bits, v_bits, sparse_thr, seed=0):
    kcent, _ = O.codebook_f32(k_bits)
    vcent, _ = O.codebook_f32(v_bits)
    return O.decode_rotated(q.astype(np.float64), kc, kn, vc, vn, seq_lens, scale, k_bits, v_bits,
                            kcent, vcent, O.sign_vector(seed), sparse_thr)
