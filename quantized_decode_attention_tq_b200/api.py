"""Thin Python binding over the C ABI (include/tq.h).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the encoder and of decode attention runs in the
library's sm_100a kernels.  There is no fallback path.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np

from ._lib import VOutliers as VOutliers_c
from ._lib import (TQ_ERR_DEVICE_BOUNDS, TQ_F16, TQ_F32, TQ_OK, Codebook, KVDesc, TQError, check,
                   lib)


def make_codebook(bits: int) -> Codebook:
    """Lloyd-Max codebook of N(0,1) with 2^bits levels (host, synchronous)."""
    cb = Codebook()
    check("tq_make_codebook", lib().tq_make_codebook(bits, ctypes.byref(cb)))
    return cb


def codebook_arrays(cb: Codebook):
    levels = 1 << cb.bits
    return (np.array(cb.centroids[:levels], dtype=np.float32),
            np.array(cb.boundaries[:levels - 1], dtype=np.float32))


def sign_vector(seed: int) -> np.ndarray:
    out = (ctypes.c_int8 * 128)()
    check("tq_sign_vector", lib().tq_sign_vector(seed, out))
    return np.frombuffer(out, dtype=np.int8).copy()


def kv_desc(batch, kv_heads, head_dim, seq_cap, k_bits, v_bits, sign_seed=0) -> KVDesc:
    return KVDesc(batch, kv_heads, head_dim, seq_cap, sign_seed, k_bits, v_bits)


@dataclass
class Cache:
    """One layer's packed cache: codes uint8, norms fp16 stored in int16 tensors."""
    desc: KVDesc
    k_codes: "object"
    k_norms: "object"
    v_codes: "object"
    v_norms: "object"


def cache_shapes(desc: KVDesc):
    nb = desc.head_dim // 128
    base = (desc.batch, desc.kv_heads, desc.seq_cap, nb)
    return {"k_codes": base + (16 * desc.k_bits,), "k_norms": base,
            "v_codes": base + (16 * desc.v_bits,), "v_norms": base}


def alloc_cache(desc: KVDesc, device="cuda") -> Cache:
    import torch
    s = cache_shapes(desc)
    return Cache(desc,
                 torch.zeros(s["k_codes"], dtype=torch.uint8, device=device),
                 torch.zeros(s["k_norms"], dtype=torch.int16, device=device),
                 torch.zeros(s["v_codes"], dtype=torch.uint8, device=device),
                 torch.zeros(s["v_norms"], dtype=torch.int16, device=device))


def _ptr(t, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return TQ_F16
    if t.dtype == torch.float32:
        return TQ_F32
    raise ValueError(f"unsupported dtype {t.dtype}: fp16 or fp32")


def encode_kv(cache: Cache, k_cb: Codebook, v_cb: Codebook, k=None, v=None, start_pos=None,
              status=None, stream=None) -> None:
    """Encode K/V rows [B, Hkv, seq_new, D] into the cache (tq_encode_kv)."""
    src = k if k is not None else v
    if src is None:
        raise ValueError("k or v is required")
    if k is not None and v is not None and (k.shape != v.shape or k.dtype != v.dtype):
        raise ValueError("k and v must have the same shape and dtype")
    seq_new = src.shape[2]
    st = lib().tq_encode_kv(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb),
        _ptr(k, "k"), _ptr(v, "v"), _dtype_code(src), seq_new, _ptr(start_pos, "start_pos"),
        _ptr(cache.k_codes, "k_codes") if k is not None else None,
        _ptr(cache.k_norms, "k_norms") if k is not None else None,
        _ptr(cache.v_codes, "v_codes") if v is not None else None,
        _ptr(cache.v_norms, "v_norms") if v is not None else None,
        _ptr(status, "status"), _stream(stream))
    check("tq_encode_kv", st)


def decode_workspace_size(desc: KVDesc, q_heads: int, sparse_thr: float = 0.0) -> int:
    return int(lib().tq_decode_workspace_size(ctypes.byref(desc), q_heads, sparse_thr))


def alloc_workspace(desc: KVDesc, q_heads: int, sparse_thr: float = 0.0, device="cuda"):
    """A zeroed workspace (the library requires zero before first use)."""
    import torch
    n = decode_workspace_size(desc, q_heads, sparse_thr)
    if n == 0:
        raise ValueError("invalid decode configuration")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_attention(cache: Cache, k_cb: Codebook, v_cb: Codebook, q, seq_lens, scale: float,
                     out, workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """Single-token decode attention over the packed cache (tq_decode_attention)."""
    q_heads = q.shape[1]
    st = lib().tq_decode_attention(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb), q_heads,
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention", st)
    return out


def decode_attention_multi(cache: Cache, k_cb: Codebook, v_cb: Codebook, q, seq_lens, scale: float,
                           out, workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """n_q query tokens per sequence, the last n_q positions, each seeing the
    positions up to its own (tq_decode_attention_multi).  q, out: [B, n_q, Hq, D];
    workspace: alloc_workspace(desc, Hq * n_q, sparse_thr)."""
    n_q, q_heads = q.shape[1], q.shape[2]
    st = lib().tq_decode_attention_multi(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb), q_heads, n_q,
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention_multi", st)
    return out


def decode_step(cache: Cache, k_cb: Codebook, v_cb: Codebook, q, k_new, v_new, seq_lens, scale: float,
                out, workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """One decode step (tq_decode_step): write each sequence's new K/V row
    [B, Hkv, D] at position seq_lens[b] - 1, then attend over the cache."""
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    q_heads = q.shape[1]
    st = lib().tq_decode_step(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb), q_heads,
        _ptr(q, "q"), _dtype_code(q), _ptr(k_new, "k_new"), _ptr(v_new, "v_new"), _dtype_code(k_new),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_step", st)
    return out


def decode_attention_noalloc(cache: Cache, k_cb: Codebook, v_cb: Codebook, q, seq_lens, scale: float,
                             out, sparse_thr: float = 0.0, status=None, stream=None):
    """Decode attention without a caller workspace (tq_decode_attention_noalloc).

    For callers that may not allocate device memory: the library's built-in
    64 MiB scratch array is used instead.  Calls must not overlap on the GPU.
    """
    q_heads = q.shape[1]
    st = lib().tq_decode_attention_noalloc(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb), q_heads,
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention_noalloc", st)
    return out


def read_device_status(status, stream=None) -> int:
    """The bits of a device status word (tq_read_device_status; synchronous).

    Returns the TQ_DEV_* bits that the kernels OR-ed into ``status`` (a
    one-element int32/uint32 CUDA tensor); 0 means no range error."""
    bits = ctypes.c_uint32(0)
    st = lib().tq_read_device_status(_ptr(status, "status"), ctypes.byref(bits), _stream(stream))
    if st not in (TQ_OK, TQ_ERR_DEVICE_BOUNDS):
        raise TQError("tq_read_device_status", st)
    return int(bits.value)


# ---- V v3: outlier-channel separation -------------------------------------

@dataclass
class VOutliers:
    """v3 side data of one layer: channels int32 [Hkv, k] (ascending) and the
    stored fp16 values [B, Hkv, seq_cap, kp] in an int16 tensor, kp = 8 for
    k <= 8 else 16."""
    k: int
    channels: "object"
    values: "object"

    def c_struct(self) -> VOutliers_c:
        return VOutliers_c(self.k, _ptr(self.channels, "channels"), _ptr(self.values, "values"))


def outlier_row(k: int) -> int:
    return 8 if k <= 8 else 16


def alloc_outliers(desc: KVDesc, channels) -> VOutliers:
    """VOutliers for `channels` (device int32 [Hkv, k]) with zeroed values."""
    import torch
    k = int(channels.shape[1])
    values = torch.zeros((desc.batch, desc.kv_heads, desc.seq_cap, outlier_row(k)), dtype=torch.int16,
                         device=channels.device)
    return VOutliers(k, channels, values)


def pick_outlier_channels(desc: KVDesc, v, k: int, stream=None):
    """The k channels of largest mean square per kv-head over v [B, Hkv, rows, D]
    (tq_pick_outlier_channels): device int32 [Hkv, k], ascending."""
    import torch
    ch = torch.empty((desc.kv_heads, k), dtype=torch.int32, device=v.device)
    st = lib().tq_pick_outlier_channels(ctypes.byref(desc), _ptr(v, "v"), _dtype_code(v), int(v.shape[2]), k,
                                        _ptr(ch, "channels"), _stream(stream))
    check("tq_pick_outlier_channels", st)
    return ch


def encode_kv_v3(cache: Cache, k_cb: Codebook, v_cb: Codebook, vo: VOutliers, k=None, v=None, start_pos=None,
                 status=None, stream=None) -> None:
    """encode_kv with the V side in v3 format (tq_encode_kv_v3)."""
    src = k if k is not None else v
    if src is None:
        raise ValueError("k or v is required")
    if k is not None and v is not None and (k.shape != v.shape or k.dtype != v.dtype):
        raise ValueError("k and v must have the same shape and dtype")
    vs = vo.c_struct()
    st = lib().tq_encode_kv_v3(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb),
        _ptr(k, "k"), _ptr(v, "v"), _dtype_code(src), src.shape[2], _ptr(start_pos, "start_pos"),
        _ptr(cache.k_codes, "k_codes") if k is not None else None,
        _ptr(cache.k_norms, "k_norms") if k is not None else None,
        _ptr(cache.v_codes, "v_codes") if v is not None else None,
        _ptr(cache.v_norms, "v_norms") if v is not None else None,
        ctypes.byref(vs), _ptr(status, "status"), _stream(stream))
    check("tq_encode_kv_v3", st)


def decode_attention_v3(cache: Cache, k_cb: Codebook, v_cb: Codebook, vo: VOutliers, q, seq_lens, scale: float,
                        out, workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """decode_attention over a v3 V cache (tq_decode_attention_v3)."""
    vs = vo.c_struct()
    st = lib().tq_decode_attention_v3(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb), q.shape[1],
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"), ctypes.byref(vs),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention_v3", st)
    return out


def decode_attention_multi_v3(cache: Cache, k_cb: Codebook, v_cb: Codebook, vo: VOutliers, q, seq_lens,
                              scale: float, out, workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """decode_attention_multi over a v3 V cache (tq_decode_attention_multi_v3).
    q, out: [B, n_q, Hq, D]; workspace: alloc_workspace(desc, Hq * n_q, sparse_thr)."""
    vs = vo.c_struct()
    n_q, q_heads = q.shape[1], q.shape[2]
    st = lib().tq_decode_attention_multi_v3(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_cb), q_heads, n_q,
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"), ctypes.byref(vs),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention_multi_v3", st)
    return out


# ---- V v2: trellis-coded quantisation --------------------------------------

def make_tcq_codebook(v_bits: int) -> Codebook:
    """The doubled codebook of the v2 format: the 2^(v_bits+1)-level Lloyd-Max
    quantiser of N(0,1)."""
    return make_codebook(v_bits + 1)


def encode_kv_v2(cache: Cache, k_cb: Codebook, v_tcq: Codebook, k=None, v=None, start_pos=None, status=None,
                 stream=None) -> None:
    """encode_kv with the V side in v2 format (tq_encode_kv_v2)."""
    src = k if k is not None else v
    if src is None:
        raise ValueError("k or v is required")
    if k is not None and v is not None and (k.shape != v.shape or k.dtype != v.dtype):
        raise ValueError("k and v must have the same shape and dtype")
    st = lib().tq_encode_kv_v2(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_tcq),
        _ptr(k, "k"), _ptr(v, "v"), _dtype_code(src), src.shape[2], _ptr(start_pos, "start_pos"),
        _ptr(cache.k_codes, "k_codes") if k is not None else None,
        _ptr(cache.k_norms, "k_norms") if k is not None else None,
        _ptr(cache.v_codes, "v_codes") if v is not None else None,
        _ptr(cache.v_norms, "v_norms") if v is not None else None,
        _ptr(status, "status"), _stream(stream))
    check("tq_encode_kv_v2", st)


def decode_attention_v2(cache: Cache, k_cb: Codebook, v_tcq: Codebook, q, seq_lens, scale: float, out,
                        workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """decode_attention over a v2 V cache (tq_decode_attention_v2)."""
    st = lib().tq_decode_attention_v2(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_tcq), q.shape[1],
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention_v2", st)
    return out


def decode_attention_multi_v2(cache: Cache, k_cb: Codebook, v_tcq: Codebook, q, seq_lens, scale: float, out,
                              workspace, sparse_thr: float = 0.0, status=None, stream=None):
    """decode_attention_multi over a v2 V cache (tq_decode_attention_multi_v2).
    q, out: [B, n_q, Hq, D]; workspace: alloc_workspace(desc, Hq * n_q, sparse_thr)."""
    n_q, q_heads = q.shape[1], q.shape[2]
    st = lib().tq_decode_attention_multi_v2(
        ctypes.byref(cache.desc), ctypes.byref(k_cb), ctypes.byref(v_tcq), q_heads, n_q,
        _ptr(q, "q"), _dtype_code(q),
        _ptr(cache.k_codes, "k_codes"), _ptr(cache.k_norms, "k_norms"),
        _ptr(cache.v_codes, "v_codes"), _ptr(cache.v_norms, "v_norms"),
        _ptr(seq_lens, "seq_lens"), float(scale), float(sparse_thr), _ptr(out, "out"),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, "status"), _stream(stream))
    check("tq_decode_attention_multi_v2", st)
    return out
