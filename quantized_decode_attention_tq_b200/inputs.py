"""Seeded synthetic workloads (numpy PCG64).  Holds no arithmetic of the method.

Recipe (one ``numpy.random.default_rng(seed)`` per workload; draws happen in
this order): sequence lengths, per-channel K scales, K, V, Q.  K and V are
drawn one batch entry at a time, in float32 (``standard_normal(dtype=
float32)``) or float64 for Student-t, then cast to the workload dtype.

Workloads (the five configurations the method is measured on):
  toy     decode: B1, Hq1/Hkv1, D128, S256, fp32 N(0,1) Q/K/V, K4/V4.
  encode  encode-only: B8, Hkv8, D128, S32768, fp16; K = N(0,1) times a
          per-(kv-head, channel) LogNormal(0,1) scale with round(0.02*D)
          channels per kv-head (chosen without replacement) scaled x20;
          V ~ Student-t(4); K3/V2.
  gqa     decode: B8, Hq32/Hkv8, D128, S32768, K3/V3, fp16 N(0,1) Q/K/V.
  long    decode: B1, Hq32/Hkv8, D128, S131072, K4/V2, fp16 N(0,1) Q/K/V,
          sparse-V threshold 1e-6 (measured on and off).
  ragged  decode: B4, lengths uniform in [16384, 65536], seq_cap 65536,
          Hq16/Hkv4, D256, K3/V2, fp16 N(0,1) Q/K/V, sparse-V threshold 1e-5.
Every decode workload uses softmax scale 1/sqrt(D) and sign seed 0.

``dist="outlier_v"`` gives any decode workload V with outlier channels (the
case the v3 format is for): K ~ N(0,1); V = N(0,1) times a per-(kv-head,
channel) LogNormal(0, 0.5) scale, round(0.05*D) channels per kv-head (chosen
without replacement) scaled x20.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

WORKLOADS = {
    "toy": dict(batch=1, q_heads=1, kv_heads=1, head_dim=128, seq=256, k_bits=4, v_bits=4,
                dtype="float32", dist="normal", sparse_thr=0.0),
    "encode": dict(batch=8, q_heads=8, kv_heads=8, head_dim=128, seq=32768, k_bits=3, v_bits=2,
                   dtype="float16", dist="outlier_t4", sparse_thr=0.0),
    "gqa": dict(batch=8, q_heads=32, kv_heads=8, head_dim=128, seq=32768, k_bits=3, v_bits=3,
                dtype="float16", dist="normal", sparse_thr=0.0),
    "long": dict(batch=1, q_heads=32, kv_heads=8, head_dim=128, seq=131072, k_bits=4, v_bits=2,
                 dtype="float16", dist="normal", sparse_thr=1e-6),
    "ragged": dict(batch=4, q_heads=16, kv_heads=4, head_dim=256, seq=65536, k_bits=3, v_bits=2,
                   dtype="float16", dist="normal", sparse_thr=1e-5, ragged=(16384, 65536)),
}


@dataclass
class Workload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    seq_cap: int
    k_bits: int
    v_bits: int
    dtype: str
    sparse_thr: float
    seq_lens: np.ndarray
    scale: float
    k: np.ndarray = field(repr=False, default=None)
    v: np.ndarray = field(repr=False, default=None)
    q: np.ndarray = field(repr=False, default=None)
    sign_seed: int = 0


def make(name: str, seed: int = 0, batch: int | None = None, seq: int | None = None,
         ragged: tuple | None = None, with_q: bool = True, dist: str | None = None) -> Workload:
    """Generate workload ``name`` (optionally with a reduced batch / length).

    ``seq`` overrides the cache length (and the ragged range is scaled to it
    unless ``ragged`` is given explicitly).  ``dist`` overrides the K/V
    distribution: "normal", "outlier_t4" (the encode-only workload's
    outlier-channel K and Student-t(4) V) or "outlier_v" (outlier-channel V)
    at the workload's own shapes.
    """
    cfg = dict(WORKLOADS[name])
    if dist is not None:
        assert dist in ("normal", "outlier_t4", "outlier_v"), dist
        cfg["dist"] = dist
    bsz = batch if batch is not None else cfg["batch"]
    seq_cap = seq if seq is not None else cfg["seq"]
    rng = np.random.default_rng(seed)
    d, hkv, hq = cfg["head_dim"], cfg["kv_heads"], cfg["q_heads"]
    dt = np.dtype(cfg["dtype"])

    # 1. lengths
    rr = ragged if ragged is not None else cfg.get("ragged")
    if rr is not None:
        if seq is not None and ragged is None:
            lo = max(1, int(round(rr[0] * seq_cap / cfg["seq"])))
            rr = (lo, seq_cap)
        lens = rng.integers(rr[0], rr[1], size=bsz, endpoint=True).astype(np.int32)
    else:
        lens = np.full(bsz, seq_cap, dtype=np.int32)

    # 2. per-channel K scales (outlier_t4), then V scales (outlier_v)
    kscale = None
    if cfg["dist"] == "outlier_t4":
        kscale = rng.lognormal(0.0, 1.0, size=(hkv, d))
        n_out = int(round(0.02 * d))
        for h in range(hkv):
            idx = rng.choice(d, size=n_out, replace=False)
            kscale[h, idx] *= 20.0
    vscale = None
    if cfg["dist"] == "outlier_v":
        vscale = rng.lognormal(0.0, 0.5, size=(hkv, d))
        n_out = int(round(0.05 * d))
        for h in range(hkv):
            idx = rng.choice(d, size=n_out, replace=False)
            vscale[h, idx] *= 20.0

    # 3. K, 4. V  (one batch entry at a time)
    k = np.empty((bsz, hkv, seq_cap, d), dtype=dt)
    v = np.empty((bsz, hkv, seq_cap, d), dtype=dt)
    for b in range(bsz):
        kb = rng.standard_normal((hkv, seq_cap, d), dtype=np.float32)
        if kscale is not None:
            kb *= kscale[:, None, :].astype(np.float32)
        k[b] = kb.astype(dt)
    for b in range(bsz):
        if cfg["dist"] == "outlier_t4":
            v[b] = rng.standard_t(4.0, size=(hkv, seq_cap, d)).astype(dt)
        else:
            vb = rng.standard_normal((hkv, seq_cap, d), dtype=np.float32)
            if vscale is not None:
                vb *= vscale[:, None, :].astype(np.float32)
            v[b] = vb.astype(dt)

    # 5. Q
    q = None
    if with_q:
        q = rng.standard_normal((bsz, hq, d), dtype=np.float32).astype(dt)

    return Workload(name=name, batch=bsz, q_heads=hq, kv_heads=hkv, head_dim=d, seq_cap=seq_cap,
                    k_bits=cfg["k_bits"], v_bits=cfg["v_bits"], dtype=cfg["dtype"],
                    sparse_thr=cfg["sparse_thr"], seq_lens=lens, scale=1.0 / math.sqrt(d),
                    k=k, v=v, q=q)
