"""The allocation-free decode entry point (tq_decode_attention_noalloc).

It serves callers that are not allowed to allocate device memory, so it takes
its scratch from an array built into the library instead of a workspace.  The
test calls it through the C ABI twice in a row and checks each result against
tq_decode_attention on the same inputs.  The file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import quantized_decode_attention_tq_b200 as tq
from quantized_decode_attention_tq_b200 import _lib, inputs

from ._parity import DECODE_REL_TOL, gpu_encode, rel_err, to_dev, torch_mod

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,sparse", [("gqa", 0.0), ("ragged", 3e-3)])
def test_noalloc_matches_workspace_entry_point(name, sparse):
    torch = torch_mod()
    w = inputs.make(name, batch=2, seq=700)
    cache, kcb, vcb = gpu_encode(w)
    q = to_dev(w.q)
    lens = to_dev(w.seq_lens.astype(np.int32))
    out_ref = torch.empty(w.batch, w.q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    ws = tq.alloc_workspace(cache.desc, w.q_heads, sparse)
    tq.decode_attention(cache, kcb, vcb, q, lens, w.scale, out_ref, ws, sparse_thr=sparse)
    torch.cuda.synchronize()
    ref = out_ref.cpu().numpy()
    for _ in range(2):  # two calls in a row share the built-in scratch
        out = torch.full_like(out_ref, float("nan"))
        tq.decode_attention_noalloc(cache, kcb, vcb, q, lens, w.scale, out, sparse_thr=sparse)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_err(got, ref) <= DECODE_REL_TOL


def test_noalloc_rejects_requests_beyond_the_scratch_limit():
    lib = tq.lib()
    desc = tq.kv_desc(64, 8, 256, 65536, 3, 3)        # sparse score buffer alone: 1 GiB
    need = tq.decode_workspace_size(desc, 32, 1e-5)
    assert need > _lib.TQ_NOALLOC_SCRATCH_BYTES
    cb = tq.make_codebook(3)
    fake = ctypes.c_void_p(0x7f0000000000)
    st = lib.tq_decode_attention_noalloc(ctypes.byref(desc), ctypes.byref(cb), ctypes.byref(cb), 32,
                                         fake, 1, fake, fake, fake, fake, fake, 0.1, 1e-5, fake,
                                         None, None)
    assert st == _lib.TQ_ERR_SCRATCH_LIMIT
