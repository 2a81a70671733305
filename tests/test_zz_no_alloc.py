"""The allocation-free decode entry point, loki_decode_attention_noalloc.

Some callers cannot allocate device memory on the decode path (a runtime whose
device memory plan is fixed at start-up, or one that cannot accept the device
synchronisation cudaMalloc may imply).  For them the library offers a decode
call whose scratch is a fixed array in its own device code.  This file checks,
through the C ABI, that two such calls in a row give what the workspace entry
point gives on the same inputs, both for query groups of 4 heads (which need no
scratch) and of 8 heads (whose rotated queries go through the fixed array),
the latter also against the fp64 oracle; that a small-group shape whose
workspace would exceed the array still runs; and that a shape needing more
scratch than the array holds is refused before anything is launched.  It is
collected last so that a failure here stops a `-x` run only after every other
test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
from workloads import Workload
from workloads import generators as gen

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _lib():
    from sparse_decode_attention_loki_b200 import _lib
    return _lib


def _case(seed, n_q_heads=8, batch=2, seq_len=3001):
    w = Workload(name=f"noalloc-{seed}", dtype="bf16", batch=batch, n_q_heads=n_q_heads, n_kv_heads=2,
                 head_dim=128, seq_len=seq_len, d_f=0.25, k_f=0.25, generator="powerlaw", alpha=1.5, n_calib=512,
                 seed=seed)
    inp = gen.decode_inputs(w)
    import oracle
    P32 = np.ascontiguousarray(np.stack([oracle.pca_basis(c)[0] for c in inp["calib"]]), dtype=np.float32)
    return w, inp, P32


def _noalloc(lib, cache, S, q, P, d, k, out, idx):
    return lib.loki_decode_attention_noalloc(cache.desc(), S, q.shape[1], ctypes.c_void_p(q.data_ptr()),
                                             ctypes.c_void_p(P.data_ptr()), d, k, 0.0,
                                             ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("n_q_heads", [8, 16])
def test_noalloc_matches_workspace_entry_point_on_two_calls(n_q_heads):
    # 8 query heads over 2 KV heads (groups of 4): the decode kernel rotates
    # its own queries; 16 (groups of 8): the rotate kernel writes the rotated
    # queries into the fixed array and the decode kernel reads them back, so
    # a wrong array address or stale contents from the first call would show
    import oracle
    import sparse_decode_attention_loki_b200 as L
    lib = _lib().load()
    w, inp, P32 = _case(11 + n_q_heads, n_q_heads=n_q_heads)
    P = torch.from_numpy(P32).to(DEV)
    cache = L.LokiCache(w.batch, w.n_kv_heads, w.head_dim, w.seq_len, dtype=torch.bfloat16, device=DEV)
    L.loki_append(cache, 0, inp["keys"].to(DEV), inp["values"].to(DEV), P)
    K_hat = cache.k_hat.double().cpu().numpy()
    V = cache.v.double().cpu().numpy()
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    S, d, k = w.seq_len, w.d, w.k
    for call in range(2):   # two calls in a row on the shared scratch, different queries
        q = torch.randn((w.batch, w.n_q_heads, w.head_dim), generator=g, device=DEV).to(torch.bfloat16)
        ref_out, ref_idx = L.loki_decode_attention(cache, S, q, P, d, k)
        out = torch.empty_like(ref_out)
        idx = torch.empty_like(ref_idx)
        st = _noalloc(lib, cache, S, q, P, d, k, out, idx)
        assert st == 0, lib.loki_last_error()
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx), f"call {call}: index sets differ"
        err = float((out - ref_out).abs().max())
        assert err <= parity.TOL["bf16"], f"call {call}: max abs difference {err}"
        q64 = q.double().cpu().numpy()
        ref = oracle.loki_decode(q64, K_hat, V, P32.astype(np.float64), S, d, k)
        parity.check_decode(out.cpu().numpy(), idx.cpu().numpy(), ref, ref["q_hat"], K_hat, V,
                            oracle.default_scale(w.head_dim), "bf16")


def test_noalloc_runs_small_groups_whatever_their_workspace_size():
    # groups of up to 4 heads use no scratch, so a shape whose workspace
    # (B * Hkv * (G + 1) * D * 4 = 1024 * 2 * 5 * 512 bytes) exceeds the fixed
    # array is not refused
    import sparse_decode_attention_loki_b200 as L
    lib = _lib().load()
    w, inp, P32 = _case(3, n_q_heads=8, batch=1024, seq_len=40)
    assert L.loki_decode_workspace_size(L.LokiCache(w.batch, 2, 128, 40, dtype=torch.bfloat16, device=DEV), 40,
                                        8) > (4 << 20)
    P = torch.from_numpy(P32).to(DEV)
    cache = L.LokiCache(w.batch, w.n_kv_heads, w.head_dim, w.seq_len, dtype=torch.bfloat16, device=DEV)
    L.loki_append(cache, 0, inp["keys"].to(DEV), inp["values"].to(DEV), P)
    q = inp["q"].to(DEV)
    ref_out, ref_idx = L.loki_decode_attention(cache, 40, q, P, w.d, w.k)
    out, idx = torch.empty_like(ref_out), torch.empty_like(ref_idx)
    assert _noalloc(lib, cache, 40, q, P, w.d, w.k, out, idx) == 0, lib.loki_last_error()
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx)
    assert float((out - ref_out).abs().max()) <= parity.TOL["bf16"]


def test_noalloc_refuses_shapes_beyond_its_scratch():
    import sparse_decode_attention_loki_b200 as L
    lib = _lib().load()
    # B * Hkv * (G + 1) * D * 4 bytes of scratch: 128 * 8 * 9 * 128 * 4 > 4 MiB
    cache = L.LokiCache(128, 8, 128, 4, dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((128, 64, 128), dtype=torch.bfloat16, device=DEV)
    P = torch.zeros((8, 128, 128), dtype=torch.float32, device=DEV)
    with pytest.raises(L.LokiError) as e:
        L.loki_decode_attention_noalloc(cache, 4, q, P, 32, 2)
    assert e.value.status == _lib().LOKI_ERR_UNSUPPORTED
    assert "fixed scratch" in str(e.value)
    torch.cuda.synchronize()
