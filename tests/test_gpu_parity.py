"""Parity of the CUDA path (through the C ABI of libloki.so) with the fp64
oracle, on seeded synthetic inputs.

The cache contents the decode kernels read are the oracle's rotated keys
(oracle.rotate_keys, rounded to the cache dtype) uploaded as they are, so that
both sides score exactly the same K_hat; the GPU append kernel is checked on its
own against the exact rotation.
"""
import contextlib
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
import parity
from workloads import Workload, get_workload, mistral_sweep_points
from workloads import generators as gen

pytestmark = pytest.mark.gpu

DEV = "cuda"
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def L():
    import sparse_decode_attention_loki_b200 as lib
    return lib


@contextlib.contextmanager
def forced_cluster(n):
    """Launches inside use n CTAs (dense) or key-stream units (Loki) per row
    (loki_set_launch_override); None leaves the planner's choice."""
    from sparse_decode_attention_loki_b200 import _lib
    _lib.check(_lib.load().loki_set_launch_override(int(n or 0)))
    try:
        yield
    finally:
        _lib.check(_lib.load().loki_set_launch_override(0))


def small_workload(dtype, D, G, S, Hkv=2, B=2, generator="powerlaw", seed=77):
    return Workload(name=f"small-{dtype}-D{D}-G{G}-S{S}", dtype=dtype, batch=B, n_q_heads=Hkv * G,
                    n_kv_heads=Hkv, head_dim=D, seq_len=S, d_f=0.25, k_f=0.25, generator=generator,
                    alpha=1.5, n_calib=max(4 * D, 512), seed=seed)


def basis(w):
    """P from the oracle's PCA of each head's calibration batch, as fp32."""
    return np.ascontiguousarray(np.stack([oracle.pca_basis(gen.calibration_keys(w, g))[0]
                                          for g in range(w.n_kv_heads)]), dtype=np.float32)


def upload_case(w, inp, P32, capacity=None):
    """Cache filled with the oracle's rotated keys; returns (cache, K_hat64, V64, q_dev, P_dev)."""
    S = inp["seq_len"]
    cap = capacity or S
    K_hat = oracle.rotate_keys(inp["keys64"], P32.astype(np.float64), w.dtype)
    td = TORCH_DTYPE[w.dtype]
    cache = L().LokiCache(len(inp["batches"]), w.n_kv_heads, w.head_dim, cap, dtype=td, device=DEV)
    cache.k_hat.zero_()
    cache.v.zero_()
    cache.k_hat[:, :, :S] = torch.from_numpy(K_hat).to(td).to(DEV)
    cache.v[:, :, :S] = inp["values"].to(DEV)
    return cache, K_hat, inp["values64"], inp["q"].to(DEV), torch.from_numpy(P32).to(DEV)


def run_decode(w, S, d, k, ncta=None, scale=0.0, inp=None, P32=None, capacity=None):
    inp = inp or gen.decode_inputs(w, seq_len=S)
    P32 = basis(w) if P32 is None else P32
    cache, K_hat, V, q, P = upload_case(w, inp, P32, capacity)
    with forced_cluster(ncta):
        out, idx = L().loki_decode_attention(cache, S, q, P, d, k, scale=scale)
    torch.cuda.synchronize()
    sc = None if scale <= 0 else scale
    ref = oracle.loki_decode(inp["q64"], K_hat, V, P32.astype(np.float64), S, d, k, scale=sc)
    return out.cpu().numpy(), idx.cpu().numpy(), ref, K_hat, V, inp, P32, cache, q, P


# ----------------------------------------------------------------------------- append
TC_MIN_VECTORS = 256   # bf16 appends of at least this many vectors per KV head run on the tensor cores


@pytest.mark.parametrize("dtype,D,n_new,pos,B,Hkv", [
    ("bf16", 128, 1, 0, 2, 3),
    ("bf16", 128, 37, 5, 3, 2),
    ("bf16", 128, 300, 100, 2, 2),     # tensor cores: 600 vectors, 5 tiles (ragged)
    ("bf16", 128, 150, 3, 3, 5),       # tensor cores: 450 vectors
    ("bf16", 128, 2048, 0, 1, 2),      # tensor cores: 16 full tiles
    ("bf16", 64, 9, 3, 1, 4),
    ("bf16", 64, 257, 11, 1, 3),       # tensor cores, D = 64
    ("f32", 64, 1, 7, 2, 2),
    ("f32", 128, 41, 0, 2, 3),
    ("f32", 128, 700, 2, 1, 2),        # fp32 caches stay on the CUDA cores
])
def test_append_matches_exact_rotation(dtype, D, n_new, pos, B, Hkv):
    w = small_workload(dtype, D, 1, n_new, Hkv=Hkv, B=B)
    inp = gen.decode_inputs(w, seq_len=n_new)
    P32 = basis(w)
    cap = pos + n_new + 11
    td = TORCH_DTYPE[dtype]
    cache = L().LokiCache(B, Hkv, D, cap, dtype=td, device=DEV)
    cache.k_hat.fill_(7.0)
    cache.v.fill_(-3.0)
    L().loki_append(cache, pos, inp["keys"].to(DEV), inp["values"].to(DEV), torch.from_numpy(P32).to(DEV))
    torch.cuda.synchronize()
    kh = cache.k_hat.to(torch.float64).cpu().numpy()
    vv = cache.v.to(torch.float64).cpu().numpy()
    tc = dtype == "bf16" and B * n_new >= TC_MIN_VECTORS
    st = parity.check_append(kh[:, :, pos:pos + n_new], inp["keys64"], P32.astype(np.float64), dtype,
                             tensor_core=tc)
    if tc:
        n = ctypes.c_uint32(0)
        L()._lib.check(L().load_library().loki_device_error_count(ctypes.byref(n)))
        assert n.value == 0, "a bounded wait of the tensor-core append timed out"
    if dtype == "bf16":
        assert st["mismatch"] <= 0.05 * st["n"]   # sanity: most values round exactly like the oracle
    np.testing.assert_array_equal(vv[:, :, pos:pos + n_new], inp["values64"])
    # nothing outside [pos, pos + n_new) is touched
    assert np.all(kh[:, :, :pos] == 7.0) and np.all(kh[:, :, pos + n_new:] == 7.0)
    assert np.all(vv[:, :, :pos] == -3.0) and np.all(vv[:, :, pos + n_new:] == -3.0)


def test_bulk_append_identity_basis_is_a_copy():
    # the tensor-core path with P = I: the split terms are 1, 0, 0 and the
    # products exact, so the cache must hold the keys bit for bit
    w = small_workload("bf16", 128, 1, 1000)
    inp = gen.decode_inputs(w, seq_len=1000)
    P = torch.eye(128, dtype=torch.float32).expand(2, 128, 128).contiguous().to(DEV)
    cache = L().LokiCache(2, 2, 128, 1000, dtype=torch.bfloat16, device=DEV)
    L().loki_append(cache, 0, inp["keys"].to(DEV), inp["values"].to(DEV), P)
    torch.cuda.synchronize()
    assert torch.equal(cache.k_hat.cpu(), inp["keys"])
    assert torch.equal(cache.v.cpu(), inp["values"])


def test_append_identity_basis_is_a_copy():
    w = small_workload("bf16", 128, 1, 64)
    inp = gen.decode_inputs(w, seq_len=64)
    P = torch.eye(128, dtype=torch.float32).expand(2, 128, 128).contiguous().to(DEV)
    cache = L().LokiCache(2, 2, 128, 64, dtype=torch.bfloat16, device=DEV)
    L().loki_append(cache, 0, inp["keys"].to(DEV), inp["values"].to(DEV), P)
    torch.cuda.synchronize()
    assert torch.equal(cache.k_hat.cpu(), inp["keys"])


# ----------------------------------------------------------------------------- decode, small shapes
DECODE_CASES = [
    # dtype, D, G, S, d, k
    ("f32", 64, 1, 256, 16, 64),
    ("bf16", 128, 1, 1000, 32, 250),
    ("bf16", 128, 4, 3001, 64, 375),
    ("bf16", 64, 2, 777, 8, 100),
    ("f32", 128, 8, 513, 128, 512),
    ("bf16", 128, 1, 300, 1, 1),
    ("bf16", 128, 4, 2048, 16, 2047),
    ("bf16", 128, 1, 1500, 32, 1500),
    ("f32", 64, 4, 100, 3, 17),
    ("bf16", 128, 8, 4097, 33, 1024),
    ("f32", 128, 2, 1, 7, 1),
]


@pytest.mark.parametrize("ncta", [None, 1, 4, 16])
@pytest.mark.parametrize("dtype,D,G,S,d,k", DECODE_CASES)
def test_decode_matches_oracle(dtype, D, G, S, d, k, ncta):
    w = small_workload(dtype, D, G, S)
    out, idx, ref, K_hat, V, inp, P32, *_ = run_decode(w, S, d, k, ncta=ncta)
    parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, oracle.default_scale(D), dtype)


def test_tiny_fp32_workload():
    w = get_workload("tiny-fp32")
    out, idx, ref, K_hat, V, *_ = run_decode(w, w.seq_len, w.d, w.k)
    st = parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, oracle.default_scale(w.head_dim), w.dtype)
    assert st["swapped_rows"] == 0


def test_decode_explicit_scale_and_capacity():
    w = small_workload("bf16", 128, 4, 900)
    out, idx, ref, K_hat, V, *_ = run_decode(w, 900, 32, 200, scale=0.3, capacity=1500)
    parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, 0.3, "bf16")


@pytest.mark.parametrize("ncta", [1, 8])
def test_exact_ties_take_lowest_index(ncta):
    # identity basis, small-integer keys and queries: every score is an exact
    # integer on both sides, with many exact ties; the selection must match the
    # oracle exactly (lower index wins)
    rng = np.random.default_rng(5)
    B, Hkv, G, D, S, d, k = 2, 2, 2, 128, 2000, 16, 333
    keys = rng.integers(-2, 3, (B, Hkv, S, D)).astype(np.float64)
    vals = rng.standard_normal((B, Hkv, S, D))
    q = rng.integers(-1, 2, (B, Hkv * G, D)).astype(np.float64)
    P = np.ascontiguousarray(np.broadcast_to(np.eye(D, dtype=np.float32), (Hkv, D, D)))
    vt, v64 = gen.to_cache_dtype(vals, "bf16")
    kt, k64 = gen.to_cache_dtype(keys, "bf16")
    qt, q64 = gen.to_cache_dtype(q, "bf16")
    inp = dict(keys64=k64, values=vt, values64=v64, q=qt, q64=q64, batches=list(range(B)), seq_len=S)
    w = small_workload("bf16", D, G, S, Hkv=Hkv, B=B)
    out, idx, ref, K_hat, V, *_ = run_decode(w, S, d, k, ncta=ncta, inp=inp, P32=P)
    np.testing.assert_array_equal(idx, ref["idx"])
    parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, oracle.default_scale(D), "bf16")


@pytest.mark.parametrize("S,ncta", [(1234, None), (1234, 16), (15000, None), (15000, 1), (20000, 16)])
def test_zero_query_selects_first_k(S, ncta):
    # every score is equal: the selection is decided by the tie rule alone;
    # the longer rows put more candidate keys in one CTA than its exchange
    # slot holds, which takes the distributed refinement path
    w = small_workload("bf16", 128, 4, S)
    inp = gen.decode_inputs(w, seq_len=S)
    inp["q"] = torch.zeros_like(inp["q"])
    inp["q64"] = np.zeros_like(inp["q64"])
    k = 77 if S < 10000 else 3001
    out, idx, ref, K_hat, V, *_ = run_decode(w, S, 32, k, ncta=ncta, inp=inp)
    assert np.all(idx == np.arange(k, dtype=np.int32))
    for h in range(w.n_q_heads):
        np.testing.assert_allclose(out[:, h], V[:, h // 4, :k].mean(axis=1), atol=5e-3)


@pytest.mark.parametrize("S,k,ncta", [(6000, 600, None), (6000, 5000, None), (30000, 3000, 2), (30000, 15000, 2),
                                     (30000, 3000, 16)])
def test_select_lists_and_their_overflow(S, k, ncta):
    # the select keeps per-warp lists of the tokens at or above the first
    # digit's bucket; a large k overflows them (and the selection falls back
    # to sweeps over every key), on short rows (one CTA selects all) and long
    # ones (the cluster selects)
    w = small_workload("bf16", 128, 2, S, Hkv=2, B=1, seed=S + k)
    out, idx, ref, K_hat, V, *_ = run_decode(w, S, 32, k, ncta=ncta)
    parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, oracle.default_scale(128), "bf16")


def test_full_budget_equals_dense():
    w = small_workload("bf16", 128, 4, 700)
    out, idx, ref, K_hat, V, inp, P32, cache, q, P = run_decode(w, 700, 128, 700)
    dense = L().dense_decode_attention(cache, 700, q, P).cpu().numpy()
    ref_dense = oracle.dense_decode(inp["q64"], K_hat, V, P32.astype(np.float64), 700)
    parity.check_dense(dense, ref_dense, "bf16")
    parity.check_dense(out, ref_dense, "bf16")
    assert np.all(idx == np.arange(700))


# ----------------------------------------------------------------------------- workspace and score tiles
def test_workspace_needs_no_initialisation_and_is_shared_across_shapes():
    # one external workspace, filled with garbage first, shared by calls of
    # different caches, lengths, d and k: every call must match the oracle
    lib = L()
    ws = torch.randint(0, 256, (32 << 20,), dtype=torch.uint8, device=DEV)
    cases = [("bf16", 128, 4, 3001, 64, 375, 2, 2), ("bf16", 128, 1, 5000, 32, 1250, 4, 3),
             ("f32", 64, 2, 700, 16, 99, 1, 2), ("bf16", 128, 4, 3001, 8, 2999, 2, 2),
             ("bf16", 128, 8, 40000, 32, 5000, 1, 1)]
    for dtype, D, G, S, d, k, Hkv, B in cases:
        w = small_workload(dtype, D, G, S, Hkv=Hkv, B=B, seed=S + d)
        inp = gen.decode_inputs(w, seq_len=S)
        P32 = basis(w)
        cache, K_hat, V, q, P = upload_case(w, inp, P32)
        assert lib.loki_decode_workspace_size(cache, S, w.n_q_heads) <= ws.numel()
        out, idx = lib.loki_decode_attention(cache, S, q, P, d, k, workspace=ws)
        torch.cuda.synchronize()
        ref = oracle.loki_decode(inp["q64"], K_hat, V, P32.astype(np.float64), S, d, k)
        parity.check_decode(out.cpu().numpy(), idx.cpu().numpy(), ref, ref["q_hat"], K_hat, V,
                            oracle.default_scale(D), dtype)


@pytest.mark.parametrize("S,B,Hkv,G", [(20000, 1, 2, 1), (4096, 16, 8, 4), (257, 3, 2, 2), (70001, 1, 1, 4),
                                       (9000, 3, 2, 8)])
def test_cluster_shapes_and_ragged_chunks(S, B, Hkv, G):
    # rows split over clusters of several CTAs with a ragged last chunk, grids
    # of several waves, and a row longer than one CTA can hold
    w = small_workload("bf16", 128, G, S, Hkv=Hkv, B=B, seed=S)
    rot, ncta, ctas, short_kernel = L().loki_decode_launch_shape(
        L().LokiCache(B, Hkv, 128, S, dtype=torch.bfloat16, device=DEV), S, Hkv * G, max(1, S // 8))
    assert rot == (B * Hkv * 4 if G == 8 else 0) and ctas == B * Hkv * ncta
    assert short_kernel in (0, 1) and (S <= 8192 or short_kernel == 0)
    assert ncta in (1, 2, 4, 8, 16) and ncta * 24576 >= S
    out, idx, ref, K_hat, V, *_ = run_decode(w, S, 32, max(1, S // 8))
    parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, oracle.default_scale(128), "bf16")


@pytest.mark.parametrize("S,B,Hkv,G", [(6144, 1, 8, 4), (5120, 4, 8, 4), (4608, 2, 2, 8), (8192, 1, 4, 1)])
def test_rows_between_4096_and_8192_tokens(S, B, Hkv, G):
    # the short-row kernel takes these only where its shared memory (the whole
    # row's keys in every CTA) keeps the long-row kernel's CTAs per SM, so both
    # kernels serve rows of this length; either way the selection and the
    # attention must match the oracle
    w = small_workload("bf16", 128, G, S, Hkv=Hkv, B=B, seed=S + G)
    rot, ncta, ctas, short_kernel = L().loki_decode_launch_shape(
        L().LokiCache(B, Hkv, 128, S, dtype=torch.bfloat16, device=DEV), S, Hkv * G, S // 4)
    assert short_kernel in (0, 1) and ctas == B * Hkv * ncta
    out, idx, ref, K_hat, V, *_ = run_decode(w, S, 32, S // 4)
    parity.check_decode(out, idx, ref, ref["q_hat"], K_hat, V, oracle.default_scale(128), "bf16")


def test_repeated_calls_are_identical():
    w = small_workload("bf16", 128, 4, 3001)
    out, idx, ref, K_hat, V, inp, P32, cache, q, P = run_decode(w, 3001, 64, 375)
    for _ in range(3):
        o2, i2 = L().loki_decode_attention(cache, 3001, q, P, 64, 375)
        torch.cuda.synchronize()
        assert np.array_equal(i2.cpu().numpy(), idx)
        assert np.array_equal(o2.cpu().numpy(), out)


# ----------------------------------------------------------------------------- Exact-TopK baseline and agreement
@pytest.mark.parametrize("rows,S,k", [(1, 10, 1), (5, 300, 7), (3, 5000, 1000), (2, 40000, 4096), (4, 8, 8)])
def test_jaccard_kernel_matches_oracle(rows, S, k):
    rng = np.random.default_rng(rows * 1000 + k)
    a = np.stack([np.sort(rng.choice(S, k, replace=False)) for _ in range(rows)]).astype(np.int32)
    b = np.stack([np.sort(rng.choice(S, k, replace=False)) for _ in range(rows)]).astype(np.int32)
    b[0] = a[0]  # identical sets
    if rows > 1 and 2 * k <= S:  # disjoint sets
        b[1] = np.sort(rng.choice(np.setdiff1d(np.arange(S), a[1]), k, replace=False))
    got = L().topk_jaccard(torch.from_numpy(a).to(DEV), torch.from_numpy(b).to(DEV)).cpu().numpy()
    # c / (2k - c) of two integers, correctly rounded to fp32 on both sides
    np.testing.assert_array_equal(got, oracle.topk_jaccard(a, b).astype(np.float32))


@pytest.mark.parametrize("dtype,G", [("bf16", 4), ("f32", 1)])
def test_exact_topk_baseline_and_agreement(dtype, G):
    # the Exact-TopK baseline is the decode with d = D; the agreement of Loki's
    # selection with it is the Jaccard similarity of the two index sets
    S, k = 3001, 375
    w = small_workload(dtype, 128, G, S)
    inp = gen.decode_inputs(w, seq_len=S)
    P32 = basis(w)
    o1, i1, ref1, K_hat, V, *_ = run_decode(w, S, 32, k, inp=inp, P32=P32)
    o2, i2, ref2, *_ = run_decode(w, S, 128, k, inp=inp, P32=P32)
    parity.check_decode(o1, i1, ref1, ref1["q_hat"], K_hat, V, oracle.default_scale(128), dtype)
    parity.check_decode(o2, i2, ref2, ref2["q_hat"], K_hat, V, oracle.default_scale(128), dtype)
    got = L().topk_jaccard(torch.from_numpy(i1).to(DEV), torch.from_numpy(i2).to(DEV)).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.topk_jaccard(i1, i2).astype(np.float32))
    if np.array_equal(i1, ref1["idx"]) and np.array_equal(i2, ref2["idx"]):
        np.testing.assert_array_equal(got, oracle.topk_jaccard(ref1["idx"], ref2["idx"]).astype(np.float32))
    assert np.all(got > 0.0) and np.all(got <= 1.0)


# ----------------------------------------------------------------------------- dense, small shapes
@pytest.mark.parametrize("ncta", [None, 1, 16])
@pytest.mark.parametrize("dtype,D,G,S", [
    ("f32", 64, 1, 256), ("bf16", 128, 1, 4096), ("bf16", 128, 4, 3001), ("f32", 128, 8, 77),
    ("bf16", 64, 2, 1), ("bf16", 128, 8, 1025),
])
def test_dense_matches_oracle(dtype, D, G, S, ncta):
    w = small_workload(dtype, D, G, S)
    inp = gen.decode_inputs(w, seq_len=S)
    P32 = basis(w)
    cache, K_hat, V, q, P = upload_case(w, inp, P32, capacity=S + 5)
    with forced_cluster(ncta):
        out = L().dense_decode_attention(cache, S, q, P)
    torch.cuda.synchronize()
    ref = oracle.dense_decode(inp["q64"], K_hat, V, P32.astype(np.float64), S)
    parity.check_dense(out.cpu().numpy(), ref, dtype)


# ----------------------------------------------------------------------------- errors
def test_invalid_arguments_raise_without_launch():
    lib = L()
    cache = lib.LokiCache(1, 2, 128, 64, dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device=DEV)
    P = torch.zeros((2, 128, 128), dtype=torch.float32, device=DEV)
    for d, k, S in [(0, 1, 10), (129, 1, 10), (8, 0, 10), (8, 11, 10), (8, 1, 65), (8, 1, 0)]:
        with pytest.raises(lib.LokiError) as e:
            lib.loki_decode_attention(cache, S, q, P, d, k)
        assert e.value.status == 1
    q3 = torch.zeros((1, 6, 128), dtype=torch.bfloat16, device=DEV)   # G = 3
    with pytest.raises(lib.LokiError) as e:
        lib.loki_decode_attention(cache, 10, q3, P, 8, 4)
    assert e.value.status == 2
    with pytest.raises(lib.LokiError) as e:
        lib.loki_append(cache, 60, torch.zeros((1, 2, 5, 128), dtype=torch.bfloat16, device=DEV),
                        torch.zeros((1, 2, 5, 128), dtype=torch.bfloat16, device=DEV), P)
    assert e.value.status == 1
    torch.cuda.synchronize()


# ----------------------------------------------------------------------------- full-size workloads
def fill_cache_on_device(w, P_dev, S, capacity, seed=123, d_lr=0, chunk=16384):
    """Whole cache through the GPU append kernel from device-drawn keys (with
    a low-rank key plane d_lr wide when d_lr > 0), `chunk` tokens per append
    so that the keys in flight stay a few GB even for the largest caches."""
    td = TORCH_DTYPE[w.dtype]
    cache = L().LokiCache(w.batch, w.n_kv_heads, w.head_dim, capacity, dtype=td, device=DEV,
                          lowrank_dim=d_lr or None)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    for t0 in range(0, S, chunk):
        n = min(chunk, S - t0)
        k_new = torch.empty((w.batch, w.n_kv_heads, n, w.head_dim), dtype=td, device=DEV)
        for h in range(w.n_kv_heads):
            k_new[:, h] = gen.device_keys(gen.make_key_model(w, h), w.batch, n, g, DEV, td)
        v_new = torch.randn((w.batch, w.n_kv_heads, n, w.head_dim), generator=g, device=DEV).to(td)
        L().loki_append(cache, t0, k_new, v_new, P_dev)
        del k_new, v_new
    return cache


def full_size_check(w, S=None, n_rows=3, seed=0):
    """The launch configuration bench.py times: a cache with a low-rank key
    plane as wide as d (rounded up to 16 bytes) when that is narrower than D."""
    S = S or w.seq_len
    k = w.k if S == w.seq_len else max(1, min(S, int(np.floor(w.k_f * S + 1e-9))))
    d = w.d
    per = 8 if w.dtype == "bf16" else 4
    d_lr = (d + per - 1) // per * per
    d_lr = d_lr if d_lr < w.head_dim else 0
    P32 = basis(w)
    P_dev = torch.from_numpy(P32).to(DEV)
    cache = fill_cache_on_device(w, P_dev, S, S, d_lr=d_lr)
    rng = np.random.default_rng(seed)
    rows = sorted({(int(rng.integers(0, w.batch)), int(rng.integers(0, w.n_kv_heads))) for _ in range(n_rows)})
    G = w.group
    td = TORCH_DTYPE[w.dtype]
    host = {}
    for (b, g) in rows:
        keys = gen.row_keys(w, b, g, S)
        kt, k64 = gen.to_cache_dtype(keys, w.dtype)
        vt, v64 = gen.to_cache_dtype(gen.row_values(w, b, g, S), w.dtype)
        K_hat = oracle.rotate_keys(k64[None, None], P32[g:g + 1].astype(np.float64), w.dtype)
        cache.k_hat[b, g, :S] = torch.from_numpy(K_hat[0, 0]).to(td).to(DEV)
        cache.v[b, g, :S] = vt.to(DEV)
        host[(b, g)] = (K_hat, v64[None, None])
    if d_lr:
        cache.k_lr.copy_(cache.k_hat[..., :d_lr])  # the plane follows the rows written above
    Q = np.stack([gen.queries(w, b) for b in range(w.batch)])
    qt, q64 = gen.to_cache_dtype(Q, w.dtype)
    out, idx = L().loki_decode_attention(cache, S, qt.to(DEV), P_dev, d, k)
    dense = L().dense_decode_attention(cache, S, qt.to(DEV), P_dev)
    torch.cuda.synchronize()
    out, idx, dense = out.cpu().numpy(), idx.cpu().numpy(), dense.cpu().numpy()
    for (b, g), (K_hat, V) in host.items():
        qs = q64[b:b + 1, g * G:(g + 1) * G]
        Pg = P32[g:g + 1].astype(np.float64)
        ref = oracle.loki_decode(qs, K_hat, V, Pg, S, d, k)
        parity.check_decode(out[b:b + 1, g * G:(g + 1) * G], idx[b:b + 1, g:g + 1], ref, ref["q_hat"], K_hat, V,
                            oracle.default_scale(w.head_dim), w.dtype)
        rd = oracle.dense_decode(qs, K_hat, V, Pg, S)
        parity.check_dense(dense[b:b + 1, g * G:(g + 1) * G], rd, w.dtype)
    # every row's selection is structurally valid
    assert idx.min() >= 0 and idx.max() < S
    assert np.all(np.diff(idx, axis=-1) > 0)
    del cache
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["llama2-7b-decode", "llama3-8b-gqa-decode"])
def test_full_size_workload(name):
    full_size_check(get_workload(name))


@pytest.mark.parametrize("S", [3073, 3328, 3584])
def test_llama2_13b_generation_lengths(S):
    w = get_workload("llama2-13b-generation")
    full_size_check(w, S=S, n_rows=2)


SWEEP_SAMPLE = [
    "mistral-7b-gqa-s4096-b1-d0.25-k0.25",
    "mistral-7b-gqa-s16384-b8-d0.125-k0.5",
    "mistral-7b-gqa-s16384-b8-d0.5-k0.5",       # the largest d and k together
    "mistral-7b-gqa-s16384-b32-d0.25-k0.25",    # 256 rows: several waves of clusters
    "mistral-7b-gqa-s16384-b64-d0.125-k0.125",  # 512 rows
    "mistral-7b-gqa-s65536-b1-d0.5-k0.125",
    "mistral-7b-gqa-s131072-b1-d0.25-k0.25",
    "mistral-7b-gqa-s131072-b8-d0.125-k0.125",
    "mistral-7b-gqa-s131072-b32-d0.25-k0.125",  # 256 rows of 131072 tokens (17 GB of cache)
    "mistral-7b-gqa-s131072-b64-d0.125-k0.25",  # 512 rows (34 GB of cache)
]


@pytest.mark.parametrize("name", SWEEP_SAMPLE)
def test_mistral_sweep_points(name):
    w = next(p for p in mistral_sweep_points() if p.name == name)
    full_size_check(w, n_rows=2)
