"""The low-rank key plane of a contiguous cache (loki_cache.k_lr, d_lr): every
call that writes keys keeps it equal to the first d_lr dims of k_hat, and a
Loki decode that streams its scores from it returns exactly what the same call
without the plane returns (the plane is a copy of the values it replaces), and
matches the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from test_gpu_parity import DEV, TORCH_DTYPE, L, basis, forced_cluster, small_workload
from workloads import generators as gen

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _plane_cache(B, Hkv, D, cap, td, d_lr):
    c = L().LokiCache(B, Hkv, D, cap, dtype=td, device=DEV, lowrank_dim=d_lr)
    c.k_hat.fill_(SENTINEL)
    c.v.fill_(SENTINEL)
    c.k_lr.fill_(SENTINEL)
    return c


@pytest.mark.parametrize("dtype,D,d_lr,n_new,pos,B,Hkv", [
    ("bf16", 128, 32, 1, 0, 2, 3),       # CUDA-core append
    ("bf16", 128, 16, 37, 5, 3, 2),
    ("bf16", 128, 64, 300, 100, 2, 2),   # tensor cores, ragged last tile
    ("bf16", 128, 128, 150, 3, 3, 5),    # tensor cores, plane as wide as the key
    ("bf16", 64, 8, 257, 11, 1, 3),      # tensor cores, D = 64
    ("f32", 64, 4, 9, 3, 1, 4),
    ("f32", 128, 36, 41, 0, 2, 3),
])
def test_append_writes_the_plane(dtype, D, d_lr, n_new, pos, B, Hkv):
    w = small_workload(dtype, D, 1, n_new, Hkv=Hkv, B=B)
    inp = gen.decode_inputs(w, seq_len=n_new)
    P = torch.from_numpy(basis(w)).to(DEV)
    cap = pos + n_new + 5
    c = _plane_cache(B, Hkv, D, cap, TORCH_DTYPE[dtype], d_lr)
    L().loki_append(c, pos, inp["keys"].to(DEV), inp["values"].to(DEV), P)
    torch.cuda.synchronize()
    # inside the range: bit-exact copy of the stored keys; outside: untouched
    assert torch.equal(c.k_lr[:, :, pos:pos + n_new], c.k_hat[:, :, pos:pos + n_new, :d_lr])
    assert bool((c.k_lr[:, :, :pos] == SENTINEL).all()) and bool((c.k_lr[:, :, pos + n_new:] == SENTINEL).all())
    assert not bool((c.k_hat[:, :, pos:pos + n_new] == SENTINEL).all())


def _twin_caches(w, inp, P32, d_lr):
    """Two caches with the same k_hat and v (the oracle's rotated keys): one
    with the plane (a copy of k_hat[..., :d_lr]), one without."""
    S = inp["seq_len"]
    td = TORCH_DTYPE[w.dtype]
    K_hat = oracle.rotate_keys(inp["keys64"], P32.astype(np.float64), w.dtype)
    B = len(inp["batches"])
    plain = L().LokiCache(B, w.n_kv_heads, w.head_dim, S, dtype=td, device=DEV)
    plain.k_hat.copy_(torch.from_numpy(K_hat).to(td))
    plain.v.copy_(inp["values"])
    lr = L().LokiCache(B, w.n_kv_heads, w.head_dim, S, dtype=td, device=DEV, k_hat=plain.k_hat, v=plain.v,
                       lowrank_dim=d_lr)
    lr.k_lr.copy_(plain.k_hat[..., :d_lr])
    return plain, lr, K_hat


@pytest.mark.parametrize("dtype,D,G,S,d,d_lr,kf,ncta", [
    ("bf16", 128, 1, 4096, 32, 32, 0.25, None),    # the llama2-7b shape, gather path
    ("bf16", 128, 4, 3000, 64, 64, 0.125, None),   # GQA, tensor-core attention
    ("bf16", 128, 4, 20000, 32, 64, 0.25, 4),      # d < d_lr, candidate path
    ("bf16", 128, 8, 1500, 16, 16, 0.25, None),    # groups of 8: rotate grid + decode
    ("bf16", 64, 2, 777, 8, 16, 0.5, 2),           # D = 64, ragged
    ("f32", 128, 1, 1000, 32, 32, 0.25, None),
    ("bf16", 128, 4, 2048, 96, 64, 0.25, None),    # d > d_lr: the plane is not read
    ("f32", 128, 2, 20000, 32, 32, 0.25, 4),       # fp32 plane, candidate path
    ("bf16", 128, 2, 9000, 40, 40, 0.125, None),   # an 80-byte plane row (not a power of two)
    ("bf16", 128, 4, 30000, 64, 64, 0.5, 2),       # k_f 0.5: the select lists overflow
])
def test_decode_with_plane_is_bit_identical(dtype, D, G, S, d, d_lr, kf, ncta):
    w = small_workload(dtype, D, G, S, Hkv=2, B=2, seed=91)
    inp = gen.decode_inputs(w, seq_len=S)
    P32 = basis(w)
    plain, lr, K_hat = _twin_caches(w, inp, P32, d_lr)
    q = inp["q"].to(DEV)
    P = torch.from_numpy(P32).to(DEV)
    k = max(1, int(kf * S))
    with forced_cluster(ncta):
        o0, i0 = L().loki_decode_attention(plain, S, q, P, d, k)
        o1, i1 = L().loki_decode_attention(lr, S, q, P, d, k)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1)
    assert torch.equal(o0, o1)
    # and against the oracle on two rows
    ref = oracle.loki_decode(inp["q64"], K_hat, inp["values64"], P32.astype(np.float64), S, d, k)
    parity.check_decode(o1.cpu().numpy(), i1.cpu().numpy(), ref, ref["q_hat"], K_hat, inp["values64"],
                        oracle.default_scale(D), dtype, rows=[(0, 0), (1, 1)])


@pytest.mark.parametrize("G", [4, 8])
def test_fused_append_keeps_the_plane(G):
    S, D, d_lr, d = 2500, 128, 32, 32
    w = small_workload("bf16", D, G, S, Hkv=2, B=3, seed=5)
    inp = gen.decode_inputs(w, seq_len=S)
    P32 = basis(w)
    plain, lr, _ = _twin_caches(w, inp, P32, d_lr)
    lr2 = L().LokiCache(3, 2, D, S, dtype=torch.bfloat16, device=DEV, lowrank_dim=d_lr)
    lr2.k_hat.copy_(plain.k_hat)
    lr2.v.copy_(plain.v)
    lr2.k_lr.copy_(lr.k_lr)
    lr2.k_lr[:, :, S - 1].fill_(SENTINEL)  # the slot the call must overwrite
    plain.k_hat[:, :, S - 1].fill_(SENTINEL)
    k_new = inp["keys"][:, :, S - 1].contiguous().to(DEV)
    v_new = inp["values"][:, :, S - 1].contiguous().to(DEV)
    q = inp["q"].to(DEV)
    P = torch.from_numpy(P32).to(DEV)
    k = S // 4
    o0, i0 = L().loki_decode_attention_append(plain, S, k_new, v_new, q, P, d, k)
    o1, i1 = L().loki_decode_attention_append(lr2, S, k_new, v_new, q, P, d, k)
    torch.cuda.synchronize()
    assert torch.equal(lr2.k_hat, plain.k_hat)
    assert torch.equal(lr2.k_lr, lr2.k_hat[..., :d_lr])
    assert torch.equal(i0, i1)
    assert torch.equal(o0, o1)
