"""Generation steps that append their token inside the decode call
(loki_decode_attention_append, dense_decode_attention_append,
loki_paged_decode_attention_append) against the oracle.

The cache holds the first S - 1 tokens (rotated by the oracle); the call must
write token S - 1 (k_new . P rounded to the cache dtype, within the fp32
accumulation bound of loki_append, and v_new exactly) and then return the Loki
(or dense) step over all S tokens of the updated cache, compared with the
oracle on the cache as read back.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from test_gpu_parity import DEV, TORCH_DTYPE, L, basis, forced_cluster, small_workload
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _setup(dtype, D, G, S, B, Hkv, seed):
    w = small_workload(dtype, D, G, S, Hkv=Hkv, B=B, seed=seed)
    inp = gen.decode_inputs(w, seq_len=S)
    P32 = basis(w)
    td = TORCH_DTYPE[dtype]
    cache = L().LokiCache(B, Hkv, D, S + 2, dtype=td, device=DEV)
    cache.k_hat.fill_(123.0)  # stale data in the slot the call must overwrite
    cache.v.fill_(123.0)
    K_hat = oracle.rotate_keys(inp["keys64"], P32.astype(np.float64), dtype)
    if S > 1:
        cache.k_hat[:, :, :S - 1] = torch.from_numpy(K_hat[:, :, :S - 1]).to(td).to(DEV)
        cache.v[:, :, :S - 1] = inp["values"][:, :, :S - 1].to(DEV)
    k_new = inp["keys"][:, :, S - 1].contiguous().to(DEV)
    v_new = inp["values"][:, :, S - 1].contiguous().to(DEV)
    return w, inp, P32, cache, k_new, v_new, inp["q"].to(DEV), torch.from_numpy(P32).to(DEV)


def _check_new_row(cache, S, inp, P32, dtype):
    got = cache.k_hat[:, :, S - 1:S].double().cpu().numpy()
    parity.check_append(got, inp["keys64"][:, :, S - 1:S], P32.astype(np.float64), dtype)
    assert np.array_equal(cache.v[:, :, S - 1].double().cpu().numpy(), inp["values64"][:, :, S - 1])


CASES = [
    # dtype, D, G, S, B, Hkv, d, k, cluster
    ("bf16", 128, 1, 4096, 1, 4, 32, 1024, None),
    ("bf16", 128, 4, 20000, 1, 2, 64, 2500, None),
    ("bf16", 128, 4, 3001, 2, 2, 32, 750, 4),
    ("f32", 64, 2, 300, 2, 2, 16, 75, None),
    ("bf16", 128, 8, 3000, 2, 1, 32, 700, None),
    ("bf16", 128, 1, 1, 2, 2, 8, 1, None),
    ("bf16", 64, 4, 257, 3, 2, 16, 60, 2),
    ("f32", 128, 1, 9000, 1, 2, 32, 2000, 8),
]


@pytest.mark.parametrize("dtype,D,G,S,B,Hkv,d,k,ncta", CASES)
def test_loki_step_with_append(dtype, D, G, S, B, Hkv, d, k, ncta):
    w, inp, P32, cache, k_new, v_new, q, P = _setup(dtype, D, G, S, B, Hkv, seed=S + G)
    with forced_cluster(ncta):
        out, idx = L().loki_decode_attention_append(cache, S, k_new, v_new, q, P, d, k)
    torch.cuda.synchronize()
    _check_new_row(cache, S, inp, P32, dtype)
    K = cache.k_hat[:, :, :S].double().cpu().numpy()
    V = cache.v[:, :, :S].double().cpu().numpy()
    ref = oracle.loki_decode(inp["q64"], K, V, P32.astype(np.float64), S, d, k)
    parity.check_decode(out.cpu().numpy(), idx.cpu().numpy(), ref, ref["q_hat"], K, V, oracle.default_scale(D), dtype)


@pytest.mark.parametrize("dtype,D,G,S,B,Hkv,ncta", [("bf16", 128, 1, 4096, 1, 4, None), ("bf16", 128, 4, 20000, 1, 2, 4),
                                                    ("f32", 64, 2, 300, 2, 2, 2), ("bf16", 128, 8, 513, 2, 1, None),
                                                    ("bf16", 128, 1, 1, 2, 2, None)])
def test_dense_step_with_append(dtype, D, G, S, B, Hkv, ncta):
    w, inp, P32, cache, k_new, v_new, q, P = _setup(dtype, D, G, S, B, Hkv, seed=7 * S + G)
    with forced_cluster(ncta):
        out = L().dense_decode_attention_append(cache, S, k_new, v_new, q, P)
    torch.cuda.synchronize()
    _check_new_row(cache, S, inp, P32, dtype)
    K = cache.k_hat[:, :, :S].double().cpu().numpy()
    V = cache.v[:, :, :S].double().cpu().numpy()
    ref = oracle.dense_decode(inp["q64"], K, V, P32.astype(np.float64), S)
    parity.check_dense(out.cpu().numpy(), ref, dtype)


def test_generation_loop_matches_the_oracle():
    """Three steps in a row, each appending its token inside the call."""
    S0, steps = 2000, 3
    w, inp, P32, cache, _, _, q, P = _setup("bf16", 128, 4, S0 + steps, 2, 2, seed=5)
    for t in range(steps):
        S = S0 + 1 + t
        k_new = inp["keys"][:, :, S - 1].contiguous().to(DEV)
        v_new = inp["values"][:, :, S - 1].contiguous().to(DEV)
        out, idx = L().loki_decode_attention_append(cache, S, k_new, v_new, q, P, 32, S // 4)
    torch.cuda.synchronize()
    S = S0 + steps
    K = cache.k_hat[:, :, :S].double().cpu().numpy()
    V = cache.v[:, :, :S].double().cpu().numpy()
    parity.check_append(K[:, :, S0:S], inp["keys64"][:, :, S0:S], P32.astype(np.float64), "bf16")
    ref = oracle.loki_decode(inp["q64"], K, V, P32.astype(np.float64), S, 32, S // 4)
    parity.check_decode(out.cpu().numpy(), idx.cpu().numpy(), ref, ref["q_hat"], K, V, oracle.default_scale(128),
                        "bf16")


def test_paged_step_with_append():
    """Per-sequence lengths: sequence b's token goes to position S_b - 1."""
    from test_gpu_paged import Setup, _check_decode_rows, _widen
    lens = [700, 33, 4000]
    su = Setup("bf16", 128, 4, 16, [S - 1 for S in lens], seed=21)
    Lb = su.L
    zeros = torch.zeros(su.B, dtype=torch.int32, device=su.dev)
    Lb.loki_paged_append(su.cache, su.seqs(), zeros, su.k_new, su.v_new, su.P_dev)
    su.scrub_past([S - 1 for S in lens])
    kt = torch.randn((su.B, su.Hkv, su.D), device=su.dev).to(torch.bfloat16)
    vt = torch.randn((su.B, su.Hkv, su.D), device=su.dev).to(torch.bfloat16)
    lens_t = torch.as_tensor(np.array(lens, dtype=np.int32)).to(su.dev)
    ks = [max(1, S // 4) for S in lens]
    ks_t = torch.as_tensor(np.array(ks, dtype=np.int32)).to(su.dev)
    out, idx = Lb.loki_paged_decode_attention_append(su.cache, su.seqs(lens_t), kt, vt, su.q, su.P_dev, 32, max(ks),
                                                     ks=ks_t)
    torch.cuda.synchronize()
    K = su.logical(su.cache.k_hat)
    for b, S in enumerate(lens):
        parity.check_append(K[b:b + 1, :, S - 1:S], _widen(kt)[b:b + 1, :, None], su.P.astype(np.float64), "bf16")
        assert np.array_equal(su.logical(su.cache.v)[b, :, S - 1], _widen(vt)[b])
    _check_decode_rows(su, lens, ks, 32, out, idx)


def test_generation_run_of_the_pages_shape():
    """The Llama2-13B-like generation run (batch 16, 40 heads, D 128, bf16):
    a prompt of 3072 tokens, then 64 consecutive steps, step t appending its
    token at position 3072 + t inside the call and attending over 3073 + t
    tokens with k = floor(S / 4), d = 32, on a cache with a 32-dim low-rank
    plane.  Checked against the oracle: every appended row of the sampled
    (batch, KV head) rows, and the last step's outputs and selections of those
    rows (on the cache as the GPU left it); every row's last selection is
    valid."""
    from test_gpu_parity import fill_cache_on_device
    from workloads import get_workload
    w = get_workload("llama2-13b-generation")
    T0, steps, d = w.prompt_len, 64, w.d
    B, Hkv, D = w.batch, w.n_kv_heads, w.head_dim
    P32 = basis(w)
    P_dev = torch.from_numpy(P32).to(DEV)
    cache = fill_cache_on_device(w, P_dev, T0, T0 + steps, d_lr=32)
    rows = [(0, 0), (7, 21), (15, 39)]
    pre = {}
    for (b, g) in rows:  # host-drawn prompts for the rows the oracle checks
        kt, k64 = gen.to_cache_dtype(gen.row_keys(w, b, g, T0), "bf16")
        vt, v64 = gen.to_cache_dtype(gen.row_values(w, b, g, T0), "bf16")
        K_hat = oracle.rotate_keys(k64[None, None], P32[g:g + 1].astype(np.float64), "bf16")
        cache.k_hat[b, g, :T0] = torch.from_numpy(K_hat[0, 0]).to(torch.bfloat16).to(DEV)
        cache.v[b, g, :T0] = vt.to(DEV)
        pre[(b, g)] = v64
    cache.k_lr[:, :, :T0].copy_(cache.k_hat[:, :, :T0, :32])
    models = [gen.make_key_model(w, g) for g in range(Hkv)]
    news = []
    for t in range(steps):
        tok = [gen.new_token(w, b, t, models) for b in range(B)]
        kn = np.stack([x[0] for x in tok])
        vn = np.stack([x[1] for x in tok])
        knt, kn64 = gen.to_cache_dtype(kn, "bf16")
        vnt, vn64 = gen.to_cache_dtype(vn, "bf16")
        Q = np.stack([gen.queries(w, b, step=t) for b in range(B)])
        qt, q64 = gen.to_cache_dtype(Q, "bf16")
        S = T0 + t + 1
        out, idx = L().loki_decode_attention_append(cache, S, knt.to(DEV), vnt.to(DEV), qt.to(DEV), P_dev, d,
                                                    S // 4)
        news.append((kn64, vn64))
    torch.cuda.synchronize()
    S = T0 + steps
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    Kall = cache.k_hat[:, :, :S].double().cpu().numpy()
    Vall = cache.v[:, :, :S].double().cpu().numpy()
    assert torch.equal(cache.k_lr[:, :, T0:S], cache.k_hat[:, :, T0:S, :32])  # the plane follows every append
    for (b, g) in rows:
        kn64 = np.stack([news[t][0][b, g] for t in range(steps)])
        vn64 = np.stack([news[t][1][b, g] for t in range(steps)])
        parity.check_append(Kall[b:b + 1, g:g + 1, T0:S], kn64[None, None], P32[g:g + 1].astype(np.float64),
                            "bf16")
        assert np.array_equal(Vall[b, g, T0:S], vn64)
        assert np.array_equal(Vall[b, g, :T0], pre[(b, g)])
        ref = oracle.loki_decode(q64[b:b + 1, g:g + 1], Kall[b:b + 1, g:g + 1], Vall[b:b + 1, g:g + 1],
                                 P32[g:g + 1].astype(np.float64), S, d, S // 4)
        parity.check_decode(out[b:b + 1, g:g + 1], idx[b:b + 1, g:g + 1], ref, ref["q_hat"],
                            Kall[b:b + 1, g:g + 1], Vall[b:b + 1, g:g + 1], oracle.default_scale(D), "bf16")
    assert idx.min() >= 0 and idx.max() < S and np.all(np.diff(idx, axis=-1) > 0)
