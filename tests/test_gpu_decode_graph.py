"""DecodeGraph: the decode step from and to pinned host memory, captured once
as a CUDA graph and replayed, returns exactly what the eager call returns, for
new queries and for cache contents that change between replays."""
import numpy as np
import pytest
import torch

import oracle
import parity
from test_gpu_parity import DEV, L, basis, small_workload, upload_case
from workloads import generators as gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,S,d,kf", [(1, 4096, 32, 0.25), (4, 20000, 64, 0.125), (8, 1500, 32, 0.25)])
def test_graph_replays_match_eager_calls(G, S, d, kf):
    w = small_workload("bf16", 128, G, S, Hkv=2, B=2, seed=400 + G)
    inp = gen.decode_inputs(w, seq_len=S)
    P32 = basis(w)
    cache, K_hat, V, q, P = upload_case(w, inp, P32)
    k = max(1, int(kf * S))
    g = L().DecodeGraph(cache, S, P, d, k, w.n_q_heads)
    rng = torch.Generator().manual_seed(9)
    for step in range(3):
        qh = torch.randn(q.shape, generator=rng).to(torch.bfloat16) if step else q.cpu()
        g.q_host.copy_(qh)
        g.replay()
        torch.cuda.synchronize()
        o_e, i_e = L().loki_decode_attention(cache, S, qh.to(DEV), P, d, k)
        torch.cuda.synchronize()
        assert torch.equal(g.idx_host, i_e.cpu())
        assert torch.equal(g.out_host, o_e.cpu())
        if step == 0:
            ref = oracle.loki_decode(inp["q64"], K_hat, V, P32.astype(np.float64), S, d, k)
            parity.check_decode(g.out_host.numpy(), g.idx_host.numpy(), ref, ref["q_hat"], K_hat, V,
                                oracle.default_scale(128), "bf16")
        # the cache changes between replays: the next replay reads the new rows
        cache.v[:, :, :64].mul_(-1.0)
