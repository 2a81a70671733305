"""Paged caches with per-sequence lengths (loki_paged_append,
loki_paged_decode_attention, dense_paged_decode_attention) against the oracle.

Per sequence the Loki step is the same computation as on a contiguous cache
over that sequence's tokens 0 .. S_b - 1, so the oracle is run one sequence at
a time on the logical token order gathered from the pages.  Page ids are a
random permutation of a pool with spare pages, and every slot a sequence does
not own (past S_b) holds a large constant, so a read past the sequence or
through a wrong page would change the results.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity

pytestmark = pytest.mark.gpu

TD = {"bf16": torch.bfloat16, "f32": torch.float32}
GARBAGE = 300.0


def _orthonormal(rng, H, D):
    return np.stack([np.linalg.qr(rng.standard_normal((D, D)))[0] for _ in range(H)]).astype(np.float32)


def _keys(rng, B, H, S, D):
    # low-rank structure plus noise, with a per-head offset
    A = rng.standard_normal((H, 8, D)) / np.sqrt(8)
    Z = rng.standard_normal((B, H, S, 8))
    return np.einsum("bhsr,hrd->bhsd", Z, A) + 0.3 * rng.standard_normal((B, H, S, D)) + \
        0.5 * rng.standard_normal((1, H, 1, D))


class Setup:
    def __init__(self, dtype, D, G, page, lens, seed, Hkv=2, spare=5):
        import sparse_decode_attention_loki_b200 as L
        self.L = L
        rng = np.random.default_rng(seed)
        self.dtype, self.D, self.G, self.page, self.lens = dtype, D, G, page, list(lens)
        self.B, self.Hkv, self.Hq = len(lens), Hkv, Hkv * G
        self.S_max = max(lens)
        self.pps = math.ceil((self.S_max + 1) / page)  # room for one generated token
        self.num_pages = self.B * self.pps + spare
        table = rng.permutation(self.num_pages)[: self.B * self.pps].reshape(self.B, self.pps).astype(np.int32)
        self.table_np = table
        td = TD[dtype]
        self.dev = torch.device("cuda", 0)
        self.cache = L.PagedLokiCache(self.num_pages, Hkv, D, page, dtype=td, device=self.dev)
        self.cache.k_hat.fill_(GARBAGE)
        self.cache.v.fill_(GARBAGE)
        self.table = torch.as_tensor(table).to(self.dev)
        self.seq_lens = torch.as_tensor(np.array(lens, dtype=np.int32)).to(self.dev)
        self.P = _orthonormal(rng, Hkv, D)
        self.P_dev = torch.as_tensor(self.P).to(self.dev)
        k64 = _keys(rng, self.B, Hkv, self.S_max, D)
        v64 = rng.standard_normal((self.B, Hkv, self.S_max, D))
        self.k_new = torch.as_tensor(k64, dtype=torch.float32).to(td).to(self.dev).contiguous()
        self.v_new = torch.as_tensor(v64, dtype=torch.float32).to(td).to(self.dev).contiguous()
        self.q = torch.as_tensor(rng.standard_normal((self.B, self.Hq, D)), dtype=torch.float32).to(td).to(
            self.dev).contiguous()
        self.rng = rng

    def seqs(self, lens=None):
        lens_t = self.seq_lens if lens is None else lens
        mx = self.S_max if lens is None else int(lens.max().item())
        return self.L.SeqTable(self.table, lens_t, mx)

    def logical(self, pool):
        """[B, Hkv, pps*page, D] fp64 in token order, gathered from the pages."""
        p = pool.float().cpu().numpy().astype(np.float64)
        out = p[self.table_np]                       # [B, pps, Hkv, page, D]
        out = out.transpose(0, 2, 1, 3, 4).reshape(self.B, self.Hkv, self.pps * self.page, self.D)
        return out

    def own_slot_mask(self, lens):
        """Slots (b, t) a sequence owns below its length."""
        m = np.zeros((self.B, self.pps * self.page), dtype=bool)
        for b, S in enumerate(lens):
            m[b, :S] = True
        return m

    def scrub_past(self, lens):
        """Write GARBAGE to every slot of a sequence's pages at or past its length."""
        pg, sl = [], []
        for b, S in enumerate(lens):
            t = np.arange(S, self.pps * self.page)
            pg.append(self.table_np[b, t // self.page])
            sl.append(t % self.page)
        pg = torch.as_tensor(np.concatenate(pg).astype(np.int64)).to(self.dev)
        sl = torch.as_tensor(np.concatenate(sl).astype(np.int64)).to(self.dev)
        self.cache.k_hat[pg, :, sl, :] = GARBAGE
        self.cache.v[pg, :, sl, :] = GARBAGE


def _widen(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_decode_rows(su, lens, ks, d, out, idx):
    K = su.logical(su.cache.k_hat)
    V = su.logical(su.cache.v)
    q64 = _widen(su.q)
    P64 = su.P.astype(np.float64)
    scale = oracle.default_scale(su.D)
    idx_np = idx.cpu().numpy()
    out_np = out.cpu().numpy()
    k_max = idx_np.shape[2]
    for b, (S, k) in enumerate(zip(lens, ks)):
        ref = oracle.loki_decode(q64[b:b + 1], K[b:b + 1, :, :S], V[b:b + 1, :, :S], P64, S, d, k)
        parity.check_decode(out_np[b:b + 1], idx_np[b:b + 1, :, :k], ref, ref["q_hat"], K[b:b + 1, :, :S],
                            V[b:b + 1, :, :S], scale, su.dtype)
        assert np.all(idx_np[b, :, k:k_max] == -1), f"sequence {b}: idx past k={k} is not -1"


CASES = [
    # dtype, D, G, page, lens, k_f, d_f
    ("bf16", 128, 1, 16, [300, 1, 77, 512], 0.25, 0.25),
    ("f32", 64, 2, 64, [257, 64, 130], 0.5, 0.25),
    ("bf16", 128, 4, 256, [4096, 1500, 3000], 0.125, 0.5),
    ("bf16", 128, 8, 32, [20000, 5000], 0.25, 0.25),
    ("f32", 128, 1, 1, [40, 9], 0.25, 0.125),
]


@pytest.mark.parametrize("dtype,D,G,page,lens,k_f,d_f", CASES)
def test_paged_append_decode_dense_and_generation(dtype, D, G, page, lens, k_f, d_f):
    su = Setup(dtype, D, G, page, lens, seed=D + G + page + len(lens))
    L = su.L
    B = su.B
    # bulk append of every sequence's first S_max tokens at position 0
    zeros = torch.zeros(B, dtype=torch.int32, device=su.dev)
    L.loki_paged_append(su.cache, su.seqs(), zeros, su.k_new, su.v_new, su.P_dev)
    torch.cuda.synchronize()
    K = su.logical(su.cache.k_hat)[:, :, :su.S_max]
    keys64 = _widen(su.k_new)
    tc = dtype == "bf16" and B * su.S_max >= 256
    for b in range(B):
        parity.check_append(K[b:b + 1], keys64[b:b + 1], su.P.astype(np.float64), dtype, tensor_core=tc)
    assert np.array_equal(su.logical(su.cache.v)[:, :, :su.S_max], _widen(su.v_new))
    su.scrub_past(lens)

    d = max(1, int(d_f * D))
    ks = [max(1, int(k_f * S)) for S in lens]
    k_max = max(ks)
    ks_t = torch.as_tensor(np.array(ks, dtype=np.int32)).to(su.dev)
    out, idx = L.loki_paged_decode_attention(su.cache, su.seqs(), su.q, su.P_dev, d, k_max, ks=ks_t)
    torch.cuda.synchronize()
    _check_decode_rows(su, lens, ks, d, out, idx)

    # without ks every sequence keeps min(S_b, k_max)
    out2, idx2 = L.loki_paged_decode_attention(su.cache, su.seqs(), su.q, su.P_dev, d, k_max)
    torch.cuda.synchronize()
    _check_decode_rows(su, lens, [min(S, k_max) for S in lens], d, out2, idx2)

    dout = L.dense_paged_decode_attention(su.cache, su.seqs(), su.q, su.P_dev)
    torch.cuda.synchronize()
    Kl, Vl = su.logical(su.cache.k_hat), su.logical(su.cache.v)
    q64 = _widen(su.q)
    for b, S in enumerate(lens):
        ref = oracle.dense_decode(q64[b:b + 1], Kl[b:b + 1, :, :S], Vl[b:b + 1, :, :S], su.P.astype(np.float64), S)
        parity.check_dense(dout[b:b + 1].cpu().numpy(), ref, dtype)

    # one generation step: each sequence appends a token at its own length
    kt = torch.as_tensor(_keys(su.rng, B, su.Hkv, 1, D), dtype=torch.float32).to(TD[dtype]).to(su.dev).contiguous()
    vt = torch.as_tensor(su.rng.standard_normal((B, su.Hkv, 1, D)), dtype=torch.float32).to(TD[dtype]).to(
        su.dev).contiguous()
    L.loki_paged_append(su.cache, su.seqs(), su.seq_lens, kt, vt, su.P_dev)
    lens1 = [S + 1 for S in lens]
    lens1_t = su.seq_lens + 1
    torch.cuda.synchronize()
    Kl = su.logical(su.cache.k_hat)
    for b, S in enumerate(lens):
        parity.check_append(Kl[b:b + 1, :, S:S + 1], _widen(kt)[b:b + 1], su.P.astype(np.float64), dtype)
        assert np.array_equal(su.logical(su.cache.v)[b, :, S], _widen(vt)[b, :, 0])
    ks1 = [max(1, int(k_f * S)) for S in lens1]
    ks1_t = torch.as_tensor(np.array(ks1, dtype=np.int32)).to(su.dev)
    out3, idx3 = L.loki_paged_decode_attention(su.cache, su.seqs(lens1_t), su.q, su.P_dev, d, max(ks1), ks=ks1_t)
    torch.cuda.synchronize()
    _check_decode_rows(su, lens1, ks1, d, out3, idx3)


@pytest.mark.parametrize("dtype,G,page", [("bf16", 1, 64), ("bf16", 4, 16), ("f32", 2, 128)])
def test_uniform_lengths_match_the_contiguous_cache_bit_for_bit(dtype, G, page):
    """With every sequence at the same length the paged call plans the same
    launch as the contiguous one and must return identical bits."""
    S, B, D = 3000, 3, 128
    su = Setup(dtype, D, G, page, [S] * B, seed=11 + G)
    L = su.L
    zeros = torch.zeros(B, dtype=torch.int32, device=su.dev)
    L.loki_paged_append(su.cache, su.seqs(), zeros, su.k_new, su.v_new, su.P_dev)
    cont = L.LokiCache(B, su.Hkv, D, S, dtype=TD[dtype], device=su.dev)
    L.loki_append(cont, 0, su.k_new, su.v_new, su.P_dev)
    torch.cuda.synchronize()
    assert torch.equal(torch.as_tensor(su.logical(su.cache.k_hat)[:, :, :S]), cont.k_hat.double().cpu())
    d, k = 32, 750
    o1, i1 = L.loki_paged_decode_attention(su.cache, su.seqs(), su.q, su.P_dev, d, k)
    o2 = torch.empty_like(o1)
    i2 = torch.empty_like(i1)
    L.loki_decode_attention(cont, S, su.q, su.P_dev, d, k, out=o2, idx=i2)
    d1 = L.dense_paged_decode_attention(su.cache, su.seqs(), su.q, su.P_dev)
    d2 = L.dense_decode_attention(cont, S, su.q, su.P_dev)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2)
    assert torch.equal(o1, o2)
    assert torch.equal(d1, d2)


def test_append_past_the_page_table_is_dropped():
    """Positions beyond pages_per_seq * page_size are not written: the pool is
    unchanged outside the slots the sequences own."""
    su = Setup("bf16", 64, 1, 16, [20, 20], seed=5)
    L = su.L
    before_k = su.cache.k_hat.clone()
    pos = torch.as_tensor(np.array([su.pps * su.page - 3, su.pps * su.page + 4], dtype=np.int32)).to(su.dev)
    kn = su.k_new[:, :, :8].contiguous()
    vn = su.v_new[:, :, :8].contiguous()
    L.loki_paged_append(su.cache, su.seqs(), pos, kn, vn, su.P_dev)
    torch.cuda.synchronize()
    changed = (su.cache.k_hat != before_k).any(dim=(1, 3)).cpu().numpy()  # [num_pages, page]
    owned = set()
    for t in range(su.pps * su.page - 3, su.pps * su.page):
        owned.add((int(su.table_np[0, t // su.page]), t % su.page))
    for pg in range(su.num_pages):
        for sl in range(su.page):
            if changed[pg, sl]:
                assert (pg, sl) in owned, (pg, sl)
    assert len(owned) == int(changed.sum())


# ----------------------------------------------------------------------------- low-rank key plane pools
def _plane_twin(su, d_lr):
    """A paged cache on the same pools with a low-rank plane pool (filled with
    GARBAGE, then kept by the appends)."""
    c = su.L.PagedLokiCache(su.num_pages, su.Hkv, su.D, su.page, dtype=TD[su.dtype], device=su.dev,
                            k_hat=su.cache.k_hat, v=su.cache.v, lowrank_dim=d_lr)
    c.k_lr.fill_(GARBAGE)
    return c


@pytest.mark.parametrize("dtype,D,G,page,lens,d,d_lr", [
    ("bf16", 128, 1, 16, [700, 333, 1024], 32, 32),     # CUDA-core append
    ("bf16", 128, 4, 64, [300, 2000], 32, 64),          # tensor-core append (B * n_new >= 256), d < d_lr
    ("f32", 64, 2, 32, [500, 129, 77], 16, 16),
])
def test_paged_plane_is_kept_and_read(dtype, D, G, page, lens, d, d_lr):
    su = Setup(dtype, D, G, page, lens, seed=17 + G)
    c = _plane_twin(su, d_lr)
    pos = torch.zeros(su.B, dtype=torch.int32, device=su.dev)
    su.L.loki_paged_append(c, su.seqs(), pos, su.k_new, su.v_new, su.P_dev)  # tokens [0, S_max) of every row
    torch.cuda.synchronize()
    # every written slot holds the first d_lr dims of its key; the rest is untouched
    wr = torch.as_tensor(su.own_slot_mask([su.S_max] * su.B)).to(su.dev)
    Kl = torch.as_tensor(su.logical(c.k_hat)).to(su.dev).permute(0, 2, 1, 3)[..., :d_lr]
    Ll = torch.as_tensor(su.logical(torch.nn.functional.pad(c.k_lr, (0, D - d_lr)))).to(su.dev)
    Ll = Ll.permute(0, 2, 1, 3)[..., :d_lr]
    assert torch.equal(Ll[wr], Kl[wr])
    assert bool((Ll[~wr] == GARBAGE).all())
    k = max(1, min(lens) // 4)
    o0, i0 = su.L.loki_paged_decode_attention(su.cache, su.seqs(), su.q, su.P_dev, d, k)
    o1, i1 = su.L.loki_paged_decode_attention(c, su.seqs(), su.q, su.P_dev, d, k)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1) and torch.equal(o0, o1)


def test_paged_fused_append_keeps_the_plane():
    # two identical setups (same seed): one read and kept through a plane, one without
    runs = []
    for plane in (False, True):
        su = Setup("bf16", 128, 4, 16, [900, 401], seed=23)
        c = _plane_twin(su, 32) if plane else su.cache
        pos = torch.zeros(su.B, dtype=torch.int32, device=su.dev)
        su.L.loki_paged_append(c, su.seqs(), pos, su.k_new, su.v_new, su.P_dev)
        lens1 = torch.as_tensor(np.array(su.lens, dtype=np.int32) + 1).to(su.dev)
        seqs1 = su.L.SeqTable(su.table, lens1, su.S_max + 1)
        kn = torch.as_tensor(su.rng.standard_normal((su.B, su.Hkv, 128)), dtype=torch.float32).to(
            torch.bfloat16).to(su.dev)
        vn = torch.as_tensor(su.rng.standard_normal((su.B, su.Hkv, 128)), dtype=torch.float32).to(
            torch.bfloat16).to(su.dev)
        out, idx = su.L.loki_paged_decode_attention_append(c, seqs1, kn, vn, su.q, su.P_dev, 32, 100)
        torch.cuda.synchronize()
        if plane:
            wr = torch.as_tensor(su.own_slot_mask([S + 1 for S in su.lens])).to(su.dev)
            Kl = torch.as_tensor(su.logical(c.k_hat)).to(su.dev).permute(0, 2, 1, 3)[..., :32]
            Ll = torch.as_tensor(su.logical(torch.nn.functional.pad(c.k_lr, (0, 96)))).to(su.dev)
            assert torch.equal(Ll.permute(0, 2, 1, 3)[..., :32][wr], Kl[wr])
        runs.append((out, idx, c.k_hat.clone()))
    assert torch.equal(runs[0][2], runs[1][2])
    assert torch.equal(runs[0][1], runs[1][1]) and torch.equal(runs[0][0], runs[1][0])
