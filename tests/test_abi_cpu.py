"""The C-ABI library loads, exports every entry point include/loki.h declares,
and rejects invalid arguments on the host before any CUDA call.  No test here
launches a kernel: every call below fails host validation (or only reads device
attributes), so the file is safe with or without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "loki.h")


def _declared():
    src = open(HEADER).read()
    return re.findall(r"LOKI_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    from sparse_decode_attention_loki_b200 import _lib
    return _lib.load()


def test_header_declares_the_abi():
    names = _declared()
    assert set(names) == {"loki_append", "loki_decode_workspace_size", "loki_decode_attention",
                          "loki_decode_attention_noalloc", "dense_decode_attention", "loki_decode_launch_shape",
                          "loki_topk_jaccard", "loki_device_error_count", "loki_pca_workspace_size",
                          "loki_paged_append", "loki_paged_decode_workspace_size", "loki_paged_decode_attention",
                          "dense_paged_decode_attention", "loki_decode_attention_append",
                          "dense_decode_attention_append", "loki_paged_decode_attention_append",
                          "loki_pca_calibrate", "loki_set_launch_override", "loki_phase_stamps", "loki_status_string", "loki_last_error",
                          "loki_version"}


def test_library_exports_every_declared_symbol(lib):
    from sparse_decode_attention_loki_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)
    # the binding declares a signature for each of them, and nothing else
    assert set(_lib.SIGNATURES) == set(_declared())


def test_library_is_built_for_sm100a():
    from sparse_decode_attention_loki_b200 import build
    comp, link = build.commands()
    for cmd in comp + [link]:
        assert "arch=compute_100a,code=sm_100a" in " ".join(cmd)


def test_version_and_status_strings(lib):
    assert lib.loki_version() == 13
    for s, word in [(0, b"LOKI_OK"), (1, b"INVALID_ARG"), (2, b"UNSUPPORTED"), (3, b"CUDA")]:
        assert word in lib.loki_status_string(s)
    assert lib.loki_status_string(99) == b"unknown loki_status"


def _cache(dtype=1, B=1, H=2, D=128, cap=64, k=4096, v=8192, k_lr=None, d_lr=0):
    from sparse_decode_attention_loki_b200 import _lib
    return _lib.loki_cache(dtype, B, H, D, cap, k, v, k_lr, d_lr)


FAKE = 1 << 20   # aligned non-null address; never dereferenced because validation fails first
WS = 1 << 24     # 256-byte aligned fake workspace address, with a size that passes the size check
WSB = 1 << 40


@pytest.mark.parametrize("cache_kw,seq,hq,d,k,status", [
    (dict(dtype=7), 10, 2, 8, 4, 1),              # bad dtype
    (dict(B=0), 10, 2, 8, 4, 1),                  # empty batch
    (dict(D=96), 10, 2, 8, 4, 2),                 # unsupported head dim
    (dict(k=0), 10, 2, 8, 4, 1),                  # null cache pointer
    (dict(k=4100), 10, 2, 8, 4, 1),               # misaligned cache pointer
    (dict(), 0, 2, 8, 4, 1),                      # empty sequence
    (dict(), 65, 2, 8, 4, 1),                     # seq_len > capacity
    (dict(), 10, 3, 8, 4, 1),                     # Hq not a multiple of Hkv
    (dict(), 10, 6, 8, 4, 2),                     # group size 3 unsupported
    (dict(), 10, 2, 0, 4, 1),                     # d = 0
    (dict(), 10, 2, 129, 4, 1),                   # d > D
    (dict(), 10, 2, 8, 0, 1),                     # k = 0
    (dict(), 10, 2, 8, 11, 1),                    # k > seq_len
])
def test_decode_validation(lib, cache_kw, seq, hq, d, k, status):
    c = _cache(**cache_kw)
    r = lib.loki_decode_attention(ctypes.byref(c), seq, hq, FAKE, FAKE, d, k, 0.0, FAKE, FAKE, WS, WSB, None)
    assert r == status, lib.loki_last_error()
    assert lib.loki_last_error() != b""


def test_decode_null_pointers(lib):
    c = _cache()
    assert lib.loki_decode_attention(None, 10, 2, FAKE, FAKE, 8, 4, 0.0, FAKE, FAKE, WS, WSB, None) == 1
    for args in [(None, FAKE, FAKE, FAKE), (FAKE, None, FAKE, FAKE), (FAKE, FAKE, None, FAKE), (FAKE, FAKE, FAKE, None)]:
        q, P, out, idx = args
        assert lib.loki_decode_attention(ctypes.byref(c), 10, 2, q, P, 8, 4, 0.0, out, idx, WS, WSB, None) == 1
    assert lib.loki_decode_attention(ctypes.byref(c), 10, 2, FAKE + 8, FAKE, 8, 4, 0.0, FAKE, FAKE, WS, WSB,
                                     None) == 1
    assert lib.dense_decode_attention(ctypes.byref(c), 10, 2, None, FAKE, 0.0, FAKE, None) == 1
    assert lib.dense_decode_attention(ctypes.byref(c), 0, 2, FAKE, FAKE, 0.0, FAKE, None) == 1


def _ws_bytes(B, Hkv, G, D, S=None):
    """The workspace regions include/loki.h documents, each 256-byte aligned:
    the rotated queries [rows, G, D] and the low-rank group queries [rows, D],
    fp32 (no dependence on the length)."""
    a = lambda x: (x + 255) // 256 * 256
    rows = B * Hkv
    return a(rows * G * D * 4) + a(rows * D * 4)


def test_workspace_size_and_validation(lib):
    c = _cache(B=3, H=2, cap=5000)
    n = ctypes.c_size_t(0)
    for S, hq in [(10, 2), (64, 4), (4999, 16), (5000, 2)]:
        assert lib.loki_decode_workspace_size(ctypes.byref(c), S, hq, ctypes.byref(n)) == 0
        assert n.value == _ws_bytes(3, 2, hq // 2, 128, S)
    assert lib.loki_decode_workspace_size(ctypes.byref(c), 5001, 2, ctypes.byref(n)) == 1
    assert lib.loki_decode_workspace_size(ctypes.byref(c), 0, 2, ctypes.byref(n)) == 1
    assert lib.loki_decode_workspace_size(ctypes.byref(c), 10, 3, ctypes.byref(n)) == 1
    assert lib.loki_decode_workspace_size(ctypes.byref(c), 10, 2, None) == 1
    need = _ws_bytes(3, 2, 1, 128, 10)
    args = (ctypes.byref(c), 10, 2, FAKE, FAKE, 8, 4, 0.0, FAKE, FAKE)
    assert lib.loki_decode_attention(*args, None, WSB, None) == 1          # no workspace
    assert lib.loki_decode_attention(*args, WS + 16, WSB, None) == 1       # not 256-byte aligned
    assert lib.loki_decode_attention(*args, WS, need - 1, None) == 1       # too small
    assert b"smaller" in lib.loki_last_error()


def test_device_error_count_validation(lib):
    assert lib.loki_device_error_count(None) == 1


def test_jaccard_validation(lib):
    assert lib.loki_topk_jaccard(FAKE, FAKE, 0, 4, FAKE, None) == 1
    assert lib.loki_topk_jaccard(FAKE, FAKE, 3, 0, FAKE, None) == 1
    assert lib.loki_topk_jaccard(None, FAKE, 3, 4, FAKE, None) == 1
    assert lib.loki_topk_jaccard(FAKE, FAKE + 2, 3, 4, FAKE, None) == 1
    assert lib.loki_topk_jaccard(FAKE, FAKE, 3, 4, None, None) == 1


def _pca_ws_bytes(H, D):
    """Means [H, D] then covariances [H, D, D], fp64, each region padded to 256 bytes."""
    a = lambda x: (x + 255) // 256 * 256
    return a(H * D * 8) + a(H * D * D * 8)


def test_pca_workspace_size_and_validation(lib):
    n = ctypes.c_size_t(0)
    for H, D in [(1, 64), (8, 128), (32, 128), (3, 64)]:
        assert lib.loki_pca_workspace_size(H, D, ctypes.byref(n)) == 0
        assert n.value == _pca_ws_bytes(H, D)
    assert lib.loki_pca_workspace_size(0, 128, ctypes.byref(n)) == 1
    assert lib.loki_pca_workspace_size(2, 96, ctypes.byref(n)) == 2
    assert lib.loki_pca_workspace_size(2, 128, None) == 1
    need = _pca_ws_bytes(2, 128)
    ok = (FAKE, 0, 2, 100, 128, FAKE, FAKE, WS, need, None)
    def call(**kw):
        names = ["keys", "dtype", "H", "N", "D", "P", "w", "ws", "wsb", "stream"]
        args = dict(zip(names, ok))
        args.update(kw)
        return lib.loki_pca_calibrate(*[args[k] for k in names])
    assert call(dtype=2) == 1
    assert call(N=0) == 1
    assert call(D=32) == 2
    assert call(H=0) == 1
    assert call(keys=None) == 1
    assert call(P=None) == 1
    assert call(ws=None) == 1
    assert call(keys=FAKE + 8) == 1      # not 16-byte aligned
    assert call(w=FAKE + 4) == 1         # eigenvalues not 8-byte aligned
    assert call(ws=WS + 64) == 1         # workspace not 256-byte aligned
    assert call(wsb=need - 1) == 1
    assert b"smaller" in lib.loki_last_error()


@pytest.mark.parametrize("pos,n_new,status", [(-1, 1, 1), (0, 0, 1), (60, 5, 1), (64, 1, 1)])
def test_append_validation(lib, pos, n_new, status):
    c = _cache()
    assert lib.loki_append(ctypes.byref(c), pos, n_new, FAKE, FAKE, FAKE, None) == status


def test_append_pointer_validation(lib):
    c = _cache()
    assert lib.loki_append(ctypes.byref(c), 0, 1, None, FAKE, FAKE, None) == 1
    assert lib.loki_append(ctypes.byref(c), 0, 1, FAKE, FAKE + 4, FAKE, None) == 1
    assert lib.loki_append(ctypes.byref(c), 0, 1, FAKE, FAKE, None, None) == 1
    assert lib.loki_append(None, 0, 1, FAKE, FAKE, FAKE, None) == 1


def _paged(dtype=1, H=2, D=128, page=16, pages=10, k=4096, v=8192, k_lr=None, d_lr=0):
    from sparse_decode_attention_loki_b200 import _lib
    return _lib.loki_paged_cache(dtype, H, D, page, pages, k, v, k_lr, d_lr)


def _seqs(B=2, pps=4, max_len=50, table=FAKE, lens=FAKE):
    from sparse_decode_attention_loki_b200 import _lib
    return _lib.loki_seq_table(B, pps, max_len, table, lens)


def test_paged_workspace_size_and_cache_validation(lib):
    n = ctypes.c_size_t(0)
    c, q = _paged(), _seqs()
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 4, ctypes.byref(n)) == 0
    assert n.value == _ws_bytes(2, 2, 2, 128, 50)
    bad_caches = [_paged(page=24), _paged(page=0), _paged(page=1 << 17), _paged(pages=0), _paged(dtype=5),
                  _paged(H=0), _paged(k=0), _paged(v=FAKE + 8)]
    for bc in bad_caches:
        assert lib.loki_paged_decode_workspace_size(ctypes.byref(bc), ctypes.byref(q), 4, ctypes.byref(n)) == 1
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(_paged(D=96)), ctypes.byref(q), 4,
                                                ctypes.byref(n)) == 2
    # a pool of 2^31 rows (num_pages * Hkv * page_size) is refused, one row less is not
    big = _seqs(pps=1, max_len=50)
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(_paged(H=2, page=1 << 16, pages=1 << 14)),
                                                ctypes.byref(big), 4, ctypes.byref(n)) == 2
    assert b"2^31" in lib.loki_last_error()
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(_paged(H=1, page=1, pages=(1 << 31) - 1)),
                                                ctypes.byref(big), 4, ctypes.byref(n)) == 1  # max_len > 1 token
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(_paged(H=1, page=64, pages=(1 << 25) - 1)),
                                                ctypes.byref(big), 4, ctypes.byref(n)) == 0
    bad_seqs = [_seqs(B=0), _seqs(pps=0), _seqs(max_len=0), _seqs(max_len=65), _seqs(table=None),
                _seqs(table=FAKE + 2), _seqs(lens=FAKE + 2)]
    for bq in bad_seqs:
        assert lib.loki_paged_decode_workspace_size(ctypes.byref(c), ctypes.byref(bq), 4, ctypes.byref(n)) == 1
    assert lib.loki_paged_decode_workspace_size(None, ctypes.byref(q), 4, ctypes.byref(n)) == 1
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(c), None, 4, ctypes.byref(n)) == 1
    # NULL seq_lens is allowed (every sequence at max_seq_len)
    assert lib.loki_paged_decode_workspace_size(ctypes.byref(c), ctypes.byref(_seqs(lens=None)), 4,
                                                ctypes.byref(n)) == 0


def test_paged_decode_validation(lib):
    c, q = _paged(), _seqs()
    need = _ws_bytes(2, 2, 2, 128, 50)
    base = dict(hq=4, qp=FAKE, P=FAKE, d=32, ks=FAKE, kmax=10, out=FAKE, idx=FAKE, ws=WS, wsb=need)
    def call(**kw):
        a = dict(base)
        a.update(kw)
        return lib.loki_paged_decode_attention(ctypes.byref(c), ctypes.byref(q), a["hq"], a["qp"], a["P"], a["d"],
                                               a["ks"], a["kmax"], 0.0, a["out"], a["idx"], a["ws"], a["wsb"], None)
    assert call(d=0) == 1
    assert call(d=129) == 1
    assert call(kmax=0) == 1
    assert call(kmax=51) == 1            # beyond max_seq_len
    assert call(ks=FAKE + 2) == 1
    assert call(idx=None) == 1
    assert call(ws=None) == 1
    assert call(ws=WS + 16) == 1
    assert call(wsb=need - 1) == 1
    assert call(hq=3) == 1
    assert call(hq=6) == 2               # group of 3
    assert call(qp=None) == 1
    assert lib.dense_paged_decode_attention(ctypes.byref(c), ctypes.byref(q), 3, FAKE, FAKE, 0.0, FAKE, None) == 1
    assert lib.dense_paged_decode_attention(ctypes.byref(c), ctypes.byref(q), 4, None, FAKE, 0.0, FAKE, None) == 1


def test_paged_append_validation(lib):
    c, q = _paged(), _seqs()
    assert lib.loki_paged_append(ctypes.byref(c), ctypes.byref(q), None, 1, FAKE, FAKE, FAKE, None) == 1
    assert lib.loki_paged_append(ctypes.byref(c), ctypes.byref(q), FAKE + 2, 1, FAKE, FAKE, FAKE, None) == 1
    assert lib.loki_paged_append(ctypes.byref(c), ctypes.byref(q), FAKE, 0, FAKE, FAKE, FAKE, None) == 1
    assert lib.loki_paged_append(ctypes.byref(c), ctypes.byref(q), FAKE, 1, None, FAKE, FAKE, None) == 1
    assert lib.loki_paged_append(ctypes.byref(c), ctypes.byref(q), FAKE, 1, FAKE, FAKE + 4, FAKE, None) == 1
    assert lib.loki_paged_append(ctypes.byref(c), ctypes.byref(q), FAKE, 1, FAKE, FAKE, None, None) == 1
    assert lib.loki_paged_append(ctypes.byref(_paged(page=3)), ctypes.byref(q), FAKE, 1, FAKE, FAKE, FAKE,
                                 None) == 1


def test_append_decode_validation(lib):
    c = _cache(B=1, H=2, cap=64)
    need = _ws_bytes(1, 2, 1, 128, 10)
    base = (ctypes.byref(c), 10, 2)
    tail = (FAKE, FAKE, 8, 4, 0.0, FAKE, FAKE, WS, need, None)
    assert lib.loki_decode_attention_append(*base, None, FAKE, *tail) == 1
    assert lib.loki_decode_attention_append(*base, FAKE, None, *tail) == 1
    assert lib.loki_decode_attention_append(*base, FAKE + 8, FAKE, *tail) == 1
    assert lib.loki_decode_attention_append(ctypes.byref(c), 65, 2, FAKE, FAKE, *tail) == 1   # seq_len > capacity
    assert lib.loki_decode_attention_append(*base, FAKE, FAKE, FAKE, FAKE, 8, 11, 0.0, FAKE, FAKE, WS, need,
                                            None) == 1   # k > seq_len
    assert lib.dense_decode_attention_append(*base, None, FAKE, FAKE, FAKE, 0.0, FAKE, None) == 1
    assert lib.dense_decode_attention_append(*base, FAKE, FAKE + 4, FAKE, FAKE, 0.0, FAKE, None) == 1
    pc, pq = _paged(), _seqs()
    pneed = _ws_bytes(2, 2, 2, 128, 50)
    assert lib.loki_paged_decode_attention_append(ctypes.byref(pc), ctypes.byref(pq), 4, None, FAKE, FAKE, FAKE, 32,
                                                  None, 10, 0.0, FAKE, FAKE, WS, pneed, None) == 1
    assert lib.loki_paged_decode_attention_append(ctypes.byref(pc), ctypes.byref(pq), 16, FAKE, FAKE, FAKE, FAKE, 32,
                                                  None, 10, 0.0, FAKE, FAKE, WS, _ws_bytes(2, 2, 8, 128), None) == 2


def test_cache_struct_layout():
    # int32 x5, then three pointers from offset 24, then d_lr: the C layout
    from sparse_decode_attention_loki_b200 import _lib
    c = _lib.loki_cache
    assert ctypes.sizeof(c) == 56
    assert (c.k_hat.offset, c.v.offset, c.k_lr.offset, c.d_lr.offset) == (24, 32, 40, 48)


@pytest.mark.parametrize("dtype,D,k_lr,d_lr,status", [
    (1, 128, FAKE, 32, 0),        # bf16 plane of 32 dims (64-byte rows)
    (1, 128, FAKE, 8, 0),         # 16-byte rows
    (1, 128, FAKE, 128, 0),       # the whole key
    (0, 64, FAKE, 4, 0),          # fp32: 16-byte rows
    (1, 128, FAKE, 0, 1),         # empty plane
    (1, 128, FAKE, 12, 1),        # 24-byte rows
    (0, 64, FAKE, 6, 1),          # fp32 24-byte rows
    (1, 128, FAKE, 136, 1),       # wider than the key
    (1, 64, FAKE, 72, 1),
    (1, 128, FAKE + 8, 32, 1),    # misaligned plane
    (1, 128, None, 12, 0),        # no plane: d_lr is ignored
])
def test_lowrank_plane_validation(lib, dtype, D, k_lr, d_lr, status):
    c = _cache(dtype=dtype, D=D, k_lr=k_lr, d_lr=d_lr)
    n = ctypes.c_size_t(0)
    assert lib.loki_decode_workspace_size(ctypes.byref(c), 10, 2, ctypes.byref(n)) == status
    # the append and the decode validate the cache the same way (stopped
    # before any launch by a bad range / a missing q)
    assert lib.loki_append(ctypes.byref(c), 64, 1, FAKE, FAKE, FAKE, None) == 1
    args = (ctypes.byref(c), 10, 2, None, FAKE, 8, 4, 0.0, FAKE, FAKE, WS, WSB, None)
    assert lib.loki_decode_attention(*args) == 1
    if status:
        assert b"plane" in lib.loki_last_error()


def test_paged_lowrank_plane_validation(lib):
    from sparse_decode_attention_loki_b200 import _lib
    assert ctypes.sizeof(_lib.loki_paged_cache) == 56
    n = ctypes.c_size_t(0)
    q = _seqs()
    for k_lr, d_lr, status in [(FAKE, 32, 0), (FAKE, 12, 1), (FAKE, 136, 1), (FAKE + 8, 32, 1), (None, 12, 0)]:
        c = _paged(k_lr=k_lr, d_lr=d_lr)
        assert lib.loki_paged_decode_workspace_size(ctypes.byref(c), ctypes.byref(q), 4, ctypes.byref(n)) == status
        if status:
            assert b"plane" in lib.loki_last_error()


def test_the_abi_is_plain_c(lib):
    # include/loki.h compiles as C99 (pedantic, warnings as errors) and a C
    # program links libloki.so and gets its validation answers (no GPU needed)
    import shutil
    from sparse_decode_attention_loki_b200 import _lib
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "tests", "c_abi", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_check")
    libdir = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-L", libdir, "-lloki",
                        "-Wl,-rpath," + libdir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr
