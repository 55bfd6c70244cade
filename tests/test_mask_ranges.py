"""Host-side check of the tile-range arithmetic that both passes use for masks (MaskSpec in the
CUDA library's kernels.h): the range functions are compiled for the CPU and compared with brute
force over the visibility rule (key j visible to query i iff i+off-wl <= j <= i+off+wr, off =
nk-nq, negative bound = unbounded; "Attention Mechanism ...", §4.4 causal, §4.5 sliding window,
§4.2 cross-attention). The forward pass's key-tile ranges, the backward pass's query-tile ranges
and the deterministic mode's first key tile must describe the same set of (query tile, key tile)
pairs, and that set must be exactly the pairs holding a visible (query, key)."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR_DIR = os.path.join(ROOT, "exact_attention_138_b200", "csrc")

SHIM = r"""
#include "kernels.h"
using namespace attn;
static MaskSpec spec(int nq, int nk, int wl, int wr) {
    return MaskSpec{nq, nk, wl, wr, (long long)nk - nq};
}
extern "C" void keys(int nq, int nk, int wl, int wr, long long a, long long b, long long* out) {
    visible_keys(spec(nq, nk, wl, wr), a, b, out[0], out[1]);
}
extern "C" void qtiles(int nq, int nk, int wl, int wr, long long c, long long e, int bq, int* out) {
    visible_query_tiles(spec(nq, nk, wl, wr), c, e, bq, out[0], out[1]);
}
extern "C" int first_ktile(int nq, int nk, int wl, int wr, long long a, int bk) {
    return first_key_tile(spec(nq, nk, wl, wr), a, bk);
}
extern "C" int last_ktile(int nq, int nk, int wl, int wr, long long a, int bq, int bk) {
    return last_key_tile(spec(nq, nk, wl, wr), a, bq, bk);
}
"""


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    gxx = shutil.which("g++")
    cuda_inc = "/usr/local/cuda/include"
    if gxx is None or not os.path.isdir(cuda_inc):
        pytest.skip("g++ or the CUDA headers are not available")
    d = tmp_path_factory.mktemp("maskshim")
    src = d / "shim.cpp"
    src.write_text(SHIM)
    so = d / "shim.so"
    subprocess.run([gxx, "-std=c++17", "-O1", "-fPIC", "-shared", "-I", HDR_DIR, "-I", cuda_inc,
                    str(src), "-o", str(so)], check=True)
    L = ctypes.CDLL(str(so))
    LL = ctypes.c_longlong
    L.keys.argtypes = [ctypes.c_int] * 4 + [LL, LL, ctypes.POINTER(LL)]
    L.qtiles.argtypes = [ctypes.c_int] * 4 + [LL, LL, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    L.first_ktile.argtypes = [ctypes.c_int] * 4 + [LL, ctypes.c_int]
    L.first_ktile.restype = ctypes.c_int
    L.last_ktile.argtypes = [ctypes.c_int] * 4 + [LL, ctypes.c_int, ctypes.c_int]
    L.last_ktile.restype = ctypes.c_int
    return L


def visibility(nq, nk, wl, wr):
    i = np.arange(nq)[:, None] + (nk - nq)
    j = np.arange(nk)[None, :]
    vis = np.ones((nq, nk), bool)
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    return vis


CASES = [(300, 300, -1, 0), (300, 300, -1, -1), (300, 300, 5, 5), (300, 300, 0, 0),
         (300, 300, 130, 0), (257, 700, -1, 0), (700, 257, -1, 0), (700, 257, -1, -1),
         (100, 1000, 20, 3), (1000, 100, 3, 20), (129, 129, 127, 128), (64, 640, 0, 0),
         (513, 130, 200, 0), (1, 1, -1, 0), (1, 500, 10, 10), (500, 1, -1, 0), (383, 383, 64, 64)]


@pytest.mark.parametrize("nq,nk,wl,wr", CASES)
def test_key_ranges_of_query_tiles(lib, nq, nk, wl, wr):
    vis = visibility(nq, nk, wl, wr)
    out = (ctypes.c_longlong * 2)()
    for a in range(0, nq, 128):
        b = min(a + 127, nq - 1)
        lib.keys(nq, nk, wl, wr, a, b, out)
        cols = np.nonzero(vis[a:b + 1].any(0))[0]
        if cols.size == 0:
            assert out[0] > out[1]
        else:
            assert (out[0], out[1]) == (cols[0], cols[-1])
            assert cols.size == cols[-1] - cols[0] + 1           # contiguous
    for i in range(nq):                                           # single rows too
        lib.keys(nq, nk, wl, wr, i, i, out)
        cols = np.nonzero(vis[i])[0]
        if cols.size == 0:
            assert out[0] > out[1]
        else:
            assert (out[0], out[1]) == (cols[0], cols[-1]) and cols.size == out[1] - out[0] + 1


@pytest.mark.parametrize("nq,nk,wl,wr", CASES)
@pytest.mark.parametrize("bq", [64, 128])
def test_both_passes_agree_on_tile_pairs(lib, nq, nk, wl, wr, bq):
    vis = visibility(nq, nk, wl, wr)
    nqt, nkt = -(-nq // bq), -(-nk // 128)
    exact = np.zeros((nqt, nkt), bool)
    for t in range(nqt):
        for s in range(nkt):
            exact[t, s] = vis[t * bq:(t + 1) * bq, s * 128:(s + 1) * 128].any()
    # backward: query tiles per key tile
    out = (ctypes.c_int * 2)()
    bwd = np.zeros_like(exact)
    for s in range(nkt):
        lib.qtiles(nq, nk, wl, wr, s * 128, min(s * 128 + 127, nk - 1), bq, out)
        bwd[out[0]:out[1], s] = True
    assert np.array_equal(bwd, exact)
    # forward: key tiles per query tile (tiles of bq rows)
    o2 = (ctypes.c_longlong * 2)()
    fwd = np.zeros_like(exact)
    for t in range(nqt):
        lib.keys(nq, nk, wl, wr, t * bq, min(t * bq + bq - 1, nq - 1), o2)
        if o2[0] <= o2[1]:
            fwd[t, o2[0] // 128:o2[1] // 128 + 1] = True
    assert np.array_equal(fwd, exact)
    # deterministic ordering: the first and last key tiles met by each query tile
    for t in range(nqt):
        if exact[t].any():
            assert lib.first_ktile(nq, nk, wl, wr, t * bq, 128) == np.nonzero(exact[t])[0][0]
            assert lib.last_ktile(nq, nk, wl, wr, t * bq, bq, 128) == np.nonzero(exact[t])[0][-1]


def test_full_visibility_test_matches_brute_force(lib):
    # a (query tile, key tile) pair needs no mask iff the keys seen by every row of the tile, i.e.
    # visible_keys(last row, first row), cover the key tile
    out = (ctypes.c_longlong * 2)()
    for nq, nk, wl, wr in CASES:
        vis = visibility(nq, nk, wl, wr)
        for a in range(0, nq, 64):
            for c in range(0, nk, 128):
                b = a + 63
                lib.keys(nq, nk, wl, wr, b, a, out)
                claim = out[0] <= c and c + 127 <= out[1]
                rows = min(b, nq - 1)
                truth = (c + 128 <= nk) and vis[a:rows + 1, c:c + 128].all() and b < nq
                # the claim may be conservative only for the partial last query tile
                if claim:
                    assert vis[a:rows + 1, c:c + 128].all() and c + 128 <= nk
                if truth:
                    assert claim
