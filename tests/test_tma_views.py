"""Host checks of the TMA views the expert-FFN kernels read their weights through.

The views' extents, strides and boxes come from the library's own `csrc/tmap.cuh`
(compiled here with the host compiler; no driver call).  For every box the kernels
place -- the CTA-pair kernel's fragment-order 128-row boxes, the decode kernel's
(gate, up) pair boxes, bf16 and int8, interleaved and chunked fc1 -- each in-bounds
element must lie inside the weight tensor (TMA fills out-of-range coordinates with
zeros, but checks no footprint), and every row a kernel keeps must be the weight row
its epilogue assumes: box row 32 Q + 8 q + j = the expert's row r0 + 32 Q + 4 j + q
(fragment order), box row 2 i + s = row 2 (i0 + i) + s of the interleaved order
(pair order), where chunked fc1 stores interleaved row 2 i + s at row s I + i.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixture_experts_ffn_15_b200", "csrc")
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")

# (E, I, H): sizes both kernels accept (I a multiple of 64, H of 128), with ragged
# 256-row pair tiles (2I = 1408, 384, 640) and a single expert
SIZES = [(1, 64, 128), (3, 192, 256), (5, 320, 384), (8, 704, 2816), (2, 1536, 4096)]


@pytest.fixture(scope="module")
def views_bin(tmp_path_factory):
    if shutil.which("g++") is None or not os.path.exists(os.path.join(CUDA_INC, "cuda.h")):
        pytest.skip("needs g++ and the CUDA headers")
    out = str(tmp_path_factory.mktemp("views") / "tma_views")
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-I", CSRC, "-I", CUDA_INC,
                        os.path.join(ROOT, "tests", "tma_views_main.cpp"), "-o", out],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def read_views(binary, E, I, H):
    r = subprocess.run([binary, str(E), str(I), str(H)], capture_output=True, text=True, check=True)
    views = {}
    for line in r.stdout.splitlines():
        f = line.split()
        name = f[0]
        assert f[1] != "refused", f"{name} refused for E={E} I={I} H={H}"
        rank, eb = int(f[1]), int(f[2])
        v = [int(x) for x in f[3:]]
        views[name] = dict(rank=rank, elem=eb, dims=v[:rank], strides=v[rank:2 * rank - 1],
                           box=v[2 * rank - 1:3 * rank - 1])
    return views


def box_rows(view, coords):
    """(box row index, byte offset of the row) of every in-bounds row of one box; the
    row dimensions are 1 .. rank-1, box rows numbered with dimension 1 fastest."""
    dims, strides, box = view["dims"], view["strides"], view["box"]
    rank = view["rank"]
    rows = []
    n = 1
    for d in range(1, rank):
        n *= box[d]
    for idx in range(n):
        rem, off, inside = idx, 0, True
        for d in range(1, rank):
            b = rem % box[d]
            rem //= box[d]
            c = coords[d] + b
            if c < 0 or c >= dims[d]:
                inside = False
                break
            off += c * strides[d - 1]
        if inside:
            rows.append((idx, off))
    return rows


def check_common(view, K):
    elem = view["elem"]
    assert view["dims"][0] == K
    assert all(s % 16 == 0 for s in view["strides"]), view["strides"]
    # one box row is one swizzle row: 128 bytes of bf16 (64 bytes of int8)
    assert view["box"][0] * elem == (64 if elem == 1 else 128)
    assert all(1 <= b <= 256 for b in view["box"])


def check_fragment_order(view, E, n, K, chunked_I=None):
    """The pair kernel: unit weight tile mt of 256 rows, CTA rank r, first row
    w_in = 256 mt + 128 r (interleaved order for fc1)."""
    check_common(view, K)
    elem = view["elem"]
    row_bytes = K * elem
    total = E * n * row_bytes
    for g in range(E):
        for mt in range((n + 255) // 256):
            for r in range(2):
                w_in = 256 * mt + 128 * r
                if chunked_I is None:
                    coords = [0, 0, 0, w_in // 32, g]
                else:
                    coords = [0, 0, 0, 0, g * (chunked_I // 8) + w_in // 32]
                for idx, off in box_rows(view, coords):
                    assert off + row_bytes <= total, (g, mt, r, idx, off)
                    Q, q, j = idx // 32, (idx % 32) // 8, idx % 8
                    lr = w_in + 32 * Q + 4 * j + q        # the epilogue's row of this lane
                    if lr >= n:
                        continue                            # dropped by the epilogue
                    if chunked_I is None:
                        want = g * n + lr
                    else:
                        want = g * n + (lr % 2) * chunked_I + lr // 2
                    assert off == want * row_bytes, (g, mt, r, idx, off // row_bytes, want)


def check_pair_order(view, E, n, K, chunked_I=None):
    """The decode kernel: m-tile mt of 128 rows, box of 64 (gate, up) pairs from pair
    64 mt; box row 2 i + s."""
    check_common(view, K)
    elem = view["elem"]
    row_bytes = K * elem
    total = E * n * row_bytes
    for g in range(E):
        for mt in range(n // 128):
            coords = [0, 0, 64 * mt, g]
            for idx, off in box_rows(view, coords):
                assert off + row_bytes <= total, (g, mt, idx, off)
                s, i = idx % 2, idx // 2
                pair = 64 * mt + i
                want = g * n + (s * chunked_I + pair if chunked_I else 2 * pair + s)
                assert off == want * row_bytes, (g, mt, idx, off // row_bytes, want)


@pytest.mark.parametrize("E,I,H", SIZES)
def test_pair_kernel_fragment_order_views(views_bin, E, I, H):
    v = read_views(views_bin, E, I, H)
    check_fragment_order(v["pair_fc1_interleaved"], E, 2 * I, H)
    check_fragment_order(v["pair_fc1_chunked"], E, 2 * I, H, chunked_I=I)
    check_fragment_order(v["pair_fc2"], E, H, I)


@pytest.mark.parametrize("E,I,H", SIZES)
def test_decode_kernel_pair_order_views(views_bin, E, I, H):
    v = read_views(views_bin, E, I, H)
    for sfx in ("", "_u8"):
        check_pair_order(v["decode_fc1_interleaved" + sfx], E, 2 * I, H)
        check_pair_order(v["decode_fc1_chunked" + sfx], E, 2 * I, H, chunked_I=I)
        check_pair_order(v["decode_fc2" + sfx], E, H, I)


def test_views_refuse_sizes_they_cannot_tile(views_bin):
    # 2I not a multiple of 32 has no fragment-order view; I not a multiple of 16 no
    # chunked one
    r = subprocess.run([views_bin, "2", "8", "128"], capture_output=True, text=True, check=True)
    refused = {l.split()[0] for l in r.stdout.splitlines() if l.endswith("refused")}
    assert {"pair_fc1_interleaved", "pair_fc1_chunked"} <= refused
