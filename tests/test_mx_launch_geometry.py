"""Launch geometry of the block-scaled MXFP8 expert FFN (csrc/expert_ffn_mx.cu),
replayed on the CPU (CPU only).

For the schedules of the seeded workloads, every tile the grouped raster
hands out is expanded into the coordinates its TMA loads and stores name and
the bytes its epilogue writes; all of them must lie inside the tensor maps
and buffers the launcher builds, every output tile must be produced exactly
once, and the shared-memory and TMEM budgets must hold for every expert count
the ABI accepts. This restates the kernel's index arithmetic in numpy; it is
the bounds check to run before the kernel's first launch on a GPU.
"""
import numpy as np
import pytest

import oracle
from combine_top_route_counting_b200 import inputs

BM, RM = 256, 8                  # pair-tile rows; M-tiles per raster chunk
BK = 128                         # E4M3 values per pipeline stage
SMEM_LIMIT = 232448              # 227 KB of dynamic shared memory per CTA
K_RING = 4


# per MODE: tile columns, accumulators, stages, B rows per CTA, scale atoms of B
GEOM = {0: dict(BN=256, ACC=1, STAGES=6, B_ROWS=128, SFB=2),
        1: dict(BN=128, ACC=2, STAGES=7, B_ROWS=64, SFB=1)}


def _smem_bytes(mode: int, E: int) -> int:
    g = GEOM[mode]
    stage = 128 * BK + g["B_ROWS"] * BK
    sf_stage = 512 * (1 + g["SFB"])
    staging = 8 * 4096 if mode == 1 else 0
    num_bars = 2 * g["STAGES"] + 2 * g["ACC"] + 1 + 2 * K_RING
    return (1024 + g["STAGES"] * (stage + sf_stage) + staging + num_bars * 8 + 16 + K_RING * 4
            + (2 * E + 1) * 4)


def _tiles(s_off: np.ndarray, s_end: np.ndarray, E: int, tiles_n: int):
    """The grouped raster (N-block-major inside chunks of RM M-tiles): tile ->
    (valid, row0, n, l) for every tile id of the launch."""
    num_tiles = (int(s_off[E]) // BM) * tiles_n
    t = np.arange(num_tiles, dtype=np.int64)
    u = t // tiles_n
    l = np.searchsorted(s_off[:E] // BM, u, side="right") - 1   # largest l with S[l]/BM <= u
    m0 = s_off[l] // BM
    mcount = s_off[l + 1] // BM - m0
    j = t - m0 * tiles_n
    mc = j // (RM * tiles_n)
    rows = np.minimum(RM, mcount - mc * RM)
    jj = j - mc * RM * tiles_n
    ng = jj // rows                              # RN = 1: one column block per group
    rr = jj - ng * rows
    n = ng
    row0 = (m0 + mc * RM + rr) * BM
    return row0 < s_end[l], row0, n, l


def _check_mode(mode: int, sh: dict, s_off, s_end, rows_max: int):
    E, H, I = sh["E"], sh["H"], sh["I"]
    K, Nout = (H, I) if mode == 0 else (I, H)
    tiles_n = Nout // 128
    kb_max = K // BK - 1
    valid, row0, n, l = _tiles(s_off, s_end, E, tiles_n)
    # a tile never straddles two experts, and every (row tile, column block)
    # of the experts' segments comes exactly once
    assert ((row0 >= s_off[l]) & (row0 + BM <= s_off[l + 1])).all()
    keys = (row0 // BM) * tiles_n + n
    assert len(np.unique(keys)) == len(keys) == (int(s_off[E]) // BM) * tiles_n
    row0, n, l = row0[valid], n[valid], l[valid]
    for rank in (0, 1):
        arow = row0 + 128 * rank
        # A codes: box 128 x 128 at (kb * 128, arow) of [rows_max, K]
        assert (kb_max * BK + BK <= K) and (arow + 128 <= rows_max).all()
        # A scale atoms: (arow / 128) * K/128 + kb < rows_max/128 * K/128
        assert ((arow // 128) * (K // BK) + kb_max < rows_max // 128 * (K // BK)).all()
        if mode == 0:
            brow = l * I + n * 128                       # W1t / W3t rows
            assert (brow + 128 <= E * I).all()
            assert ((brow // 128) * (K // BK) + kb_max < E * I // 128 * (K // BK)).all()
        else:
            brow = l * H + n * 128                       # W2t rows of the tile
            assert (brow + 64 * rank + 64 <= E * H).all()
            assert ((brow // 128) * (K // BK) + kb_max < E * H // 128 * (K // BK)).all()
    # epilogue: rows row0 .. row0 + 255 of the tile
    last_row = row0 + 255
    assert (last_row < rows_max).all()
    if mode == 0:
        last_col = n * 128 + 64 + 32                     # half 1, chunk 1: 32 codes
        assert (last_col <= I).all()
        kblk = I // 32
        last_sc = ((last_row // 128) * (kblk // 4) + (kblk - 1) // 4) * 512 + 31 * 16 + 3 * 4 + 3
        assert (last_sc < rows_max * I // 32).all()
    else:
        # y: 32 x 32 fp32 boxes at (n*128 + half*64 + c*32, row0 + rank*128 + q*32)
        assert (n * 128 + 64 + 32 + 32 <= H).all()


@pytest.mark.parametrize("name", ["tiny", "tiny_bwd", "mid", "kimi", "zipf", "kimi_e16"])
def test_mx_ffn_tiles_stay_inside_their_buffers(name):
    w = inputs.WORKLOADS[name]
    sh = w.shape()
    ids, _, _ = oracle.route_topk(inputs.make_logits(w), w.k)
    s = oracle.schedule(ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, w.pad)
    s_off = s["offsets"].astype(np.int64)
    s_end = s_off[:-1] + s["counts"].sum(axis=1)
    rows_max = (w.P * w.N * w.k + w.E * (w.pad - 1) + 255) // 256 * 256
    assert s_off[-1] <= rows_max and (s_off % BM == 0).all()
    for mode in (0, 1):
        _check_mode(mode, sh, s_off, s_end, rows_max)


@pytest.mark.parametrize("E", [1, 8, 384, 1024])
def test_mx_ffn_budgets(E):
    for mode in (0, 1):
        g = GEOM[mode]
        assert _smem_bytes(mode, E) <= SMEM_LIMIT
        sf_cols = 8 if g["SFB"] == 1 else 16
        assert g["ACC"] * g["BN"] + g["STAGES"] * sf_cols <= 512   # accumulators + scales
        assert 4 * (1 + g["SFB"]) <= sf_cols                        # A atom + B atoms per stage
        assert (g["ACC"] * g["BN"]) % 4 == 0 and sf_cols % 4 == 0   # copies start on 4 columns


@pytest.mark.parametrize("E,K,N", [(1, 128, 128), (3, 256, 384), (384, 7168, 2048), (384, 2048, 7168)])
def test_mx_weight_quantisation_blocks_stay_inside_their_buffers(E, K, N):
    """mx_weights_kernel: block b -> (expert, 128-row K tile, 64-column N tile);
    each thread reads one column's 32-value K block and writes 32 codes of the
    transposed row and one tiled scale."""
    tiles_n, tiles_k = N // 64, K // 128
    blocks = E * tiles_k * tiles_n
    assert blocks < 2 ** 31
    b = np.array([0, 1, tiles_n - 1, tiles_n, blocks // 2, blocks - 1], dtype=np.int64)
    b = b[b < blocks]
    nt, kt, e = b % tiles_n, (b // tiles_n) % tiles_k, b // (tiles_n * tiles_k)
    assert (e < E).all()
    # loads: rows e*K + kt*128 + [0, 128), columns nt*64 + [0, 64) of [E*K, N]
    assert ((e * K + kt * 128 + 127) * N + nt * 64 + 63 < E * K * N).all()
    # stores: row e*N + nt*64 + n (n < 64), codes [32 (kt*4 + j), +32) of a K-row
    row = e * N + nt * 64 + 63
    assert ((row * K + (kt * 4 + 3) * 32 + 32) <= E * N * K).all()
    kblk = K // 32
    sc = ((row // 128) * (kblk // 4) + (kt * 4 + 3) // 4) * 512 + (row % 32) * 16 + ((row // 32) % 4) * 4 + 3
    assert (sc < E * N * K // 32).all()
