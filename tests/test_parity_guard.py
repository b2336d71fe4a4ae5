"""The GPU parity tests' own checks, pinned on the CPU: the bf16 per-element
guard passes the oracle's own rounded output and fails one wrong element, and
the tile-covering row choice puts a checked row in every m-tile."""
import numpy as np
import pytest

import oracle
from gpu_helpers import assert_elementwise, compact_rows, tile_cover_tokens
from mixture_experts_sparse_b200 import inputs


def _layer(T=512, d=256, dff=512, N=8, k=1, cf=2.0, seed=3):
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, dtype="bf16", seed=seed)
    C = oracle.capacity(T, N, k, cf)
    W = {key: L[key] for key in ("w1", "b1", "w3", "b3", "w2", "b2")}
    return L, oracle.forward(L["x"], L["w_r"], L["b_r"], W, k=k, C=C, out_dtype=oracle.BF16)


def test_guard_passes_rounding_and_fails_one_wrong_element():
    _, res = _layer()
    ref = res["out_exact"]
    got = res["out"].astype(np.float64)          # the oracle's own bf16-rounded output
    assert_elementwise(got, ref)
    for (r, c, src) in [(100, 17, 200), (0, 0, 255), (511, 128, 3)]:
        if ref[r].any():
            bad = got.copy()
            bad[r, c] = got[r, src]               # a value from another column, as a wrong tile would give
            with pytest.raises(AssertionError):
                assert_elementwise(bad, ref)
    bad = got.copy()
    bad[7] = 0.0                                  # a kept token's row lost
    if ref[7].any():
        with pytest.raises(AssertionError):
            assert_elementwise(bad, ref)


def test_guard_dropped_rows_must_be_exact_zeros():
    ref = np.zeros((2, 8))
    assert_elementwise(np.zeros((2, 8)), ref)
    got = np.zeros((2, 8))
    got[1, 3] = 1e-30
    with pytest.raises(AssertionError):
        assert_elementwise(got, ref)


@pytest.mark.parametrize("block", [128, 256])
def test_tile_cover_hits_every_block(block):
    L, res = _layer(T=3000, N=5, k=2, cf=1.0, seed=8)
    idx, disp = res["routing"]["idx"], res["disp"]
    toks = set(tile_cover_tokens(idx, disp, block).tolist())
    row_token, row_expert = compact_rows(idx, disp)
    off = disp["offsets"]
    for e in range(off.size - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        for b in range(lo, hi, block):
            rows = range(b, min(b + block, hi))
            assert any(int(row_token[r]) in toks for r in rows), (e, b)
            assert int(row_token[min(b + block, hi) - 1]) in toks     # last row of the tile
