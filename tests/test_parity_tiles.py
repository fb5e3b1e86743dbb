"""The tile-local parity checks (tests/parity_tiles.py) on the CPU: a result
with one output tile that lost its LoRA term, or one dA block off by a few
percent, passes the whole-tensor relative Frobenius bar but fails the tile
check.  The wrong result is made here, from the oracle's own output; no
kernel is involved."""
import numpy as np
import pytest

import parity_tiles as pt
from bit_nf4_quantized_24_b200 import workloads as wl

TOL = 1e-2


def _bf16_round(x):
    """Round fp64 values to bf16 (round to nearest even), back as fp64: what a
    kernel's bf16 output of the exact value holds."""
    f = np.asarray(x, np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def test_rows_every_tile_covers_every_band():
    for M in (1, 255, 256, 257, 4096, 8192, 1000):
        rows = pt.rows_every_tile(M, seed=3)
        assert rows[0] == 0 and rows[-1] == M - 1
        assert set(np.unique(rows // 256)) == set(range((M + 255) // 256))
        assert np.all(np.diff(rows) > 0)
    assert len(pt.rows_every_tile(4096, 1, per_tile=3)) >= 48


@pytest.fixture(scope="module")
def layer(oracle):
    M, N, K, r = 4096, 2048, 1024, 16
    p = wl.draw_small(4242, M, N, K, r, 32.0)
    oc, oa, od, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(oc, oa, od, N, K)
    rows = pt.rows_every_tile(M, seed=5)
    X16, A16, B16 = wl.bf16_bits(p["X"]), wl.bf16_bits(p["A"]), wl.bf16_bits(p["B"])
    Y = oracle.linear_fwd(X16, Wp, A16, B16, p["scale"], rows=rows)
    Y0 = oracle.linear_fwd(X16, Wp, A16, np.zeros_like(B16), p["scale"], rows=rows)  # base only
    return {"rows": rows, "Y": Y, "Y0": Y0, "M": M, "N": N}


def test_a_tile_without_its_lora_term_fails_only_the_tile_check(layer):
    rows, Y, Y0 = layer["rows"], layer["Y"], layer["Y0"]
    good = _bf16_round(Y)
    assert pt.assert_tiles("Y", good, Y, rows, TOL) < 4e-3  # bf16 output rounding only
    bad = good.copy()
    band, col = 7, 3                                  # token rows 1792..2047, outputs 768..1023
    sel = rows // 256 == band
    bad[sel, 256 * col:256 * (col + 1)] = _bf16_round(Y0[sel, 256 * col:256 * (col + 1)])
    whole = np.linalg.norm(bad - Y) / np.linalg.norm(Y)
    assert whole <= TOL, "the whole-tensor error must hide the fault for this test to mean anything"
    errs = pt.tile_errors(bad, Y, rows)
    k, e = pt.worst(errs)
    assert k == (band, col) and e > TOL
    with pytest.raises(AssertionError):
        pt.assert_tiles("Y", bad, Y, rows, TOL)


def test_a_wrong_dA_block_fails_only_the_block_check(oracle):
    M, N, K, r = 512, 256, 1024, 16
    p = wl.draw_small(4343, M, N, K, r, 32.0)
    oc, oa, od, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(oc, oa, od, N, K)
    _, dA, dB, _ = oracle.linear_bwd(wl.bf16_bits(p["X"]), wl.bf16_bits(p["dY"]), Wp, wl.bf16_bits(p["A"]),
                                     wl.bf16_bits(p["B"]), p["scale"], want_dx=False)
    good = _bf16_round(dA)
    assert pt.assert_blocks("dA", good, dA, TOL) < 4e-3
    bad = good.copy()
    bad[0:16, 512:528] *= 1.05                         # one 16 x 16 block 5 % off
    assert np.linalg.norm(bad - dA) / np.linalg.norm(dA) <= TOL
    k, e = pt.worst(pt.block_errors(bad, dA))
    assert k == (0, 32) and e > TOL
    with pytest.raises(AssertionError):
        pt.assert_blocks("dA", bad, dA, TOL)
    assert pt.assert_blocks("dB", _bf16_round(dB), dB, TOL) < 4e-3


def test_blocks_with_zero_reference_are_skipped():
    ref = np.zeros((32, 32))
    ref[:16, :16] = 1.0
    got = ref.copy()
    got[16:, 16:] = 5.0  # nonzero where the reference is zero: not a relative error
    assert set(pt.block_errors(got, ref)) == {(0, 0)}
