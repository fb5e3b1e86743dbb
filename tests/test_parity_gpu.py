"""Parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Bars: NF4 codes, absmax codes and double-quant scales bit-exact; dequantized
bf16 weights bit-exact; Y, dX, dA, dB within a relative Frobenius error of 1e-2
(the layer's stated tolerance; the expected error is the bf16 rounding of the
outputs, ~3e-3), both over the whole tensor and tile by tile: every 256-token x
256-output tile of Y and dX and every 16 x 16 block of dA and dB must meet it on
its own (tests/parity_tiles.py), so a fault confined to one tile cannot hide in
the norm of the rest.  Small cases span several tiles with ragged tails and are
checked in full; the five workloads are checked at full size on rows sampled
from every 256-token tile (plus the last, ragged row) of Y and dX and on all of
dA and dB, with the same launches the benchmark times.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import parity_tiles as pt
from bit_nf4_quantized_24_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def qb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_nf4_quantized_24_b200 import binding, build
    build.build()
    binding.lib()
    return binding


def relfro(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.linalg.norm(got - ref)
    n = np.linalg.norm(ref)
    return d / n if n > 0 else d


def bits(t):
    return wl.bf16_bits(t.cpu())


def quantize_both(qb, oracle, W, block=64, dq_block=256):
    """GPU and oracle quantization of the same fp32 weight; asserts bit-exact."""
    q = qb.nf4_quantize(W.cuda(), block, dq_block)
    oc, oa, od, _ = oracle.nf4_quantize(W.numpy(), block=block, dq_block=dq_block)
    assert np.array_equal(q.codes.cpu().numpy(), oc), "NF4 codes differ"
    assert np.array_equal(q.absmax_q.cpu().numpy(), oa), "absmax codes differ"
    assert q.dq_scale.cpu().numpy().tobytes() == od.tobytes(), "scales differ"
    _, Wp = oracle.nf4_dequantize(oc, oa, od, W.shape[0], W.shape[1], block=block, dq_block=dq_block)
    return q, Wp


def run_fwd_check(qb, oracle, p, rows=None, q=None, Wp=None):
    if q is None:
        q, Wp = quantize_both(qb, oracle, p["W"])
    X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
    Y, H = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    torch.cuda.synchronize()
    Yref = oracle.linear_fwd(bits(p["X"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"], rows=rows)
    Yg = Y.float().cpu().numpy()
    if rows is not None:
        Yg = Yg[rows]
    e = relfro(Yg, Yref)
    assert e <= TOL, f"Y rel err {e}"
    pt.assert_tiles("Y", Yg, Yref, rows if rows is not None else np.arange(Yg.shape[0]), TOL)
    Href = oracle.lora_h(bits(p["X"][rows] if rows is not None else p["X"]), bits(p["A"]))
    Hg = H.float().cpu().numpy()
    eh = relfro(Hg[rows] if rows is not None else Hg, Href)
    assert eh <= TOL, f"H rel err {eh}"
    return e, q, Wp


def run_bwd_check(qb, oracle, p, rows=None, q=None, Wp=None, use_saved_h=True):
    if q is None:
        q, Wp = quantize_both(qb, oracle, p["W"])
    X, A, B, dY = p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["dY"].cuda()
    H = None
    if use_saved_h:
        _, H = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    dX, dA, dB = qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"], H=H)
    torch.cuda.synchronize()
    dXr, dAr, dBr, _ = oracle.linear_bwd(bits(p["X"]), bits(p["dY"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"],
                                         rows=rows)
    dXg = dX.float().cpu().numpy()
    if rows is not None:
        dXg = dXg[rows]
    dAg, dBg = dA.float().cpu().numpy(), dB.float().cpu().numpy()
    errs = (relfro(dXg, dXr), relfro(dAg, dAr), relfro(dBg, dBr))
    assert max(errs) <= TOL, f"dX/dA/dB rel err {errs}"
    pt.assert_tiles("dX", dXg, dXr, rows if rows is not None else np.arange(dXg.shape[0]), TOL)
    pt.assert_blocks("dA", dAg, dAr, TOL)
    pt.assert_blocks("dB", dBg, dBr, TOL)
    return errs


@pytest.mark.parametrize("M,N,K", [(600, 2048, 2048), (1100, 2048, 3072)])
def test_split_tiles_match_whole_tiles(qb, oracle, M, N, K):
    """Shapes whose tiles leave a partial last wave run those tiles split along
    the contraction (fp32 partial sums added in piece order by a second
    kernel).  With the workspace the plan asks for, Y and dX match the oracle
    tile by tile, repeat bit for bit, and agree with a run whose workspace has
    no room for the partial sums (every tile whole) to fp32 summation order."""
    r = 16
    for mode in (0, 1):
        ns, nt, pb = qb.gemm_split_plan(mode, M, N, K)
        assert ns >= 2 and nt >= 1 and pb == nt * ns * 512 * 256 * 4, (mode, ns, nt, pb)
    p = wl.draw_small(1200 + M, M, N, K, r, 2.0 * r)
    q, Wp = quantize_both(qb, oracle, p["W"])
    X, A, B, dY = p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["dY"].cuda()
    full_f = torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    small_f = torch.empty(full_f.numel() - qb.gemm_split_plan(0, M, N, K)[2], dtype=torch.uint8, device="cuda")
    Y1, H = qb.qlora_linear_fwd(q, X, A, B, p["scale"], workspace=full_f)
    Y2, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"], workspace=full_f)
    L, P = qb.lib(), qb._ptr
    Yw = torch.empty_like(Y1)  # a workspace without room for the partial sums (the binding would enlarge it)
    assert L.qlora_linear_fwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(X), M, P(A), P(B), r,
                              ctypes.c_float(p["scale"]), P(Yw), None, P(small_f), small_f.numel(), None) == 0
    full_b = torch.empty(qb.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    small_b = torch.empty(full_b.numel() - qb.gemm_split_plan(1, M, N, K)[2], dtype=torch.uint8, device="cuda")
    dX1, _, _ = qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"], H=H, workspace=full_b)
    dX2, _, _ = qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"], H=H, workspace=full_b)
    dXw, dAw, dBw = torch.empty_like(dX1), torch.empty(r, K, dtype=torch.bfloat16, device="cuda"), \
        torch.empty(N, r, dtype=torch.bfloat16, device="cuda")
    assert L.qlora_linear_bwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(X), P(dY), M, P(A), P(B), r,
                              ctypes.c_float(p["scale"]), P(H), P(dXw), P(dAw), P(dBw), P(small_b), small_b.numel(),
                              None) == 0
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(dX1, dX2), "split tiles are not repeatable"
    assert relfro(Y1.float().cpu().numpy(), Yw.float().cpu().numpy()) < 2e-3
    assert relfro(dX1.float().cpu().numpy(), dXw.float().cpu().numpy()) < 2e-3
    rows = pt.rows_every_tile(M, 1300 + M, per_tile=2)
    Yref = oracle.linear_fwd(bits(p["X"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"], rows=rows)
    pt.assert_tiles("Y", Y1.float().cpu().numpy()[rows], Yref, rows, TOL)
    dXr, _, _, _ = oracle.linear_bwd(bits(p["X"]), bits(p["dY"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"],
                                     rows=rows)
    pt.assert_tiles("dX", dX1.float().cpu().numpy()[rows], dXr, rows, TOL)


# ------------------------------------------------------------------ codec


@pytest.mark.parametrize("N,K,seed", [(1, 64, 0), (3, 192, 1), (5, 320, 2), (37, 4160, 3), (300, 1024, 4)])
def test_quantize_bit_exact(qb, oracle, N, K, seed):
    W = wl.draw_weight(wl.generator(seed), N, K, 0.02, 0.02)
    W[0, :64] = 0.0                      # an all-zero block
    if N > 2:
        W[2, :] *= 1e-30                 # tiny magnitudes
    quantize_both(qb, oracle, W)


def test_quantize_codebook_values_and_ties(qb, oracle):
    _, l32, m32 = oracle.nf4_codebook()
    rows = []
    for e in (-7, 0, 3):
        idx = np.arange(64) % 16
        rows.append(l32[idx] * np.float32(2.0 ** e))
    for i in range(15):
        r = np.zeros(64, np.float32)
        r[0] = 1.0
        r[1] = m32[i]
        r[2] = np.nextafter(m32[i], np.float32(2))
        r[3] = np.nextafter(m32[i], np.float32(-2))
        r[4:] = np.float32(-1.0)
        rows.append(r)
    W = torch.from_numpy(np.stack(rows).astype(np.float32))
    quantize_both(qb, oracle, W)


def test_quantize_near_midpoints_any_scale(qb, oracle):
    """Weights within a few ulps of m * midpoint for block absmax m of every
    size (not powers of two), so that the quotient w / m lands next to a
    midpoint: the GPU's division and code lookup must match the oracle's
    IEEE division and midpoint count bit for bit."""
    _, _, m32 = oracle.nf4_codebook()
    g = np.random.default_rng(123)
    rows = []
    for e in (-110, -60, -20, -7, -1, 0, 3, 40, 90, 110):
        for _ in range(40):
            m = np.float32(g.uniform(1.0, 2.0) * 2.0 ** e)
            r = np.empty(64, np.float32)
            r[0] = m
            for j in range(1, 64):
                mid = m32[g.integers(0, 15)]
                w = np.float32(np.float64(mid) * np.float64(m))
                for _ in range(int(g.integers(-3, 4))):
                    w = np.nextafter(w, np.float32(np.inf) if g.random() < 0.5 else np.float32(-np.inf))
                r[j] = np.clip(w, -m, m)
            rows.append(r)
    W = torch.from_numpy(np.stack(rows).astype(np.float32))
    quantize_both(qb, oracle, W)


@pytest.mark.parametrize("block", [32, 64, 128, 256])
@pytest.mark.parametrize("dq_block", [256, 0])
def test_codec_other_formats_bit_exact(qb, oracle, block, dq_block):
    """Every block size with and without double quantization: codes, absmax
    codes and scales bit-exact; the dequantized weight bit-exact.  37 rows of
    2048 make the last group of 256 blocks ragged for every block size."""
    N, K = 37, 2048
    W = wl.draw_weight(wl.generator(500 + block + dq_block), N, K, 0.02, 0.02)
    W[0, :block] = 0.0  # an all-zero block
    W[3, :] *= 1e-30    # tiny magnitudes
    q, Wp = quantize_both(qb, oracle, W, block, dq_block)
    assert (q.block, q.dq_block) == (block, dq_block)
    Wd = qb.nf4_dequantize(q)
    o16, _ = oracle.nf4_dequantize(q.codes.cpu().numpy(), q.absmax_q.cpu().numpy(), q.dq_scale.cpu().numpy(),
                                   N, K, block=block, dq_block=dq_block)
    assert np.array_equal(Wd.view(torch.int16).cpu().numpy().view(np.uint16), o16)


@pytest.mark.parametrize("block,dq_block", [(32, 256), (128, 0), (256, 256), (64, 0), (128, 256), (256, 0)])
def test_layer_other_formats(qb, oracle, block, dq_block):
    """Every codec format through the layer: the fused GEMM (forward and
    backward at a GEMM size) and, at a decode size, the row-major decode
    kernel and the decode-tile kernel (blocks 64 to 256; block 32 keeps the
    GEMM), against the oracle's dequantized weight of the same format."""
    M, N, K, r = 150, 264, 1024, 16
    p = wl.draw_small(600 + block + dq_block, M, N, K, r, 2.0 * r)
    q, Wp = quantize_both(qb, oracle, p["W"], block, dq_block)
    run_fwd_check(qb, oracle, p, q=q, Wp=Wp)
    run_bwd_check(qb, oracle, p, q=q, Wp=Wp)
    for Md in (5, 12):
        p2 = dict(p)
        p2["X"] = p["X"][:Md].contiguous()
        run_fwd_check(qb, oracle, p2, q=q, Wp=Wp)
        if block >= 64:
            T = qb.nf4_decode_tiles(q)
            Y, _ = qb.qlora_linear_fwd_tiles(q, T, p2["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["scale"])
            torch.cuda.synchronize()
            Yref = oracle.linear_fwd(bits(p2["X"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"])
            assert relfro(Y.float().cpu().numpy(), Yref) <= TOL
        else:
            with pytest.raises(qb.QloraError) as ei:
                qb.qlora_linear_fwd_tiles(q, qb.nf4_decode_tiles(q), p2["X"].cuda(), p["A"].cuda(), p["B"].cuda(),
                                          p["scale"])
            assert ei.value.status == -7


@pytest.mark.parametrize("fmt_in,fmt_out,r", [((64, 256), (64, 256), 16), ((32, 0), (128, 256), 8),
                                               ((256, 256), (64, 0), 64), ((64, 256), (64, 256), 3)])
def test_merge_lora_bit_exact(qb, oracle, fmt_in, fmt_out, r):
    """Merge-and-requantize on the GPU equals the oracle bit for bit (codes,
    absmax codes, scales), for changes of format and any r."""
    N, K = 37, 1024
    W = wl.draw_weight(wl.generator(700 + r), N, K, 0.02, 0.02)
    W[2, :256] = 0.0
    q, _ = quantize_both(qb, oracle, W, *fmt_in)
    g = wl.generator(800 + r)
    A = ((torch.rand(r, K, generator=g) * 2 - 1) / np.sqrt(K)).bfloat16()
    B = (torch.randn(N, r, generator=g) * 0.05).bfloat16()
    m = qb.nf4_merge_lora(q, A.cuda(), B.cuda(), 0.5, *fmt_out)
    oc, oa, od, _ = oracle.nf4_merge_lora(q.codes.cpu().numpy(), q.absmax_q.cpu().numpy(), q.dq_scale.cpu().numpy(),
                                          N, K, bits(A), bits(B), 0.5, *fmt_in, *fmt_out)
    assert np.array_equal(m.codes.cpu().numpy(), oc), "codes differ"
    assert np.array_equal(m.absmax_q.cpu().numpy(), oa), "absmax codes differ"
    assert m.dq_scale.cpu().numpy().tobytes() == od.tobytes(), "scales differ"


@pytest.mark.parametrize("N,K,fmt_in,r", [(45, 3072, (128, 0), 64), (16, 2048, (64, 256), 1), (3, 1024, (32, 256), 16),
                                           (40, 1024, (256, 256), 8), (50, 1024, (128, 256), 5)])
def test_merge_lora_tiled_shapes(qb, oracle, N, K, fmt_in, r):
    """Merges into the default format with K a multiple of 1024 (the tiled
    path: 16 rows per CTA, groups of 256 blocks that start inside a row when
    K / 64 is not a multiple of 256, a ragged last row range) equal the oracle
    bit for bit; a row whose merged values are all zero codes the zero level."""
    W = wl.draw_weight(wl.generator(710 + N), N, K, 0.02, 0.02)
    W[N - 1, :] = 0.0
    q, _ = quantize_both(qb, oracle, W, *fmt_in)
    g = wl.generator(810 + r)
    A = ((torch.rand(r, K, generator=g) * 2 - 1) / np.sqrt(K)).bfloat16()
    B = (torch.randn(N, r, generator=g) * 0.05).bfloat16()
    B[N - 1, :] = 0.0
    m = qb.nf4_merge_lora(q, A.cuda(), B.cuda(), 1.5, 64, 256)
    oc, oa, od, _ = oracle.nf4_merge_lora(q.codes.cpu().numpy(), q.absmax_q.cpu().numpy(), q.dq_scale.cpu().numpy(),
                                          N, K, bits(A), bits(B), 1.5, *fmt_in, 64, 256)
    assert np.array_equal(m.codes.cpu().numpy(), oc), "codes differ"
    assert np.array_equal(m.absmax_q.cpu().numpy(), oa), "absmax codes differ"
    assert m.dq_scale.cpu().numpy().tobytes() == od.tobytes(), "scales differ"


def test_merge_lora_reports_overflow(qb):
    """A merge whose values overflow fp32 (a huge scale) is reported as
    non-finite, as a quantize of such weights is."""
    N, K, r = 20, 1024, 4
    q = qb.nf4_quantize(wl.draw_weight(wl.generator(720), N, K, 0.02, 0.0).cuda())
    A = torch.ones(r, K, dtype=torch.bfloat16, device="cuda")
    B = torch.ones(N, r, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qb.QloraError) as ei:
        qb.nf4_merge_lora(q, A, B, 3.0e38)
    assert ei.value.status == -3


def test_merge_lora_at_decode_scale(qb, oracle):
    """The 70B-shaped up projection merged with its r = 16 adapter: sampled
    rows against the oracle (the merge of a row depends only on that row)."""
    w = wl.WORKLOADS["decode_70b_up"]
    p = wl.draw_linear(w, M=1)
    q = qb.nf4_quantize(p["W"].cuda())
    m = qb.nf4_merge_lora(q, p["A"].cuda(), p["B"].cuda(), p["scale"])
    N, K = p["N"], p["K"]
    rows = np.array([0, 1, 4097, N - 2, N - 1])
    bpr = K // 64  # blocks per row; 128 per row -> whole double-quant groups are 2 rows
    for n in rows:
        n0 = n - n % 2  # the pair of rows that shares a group of 256 blocks
        sl = slice(n0 * K // 2, (n0 + 2) * K // 2)
        bs = slice(n0 * bpr, (n0 + 2) * bpr)
        oc, oa, od, _ = oracle.nf4_merge_lora(q.codes[sl].cpu().numpy(), q.absmax_q[bs].cpu().numpy(),
                                              q.dq_scale[n0 // 2: n0 // 2 + 1].cpu().numpy(), 2, K,
                                              bits(p["A"]), bits(p["B"][n0:n0 + 2]), p["scale"])
        assert np.array_equal(m.codes[sl].cpu().numpy(), oc)
        assert np.array_equal(m.absmax_q[bs].cpu().numpy(), oa)
        assert m.dq_scale[n0 // 2: n0 // 2 + 1].cpu().numpy().tobytes() == od.tobytes()


@pytest.mark.parametrize("M,r", [(1, 16), (5, 64), (12, 16), (16, 64)])
def test_multi_adapter_decode(qb, oracle, M, r):
    """Decode with a stack of 3 adapters and a per-token index against the
    oracle's multi-adapter forward; a token with an index outside the stack
    gets the base output only."""
    N, K, na = 1000, 2048, 3
    p = wl.draw_small(900 + M + r, M, N, K, r, 2.0 * r, with_dy=False)
    q, Wp = quantize_both(qb, oracle, p["W"])
    g = wl.generator(950 + M)
    A_all = ((torch.rand(na, r, K, generator=g) * 2 - 1) / np.sqrt(K)).bfloat16()
    B_all = (torch.randn(na, N, r, generator=g) * 0.5).bfloat16()
    scales = torch.tensor([2.0, 0.5, 4.0], dtype=torch.float32)
    idx = torch.tensor([(3 * m + 1) % na for m in range(M)], dtype=torch.int32)
    bad = M > 3
    if bad:
        idx[3] = 7  # outside the stack: no LoRA term
    Y = qb.qlora_linear_fwd_multi(q, p["X"].cuda(), A_all.cuda(), B_all.cuda(), scales.cuda(), idx.cuda())
    torch.cuda.synchronize()
    X16 = bits(p["X"])
    ref_idx = idx.numpy().copy()
    if bad:
        ref_idx[3] = 0
    Yref = oracle.linear_fwd_multi(X16, Wp, bits(A_all), bits(B_all), scales.double().numpy(), ref_idx)
    if bad:
        zeroB = np.zeros((N, r), np.uint16)
        Yref[3] = oracle.linear_fwd(X16, Wp, bits(A_all[0]), zeroB, 1.0, rows=np.array([3]))[0]
    e = relfro(Y.float().cpu().numpy(), Yref)
    assert e <= TOL, f"Y rel err {e}"


@pytest.mark.parametrize("M", [200, 5])
def test_lora_dropout(qb, oracle, M):
    """LoRA dropout on the adapter input (p = 0.1, mask drawn on the host):
    forward through the GEMM (M = 200) or the decode kernel (M = 5), and the
    backward, against the oracle."""
    N, K, r = 264, 1024, 16
    p = wl.draw_small(1100 + M, M, N, K, r, 32.0, b_std=0.5)
    q, Wp = quantize_both(qb, oracle, p["W"])
    g = np.random.default_rng(1200 + M)
    mask = (g.random((M, K)) >= 0.1).astype(np.uint8)
    keep = float(np.float32(1.0 / 0.9))
    X, A, B, dY = p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["dY"].cuda()
    mk = torch.from_numpy(mask).cuda()
    Y, H = qb.qlora_linear_fwd_dropout(q, X, A, B, p["scale"], mk, keep)
    X16, A16, B16, dY16 = bits(p["X"]), bits(p["A"]), bits(p["B"]), bits(p["dY"])
    Yref = oracle.linear_fwd_dropout(X16, mask, keep, Wp, A16, B16, p["scale"])
    assert relfro(Y.float().cpu().numpy(), Yref) <= TOL
    Href = oracle._bf16_to_f64(oracle.dropout_input(X16, mask, keep)) @ oracle._bf16_to_f64(A16).T
    assert relfro(H.float().cpu().numpy(), Href) <= TOL
    dX, dA, dB = qb.qlora_linear_bwd_dropout(q, X, dY, A, B, p["scale"], mk, keep, H=H)
    rX, rA, rB = oracle.linear_bwd_dropout(X16, mask, keep, dY16, Wp, A16, B16, p["scale"])
    errs = (relfro(dX.float().cpu().numpy(), rX), relfro(dA.float().cpu().numpy(), rA),
            relfro(dB.float().cpu().numpy(), rB))
    assert max(errs) <= TOL, f"dX/dA/dB rel err {errs}"
    _, dA2, _ = qb.qlora_linear_bwd_dropout(q, X, dY, A, B, p["scale"], mk, keep, want_dx=False)  # H recomputed
    assert relfro(dA2.float().cpu().numpy(), rA) <= TOL


@pytest.mark.parametrize("M,K", [(2048, 4096), (300, 1024)])
def test_lora_dropout_mask_inside_the_adapter_kernels(qb, M, K):
    """For M > 16 the dropout entry points apply the keep mask to the X tiles
    inside the H and dA kernels instead of writing Xd to memory.  Their H and
    dA equal, bit for bit, those of the plain layer run on Xd made by torch
    (bf16(fl32(x * keep)) where kept, else 0), which the oracle tests cover;
    (2048, 4096) takes the 256-column dA kernel, (300, 1024) the 64-column one."""
    N, r = 512, 16
    p = wl.draw_small(1500 + M, M, N, K, r, 32.0, b_std=0.5)
    q = qb.nf4_quantize(p["W"].cuda())
    g = torch.Generator().manual_seed(1600 + M)
    mask = (torch.rand(M, K, generator=g) >= 0.1).to(torch.uint8)
    keep = float(np.float32(1.0 / 0.9))
    X, A, B, dY = p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["dY"].cuda()
    mk = mask.cuda()
    Xd = torch.where(mk.bool(), (X.float() * keep).bfloat16(), torch.zeros_like(X))
    _, H = qb.qlora_linear_fwd_dropout(q, X, A, B, p["scale"], mk, keep)
    _, Hp = qb.qlora_linear_fwd(q, Xd, A, B, p["scale"])
    _, dA, _ = qb.qlora_linear_bwd_dropout(q, X, dY, A, B, p["scale"], mk, keep, H=H, want_dx=False)
    _, dAp, _ = qb.qlora_linear_bwd(q, Xd, dY, A, B, p["scale"], H=Hp, want_dx=False)
    _, dA2, _ = qb.qlora_linear_bwd_dropout(q, X, dY, A, B, p["scale"], mk, keep, want_dx=False)  # H recomputed
    torch.cuda.synchronize()
    assert torch.equal(H, Hp), "H differs from the materialised-Xd path"
    assert torch.equal(dA, dAp), "dA differs from the materialised-Xd path"
    assert torch.equal(dA2, dAp), "dA (H recomputed) differs from the materialised-Xd path"


def test_noalloc_entry_reads_default_format_only(qb):
    q = qb.nf4_quantize(torch.randn(64, 256, device="cuda") * 0.02, 128, 0)
    X = torch.randn(32, 256, device="cuda").bfloat16()
    A = torch.randn(16, 256, device="cuda").bfloat16()
    B = torch.randn(64, 16, device="cuda").bfloat16()
    with pytest.raises(qb.QloraError) as ei:
        qb.qlora_linear_fwd_noalloc(q, X, A, B, 2.0)
    assert ei.value.status == -7


def test_quantize_rejects_nonfinite(qb):
    for bad in (float("nan"), float("inf"), -float("inf")):
        W = torch.zeros(4, 128, device="cuda")
        W[2, 77] = bad
        with pytest.raises(qb.QloraError) as ei:
            qb.nf4_quantize(W)
        assert ei.value.status == -3


@pytest.mark.parametrize("N,K,seed", [(7, 192, 5), (64, 4096, 6)])
def test_dequantize_bit_exact(qb, oracle, N, K, seed):
    W = wl.draw_weight(wl.generator(seed), N, K, 0.02, 0.01)
    q, _ = quantize_both(qb, oracle, W)
    Wd = qb.nf4_dequantize(q)
    torch.cuda.synchronize()
    o16, _ = oracle.nf4_dequantize(q.codes.cpu().numpy(), q.absmax_q.cpu().numpy(), q.dq_scale.cpu().numpy(), N, K)
    assert np.array_equal(bits(Wd), o16)


# ----------------------------------------------------------- layer, small


SMALL = [
    # M, N, K, r        (GEMM path: M > 16)
    (17, 64, 64, 8),
    (128, 256, 128, 16),
    (200, 264, 320, 16),
    (300, 520, 1024, 64),
    (700, 264, 4160, 64),    # r = 64 on the tensor-core adapter kernels: uneven stage split, ragged last tile
    (257, 1000, 192, 24),
]


@pytest.mark.parametrize("M,N,K,r", SMALL)
def test_forward_small(qb, oracle, M, N, K, r):
    p = wl.draw_small(1000 + M + N + K, M, N, K, r, 2.0 * r, with_dy=False)
    run_fwd_check(qb, oracle, p)


DECODE = [
    (1, 64, 64, 8),
    (4, 264, 320, 16),
    (16, 1000, 1024, 64),
    (9, 72, 4096, 8),
    (8, 136, 2112, 24),    # 33 blocks per row: the last stage holds one block
    (13, 520, 11008, 40),  # 172 blocks per row, r not a multiple of 16
    (2, 8, 64, 8),         # a single half tile
]


@pytest.mark.parametrize("M,N,K,r", DECODE)
def test_forward_decode_small(qb, oracle, M, N, K, r):
    p = wl.draw_small(2000 + M + N, M, N, K, r, 2.0 * r, with_dy=False)
    run_fwd_check(qb, oracle, p)


# ------------------------------------------------------------ decode tiles


def tiles_from_codes(codes, N, K):
    """The decode-tile arrangement of row-major codes as the header states it,
    restated by index arithmetic: unit (tau, kb) at (tau * K/64 + kb) * 512,
    lane i = 4g + t at 16 i holding row 16 tau + g bytes 32 kb + 8t .. +7, then
    row 16 tau + g + 8; rows past N are zeros."""
    c = np.asarray(codes, np.uint8).reshape(N, K // 2)
    T = -(-N // 16)
    pad = np.zeros((T * 16, K // 2), np.uint8)
    pad[:N] = c
    v = pad.reshape(T, 2, 8, K // 64, 4, 8)  # [tau][row half h][g][kb][t][byte]
    return np.ascontiguousarray(v.transpose(0, 3, 2, 4, 1, 5)).reshape(-1)


@pytest.mark.parametrize("N,K", [(8, 1024), (40, 1024), (1000, 2048), (64, 3072)])
def test_decode_tiles_layout(qb, N, K):
    W = torch.randn(N, K, generator=wl.generator(N + K)) * 0.05
    q = qb.nf4_quantize(W.cuda())
    T = qb.nf4_decode_tiles(q)
    torch.cuda.synchronize()
    assert T.numel() == qb.nf4_decode_tiles_bytes(N, K) == -(-N // 16) * (K // 64) * 512
    assert np.array_equal(T.cpu().numpy(), tiles_from_codes(q.codes.cpu().numpy(), N, K))


def run_fwd_tiles_check(qb, oracle, p, rows=None):
    q, Wp = quantize_both(qb, oracle, p["W"])
    T = qb.nf4_decode_tiles(q)
    X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
    Y, H = qb.qlora_linear_fwd_tiles(q, T, X, A, B, p["scale"])
    Yrow, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"])  # row-major decode kernel
    torch.cuda.synchronize()
    Yref = oracle.linear_fwd(bits(p["X"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"], rows=rows)
    Yg, Yr = Y.float().cpu().numpy(), Yrow.float().cpu().numpy()
    if rows is not None:
        Yg, Yr = Yg[rows], Yr[rows]
    e = relfro(Yg, Yref)
    assert e <= TOL, f"Y rel err {e}"
    assert relfro(Yg, Yr) <= 5e-3, "tiles and row-major decode disagree"
    Href = oracle.lora_h(bits(p["X"]), bits(p["A"]))
    assert relfro(H.float().cpu().numpy(), Href) <= TOL
    return e


DECODE_TILES = [
    (1, 40, 1024, 8),      # one item per tile, a ragged last tile
    (4, 264, 2048, 16),
    (8, 1000, 4096, 64),   # ragged last tile (1000 = 62 * 16 + 8)
    (9, 72, 1024, 8),      # two token tiles
    (16, 520, 3072, 40),   # three items per tile, r not a multiple of 16
    (3, 8, 1024, 24),      # a single half tile
    (2, 4096, 5120, 16),   # more tiles than SMs
    (12, 64, 28672, 16),   # 56 chunks per row: long chunk sequences per half
    (5, 40008, 1024, 16),  # more than 14 tiles per CTA: two rounds of tile pairs, odd counts, ragged last tile
]


@pytest.mark.parametrize("M,N,K,r", DECODE_TILES)
def test_forward_decode_tiles(qb, oracle, M, N, K, r):
    p = wl.draw_small(2500 + M + N, M, N, K, r, 2.0 * r, with_dy=False)
    run_fwd_tiles_check(qb, oracle, p)


def test_decode_tiles_repeatable(qb):
    """Items of a tile are added in item order: two calls give the same bits."""
    p = wl.draw_small(2600, 7, 2056, 4096, 16, 32.0, with_dy=False)
    q = qb.nf4_quantize(p["W"].cuda())
    T = qb.nf4_decode_tiles(q)
    X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
    Y1, _ = qb.qlora_linear_fwd_tiles(q, T, X, A, B, p["scale"])
    Y2, _ = qb.qlora_linear_fwd_tiles(q, T, X, A, B, p["scale"])
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("M,r", [(1, 16), (12, 64)])
def test_multi_adapter_decode_tiles(qb, oracle, M, r):
    N, K, na = 1000, 2048, 3
    p = wl.draw_small(960 + M + r, M, N, K, r, 2.0 * r, with_dy=False)
    q, Wp = quantize_both(qb, oracle, p["W"])
    T = qb.nf4_decode_tiles(q)
    g = wl.generator(970 + M)
    A_all = ((torch.rand(na, r, K, generator=g) * 2 - 1) / np.sqrt(K)).bfloat16()
    B_all = (torch.randn(na, N, r, generator=g) * 0.5).bfloat16()
    scales = torch.tensor([2.0, 0.5, 4.0], dtype=torch.float32)
    idx = torch.tensor([(2 * m + 1) % na for m in range(M)], dtype=torch.int32)
    Y = qb.qlora_linear_fwd_multi_tiles(q, T, p["X"].cuda(), A_all.cuda(), B_all.cuda(), scales.cuda(), idx.cuda())
    torch.cuda.synchronize()
    Yref = oracle.linear_fwd_multi(bits(p["X"]), Wp, bits(A_all), bits(B_all), scales.double().numpy(),
                                   idx.numpy().copy())
    e = relfro(Y.float().cpu().numpy(), Yref)
    assert e <= TOL, f"Y rel err {e}"


def test_decode_tiles_rejects_shapes(qb):
    q = qb.nf4_quantize(torch.randn(64, 1088, device="cuda") * 0.02)
    with pytest.raises(qb.QloraError):
        qb.nf4_decode_tiles(q)  # K % 1024 != 0
    q = qb.nf4_quantize(torch.randn(64, 1024, device="cuda") * 0.02)
    T = qb.nf4_decode_tiles(q)
    X = torch.randn(17, 1024, device="cuda").bfloat16()
    A = torch.randn(16, 1024, device="cuda").bfloat16()
    B = torch.randn(64, 16, device="cuda").bfloat16()
    with pytest.raises(qb.QloraError):
        qb.qlora_linear_fwd_tiles(q, T, X, A, B, 2.0)  # M > 16
    assert qb.device_status() == 0


def test_decode_repeatable(qb):
    """The decode kernel sums its K-split partials in a fixed order: two calls
    give the same bits."""
    p = wl.draw_small(2100, 5, 2056, 4160, 16, 32.0, with_dy=False)
    q = qb.nf4_quantize(p["W"].cuda())
    X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
    Y1, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    Y2, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("M,N,K,r", SMALL)
def test_backward_small(qb, oracle, M, N, K, r):
    p = wl.draw_small(3000 + M + N + K, M, N, K, r, 2.0 * r)
    run_bwd_check(qb, oracle, p)
    run_bwd_check(qb, oracle, p, use_saved_h=False)


@pytest.mark.parametrize("M,N,K,r", [(5, 264, 1024, 64), (16, 1000, 2048, 64), (3, 72, 320, 16)])
def test_backward_few_tokens(qb, oracle, M, N, K, r):
    """The backward at decode-sized token counts (one partly filled token tile
    in every adapter kernel, the GEMM's single token pair)."""
    p = wl.draw_small(3500 + M + N + K, M, N, K, r, 2.0 * r)
    run_bwd_check(qb, oracle, p)
    run_bwd_check(qb, oracle, p, use_saved_h=False)


def test_adapter_isolating_cases(qb, oracle):
    """W = 0 makes Y and dX pure LoRA; a large B makes the adapter dominate."""
    M, N, K, r = 150, 320, 256, 16
    p = wl.draw_small(77, M, N, K, r, 32.0)
    p["W"] = torch.zeros(N, K)
    run_fwd_check(qb, oracle, p)
    run_bwd_check(qb, oracle, p)
    p = wl.draw_small(78, M, N, K, r, 32.0, b_std=1.0)
    run_fwd_check(qb, oracle, p)
    run_bwd_check(qb, oracle, p)
    p = wl.draw_small(79, 12, N, K, r, 32.0, b_std=1.0, with_dy=False)  # decode path
    p["W"] = torch.zeros(N, K)
    run_fwd_check(qb, oracle, p)


def test_zero_B_gives_base_and_zero_dA(qb, oracle):
    M, N, K, r = 130, 256, 256, 16
    p = wl.draw_small(81, M, N, K, r, 32.0)
    p["B"] = torch.zeros(N, r, dtype=torch.bfloat16)
    q, Wp = quantize_both(qb, oracle, p["W"])
    X, A, B, dY = p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["dY"].cuda()
    Y1, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    Y2, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    assert torch.equal(Y1, Y2)
    Yb = oracle.linear_fwd(bits(p["X"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"])
    assert relfro(Y1.float().cpu().numpy(), Yb) <= TOL
    _, dA, dB = qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"])
    assert torch.count_nonzero(dA).item() == 0
    assert torch.count_nonzero(dB).item() > 0


def test_no_tokens(qb):
    N, K, r = 128, 128, 16
    q = qb.nf4_quantize(torch.randn(N, K, device="cuda") * 0.02)
    X = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    A = torch.randn(r, K, device="cuda").bfloat16()
    B = torch.randn(N, r, device="cuda").bfloat16()
    Y, _ = qb.qlora_linear_fwd(q, X, A, B, 2.0)
    assert Y.shape == (0, N)
    dX, dA, dB = qb.qlora_linear_bwd(q, X, torch.empty(0, N, dtype=torch.bfloat16, device="cuda"), A, B, 2.0)
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


def test_decode_and_gemm_paths_agree(qb):
    """M <= 16 runs the decode kernel, M > 16 the tensor-core GEMM; the same
    rows must agree within tolerance."""
    N, K, r = 1024, 2048, 16
    p = wl.draw_small(91, 17, N, K, r, 32.0, with_dy=False)
    q = qb.nf4_quantize(p["W"].cuda())
    X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
    Yg, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"])          # GEMM
    Yd, _ = qb.qlora_linear_fwd(q, X[:16].contiguous(), A, B, p["scale"])  # decode
    assert relfro(Yd.float().cpu().numpy(), Yg[:16].float().cpu().numpy()) <= 5e-3


def test_backward_repeatable_large(qb):
    """dA and dB come out bit for bit the same on every call, with the dX GEMM
    (dA, dB on the side stream) and without it, at a shape with thousands of
    column-kernel CTAs: the TMA rings release a stage only after the
    consumers' reads of it are ordered before the refill."""
    M, N, K, r = 4096, 8192, 28672, 64
    g = wl.generator(97)
    X = torch.randn(M, K, generator=g).bfloat16().cuda()
    dY = torch.randn(M, N, generator=g).bfloat16().cuda()
    A = ((torch.rand(r, K, generator=g) * 2 - 1) / np.sqrt(K)).bfloat16().cuda()
    B = (torch.randn(N, r, generator=g) * 0.01).bfloat16().cuda()
    q = qb.nf4_quantize(torch.randn(N, K, generator=g).cuda() * 0.02)
    H = (X.float() @ A.float().t()).bfloat16()
    ref = None
    for want_dx in (True, False, True, False, True):
        _, dA, dB = qb.qlora_linear_bwd(q, X, dY, A, B, 0.25, H=H, want_dx=want_dx)
        torch.cuda.synchronize()
        if ref is None:
            ref = (dA.clone(), dB.clone())
        assert torch.equal(dA, ref[0]) and torch.equal(dB, ref[1])
    dH = (0.25 * (dY.float() @ B.float())).bfloat16().float()
    dA_t = dH.t() @ X.float()
    assert relfro(ref[0].float().cpu().numpy(), dA_t.cpu().numpy()) <= 5e-3
    assert qb.device_status() == 0


def test_fwd_bwd_in_cuda_graph(qb):
    """The backward forks dA and dB onto a side stream and joins it: the same
    calls captured in a CUDA graph and replayed give the eager results."""
    M, N, K, r = 1040, 1024, 2048, 16
    p = wl.draw_small(95, M, N, K, r, 32.0)
    q = qb.nf4_quantize(p["W"].cuda())
    X, A, B, dY = p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["dY"].cuda()
    Y0, H0 = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
    dX0, dA0, dB0 = qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"], H=H0)
    torch.cuda.synchronize()
    Y = torch.empty_like(Y0)
    H = torch.empty_like(H0)
    dX, dA, dB = torch.empty_like(dX0), torch.empty_like(dA0), torch.empty_like(dB0)
    wsf = torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    wsb = torch.empty(qb.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    L = qb.lib()
    import ctypes

    def step():
        st = qb._stream()
        assert L.qlora_linear_fwd(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), N, K, qb._ptr(X), M,
                                  qb._ptr(A), qb._ptr(B), r, ctypes.c_float(p["scale"]), qb._ptr(Y), qb._ptr(H),
                                  qb._ptr(wsf), wsf.numel(), st) == 0
        assert L.qlora_linear_bwd(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), N, K, qb._ptr(X),
                                  qb._ptr(dY), M, qb._ptr(A), qb._ptr(B), r, ctypes.c_float(p["scale"]), qb._ptr(H),
                                  qb._ptr(dX), qb._ptr(dA), qb._ptr(dB), qb._ptr(wsb), wsb.numel(), st) == 0

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in (Y, H, dX, dA, dB):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for got, ref in ((Y, Y0), (H, H0), (dX, dX0), (dA, dA0), (dB, dB0)):
        assert torch.equal(got, ref)
    del g
    assert qb.device_status() == 0


def test_backward_on_two_unordered_streams(qb, oracle):
    """Two backward calls on two streams with no ordering between them (each
    caller stream has its own side stream for dA and dB): both match the
    oracle, and a CUDA graph captured on a third stream still works."""
    cases = []
    for seed, (M, N, K, r) in ((501, (300, 520, 1024, 16)), (502, (260, 264, 2048, 64))):
        p = wl.draw_small(seed, M, N, K, r, 2.0 * r, b_std=0.5)
        q, Wp = quantize_both(qb, oracle, p["W"])
        cases.append((p, q, Wp))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    torch.cuda.synchronize()
    for (p, q, _), st in zip(cases, streams):
        with torch.cuda.stream(st):
            X, A, B, dY = (p[k].cuda(non_blocking=True) for k in ("X", "A", "B", "dY"))
            outs.append(qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"], stream=st) + (X, A, B, dY))
    torch.cuda.synchronize()
    for (p, q, Wp), (dX, dA, dB, *_keep) in zip(cases, outs):
        dXr, dAr, dBr, _ = oracle.linear_bwd(bits(p["X"]), bits(p["dY"]), Wp, bits(p["A"]), bits(p["B"]),
                                             p["scale"])
        errs = (relfro(dX.float().cpu().numpy(), dXr), relfro(dA.float().cpu().numpy(), dAr),
                relfro(dB.float().cpu().numpy(), dBr))
        assert max(errs) <= TOL, errs
    assert qb.device_status() == 0


def test_quantize_from_two_threads(qb, oracle):
    """nf4_quantize from two host threads on two streams at once: each call has
    its own non-finite flag, so the call with a NaN reports it and the other
    returns its codes bit-exact."""
    import threading
    good = wl.draw_weight(wl.generator(511), 512, 4096, 0.02)
    bad = wl.draw_weight(wl.generator(512), 512, 4096, 0.02)
    bad[300, 17] = float("nan")
    res = {}

    def run(name, W):
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            Wd = W.cuda(non_blocking=True)
            for _ in range(20):
                try:
                    res[name] = qb.nf4_quantize(Wd, stream=st)
                except qb.QloraError as e:
                    res[name] = e.status

    ts = [threading.Thread(target=run, args=("good", good)), threading.Thread(target=run, args=("bad", bad))]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert res["bad"] == -3
    oc, oa, od, _ = oracle.nf4_quantize(good.numpy())
    q = res["good"]
    assert np.array_equal(q.codes.cpu().numpy(), oc) and np.array_equal(q.absmax_q.cpu().numpy(), oa)
    assert q.dq_scale.cpu().numpy().tobytes() == od.tobytes()


def test_bounded_wait_runs_out_and_the_next_call_is_correct(qb, oracle):
    """The decode kernel's testing aid withholds one code stage per CTA with a
    1 ms wait limit: the consumers' bounded wait runs out, the kernel drains
    what it issued and returns, the device status reports QLORA_ERR_TIMEOUT
    (and is cleared by reading it), and the next normal call on the same
    buffers matches the oracle."""
    import ctypes
    M, N, K, r = 3, 4096, 4096, 16   # every CTA has at least two code stages
    p = wl.draw_small(520, M, N, K, r, 32.0, with_dy=False)
    q, Wp = quantize_both(qb, oracle, p["W"])
    X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
    assert qb.device_status() == 0
    L = qb.lib()
    st = L.qlora_test_decode_timeout(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), N, K, qb._ptr(X), M,
                                     qb._ptr(A), qb._ptr(B), r, ctypes.c_float(p["scale"]), qb._ptr(Y), qb._ptr(ws),
                                     ws.numel(), qb._stream())
    assert st == 0
    torch.cuda.synchronize()
    assert qb.device_status() == -6   # QLORA_ERR_TIMEOUT
    assert qb.device_status() == 0    # read and cleared
    Y2, _ = qb.qlora_linear_fwd(q, X, A, B, p["scale"], out=Y, workspace=ws)
    torch.cuda.synchronize()
    Yref = oracle.linear_fwd(bits(p["X"]), Wp, bits(p["A"]), bits(p["B"]), p["scale"])
    assert relfro(Y2.float().cpu().numpy(), Yref) <= TOL
    assert qb.device_status() == 0


def test_argument_errors_on_device(qb):
    q = qb.nf4_quantize(torch.randn(64, 128, device="cuda") * 0.02)
    X = torch.randn(32, 128, device="cuda").bfloat16()
    A = torch.randn(16, 128, device="cuda").bfloat16()
    B = torch.randn(64, 16, device="cuda").bfloat16()
    L = qb.lib()
    import ctypes
    Y = torch.empty(32, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    st = L.qlora_linear_fwd(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), 64, 128, qb._ptr(X), 32,
                            qb._ptr(A), qb._ptr(B), 16, ctypes.c_float(2.0), qb._ptr(Y), None, qb._ptr(ws), 64,
                            qb._stream())
    assert st == -4  # workspace too small
    assert qb.device_status() == 0


# ---------------------------------------------------- workloads, full size


def _rows(M, per_tile, seed):
    """Rows of every 256-token tile (the GEMM's CTA token tile), plus the first
    and the last (ragged) row."""
    return pt.rows_every_tile(M, seed, tile=256, per_tile=per_tile)


def test_workload_fwd_2048(qb, oracle):
    p = wl.draw_linear(wl.WORKLOADS["fwd_2048"])
    run_fwd_check(qb, oracle, p)


def test_workload_qproj_7b(qb, oracle):
    w = wl.WORKLOADS["qproj_7b"]
    p = wl.draw_linear(w)
    rows = _rows(p["M"], 3, 1)
    _, q, Wp = run_fwd_check(qb, oracle, p, rows=rows)
    run_bwd_check(qb, oracle, p, rows=rows, q=q, Wp=Wp)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_workload_decode_70b_up(qb, oracle, M):
    w = wl.WORKLOADS["decode_70b_up"]
    p = wl.draw_linear(w, M=M)
    run_fwd_check(qb, oracle, p)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_workload_decode_70b_up_tiles(qb, oracle, M):
    """The decode workload through the decode tiles, the launch the benchmark times."""
    w = wl.WORKLOADS["decode_70b_up"]
    p = wl.draw_linear(w, M=M)
    run_fwd_tiles_check(qb, oracle, p)


@pytest.mark.parametrize("proj", [0, 1, 2])
def test_workload_mlp_7b(qb, oracle, proj):
    w = wl.WORKLOADS["mlp_7b"]
    p = wl.draw_linear(w, proj)
    rows = _rows(p["M"], 1, 10 + proj)
    _, q, Wp = run_fwd_check(qb, oracle, p, rows=rows)
    run_bwd_check(qb, oracle, p, rows=rows, q=q, Wp=Wp)


@pytest.mark.parametrize("proj", range(7))
def test_workload_layer_70b(qb, oracle, proj):
    w = wl.WORKLOADS["layer_70b"]
    p = wl.draw_linear(w, proj)
    rows = _rows(p["M"], 1, 20 + proj)
    _, q, Wp = run_fwd_check(qb, oracle, p, rows=rows)
    run_bwd_check(qb, oracle, p, rows=rows, q=q, Wp=Wp)


def test_workload_qproj_7b_adapter_only(qb, oracle):
    """The q_proj workload at full size with W = 0: Y and dX are then the LoRA
    terms alone, so an output tile that drops or misplaces its adapter product
    fails the tile check outright ("QLoRA: fine-tuning a large model on one
    GPU", LoRA, stated once: h = W0 x + (alpha/r) B A x)."""
    w = wl.WORKLOADS["qproj_7b"]
    p = wl.draw_linear(w)
    p["W"] = torch.zeros_like(p["W"])
    rows = _rows(p["M"], 1, 31)
    _, q, Wp = run_fwd_check(qb, oracle, p, rows=rows)
    assert not np.any(Wp)
    run_bwd_check(qb, oracle, p, rows=rows, q=q, Wp=Wp)


def test_device_status_clean(qb):
    assert qb.device_status() == 0
