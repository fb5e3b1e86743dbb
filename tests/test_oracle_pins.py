"""Pins for the CPU oracle (runs without a GPU).

Every check compares the oracle with something other than itself: numbers the
QLoRA pages print (tests/golden/page_numbers.txt), closed forms of the codebook
construction evaluated with Python's own normal distribution, textbook bf16
rounding, brute-force nearest-level search, numpy matrix products, and the
exact linearity identities that tie a backward pass to its forward pass.
"""
import math
import os
import statistics

import numpy as np
import pytest
import torch

from bit_nf4_quantized_24_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_numbers.txt")


def golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, value, _unit, _cite = [p.strip() for p in line.split("|", 3)]
        out[name] = float(value)
    return out


def unpack(codes):
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=1).reshape(-1)


# ----------------------------------------------------------------- codebook


def test_codebook_structure(oracle):
    g = golden()
    l64, l32, m32 = oracle.nf4_codebook()
    assert len(l32) == g["nf4_levels"] == 16
    assert np.all(np.diff(l32) > 0), "levels strictly ascending"
    assert l32[0] == -1.0 and l32[7] == 0.0 and l32[15] == 1.0
    assert np.array_equal(l32, l64.astype(np.float32))
    for i in range(15):
        assert l32[i] < m32[i] < l32[i + 1]
        assert m32[i] == np.float32(np.float32(l32[i] + l32[i + 1]) * np.float32(0.5))


def test_codebook_is_equal_mass_normal_quantiles(oracle):
    """The levels sit at equally spaced probabilities of N(0,1) on each side of
    the exact zero (8 positive, 7 negative), scaled so the outermost level is 1.
    Evaluated with Python's statistics.NormalDist, not the oracle's inverse."""
    nd = statistics.NormalDist()
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    assert oracle.nf4_delta() == delta
    z = nd.inv_cdf(delta)
    l64, l32, _ = oracle.nf4_codebook()
    for i in range(8, 16):
        assert abs(nd.cdf(l64[i] * z) - (0.5 + (i - 7) * (delta - 0.5) / 8)) < 1e-12
    for i in range(0, 7):
        assert abs(nd.cdf(l64[i] * z) - (0.5 - (7 - i) * (delta - 0.5) / 7)) < 1e-12
    # a bell-curve shape: gaps widen away from zero on both sides
    gaps = np.diff(l64)
    assert np.all(np.diff(gaps[7:]) > 0) and np.all(np.diff(gaps[:7]) < 0)


# ----------------------------------------------------------------- quantize


@pytest.mark.parametrize("e", [-9, -3, 0, 4])
def test_codebook_values_round_trip(oracle, e):
    """A block made of the levels times a power-of-two absmax encodes to the
    level indices; the even element sits in the low nibble."""
    _, l32, _ = oracle.nf4_codebook()
    a = np.float32(2.0 ** e)
    idx = np.array(list(range(16)) + list(range(15, -1, -1)) + [0, 15] * 8 + list(range(16)), np.int64)
    assert idx.size == 64
    W = (l32[idx] * a).astype(np.float32).reshape(1, 64)
    codes, aq, dq, absmax = oracle.nf4_quantize(W)
    assert absmax[0] == a
    assert np.array_equal(unpack(codes), idx)
    assert codes[0] == (idx[0] | (idx[1] << 4))


def test_tie_rule_and_next_float(oracle):
    _, l32, m32 = oracle.nf4_codebook()
    rows = []
    expect = []
    for i in range(15):
        blk = np.zeros(64, np.float32)
        blk[0] = 1.0  # absmax 1: t == x exactly
        blk[1] = m32[i]
        blk[2] = np.nextafter(m32[i], np.float32(np.inf))
        blk[3] = np.nextafter(m32[i], np.float32(-np.inf))
        rows.append(blk)
        e = np.full(64, 7)
        e[0], e[1], e[2], e[3] = 15, i, i + 1, i
        expect.append(e)
    codes, _, _, _ = oracle.nf4_quantize(np.stack(rows))
    assert np.array_equal(unpack(codes), np.concatenate(expect))


def test_zero_block_and_zero_group(oracle):
    W = np.zeros((2, 128), np.float32)
    W[1, 64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    codes, aq, dq, absmax = oracle.nf4_quantize(W)
    c = unpack(codes)
    assert np.all(c[:192] == 7)
    assert absmax[0] == 0 and aq[0] == 0 and aq[3] == 255
    W0 = np.zeros((4, 64), np.float32)
    codes, aq, dq, _ = oracle.nf4_quantize(W0)
    assert np.all(codes == 0x77) and np.all(aq == 0) and np.all(dq == 0)


@pytest.mark.parametrize("shape,seed", [((4, 128), 0), ((64, 64), 1), ((3, 192), 2)])
def test_brute_force_nearest_level(oracle, shape, seed):
    """Nearest level by exhaustive fp64 search on t = fl32(x / a) agrees with the
    oracle's midpoint count everywhere except within one ulp of a midpoint."""
    g = wl.generator(100 + seed)
    W = wl.draw_weight(g, shape[0], shape[1], 0.02, 0.05).numpy()
    _, l32, m32 = oracle.nf4_codebook()
    codes, _, _, absmax = oracle.nf4_quantize(W)
    c = unpack(codes)
    blocks = W.reshape(-1, 64)
    a = np.abs(blocks).max(axis=1)
    assert np.array_equal(a, absmax)
    t = (blocks / a[:, None].astype(np.float32)).astype(np.float32).reshape(-1)
    brute = np.argmin(np.abs(t.astype(np.float64)[:, None] - l32.astype(np.float64)[None, :]), axis=1)
    diff = brute != c
    near = np.min(np.abs(t[:, None] - m32[None, :]), axis=1) <= np.spacing(np.abs(t))
    assert not np.any(diff & ~near)
    assert diff.sum() == 0


def test_nonfinite_and_bad_shape_rejected(oracle):
    W = np.zeros((2, 64), np.float32)
    W[1, 5] = np.nan
    with pytest.raises(oracle.OracleError, match="NONFINITE"):
        oracle.nf4_quantize(W)
    W[1, 5] = np.inf
    with pytest.raises(oracle.OracleError, match="NONFINITE"):
        oracle.nf4_quantize(W)
    with pytest.raises(oracle.OracleError, match="SHAPE"):
        oracle.nf4_quantize(np.zeros((2, 96), np.float32))


# ------------------------------------------------------------ double quant


def test_double_quant_code_bounds(oracle):
    g = wl.generator(7)
    W = wl.draw_weight(g, 8, 4096 + 64 * 3, 0.02, 0.01).numpy()  # 524 blocks: 2 full groups + a short one
    codes, aq, dq, a = oracle.nf4_quantize(W)
    nb = a.size
    assert dq.size == math.ceil(nb / 256)
    for gi in range(dq.size):
        grp = slice(gi * 256, min(nb, (gi + 1) * 256))
        c2 = a[grp].max()
        assert dq[gi] == np.float32(c2 / np.float32(255))
        assert aq[grp][np.argmax(a[grp])] == 255
        ap = (aq[grp].astype(np.float32) * dq[gi]).astype(np.float32)
        assert np.all(np.abs(ap.astype(np.float64) - a[grp]) <= 0.5 * dq[gi] * (1 + 2 ** -20) + np.spacing(a[grp]))


def test_format_bits_and_footprints_match_pages(oracle):
    g = golden()
    N = K = 8192
    cb, ab, dc = oracle.nf4_sizes(N, K)
    numel = N * K
    bits = 8.0 * (cb + ab + 4 * dc) / numel
    assert bits == 4 + 8 / 64 + 32 / (64 * 256)
    fp32_scale_bits = 32 / g["nf4_block"]
    assert fp32_scale_bits == g["scale_overhead_fp32_block64_bits"]
    saving = fp32_scale_bits - (bits - 4)
    assert round(saving, 2) == g["double_quant_saving_bits"]
    assert round(saving, 1) == g["double_quant_saving_bits_rough"]
    assert cb / numel == g["bytes_per_weight_4bit"]
    assert 65e9 * cb / numel / 1e9 == g["weights_65b_4bit_gb"]
    gb70 = 70e9 * bits / 8 / 1e9
    assert g["weights_70b_4bit_gb_low"] <= gb70 <= g["weights_70b_4bit_gb_high"]


# ------------------------------------------------------------ dequantize


def test_bf16_rounding_textbook(oracle):
    f = oracle.f32_to_bf16_bits
    assert f(1.0) == 0x3F80
    assert f(1.0 + 2 ** -8) == 0x3F80          # tie -> even
    assert f(1.0 + 3 * 2 ** -8) == 0x3F82      # tie -> even (up)
    assert f(1.0 + 2 ** -8 + 2 ** -20) == 0x3F81
    assert f(-(1.0 + 2 ** -8)) == 0xBF80
    assert f(float("inf")) == 0x7F80
    assert f(3.4028234663852886e38) == 0x7F80  # rounds past the largest bf16
    assert f(float("nan")) & 0x7FC0 == 0x7FC0
    x = torch.randn(4096, generator=wl.generator(3)) * 10.0 ** torch.randint(-20, 20, (4096,), generator=wl.generator(4))
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([f(float(v)) for v in x.numpy()], np.uint16)
    assert np.array_equal(ref, got)


def test_dequant_round_trip_error_bound(oracle):
    g = wl.generator(9)
    N, K = 16, 512
    W = wl.draw_weight(g, N, K, 0.02, 0.01).numpy()
    _, l32, _ = oracle.nf4_codebook()
    codes, aq, dq, a = oracle.nf4_quantize(W)
    w16, w32 = oracle.nf4_dequantize(codes, aq, dq, N, K)
    assert np.array_equal(w16.view(np.uint16), torch.from_numpy(w32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    half_gap = np.max(np.diff(l32.astype(np.float64))) / 2
    ap = (aq.astype(np.float64) * np.repeat(dq, 256)[: aq.size])
    blk_a = np.repeat(a.astype(np.float64), 64).reshape(N, K)
    blk_ap = np.repeat(ap, 64).reshape(N, K)
    bound = blk_a * half_gap + np.abs(blk_ap - blk_a) + np.abs(W) * 2 ** -8 + 1e-30
    assert np.all(np.abs(w32.astype(np.float64) - W) <= bound)


# ------------------------------------------------------------------ layer


def _small(seed=11, M=8, N=24, K=128, r=4, alpha=8.0):
    p = wl.draw_small(seed, M, N, K, r, alpha)
    p["B"] = (torch.randn(N, r, generator=wl.generator(seed + 1)) * 0.5).to(torch.bfloat16)
    return p


def _bits(t):
    return wl.bf16_bits(t)


def test_adapter_parameter_counts_match_pages(oracle):
    g = golden()
    d = k = 4096
    r = 16
    A = np.zeros((r, k), np.uint16)
    B = np.zeros((d, r), np.uint16)
    X = np.zeros((1, k), np.uint16)
    Wp = np.zeros((d, k), np.float32)
    oracle.linear_fwd(X, Wp, A, B, 2.0)  # the oracle accepts exactly these adapter shapes
    count = A.size + B.size
    assert count == g["lora_params_4096_r16"]
    assert round(100 * count / (d * k), 2) == g["lora_fraction_4096_r16_pct"]
    assert d * k / count == g["lora_reduction_factor_4096_r16"]


def test_adapter_counts_of_the_practice_question_and_bert_tiny(oracle):
    """quantmemo, Practice 1: a 2048 x 2048 weight at r = 8.  katajob, "What an
    adapter actually adds": BERT-tiny (hidden 128, 2 layers) with r = 8 on the
    query and value projections and its 2-class head trainable prints 8,450.
    The adapter shapes are the ones the oracle's layer accepts."""
    g = golden()

    def adapter(d, k, r):
        A = np.zeros((r, k), np.uint16)
        B = np.zeros((d, r), np.uint16)
        oracle.linear_fwd(np.zeros((1, k), np.uint16), np.zeros((d, k), np.float32), A, B, 2.0)
        return A.size + B.size

    c = adapter(2048, 2048, 8)
    assert c == g["lora_params_2048_r8"]
    assert round(100 * c / (2048 * 2048), 2) == g["lora_fraction_2048_r8_pct"]
    per_projection = adapter(128, 128, 8)
    head = 2 * 128 + 2  # classifier weight [2, 128] and bias [2]
    assert 2 * 2 * per_projection + head == g["bert_tiny_trainable_params"]


def test_forward_equals_merged_weight_product(oracle):
    """Y = X (W' + s B A)^T: the merge identity, with numpy's matmul."""
    p = _small()
    codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(codes, aq, dq, p["N"], p["K"])
    X = p["X"].double().numpy()
    A = p["A"].double().numpy()
    B = p["B"].double().numpy()
    s = p["scale"]
    ref = X @ (Wp.astype(np.float64) + s * B @ A).T
    Y = oracle.linear_fwd(_bits(p["X"]), Wp, _bits(p["A"]), _bits(p["B"]), s)
    assert np.max(np.abs(Y - ref)) <= 1e-12 * np.max(np.abs(ref))
    rows = np.array([5, 0, 7])
    Yr = oracle.linear_fwd(_bits(p["X"]), Wp, _bits(p["A"]), _bits(p["B"]), s, rows=rows)
    assert np.array_equal(Yr, Y[rows])
    H = oracle.lora_h(_bits(p["X"]), _bits(p["A"]))
    assert np.max(np.abs(H - X @ A.T)) <= 1e-13


def _loss_of_forward(oracle, X16, Wp, A16, B16, s, dY):
    return float(np.sum(dY * oracle.linear_fwd(X16, Wp, A16, B16, s)))


def test_backward_is_adjoint_of_forward(oracle):
    """<dY, Y(V)> = <dX, V> (Y is linear in X), and likewise for A and B with
    the base term removed: the backward is the exact adjoint of the forward."""
    p = _small(seed=21, M=6, N=40, K=192, r=8)
    codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(codes, aq, dq, p["N"], p["K"])
    s = p["scale"]
    dY = p["dY"].double().numpy()
    dX, dA, dB, dH = oracle.linear_bwd(_bits(p["X"]), _bits(p["dY"]), Wp, _bits(p["A"]), _bits(p["B"]), s)
    g = wl.generator(99)
    Vx = torch.randn(p["M"], p["K"], generator=g).to(torch.bfloat16)
    Va = torch.randn(p["r"], p["K"], generator=g).to(torch.bfloat16)
    Vb = torch.randn(p["N"], p["r"], generator=g).to(torch.bfloat16)
    zero = np.zeros_like(Wp)
    lx = _loss_of_forward(oracle, _bits(Vx), Wp, _bits(p["A"]), _bits(p["B"]), s, dY)
    assert abs(lx - np.sum(dX * Vx.double().numpy())) <= 1e-10 * (abs(lx) + 1)
    la = _loss_of_forward(oracle, _bits(p["X"]), zero, _bits(Va), _bits(p["B"]), s, dY)
    assert abs(la - np.sum(dA * Va.double().numpy())) <= 1e-10 * (abs(la) + 1)
    lb = _loss_of_forward(oracle, _bits(p["X"]), zero, _bits(p["A"]), _bits(Vb), s, dY)
    assert abs(lb - np.sum(dB * Vb.double().numpy())) <= 1e-10 * (abs(lb) + 1)
    # dH is the gradient at the adapter's hidden activations H = X A^T
    assert np.allclose(dH, s * dY @ p["B"].double().numpy(), rtol=0, atol=1e-12)
    rows = np.array([3, 1])
    dXr, _, _, _ = oracle.linear_bwd(_bits(p["X"]), _bits(p["dY"]), Wp, _bits(p["A"]), _bits(p["B"]), s, rows=rows)
    assert np.array_equal(dXr, dX[rows])


def test_zero_adapter_B_gives_base_output_and_zero_dA(oracle):
    """With B = 0 the update BA is zero (the adapter's initial state): Y is the
    base product and dA vanishes exactly."""
    p = _small(seed=31)
    codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(codes, aq, dq, p["N"], p["K"])
    B0 = np.zeros((p["N"], p["r"]), np.uint16)
    Y = oracle.linear_fwd(_bits(p["X"]), Wp, _bits(p["A"]), B0, p["scale"])
    assert np.array_equal(Y, p["X"].double().numpy() @ Wp.astype(np.float64).T) or \
        np.max(np.abs(Y - p["X"].double().numpy() @ Wp.astype(np.float64).T)) < 1e-12
    _, dA, dB, _ = oracle.linear_bwd(_bits(p["X"]), _bits(p["dY"]), Wp, _bits(p["A"]), B0, p["scale"])
    assert np.all(dA == 0.0)
    assert np.any(dB != 0.0)


# --------------------------------------- other block sizes, double quant off


@pytest.mark.parametrize("block", [32, 64, 128, 256])
@pytest.mark.parametrize("dq_block", [256, 0])
def test_levels_round_trip_any_block(oracle, block, dq_block):
    """Blocks made of the levels times a power-of-two absmax encode to the level
    indices whatever the block size; with double quantization off the stored
    scale is that absmax exactly and each weight dequantizes to its own bf16
    rounding."""
    _, l32, _ = oracle.nf4_codebook()
    rows = 3
    idx = (np.arange(rows * block) * 7 + 3) % 16
    idx[::block] = 15  # each block holds level 1 (its absmax) once
    e = np.repeat(np.array([-6, 0, 5])[: rows], block)
    W = (l32[idx] * (2.0 ** e)).astype(np.float32).reshape(rows, block)
    codes, aq, dq, absmax = oracle.nf4_quantize(W, block=block, dq_block=dq_block)
    assert np.array_equal(unpack(codes), idx)
    assert np.array_equal(absmax, (2.0 ** np.array([-6, 0, 5])).astype(np.float32))
    if dq_block == 0:
        assert aq.size == 0 and np.array_equal(dq, absmax)
        w16, w32 = oracle.nf4_dequantize(codes, aq, dq, rows, block, block=block, dq_block=0)
        # L * 2^e is exact in fp32, so the dequantized value is bf16(W) itself
        assert np.array_equal(w32, torch.from_numpy(W).to(torch.bfloat16).float().numpy())
    else:
        assert aq.size == rows


@pytest.mark.parametrize("block", [32, 128, 256])
def test_brute_force_nearest_level_any_block(oracle, block):
    """The nearest-level rule holds with the block's own absmax for every block
    size (exhaustive fp64 search on t = fl32(x / a))."""
    W = wl.draw_weight(wl.generator(300 + block), 6, 512, 0.02, 0.05).numpy()
    _, l32, _ = oracle.nf4_codebook()
    codes, _, _, absmax = oracle.nf4_quantize(W, block=block)
    blocks = W.reshape(-1, block)
    a = np.abs(blocks).max(axis=1)
    assert np.array_equal(a, absmax)
    t = (blocks / a[:, None]).astype(np.float32).reshape(-1)
    brute = np.argmin(np.abs(t.astype(np.float64)[:, None] - l32.astype(np.float64)[None, :]), axis=1)
    assert np.array_equal(brute, unpack(codes))


def test_double_quant_off_stores_exact_scales(oracle):
    """Without double quantization the block scale is the exact absmax: the
    element of largest magnitude dequantizes to +-bf16(absmax), and the whole
    block's error is bounded by half the widest level gap times absmax plus
    the bf16 rounding -- with no second-level term."""
    W = wl.draw_weight(wl.generator(77), 8, 256, 0.02, 0.05).numpy()
    _, l32, _ = oracle.nf4_codebook()
    codes, aq, dq, a = oracle.nf4_quantize(W, block=64, dq_block=0)
    assert aq.size == 0 and np.array_equal(dq, a)
    w16, w32 = oracle.nf4_dequantize(codes, aq, dq, 8, 256, block=64, dq_block=0)
    blocks = W.reshape(-1, 64)
    i = np.abs(blocks).argmax(axis=1)
    top = w32.reshape(-1, 64)[np.arange(blocks.shape[0]), i]
    want = torch.from_numpy(np.sign(blocks[np.arange(blocks.shape[0]), i]) * a).to(torch.bfloat16).float().numpy()
    assert np.array_equal(top, want)
    half_gap = np.max(np.diff(l32.astype(np.float64))) / 2
    bound = np.repeat(a.astype(np.float64), 64).reshape(8, 256) * half_gap + np.abs(W) * 2 ** -8 + 1e-30
    assert np.all(np.abs(w32.astype(np.float64) - W) <= bound)


@pytest.mark.parametrize("block,dq_block,bits", [(64, 256, 4 + 8 / 64 + 32 / (64 * 256)), (64, 0, 4.5),
                                                  (32, 0, 5.0), (128, 256, 4 + 8 / 128 + 32 / (128 * 256)),
                                                  (256, 0, 4.125)])
def test_format_bits_per_parameter(oracle, block, dq_block, bits):
    """Storage per weight: 4 code bits + the block's scale (8 bits, or 32 bits
    without double quantization) / block + 32 bits per group of 256 blocks."""
    N, K = 64, 4096
    cb, ab, dc = oracle.nf4_sizes(N, K, block, dq_block)
    assert (8 * (cb + ab) + 32 * dc) / (N * K) == pytest.approx(bits, rel=1e-12)


# ------------------------------------------------- merge and re-quantize (f2)


def _quantized(oracle, seed, N=12, K=512, block=64, dq_block=256):
    W = wl.draw_weight(wl.generator(seed), N, K, 0.02, 0.05).numpy()
    W[1, :block] = 0.0  # an all-zero block
    codes, aq, dq, _ = oracle.nf4_quantize(W, block=block, dq_block=dq_block)
    _, wp = oracle.nf4_dequantize(codes, aq, dq, N, K, block=block, dq_block=dq_block)
    return codes, aq, dq, wp


@pytest.mark.parametrize("block,dq_block", [(64, 256), (32, 0), (256, 256)])
def test_merge_with_zero_adapter_is_idempotent(oracle, block, dq_block):
    """B = 0: the merged weight is the dequantized weight itself, and quantizing
    it again returns the same codes (each block's largest weight sits on level
    +-1, and bf16 rounding moves w'/a far less than the level spacing)."""
    N, K, r = 12, 512, 8
    codes, aq, dq, wp = _quantized(oracle, 31, N, K, block, dq_block)
    A = wl.bf16_bits(torch.randn(r, K).bfloat16())
    B = np.zeros((N, r), np.uint16)
    oc, oa, od, merged = oracle.nf4_merge_lora(codes, aq, dq, N, K, A, B, 2.0, block, dq_block, block, dq_block)
    assert np.array_equal(merged, wp)
    assert np.array_equal(oc, codes)


def test_merge_closed_form_shift(oracle):
    """r = 1, A = 1, B = 0.25, s = 2: every weight moves by exactly 0.5."""
    N, K = 4, 128
    codes, aq, dq, wp = _quantized(oracle, 32, N, K)
    one = np.uint16(0x3F80)      # bf16 1.0
    quarter = np.uint16(0x3E80)  # bf16 0.25
    A = np.full((1, K), one, np.uint16)
    B = np.full((N, 1), quarter, np.uint16)
    _, _, _, merged = oracle.nf4_merge_lora(codes, aq, dq, N, K, A, B, 2.0)
    assert np.array_equal(merged.astype(np.float64) - wp.astype(np.float64), np.full((N, K), 0.5))


@pytest.mark.parametrize("out_block,out_dq", [(64, 256), (128, 0)])
def test_merge_matches_real_sum_within_quantization_error(oracle, out_block, out_dq):
    """The re-quantized merge dequantizes to w' + s B A (fp64) within the NF4
    error of its own blocks: half the widest level gap times the block absmax,
    plus the scale coding and bf16 rounding."""
    N, K, r, s = 16, 512, 16, 0.25
    codes, aq, dq, wp = _quantized(oracle, 33, N, K)
    g = wl.generator(34)
    A = (torch.rand(r, K, generator=g) * 2 - 1) / np.sqrt(K)
    B = torch.randn(N, r, generator=g) * 0.05
    A16, B16 = wl.bf16_bits(A.bfloat16()), wl.bf16_bits(B.bfloat16())
    oc, oa, od, merged = oracle.nf4_merge_lora(codes, aq, dq, N, K, A16, B16, s, 64, 256, out_block, out_dq)
    exact = wp.astype(np.float64) + s * (B.bfloat16().double().numpy() @ A.bfloat16().double().numpy())
    assert np.max(np.abs(merged - exact)) <= 1e-6 * np.max(np.abs(exact))
    _, back = oracle.nf4_dequantize(oc, oa, od, N, K, block=out_block, dq_block=out_dq)
    _, l32, _ = oracle.nf4_codebook()
    half_gap = np.max(np.diff(l32.astype(np.float64))) / 2
    amax = np.repeat(np.abs(merged.reshape(-1, out_block)).max(axis=1), out_block).reshape(N, K).astype(np.float64)
    bound = amax * (half_gap + 1.0 / 255) + np.abs(exact) * 2 ** -8 + 1e-30
    assert np.all(np.abs(back - exact) <= bound)


# ------------------------------------------------- multi-adapter decode (f3)


def test_multi_adapter_forward_reduces_to_single_adapter(oracle):
    """A stack of adapters with a per-token index: every token's output row is
    the single-adapter forward with its own adapter and scale, and a uniform
    index is the single-adapter forward itself."""
    M, N, K, r, na = 6, 40, 256, 8, 3
    p = wl.draw_small(41, M, N, K, r, 16.0)
    codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(codes, aq, dq, N, K)
    g = wl.generator(42)
    A_all = np.stack([wl.bf16_bits((torch.rand(r, K, generator=g) - 0.5).bfloat16()) for _ in range(na)])
    B_all = np.stack([wl.bf16_bits((torch.randn(N, r, generator=g) * 0.1).bfloat16()) for _ in range(na)])
    scales = [2.0, 0.5, 4.0]
    idx = np.array([2, 0, 1, 1, 2, 0], np.int32)
    X16 = _bits(p["X"])
    Y = oracle.linear_fwd_multi(X16, Wp, A_all, B_all, scales, idx)
    for m in range(M):
        a = idx[m]
        ref = oracle.linear_fwd(X16, Wp, A_all[a], B_all[a], scales[a], rows=np.array([m]))
        assert np.array_equal(Y[m], ref[0])
    Y1 = oracle.linear_fwd_multi(X16, Wp, A_all, B_all, scales, np.ones(M, np.int32))
    assert np.array_equal(Y1, oracle.linear_fwd(X16, Wp, A_all[1], B_all[1], scales[1]))
    with pytest.raises(RuntimeError):
        oracle.linear_fwd_multi(X16, Wp, A_all, B_all, scales, np.array([0, 1, 3, 0, 0, 0], np.int32))


# ------------------------------------------------------ LoRA dropout (f4)


def _dropout_case(oracle, seed=51, M=10, N=24, K=128, r=8):
    p = _small(seed, M, N, K, r)
    codes, aq, dq, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(codes, aq, dq, N, K)
    return p, Wp


def test_dropout_input_rounding(oracle):
    """Xd = mask ? bf16(fl32(x * keep)) : 0: keep = 2 scales exactly, a kept
    element of 1.0 times 1/(1-0.1) rounds to the bf16 nearest fl32(1/0.9)."""
    X = np.array([0x3F80, 0xC040, 0x3F80, 0x0000], np.uint16)  # 1, -3, 1, 0
    m = np.array([1, 1, 0, 1], np.uint8)
    Xd = oracle.dropout_input(X, m, 2.0)
    assert list(Xd) == [0x4000, 0xC0C0, 0, 0]                  # 2, -6, 0, 0
    keep = float(np.float32(1.0 / 0.9))
    Xd = oracle.dropout_input(X[:1], np.ones(1, np.uint8), keep)
    want = torch.tensor([np.float32(keep)]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert Xd[0] == want[0]


def test_dropout_keep_all_is_the_plain_layer(oracle):
    p, Wp = _dropout_case(oracle)
    X16, A16, B16, dY16 = _bits(p["X"]), _bits(p["A"]), _bits(p["B"]), _bits(p["dY"])
    ones = np.ones(X16.shape, np.uint8)
    Y = oracle.linear_fwd_dropout(X16, ones, 1.0, Wp, A16, B16, p["scale"])
    assert np.allclose(Y, oracle.linear_fwd(X16, Wp, A16, B16, p["scale"]), rtol=1e-12, atol=1e-12)
    dX, dA, dB = oracle.linear_bwd_dropout(X16, ones, 1.0, dY16, Wp, A16, B16, p["scale"])
    rX, rA, rB, _ = oracle.linear_bwd(X16, dY16, Wp, A16, B16, p["scale"])
    for a, b in ((dX, rX), (dA, rA), (dB, rB)):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_dropout_drop_all_removes_the_adapter(oracle):
    p, Wp = _dropout_case(oracle)
    X16, A16, B16, dY16 = _bits(p["X"]), _bits(p["A"]), _bits(p["B"]), _bits(p["dY"])
    zeros = np.zeros(X16.shape, np.uint8)
    B0 = np.zeros_like(B16)
    Y = oracle.linear_fwd_dropout(X16, zeros, 1.25, Wp, A16, B16, p["scale"])
    assert np.allclose(Y, oracle.linear_fwd(X16, Wp, A16, B0, p["scale"]), rtol=1e-12, atol=1e-12)
    dX, dA, dB = oracle.linear_bwd_dropout(X16, zeros, 1.25, dY16, Wp, A16, B16, p["scale"])
    rX, _, _, _ = oracle.linear_bwd(X16, dY16, Wp, A16, B0, p["scale"])
    assert np.allclose(dX, rX, rtol=1e-12, atol=1e-12)
    assert not dA.any() and not dB.any()


def test_dropout_backward_is_adjoint_of_forward(oracle):
    """keep = 2 makes Xd = 2 * mask * X exact, so the layer is linear in X and
    in A; the backward must be its adjoint: <dY, J V> = <dX, V>."""
    p, Wp = _dropout_case(oracle)
    M, K = p["X"].shape
    X16, A16, B16, dY16 = _bits(p["X"]), _bits(p["A"]), _bits(p["B"]), _bits(p["dY"])
    g = np.random.default_rng(52)
    mask = (g.random((M, K)) < 0.5).astype(np.uint8)
    s = p["scale"]
    dX, dA, dB = oracle.linear_bwd_dropout(X16, mask, 2.0, dY16, Wp, A16, B16, s)
    dY = oracle._bf16_to_f64(dY16)
    A, B = oracle._bf16_to_f64(A16), oracle._bf16_to_f64(B16)
    V = g.standard_normal((M, K))
    JV = V @ Wp.astype(np.float64).T + s * ((2.0 * mask * V) @ A.T) @ B.T
    assert np.isclose(np.sum(dY * JV), np.sum(dX * V), rtol=1e-10)
    Xd = oracle._bf16_to_f64(oracle.dropout_input(X16, mask, 2.0))
    VA = g.standard_normal(A.shape)
    assert np.isclose(np.sum(dY * (s * (Xd @ VA.T) @ B.T)), np.sum(dA * VA), rtol=1e-10)
