"""qlora_linear_fwd_noalloc: the forward entry point for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the
library).  Called through the C ABI and compared with qlora_linear_fwd, which
takes a caller-allocated workspace, and with the CPU oracle, on two calls in a
row with different inputs, on both the decode path (M <= 16) and the
tensor-core GEMM path, with and without H; once more through the Python
wrapper.

This file is collected last so that a run that stops at the first failure has
run every other test before it; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

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


def _relfro(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _call_noalloc(qb, q, X, A, B, scale, Y, H):
    L = qb.lib()
    return L.qlora_linear_fwd_noalloc(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), q.N, q.K,
                                      qb._ptr(X), X.shape[0], qb._ptr(A), qb._ptr(B), A.shape[0],
                                      ctypes.c_float(scale), qb._ptr(Y), qb._ptr(H), qb._stream())


def _call_with_workspace(qb, q, X, A, B, scale):
    M, r = X.shape[0], A.shape[0]
    Y = torch.empty(M, q.N, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(qb.fwd_workspace_bytes(M, q.N, q.K, r), dtype=torch.uint8, device="cuda")
    L = qb.lib()
    st = L.qlora_linear_fwd(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), q.N, q.K, qb._ptr(X), M,
                            qb._ptr(A), qb._ptr(B), r, ctypes.c_float(scale), qb._ptr(Y), qb._ptr(H), qb._ptr(ws),
                            ws.numel(), qb._stream())
    assert st == 0
    return Y, H


def _oracle_y(oracle, q, p):
    """The oracle's Y for the GPU-quantized weight (the oracle dequantizes the
    same codes; the quantizer itself is compared bit for bit elsewhere)."""
    _, Wp = oracle.nf4_dequantize(q.codes.cpu().numpy(), q.absmax_q.cpu().numpy(), q.dq_scale.cpu().numpy(),
                                  q.N, q.K)
    return oracle.linear_fwd(wl.bf16_bits(p["X"]), Wp, wl.bf16_bits(p["A"]), wl.bf16_bits(p["B"]), p["scale"])


@pytest.mark.parametrize("save_h", [True, False])
@pytest.mark.parametrize("M,N,K,r", [(200, 520, 1024, 16), (7, 264, 2048, 64)])
def test_noalloc_matches_workspace_entry_point_twice(qb, oracle, M, N, K, r, save_h):
    """Two calls in a row with different inputs, through the C ABI: Y (and H
    when asked for) agree with the workspace entry point and with the oracle."""
    q = qb.nf4_quantize(wl.draw_weight(wl.generator(5 + M), N, K, 0.02).cuda())
    for call in range(2):  # the second call must not see the first call's scratch
        p = wl.draw_small(600 + 10 * call + M, M, N, K, r, 2.0 * r, b_std=0.5, with_dy=False)
        X, A, B = p["X"].cuda(), p["A"].cuda(), p["B"].cuda()
        Yref, Href = _call_with_workspace(qb, q, X, A, B, p["scale"])
        Y = torch.empty_like(Yref)
        H = torch.empty_like(Href) if save_h else None
        assert _call_noalloc(qb, q, X, A, B, p["scale"], Y, H) == 0
        torch.cuda.synchronize()
        assert _relfro(Y, Yref) <= TOL
        if save_h:
            assert _relfro(H, Href) <= TOL
        Yo = _oracle_y(oracle, q, p)
        err = np.linalg.norm(Y.float().cpu().numpy().astype(np.float64) - Yo) / np.linalg.norm(Yo)
        assert err <= TOL, f"Y against the oracle: {err}"


def test_noalloc_through_the_binding(qb, oracle):
    """The Python wrapper of the entry point, without H."""
    M, N, K, r = 40, 136, 1024, 8
    q = qb.nf4_quantize(wl.draw_weight(wl.generator(41), N, K, 0.02).cuda())
    p = wl.draw_small(640, M, N, K, r, 16.0, b_std=0.5, with_dy=False)
    Y, H = qb.qlora_linear_fwd_noalloc(q, p["X"].cuda(), p["A"].cuda(), p["B"].cuda(), p["scale"], save_h=False)
    torch.cuda.synchronize()
    assert H is None
    Yo = _oracle_y(oracle, q, p)
    err = np.linalg.norm(Y.float().cpu().numpy().astype(np.float64) - Yo) / np.linalg.norm(Yo)
    assert err <= TOL


def test_noalloc_rejects_more_than_its_scratch(qb):
    N, K, r = 64, 64, 64
    q = qb.nf4_quantize(torch.randn(N, K, device="cuda") * 0.02)
    M = (1 << 20) // r + 1  # one token more than the fixed scratch holds
    # a real X / Y are not needed: the size check comes before anything is read
    X = torch.empty(16, K, dtype=torch.bfloat16, device="cuda")
    A = torch.empty(r, K, dtype=torch.bfloat16, device="cuda")
    B = torch.empty(N, r, dtype=torch.bfloat16, device="cuda")
    L = qb.lib()
    st = L.qlora_linear_fwd_noalloc(qb._ptr(q.codes), qb._ptr(q.absmax_q), qb._ptr(q.dq_scale), N, K, qb._ptr(X), M,
                                    qb._ptr(A), qb._ptr(B), r, ctypes.c_float(1.0), qb._ptr(X), None, qb._stream())
    assert st == -4  # QLORA_ERR_WORKSPACE
    assert qb.device_status() == 0
