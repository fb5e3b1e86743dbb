"""The C-ABI library loads, exports every function the header declares, and
rejects bad arguments before touching the GPU.  Runs without a GPU."""
import ctypes

import numpy as np
import pytest

from bit_nf4_quantized_24_b200 import binding as qb


@pytest.fixture(scope="module")
def L():
    from bit_nf4_quantized_24_b200 import build
    build.build()
    return qb.lib()


def test_exports_every_declared_function(L):
    names = qb.header_functions()
    for must in ["nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd", "nf4_quantized_sizes",
                 "nf4_codebook", "qlora_linear_fwd_workspace", "qlora_linear_bwd_workspace"]:
        assert must in names
    for n in names:
        assert hasattr(L, n), f"library does not export {n}"


def test_status_strings_and_version(L):
    for code in range(0, -8, -1):
        assert qb.status_string(code).startswith(qb.STATUS[code])
    assert qb.version() >> 16 == 1


def test_codebook_matches_oracle_bit_for_bit(L, oracle):
    """The library computes its table with its own code (Newton on erfc); the
    oracle with bisection.  Both must round to the same fp32 levels."""
    lib_levels = np.array(qb.nf4_codebook(), np.float32)
    _, o32, _ = oracle.nf4_codebook()
    assert lib_levels.tobytes() == o32.tobytes()


def test_sizes_match_oracle_format(L, oracle):
    for N, K in [(1, 64), (3, 192), (4096, 4096), (28672, 8192), (11008, 4096)]:
        cb, ab, db = qb.nf4_quantized_sizes(N, K)
        ocb, oab, odc = oracle.nf4_sizes(N, K)
        assert (cb, ab, db) == (ocb, oab, 4 * odc)
    for block in (32, 64, 128, 256):
        for dq in (256, 0):
            cb, ab, db = qb.nf4_quantized_sizes(7, 1024, block, dq)
            assert (cb, ab, db) == tuple(v * (4 if k == 2 else 1)
                                         for k, v in enumerate(oracle.nf4_sizes(7, 1024, block, dq)))


def test_argument_errors_return_before_any_device_work(L):
    i = ctypes.c_size_t()
    assert L.nf4_quantized_sizes(4, 96, 64, 256, ctypes.byref(i), ctypes.byref(i), ctypes.byref(i)) == -2
    assert L.nf4_quantized_sizes(4, 192, 48, 256, ctypes.byref(i), ctypes.byref(i), ctypes.byref(i)) == -7
    assert L.nf4_quantized_sizes(4, 128, 64, 128, ctypes.byref(i), ctypes.byref(i), ctypes.byref(i)) == -7
    assert L.nf4_quantized_sizes(-1, 64, 64, 256, ctypes.byref(i), ctypes.byref(i), ctypes.byref(i)) == -1
    assert L.nf4_codebook(None) == -1
    assert L.qlora_linear_fwd_workspace(16, 64, 64, 12, ctypes.byref(i)) == -7
    assert L.qlora_linear_fwd_workspace(16, 64, 64, 0, ctypes.byref(i)) == -1
    assert L.qlora_linear_fwd_workspace(16, 64, 96, 16, ctypes.byref(i)) == -2
    assert L.qlora_linear_bwd_workspace(16, 60, 64, 16, ctypes.byref(i)) == -2
    # null tensors are rejected before any launch
    assert L.qlora_linear_fwd(None, None, None, 64, 64, None, 16, None, None, 16, ctypes.c_float(2.0), None, None,
                              None, 0, None) == -1
    assert L.qlora_linear_bwd(None, None, None, 64, 64, None, None, 16, None, None, 16, ctypes.c_float(2.0), None,
                              None, None, None, None, 0, None) == -1
    assert L.qlora_trace_gemm_events(None, -1) == -1
    # decode tiles: K % 1024 == 0, M <= 16
    assert L.nf4_decode_tiles_bytes(40, 1088, ctypes.byref(i)) == -2
    assert L.nf4_decode_tiles_bytes(0, 1024, ctypes.byref(i)) == -1
    assert L.nf4_decode_tiles_bytes(40, 1024, ctypes.byref(i)) == 0 and i.value == 3 * 16 * 512
    assert L.nf4_decode_tiles(None, 40, 1024, None, None) == -1
    f2 = ctypes.c_float(2.0)
    assert L.qlora_linear_fwd_tiles(None, None, None, 64, 1024, None, 17, None, None, 16, f2, None, None, None, 0,
                                    None) == -7
    assert L.qlora_linear_fwd_tiles(None, None, None, 64, 1088, None, 4, None, None, 16, f2, None, None, None, 0,
                                    None) == -2
    assert L.qlora_linear_fwd_tiles(None, None, None, 64, 1024, None, 4, None, None, 16, f2, None, None, None, 0,
                                    None) == -1
    assert L.qlora_linear_fwd_multi_tiles(None, None, None, 64, 1024, None, 4, None, None, 2, 16, None, None, None,
                                          None, 0, None) == -1


def test_workspace_sizes_grow_with_shape(L):
    a = qb.fwd_workspace_bytes(128, 2048, 2048, 8)
    b = qb.fwd_workspace_bytes(4096, 4096, 4096, 16)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    assert qb.bwd_workspace_bytes(4096, 4096, 4096, 16) > qb.bwd_workspace_bytes(128, 2048, 2048, 8)


def test_split_plan_without_a_device(L):
    """The fused GEMM's split plan needs the device's resident CTA pairs:
    without a device every tile runs whole and the workspace functions add no
    room for partial sums; bad arguments are rejected."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("checks the host-only answer")
    for mode in (0, 1):
        assert qb.gemm_split_plan(mode, 4096, 1024, 8192) == (1, 0, 0)
    ns, nt, pb = ctypes.c_int(), ctypes.c_int64(), ctypes.c_size_t()
    assert L.qlora_gemm_split_plan(2, 4096, 1024, 8192, ctypes.byref(ns), ctypes.byref(nt), ctypes.byref(pb)) == -1
    assert L.qlora_gemm_split_plan(0, -1, 1024, 8192, None, None, None) == -1
    assert L.qlora_gemm_split_plan(0, 4096, 1024, 8192, None, None, None) == 0  # NULL outputs allowed
    M, r = 4096, 64
    assert qb.fwd_workspace_bytes(M, 1024, 8192, r) == M * r * 2  # Hs only


def test_midpoints_avoid_the_quantizer_cell_edges(L):
    """The GPU quantizer finds a code from the 1/64-wide cell that holds
    t = w / absmax (cell edges at odd multiples of 1/128) plus one compare with
    the single midpoint inside the cell.  That is exact only if cells are
    narrower than the midpoint spacing and no midpoint sits on a cell edge."""
    lv = (ctypes.c_float * 16)()
    assert L.nf4_codebook(lv) == 0
    levels = np.array(list(lv), dtype=np.float32)
    mids = ((levels[:-1] + levels[1:]) * np.float32(0.5)).astype(np.float32)
    assert np.all(np.diff(mids.astype(np.float64)) > 1.0 / 64)
    scaled = mids.astype(np.float64) * 128.0
    on_edge = (scaled == np.round(scaled)) & (np.round(scaled) % 2 == 1)
    assert not on_edge.any()


def test_cuda_failure_is_reported_by_both_forward_entry_points(L):
    """Without a usable CUDA device (this test runs only where there is none),
    the first CUDA call of a forward fails on the host: the workspace entry
    point and the no-workspace one both return QLORA_ERR_CUDA and record the
    CUDA error for qlora_last_cuda_error() on the calling thread.  The pointers
    are never dereferenced (nothing reaches a device)."""
    import threading

    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a host without a usable CUDA device")
    P = ctypes.c_void_p
    fake, ws = P(0x10000), P(0x20000)
    res = {}

    def run(name, call):
        res[name] = (L.qlora_last_cuda_error(), call(), L.qlora_last_cuda_error())

    calls = {
        "noalloc": lambda: L.qlora_linear_fwd_noalloc(fake, fake, fake, 256, 256, fake, 32, fake, fake, 16,
                                                      ctypes.c_float(2.0), fake, None, None),
        "workspace": lambda: L.qlora_linear_fwd(fake, fake, fake, 256, 256, fake, 32, fake, fake, 16,
                                                ctypes.c_float(2.0), fake, None, ws, 1 << 20, None),
    }
    for name, call in calls.items():  # a fresh host thread each: its last error starts at 0
        t = threading.Thread(target=run, args=(name, call))
        t.start()
        t.join()
        before, status, after = res[name]
        assert before == 0 and status == -5 and after != 0, (name, res[name])
