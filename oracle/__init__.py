"""CPU oracle for the QLoRA NF4 linear layer -- TEST INFRASTRUCTURE ONLY.

A plain fp64 C implementation (``nf4_oracle.c``) of what the hot path computes:
the NF4 codebook, blockwise absmax quantization with 8-bit double quantization,
dequantization to bf16, and the layer forward/backward.  Only ``tests/``, the
package's ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this module.  It shares no code with the CUDA library under
``bit_nf4_quantized_24_b200/``; the product path never calls it.

Sources (web pages on QLoRA, by title and section): "What does QLoRA change
compared with plain LoRA when fine-tuning Llama?" (NF4, double quantization),
"QLoRA and Quantized Fine-Tuning" (W' = W_4bit + BA), "QLoRA: fine-tuning a
large model on one GPU" ("LoRA, stated once": h = W0 x + (alpha/r) B A x).

Arrays are numpy.  bf16 tensors travel as their raw ``uint16`` bits.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``nf4_oracle.c`` into ``liboracle.so`` (gcc, OpenMP, -O2).

    Plain IEEE arithmetic: no -ffast-math, so fp32 and fp64 operations round
    exactly as written in the source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.or_nf4_delta.restype = ctypes.c_double
    lib.or_nf4_codebook.argtypes = [P, P, P]
    lib.or_nf4_sizes.argtypes = [i64, i64, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.or_nf4_quantize.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, P, P, P, P]
    lib.or_nf4_dequantize.argtypes = [P, P, P, i64, i64, ctypes.c_int, ctypes.c_int, P, P]
    lib.or_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.or_f32_to_bf16.restype = ctypes.c_uint16
    lib.or_lora_h.argtypes = [P, i64, i64, P, ctypes.c_int, P]
    lib.or_linear_fwd.argtypes = [P, i64, i64, P, i64, P, P, ctypes.c_int, ctypes.c_double,
                                  P, i64, P]
    lib.or_linear_bwd.argtypes = [P, P, i64, i64, P, i64, P, P, ctypes.c_int, ctypes.c_double,
                                  P, i64, P, P, P, P]
    lib.or_num_threads.restype = ctypes.c_int
    lib.or_dropout_input.argtypes = [P, P, ctypes.c_float, i64, P]
    lib.or_linear_fwd_multi.argtypes = [P, i64, i64, P, i64, P, P, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.or_nf4_merge_lora.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, i64, i64, P, P, ctypes.c_int,
                                      ctypes.c_float, ctypes.c_int, ctypes.c_int, P, P, P, P]
    _lib = lib
    return lib


class OracleError(RuntimeError):
    pass


def _check(st: int, what: str):
    if st != 0:
        names = {-1: "ARG", -2: "SHAPE", -3: "NONFINITE"}
        raise OracleError(f"{what}: oracle status {st} ({names.get(st, '?')})")


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().or_num_threads())


def nf4_delta() -> float:
    return float(_load().or_nf4_delta())


def nf4_codebook():
    """Returns (levels_fp64[16], levels_fp32[16], midpoints_fp32[15])."""
    lib = _load()
    l64 = np.zeros(16, np.float64)
    l32 = np.zeros(16, np.float32)
    m32 = np.zeros(15, np.float32)
    _check(lib.or_nf4_codebook(_p(l64), _p(l32), _p(m32)), "codebook")
    return l64, l32, m32


def nf4_sizes(N: int, K: int, block: int = 64, dq_block: int = 256):
    """(codes bytes, absmax_q bytes, dq_scale count) of the NF4 format."""
    lib = _load()
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib.or_nf4_sizes(N, K, block, dq_block, ctypes.byref(a), ctypes.byref(b),
                            ctypes.byref(c)), "sizes")
    return a.value, b.value, c.value


def nf4_quantize(W: np.ndarray, block: int = 64, dq_block: int = 256):
    """W fp32 [N, K] -> (codes u8 [N*K/2], absmax_q u8 [N*K/block],
    dq_scale f32 [groups], absmax f32 [N*K/block] (exact first-level scales)).
    dq_block = 0: no double quantization; absmax_q is empty and dq_scale holds
    the exact fp32 absmax of every block."""
    lib = _load()
    W = _c(W, np.float32)
    N, K = W.shape
    cb, ab, dc = nf4_sizes(N, K, block, dq_block)
    codes = np.zeros(cb, np.uint8)
    aq = np.zeros(max(ab, 1), np.uint8)[:ab]
    dq = np.zeros(dc, np.float32)
    a = np.zeros(N * K // block, np.float32)
    _check(lib.or_nf4_quantize(_p(W), N, K, block, dq_block, _p(codes), _p(aq), _p(dq), _p(a)),
           "quantize")
    return codes, aq, dq, a


def nf4_dequantize(codes, absmax_q, dq_scale, N: int, K: int, block: int = 64,
                   dq_block: int = 256):
    """Returns (bf16 bits u16 [N, K], the same values as fp32 [N, K])."""
    lib = _load()
    codes = _c(codes, np.uint8)
    absmax_q = _c(absmax_q, np.uint8)
    dq_scale = _c(dq_scale, np.float32)
    out16 = np.zeros((N, K), np.uint16)
    out32 = np.zeros((N, K), np.float32)
    _check(lib.or_nf4_dequantize(_p(codes), _p(absmax_q), _p(dq_scale), N, K, block, dq_block,
                                 _p(out16), _p(out32)), "dequantize")
    return out16, out32


def nf4_merge_lora(codes, absmax_q, dq_scale, N: int, K: int, A16, B16, scale: float, block: int = 64,
                   dq_block: int = 256, out_block: int = 64, out_dq_block: int = 256):
    """Merge s * B A into the NF4 weight and quantize the sum again.
    A16: bf16 bits u16 [r, K]; B16: bf16 bits u16 [N, r].  Returns
    (codes, absmax_q, dq_scale, merged fp32 [N, K]) in the output format."""
    lib = _load()
    A16 = _c(A16, np.uint16)
    B16 = _c(B16, np.uint16)
    r = A16.shape[0]
    cb, ab, dc = nf4_sizes(N, K, out_block, out_dq_block)
    oc = np.zeros(cb, np.uint8)
    oa = np.zeros(max(ab, 1), np.uint8)[:ab]
    od = np.zeros(dc, np.float32)
    merged = np.zeros((N, K), np.float32)
    _check(lib.or_nf4_merge_lora(_p(_c(codes, np.uint8)), _p(_c(absmax_q, np.uint8)), _p(_c(dq_scale, np.float32)),
                                 block, dq_block, N, K, _p(A16), _p(B16), r, float(scale), out_block, out_dq_block,
                                 _p(oc), _p(oa), _p(od), _p(merged)), "merge_lora")
    return oc, oa, od, merged


def f32_to_bf16_bits(x: float) -> int:
    return int(_load().or_f32_to_bf16(ctypes.c_float(x)))


def lora_h(X16, A16):
    """H = X A^T (fp64) from bf16 bits X [M,K], A [r,K]."""
    lib = _load()
    X16 = _c(X16, np.uint16)
    A16 = _c(A16, np.uint16)
    M, K = X16.shape
    r = A16.shape[0]
    H = np.zeros((M, r), np.float64)
    _check(lib.or_lora_h(_p(X16), M, K, _p(A16), r, _p(H)), "lora_h")
    return H


def linear_fwd(X16, Wp32, A16, B16, scale: float, rows=None):
    """Y = X Wp^T + s (X A^T) B^T in fp64 for the given rows (all when None).

    X16 bf16 bits [M,K]; Wp32 the dequantized weight [N,K] (fp32 holding bf16
    values); A16 [r,K]; B16 [N,r]."""
    lib = _load()
    X16 = _c(X16, np.uint16)
    Wp32 = _c(Wp32, np.float32)
    A16 = _c(A16, np.uint16)
    B16 = _c(B16, np.uint16)
    M, K = X16.shape
    N = Wp32.shape[0]
    r = A16.shape[0]
    assert Wp32.shape == (N, K) and A16.shape == (r, K) and B16.shape == (N, r)
    rows_a = None if rows is None else _c(rows, np.int64)
    nrows = M if rows is None else len(rows_a)
    Y = np.zeros((nrows, N), np.float64)
    _check(lib.or_linear_fwd(_p(X16), M, K, _p(Wp32), N, _p(A16), _p(B16), r, float(scale),
                             _p(rows_a), nrows, _p(Y)), "linear_fwd")
    return Y


def dropout_input(X16, mask, keep: float):
    """Xd = mask ? bf16(fl32(X * keep)) : 0, as bf16 bits (mask: 1 = keep)."""
    lib = _load()
    X16 = _c(X16, np.uint16)
    mask = _c(mask, np.uint8)
    Xd = np.zeros(X16.shape, np.uint16)
    _check(lib.or_dropout_input(_p(X16), _p(mask), float(keep), X16.size, _p(Xd)), "dropout_input")
    return Xd


def _bf16_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def linear_fwd_dropout(X16, mask, keep, Wp32, A16, B16, scale: float, rows=None):
    """Y with LoRA dropout on the adapter input: the base product uses X, the
    adapter uses Xd = dropout_input(X) (fp64, library matmuls as steps)."""
    B0 = np.zeros_like(_c(B16, np.uint16))
    Y = linear_fwd(X16, Wp32, A16, B0, scale, rows=rows)        # base only
    Xd = _bf16_to_f64(dropout_input(X16, mask, keep))
    if rows is not None:
        Xd = Xd[rows]
    H = Xd @ _bf16_to_f64(A16).T
    return Y + scale * (H @ _bf16_to_f64(B16).T)


def linear_bwd_dropout(X16, mask, keep, dY16, Wp32, A16, B16, scale: float):
    """(dX, dA, dB) with LoRA dropout: dH = s dY B, H = Xd A^T,
    dX = dY Wp + (dH A) * mask * keep, dA = dH^T Xd, dB = s dY^T H."""
    B0 = np.zeros_like(_c(B16, np.uint16))
    dX, _, _, _ = linear_bwd(X16, dY16, Wp32, A16, B0, scale)   # dY Wp (the adapter term is added below)
    Xd = _bf16_to_f64(dropout_input(X16, mask, keep))
    A = _bf16_to_f64(A16)
    B = _bf16_to_f64(B16)
    dY = _bf16_to_f64(dY16)
    dH = scale * (dY @ B)
    dX = dX + (dH @ A) * (np.asarray(mask, np.float64) * float(np.float32(keep)))
    H = Xd @ A.T
    return dX, dH.T @ Xd, scale * (dY.T @ H)


def linear_fwd_multi(X16, Wp32, A16_all, B16_all, scales, idx):
    """Y [M, N] (fp64) of the multi-adapter forward: token m uses adapter
    idx[m] of A16_all [na, r, K], B16_all [na, N, r] with scale scales[na]."""
    lib = _load()
    X16 = _c(X16, np.uint16)
    Wp32 = _c(Wp32, np.float32)
    A16_all = _c(A16_all, np.uint16)
    B16_all = _c(B16_all, np.uint16)
    sc = _c(np.asarray(scales, np.float64), np.float64)
    ix = _c(np.asarray(idx, np.int32), np.int32)
    M, K = X16.shape
    N = Wp32.shape[0]
    na, r = A16_all.shape[0], A16_all.shape[1]
    Y = np.zeros((M, N), np.float64)
    _check(lib.or_linear_fwd_multi(_p(X16), M, K, _p(Wp32), N, _p(A16_all), _p(B16_all), na, r, _p(sc), _p(ix),
                                   _p(Y)), "linear_fwd_multi")
    return Y


def linear_bwd(X16, dY16, Wp32, A16, B16, scale: float, rows=None, want_dx=True):
    """Returns (dX [nrows,K] or None, dA [r,K], dB [N,r], dH [M,r]) in fp64."""
    lib = _load()
    X16 = _c(X16, np.uint16)
    dY16 = _c(dY16, np.uint16)
    Wp32 = _c(Wp32, np.float32)
    A16 = _c(A16, np.uint16)
    B16 = _c(B16, np.uint16)
    M, K = X16.shape
    N = Wp32.shape[0]
    r = A16.shape[0]
    assert dY16.shape == (M, N) and Wp32.shape == (N, K)
    rows_a = None if rows is None else _c(rows, np.int64)
    nrows = (M if rows is None else len(rows_a)) if want_dx else 0
    if not want_dx:
        rows_a = None
    dX = np.zeros((max(nrows, 1), K), np.float64)
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    dH = np.zeros((M, r), np.float64)
    st = lib.or_linear_bwd(_p(X16), _p(dY16), M, K, _p(Wp32), N, _p(A16), _p(B16), r,
                           float(scale), _p(rows_a) if want_dx else None,
                           nrows if (want_dx and rows is not None) else (M if want_dx else 0),
                           _p(dX), _p(dA), _p(dB), _p(dH))
    _check(st, "linear_bwd")
    return (dX[:nrows] if want_dx else None), dA, dB, dH
