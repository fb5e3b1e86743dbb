"""ctypes binding of libqlora_nf4.so (the C ABI in include/qlora_nf4.h).

Argument marshalling only: torch CUDA tensors in, data pointers and the
current stream out, status codes checked.  Every step of the computation runs
in the library's CUDA kernels; if the library is missing this module raises --
there is no CPU fallback.

Function names follow the C ABI: ``nf4_quantize``, ``nf4_dequantize``,
``qlora_linear_fwd``, ``qlora_linear_bwd`` (plus the size and codebook queries).
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlora_nf4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "qlora_nf4.h")

BLOCK = 64
DQ_BLOCK = 256

STATUS = {0: "QLORA_OK", -1: "QLORA_ERR_ARG", -2: "QLORA_ERR_SHAPE", -3: "QLORA_ERR_NONFINITE",
          -4: "QLORA_ERR_WORKSPACE", -5: "QLORA_ERR_CUDA", -6: "QLORA_ERR_TIMEOUT", -7: "QLORA_ERR_UNSUPPORTED"}


class QloraError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        extra = ""
        if status == -5:
            extra = f" (cudaError {lib().qlora_last_cuda_error()})"
        super().__init__(f"{what}: {STATUS.get(status, status)}{extra}")


_lib = None


def lib():
    """Loads the library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_nf4_quantized_24_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.qlora_status_string.restype = ctypes.c_char_p
    L.qlora_status_string.argtypes = [i32]
    L.qlora_last_cuda_error.restype = i32
    L.qlora_version.restype = i32
    L.nf4_quantized_sizes.argtypes = [i64, i64, i32, i32, P, P, P]
    L.nf4_codebook.argtypes = [P]
    L.nf4_quantize.argtypes = [P, i64, i64, i32, i32, P, P, P, P]
    L.nf4_dequantize.argtypes = [P, P, P, i64, i64, i32, i32, P, P]
    L.qlora_linear_fwd_workspace.argtypes = [i64, i64, i64, i32, P]
    L.qlora_linear_bwd_workspace.argtypes = [i64, i64, i64, i32, P]
    L.qlora_linear_fwd.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, f32, P, P, P, sz, P]
    L.qlora_linear_bwd.argtypes = [P, P, P, i64, i64, P, P, i64, P, P, i32, f32, P, P, P, P, P, sz, P]
    L.qlora_linear_fwd_noalloc.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, f32, P, P, P]
    L.qlora_linear_fwd_fmt.argtypes = [P, P, P, i32, i32, i64, i64, P, i64, P, P, i32, f32, P, P, P, sz, P]
    L.nf4_merge_lora.argtypes = [P, P, P, i32, i32, i64, i64, P, P, i32, f32, i32, i32, P, P, P, P]
    L.qlora_linear_fwd_multi.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, i32, P, P, P, P, sz, P]
    L.qlora_linear_dropout_workspace.argtypes = [i64, i64, i64, i32, P]
    L.nf4_decode_tiles_bytes.argtypes = [i64, i64, P]
    L.nf4_decode_tiles.argtypes = [P, i64, i64, P, P]
    L.qlora_linear_fwd_tiles.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, f32, P, P, P, sz, P]
    L.qlora_linear_fwd_tiles_fmt.argtypes = [P, P, P, i32, i32, i64, i64, P, i64, P, P, i32, f32, P, P, P, sz, P]
    L.qlora_linear_fwd_multi_tiles.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, i32, P, P, P, P, sz, P]
    L.qlora_linear_fwd_dropout.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, f32, P, f32, P, P, P, sz, P]
    L.qlora_linear_bwd_dropout.argtypes = [P, P, P, i64, i64, P, P, i64, P, P, i32, f32, P, f32, P, P, P, P, P, sz,
                                           P]
    L.qlora_linear_bwd_fmt.argtypes = [P, P, P, i32, i32, i64, i64, P, P, i64, P, P, i32, f32, P, P, P, P, P, sz,
                                       P]
    L.qlora_device_status.restype = i32
    L.qlora_test_decode_timeout.argtypes = [P, P, P, i64, i64, P, i64, P, P, i32, f32, P, P, sz, P]
    L.qlora_trace_gemm_events.argtypes = [P, i32]
    L.qlora_trace_gemm_count.restype = i32
    L.qlora_gemm_resident_pairs.argtypes = [i32]
    L.qlora_gemm_resident_pairs.restype = i32
    L.qlora_gemm_split_plan.argtypes = [i32, i64, i64, i64, P, P, P]
    _lib = L
    return L


def header_functions() -> list[str]:
    """Names of the functions include/qlora_nf4.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)


def _check(status: int, what: str):
    if status != 0:
        raise QloraError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _req(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def version() -> int:
    return lib().qlora_version()


def status_string(status: int) -> str:
    return lib().qlora_status_string(status).decode()


def nf4_quantized_sizes(N: int, K: int, block: int = BLOCK, dq_block: int = DQ_BLOCK):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().nf4_quantized_sizes(N, K, block, dq_block, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "nf4_quantized_sizes")
    return a.value, b.value, c.value


def nf4_codebook():
    out = (ctypes.c_float * 16)()
    _check(lib().nf4_codebook(ctypes.cast(out, ctypes.c_void_p)), "nf4_codebook")
    return list(out)


class NF4Weight:
    """The three buffers of a quantized [N, K] weight (device tensors) and its
    format: `block` weights per absmax, `dq_block` blocks per second-level
    scale (0: no double quantization; dq_scale then holds each block's fp32
    absmax and absmax_q is empty)."""

    def __init__(self, codes, absmax_q, dq_scale, N, K, block=BLOCK, dq_block=DQ_BLOCK):
        self.codes, self.absmax_q, self.dq_scale = codes, absmax_q, dq_scale
        self.N, self.K = int(N), int(K)
        self.block, self.dq_block = int(block), int(dq_block)

    def _layer_format(self):
        if (self.block, self.dq_block) != (BLOCK, DQ_BLOCK):
            raise QloraError(-7, f"this entry point reads the default NF4 format "
                                 f"(block {BLOCK}, dq_block {DQ_BLOCK}), not ({self.block}, {self.dq_block})")

    @property
    def nbytes(self):
        return self.codes.numel() + self.absmax_q.numel() + 4 * self.dq_scale.numel()


def nf4_quantize(W: torch.Tensor, block: int = BLOCK, dq_block: int = DQ_BLOCK, stream=None) -> NF4Weight:
    _req(W, torch.float32, "W")
    N, K = W.shape
    cb, ab, db = nf4_quantized_sizes(N, K, block, dq_block)
    dev = W.device
    codes = torch.empty(cb, dtype=torch.uint8, device=dev)
    absmax_q = torch.empty(ab, dtype=torch.uint8, device=dev)
    dq_scale = torch.empty(db // 4, dtype=torch.float32, device=dev)
    _check(lib().nf4_quantize(_ptr(W), N, K, block, dq_block, _ptr(codes), _ptr(absmax_q) if ab else None,
                              _ptr(dq_scale), _stream(stream)), "nf4_quantize")
    return NF4Weight(codes, absmax_q, dq_scale, N, K, block, dq_block)


def nf4_dequantize(w: NF4Weight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(w.N, w.K, dtype=torch.bfloat16, device=w.codes.device)
    _req(out, torch.bfloat16, "out", (w.N, w.K))
    _check(lib().nf4_dequantize(_ptr(w.codes), _ptr(w.absmax_q) if w.absmax_q.numel() else None, _ptr(w.dq_scale),
                                w.N, w.K, w.block, w.dq_block, _ptr(out), _stream(stream)), "nf4_dequantize")
    return out


def nf4_merge_lora(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, scale: float, block: int | None = None,
                   dq_block: int | None = None, stream=None) -> NF4Weight:
    """A new NF4 weight holding deq(W) + scale * B A, quantized again (in w's
    format unless block / dq_block are given)."""
    r = A.shape[0]
    _req(A, torch.bfloat16, "A", (r, w.K))
    _req(B, torch.bfloat16, "B", (w.N, r))
    block = w.block if block is None else block
    dq_block = w.dq_block if dq_block is None else dq_block
    cb, ab, db = nf4_quantized_sizes(w.N, w.K, block, dq_block)
    dev = w.codes.device
    codes = torch.empty(cb, dtype=torch.uint8, device=dev)
    absmax_q = torch.empty(ab, dtype=torch.uint8, device=dev)
    dq_scale = torch.empty(db // 4, dtype=torch.float32, device=dev)
    _check(lib().nf4_merge_lora(_ptr(w.codes), _ptr(w.absmax_q) if w.absmax_q.numel() else None, _ptr(w.dq_scale),
                                w.block, w.dq_block, w.N, w.K, _ptr(A), _ptr(B), r, float(scale), block, dq_block,
                                _ptr(codes), _ptr(absmax_q) if ab else None, _ptr(dq_scale), _stream(stream)),
           "nf4_merge_lora")
    return NF4Weight(codes, absmax_q, dq_scale, w.N, w.K, block, dq_block)


def fwd_workspace_bytes(M, N, K, r) -> int:
    b = ctypes.c_size_t()
    _check(lib().qlora_linear_fwd_workspace(M, N, K, r, ctypes.byref(b)), "qlora_linear_fwd_workspace")
    return b.value


def bwd_workspace_bytes(M, N, K, r) -> int:
    b = ctypes.c_size_t()
    _check(lib().qlora_linear_bwd_workspace(M, N, K, r, ctypes.byref(b)), "qlora_linear_bwd_workspace")
    return b.value


def _workspace(nbytes, device, ws):
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def qlora_linear_fwd(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, scale: float,
                     save_h: bool = True, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     stream=None):
    """Y = X deq(W)^T + scale (X A^T) B^T.  Returns (Y, H) with H = X A^T (bf16) or None."""
    M = X.shape[0]
    r = A.shape[0]
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(A, torch.bfloat16, "A", (r, w.K))
    _req(B, torch.bfloat16, "B", (w.N, r))
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _req(out, torch.bfloat16, "Y", (M, w.N))
    H = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if save_h else None
    nbytes = fwd_workspace_bytes(M, w.N, w.K, r)
    ws = _workspace(nbytes, X.device, workspace)
    _check(lib().qlora_linear_fwd_fmt(_ptr(w.codes), _ptr(w.absmax_q) if w.absmax_q.numel() else None,
                                      _ptr(w.dq_scale), w.block, w.dq_block, w.N, w.K, _ptr(X), M, _ptr(A), _ptr(B),
                                      r, float(scale), _ptr(out), _ptr(H), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_linear_fwd")
    return out, H


def dropout_workspace_bytes(M, N, K, r) -> int:
    b = ctypes.c_size_t()
    _check(lib().qlora_linear_dropout_workspace(M, N, K, r, ctypes.byref(b)), "qlora_linear_dropout_workspace")
    return b.value


def qlora_linear_fwd_dropout(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, scale: float,
                             keep_mask: torch.Tensor, keep_scale: float, save_h: bool = True, out=None,
                             workspace=None, stream=None):
    """Forward with LoRA dropout on the adapter input (keep_mask uint8 [M, K],
    1 = keep; keep_scale = 1 / (1 - p)).  Returns (Y, H) with H = Xd A^T."""
    w._layer_format()
    M = X.shape[0]
    r = A.shape[0]
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(A, torch.bfloat16, "A", (r, w.K))
    _req(B, torch.bfloat16, "B", (w.N, r))
    _req(keep_mask, torch.uint8, "keep_mask", (M, w.K))
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    H = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if save_h else None
    ws = _workspace(dropout_workspace_bytes(M, w.N, w.K, r), X.device, workspace)
    _check(lib().qlora_linear_fwd_dropout(_ptr(w.codes), _ptr(w.absmax_q), _ptr(w.dq_scale), w.N, w.K, _ptr(X), M,
                                          _ptr(A), _ptr(B), r, float(scale), _ptr(keep_mask), float(keep_scale),
                                          _ptr(out), _ptr(H), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_linear_fwd_dropout")
    return out, H


def qlora_linear_bwd_dropout(w: NF4Weight, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                             scale: float, keep_mask: torch.Tensor, keep_scale: float, H=None, want_dx=True,
                             workspace=None, stream=None):
    """Backward with LoRA dropout; returns (dX or None, dA, dB)."""
    w._layer_format()
    M = X.shape[0]
    r = A.shape[0]
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(dY, torch.bfloat16, "dY", (M, w.N))
    _req(keep_mask, torch.uint8, "keep_mask", (M, w.K))
    dX = torch.empty(M, w.K, dtype=torch.bfloat16, device=X.device) if want_dx else None
    dA = torch.empty(r, w.K, dtype=torch.bfloat16, device=X.device)
    dB = torch.empty(w.N, r, dtype=torch.bfloat16, device=X.device)
    ws = _workspace(dropout_workspace_bytes(M, w.N, w.K, r), X.device, workspace)
    _check(lib().qlora_linear_bwd_dropout(_ptr(w.codes), _ptr(w.absmax_q), _ptr(w.dq_scale), w.N, w.K, _ptr(X),
                                          _ptr(dY), M, _ptr(A), _ptr(B), r, float(scale), _ptr(keep_mask),
                                          float(keep_scale), _ptr(H), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                                          ws.numel(), _stream(stream)), "qlora_linear_bwd_dropout")
    return dX, dA, dB


def qlora_linear_fwd_multi(w: NF4Weight, X: torch.Tensor, A_all: torch.Tensor, B_all: torch.Tensor,
                           scales: torch.Tensor, adapter_idx: torch.Tensor, out: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, stream=None):
    """Decode with one adapter per token: Y[m] = X[m] deq(W)^T +
    scales[a] (X[m] A_a^T) B_a^T, a = adapter_idx[m] (M <= 16)."""
    w._layer_format()
    M = X.shape[0]
    na, r = A_all.shape[0], A_all.shape[1]
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(A_all, torch.bfloat16, "A_all", (na, r, w.K))
    _req(B_all, torch.bfloat16, "B_all", (na, w.N, r))
    _req(scales, torch.float32, "scales", (na,))
    _req(adapter_idx, torch.int32, "adapter_idx", (M,))
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _req(out, torch.bfloat16, "Y", (M, w.N))
    ws = _workspace(fwd_workspace_bytes(M, w.N, w.K, r), X.device, workspace)
    _check(lib().qlora_linear_fwd_multi(_ptr(w.codes), _ptr(w.absmax_q), _ptr(w.dq_scale), w.N, w.K, _ptr(X), M,
                                        _ptr(A_all), _ptr(B_all), na, r, _ptr(scales), _ptr(adapter_idx), _ptr(out),
                                        _ptr(ws), ws.numel(), _stream(stream)), "qlora_linear_fwd_multi")
    return out


def nf4_decode_tiles_bytes(N: int, K: int) -> int:
    b = ctypes.c_size_t()
    _check(lib().nf4_decode_tiles_bytes(N, K, ctypes.byref(b)), "nf4_decode_tiles_bytes")
    return b.value


def nf4_decode_tiles(w: NF4Weight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The decode-tile copy of w's codes (uint8, nf4_decode_tiles_bytes(N, K)
    bytes) for qlora_linear_fwd_tiles / qlora_linear_fwd_multi_tiles (the
    arrangement of the code bytes does not depend on the format)."""
    nbytes = nf4_decode_tiles_bytes(w.N, w.K)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=w.codes.device)
    _req(out, torch.uint8, "tiles", (nbytes,))
    _check(lib().nf4_decode_tiles(_ptr(w.codes), w.N, w.K, _ptr(out), _stream(stream)), "nf4_decode_tiles")
    return out


def qlora_linear_fwd_tiles(w: NF4Weight, tiles: torch.Tensor, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                           scale: float, save_h: bool = True, out: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, stream=None):
    """qlora_linear_fwd for M <= 16 tokens reading the decode tiles of w's
    codes (w supplies absmax_q, dq_scale, the format and the shape; block 64,
    128 or 256).  Returns (Y, H)."""
    M = X.shape[0]
    r = A.shape[0]
    _req(tiles, torch.uint8, "tiles", (nf4_decode_tiles_bytes(w.N, w.K),))
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(A, torch.bfloat16, "A", (r, w.K))
    _req(B, torch.bfloat16, "B", (w.N, r))
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _req(out, torch.bfloat16, "Y", (M, w.N))
    H = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if save_h else None
    ws = _workspace(fwd_workspace_bytes(M, w.N, w.K, r), X.device, workspace)
    _check(lib().qlora_linear_fwd_tiles_fmt(_ptr(tiles), _ptr(w.absmax_q) if w.absmax_q.numel() else None,
                                            _ptr(w.dq_scale), w.block, w.dq_block, w.N, w.K, _ptr(X), M, _ptr(A),
                                            _ptr(B), r, float(scale), _ptr(out), _ptr(H), _ptr(ws), ws.numel(),
                                            _stream(stream)), "qlora_linear_fwd_tiles")
    return out, H


def qlora_linear_fwd_multi_tiles(w: NF4Weight, tiles: torch.Tensor, X: torch.Tensor, A_all: torch.Tensor,
                                 B_all: torch.Tensor, scales: torch.Tensor, adapter_idx: torch.Tensor,
                                 out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """qlora_linear_fwd_multi reading the decode tiles of w's codes."""
    w._layer_format()
    M = X.shape[0]
    na, r = A_all.shape[0], A_all.shape[1]
    _req(tiles, torch.uint8, "tiles", (nf4_decode_tiles_bytes(w.N, w.K),))
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(A_all, torch.bfloat16, "A_all", (na, r, w.K))
    _req(B_all, torch.bfloat16, "B_all", (na, w.N, r))
    _req(scales, torch.float32, "scales", (na,))
    _req(adapter_idx, torch.int32, "adapter_idx", (M,))
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _req(out, torch.bfloat16, "Y", (M, w.N))
    ws = _workspace(fwd_workspace_bytes(M, w.N, w.K, r), X.device, workspace)
    _check(lib().qlora_linear_fwd_multi_tiles(_ptr(tiles), _ptr(w.absmax_q), _ptr(w.dq_scale), w.N, w.K, _ptr(X), M,
                                              _ptr(A_all), _ptr(B_all), na, r, _ptr(scales), _ptr(adapter_idx),
                                              _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_linear_fwd_multi_tiles")
    return out


def qlora_linear_bwd(w: NF4Weight, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     scale: float, H: torch.Tensor | None = None, want_dx: bool = True,
                     outs=None, workspace: torch.Tensor | None = None, stream=None):
    """Returns (dX or None, dA, dB) for Y = X deq(W)^T + scale (X A^T) B^T."""
    M = X.shape[0]
    r = A.shape[0]
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(dY, torch.bfloat16, "dY", (M, w.N))
    _req(A, torch.bfloat16, "A", (r, w.K))
    _req(B, torch.bfloat16, "B", (w.N, r))
    if H is not None:
        _req(H, torch.bfloat16, "H", (M, r))
    if outs is None:
        dX = torch.empty(M, w.K, dtype=torch.bfloat16, device=X.device) if want_dx else None
        dA = torch.empty(r, w.K, dtype=torch.bfloat16, device=X.device)
        dB = torch.empty(w.N, r, dtype=torch.bfloat16, device=X.device)
    else:
        dX, dA, dB = outs
    nbytes = bwd_workspace_bytes(M, w.N, w.K, r)
    ws = _workspace(nbytes, X.device, workspace)
    _check(lib().qlora_linear_bwd_fmt(_ptr(w.codes), _ptr(w.absmax_q) if w.absmax_q.numel() else None,
                                      _ptr(w.dq_scale), w.block, w.dq_block, w.N, w.K, _ptr(X), _ptr(dY), M, _ptr(A),
                                      _ptr(B), r, float(scale), _ptr(H), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                                      ws.numel(), _stream(stream)), "qlora_linear_bwd")
    return dX, dA, dB


def qlora_linear_fwd_noalloc(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, scale: float,
                             save_h: bool = True, out: torch.Tensor | None = None, stream=None):
    """qlora_linear_fwd without a workspace: the library's fixed device scratch
    is used instead (M * r <= QLORA_NOALLOC_MAX_TOKENS_X_RANK).  Returns (Y, H)."""
    w._layer_format()
    M = X.shape[0]
    r = A.shape[0]
    _req(X, torch.bfloat16, "X", (M, w.K))
    _req(A, torch.bfloat16, "A", (r, w.K))
    _req(B, torch.bfloat16, "B", (w.N, r))
    if out is None:
        out = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _req(out, torch.bfloat16, "Y", (M, w.N))
    H = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if save_h else None
    _check(lib().qlora_linear_fwd_noalloc(_ptr(w.codes), _ptr(w.absmax_q), _ptr(w.dq_scale), w.N, w.K, _ptr(X), M,
                                          _ptr(A), _ptr(B), r, float(scale), _ptr(out), _ptr(H), _stream(stream)),
           "qlora_linear_fwd_noalloc")
    return out, H


def gemm_resident_pairs(mode: int = 0) -> int:
    """CTA pairs of the fused GEMM that fit on the current device at once."""
    return lib().qlora_gemm_resident_pairs(mode)


def gemm_split_plan(mode: int, M: int, N: int, K: int) -> tuple[int, int, int]:
    """(pieces per split tile, split tiles, bytes of fp32 partial sums) of the
    fused GEMM for an M x N x K layer on the current device."""
    ns, nt, pb = ctypes.c_int(), ctypes.c_int64(), ctypes.c_size_t()
    _check(lib().qlora_gemm_split_plan(mode, M, N, K, ctypes.byref(ns), ctypes.byref(nt), ctypes.byref(pb)),
           "qlora_gemm_split_plan")
    return ns.value, nt.value, pb.value


def device_status() -> int:
    """Reads and clears the device status word (synchronizes the device)."""
    return lib().qlora_device_status()


class GemmTrace:
    """Records CUDA events around every fused dequant-GEMM launch (up to
    `capacity` launches) while active; ``times_ms()`` returns their durations."""

    def __init__(self, capacity: int):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:  # torch creates the CUDA event lazily, on first record
            e.record()
        self._arr = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self.capacity = capacity

    def __enter__(self):
        _check(lib().qlora_trace_gemm_events(ctypes.cast(self._arr, ctypes.c_void_p), self.capacity), "trace")
        return self

    def __exit__(self, *exc):
        self.count = lib().qlora_trace_gemm_count()
        lib().qlora_trace_gemm_events(None, 0)
        return False

    def times_ms(self):
        torch.cuda.synchronize()
        return [self.events[2 * i].elapsed_time(self.events[2 * i + 1]) for i in range(self.count)]
