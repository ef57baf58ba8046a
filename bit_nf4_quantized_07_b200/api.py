"""Thin ctypes binding of libqlora_nf4.so (the C ABI in include/qlora_nf4.h).

Argument marshalling only: tensors are torch CUDA tensors (torch provides the
device memory and the current stream); every step of the computation runs in
the library's CUDA kernels.  There is no fallback: if the library is missing
or a call fails, an exception is raised.

Function names follow the C entry points: ``nf4_quantize``,
``nf4_double_quant``, ``nf4_dequant``, ``qlora_linear_fwd``,
``qlora_linear_bwd``, plus ``workspace_bytes``, ``codebook``, ``version``.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLN_OK = 0
STATUS_NAMES = {0: "QLN_OK", 1: "QLN_ERR_NULL", 2: "QLN_ERR_SHAPE", 3: "QLN_ERR_ALIGN", 4: "QLN_ERR_WORKSPACE",
                5: "QLN_ERR_ARCH", 6: "QLN_ERR_CUDA", 7: "QLN_ERR_TIMEOUT", 8: "QLN_ERR_INTERNAL"}
OP_DOUBLE_QUANT, OP_LINEAR_FWD, OP_LINEAR_BWD, OP_QUANTIZE_DQ_BATCH = 1, 2, 3, 4

#: Every symbol include/qlora_nf4.h declares.
EXPORTS = ("nf4_quantize", "nf4_quantize_ex", "nf4_quantize_dq", "nf4_quantize_dq_batch", "nf4_double_quant", "nf4_double_quant_ex", "nf4_double_quant_noalloc",
           "nf4_dequant",
           "nf4_dequant_flat", "qlora_linear_fwd", "qlora_linear_bwd", "qln_workspace_bytes", "qln_codebook",
           "qln_status_str", "qln_version", "qln_launch_count", "qln_adamw_step")
DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2
DQ_FORMATS = {"int8": 0, "e4m3": 1}


class QLNError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class CAdamWConfig(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


ADAMW_PAGE_IN, ADAMW_PAGE_OUT = 1, 2


class CQuantJob(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("numel", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("dq_format", ctypes.c_int32), ("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("qabs", ctypes.c_void_p), ("dq_scale", ctypes.c_void_p), ("dq_mean", ctypes.c_void_p)]


class CNF4Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p), ("qabs", ctypes.c_void_p),
                ("dq_scale", ctypes.c_void_p), ("dq_mean", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("dq_format", ctypes.c_int32)]


_lib = None


def lib():
    """Load libqlora_nf4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with bit_nf4_quantized_07_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
        WP = ctypes.POINTER(CNF4Weight)
        sig = {
            "nf4_quantize": ([P, I64, P, P, P], I32),
            "nf4_quantize_ex": ([P, I32, I64, P, P, P], I32),
            "nf4_quantize_dq": ([P, I32, I64, I32, P, P, P, P, P, P, SZ, P], I32),
            "nf4_quantize_dq_batch": ([P, I32, P, SZ, P], I32),
            "nf4_double_quant": ([P, I64, P, P, P, P, SZ, P], I32),
            "nf4_double_quant_ex": ([P, I64, I32, P, P, P, P, SZ, P], I32),
            "nf4_double_quant_noalloc": ([P, I64, P, P, P, P], I32),
            "nf4_dequant": ([WP, P, P], I32),
            "nf4_dequant_flat": ([WP, I64, P, P], I32),
            "qlora_linear_fwd": ([WP, P, I64, P, P, I32, F, P, P, P, SZ, P], I32),
            "qlora_linear_bwd": ([WP, P, I64, P, P, I32, F, P, P, P, P, P, P, SZ, P], I32),
            "qln_workspace_bytes": ([I32, I64, I64, I64, I32], SZ),
            "qln_codebook": ([P], None),
            "qln_status_str": ([I32], ctypes.c_char_p),
            "qln_version": ([], I32),
            "qln_launch_count": ([], ctypes.c_uint64),
            "qln_adamw_step": ([P, P, P, P, P, I64, ctypes.POINTER(CAdamWConfig), P, I32, P], I32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(fn, st):
    if st != QLN_OK:
        raise QLNError(fn, st)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def version() -> int:
    return lib().qln_version()


def launch_count() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(lib().qln_launch_count())


def codebook() -> torch.Tensor:
    """The 16 fp32 NF4 values the kernels use (host copy)."""
    out = (ctypes.c_float * 16)()
    lib().qln_codebook(out)
    return torch.tensor(list(out), dtype=torch.float32)


def status_str(st: int) -> str:
    return lib().qln_status_str(st).decode()


def workspace_bytes(op: int, rows: int, cols: int = 0, n: int = 0, r: int = 0) -> int:
    return int(lib().qln_workspace_bytes(op, rows, cols, n, r))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Device scratch (torch-allocated, 256-byte aligned by the caching
    allocator), zero-filled: the counters in the workspace header must start
    at zero, and every call leaves them there."""
    t = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")
    assert t.data_ptr() % 256 == 0
    return t


@dataclass
class NF4Weight:
    """An NF4 weight [rows][cols] as stored on the device."""
    codes: torch.Tensor                    # uint8 [rows*cols/2]
    rows: int
    cols: int
    absmax: Optional[torch.Tensor] = None  # fp32 [nb]
    qabs: Optional[torch.Tensor] = None    # int8 [nb]
    dq_scale: Optional[torch.Tensor] = None
    dq_mean: Optional[torch.Tensor] = None
    dq_format: str = "int8"                # how qabs is stored: "int8" or "e4m3"

    def c_struct(self) -> CNF4Weight:
        return CNF4Weight(self.codes.data_ptr(), self.absmax.data_ptr() if self.absmax is not None else None,
                          self.qabs.data_ptr() if self.qabs is not None else None,
                          self.dq_scale.data_ptr() if self.dq_scale is not None else None,
                          self.dq_mean.data_ptr() if self.dq_mean is not None else None, self.rows, self.cols,
                          DQ_FORMATS[self.dq_format])


_DTYPES = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}


def nf4_quantize(W: torch.Tensor, codes: Optional[torch.Tensor] = None, absmax: Optional[torch.Tensor] = None):
    """W (fp32, bf16 or fp16; any shape and numel) -> (codes uint8 [ceil(numel/2)],
    absmax fp32 [ceil(numel/64)]).  fp32 weights in whole 64-blocks go through
    nf4_quantize, everything else through nf4_quantize_ex (same bits for the
    same values)."""
    n = W.numel()
    if W.dtype not in _DTYPES:
        raise ValueError(f"unsupported weight dtype {W.dtype}")
    if codes is None:
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=W.device)
    if absmax is None:
        absmax = torch.empty((n + 63) // 64, dtype=torch.float32, device=W.device)
    _need_cuda(W, codes, absmax)
    if W.dtype == torch.float32 and n % 64 == 0:
        _check("nf4_quantize", lib().nf4_quantize(_p(W), n, _p(codes), _p(absmax), _stream()))
    else:
        _check("nf4_quantize_ex", lib().nf4_quantize_ex(_p(W), _DTYPES[W.dtype], n, _p(codes), _p(absmax),
                                                        _stream()))
    return codes, absmax


def nf4_quantize_dq(W: torch.Tensor, codes=None, absmax=None, qabs=None, dq_scale=None, dq_mean=None, ws=None,
                    fmt: str = "int8"):
    """W (fp32/bf16/fp16) -> (codes, absmax, qabs, dq_scale, dq_mean): nf4_quantize
    then nf4_double_quant in one call (nf4_quantize_dq), the same bits."""
    if W.dtype not in _DTYPES:
        raise ValueError(f"unsupported weight dtype {W.dtype}")
    n = W.numel()
    nb = (n + 63) // 64
    dev = W.device
    if codes is None:
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev)
    if absmax is None:
        absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    if qabs is None:
        qabs = torch.empty(nb, dtype=torch.int8 if fmt == "int8" else torch.uint8, device=dev)
    if dq_scale is None:
        dq_scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    if dq_mean is None:
        dq_mean = torch.empty(1, dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_DOUBLE_QUANT, nb), dev)
    _need_cuda(W, codes, absmax, qabs, dq_scale, dq_mean, ws)
    _check("nf4_quantize_dq", lib().nf4_quantize_dq(_p(W), _DTYPES[W.dtype], n, DQ_FORMATS[fmt], _p(codes),
                                                    _p(absmax), _p(qabs), _p(dq_scale), _p(dq_mean), _p(ws),
                                                    ws.numel(), _stream()))
    return codes, absmax, qabs, dq_scale, dq_mean


def nf4_quantize_dq_batch(jobs, ws=None):
    """nf4_quantize_dq of several weights in one call (nf4_quantize_dq_batch).

    jobs: a sequence of (W, codes, absmax, qabs, dq_scale, dq_mean, fmt)
    tuples with the outputs allocated as nf4_quantize_dq would."""
    jobs = list(jobs)
    arr = (CQuantJob * len(jobs))()
    dev = jobs[0][0].device if jobs else None
    for i, (W, codes, absmax, qabs, dq_scale, dq_mean, fmt) in enumerate(jobs):
        if W.dtype not in _DTYPES:
            raise ValueError(f"unsupported weight dtype {W.dtype}")
        if fmt not in DQ_FORMATS:
            raise ValueError(f"job {i}: unknown double-quantization format {fmt!r}")
        n = W.numel()
        nb = (n + 63) // 64
        # the library writes through raw pointers: check dtypes, sizes and layout here
        for name, t, dts, need in (("codes", codes, (torch.uint8,), (n + 1) // 2),
                                   ("absmax", absmax, (torch.float32,), nb),
                                   ("qabs", qabs, (torch.int8, torch.uint8), nb),
                                   ("dq_scale", dq_scale, (torch.float32,), (nb + 255) // 256),
                                   ("dq_mean", dq_mean, (torch.float32,), 1)):
            if t.dtype not in dts:
                raise ValueError(f"job {i}: {name} must be {' or '.join(map(str, dts))}, got {t.dtype}")
            if t.numel() < need:
                raise ValueError(f"job {i}: {name} holds {t.numel()} elements, needs {need}")
            if not t.is_contiguous():
                raise ValueError(f"job {i}: {name} must be contiguous")
            if t.device != W.device:
                raise ValueError(f"job {i}: {name} is on {t.device}, W on {W.device}")
        _need_cuda(W, codes, absmax, qabs, dq_scale, dq_mean)
        arr[i] = CQuantJob(_p(W), n, _DTYPES[W.dtype], DQ_FORMATS[fmt], _p(codes), _p(absmax), _p(qabs),
                           _p(dq_scale), _p(dq_mean))
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_QUANTIZE_DQ_BATCH, len(jobs)), dev)
    _need_cuda(ws)
    _check("nf4_quantize_dq_batch", lib().nf4_quantize_dq_batch(arr, len(jobs), _p(ws), ws.numel(), _stream()))


def nf4_double_quant(absmax: torch.Tensor, qabs=None, dq_scale=None, dq_mean=None, ws=None, fmt: str = "int8"):
    """fp32 absmax [nb] -> (qabs [nb], dq_scale fp32 [ceil(nb/256)], dq_mean fp32 [1]).

    fmt "int8": qabs int8 (nf4_double_quant); "e4m3": qabs uint8 E4M3 codes
    (nf4_double_quant_ex) -- set NF4Weight.dq_format to match."""
    nb = absmax.numel()
    dev = absmax.device
    if qabs is None:
        qabs = torch.empty(nb, dtype=torch.int8 if fmt == "int8" else torch.uint8, device=dev)
    if dq_scale is None:
        dq_scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    if dq_mean is None:
        dq_mean = torch.empty(1, dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_DOUBLE_QUANT, nb), dev)
    _need_cuda(absmax, qabs, dq_scale, dq_mean, ws)
    if fmt == "int8":
        _check("nf4_double_quant", lib().nf4_double_quant(_p(absmax), nb, _p(qabs), _p(dq_scale), _p(dq_mean),
                                                          _p(ws), ws.numel(), _stream()))
    else:
        _check("nf4_double_quant_ex", lib().nf4_double_quant_ex(_p(absmax), nb, DQ_FORMATS[fmt], _p(qabs),
                                                                _p(dq_scale), _p(dq_mean), _p(ws), ws.numel(),
                                                                _stream()))
    return qabs, dq_scale, dq_mean


def nf4_double_quant_noalloc(absmax: torch.Tensor, qabs, dq_scale, dq_mean):
    """nf4_double_quant into caller-provided outputs, with no device workspace:
    for callers that cannot allocate device memory (see the header)."""
    nb = absmax.numel()
    # the library writes nb codes, ceil(nb / 256) scales and one mean through
    # raw pointers: check dtypes, sizes, layout and device here
    ng = (nb + 255) // 256
    for name, t, dt, need in (("absmax", absmax, torch.float32, nb), ("qabs", qabs, torch.int8, nb),
                              ("dq_scale", dq_scale, torch.float32, ng), ("dq_mean", dq_mean, torch.float32, 1)):
        if t.dtype != dt:
            raise ValueError(f"{name} must be {dt}, got {t.dtype}")
        if t.numel() < need:
            raise ValueError(f"{name} holds {t.numel()} elements, needs {need}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device != absmax.device:
            raise ValueError(f"{name} is on {t.device}, absmax on {absmax.device}")
    _need_cuda(absmax, qabs, dq_scale, dq_mean)
    _check("nf4_double_quant_noalloc", lib().nf4_double_quant_noalloc(_p(absmax), nb, _p(qabs), _p(dq_scale),
                                                                      _p(dq_mean), _stream()))
    return qabs, dq_scale, dq_mean


def quantize_weight(W: torch.Tensor, double_quant: bool = True, ws=None, dq_format: str = "int8") -> NF4Weight:
    """nf4_quantize_dq (or nf4_quantize alone without double quantization)
    of a [rows][cols] weight (fp32, bf16 or fp16)."""
    rows, cols = W.shape
    if double_quant:
        codes, absmax, qabs, scale, mean = nf4_quantize_dq(W, ws=ws, fmt=dq_format)
        return NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax, qabs=qabs, dq_scale=scale, dq_mean=mean,
                         dq_format=dq_format)
    codes, absmax = nf4_quantize(W)
    w = NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax)
    return w


def nf4_dequant(w: NF4Weight, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """doubleDequant to BF16 [rows][cols]."""
    if out is None:
        out = torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=w.codes.device)
    _need_cuda(w.codes, out)
    cw = w.c_struct()
    _check("nf4_dequant", lib().nf4_dequant(ctypes.byref(cw), _p(out), _stream()))
    return out


def nf4_dequant_flat(w: NF4Weight, numel: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """doubleDequant of a flat weight of any numel to BF16 [numel] (w.rows and
    w.cols are not used)."""
    if out is None:
        out = torch.empty(numel, dtype=torch.bfloat16, device=w.codes.device)
    _need_cuda(w.codes, out)
    cw = w.c_struct()
    _check("nf4_dequant_flat", lib().nf4_dequant_flat(ctypes.byref(cw), int(numel), _p(out), _stream()))
    return out


def qlora_linear_fwd(w: NF4Weight, X, A, B, s: float, Y=None, U_out=None, ws=None, want_u: bool = True):
    """Y = X W'^T + s (X A^T) B^T.  Returns (Y [n][dout] bf16, U [n][r] bf16 or None)."""
    n = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty(n, w.rows, dtype=torch.bfloat16, device=dev)
    if U_out is None and want_u:
        U_out = torch.empty(n, r, dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_LINEAR_FWD, w.rows, w.cols, n, r), dev)
    _need_cuda(X, A, B, Y, U_out, ws)
    cw = w.c_struct()
    _check("qlora_linear_fwd", lib().qlora_linear_fwd(ctypes.byref(cw), _p(X), n, _p(A), _p(B), r, float(s), _p(Y),
                                                      _p(U_out), _p(ws), ws.numel(), _stream()))
    return Y, U_out


def qlora_linear_bwd(w: NF4Weight, X, A, B, s: float, dY, U=None, dX=None, dA=None, dB=None, ws=None):
    """Returns (dX [n][din] bf16, dA [r][din] fp32, dB [dout][r] fp32)."""
    n = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if dX is None:
        dX = torch.empty(n, w.cols, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(r, w.cols, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(w.rows, r, dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_LINEAR_BWD, w.rows, w.cols, n, r), dev)
    _need_cuda(X, A, B, dY, U, dX, dA, dB, ws)
    cw = w.c_struct()
    _check("qlora_linear_bwd", lib().qlora_linear_bwd(ctypes.byref(cw), _p(X), n, _p(A), _p(B), r, float(s), _p(dY),
                                                      _p(U), _p(dX), _p(dA), _p(dB), _p(ws), ws.numel(), _stream()))
    return dX, dA, dB


def device_status(ws: torch.Tensor) -> int:
    """The int32 status word at workspace offset 0 (synchronises the current stream)."""
    return int(ws[:4].view(torch.int32).item())


def adamw_step(param: torch.Tensor, grad: torch.Tensor, m: torch.Tensor, v: torch.Tensor, step: torch.Tensor,
               lr: float, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
               param_bf16: Optional[torch.Tensor] = None, flags: int = 0):
    """One AdamW update of an fp32 master tensor in place (qln_adamw_step).
    ``step`` is a device int64 tensor holding the step number t >= 1."""
    n = param.numel()
    _need_cuda(param, grad, m, v, step, param_bf16)
    cfg = CAdamWConfig(lr, betas[0], betas[1], eps, weight_decay)
    _check("qln_adamw_step", lib().qln_adamw_step(_p(param), _p(grad), _p(m), _p(v), _p(param_bf16), n,
                                                  ctypes.byref(cfg), _p(step), flags, _stream()))
