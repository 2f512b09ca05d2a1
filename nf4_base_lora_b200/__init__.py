"""Python binding of libnf4lora (the NF4-LoRA linear layer for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``lib/libnf4lora.so`` behind the C ABI declared in
``include/nf4lora.h``.  PyTorch provides device memory and the current CUDA
stream.  Importing fails loudly if the shared library has not been built
(``python -m nf4_base_lora_b200.build``); there is no fallback.

Layer (QLoRA frozen-base linear, "第 04 篇：QLoRA 原理" §2.2-§2.4, §6.1-§6.4):

    Y  = X W_hat^T + s (X A^T) B^T
    dX = dY W_hat + s (dY B) A,   dA = s (dY B)^T X,   dB = s dY^T (X A^T)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# NF4LORA_DEBUG=1 loads the bounds-checking build (python nf4_base_lora_b200/build.py --debug)
LIB_PATH = os.path.join(_HERE, "lib", "libnf4lora_debug.so" if os.environ.get("NF4LORA_DEBUG") == "1"
                        else "libnf4lora.so")

NF4_OK = 0
STATUS_NAMES = {0: "NF4_OK", -1: "NF4_ERR_INVALID_ARG", -2: "NF4_ERR_UNSUPPORTED_SHAPE",
                -3: "NF4_ERR_MISALIGNED", -4: "NF4_ERR_WORKSPACE", -5: "NF4_ERR_CUDA",
                -6: "NF4_ERR_TIMEOUT", -7: "NF4_ERR_DEVICE"}

# Every symbol the C ABI exports (include/nf4lora.h), in declaration order.
ABI_SYMBOLS = ("nf4_packed_bytes", "nf4_tensor_from_buffer", "nf4_packed_bytes_nodq",
               "nf4_tensor_from_buffer_nodq", "nf4_quantize_workspace_bytes",
               "qlora_fwd_workspace_bytes", "qlora_bwd_workspace_bytes", "nf4_quantize",
               "nf4_quantize_noalloc", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd",
               "nf4_merge_workspace_bytes", "nf4_merge_lora", "nf4_merge_requantize",
               "lora_adamw_step", "nf4lora_last_error_string", "nf4lora_device_status", "nf4lora_check_bounded_wait",
               "nf4lora_debug_site", "nf4lora_debug_build", "nf4lora_trace_start",
               "nf4lora_trace_stop", "nf4lora_trace_count", "nf4lora_trace_get", "nf4lora_version")


class Nf4TensorStruct(ctypes.Structure):
    _fields_ = [("d_out", ctypes.c_int64), ("d_in", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("qscale", ctypes.c_void_p),
                ("scale2", ctypes.c_void_p), ("scale_mean", ctypes.c_void_p),
                ("absmax", ctypes.c_void_p)]


class AdamwTensorStruct(ctypes.Structure):
    _fields_ = [("master", ctypes.c_void_p), ("param", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("m", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n", ctypes.c_int64)]


class AdamwHparamsStruct(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


class Nf4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s (%d): %s" % (STATUS_NAMES.get(status, "?"), status, message))
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("%s is not built; run python nf4_base_lora_b200/build.py%s"
                          % (LIB_PATH, " --debug" if "debug" in os.path.basename(LIB_PATH) else ""))
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, SZ, I, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int,
                        ctypes.c_float)
    S = ctypes.POINTER(Nf4TensorStruct)
    sig = {
        "nf4_packed_bytes": (SZ, [I64, I64]),
        "nf4_tensor_from_buffer": (I, [S, P, SZ, I64, I64]),
        "nf4_packed_bytes_nodq": (SZ, [I64, I64]),
        "nf4_tensor_from_buffer_nodq": (I, [S, P, SZ, I64, I64]),
        "nf4_quantize_workspace_bytes": (SZ, [I64, I64]),
        "qlora_fwd_workspace_bytes": (SZ, [I64, I64, I64, I]),
        "qlora_bwd_workspace_bytes": (SZ, [I64, I64, I64, I]),
        "nf4_quantize": (I, [P, I64, I64, S, P, SZ, P]),
        "nf4_quantize_noalloc": (I, [P, I64, I64, S, P]),
        "nf4_dequantize": (I, [S, P, P]),
        "qlora_linear_fwd": (I, [S, P, P, I, F, P, I64, P, P, P, SZ, P]),
        "qlora_linear_bwd": (I, [S, P, P, I, F, P, P, P, I64, P, P, P, I, P, SZ, P]),
        "nf4_merge_workspace_bytes": (SZ, [I64, I64]),
        "nf4_merge_lora": (I, [S, P, P, I, F, P, P]),
        "nf4_merge_requantize": (I, [S, P, P, I, F, S, P, SZ, P]),
        "lora_adamw_step": (I, [ctypes.POINTER(AdamwTensorStruct), I, ctypes.POINTER(AdamwHparamsStruct), P]),
        "nf4lora_last_error_string": (ctypes.c_char_p, []),
        "nf4lora_device_status": (I, [P]),
        "nf4lora_check_bounded_wait": (I, [I64, P]),
        "nf4lora_debug_site": (I, [P, ctypes.POINTER(ctypes.c_uint)]),
        "nf4lora_debug_build": (I, []),
        "nf4lora_trace_start": (I, [I]),
        "nf4lora_trace_stop": (I, []),
        "nf4lora_trace_count": (I, []),
        "nf4lora_trace_get": (I, [I, ctypes.c_char_p, SZ, ctypes.POINTER(ctypes.c_float)]),
        "nf4lora_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int) -> None:
    if status != NF4_OK:
        raise Nf4Error(status, lib.nf4lora_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous bfloat16 CUDA tensor" % name)
    return t


def _workspace(nbytes: int, device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- sizing
def nf4_packed_bytes(d_out: int, d_in: int) -> int:
    return int(lib.nf4_packed_bytes(d_out, d_in))


def nf4_packed_bytes_nodq(d_out: int, d_in: int) -> int:
    return int(lib.nf4_packed_bytes_nodq(d_out, d_in))


def nf4_quantize_workspace_bytes(d_out: int, d_in: int) -> int:
    return int(lib.nf4_quantize_workspace_bytes(d_out, d_in))


def qlora_fwd_workspace_bytes(M: int, d_out: int, d_in: int, r: int) -> int:
    return int(lib.qlora_fwd_workspace_bytes(M, d_out, d_in, r))


def qlora_bwd_workspace_bytes(M: int, d_out: int, d_in: int, r: int) -> int:
    return int(lib.qlora_bwd_workspace_bytes(M, d_out, d_in, r))


class NF4Tensor:
    """An encoded weight: one device buffer holding the packed codes and the
    block scales: with double_quant (the default) the int8 scale codes, the
    fp32 group scales and the fp32 mean; without it one fp32 scale per block
    of 64 weights."""

    def __init__(self, d_out: int, d_in: int, device="cuda", buffer: Optional[torch.Tensor] = None,
                 double_quant: bool = True):
        nbytes = nf4_packed_bytes(d_out, d_in) if double_quant else nf4_packed_bytes_nodq(d_out, d_in)
        if nbytes == 0:
            raise Nf4Error(-2, "unsupported weight shape [%d, %d]" % (d_out, d_in))
        self.buffer = buffer if buffer is not None else torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.struct = Nf4TensorStruct()
        fill = lib.nf4_tensor_from_buffer if double_quant else lib.nf4_tensor_from_buffer_nodq
        _check(fill(ctypes.byref(self.struct), _ptr(self.buffer), self.buffer.numel(), d_out, d_in))
        self.d_out, self.d_in = d_out, d_in
        self.double_quant = double_quant

    def _view(self, attr: str, dtype, count: int) -> torch.Tensor:
        off = getattr(self.struct, attr) - self.buffer.data_ptr()
        itemsize = torch.empty((), dtype=dtype).element_size()
        return self.buffer[off:off + count * itemsize].view(dtype)

    @property
    def codes(self) -> torch.Tensor:
        return self._view("codes", torch.uint8, self.d_out * self.d_in // 2)

    @property
    def qscale(self) -> torch.Tensor:
        return self._view("qscale", torch.int8, self.d_out * self.d_in // 64)

    @property
    def scale2(self) -> torch.Tensor:
        nb = self.d_out * self.d_in // 64
        return self._view("scale2", torch.float32, (nb + 255) // 256)

    @property
    def scale_mean(self) -> torch.Tensor:
        return self._view("scale_mean", torch.float32, 1)

    @property
    def absmax(self) -> torch.Tensor:
        """fp32 block scales (only without double quantisation)."""
        if self.double_quant:
            raise AttributeError("a double-quantised tensor stores no fp32 block scales")
        return self._view("absmax", torch.float32, self.d_out * self.d_in // 64)


# ---------------------------------------------------------------- entry points
def nf4_quantize(W: torch.Tensor, out: Optional[NF4Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, double_quant: bool = True) -> NF4Tensor:
    """Encode fp32 W [d_out, d_in] (CUDA) to NF4 codes with double-quantised
    scales, or with fp32 block scales when double_quant is False (the format
    of `out` decides when it is given).  `workspace` (uint8, >=
    nf4_quantize_workspace_bytes; only the double-quantised format uses it)
    is allocated when not given."""
    if W.dtype != torch.float32 or not W.is_cuda or not W.is_contiguous() or W.dim() != 2:
        raise ValueError("W must be a contiguous 2-D float32 CUDA tensor")
    d_out, d_in = W.shape
    out = out if out is not None else NF4Tensor(d_out, d_in, W.device, double_quant=double_quant)
    ws = workspace
    if ws is None and out.double_quant:
        ws = _workspace(nf4_quantize_workspace_bytes(d_out, d_in), W.device)
    _check(lib.nf4_quantize(_ptr(W), d_out, d_in, ctypes.byref(out.struct), _ptr(ws),
                            0 if ws is None else ws.numel(), _stream()))
    return out


def nf4_quantize_noalloc(W: torch.Tensor, out: NF4Tensor) -> NF4Tensor:
    """nf4_quantize for callers that cannot allocate device memory: the
    library's built-in scratch replaces the workspace (at most 268,435,456
    weights; calls that overlap on the GPU share that scratch and race)."""
    if W.dtype != torch.float32 or not W.is_cuda or not W.is_contiguous() or W.dim() != 2:
        raise ValueError("W must be a contiguous 2-D float32 CUDA tensor")
    d_out, d_in = W.shape
    status = lib.nf4_quantize_noalloc(_ptr(W), d_out, d_in, ctypes.byref(out.struct), _stream())
    if status != NF4_OK:
        raise Nf4Error(status, "nf4_quantize_noalloc failed")
    return out


def nf4_dequantize(w: NF4Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Materialise W_hat [d_out, d_in] in bfloat16."""
    out = out if out is not None else torch.empty((w.d_out, w.d_in), dtype=torch.bfloat16,
                                                  device=w.buffer.device)
    _check(lib.nf4_dequantize(ctypes.byref(w.struct), _ptr(out), _stream()))
    return out


def qlora_linear_fwd(w: NF4Tensor, A: torch.Tensor, B: torch.Tensor, scaling: float, X: torch.Tensor,
                     save_t: bool = True, Y: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None,
                     T: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Y = X W_hat^T + s (X A^T) B^T.  Returns (Y, T) with T = s X A^T in
    fp32 (or None when save_t is False), for reuse by the backward; T may be
    given as a contiguous float32 [M, r] output buffer."""
    _bf16(A, "A"), _bf16(B, "B"), _bf16(X, "X")
    r = A.shape[0]
    M = X.shape[0]
    Y = Y if Y is not None else torch.empty((M, w.d_out), dtype=torch.bfloat16, device=X.device)
    if not save_t:
        T = None
    elif T is None:
        T = torch.empty((M, r), dtype=torch.float32, device=X.device)
    elif T.dtype != torch.float32 or not T.is_contiguous() or tuple(T.shape) != (M, r):
        raise ValueError("T must be a contiguous float32 [M, r] tensor")
    need = qlora_fwd_workspace_bytes(M, w.d_out, w.d_in, r)
    ws = workspace if workspace is not None else _workspace(need, X.device)
    _check(lib.qlora_linear_fwd(ctypes.byref(w.struct), _ptr(A), _ptr(B), r, ctypes.c_float(scaling),
                                _ptr(X), M, _ptr(Y), _ptr(T), _ptr(ws), 0 if ws is None else ws.numel(),
                                _stream()))
    return Y, T


def qlora_linear_bwd(w: NF4Tensor, A: torch.Tensor, B: torch.Tensor, scaling: float,
                     X: Optional[torch.Tensor], T: Optional[torch.Tensor], dY: torch.Tensor,
                     need_dx: bool = True, need_da: bool = True, need_db: bool = True,
                     dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                     accumulate: bool = False, dX: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None):
    """Returns (dX, dA, dB); an output not requested is None.  T is the fp32
    [M, r] array the forward saved (or None: recomputed from X).  With
    accumulate=True the gradients are added into the given dA / dB."""
    _bf16(A, "A"), _bf16(B, "B"), _bf16(dY, "dY")
    if T is not None and (T.dtype != torch.float32 or not T.is_contiguous()):
        raise ValueError("T must be the contiguous float32 array saved by the forward")
    r = A.shape[0]
    M = dY.shape[0]
    dev = dY.device
    if need_dx and dX is None:
        dX = torch.empty((M, w.d_in), dtype=torch.bfloat16, device=dev)
    if need_da and dA is None:
        dA = torch.zeros((r, w.d_in), dtype=torch.bfloat16, device=dev)
    if need_db and dB is None:
        dB = torch.zeros((w.d_out, r), dtype=torch.bfloat16, device=dev)
    dX = dX if need_dx else None
    dA = dA if need_da else None
    dB = dB if need_db else None
    need = qlora_bwd_workspace_bytes(M, w.d_out, w.d_in, r)
    ws = workspace if workspace is not None else _workspace(need, dev)
    _check(lib.qlora_linear_bwd(ctypes.byref(w.struct), _ptr(A), _ptr(B), r, ctypes.c_float(scaling),
                                _ptr(X), _ptr(T), _ptr(dY), M, _ptr(dX), _ptr(dA), _ptr(dB),
                                1 if accumulate else 0, _ptr(ws), 0 if ws is None else ws.numel(),
                                _stream()))
    return dX, dA, dB


def nf4_merge_workspace_bytes(d_out: int, d_in: int) -> int:
    return int(lib.nf4_merge_workspace_bytes(d_out, d_in))


def _adapter(w: NF4Tensor, A: torch.Tensor, B: torch.Tensor) -> int:
    _bf16(A, "A")
    _bf16(B, "B")
    r = A.shape[0]
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != w.d_in or tuple(B.shape) != (w.d_out, r):
        raise ValueError("A must be [r, d_in] and B [d_out, r]")
    return r


def nf4_merge_lora(w: NF4Tensor, A: torch.Tensor, B: torch.Tensor, scaling: float,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """fp32 W_hat + s B A [d_out, d_in] (the adapter folded into the base)."""
    r = _adapter(w, A, B)
    out = out if out is not None else torch.empty((w.d_out, w.d_in), dtype=torch.float32, device=A.device)
    _check(lib.nf4_merge_lora(ctypes.byref(w.struct), _ptr(A), _ptr(B), r, scaling, _ptr(out), _stream()))
    return out


def nf4_merge_requantize(w: NF4Tensor, A: torch.Tensor, B: torch.Tensor, scaling: float,
                         out: Optional[NF4Tensor] = None, workspace: Optional[torch.Tensor] = None) -> NF4Tensor:
    """The merged weight encoded again, in the format of `out` (when not
    given, that of `w`); `out` may be `w`."""
    r = _adapter(w, A, B)
    out = out if out is not None else NF4Tensor(w.d_out, w.d_in, A.device, double_quant=w.double_quant)
    ws = workspace if workspace is not None else _workspace(nf4_merge_workspace_bytes(w.d_out, w.d_in), A.device)
    _check(lib.nf4_merge_requantize(ctypes.byref(w.struct), _ptr(A), _ptr(B), r, scaling, ctypes.byref(out.struct),
                                    _ptr(ws), 0 if ws is None else ws.numel(), _stream()))
    return out


def lora_adamw_step(tensors, lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                    weight_decay: float = 0.0, step: int = 1) -> None:
    """One AdamW update, in place, of adapter tensors given as tuples
    (master fp32, param bf16 or None, grad bf16, m fp32, v fp32), all
    contiguous CUDA tensors of one size per tuple."""
    arr = (AdamwTensorStruct * max(1, len(tensors)))()
    for i, (master, param, grad, m, v) in enumerate(tensors):
        n = master.numel()
        for t, dt, name in ((master, torch.float32, "master"), (grad, torch.bfloat16, "grad"),
                            (m, torch.float32, "m"), (v, torch.float32, "v"), (param, torch.bfloat16, "param")):
            if t is None and name == "param":
                continue
            if t.dtype != dt or not t.is_cuda or not t.is_contiguous() or t.numel() != n:
                raise ValueError("tensor %d: %s must be a contiguous %s CUDA tensor of %d elements"
                                 % (i, name, dt, n))
        arr[i] = AdamwTensorStruct(master.data_ptr(), None if param is None else param.data_ptr(),
                                   grad.data_ptr(), m.data_ptr(), v.data_ptr(), n)
    h = AdamwHparamsStruct(lr, beta1, beta2, eps, weight_decay, step)
    _check(lib.lora_adamw_step(arr, len(tensors), ctypes.byref(h), _stream()))


def device_status() -> None:
    """Raise Nf4Error(NF4_ERR_TIMEOUT) if a kernel abandoned a bounded wait."""
    _check(lib.nf4lora_device_status(_stream()))


def check_bounded_wait(limit_ns: int = 1000000) -> None:
    """Enqueue the library's self-check of its bounded waits: a kernel whose
    wait on a barrier nothing arrives on gives up after limit_ns.  The next
    device_status() then raises Nf4Error(NF4_ERR_TIMEOUT)."""
    _check(lib.nf4lora_check_bounded_wait(int(limit_ns), _stream()))


def debug_site() -> int:
    """The first failed access check of a debug build, as (site << 16) | line,
    since the last call (0: none; always 0 in a release build)."""
    v = ctypes.c_uint(0)
    _check(lib.nf4lora_debug_site(_stream(), ctypes.byref(v)))
    return int(v.value)


def trace_start(max_launches: int = 4096) -> None:
    """Time every kernel the library launches from now on (see trace_records)."""
    _check(lib.nf4lora_trace_start(max_launches))


def trace_stop() -> None:
    _check(lib.nf4lora_trace_stop())


def trace_count() -> int:
    return int(lib.nf4lora_trace_count())


def trace_records(limit: Optional[int] = None):
    """[(kernel name, device ms), ...] of the recorded launches."""
    out = []
    n = trace_count() if limit is None else limit
    for i in range(n):
        name = ctypes.create_string_buffer(64)
        ms = ctypes.c_float(0.0)
        if lib.nf4lora_trace_get(i, name, 64, ctypes.byref(ms)) != NF4_OK:
            break
        out.append((name.value.decode(), float(ms.value)))
    return out


def version() -> str:
    return lib.nf4lora_version().decode()
