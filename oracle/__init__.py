"""CPU oracle of the QLoRA frozen-base linear layer.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product path (the CUDA library
and its Python binding) never imports it, and it imports nothing from them.

Two parts:

* ``nf4_oracle.c`` (plain C, built here with gcc) states the encoding:
  codebook, blockwise absmax, nearest-level codes, nibble packing, double
  quantisation of the scales and the bit-exact dequantisation.
* This module states the layer arithmetic in fp64 with numpy matrix products
  (a library primitive used as a step, nothing fused or reordered):

  forward   T = s * X A^T,   Y = X W_hat^T + T B^T
  backward  U = dY B,  dX = dY W_hat + s U A,  dA = s U^T X,
            dB = s dY^T (X A^T)

  with ``W_hat`` the bfloat16 dequantised weight ([d_out, d_in]), ``A``
  [r, d_in], ``B`` [d_out, r], ``X`` [M, d_in], ``dY`` [M, d_out], and
  ``s = alpha / r``.

Sources: "第 04 篇：QLoRA 原理" (jupiter-lab.pages.dev) §2.2 (LoRA branch),
§2.4 (gradient path: the frozen base passes the input gradient and forms no
weight gradient), §6.1-§6.3 (dequantise on demand, BF16 compute, add the
branches); the compassingai.com QLoRA concept page (compute graph; LoRA
shapes B in R^{d x r}, A in R^{r x k}); the LoRA formula Y = dequant(W)X +
(BA)X of the QLoRA tutorial page (124.221.106.7, "QLoRA在资源受限…", §1.1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

NF4_BLOCK = 64
DQ_BLOCK = 256


def build(force: bool = False) -> str:
    """Compile the C part with gcc (no GPU involved)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=gnu99", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        lib.oracle_norm_ppf.restype = ctypes.c_double
        lib.oracle_norm_ppf.argtypes = [ctypes.c_double]
        lib.oracle_nf4_levels.argtypes = [P]
        lib.oracle_nf4_build_codebook.argtypes = [P]
        lib.oracle_nf4_midpoints.argtypes = [P]
        lib.oracle_nf4_absmax.argtypes = [P, I64, P]
        lib.oracle_nf4_encode.argtypes = [P, I64, P, P]
        lib.oracle_nf4_pack.argtypes = [P, I64, P]
        lib.oracle_nf4_unpack.argtypes = [P, I64, P]
        lib.oracle_dq_mean.restype = F
        lib.oracle_dq_mean.argtypes = [P, I64]
        lib.oracle_dq_quantize.argtypes = [P, I64, F, P, P]
        lib.oracle_dq_scales.argtypes = [P, P, F, I64, P]
        lib.oracle_bf16_bits.restype = ctypes.c_uint16
        lib.oracle_bf16_bits.argtypes = [F]
        lib.oracle_nf4_dequantize.argtypes = [P, P, P, F, I64, P]
        lib.oracle_num_blocks.restype = I64
        lib.oracle_num_blocks.argtypes = [I64]
        lib.oracle_num_groups.restype = I64
        lib.oracle_num_groups.argtypes = [I64]
        lib.oracle_packed_bytes.restype = I64
        lib.oracle_packed_bytes.argtypes = [I64]
        lib.oracle_nf4_dequantize_scales.argtypes = [P, P, I64, P]
        lib.oracle_packed_bytes_nodq.restype = I64
        lib.oracle_packed_bytes_nodq.argtypes = [I64]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- codebook
def norm_ppf(p: float) -> float:
    return _load().oracle_norm_ppf(float(p))


def levels() -> np.ndarray:
    out = np.zeros(16, np.float32)
    _load().oracle_nf4_levels(_p(out))
    return out


def build_codebook() -> np.ndarray:
    out = np.zeros(16, np.float64)
    _load().oracle_nf4_build_codebook(_p(out))
    return out


def midpoints() -> np.ndarray:
    out = np.zeros(15, np.float32)
    _load().oracle_nf4_midpoints(_p(out))
    return out


# ---------------------------------------------------------------- encoding
def num_blocks(n: int) -> int:
    return int(_load().oracle_num_blocks(n))


def num_groups(n: int) -> int:
    return int(_load().oracle_num_groups(n))


def packed_bytes(n: int) -> int:
    return int(_load().oracle_packed_bytes(n))


def packed_bytes_nodq(n: int) -> int:
    """Storage of the encoding without double quantisation (codes and one
    fp32 scale per block)."""
    return int(_load().oracle_packed_bytes_nodq(n))


def absmax(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, np.float32).reshape(-1)
    out = np.zeros(num_blocks(w.size), np.float32)
    _load().oracle_nf4_absmax(_p(w), w.size, _p(out))
    return out


def encode(w: np.ndarray, amax: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, np.float32).reshape(-1)
    codes = np.zeros(w.size, np.uint8)
    _load().oracle_nf4_encode(_p(w), w.size, _p(np.ascontiguousarray(amax, np.float32)), _p(codes))
    return codes


def pack(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8).reshape(-1)
    out = np.zeros((codes.size + 1) // 2, np.uint8)
    _load().oracle_nf4_pack(_p(codes), codes.size, _p(out))
    return out


def unpack(packed: np.ndarray, n: int) -> np.ndarray:
    out = np.zeros(n, np.uint8)
    _load().oracle_nf4_unpack(_p(np.ascontiguousarray(packed, np.uint8)), n, _p(out))
    return out


def dq_mean(amax: np.ndarray) -> np.float32:
    amax = np.ascontiguousarray(amax, np.float32)
    return np.float32(_load().oracle_dq_mean(_p(amax), amax.size))


def dq_quantize(amax: np.ndarray, mu: float):
    amax = np.ascontiguousarray(amax, np.float32)
    nb = amax.size
    q = np.zeros(nb, np.int8)
    a2 = np.zeros((nb + DQ_BLOCK - 1) // DQ_BLOCK, np.float32)
    _load().oracle_dq_quantize(_p(amax), nb, ctypes.c_float(mu), _p(q), _p(a2))
    return q, a2


def dq_scales(q: np.ndarray, a2: np.ndarray, mu: float) -> np.ndarray:
    q = np.ascontiguousarray(q, np.int8)
    out = np.zeros(q.size, np.float32)
    _load().oracle_dq_scales(_p(q), _p(np.ascontiguousarray(a2, np.float32)),
                             ctypes.c_float(mu), q.size, _p(out))
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    lib = _load()
    x = np.asarray(x, np.float32).reshape(-1)
    return np.array([lib.oracle_bf16_bits(ctypes.c_float(v)) for v in x], np.uint16)


def quantize(w: np.ndarray) -> Dict[str, np.ndarray]:
    """Encode one fp32 tensor (row-major flattened).  Returns the packed
    codes, int8 scale codes ``q``, fp32 group scales ``a2``, fp32 mean ``mu``
    and, for inspection, the first-level scales ``absmax`` and raw codes."""
    w = np.ascontiguousarray(w, np.float32)
    amax = absmax(w)
    codes = encode(w, amax)
    mu = dq_mean(amax)
    q, a2 = dq_quantize(amax, mu)
    return {"packed": pack(codes), "q": q, "a2": a2, "mu": np.float32(mu),
            "absmax": amax, "codes": codes}


def dequantize_bits(packed: np.ndarray, q: np.ndarray, a2: np.ndarray, mu: float,
                    n: int) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of the dequantised weight, length n."""
    out = np.zeros(n, np.uint16)
    _load().oracle_nf4_dequantize(_p(np.ascontiguousarray(packed, np.uint8)),
                                  _p(np.ascontiguousarray(q, np.int8)),
                                  _p(np.ascontiguousarray(a2, np.float32)),
                                  ctypes.c_float(mu), n, _p(out))
    return out


def quantize_nodq(w: np.ndarray) -> Dict[str, np.ndarray]:
    """The encoding without double quantisation ("第 04 篇" §5.1: one fp32
    scale per block of 64): packed codes and the fp32 absmax of each block,
    stored as is."""
    w = np.ascontiguousarray(w, np.float32)
    amax = absmax(w)
    codes = encode(w, amax)
    return {"packed": pack(codes), "absmax": amax, "codes": codes}


def dequantize_scales_bits(packed: np.ndarray, scales: np.ndarray, n: int) -> np.ndarray:
    """bfloat16 bit patterns of bf16(level[code] * s_b) with the fp32 block
    scales given, length n."""
    out = np.zeros(n, np.uint16)
    _load().oracle_nf4_dequantize_scales(_p(np.ascontiguousarray(packed, np.uint8)),
                                         _p(np.ascontiguousarray(scales, np.float32)), n, _p(out))
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def dequantize(qt: Dict[str, np.ndarray], shape) -> np.ndarray:
    """Dequantised weight as fp32 (every value exactly a bfloat16), from
    either encoding (``quantize`` or ``quantize_nodq``)."""
    n = int(np.prod(shape))
    if "q" not in qt:
        return bf16_bits_to_f32(dequantize_scales_bits(qt["packed"], qt["absmax"], n)).reshape(shape)
    bits = dequantize_bits(qt["packed"], qt["q"], qt["a2"], float(qt["mu"]), n)
    return bf16_bits_to_f32(bits).reshape(shape)


# ---------------------------------------------------------------- layer
def _f64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().float().numpy()
    return np.asarray(t, np.float64)


def forward(W_hat, A, B, X, scaling: float):
    """Y = X W_hat^T + s (X A^T) B^T in fp64; also returns T = s X A^T."""
    W_hat, A, B, X = map(_f64, (W_hat, A, B, X))
    T = scaling * (X @ A.T)
    Y = X @ W_hat.T + T @ B.T
    return Y, T


def backward(W_hat, A, B, X, dY, scaling: float):
    """Gradients of <dY, Y> for the forward above, in fp64.

    dX = dY W_hat + s (dY B) A     (the input gradient passes the frozen base)
    dA = s (dY B)^T X
    dB = s dY^T (X A^T)
    No weight gradient of the base is formed."""
    W_hat, A, B, X, dY = map(_f64, (W_hat, A, B, X, dY))
    U = dY @ B
    dX = dY @ W_hat + scaling * (U @ A)
    dA = scaling * (U.T @ X)
    dB = scaling * (dY.T @ (X @ A.T))
    return dX, dA, dB


def input_grad_rows(W_hat, A, B, dY_rows, scaling: float):
    """dX for a subset of token rows (rows of dX depend only on their dY row)."""
    W_hat, A, B, dY_rows = map(_f64, (W_hat, A, B, dY_rows))
    return dY_rows @ W_hat + scaling * ((dY_rows @ B) @ A)


def output_rows(W_hat, A, B, X_rows, scaling: float):
    """Y for a subset of token rows."""
    return forward(W_hat, A, B, X_rows, scaling)[0]


def lora_grads(A, B, X, dY, scaling: float):
    """dA and dB alone (no pass over the base weight)."""
    A, B, X, dY = map(_f64, (A, B, X, dY))
    U = dY @ B
    dA = scaling * (U.T @ X)
    dB = scaling * (dY.T @ (X @ A.T))
    return dA, dB


def trainable_parameters(d_in: int, d_out: int, r: int) -> int:
    """Entries of A and B, the only trainable tensors of the layer."""
    return r * d_in + d_out * r


# ---------------------------------------------------------------- the adapter's optimizer step
def adamw_step(p, g, m, v, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
               eps: float = 1e-8, weight_decay: float = 0.0):
    """One AdamW update of a trainable tensor (the adapter A or B), in fp64.

    "第 04 篇：QLoRA 原理" §7.3 and §8.3 keep two fp32 moments per trainable
    parameter (first m, second v) and optionally a separate master copy of
    the parameter; the pages print no update rule, so this is the decoupled
    weight-decay AdamW of Loshchilov and Hutter with bias-corrected moments
    (t = step, counted from 1):

        p <- p (1 - lr wd)
        m <- b1 m + (1 - b1) g
        v <- b2 v + (1 - b2) g^2
        p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)

    Returns the new (p, m, v) as fp64 arrays."""
    p, g, m, v = map(_f64, (p, g, m, v))
    if step < 1:
        raise ValueError("step counts from 1")
    p = p * (1.0 - lr * weight_decay)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    p = p - (lr / bc1) * m / (np.sqrt(v) / np.sqrt(bc2) + eps)
    return p, m, v


# ---------------------------------------------------------------- adapter merge
def merge_lora(W_hat, A, B, scaling: float) -> np.ndarray:
    """The merged weight fp32(W_hat + s B A) ("第 04 篇：QLoRA 原理" §12.3: merge
    the adapter into the base, W + s B A, for deployment; §12.4: the effective
    weight of QLoRA is the dequantised base plus the adapter).

    W_hat is the bf16 dequantised base ([d_out, d_in]; the fp32 original is
    not kept), A [r, d_in], B [d_out, r] bf16.  Each product B[n, j] A[j, k]
    of two bf16 values is exact in fp64; the rank-r sum is taken in fp64 in
    ascending j, then multiplied by s (fp32) and added to W_hat, each in fp64
    and rounded once, and the result is rounded to fp32 (to nearest even)."""
    W_hat, A, B = map(_f64, (W_hat, A, B))
    acc = np.zeros(W_hat.shape, np.float64)
    for j in range(A.shape[0]):
        acc = acc + B[:, j:j + 1] * A[j:j + 1, :]
    s = np.float64(np.float32(scaling))
    return (W_hat + s * acc).astype(np.float32)


def merge_requantize(qt: Dict[str, np.ndarray], shape, A, B, scaling: float) -> Dict[str, np.ndarray]:
    """§12.3's deployment path: the merged weight encoded again with the same
    NF4 + double quantisation (a second rounding of the weight)."""
    return quantize(merge_lora(dequantize(qt, shape), A, B, scaling))
