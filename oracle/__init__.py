"""CPU oracle for the N:M sparse weight x dense activation GEMM -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and this
package imports nothing from the product library: the two share no code.

What it computes follows "Realizable N:M Sparse Transformer Inference via
Search-Kernel Co-Design" (arXiv 2607.12505):

* section 2.1 -- N:M sparsity: every group of M weights keeps N non-zeros;
* section 4.2 -- micro-dense execution materialises only those N values per
  window and runs dense MMA on them, so the product equals the dense GEMM over
  the masked weight; the packed format carries values and in-window positions.

The arithmetic lives in ``nm_oracle.c`` (plain C, one OpenMP loop over output
rows, ``-ffp-contract=off``).  This module only builds it, marshals numpy
arrays, and states the readings of the paper that the C code follows:

* groups run along K, contiguous, aligned at k = 0;
* top-N by magnitude, ties to the lower in-group position;
* exactly N slots per group, kept values in ascending position;
* ``idx`` holds one 4-bit position per kept element, two per byte, low nibble
  first, each row padded to whole bytes;
* tile-shared compress (``compress_tile``, the vector-wise reading of the
  micro-dense format): the rows of a tile of consecutive output channels keep
  one pattern, chosen by the same rule with the tile's column mass (sum of |w|)
  as the magnitude, so that one gather of the activations serves the tile.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nm_oracle.c")
_LIB = os.path.join(_HERE, "libnm_oracle.so")
# Test hook: a prebuilt oracle library to load instead (the mutation tests load
# deliberately broken builds of nm_oracle.c through it); never rebuilt here.
_LIB_OVERRIDE = os.environ.get("NM_ORACLE_LIB")

DTYPES = {"int8": 0, "fp16": 1, "bf16": 2}
_lib = None


def build(force: bool = False) -> str:
    """Compile ``nm_oracle.c`` into ``libnm_oracle.so`` next to it."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
             "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, p, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        lib.oracle_compress.argtypes = [p, i64, i64, i32, i32, i32, p, p]
        lib.oracle_compress_tile.argtypes = [p, i64, i64, i32, i32, i32, i64, p, p]
        lib.oracle_decompress.argtypes = [p, p, i64, i64, i32, i32, i32, p]
        lib.oracle_gemm_i8.argtypes = [p, i64, i64, p, i64, p, p, p]
        lib.oracle_gemm_f16.argtypes = [p, i64, i64, p, i64, i32, p, p]
        lib.oracle_idx_pitch.argtypes = [i64, i32, i32]
        lib.oracle_idx_pitch.restype = i64
        lib.oracle_epilogue_i8.argtypes = [p, i64, i64, p, p, i32, ctypes.c_float, p, p, p]
        lib.oracle_epilogue_f.argtypes = [p, i64, i64, p, p, i32, p]
        lib.oracle_gelu.argtypes = [ctypes.c_double]
        lib.oracle_gelu.restype = ctypes.c_double
        lib.oracle_threads.restype = i32
        lib.oracle_set_threads.argtypes = [i32]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _dtype_code(a: np.ndarray, dtype: str | None) -> int:
    if dtype is None:
        if a.dtype == np.int8:
            dtype = "int8"
        elif a.dtype == np.float16:
            dtype = "fp16"
        else:
            raise ValueError("pass dtype='bf16' for raw uint16 bfloat16 bits")
    return DTYPES[dtype]


def threads() -> int:
    return _load().oracle_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def idx_pitch(k: int, N: int, M: int) -> int:
    return int(_load().oracle_idx_pitch(k, N, M))


def compress(W: np.ndarray, N: int, M: int, dtype: str | None = None):
    """Top-N-of-M compression of W [n_out, k] along k.

    ``W`` is int8, float16, or uint16 holding bfloat16 bits (``dtype='bf16'``).
    Returns ``(values [n_out, k//M, N], idx [n_out, idx_pitch] uint8)``.
    """
    W = np.ascontiguousarray(W)
    n_out, k = W.shape
    code = _dtype_code(W, dtype)
    values = np.zeros((n_out, k // M, N), dtype=W.dtype)
    idx = np.zeros((n_out, idx_pitch(k, N, M)), dtype=np.uint8)
    rc = _load().oracle_compress(_ptr(W), n_out, k, code, N, M, _ptr(values), _ptr(idx))
    if rc != 0:
        raise ValueError(f"oracle_compress rejected the arguments (rc={rc})")
    return values, idx


def compress_tile(W: np.ndarray, N: int, M: int, tile: int = 128, dtype: str | None = None):
    """Tile-shared top-N-of-M compression: the rows of each tile of ``tile``
    consecutive rows keep the same positions, those of largest column mass
    (sum of |w| over the tile), ties to the lower position.  int8 or float16
    only.  Same return layout as ``compress``.
    """
    W = np.ascontiguousarray(W)
    n_out, k = W.shape
    code = _dtype_code(W, dtype)
    values = np.zeros((n_out, k // M, N), dtype=W.dtype)
    idx = np.zeros((n_out, idx_pitch(k, N, M)), dtype=np.uint8)
    rc = _load().oracle_compress_tile(_ptr(W), n_out, k, code, N, M, tile, _ptr(values), _ptr(idx))
    if rc != 0:
        raise ValueError(f"oracle_compress_tile rejected the arguments (rc={rc})")
    return values, idx


def decompress(values: np.ndarray, idx: np.ndarray, n_out: int, k: int, N: int, M: int,
               dtype: str | None = None) -> np.ndarray:
    """Scatter the kept values back into a dense masked W [n_out, k]."""
    values = np.ascontiguousarray(values)
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    code = _dtype_code(values, dtype)
    Wm = np.zeros((n_out, k), dtype=values.dtype)
    rc = _load().oracle_decompress(_ptr(values), _ptr(idx), n_out, k, code, N, M, _ptr(Wm))
    if rc != 0:
        raise ValueError(f"oracle_decompress rejected the arguments (rc={rc})")
    return Wm


def gemm(X: np.ndarray, Wm: np.ndarray, scale: np.ndarray | None = None,
         dtype: str | None = None) -> np.ndarray:
    """Y = X @ Wm.T over the masked weight.

    int8 inputs: int32 result, or float32 ``(float)acc * scale[n]`` when
    ``scale`` is given.  fp16/bf16 inputs: float64 result (times ``scale``).
    """
    X = np.ascontiguousarray(X)
    Wm = np.ascontiguousarray(Wm)
    T, K = X.shape
    n_out, K2 = Wm.shape
    if K != K2:
        raise ValueError("K mismatch")
    code = _dtype_code(X, dtype)
    lib = _load()
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float32)
    sp = None if sc is None else _ptr(sc)
    if code == 0:
        if sc is None:
            Y = np.zeros((T, n_out), dtype=np.int32)
            rc = lib.oracle_gemm_i8(_ptr(X), T, K, _ptr(Wm), n_out, None, _ptr(Y), None)
        else:
            Y = np.zeros((T, n_out), dtype=np.float32)
            rc = lib.oracle_gemm_i8(_ptr(X), T, K, _ptr(Wm), n_out, sp, None, _ptr(Y))
    else:
        Y = np.zeros((T, n_out), dtype=np.float64)
        rc = lib.oracle_gemm_f16(_ptr(X), T, K, _ptr(Wm), n_out, code, sp, _ptr(Y))
    if rc != 0:
        raise ValueError(f"oracle gemm failed (rc={rc})")
    return Y


def spmm(X: np.ndarray, W: np.ndarray, N: int, M: int, scale: np.ndarray | None = None,
         dtype: str | None = None) -> np.ndarray:
    """The whole path: compress W, decompress, dense GEMM over the masked W."""
    values, idx = compress(W, N, M, dtype)
    Wm = decompress(values, idx, W.shape[0], W.shape[1], N, M, dtype)
    return gemm(X, Wm, scale, dtype)


ACTS = {"none": 0, "gelu": 1}
OUTS = ("float32", "float16", "bfloat16", "int8")


def gelu(x: float) -> float:
    """The erf form of GELU, x/2 * (1 + erf(x / sqrt 2)), in fp64."""
    return float(_load().oracle_gelu(float(x)))


def epilogue(acc: np.ndarray, scale: np.ndarray | None = None, bias: np.ndarray | None = None,
             act: str = "none", out: str = "float32", out_scale: float = 1.0) -> dict:
    """The fused output stage on a GEMM accumulator [T, n_out].

    ``acc`` int32 (INT8 path) or float64 (FP16/BF16 path, the fp64 sum).
    Returns a dict with
      ``pre``   -- float64 value after scale, bias and activation;
      ``exact`` -- the output tensor the kernel must reproduce bit for bit,
                   or None where several results are correct (GELU: the
                   kernel evaluates erf in fp32; FP16/BF16 inputs: any
                   summation order);
      ``q``     -- for ``out='int8'``: the int8 codes decided from ``pre``
                   (exact when ``exact`` is not None);
      ``q_pre`` -- for ``out='int8'``: the value that was rounded (fp64).
    Rounding to float16 uses numpy's float32 -> float16 conversion and to
    bfloat16 torch's, both round-to-nearest-even, applied to the exact fp32
    result of the INT8 path.
    """
    if act not in ACTS or out not in OUTS:
        raise ValueError("bad act/out")
    acc = np.ascontiguousarray(acc)
    T, n_out = acc.shape
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float32)
    bi = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    lib = _load()
    pre = np.zeros((T, n_out), dtype=np.float64)
    res = {"pre": pre, "exact": None}
    if acc.dtype == np.int32:
        v32 = np.zeros((T, n_out), dtype=np.float32)
        q = np.zeros((T, n_out), dtype=np.int8)
        rc = lib.oracle_epilogue_i8(_ptr(acc), T, n_out, None if sc is None else _ptr(sc),
                                    None if bi is None else _ptr(bi), ACTS[act], float(out_scale),
                                    _ptr(pre), _ptr(v32), _ptr(q))
        if rc != 0:
            raise ValueError(f"oracle_epilogue_i8 failed (rc={rc})")
        if out == "int8":
            res["q"] = q
            res["q_pre"] = pre * np.float64(np.float32(out_scale)) if act == "gelu" else \
                (v32 * np.float32(out_scale)).astype(np.float64)
            if act == "none":
                res["exact"] = q
        elif act == "none":
            if out == "float32":
                res["exact"] = v32
            elif out == "float16":
                with np.errstate(over="ignore"):  # beyond the fp16 range rounds to +-inf, as defined
                    res["exact"] = v32.astype(np.float16)
            else:
                import torch
                res["exact"] = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        return res
    if acc.dtype != np.float64 or out == "int8":
        raise ValueError("float path: float64 accumulator, float output")
    rc = lib.oracle_epilogue_f(_ptr(acc), T, n_out, None if sc is None else _ptr(sc),
                               None if bi is None else _ptr(bi), ACTS[act], _ptr(pre))
    if rc != 0:
        raise ValueError(f"oracle_epilogue_f failed (rc={rc})")
    return res


def spmm_epilogue(X: np.ndarray, W: np.ndarray, N: int, M: int, scale=None, bias=None, act="none",
                  out="float32", out_scale=1.0, dtype: str | None = None) -> dict:
    """The whole path with the fused output stage: compress, decompress, the
    raw GEMM accumulator (int32 or fp64), then ``epilogue``."""
    values, idx = compress(W, N, M, dtype)
    Wm = decompress(values, idx, W.shape[0], W.shape[1], N, M, dtype)
    acc = gemm(X, Wm, None, dtype)
    return epilogue(acc, scale, bias, act, out, out_scale)
