"""B200-native N:M semi-structured sparse weight x dense activation GEMM.

A thin ctypes binding over ``libnmspmm.so`` (C ABI in ``include/nmspmm.h``).
Every step of the path runs in the library's sm_100a kernels; this module only
marshals torch tensors (device memory and streams) into the C calls, with the
same names.  There is no fallback: if the library is missing or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnmspmm.so")

NM_OK, NM_ERR_INVALID, NM_ERR_UNSUPPORTED, NM_ERR_CUDA, NM_ERR_OOM, NM_ERR_TIMEOUT = range(6)
STATUS_NAMES = {0: "NM_OK", 1: "NM_ERR_INVALID", 2: "NM_ERR_UNSUPPORTED", 3: "NM_ERR_CUDA",
                4: "NM_ERR_OOM", 5: "NM_ERR_TIMEOUT"}
NM_INT8, NM_FP16, NM_BF16 = 0, 1, 2
_TORCH_DT = {torch.int8: NM_INT8, torch.float16: NM_FP16, torch.bfloat16: NM_BF16}
_ELEM = {NM_INT8: torch.int8, NM_FP16: torch.float16, NM_BF16: torch.bfloat16}

# Every symbol include/nmspmm.h declares.
EXPORTS = ("nm_compress", "nm_compress_tile", "nm_recompress", "nm_spmm", "nm_spmm_ex", "nm_spmm_gather",
           "nm_spmm_gather_ex", "nm_spmm_noalloc", "nm_decompress", "nm_export", "nm_export_sizes", "nm_query",
           "nm_plan_query", "nm_plan_for_shape", "nm_device_status", "nm_destroy", "nm_last_error", "nm_version",
           "nm_test_spmm_skip_stage")


class NMPlanInfo(ctypes.Structure):
    """nm_plan_info of include/nmspmm.h."""
    _fields_ = [("pair", ctypes.c_int), ("bn", ctypes.c_int), ("splits", ctypes.c_int),
                ("cluster", ctypes.c_int), ("grid", ctypes.c_int), ("units", ctypes.c_int)]


class NMError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnmspmm.so (built in-tree by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m structured_sparse_gemm_compress_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.nm_compress.argtypes = [vp, i64, i64, i32, i32, i32, vp, ctypes.POINTER(vp)]
        L.nm_compress_tile.argtypes = [vp, i64, i64, i32, i32, i32, vp, ctypes.POINTER(vp)]
        L.nm_spmm_gather.argtypes = [vp, vp, i64, i64, vp, vp, vp]
        L.nm_spmm_gather_ex.argtypes = [vp, vp, i64, i64, vp, ctypes.POINTER(NMEpilogue), vp]
        L.nm_recompress.argtypes = [vp, vp, vp]
        L.nm_spmm.argtypes = [vp, vp, i64, vp, vp, vp]
        L.nm_spmm_noalloc.argtypes = [vp, vp, i64, vp, vp, vp]
        L.nm_spmm_ex.argtypes = [vp, vp, i64, vp, ctypes.POINTER(NMEpilogue), vp]
        L.nm_test_spmm_skip_stage.argtypes = [vp, vp, i64, vp, vp, vp, i32, i64]
        L.nm_decompress.argtypes = [vp, vp, vp]
        L.nm_export.argtypes = [vp, vp, vp]
        L.nm_export_sizes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
        L.nm_query.argtypes = [vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i32),
                               ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.nm_plan_query.argtypes = [vp, i64, i32, ctypes.POINTER(NMPlanInfo)]
        L.nm_plan_for_shape.argtypes = [i32, i64, i64, i32, i32, i64, i32, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                        ctypes.POINTER(NMPlanInfo)]
        L.nm_device_status.argtypes = [vp]
        L.nm_destroy.argtypes = [vp]
        L.nm_destroy.restype = None
        L.nm_last_error.restype = ctypes.c_char_p
        L.nm_version.restype = ctypes.c_char_p
        for name in ("nm_compress", "nm_compress_tile", "nm_recompress", "nm_spmm", "nm_spmm_gather",
                     "nm_spmm_gather_ex", "nm_spmm_noalloc",
                     "nm_test_spmm_skip_stage", "nm_decompress", "nm_export", "nm_export_sizes", "nm_query",
                     "nm_plan_query", "nm_plan_for_shape", "nm_device_status"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != NM_OK:
        raise NMError(status, lib().nm_last_error().decode(errors="replace"))


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


class NMHandle:
    """One compressed weight (owns the library handle and its device memory)."""

    def __init__(self, raw: int, n_out: int, k: int, N: int, M: int, dt: int, tile: bool = False):
        self._raw = ctypes.c_void_p(raw)
        self.n_out, self.k, self.N, self.M, self.dt = n_out, k, N, M, dt
        self.tile = tile  # one pattern per 128-channel tile (nm_compress_tile)

    @property
    def raw(self) -> ctypes.c_void_p:
        if not self._raw:
            raise RuntimeError("handle already destroyed")
        return self._raw

    @property
    def dtype(self) -> torch.dtype:
        return _ELEM[self.dt]

    def destroy(self) -> None:
        if self._raw and _lib is not None:
            _lib.nm_destroy(self._raw)
        self._raw = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def nm_compress(W: torch.Tensor, N: int, M: int, stream=None) -> NMHandle:
    """Prune W [n_out, k] (int8 / fp16 / bf16, on the GPU) to N:M and pack it."""
    if not W.is_cuda:
        raise ValueError("W must be a CUDA tensor")
    if W.dtype not in _TORCH_DT:
        raise ValueError(f"unsupported dtype {W.dtype}")
    W = W.contiguous()
    n_out, k = W.shape
    out = ctypes.c_void_p()
    _check(lib().nm_compress(_ptr(W), n_out, k, _TORCH_DT[W.dtype], N, M, _stream(stream), ctypes.byref(out)))
    return NMHandle(out.value, n_out, k, N, M, _TORCH_DT[W.dtype])


def nm_compress_tile(W: torch.Tensor, N: int, M: int, stream=None) -> NMHandle:
    """Prune W [n_out, k] (int8 / fp16, on the GPU) to N:M with one pattern per
    128-row tile (largest column mass) and pack it for ``nm_spmm_gather``."""
    if not W.is_cuda:
        raise ValueError("W must be a CUDA tensor")
    if W.dtype not in _TORCH_DT:
        raise ValueError(f"unsupported dtype {W.dtype}")
    W = W.contiguous()
    n_out, k = W.shape
    out = ctypes.c_void_p()
    _check(lib().nm_compress_tile(_ptr(W), n_out, k, _TORCH_DT[W.dtype], N, M, _stream(stream), ctypes.byref(out)))
    return NMHandle(out.value, n_out, k, N, M, _TORCH_DT[W.dtype], tile=True)


def nm_recompress(h: NMHandle, W: torch.Tensor, stream=None) -> NMHandle:
    """Re-prune and re-pack a new weight of the same shape/dtype into ``h`` (no allocation)."""
    if not W.is_cuda or W.dtype != h.dtype or tuple(W.shape) != (h.n_out, h.k) or not W.is_contiguous():
        raise ValueError("W must be a contiguous CUDA tensor of the handle's shape and dtype")
    _check(lib().nm_recompress(h.raw, _ptr(W), _stream(stream)))
    return h


def out_dtype(h: NMHandle, scaled: bool) -> torch.dtype:
    if h.dt == NM_INT8:
        return torch.float32 if scaled else torch.int32
    return _ELEM[h.dt]


def nm_spmm(h: NMHandle, X: torch.Tensor, Y: torch.Tensor | None = None, scale: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """Y = X @ Wm^T for the compressed weight of ``h`` (see include/nmspmm.h)."""
    if X.dtype != h.dtype or not X.is_cuda or not X.is_contiguous() or X.dim() != 2 or X.shape[1] != h.k:
        raise ValueError("X must be a contiguous CUDA [T, k] tensor of the handle's dtype")
    T = X.shape[0]
    want = out_dtype(h, scale is not None)
    if Y is None:
        Y = torch.empty((T, h.n_out), dtype=want, device=X.device)
    elif Y.dtype != want or tuple(Y.shape) != (T, h.n_out) or not Y.is_contiguous():
        raise ValueError(f"Y must be a contiguous [{T}, {h.n_out}] {want} tensor")
    if scale is not None and (scale.dtype != torch.float32 or scale.numel() != h.n_out or not scale.is_cuda):
        raise ValueError("scale must be a CUDA float32 tensor of n_out elements")
    _check(lib().nm_spmm(h.raw, _ptr(X), T, _ptr(Y), _ptr(scale), _stream(stream)))
    return Y


def nm_spmm_gather(h: NMHandle, Xt: torch.Tensor, T: int | None = None, Y: torch.Tensor | None = None,
                   scale: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X @ Wm^T for a tile-shared handle, X given feature-major as
    ``Xt`` [k, ldx] (``Xt[kk, t] = X[t, kk]``, rows contiguous, ldx = the row
    stride); T defaults to ``Xt.shape[1]``."""
    if Xt.dtype != h.dtype or not Xt.is_cuda or Xt.dim() != 2 or Xt.shape[0] != h.k or Xt.stride(1) != 1:
        raise ValueError("Xt must be a CUDA [k, T] tensor of the handle's dtype with contiguous rows")
    T = Xt.shape[1] if T is None else int(T)
    want = out_dtype(h, scale is not None)
    if Y is None:
        Y = torch.empty((T, h.n_out), dtype=want, device=Xt.device)
    elif Y.dtype != want or tuple(Y.shape) != (T, h.n_out) or not Y.is_contiguous():
        raise ValueError(f"Y must be a contiguous [{T}, {h.n_out}] {want} tensor")
    if scale is not None and (scale.dtype != torch.float32 or scale.numel() != h.n_out or not scale.is_cuda):
        raise ValueError("scale must be a CUDA float32 tensor of n_out elements")
    ldx = Xt.stride(0) if Xt.shape[0] > 1 else Xt.shape[1]
    _check(lib().nm_spmm_gather(h.raw, _ptr(Xt), ldx, T, _ptr(Y), _ptr(scale), _stream(stream)))
    return Y


class NMEpilogue(ctypes.Structure):
    """``nm_epilogue`` of include/nmspmm.h."""
    _fields_ = [("out", ctypes.c_int), ("act", ctypes.c_int), ("scale", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("out_scale", ctypes.c_float)]


OUT_TYPES = {"default": 0, "int32": 1, "float32": 2, "float16": 3, "bfloat16": 4, "int8": 5}
ACTS = {"none": 0, "gelu": 1}
_OUT_TORCH = {"int32": torch.int32, "float32": torch.float32, "float16": torch.float16,
              "bfloat16": torch.bfloat16, "int8": torch.int8}


def resolve_out(h: NMHandle, out: str, scale, bias, act: str) -> str:
    """The output type ``NM_OUT_DEFAULT`` stands for, by the header's rule."""
    if out != "default":
        return out
    if h.dtype == torch.int8:
        return "int32" if scale is None and bias is None and act == "none" else "float32"
    return "float16" if h.dtype == torch.float16 else "bfloat16"


def nm_spmm_ex(h: NMHandle, X: torch.Tensor, Y: torch.Tensor | None = None, scale: torch.Tensor | None = None,
               bias: torch.Tensor | None = None, act: str = "none", out: str = "default",
               out_scale: float = 1.0, stream=None) -> torch.Tensor:
    """Y = out(act(X @ Wm^T * scale + bias)) with the fused output stage of
    ``nm_spmm_ex`` (include/nmspmm.h).  ``out`` is one of ``OUT_TYPES``, ``act``
    one of ``ACTS``.  Only argument marshalling happens here."""
    if X.dtype != h.dtype or not X.is_cuda or not X.is_contiguous() or X.dim() != 2 or X.shape[1] != h.k:
        raise ValueError("X must be a contiguous CUDA [T, k] tensor of the handle's dtype")
    if out not in OUT_TYPES or act not in ACTS:
        raise ValueError(f"out must be one of {tuple(OUT_TYPES)}, act one of {tuple(ACTS)}")
    for name, v in (("scale", scale), ("bias", bias)):
        if v is not None and (v.dtype != torch.float32 or v.numel() != h.n_out or not v.is_cuda):
            raise ValueError(f"{name} must be a CUDA float32 tensor of n_out elements")
    T = X.shape[0]
    res = resolve_out(h, out, scale, bias, act)
    want = _OUT_TORCH[res]
    if Y is None:
        Y = torch.empty((T, h.n_out), dtype=want, device=X.device)
    elif Y.dtype != want or tuple(Y.shape) != (T, h.n_out) or not Y.is_contiguous():
        raise ValueError(f"Y must be a contiguous [{T}, {h.n_out}] {want} tensor")
    ep = NMEpilogue(OUT_TYPES[out], ACTS[act], _ptr(scale), _ptr(bias), float(out_scale))
    _check(lib().nm_spmm_ex(h.raw, _ptr(X), T, _ptr(Y), ctypes.byref(ep), _stream(stream)))
    return Y


def nm_spmm_gather_ex(h: NMHandle, Xt: torch.Tensor, T: int | None = None, Y: torch.Tensor | None = None,
                      scale: torch.Tensor | None = None, bias: torch.Tensor | None = None, act: str = "none",
                      out: str = "default", out_scale: float = 1.0, stream=None) -> torch.Tensor:
    """``nm_spmm_gather`` (feature-major ``Xt`` [k, ldx], tile-shared handle)
    with the fused output stage of ``nm_spmm_ex``."""
    if Xt.dtype != h.dtype or not Xt.is_cuda or Xt.dim() != 2 or Xt.shape[0] != h.k or Xt.stride(1) != 1:
        raise ValueError("Xt must be a CUDA [k, T] tensor of the handle's dtype with contiguous rows")
    if out not in OUT_TYPES or act not in ACTS:
        raise ValueError(f"out must be one of {tuple(OUT_TYPES)}, act one of {tuple(ACTS)}")
    for name, v in (("scale", scale), ("bias", bias)):
        if v is not None and (v.dtype != torch.float32 or v.numel() != h.n_out or not v.is_cuda):
            raise ValueError(f"{name} must be a CUDA float32 tensor of n_out elements")
    T = Xt.shape[1] if T is None else int(T)
    want = _OUT_TORCH[resolve_out(h, out, scale, bias, act)]
    if Y is None:
        Y = torch.empty((T, h.n_out), dtype=want, device=Xt.device)
    elif Y.dtype != want or tuple(Y.shape) != (T, h.n_out) or not Y.is_contiguous():
        raise ValueError(f"Y must be a contiguous [{T}, {h.n_out}] {want} tensor")
    ep = NMEpilogue(OUT_TYPES[out], ACTS[act], _ptr(scale), _ptr(bias), float(out_scale))
    ldx = Xt.stride(0) if Xt.shape[0] > 1 else Xt.shape[1]
    _check(lib().nm_spmm_gather_ex(h.raw, _ptr(Xt), ldx, T, _ptr(Y), ctypes.byref(ep), _stream(stream)))
    return Y


def nm_spmm_noalloc(h: NMHandle, X: torch.Tensor, Y: torch.Tensor, scale: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """nm_spmm for callers that cannot allocate: split-K scratch lives in a fixed
    array inside the library (limits and ordering rules in include/nmspmm.h)."""
    _check(lib().nm_spmm_noalloc(h.raw, _ptr(X), X.shape[0], _ptr(Y), _ptr(scale), _stream(stream)))
    return Y


def nm_test_spmm_skip_stage(h: NMHandle, X: torch.Tensor, Y: torch.Tensor, scale: torch.Tensor | None,
                            skip_stage: int, timeout_ns: int, stream=None) -> int:
    """Test hook: run the SpMM with one producer stage left unfilled; returns the launch status."""
    return lib().nm_test_spmm_skip_stage(h.raw, _ptr(X), X.shape[0], _ptr(Y), _ptr(scale), _stream(stream),
                                         skip_stage, timeout_ns)


def nm_decompress(h: NMHandle, stream=None) -> torch.Tensor:
    """Masked dense W decoded from the packed operand image the SpMM reads."""
    out = torch.empty((h.n_out, h.k), dtype=h.dtype, device="cuda")
    _check(lib().nm_decompress(h.raw, _ptr(out), _stream(stream)))
    return out


def nm_export_sizes(h: NMHandle) -> tuple[int, int]:
    vb, ib = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().nm_export_sizes(h.raw, ctypes.byref(vb), ctypes.byref(ib)))
    return vb.value, ib.value


def nm_export(h: NMHandle):
    """Canonical format on the host: (values [n_out, k/M, N], idx [n_out, pitch] uint8) as torch CPU tensors."""
    vb, ib = nm_export_sizes(h)
    values = torch.empty((h.n_out, h.k // h.M, h.N), dtype=h.dtype)
    idx = torch.empty((h.n_out, ib // h.n_out), dtype=torch.uint8)
    assert values.numel() * values.element_size() == vb
    _check(lib().nm_export(h.raw, _ptr(values), _ptr(idx)))
    return values, idx


def nm_query(h: NMHandle) -> dict:
    n, k, N, M, dt = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().nm_query(h.raw, ctypes.byref(n), ctypes.byref(k), ctypes.byref(N), ctypes.byref(M),
                          ctypes.byref(dt)))
    return {"n_out": n.value, "k": k.value, "N": N.value, "M": M.value, "dtype": dt.value}


def nm_plan_query(h: NMHandle, T: int, scaled: bool = False) -> dict:
    """The launch plan the SpMM call would use for T tokens (kernel, token tile, splits, cluster, grid)."""
    info = NMPlanInfo()
    _check(lib().nm_plan_query(h.raw, int(T), int(bool(scaled)), ctypes.byref(info)))
    return {f: getattr(info, f) for f, _ in NMPlanInfo._fields_}


def nm_plan_for_shape(dtype: torch.dtype, n_out: int, k: int, N: int, M: int, T: int, sms: int,
                      pair_clusters=(74, 74, 74), stream_clusters=(148, 74, 48, 37, 28, 24, 21, 18)) -> dict:
    """The plan nm_plan_query would report for a handle of this shape on a GPU
    with ``sms`` SMs and the given resident-cluster capacities (two-SM kernel
    pairs at token tiles 224/192/128; clusters of 1..8 one-SM CTAs).  Needs no
    GPU: a test and diagnostic hook of the planner."""
    if dtype not in _TORCH_DT or len(pair_clusters) != 3 or len(stream_clusters) != 8:
        raise ValueError("dtype must be int8/float16/bfloat16, pair_clusters 3 values, stream_clusters 8")
    pc = (ctypes.c_int * 3)(*[int(v) for v in pair_clusters])
    sc = (ctypes.c_int * 8)(*[int(v) for v in stream_clusters])
    info = NMPlanInfo()
    _check(lib().nm_plan_for_shape(_TORCH_DT[dtype], int(n_out), int(k), int(N), int(M), int(T), int(sms), pc, sc,
                                   ctypes.byref(info)))
    return {f: getattr(info, f) for f, _ in NMPlanInfo._fields_}


def nm_device_status(h: NMHandle) -> int:
    """NM_OK, or NM_ERR_TIMEOUT if a kernel gave up a bounded wait (clears the word)."""
    return lib().nm_device_status(h.raw)


def nm_last_error() -> str:
    return lib().nm_last_error().decode(errors="replace")


def nm_version() -> str:
    return lib().nm_version().decode()
