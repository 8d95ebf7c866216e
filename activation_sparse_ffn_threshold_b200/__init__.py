"""Activation-sparse FFN decode on B200: Python binding of the C ABI in include/sfnn.h.

This module only marshals arguments into ``libsfnn.so`` (ctypes): every step of
the computation runs in the library's CUDA kernels.  PyTorch provides device
memory and streams.  If the library is missing the import of the binding
fails loudly; there is no fallback implementation.

    layer = SparseFFN(w_up, w_down, b, A, B, c, act="relu", hotness=p)  # CUDA tensors
    y = layer.forward(x)               # predictor + sparse FFN for one token
    idx, count = layer.predict(x)      # the predicted set only
    Y = layer.forward_batch(X)         # b tokens through the union of their sets
    XL = forward_stack([l0, l1], X0)   # residual stack
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

__all__ = ["SparseFFN", "SfnnError", "forward_stack", "predict_noalloc", "hotness_order", "library_path",
           "load_library",
           "RELU", "REGLU", "F32", "F16", "I8", "I4", "BATCH_AUTO", "BATCH_CUDA_CORE", "BATCH_TENSOR_CORE",
           "BATCH_FUSED"]

RELU, REGLU = 0, 1
F32, F16, I8, I4 = 0, 1, 2, 3
BATCH_AUTO, BATCH_CUDA_CORE, BATCH_TENSOR_CORE, BATCH_FUSED = 0, 1, 2, 3
STATUS = {0: "SFNN_OK", 1: "SFNN_ERR_INVALID_ARG", 2: "SFNN_ERR_CUDA", 3: "SFNN_ERR_OOM",
          4: "SFNN_ERR_UNSUPPORTED", 5: "SFNN_ERR_TIMEOUT"}
STATUS_CODES = {v: k for k, v in STATUS.items()}

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libsfnn.so")
_lib = None


def library_path() -> str:
    return _LIB_PATH


class SfnnError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_str(status)})")
        self.status = status


class LayerDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("n", ctypes.c_int32), ("r", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("act", ctypes.c_int32), ("wdtype", ctypes.c_int32),
                ("w_up", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("b", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p), ("pa", ctypes.c_void_p), ("pb", ctypes.c_void_p),
                ("pc", ctypes.c_void_p), ("hotness", ctypes.POINTER(ctypes.c_float)),
                ("rows_dtype", ctypes.c_int32), ("order", ctypes.c_int32)]


class Info(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("n", ctypes.c_int32), ("r", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("act", ctypes.c_int32), ("wdtype", ctypes.c_int32),
                ("num_sms", ctypes.c_int32), ("batch_path", ctypes.c_int32),
                ("weight_bytes", ctypes.c_int64), ("scratch_bytes", ctypes.c_int64),
                ("predictor_bytes", ctypes.c_int64), ("row_bytes_per_neuron", ctypes.c_int64),
                ("launches", ctypes.c_int64)]


def load_library():
    """Load libsfnn.so and declare its signatures (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          f"`python -m activation_sparse_ffn_threshold_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int
    sig = {
        "sfnn_create": ([ctypes.POINTER(LayerDesc), P, ctypes.POINTER(P)], S),
        "sfnn_destroy": ([P], S),
        "sfnn_predict": ([P, P, P, P, P], S),
        "sfnn_forward": ([P, P, P, P, P, P], S),
        "sfnn_forward_batch": ([P, P, I, P, P, P, P], S),
        "sfnn_forward_stack": ([P, I, P, I, P, P, P, P], S),
        "sfnn_forward_stack_lookahead": ([P, I, P, I, P, P, P, P], S),
        "sfnn_set_batch_path": ([P, I], S),
        "sfnn_set_fused_decode": ([P, I], S),
        "sfnn_set_hot_prefix": ([P, I], S),
        "sfnn_set_fused_quota": ([P, I], S),
        "sfnn_set_batch_quota": ([P, I], S),
        "sfnn_set_batch_depths": ([P, I, I, I, I], S),
        "sfnn_set_batch_tc_shape": ([P, I, I, I], S),
        "sfnn_tune_batch_paths": ([P, P, P], S),
        "sfnn_set_fused_depths": ([P, I, I, I, I], S),
        "sfnn_debug_stall_next_barrier": ([P, P], S),
        "sfnn_set_profile_events": ([P, P, P], S),
        "sfnn_query": ([P, ctypes.POINTER(Info)], S),
        "sfnn_get_error": ([P], S),
        "sfnn_status_str": ([S], ctypes.c_char_p),
        "sfnn_hotness_order": ([ctypes.POINTER(ctypes.c_float), I, ctypes.POINTER(ctypes.c_int32)], S),
        "sfnn_predict_noalloc": ([P, P, P, P, I, I, I, I, P, P, P], S),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _status_str(status: int) -> str:
    try:
        return load_library().sfnn_status_str(int(status)).decode()
    except Exception:  # pragma: no cover - only when the library itself is unusable
        return "?"


def _check(status: int, what: str):
    if status != 0:
        raise SfnnError(what, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float16:
        return F16
    if dt == torch.float32:
        return F32
    raise TypeError(f"weights must be fp16 or fp32, got {dt}")


def _as_dev(t, device, dtype=None):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(t))
    t = t.to(device=device, dtype=dtype) if dtype is not None else t.to(device=device)
    return t.contiguous()


def hotness_order(hotness) -> np.ndarray:
    """The storage order the library uses: hotness descending, ties by index, NaN last."""
    h = np.ascontiguousarray(hotness, dtype=np.float32)
    perm = np.empty(h.size, dtype=np.int32)
    _check(load_library().sfnn_hotness_order(h.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), h.size,
                                             perm.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))),
           "sfnn_hotness_order")
    return perm


class SparseFFN:
    """One activation-sparse FFN layer resident on a CUDA device.

    Weights are given in PyTorch layouts (w_up/w_gate [n, d], w_down [d, n],
    A [d, r], B [r, n], b/c [n]) as CUDA tensors or numpy arrays of one dtype
    (fp16 or fp32); they are copied and re-laid-out by the library and may be
    dropped afterwards.  ``hotness`` [n] is the offline activation frequency.
    """

    def __init__(self, w_up, w_down, b, A, B, c, act: str = "relu", w_gate=None, hotness=None,
                 max_batch: int = 1, device=None, stream=None, rows: str | None = None, order: str = "dealt"):
        """``rows="int8"`` / ``"int4"`` stores the FFN rows as int8 / int4 codes with
        per-row fp32 scales (fp16 layers; single-token fused path only, see
        sfnn_layer_desc.rows_dtype).  ``order`` ("dealt" or "packed") is the storage
        order of the neurons by hotness (sfnn_layer_desc.order)."""
        if rows not in (None, "int8", "int4"):
            raise ValueError("rows must be None, 'int8' or 'int4'")
        if order not in ("dealt", "packed"):
            raise ValueError("order must be 'dealt' or 'packed'")
        lib = load_library()
        device = torch.device(device or "cuda")
        dtype = w_up.dtype if isinstance(w_up, torch.Tensor) else torch.from_numpy(np.asarray(w_up[:1])).dtype
        ts = [_as_dev(t, device, dtype) for t in (w_up, w_gate, b, w_down, A, B, c)]
        w_up_t, w_gate_t, b_t, w_down_t, A_t, B_t, c_t = ts
        n, d = w_up_t.shape
        r = A_t.shape[1]
        if w_down_t.shape != (d, n) or A_t.shape != (d, r) or B_t.shape != (r, n) or b_t.shape != (n,) \
                or c_t.shape != (n,) or (w_gate_t is not None and w_gate_t.shape != (n, d)):
            raise ValueError("inconsistent layer shapes")
        self.act = REGLU if act == "reglu" else RELU
        if self.act == REGLU and w_gate_t is None:
            raise ValueError("ReGLU needs w_gate")
        self.d, self.n, self.r, self.max_batch = int(d), int(n), int(r), int(max_batch)
        self.dtype = dtype
        self.device = device
        self._hot = None
        if hotness is not None:
            self._hot = np.ascontiguousarray(np.asarray(hotness, dtype=np.float32))
        desc = LayerDesc(self.d, self.n, self.r, self.max_batch, self.act, _dtype_code(dtype),
                         w_up_t.data_ptr(), w_gate_t.data_ptr() if w_gate_t is not None else None,
                         b_t.data_ptr(), w_down_t.data_ptr(), A_t.data_ptr(), B_t.data_ptr(), c_t.data_ptr(),
                         self._hot.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if self._hot is not None
                         else None, {"int8": I8, "int4": I4}.get(rows, 0), 0 if order == "dealt" else 1)
        self.rows = rows
        self._h = ctypes.c_void_p()
        with torch.cuda.device(device):
            _check(lib.sfnn_create(ctypes.byref(desc), _stream(stream), ctypes.byref(self._h)), "sfnn_create")
        self._lib = lib

    @classmethod
    def from_layer(cls, layer, max_batch: int = 1, use_hotness: bool = True, device=None, stream=None,
                   rows: str | None = None, order: str = "dealt"):
        """Build from a record with w_up, w_gate, b, w_down, A, B, c, p and cfg.act (numpy arrays)."""
        return cls(layer.w_up, layer.w_down, layer.b, layer.A, layer.B, layer.c, act=layer.cfg.act,
                   w_gate=layer.w_gate, hotness=layer.p if use_hotness else None, max_batch=max_batch,
                   device=device, stream=stream, rows=rows, order=order)

    # ------------------------------------------------------------------ helpers
    def _check_x(self, x, rows=None):
        if not isinstance(x, torch.Tensor) or x.device.type != "cuda" or x.dtype != self.dtype \
                or not x.is_contiguous():
            raise TypeError(f"x must be a contiguous CUDA tensor of {self.dtype}")
        if rows is None and x.numel() != self.d:
            raise ValueError(f"x must have {self.d} elements")
        if rows is not None and x.numel() != rows * self.d:
            raise ValueError(f"X must have {rows}x{self.d} elements")

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    # ------------------------------------------------------------------ API
    def predict(self, x, idx=None, count=None, stream=None):
        """The predicted set of one token: (idx [n] int32, count [1] int32); idx[:count] is the set."""
        self._check_x(x)
        idx = idx if idx is not None else torch.empty(self.n, dtype=torch.int32, device=x.device)
        count = count if count is not None else torch.empty(1, dtype=torch.int32, device=x.device)
        _check(self._lib.sfnn_predict(self._h, _ptr(x), _ptr(idx), _ptr(count), _stream(stream)), "sfnn_predict")
        return idx, count

    def forward(self, x, y=None, idx=None, count=None, stream=None):
        """y [d] fp32 for one token; ``idx``/``count`` (device int32) replace the predicted set."""
        self._check_x(x)
        y = y if y is not None else torch.empty(self.d, dtype=torch.float32, device=x.device)
        if idx is not None and count is None:
            count = torch.tensor([idx.numel()], dtype=torch.int32, device=x.device)
        _check(self._lib.sfnn_forward(self._h, _ptr(x), _ptr(idx), _ptr(count), _ptr(y), _stream(stream)),
               "sfnn_forward")
        return y

    def forward_batch(self, X, Y=None, idx=None, counts=None, return_sets: bool = False, stream=None):
        """Y [b, d] fp32 for b tokens; with return_sets also (idx [b, n], counts [b])."""
        b = X.shape[0]
        self._check_x(X, rows=b)
        Y = Y if Y is not None else torch.empty((b, self.d), dtype=torch.float32, device=X.device)
        if return_sets:
            idx = idx if idx is not None else torch.empty((b, self.n), dtype=torch.int32, device=X.device)
            counts = counts if counts is not None else torch.empty(b, dtype=torch.int32, device=X.device)
        _check(self._lib.sfnn_forward_batch(self._h, _ptr(X), b, _ptr(Y), _ptr(idx), _ptr(counts),
                                            _stream(stream)), "sfnn_forward_batch")
        return (Y, idx, counts) if return_sets else Y

    def set_batch_path(self, path: int):
        _check(self._lib.sfnn_set_batch_path(self._h, int(path)), "sfnn_set_batch_path")

    def set_fused_decode(self, enable: bool):
        _check(self._lib.sfnn_set_fused_decode(self._h, int(bool(enable))), "sfnn_set_fused_decode")

    def set_fused_quota(self, quota: int):
        """The single-token kernel's rebalancing quota (0: off; -1: the profile's default)."""
        _check(self._lib.sfnn_set_fused_quota(self._h, int(quota)), "sfnn_set_fused_quota")

    def set_batch_depths(self, bstages: int = -1, c2pre: int = -1, c1depth: int = -1, c2stages: int = -1):
        """The few-token kernel's request depths (B^T half rows per warp, W_down rows requested
        during the up/gate stream, up/gate segments in flight per warp, W_down rows in flight
        in the down phase); -1 keeps a value."""
        _check(self._lib.sfnn_set_batch_depths(self._h, int(bstages), int(c2pre), int(c1depth), int(c2stages)),
               "sfnn_set_batch_depths")

    def set_batch_tc_shape(self, up_ctas_per_sm: int = -1, up_chunks_per_step: int = -1,
                           down_tiles_per_cta: int = -1):
        """The tensor-core path's kernel shapes: the up projection's CTAs per SM (1 or 2) and
        64-wide K chunks of every row staged per step (1 or 2), the down projection's
        128-column output tiles per CTA (1 or 2); -1 keeps a value."""
        _check(self._lib.sfnn_set_batch_tc_shape(self._h, int(up_ctas_per_sm), int(up_chunks_per_step),
                                                 int(down_tiles_per_cta)), "sfnn_set_batch_tc_shape")

    def tune_batch_paths(self, stream=None):
        """Measure which path serves AUTO batches just above the few-token kernel's size
        faster (two few-token launches or tensor cores) and make AUTO take it (set-up call).
        Returns {b: (ms of two launches, ms of tensor cores)} for the b it measured."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        ms = (ctypes.c_float * 18)()
        with torch.cuda.device(self.device):
            _check(self._lib.sfnn_tune_batch_paths(self._h, ms, ctypes.c_void_p(s.cuda_stream)), "sfnn_tune_batch_paths")
        return {b: (ms[2 * b], ms[2 * b + 1]) for b in range(9) if ms[2 * b + 1] > 0}

    def set_batch_quota(self, enable: bool):
        """The few-token kernel's rebalancing (off: each token's y independent of the batch)."""
        _check(self._lib.sfnn_set_batch_quota(self._h, 1 if enable else 0), "sfnn_set_batch_quota")

    def set_fused_depths(self, bstages: int = -1, c2pre: int = -1, c1depth: int = -1, c2stages: int = -1):
        """The single-token kernel's request depths (B^T stages per warp, W_down rows requested
        during the up/gate stream, up/gate segments in flight per warp, W_down rows in flight
        in the down phase); -1 keeps a value."""
        _check(self._lib.sfnn_set_fused_depths(self._h, int(bstages), int(c2pre), int(c1depth), int(c2stages)),
               "sfnn_set_fused_depths")

    def set_hot_prefix(self, enable: bool):
        """Read the hot prefix densely on the fused few-token path (default on)."""
        _check(self._lib.sfnn_set_hot_prefix(self._h, int(bool(enable))), "sfnn_set_hot_prefix")

    def debug_stall_next_barrier(self, stream=None):
        _check(self._lib.sfnn_debug_stall_next_barrier(self._h, _stream(stream)), "sfnn_debug_stall_next_barrier")

    def set_profile_events(self, before, after):
        """torch.cuda.Event pair bracketing the next forward call's kernels (events must exist)."""
        _check(self._lib.sfnn_set_profile_events(self._h, ctypes.c_void_p(before.cuda_event),
                                                 ctypes.c_void_p(after.cuda_event)), "sfnn_set_profile_events")

    def info(self) -> dict:
        inf = Info()
        _check(self._lib.sfnn_query(self._h, ctypes.byref(inf)), "sfnn_query")
        return {k: getattr(inf, k) for k, _ in Info._fields_}

    def get_error(self) -> int:
        return int(self._lib.sfnn_get_error(self._h))

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            self._lib.sfnn_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


NOALLOC_SCRATCH_BYTES = 64 * 1024


def predict_noalloc(x, A, B, c, idx=None, count=None, stream=None):
    """The predicted set of one token without a handle or any allocation in the library.

    For callers that cannot allocate device memory (see sfnn_predict_noalloc in
    include/sfnn.h).  x [d], A [d, r], B [r, n], c [n]: CUDA tensors of one dtype;
    returns (idx [n] int32, count [1] int32), idx[:count] ascending.
    """
    lib = load_library()
    for t in (x, A, B, c):
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda" or not t.is_contiguous() or t.dtype != A.dtype:
            raise TypeError("x, A, B, c must be contiguous CUDA tensors of one dtype")
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A must be [d, r] and B [r, n]")
    d, r = A.shape
    n = B.shape[1]
    if x.numel() != d or B.shape[0] != r or c.numel() != n:
        raise ValueError(f"inconsistent shapes: x {tuple(x.shape)}, A {tuple(A.shape)}, B {tuple(B.shape)}, "
                         f"c {tuple(c.shape)}")
    idx = idx if idx is not None else torch.empty(n, dtype=torch.int32, device=A.device)
    count = count if count is not None else torch.empty(1, dtype=torch.int32, device=A.device)
    for name, t, need in (("idx", idx, n), ("count", count, 1)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda" or t.dtype != torch.int32 \
                or not t.is_contiguous() or t.numel() < need:
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of at least {need} elements")
    if any(t.device != A.device for t in (x, B, c, idx, count)):
        raise ValueError("all tensors must be on one device")
    with torch.cuda.device(A.device):  # the library runs on, and takes its scratch of, the current device
        _check(lib.sfnn_predict_noalloc(_ptr(x), _ptr(A), _ptr(B), _ptr(c), d, r, n, _dtype_code(A.dtype),
                                        _ptr(idx), _ptr(count), _stream(stream)), "sfnn_predict_noalloc")
    return idx, count


def forward_stack(layers, X0, XL=None, idx=None, counts=None, return_sets: bool = False, lookahead: bool = False,
                  stream=None):
    """Residual stack X_{l+1} = X_l + FFN_l(round(X_l)); X0 [b, d] (or [d]) fp32 CUDA tensor.

    ``lookahead``: layer l+1's set is predicted from layer l's input, one layer early
    (sfnn_forward_stack_lookahead)."""
    lib = load_library()
    if X0.dtype != torch.float32 or X0.device.type != "cuda" or not X0.is_contiguous():
        raise TypeError("X0 must be a contiguous fp32 CUDA tensor")
    b = 1 if X0.dim() == 1 else X0.shape[0]
    XL = XL if XL is not None else torch.empty_like(X0)
    n = layers[0].n
    if return_sets:
        idx = idx if idx is not None else torch.empty((len(layers), b, n), dtype=torch.int32, device=X0.device)
        counts = counts if counts is not None else torch.empty((len(layers), b), dtype=torch.int32,
                                                               device=X0.device)
    arr = (ctypes.c_void_p * len(layers))(*[l.handle.value for l in layers])
    name = "sfnn_forward_stack_lookahead" if lookahead else "sfnn_forward_stack"
    _check(getattr(lib, name)(arr, len(layers), _ptr(X0), b, _ptr(XL), _ptr(idx), _ptr(counts), _stream(stream)),
           name)
    return (XL, idx, counts) if return_sets else XL
