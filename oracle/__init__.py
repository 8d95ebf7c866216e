"""CPU oracle for activation-sparse FFN decode (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The CUDA library does not, and this package
imports nothing from it: the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, no blocking or
reordering beyond the definitions); this module builds it with gcc, marshals
numpy arrays into it, and adds the parts that are pure bookkeeping: looping
over the tokens of a batch, the residual stack, and the arbitration rule for
neurons whose logit lies within 1e-3 of the threshold.

Definitions (see ``oracle.c`` for the passages they follow):
  predictor   h = relu(x A), z = h B + c, S = {i : z_i > 0}  (sigmoid(z) > 0.5)
  FFN         y = sum_{i in S} act_i(x) W_down[:, i]
              ReLU  act_i = relu(W_up[i].x + b_i)
              ReGLU act_i = relu(W_gate[i].x + b_i) * (W_up[i].x)
  stack       x_{l+1} = x_l + y_l  (double), next layer's input = x_{l+1}
              rounded to the storage dtype (round to nearest even).
  look-ahead  the same stack, but layer l+1's set is predicted from layer l's
              input (its predictor applied one layer early); layer 0's from its own.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

RELU, REGLU = 0, 1
F32, F16 = 0, 1
ARBITRATION_BAND = 1e-3


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, IEEE double, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-std=c99", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, L = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.oracle_decode.argtypes = [P, I, L, P]
        lib.oracle_decode.restype = None
        lib.oracle_predictor.argtypes = [I, I, I, I, P, P, P, P, P, P, P, I]
        lib.oracle_predictor.restype = I
        lib.oracle_preact.argtypes = [I, I, I, I, P, P, P, P, P, I]
        lib.oracle_preact.restype = None
        lib.oracle_ffn_masked.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, I]
        lib.oracle_ffn_masked.restype = None
        lib.oracle_forward.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, I]
        lib.oracle_forward.restype = I
        lib.oracle_quantize.argtypes = [I, I, I, P, L, L, I, P, P]
        lib.oracle_quantize.restype = None
        lib.oracle_ffn_masked_q.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, I]
        lib.oracle_ffn_masked_q.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = I
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _dt(arr: np.ndarray) -> int:
    if arr.dtype == np.float16:
        return F16
    if arr.dtype == np.float32:
        return F32
    raise TypeError(f"oracle takes fp16 or fp32 parameters, got {arr.dtype}")


def _c(arr):
    if arr is None:
        return None
    return np.ascontiguousarray(arr)


def _p(arr):
    return None if arr is None else arr.ctypes.data_as(ctypes.c_void_p)


def _act_code(act) -> int:
    if isinstance(act, str):
        return REGLU if act == "reglu" else RELU
    return int(act)


def decode(arr: np.ndarray) -> np.ndarray:
    """The oracle's exact conversion of stored elements to double."""
    a = _c(arr)
    out = np.empty(a.size, dtype=np.float64)
    _load().oracle_decode(_p(a), _dt(a), a.size, _p(out))
    return out.reshape(a.shape)


@dataclass
class Step:
    h: np.ndarray  # [r]
    z: np.ndarray  # [n]
    mask: np.ndarray  # [n] uint8
    a: np.ndarray  # [n]
    y: np.ndarray  # [d]

    @property
    def idx(self) -> np.ndarray:
        return np.flatnonzero(self.mask).astype(np.int32)


def predictor(x, A, B, c, nthreads: int = 1):
    """h = relu(x A), z = h B + c, mask = z > 0.  Returns (h, z, mask)."""
    x, A, B, c = _c(x), _c(A), _c(B), _c(c)
    d, r = A.shape
    n = B.shape[1]
    assert B.shape[0] == r and x.shape == (d,) and c.shape == (n,)
    h = np.empty(r, np.float64)
    z = np.empty(n, np.float64)
    mask = np.empty(n, np.uint8)
    _load().oracle_predictor(d, r, n, _dt(A), _p(x), _p(A), _p(B), _p(c), _p(h), _p(z), _p(mask), nthreads)
    return h, z, mask


def preact(x, w_up, w_gate, b, act, nthreads: int = 1) -> np.ndarray:
    """g_i = W[i].x + b_i of the ReLU'd projection (W_up for ReLU, W_gate for ReGLU)."""
    x, w_up, w_gate, b = _c(x), _c(w_up), _c(w_gate), _c(b)
    n, d = w_up.shape
    g = np.empty(n, np.float64)
    _load().oracle_preact(d, n, _act_code(act), _dt(w_up), _p(x), _p(w_up), _p(w_gate), _p(b), _p(g), nthreads)
    return g


def ffn_masked(x, w_up, w_gate, b, w_down, mask, act, nthreads: int = 1):
    """FFN over the neurons with mask != 0.  Returns (a [n], y [d])."""
    x, w_up, w_gate, b, w_down = _c(x), _c(w_up), _c(w_gate), _c(b), _c(w_down)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    n, d = w_up.shape
    assert w_down.shape == (d, n) and mask.shape == (n,)
    a = np.empty(n, np.float64)
    y = np.empty(d, np.float64)
    _load().oracle_ffn_masked(d, n, _act_code(act), _dt(w_up), _p(x), _p(w_up), _p(w_gate), _p(b), _p(w_down),
                              _p(mask), _p(a), _p(y), nthreads)
    return a, y


def forward(layer, x, nthreads: int = 1) -> Step:
    """One decode step of ``layer`` (any object with w_up, w_gate, b, w_down, A, B, c and cfg.act)."""
    h, z, mask = predictor(x, layer.A, layer.B, layer.c, nthreads)
    a, y = ffn_masked(x, layer.w_up, layer.w_gate, layer.b, layer.w_down, mask, layer.cfg.act, nthreads)
    return Step(h, z, mask, a, y)


# ---------------------------------------------------------------- int8 rows
@dataclass
class QRows:
    """A layer's FFN rows as int8 codes and fp32 scales, one scale per neuron and
    projection; q_down is neuron-major (neuron i's down row = column i of w_down)."""
    q_up: np.ndarray
    s_up: np.ndarray
    q_gate: np.ndarray | None
    s_gate: np.ndarray | None
    q_down: np.ndarray
    s_down: np.ndarray


QMAX = {8: 127, 4: 7}


def quantize(w, units_along_rows: bool = True, bits: int = 8):
    """Per-unit symmetric codes of a 2-D array (units = rows, or columns when
    ``units_along_rows`` is False), 8 or 4 bits: fp32 scale = absmax / qmax (127 or 7),
    codes rounded to nearest even in fp32 and clamped to [-qmax, qmax].
    Returns (q [units, len] int8, one code per byte; s [units])."""
    w = _c(w)
    assert w.ndim == 2
    rows, cols = w.shape
    units, length = (rows, cols) if units_along_rows else (cols, rows)
    ustride, estride = (cols, 1) if units_along_rows else (1, cols)
    q = np.empty((units, length), np.int8)
    sc = np.empty(units, np.float32)
    _load().oracle_quantize(units, length, _dt(w), _p(w), ustride, estride, QMAX[bits], _p(q), _p(sc))
    return q, sc


def quantize_layer(layer, bits: int = 8) -> QRows:
    q_up, s_up = quantize(layer.w_up, bits=bits)
    q_gate = s_gate = None
    if layer.w_gate is not None:
        q_gate, s_gate = quantize(layer.w_gate, bits=bits)
    q_down, s_down = quantize(layer.w_down, units_along_rows=False, bits=bits)
    return QRows(q_up, s_up, q_gate, s_gate, q_down, s_down)


def ffn_masked_q(x, qr: QRows, b, mask, act, nthreads: int = 1):
    """The FFN over the neurons with mask != 0, weights = codes * scales.  Returns (a, y)."""
    x, b = _c(x), _c(b)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    n, d = qr.q_up.shape
    assert qr.q_down.shape == (n, d) and mask.shape == (n,)
    a = np.empty(n, np.float64)
    y = np.empty(d, np.float64)
    gate_q = qr.q_gate if qr.q_gate is not None else qr.q_up
    gate_s = qr.s_gate if qr.s_gate is not None else qr.s_up
    _load().oracle_ffn_masked_q(d, n, _act_code(act), _dt(x), _p(x), _p(np.ascontiguousarray(qr.q_up)),
                                _p(np.ascontiguousarray(qr.s_up)), _p(np.ascontiguousarray(gate_q)),
                                _p(np.ascontiguousarray(gate_s)), _p(b), _p(np.ascontiguousarray(qr.q_down)),
                                _p(np.ascontiguousarray(qr.s_down)), _p(mask), _p(a), _p(y), nthreads)
    return a, y


def forward_q(layer, qr: QRows, x, nthreads: int = 1) -> Step:
    """One decode step with int8 rows: the predictor as in ``forward``, then the FFN on
    the dequantized rows."""
    h, z, mask = predictor(x, layer.A, layer.B, layer.c, nthreads)
    a, y = ffn_masked_q(x, qr, layer.b, mask, layer.cfg.act, nthreads)
    return Step(h, z, mask, a, y)


def forward_q_with_mask(layer, qr: QRows, x, mask, nthreads: int = 1) -> np.ndarray:
    return ffn_masked_q(x, qr, layer.b, mask, layer.cfg.act, nthreads)[1]


def forward_batch(layer, X, nthreads: int = 1) -> list[Step]:
    """Each token of a batch is independent: row t equals the single-token step of X[t]."""
    return [forward(layer, X[t], nthreads) for t in range(X.shape[0])]


def arbitrate(z_ref: np.ndarray, mask_ref: np.ndarray, mask_other: np.ndarray,
              band: float = ARBITRATION_BAND):
    """Resolve the active-set comparison.

    Neurons with |z_ref| < band may go either way; for them the other side's
    decision is taken.  Returns (mask_to_use, mismatches) where ``mismatches``
    lists neurons outside the band on which the two sets differ (must be empty).
    """
    mask_ref = np.asarray(mask_ref, dtype=bool)
    mask_other = np.asarray(mask_other, dtype=bool)
    near = np.abs(z_ref) < band
    mismatches = np.flatnonzero((mask_ref != mask_other) & ~near)
    use = np.where(near, mask_other, mask_ref)
    return use.astype(np.uint8), mismatches


def forward_with_mask(layer, x, mask, nthreads: int = 1) -> np.ndarray:
    """y for an explicitly given set (used after arbitration)."""
    return ffn_masked(x, layer.w_up, layer.w_gate, layer.b, layer.w_down, mask, layer.cfg.act, nthreads)[1]


def forward_stack(layers, x0, masks_other=None, nthreads: int = 1):
    """Residual stack: x_{l+1} = x_l + y_l in double; layer inputs rounded to the storage dtype.

    ``masks_other``: optional per-layer predicted sets from another implementation;
    when given, each layer's set is arbitrated against it (see ``arbitrate``) and
    the arbitrated set is used for that layer.  Returns (x_L, per-layer records).
    """
    dt = layers[0].w_up.dtype
    resid = np.asarray(x0, dtype=np.float64).copy()
    records = []
    for li, layer in enumerate(layers):
        xin = resid.astype(dt)  # round to nearest even
        h, z, mask = predictor(xin, layer.A, layer.B, layer.c, nthreads)
        mismatches = np.empty(0, np.int64)
        if masks_other is not None:
            mask, mismatches = arbitrate(z, mask, masks_other[li])
        a, y = ffn_masked(xin, layer.w_up, layer.w_gate, layer.b, layer.w_down, mask, layer.cfg.act, nthreads)
        records.append(dict(x_in=xin, z=z, mask=mask, y=y, mismatches=mismatches))
        resid = resid + y
    return resid, records


def forward_stack_lookahead(layers, x0, masks_other=None, nthreads: int = 1, qrows=None):
    """Residual stack whose sets are predicted one layer ahead.

    Follows the asynchronous predictor of DejaVu (53ai.com "sparsity for LLM inference"
    page, section "如何推理加速"): the next layer's sparsity is predicted one step in
    advance, so that the prediction can run beside the current layer.  Reading: layer l+1's
    predictor (its own A, B, c) takes layer l's input u_l = round(x_l); layer 0, which
    has no earlier input, predicts from u_0.  Everything else is ``forward_stack``:
    x_{l+1} = x_l + y_l in double, u_{l+1} = round(x_{l+1}), y_l computed on u_l.
    ``masks_other`` and the records are as in ``forward_stack``; each record adds
    ``x_pred``, the input its set was predicted from.  ``qrows`` (one ``QRows`` per
    layer) runs every layer's FFN on int8 rows (``ffn_masked_q``).
    """
    dt = layers[0].w_up.dtype
    resid = np.asarray(x0, dtype=np.float64).copy()
    records = []
    for li, layer in enumerate(layers):
        xin = resid.astype(dt)  # round to nearest even
        xpred = xin if li == 0 else records[li - 1]["x_in"]
        h, z, mask = predictor(xpred, layer.A, layer.B, layer.c, nthreads)
        mismatches = np.empty(0, np.int64)
        if masks_other is not None:
            mask, mismatches = arbitrate(z, mask, masks_other[li])
        if qrows is not None:
            a, y = ffn_masked_q(xin, qrows[li], layer.b, mask, layer.cfg.act, nthreads)
        else:
            a, y = ffn_masked(xin, layer.w_up, layer.w_gate, layer.b, layer.w_down, mask, layer.cfg.act, nthreads)
        records.append(dict(x_in=xin, x_pred=xpred, z=z, mask=mask, y=y, mismatches=mismatches))
        resid = resid + y
    return resid, records


def within_tolerance(y, y_ref, rel: float = 2e-3) -> tuple[bool, float]:
    """max|y - y_ref| <= rel * max|y_ref| (y_ref == 0 requires y == 0).  Returns (ok, ratio)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    scale = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    err = float(np.max(np.abs(y - y_ref))) if y_ref.size else 0.0
    if scale == 0.0:
        return err == 0.0, (0.0 if err == 0.0 else float("inf"))
    return err <= rel * scale, err / scale
