"""Shared helpers of the GPU parity tests: compare the CUDA library with the CPU oracle.

The comparison rule: the active sets must be identical except for neurons whose
oracle logit lies within 1e-3 of the threshold, where the GPU's decision is
taken; the oracle then recomputes y with that set and the GPU's y must be
within max|y - y_ref| <= 2e-3 * max|y_ref| (exact zero when y_ref is zero).
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

REL_TOL = 2e-3
NTHREADS = max(1, min(32, os.cpu_count() or 1))


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def mask_from_idx(idx_row, count, n):
    m = np.zeros(n, np.uint8)
    k = int(count)
    sel = np.asarray(idx_row[:k], dtype=np.int64)
    assert np.all((sel >= 0) & (sel < n)), "index out of range"
    assert np.unique(sel).size == sel.size, "duplicate index in a set"
    m[sel] = 1
    return m


def check_token(layer, x, y_gpu, mask_gpu, what=""):
    """Oracle step for token x; arbitrate the sets; tolerance on y.  Returns the error ratio."""
    ref = oracle.forward(layer, x, NTHREADS)
    use, mism = oracle.arbitrate(ref.z, ref.mask, mask_gpu)
    assert mism.size == 0, f"{what}: sets differ outside the arbitration band at {mism[:10]}"
    y_ref = ref.y if np.array_equal(use, ref.mask) else oracle.forward_with_mask(layer, x, use, NTHREADS)
    ok, ratio = oracle.within_tolerance(y_gpu, y_ref, REL_TOL)
    assert ok, f"{what}: max|dy|/max|y_ref| = {ratio:.3e} > {REL_TOL}"
    return ratio


class L:
    """Minimal layer record (duck-typed like workload.Layer)."""

    def __init__(self, act, w_up, w_gate, b, w_down, A, B, c, p=None):
        class C:
            pass
        self.cfg = C()
        self.cfg.act = act
        self.w_up, self.w_gate, self.b, self.w_down, self.A, self.B, self.c = w_up, w_gate, b, w_down, A, B, c
        self.p = p
