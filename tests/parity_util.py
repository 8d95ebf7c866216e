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


GUARD = 64  # canary words on each side of an output buffer
_PAT = 0x7FC0DEAD  # a NaN bit pattern that no kernel writes


def guarded(shape, dtype=torch.float32):
    """(raw, inner): an output buffer `inner` with canary words on both sides in `raw`
    (the kernels must write inside it only).  inner starts 256 bytes into raw."""
    n = int(np.prod(shape))
    raw = torch.full((n + 2 * GUARD,), _PAT, dtype=torch.int32, device="cuda")
    return raw, raw[GUARD:GUARD + n].view(dtype).view(shape)


def assert_guards(*raws):
    for raw in raws:
        r = raw.cpu().numpy()
        assert (r[:GUARD] == _PAT).all() and (r[-GUARD:] == _PAT).all(), "a kernel wrote outside its output buffer"


def fused_step(h, xd):
    """One token through the fused single-token kernel with the set that kernel itself
    decided and read (forward_batch at b = 1), outputs inside canary words: (y, mask)."""
    gy, Y = guarded((1, h.d))
    gi, idx = guarded((1, h.n), torch.int32)
    gc, cnt = guarded((1,), torch.int32)
    h.forward_batch(xd.reshape(1, -1), Y, idx=idx, counts=cnt, return_sets=True)
    assert_guards(gy, gi, gc)
    return Y[0].cpu().numpy(), mask_from_idx(idx[0].cpu().numpy(), cnt[0].item(), h.n)


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
