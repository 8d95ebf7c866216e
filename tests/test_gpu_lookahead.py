"""The look-ahead residual stack: layer l+1's set predicted from layer l's input.

* the fused look-ahead kernel (one launch per layer plus one) and the multi-kernel
  look-ahead path both match the oracle's look-ahead stack, with every layer's set --
  each path's own: the lists the fused launches consumed, the masks the multi-kernel
  path compacted -- arbitrated against the oracle's, for ReLU and ReGLU, at a reduced
  size and at the full LLaMA-7B-shaped 4-layer ReGLU stack;
* the sets really are predicted one layer early: they differ from the plain stack's;
* one layer (nothing to look ahead of) gives the plain stack's result;
* batches of tokens through the multi-kernel path, on tensor and CUDA cores;
* a stack of one handle used for every layer, int8 rows, sets that are empty
  (y = 0, so XL = X0 exactly), and a grid barrier that times out (reported, then the
  stack recovers and reproduces its result).
"""
import numpy as np
import pytest
import torch

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import NTHREADS, mask_from_idx

pytestmark = pytest.mark.gpu


def _x0(cfg, seed):
    return W.make_tokens(cfg, 1, seed=seed)[0].astype(np.float32)


def _stack_sets(hs, X0):
    XL, sidx, scnt = sf.forward_stack(hs, X0, return_sets=True, lookahead=True)
    n = hs[0].n
    return XL.cpu().numpy(), [mask_from_idx(sidx[l, 0].cpu().numpy(), scnt[l, 0].item(), n) for l in range(len(hs))]


def _run(hs, x0):
    """[(what, XL, per-layer masks)] of the fused path and of the multi-kernel path, each
    with the sets it used itself (the fused kernel's set output is checked against its
    plain call, which must give bitwise the same XL)."""
    X0 = torch.from_numpy(x0).cuda()
    XL_plain = sf.forward_stack(hs, X0, lookahead=True).cpu().numpy()
    XL_fused, m_fused = _stack_sets(hs, X0)
    distinct = all(a is not b for a, b in zip(hs, hs[1:]))
    if distinct:  # the fused path serves a set request (else the multi-kernel path does)
        assert np.array_equal(XL_plain, XL_fused)
    for h in hs:
        h.set_fused_decode(False)
    try:
        XL_multi, m_multi = _stack_sets(hs, X0)
    finally:
        for h in hs:
            h.set_fused_decode(True)
    out = [("multi-kernel", XL_multi, m_multi)]
    out.append(("fused", XL_fused, m_fused) if distinct else ("fused (its sets unreported)", XL_plain, m_multi))
    return out


def _check(layers, hs, x0, qrows=None):
    runs = _run(hs, x0)
    base = x0.astype(np.float64)
    for what, XL, masks in runs:
        xref, recs = oracle.forward_stack_lookahead(layers, x0.astype(np.float64), masks_other=masks,
                                                    nthreads=NTHREADS, qrows=qrows)
        for l, rec in enumerate(recs):
            assert rec["mismatches"].size == 0, f"{what}, layer {l}: sets differ outside the arbitration band"
        ok, ratio = oracle.within_tolerance(XL.astype(np.float64) - base, xref - base)
        assert ok, f"{what}: max|dx|/max|dx_ref| = {ratio:.3e}"
    for h in hs:
        assert h.get_error() == 0
    return runs[-1][1], runs[-1][2], None


@pytest.mark.parametrize("base", ["llama7b_reglu_stack", "opt6.7b_relu"])
def test_lookahead_stack_matches_oracle(base):
    cfg = W.small_config(W.CONFIGS[base], d=1024, n=2500, r=128)
    layers = [W.make_layer(cfg, seed=51, layer=l) for l in range(4)]
    hs = [sf.SparseFFN.from_layer(l) for l in layers]
    x0 = _x0(cfg, 52)
    _, masks, _ = _check(layers, hs, x0)
    # predicted one layer early: some layer's set differs from the plain stack's
    _, sidx, scnt = sf.forward_stack(hs, torch.from_numpy(x0).cuda(), return_sets=True)
    plain = [mask_from_idx(sidx[l, 0].cpu().numpy(), scnt[l, 0].item(), cfg.n) for l in range(4)]
    # layer 0 predicts from its own input either way (the two kernels sum the predictor in
    # different orders: they may part only within the arbitration band)
    _, z0, _ = oracle.predictor(x0.astype(cfg.np_dtype), layers[0].A, layers[0].B, layers[0].c, NTHREADS)
    assert oracle.arbitrate(z0, masks[0], plain[0])[1].size == 0
    assert any(not np.array_equal(masks[l], plain[l]) for l in range(1, 4))


@pytest.mark.parametrize("path", ["tensor_core", "cuda_core"])
def test_lookahead_batch_of_tokens(path):
    # b > 1 runs the multi-kernel path (tensor cores for the rows under AUTO at d = 1024,
    # or CUDA cores); every token is its own look-ahead stack
    cfg = W.small_config(W.CONFIGS["llama7b_reglu_stack"], d=1024, n=2500, r=128)
    layers = [W.make_layer(cfg, seed=64, layer=l) for l in range(3)]
    hs = [sf.SparseFFN.from_layer(l, max_batch=4) for l in layers]
    for h in hs:
        h.set_batch_path(sf.BATCH_TENSOR_CORE if path == "tensor_core" else sf.BATCH_CUDA_CORE)
    X0 = W.make_tokens(cfg, 3, seed=65).astype(np.float32)
    XL, sidx, scnt = sf.forward_stack(hs, torch.from_numpy(X0).cuda(), return_sets=True, lookahead=True)
    XL = XL.cpu().numpy()
    for t in range(3):
        masks = [mask_from_idx(sidx[l, t].cpu().numpy(), scnt[l, t].item(), cfg.n) for l in range(3)]
        xref, recs = oracle.forward_stack_lookahead(layers, X0[t].astype(np.float64), masks_other=masks,
                                                    nthreads=NTHREADS)
        assert all(r["mismatches"].size == 0 for r in recs)
        base = X0[t].astype(np.float64)
        ok, ratio = oracle.within_tolerance(XL[t].astype(np.float64) - base, xref - base)
        assert ok, f"token {t}: {ratio:.3e}"
    assert all(h.get_error() == 0 for h in hs)


def test_lookahead_full_size_llama7b_reglu_stack():
    cfg = W.CONFIGS["llama7b_reglu_stack"]
    layers = W.make_stack(cfg, seed=0)
    hs = [sf.SparseFFN.from_layer(l) for l in layers]
    _check(layers, hs, _x0(cfg, 53))


def test_lookahead_one_layer_is_the_plain_stack():
    cfg = W.small_config(W.CONFIGS["llama7b_reglu_stack"], d=2048, n=3001, r=256)
    lay = W.make_layer(cfg, seed=54)
    h = sf.SparseFFN.from_layer(lay)
    x0 = _x0(cfg, 55)
    X0 = torch.from_numpy(x0).cuda()
    a = sf.forward_stack([h], X0, lookahead=True).cpu().numpy()
    b = sf.forward_stack([h], X0).cpu().numpy()
    # the same set (the predictors' orders are the same); the rows are shared out to the
    # CTAs differently, so y agrees within the tolerance, and with the oracle's
    _, masks = _stack_sets([h], X0)
    xref, recs = oracle.forward_stack([lay], x0.astype(np.float64), masks_other=masks)
    assert recs[0]["mismatches"].size == 0
    base = x0.astype(np.float64)
    for XL in (a, b):
        assert oracle.within_tolerance(XL.astype(np.float64) - base, xref - base)[0]
    assert oracle.within_tolerance(a.astype(np.float64) - base, b.astype(np.float64) - base)[0]
    assert h.get_error() == 0


def test_lookahead_one_handle_for_every_layer():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1024, n=2000, r=128)
    lay = W.make_layer(cfg, seed=56)
    h = sf.SparseFFN.from_layer(lay)
    _check([lay] * 3, [h] * 3, _x0(cfg, 57))


@pytest.mark.parametrize("rows", ["int8", "int4"])
def test_lookahead_quantized_rows(rows):
    # int8 / int4 rows run the fused kernel only; its set output gives the sets it used
    cfg = W.small_config(W.CONFIGS["llama7b_reglu_stack"], d=1024, n=2500, r=128)
    layers = [W.make_layer(cfg, seed=58, layer=l) for l in range(3)]
    hs = [sf.SparseFFN.from_layer(l, rows=rows) for l in layers]
    x0 = _x0(cfg, 59)
    X0 = torch.from_numpy(x0).cuda()
    XL = sf.forward_stack(hs, X0, lookahead=True).cpu().numpy()
    XL_sets, masks = _stack_sets(hs, X0)
    assert np.array_equal(XL, XL_sets)
    qrows = [oracle.quantize_layer(l, bits=8 if rows == "int8" else 4) for l in layers]
    xref, recs = oracle.forward_stack_lookahead(layers, x0.astype(np.float64), masks_other=masks,
                                                nthreads=NTHREADS, qrows=qrows)
    assert all(r["mismatches"].size == 0 for r in recs)
    base = x0.astype(np.float64)
    assert oracle.within_tolerance(XL.astype(np.float64) - base, xref - base)[0]
    assert all(h.get_error() == 0 for h in hs)


def test_lookahead_empty_sets_leave_the_input():
    cfg = W.small_config(W.CONFIGS["llama7b_reglu_stack"], d=1024, n=1500, r=128)
    layers = [W.make_layer(cfg, seed=60, layer=l) for l in range(3)]
    for l in layers:
        l.c = np.full_like(l.c, -1e4)  # every logit far below the threshold
    hs = [sf.SparseFFN.from_layer(l) for l in layers]
    x0 = _x0(cfg, 61)
    for _, XL, masks in _run(hs, x0):
        assert all(m.sum() == 0 for m in masks)
        assert np.array_equal(XL, x0)


def test_lookahead_barrier_timeout_is_reported_and_recovers():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1024, n=3000, r=128)
    layers = [W.make_layer(cfg, seed=62, layer=l) for l in range(2)]
    hs = [sf.SparseFFN.from_layer(l) for l in layers]
    X0 = torch.from_numpy(_x0(cfg, 63)).cuda()
    ok = sf.forward_stack(hs, X0, lookahead=True).cpu().numpy()
    assert all(h.get_error() == 0 for h in hs)
    hs[0].debug_stall_next_barrier()
    sf.forward_stack(hs, X0, lookahead=True)
    torch.cuda.synchronize()  # returns: the launches on layer 0's counter gave up after their bound
    assert hs[0].get_error() == sf.STATUS_CODES["SFNN_ERR_TIMEOUT"]
    assert hs[1].get_error() == 0
    again = sf.forward_stack(hs, X0, lookahead=True).cpu().numpy()
    assert np.array_equal(again, ok)
    assert all(h.get_error() == 0 for h in hs)
