"""The multi-token fused kernel: a batch of 2 to 4 tokens in one launch on CUDA cores.

* every token agrees with the oracle, with the set that kernel itself decided and read
  (its per-token set output) arbitrated against the oracle's, for ReLU and ReGLU,
  ragged n, d up to 8192 and 2, 3 or 4 tokens;
* it agrees with the tensor-core path within the tolerance, is bitwise reproducible,
  and its set output changes nothing (the plain call gives bitwise the same Y);
* with the rebalancing of union rows over the CTAs switched off, a token's row of Y does
  not depend on which other tokens share the batch (a row applies only to the tokens
  whose sets hold it); with it on (the full-size 70B-shaped layer), the sets are the
  same, Y agrees within rounding and is bitwise reproducible for a given batch;
* AUTO takes it for 2 to 4 tokens on the full OPT-30B- and 70B-shaped layers, and the
  residual stack runs through it;
* 5 to 8 tokens as two few-token launches (FUSED, and AUTO after the measured choice)
  agree with the oracle per token;
* its request depths change nothing in the result (bitwise the same Y and sets);
* outputs stay inside their buffers (canary words on both sides).
"""
import numpy as np
import pytest
import torch

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import NTHREADS, assert_guards, check_token, dev, guarded, mask_from_idx

pytestmark = pytest.mark.gpu

SHAPES = [
    ("opt6.7b_relu", 1024, 3001, 128),
    ("70b_reglu", 2048, 5003, 256),
    ("opt30b_relu", 7168, 4099, 1024),
    ("70b_reglu", 8192, 1500, 1024),
]


def run_multi(h, X, sets=True):
    """(Y, per-token masks) of one forward_batch call, outputs inside canary words."""
    b = X.shape[0]
    gy, Y = guarded((b, h.d))
    if not sets:
        h.forward_batch(dev(X), Y)
        assert_guards(gy)
        return Y.cpu().numpy(), None
    gi, idx = guarded((b, h.n), torch.int32)
    gc, cnt = guarded((b,), torch.int32)
    h.forward_batch(dev(X), Y, idx=idx, counts=cnt, return_sets=True)
    assert_guards(gy, gi, gc)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    return Y.cpu().numpy(), [mask_from_idx(idx[t], cnt[t], h.n) for t in range(b)]


@pytest.mark.parametrize("b", [2, 3, 4])
@pytest.mark.parametrize("base,d,n,r", SHAPES)
def test_multi_matches_oracle(base, d, n, r, b):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=71)
    h = sf.SparseFFN.from_layer(lay, max_batch=4)
    h.set_batch_path(sf.BATCH_FUSED)
    X = W.make_tokens(cfg, b, seed=72 + b)
    Y, masks = run_multi(h, X)
    for t in range(b):
        check_token(lay, X[t], Y[t], masks[t], f"{base} d={d} b={b} t={t}")
    Y2, _ = run_multi(h, X, sets=False)
    assert np.array_equal(Y, Y2)  # the set output changes nothing; bitwise reproducible
    Y3, masks3 = run_multi(h, X)
    assert np.array_equal(Y, Y3) and all(np.array_equal(a, c) for a, c in zip(masks, masks3))
    if d % 128 == 0:
        h.set_batch_path(sf.BATCH_TENSOR_CORE)
        Yt, masks_t = run_multi(h, X)
        for t in range(b):
            if np.array_equal(masks[t], masks_t[t]):
                assert oracle.within_tolerance(Y[t], Yt[t].astype(np.float64))[0]
    assert h.get_error() == 0


def test_rows_do_not_depend_on_the_other_tokens():
    cfg = W.small_config(W.CONFIGS["70b_reglu"], d=2048, n=5003, r=256)
    lay = W.make_layer(cfg, seed=73)
    h = sf.SparseFFN.from_layer(lay, max_batch=4)
    h.set_batch_path(sf.BATCH_FUSED)
    h.set_batch_quota(False)
    X = W.make_tokens(cfg, 6, seed=74)
    Ya, ma = run_multi(h, X[[0, 1, 2, 3]])
    Yb, mb = run_multi(h, X[[4, 0, 5]])
    assert np.array_equal(ma[0], mb[1])
    # the same rows, the same order of every sum: token 0's output is bitwise the same
    assert np.array_equal(Ya[0], Yb[1])
    y1, m1 = run_multi(h, X[[0, 5]])
    assert np.array_equal(Ya[0], y1[0])
    assert h.get_error() == 0


@pytest.mark.parametrize("name,batches", [("opt30b_relu", (2, 4)), ("70b_reglu", (2, 3, 4))])
def test_multi_full_size_auto(name, batches):
    cfg = W.CONFIGS[name]
    lay = W.make_layer(cfg, seed=0)
    h = sf.SparseFFN.from_layer(lay, max_batch=max(batches))
    assert h.info()["batch_path"] == sf.BATCH_AUTO
    for b in batches:
        X = W.make_tokens(cfg, b, seed=75, stream_key=b)
        Y, masks = run_multi(h, X)
        for t in range(b):
            check_token(lay, X[t], Y[t], masks[t], f"{name} b={b} t={t}")
    assert h.get_error() == 0
    del h
    torch.cuda.empty_cache()


def test_rebalanced_union_rows():
    cfg = W.CONFIGS["70b_reglu"]
    lay = W.make_layer(cfg, seed=0)
    h = sf.SparseFFN.from_layer(lay, max_batch=2)
    h.set_batch_path(sf.BATCH_FUSED)
    X = W.make_tokens(cfg, 2, seed=80)
    Y_on, m_on = run_multi(h, X)
    assert np.array_equal(run_multi(h, X)[0], Y_on)  # deterministic for a given batch
    h.set_batch_quota(False)
    Y_off, m_off = run_multi(h, X)
    h.set_batch_quota(True)
    assert all(np.array_equal(a, c) for a, c in zip(m_on, m_off))
    for t in range(2):
        assert oracle.within_tolerance(Y_on[t].astype(np.float64), Y_off[t].astype(np.float64))[0]
        check_token(lay, X[t], Y_on[t], m_on[t], f"70b b=2 rebalanced t={t}")
    assert h.get_error() == 0
    del h
    torch.cuda.empty_cache()


def test_stack_of_two_tokens_through_the_multi_kernel():
    cfg = W.small_config(W.CONFIGS["llama7b_reglu_stack"], d=1024, n=2500, r=128)
    layers = [W.make_layer(cfg, seed=76, layer=l) for l in range(3)]
    hs = [sf.SparseFFN.from_layer(l, max_batch=2) for l in layers]
    X0 = W.make_tokens(cfg, 2, seed=77).astype(np.float32)
    XL, sidx, scnt = sf.forward_stack(hs, torch.from_numpy(X0).cuda(), return_sets=True)
    XL_plain = sf.forward_stack(hs, torch.from_numpy(X0).cuda())
    assert torch.equal(XL, XL_plain)
    XL = XL.cpu().numpy()
    for t in range(2):
        masks = [mask_from_idx(sidx[l, t].cpu().numpy(), scnt[l, t].item(), cfg.n) for l in range(3)]
        xref, recs = oracle.forward_stack(layers, X0[t].astype(np.float64), masks_other=masks, nthreads=NTHREADS)
        assert all(r["mismatches"].size == 0 for r in recs)
        base = X0[t].astype(np.float64)
        assert oracle.within_tolerance(XL[t].astype(np.float64) - base, xref - base)[0]
    assert all(h.get_error() == 0 for h in hs)


@pytest.mark.parametrize("base", ["opt6.7b_relu", "70b_reglu"])
def test_hot_prefix_changes_nothing(base):
    """The hot prefix only moves the hottest rows' gate/up dots ahead of the predictor's
    barrier: the same dots, the same sums, bitwise the same Y and sets."""
    cfg = W.small_config(W.CONFIGS[base], d=2048, n=5003, r=256)
    lay = W.make_layer(cfg, seed=78)
    h = sf.SparseFFN.from_layer(lay, max_batch=4)
    h.set_batch_path(sf.BATCH_FUSED)
    for b in (2, 3, 4):
        X = W.make_tokens(cfg, b, seed=79 + b)
        Y_on, m_on = run_multi(h, X)
        h.set_hot_prefix(False)
        Y_off, m_off = run_multi(h, X)
        h.set_hot_prefix(True)
        assert np.array_equal(Y_on, Y_off)
        assert all(np.array_equal(a, c) for a, c in zip(m_on, m_off))
        for t in range(b):
            check_token(lay, X[t], Y_on[t], m_on[t], f"{base} b={b} t={t}")
    # without a hotness profile there is no prefix, and the layer still decodes correctly
    h0 = sf.SparseFFN.from_layer(lay, max_batch=4, use_hotness=False)
    X = W.make_tokens(cfg, 3, seed=90)
    Y, masks = run_multi(h0, X)
    for t in range(3):
        check_token(lay, X[t], Y[t], masks[t], f"{base} identity order t={t}")
    assert h.get_error() == 0 and h0.get_error() == 0


@pytest.mark.parametrize("base,d,n,r", [("70b_reglu", 8192, 5003, 1024), ("opt6.7b_relu", 4096, 9000, 1024)])
def test_batch_request_depths_do_not_change_the_result(base, d, n, r):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=33)
    h = sf.SparseFFN.from_layer(lay, max_batch=3)
    h.set_batch_path(sf.BATCH_FUSED)
    X = W.make_tokens(cfg, 3, seed=34)
    ref = run_multi(h, X)
    for depths in [(2, 0, 1, 1), (4, 8, 2, 2), (8, 1, 1, 8), (6, 4, 2, 4)]:
        try:
            h.set_batch_depths(*depths)
        except RuntimeError as e:  # 8 W_down stages of 16 KB rows, or 8 B^T stages, may not fit
            assert "UNSUPPORTED" in str(e) or "INVALID" in str(e), e
            continue
        Y, m = run_multi(h, X)
        assert np.array_equal(Y, ref[0]), depths
        assert all(np.array_equal(a, c) for a, c in zip(m, ref[1])), depths
    for bad in [(3, -1, -1, -1), (-1, 9, -1, -1), (-1, -1, 0, -1), (-1, -1, -1, 16)]:
        with pytest.raises(RuntimeError):
            h.set_batch_depths(*bad)
    assert h.get_error() == 0


@pytest.mark.parametrize("b", [5, 6, 8])
def test_two_launch_batches(b):
    cfg = W.small_config(W.CONFIGS["70b_reglu"], d=2048, n=5003, r=256)
    lay = W.make_layer(cfg, seed=35)
    h = sf.SparseFFN.from_layer(lay, max_batch=8)
    X = W.make_tokens(cfg, b, seed=36 + b)
    h.set_batch_path(sf.BATCH_FUSED)
    Y, masks = run_multi(h, X)
    for t in range(b):
        check_token(lay, X[t], Y[t], masks[t], f"two launches b={b} t={t}")
    # each half is exactly the few-token kernel's result on that half alone
    h.set_batch_quota(False)
    Yq, _ = run_multi(h, X)
    Ya, _ = run_multi(h, X[: (b + 1) // 2])
    assert np.array_equal(Yq[: (b + 1) // 2], Ya)
    h.set_batch_quota(True)
    h.set_batch_path(sf.BATCH_AUTO)
    h.tune_batch_paths()
    Y2, m2 = run_multi(h, X)
    for t in range(b):
        check_token(lay, X[t], Y2[t], m2[t], f"auto after tuning b={b} t={t}")
    assert h.get_error() == 0
