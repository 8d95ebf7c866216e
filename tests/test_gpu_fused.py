"""The fused single-token decode kernel (one launch per token).

* it agrees with the multi-kernel path and with the oracle -- its own set (the
  positions each tile decided and read, reported by the kernel) against the oracle's
  set, then y -- on layers whose
  tiles hold one or several B^T chunks and whose rows need one or several
  columns per thread (fp32 and fp16, ReLU and ReGLU, ragged n);
* consecutive launches on the same handle (programmatic dependent launch lets
  the next one start early) stay correct and bitwise reproducible, also with other
  kernels writing the input right before each call and reading the output right after
  (single token, few-token batches, the look-ahead stack);
* the residual stack runs through it;
* its request depths (B^T stages, W_down rows requested early, up/gate segments in
  flight) change nothing in the result: bitwise the same sets and y;
* its rebalancing of active rows over the CTAs (forced quotas, on a hot-packed layer
  whose tiles hold very different counts; the wait for the shared-out rows before the
  own rows' stream and inside it) gives the same sets and y within rounding, reproducibly;
* a grid barrier that cannot complete runs out after its bound, latches
  SFNN_ERR_TIMEOUT, leaves the context usable, and the handle recovers.
"""
import numpy as np
import pytest
import torch

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import check_token, dev, fused_step, mask_from_idx

pytestmark = pytest.mark.gpu

SHAPES = [
    ("tiny_relu_f32", 512, 2048, 64),
    ("opt6.7b_relu", 1024, 3001, 128),
    ("70b_reglu", 2048, 5003, 256),
    ("opt30b_relu", 7168, 4099, 1024),
    ("70b_reglu", 8192, 1500, 1024),
]


@pytest.mark.parametrize("base,d,n,r", SHAPES)
def test_fused_matches_multikernel_and_oracle(base, d, n, r):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=11)
    h = sf.SparseFFN.from_layer(lay)
    X = W.make_tokens(cfg, 4, seed=12)
    for t in range(4):
        xd = dev(X[t])
        h.set_fused_decode(True)
        yf, mf = fused_step(h, xd)
        assert np.array_equal(h.forward(xd).cpu().numpy(), yf)
        h.set_fused_decode(False)
        ym = h.forward(xd).cpu().numpy()
        _, idx, cnt = h.forward_batch(xd.reshape(1, -1), return_sets=True)
        h.set_fused_decode(True)
        assert oracle.within_tolerance(yf, ym.astype(np.float64))[0]
        check_token(lay, X[t], yf, mf, f"{base} t={t} fused")
        check_token(lay, X[t], ym, mask_from_idx(idx[0].cpu().numpy(), cnt[0].item(), cfg.n), f"{base} t={t} multi")
    assert h.get_error() == 0


def test_back_to_back_launches_same_handle():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=2048, n=6000, r=256)
    lay = W.make_layer(cfg, seed=13)
    h = sf.SparseFFN.from_layer(lay)
    X = dev(W.make_tokens(cfg, 16, seed=14))
    Y1 = torch.empty((16, cfg.d), dtype=torch.float32, device="cuda")
    for t in range(16):
        h.forward(X[t], Y1[t])
    torch.cuda.synchronize()
    Y2 = torch.stack([h.forward(X[t]) for t in range(16)])
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    Xh = X.cpu().numpy()
    for t in (0, 7, 15):
        y, m = fused_step(h, X[t])
        assert np.array_equal(y, Y1[t].cpu().numpy())
        check_token(lay, Xh[t], y, m)
    assert h.get_error() == 0


def test_fused_paths_in_stream_order_with_other_kernels():
    # the fused kernels start early (dependent launch) and read only weights before their
    # wait: inputs written by another kernel right before each call and outputs read right
    # after, on one stream with no host synchronisation, give the isolated calls' results
    # bitwise -- single token, few-token batches, and the look-ahead stack
    cfg = W.small_config(W.CONFIGS["70b_reglu"], d=2048, n=5003, r=256)
    layers = [W.make_layer(cfg, seed=15 + l, layer=l) for l in range(2)]
    hs = [sf.SparseFFN.from_layer(l, max_batch=4) for l in layers]
    h = hs[0]
    X = dev(W.make_tokens(cfg, 12, seed=16))
    X32 = X.float()
    plan = [("one", 1), ("batch", 2), ("one", 1), ("batch", 4), ("stack", 1), ("batch", 3), ("one", 1)]

    def call(kind, x, y, stream=None):
        if kind == "one":
            return h.forward(x[0], y[0], stream=stream)
        if kind == "batch":
            return h.forward_batch(x, y, stream=stream)
        return sf.forward_stack(hs, x[0], y[0], lookahead=True, stream=stream)

    ref = []
    for i, (kind, b) in enumerate(plan):  # isolated
        x = (X32 if kind == "stack" else X)[i:i + b]
        y = torch.empty((b, cfg.d), dtype=torch.float32, device="cuda")
        call(kind, x.clone(), y)
        torch.cuda.synchronize()
        ref.append(y.clone())
    s = torch.cuda.Stream()
    xin = torch.empty((4, cfg.d), dtype=X.dtype, device="cuda")
    xin32 = torch.empty((4, cfg.d), dtype=torch.float32, device="cuda")
    yout = torch.empty((4, cfg.d), dtype=torch.float32, device="cuda")
    outs = []
    with torch.cuda.stream(s):
        for i, (kind, b) in enumerate(plan):
            buf = xin32 if kind == "stack" else xin
            buf[:b].copy_((X32 if kind == "stack" else X)[i:i + b] * 1.0)  # written right before
            call(kind, buf[:b], yout[:b], stream=s)
            outs.append(yout[:b] * 1.0)  # read right after
    torch.cuda.synchronize()
    for i, (a, e) in enumerate(zip(outs, ref)):
        assert torch.equal(a, e), f"call {i} ({plan[i][0]}, b = {plan[i][1]})"
    assert all(x.get_error() == 0 for x in hs)


def test_stack_through_fused_kernel():
    cfg = W.small_config(W.CONFIGS["llama7b_reglu_stack"], d=1024, n=2500, r=128)
    layers = [W.make_layer(cfg, seed=15, layer=l) for l in range(3)]
    hs = [sf.SparseFFN.from_layer(l) for l in layers]
    x0 = W.make_tokens(cfg, 1, seed=16)[0]
    X0 = torch.from_numpy(x0.astype(np.float32)).cuda()
    XL_fused = sf.forward_stack(hs, X0).cpu().numpy()
    XL_sets, sidx, scnt = sf.forward_stack(hs, X0, return_sets=True)
    masks = [mask_from_idx(sidx[l, 0].cpu().numpy(), scnt[l, 0].item(), cfg.n) for l in range(3)]
    xref, recs = oracle.forward_stack(layers, x0.astype(np.float64), masks_other=masks)
    assert all(r["mismatches"].size == 0 for r in recs)
    base = x0.astype(np.float64)
    assert oracle.within_tolerance(XL_fused.astype(np.float64) - base, xref - base)[0]
    assert oracle.within_tolerance(XL_sets.cpu().numpy().astype(np.float64) - base, xref - base)[0]


def test_grid_barrier_timeout_is_reported_and_recovers():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1024, n=3000, r=128)
    lay = W.make_layer(cfg, seed=17)
    h = sf.SparseFFN.from_layer(lay)
    xd = dev(W.make_tokens(cfg, 1, seed=18)[0])
    y_ok = h.forward(xd).cpu().numpy()
    assert h.get_error() == 0
    h.debug_stall_next_barrier()
    h.forward(xd)
    torch.cuda.synchronize()  # returns: the kernel gave up after its bound
    assert h.get_error() == sf.STATUS_CODES["SFNN_ERR_TIMEOUT"]
    assert h.get_error() == 0
    y_again = h.forward(xd).cpu().numpy()
    assert np.array_equal(y_again, y_ok)
    assert h.get_error() == 0


def test_fused_kernels_beside_a_kernel_on_another_stream():
    """The fused kernels' grid barriers need all their CTAs resident; a kernel that holds
    an SM on another stream (a bounded spin of ~20 ms here) delays the CTAs that would
    run there, and the barriers wait for them (well inside their one-second bound):
    results stay exact and no error is latched."""
    cfg = W.small_config(W.CONFIGS["70b_reglu"], d=2048, n=5003, r=256)
    lay = W.make_layer(cfg, seed=19)
    h = sf.SparseFFN.from_layer(lay, max_batch=4)
    X = dev(W.make_tokens(cfg, 4, seed=20))
    y_ref = h.forward(X[0]).clone()
    Y_ref = h.forward_batch(X).clone()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    for _ in range(2):
        with torch.cuda.stream(side):
            torch.cuda._sleep(40_000_000)  # ~20 ms at the B200's clocks
        y = h.forward(X[0])
        Y = h.forward_batch(X)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(Y, Y_ref)
    assert h.get_error() == 0


@pytest.mark.parametrize("base,d,n,r,quota", [
    ("70b_reglu", 1024, 5003, 128, 2),     # few own segments: the wait comes before the stream
    ("70b_reglu", 8192, 3001, 1024, 12),   # the wait inside the stream of own segments
    ("opt6.7b_relu", 4096, 9000, 512, 6),
])
def test_rebalanced_rows_match(base, d, n, r, quota):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=21)
    h = sf.SparseFFN.from_layer(lay, order="packed")  # the hottest neurons fill the first tiles
    X = W.make_tokens(cfg, 3, seed=22)
    for t in range(3):
        xd = dev(X[t])
        h.set_fused_quota(0)
        y0, m0 = fused_step(h, xd)
        h.set_fused_quota(quota)
        y1, m1 = fused_step(h, xd)
        assert np.array_equal(m0, m1)
        assert oracle.within_tolerance(y1, y0.astype(np.float64))[0]
        assert np.array_equal(h.forward(xd).cpu().numpy(), y1)  # deterministic for a quota
        check_token(lay, X[t], y1, m1, f"{base} quota {quota} t={t}")
    h.set_fused_quota(-1)
    assert h.get_error() == 0


@pytest.mark.parametrize("base,d,n,r", [("70b_reglu", 8192, 5003, 1024), ("opt6.7b_relu", 4096, 9000, 1024),
                                        ("tiny_relu_f32", 512, 2048, 64)])
def test_request_depths_do_not_change_the_result(base, d, n, r):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=31)
    h = sf.SparseFFN.from_layer(lay)
    h.set_fused_quota(3)  # the rebalancing's wait runs beside the up/gate stream
    X = W.make_tokens(cfg, 2, seed=32)
    ref = [fused_step(h, dev(X[t])) for t in range(2)]
    for depths in [(1, 0, 1, 1), (3, 16, 2, 16), (6, 2, 1, 2), (8, 5, 2, 4), (4, 8, 2, 8), (2, 4, 1, 8)]:
        try:
            h.set_fused_depths(*depths)
        except RuntimeError as e:  # 8 stages of a 2 KB row do not fit beside a large x
            assert "UNSUPPORTED" in str(e) and depths[0] == 8, e
            continue
        for t in range(2):
            y, m = fused_step(h, dev(X[t]))
            assert np.array_equal(m, ref[t][1]) and np.array_equal(y, ref[t][0]), depths
    for bad in [(5, -1, -1, -1), (-1, 17, -1, -1), (-1, -1, 3, -1), (-1, -1, -1, 3)]:
        with pytest.raises(RuntimeError):
            h.set_fused_depths(*bad)
    assert h.get_error() == 0
