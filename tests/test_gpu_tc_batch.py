"""The tensor-core (tcgen05) path of the batched union FFN.

* every token of a batch agrees with the oracle (sets exact outside the arbitration
  band, y within the tolerance), for ReLU and ReGLU, d a multiple of 128 up to 8192,
  ragged n (the union's last tile and the down GEMM's last K chunk are partial), and
  batch sizes on both sides of the MMA's N = 16 / 32 (2, 5, 16, 17, 32);
* the batch's predictor runs on the tensor cores too (hidden layer split over d, logits
  with h as an fp16 hi + lo pair): its sets pass the same arbitration;
* it agrees with the CUDA-core path within the tolerance wherever both predict the same
  set, and is bitwise reproducible;
* the up projection's tiles are shared out stream-K (each CTA runs an equal run of
  (tile, K chunk) steps; a tile split between CTAs is finished by the last to arrive):
  unions smaller than the grid (one K chunk per CTA, every tile split), and a union of
  50003 rows at d = 128 whose runs hold whole tiles between split ones, both reproducible
  launch after launch (the per-tile counters return to zero), for one and two CTAs per SM
  and one and two K chunks per step; the down projection with one and two 128-column
  tiles per CTA;
* in stream order with other kernels writing its input just before and reading its
  output just after (no host synchronisation), it gives the isolated calls' results
  bitwise;
* the full-size batch configurations (OPT-30B-shaped b = 8, 70B-shaped b = 32) match
  the oracle on every token;
* layers it cannot serve (fp32 weights, d not a multiple of 128) refuse the path.
"""
import numpy as np
import pytest

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import check_token, dev, mask_from_idx

pytestmark = pytest.mark.gpu

SHAPES = [
    ("opt6.7b_relu", 1024, 3001, 128),
    ("70b_reglu", 2048, 5003, 256),
    ("opt30b_relu", 7168, 4099, 1024),
    ("70b_reglu", 8192, 1500, 1024),
]


def run_batch(h, X, path):
    h.set_batch_path(path)
    Y, idx, cnt = h.forward_batch(dev(X), return_sets=True)
    return Y.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("base,d,n,r", SHAPES)
def test_tc_batch_matches_oracle_and_cuda_cores(base, d, n, r):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=41)
    h = sf.SparseFFN.from_layer(lay, max_batch=32)
    for b in (2, 5, 16, 17, 32):
        X = W.make_tokens(cfg, b, seed=42, stream_key=b)
        Yt, idx, cnt = run_batch(h, X, sf.BATCH_TENSOR_CORE)
        Yc, idx_c, cnt_c = run_batch(h, X, sf.BATCH_CUDA_CORE)
        for t in range(b):
            mt = mask_from_idx(idx[t], cnt[t], n)
            mc = mask_from_idx(idx_c[t], cnt_c[t], n)
            check_token(lay, X[t], Yt[t], mt, f"{base} d={d} b={b} t={t}")
            # the two predictors sum in different orders: they may part only where the
            # oracle's logit is within the arbitration band, and agree on y where they agree
            if np.array_equal(mt, mc):
                assert oracle.within_tolerance(Yt[t], Yc[t].astype(np.float64))[0]
        Yt2, _, _ = run_batch(h, X, sf.BATCH_TENSOR_CORE)
        assert np.array_equal(Yt, Yt2)
    assert h.get_error() == 0


@pytest.mark.parametrize("name,b", [("opt30b_relu", 8), ("70b_reglu", 32)])
def test_tc_batch_full_size(name, b):
    cfg = W.CONFIGS[name]
    lay = W.make_layer(cfg, seed=0)
    h = sf.SparseFFN.from_layer(lay, max_batch=b)
    X = W.make_tokens(cfg, b, seed=43)
    Y, idx, cnt = run_batch(h, X, sf.BATCH_TENSOR_CORE)
    for t in range(b):
        check_token(lay, X[t], Y[t], mask_from_idx(idx[t], cnt[t], cfg.n), f"{name} b={b} t={t}")
    assert h.get_error() == 0


@pytest.mark.parametrize("base", ["opt6.7b_relu", "70b_reglu"])
@pytest.mark.parametrize("b", [4, 20])
@pytest.mark.parametrize("shape", [(2, 1, 1), (1, 2, 2)])
def test_tc_batch_runs_of_whole_tiles(base, b, shape):
    # every neuron on: the union is all 50003 rows, 391 tiles of 2 K chunks, more steps
    # than the grid has CTAs
    cfg = W.small_config(W.CONFIGS[base], d=128, n=50003, r=64)
    lay = W.make_layer(cfg, seed=46)
    lay.c = np.full(cfg.n, 1.0e4, dtype=lay.c.dtype)
    h = sf.SparseFFN.from_layer(lay, max_batch=32)
    h.set_batch_tc_shape(*shape)
    X = W.make_tokens(cfg, b, seed=47)
    Y, idx, cnt = run_batch(h, X, sf.BATCH_TENSOR_CORE)
    assert (cnt[:b] == cfg.n).all()
    for t in range(b):
        check_token(lay, X[t], Y[t], mask_from_idx(idx[t], cnt[t], cfg.n), f"{base} b={b} t={t}")
    for _ in range(3):
        assert np.array_equal(run_batch(h, X, sf.BATCH_TENSOR_CORE)[0], Y)
    assert h.get_error() == 0


@pytest.mark.parametrize("base,d,n,r", [SHAPES[1], SHAPES[3], ("opt6.7b_relu", 1152, 2001, 128)])
def test_tc_batch_kernel_shapes(base, d, n, r):
    # up CTAs per SM x K chunks per step x down tiles per CTA: the same sets, y within the
    # tolerance of the oracle (d = 1152: two down tiles per CTA fall back to one)
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=48)
    h = sf.SparseFFN.from_layer(lay, max_batch=32)
    for b in (3, 32):
        X = W.make_tokens(cfg, b, seed=49, stream_key=b)
        for shape in [(1, 1, 1), (2, 1, 2), (1, 2, 1), (2, 2, 2)]:
            h.set_batch_tc_shape(*shape)
            Y, idx, cnt = run_batch(h, X, sf.BATCH_TENSOR_CORE)
            for t in range(b):
                check_token(lay, X[t], Y[t], mask_from_idx(idx[t], cnt[t], n), f"{base} {shape} b={b} t={t}")
            assert np.array_equal(run_batch(h, X, sf.BATCH_TENSOR_CORE)[0], Y)
    for bad in [(3, 1, 1), (1, 4, 1), (1, 1, 3), (0, 1, 1)]:
        with pytest.raises(sf.SfnnError):
            h.set_batch_tc_shape(*bad)
    assert h.get_error() == 0


@pytest.mark.parametrize("base,d,n,r", [SHAPES[1], SHAPES[2]])
def test_tc_batch_in_stream_order_with_other_kernels(base, d, n, r):
    # the chain's kernels start early (dependent launch) and read only weights before their
    # wait: an input written by another kernel just before the call, and an output read by
    # one just after, on the same stream with no host synchronisation, are what isolated
    # calls give, bitwise
    import torch
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=50)
    h = sf.SparseFFN.from_layer(lay, max_batch=32)
    h.set_batch_path(sf.BATCH_TENSOR_CORE)
    bs = [8, 3, 32, 17, 8]
    Xs = [torch.from_numpy(W.make_tokens(cfg, b, seed=60 + i, stream_key=b)).cuda() for i, b in enumerate(bs)]
    ref = []
    for X in Xs:  # isolated
        ref.append(h.forward_batch(X).clone())
        torch.cuda.synchronize()
    s = torch.cuda.Stream()
    xin = torch.empty((32, d), dtype=Xs[0].dtype, device="cuda")
    y = torch.empty((32, d), dtype=torch.float32, device="cuda")
    outs = []
    with torch.cuda.stream(s):
        for X in Xs:
            b = X.shape[0]
            xin[:b].copy_(X * 1.0)  # a kernel writes the input right before the call
            h.forward_batch(xin[:b], y[:b], stream=s)
            outs.append(y[:b] * 1.0)  # and one reads the output right after
    torch.cuda.synchronize()
    for i, (a, e) in enumerate(zip(outs, ref)):
        assert torch.equal(a, e), f"batch {i} (b = {bs[i]})"
    assert h.get_error() == 0


def test_tc_batch_refused_where_it_cannot_run():
    cfg32 = W.small_config(W.CONFIGS["tiny_relu_f32"], d=512, n=2048, r=64)
    h = sf.SparseFFN.from_layer(W.make_layer(cfg32, seed=44), max_batch=4)
    with pytest.raises(sf.SfnnError) as e:
        h.set_batch_path(sf.BATCH_TENSOR_CORE)
    assert e.value.status == 4
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1032, n=1000, r=64)  # d % 128 != 0
    h = sf.SparseFFN.from_layer(W.make_layer(cfg, seed=45), max_batch=4)
    with pytest.raises(sf.SfnnError) as e:
        h.set_batch_path(sf.BATCH_TENSOR_CORE)
    assert e.value.status == 4
    h.set_batch_path(sf.BATCH_CUDA_CORE)
