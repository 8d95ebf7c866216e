"""GPU parity: the CUDA library against the CPU oracle, through the C ABI.

* the hand-derived worked example (PowerInfer's single-layer sets) bit-exact;
* integer-exact layers (small integers, half-integer biases): fp16/fp32 inputs
  with fp32 accumulation are exact, so sets and y must equal the oracle
  bit-for-bit whatever the summation order -- this pins the kernels' indexing
  across several tiles and a ragged tail of neurons;
* explicit sets: the exact active set and the all-ones set reproduce the dense
  FFN, the empty set gives exact zeros, duplicates count once, out-of-range
  indices latch an error;
* reduced shapes with ragged n, and determinism and hotness-order invariance.
"""
import json
import os

import numpy as np
import pytest
import torch

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import L, NTHREADS, check_token, dev, fused_step, mask_from_idx

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "powerinfer_example.json")


def _pad(a, rows=None, cols=None):
    a = np.asarray(a, np.float64)
    if a.ndim == 1:
        return np.pad(a, (0, (rows or a.shape[0]) - a.shape[0]))
    return np.pad(a, ((0, (rows or a.shape[0]) - a.shape[0]), (0, (cols or a.shape[1]) - a.shape[1])))


def _golden_layers(dtype):
    """The worked example padded with zeros to the kernels' vector width (an identical layer)."""
    g = json.load(open(GOLDEN))
    d = 8 if dtype == np.float16 else 4
    r = 8 if dtype == np.float16 else 4
    f = lambda a: np.ascontiguousarray(a, dtype=dtype)
    A = f(_pad(g["A_dxr"], d, r))
    B = f(_pad(g["B_rxn"], r, 8))
    relu = L("relu", f(_pad(g["W_relu_nxd"], 8, d)), None, f(g["b"]), f(_pad(g["W_down_dxn"], d, 8)), A, B,
             f(g["c"]), np.array(g["hotness"]))
    reglu = L("reglu", f(_pad(g["W_up_reglu_nxd"], 8, d)), f(_pad(g["W_relu_nxd"], 8, d)), f(g["b"]),
              f(_pad(g["W_down_dxn"], d, 8)), A, B, f(g["c"]), np.array(g["hotness"]))
    x = f(_pad(g["x"], d))
    return g, relu, reglu, x, d


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
@pytest.mark.parametrize("use_hot", [False, True])
def test_golden_example(dtype, use_hot):
    g, relu, reglu, x, d = _golden_layers(dtype)
    e = g["expected"]
    h = sf.SparseFFN.from_layer(relu, use_hotness=use_hot)
    idx, cnt = h.predict(dev(x))
    k = int(cnt.item())
    assert sorted(idx[:k].cpu().tolist()) == e["predicted_set"] == [3, 4, 5]
    y = h.forward(dev(x)).cpu().numpy()
    assert y[:4].tolist() == e["relu_y"] and not y[4:].any()
    h2 = sf.SparseFFN.from_layer(reglu, use_hotness=use_hot)
    y2 = h2.forward(dev(x)).cpu().numpy()
    assert y2[:4].tolist() == e["reglu_y"]
    # two copies of the ReLU layer as a residual stack
    X0 = torch.zeros(d, dtype=torch.float32, device="cuda")
    X0[:4] = torch.tensor(g["x"], dtype=torch.float32)
    XL, sidx, scnt = sf.forward_stack([h, h], X0, return_sets=True)
    assert XL[:4].cpu().tolist() == e["stack2_relu"]["x_out"]
    sets = [sorted(sidx[l, 0, :int(scnt[l, 0])].cpu().tolist()) for l in range(2)]
    assert sets == e["stack2_relu"]["sets"]
    assert h.get_error() == 0


def _integer_layer(rng, d, n, r, act, dtype, density=0.05):
    def tern(shape, p):
        v = rng.choice([-1.0, 1.0], size=shape) * (rng.random(shape) < p)
        return v.astype(dtype)
    w_up = tern((n, d), density)
    w_gate = tern((n, d), density) if act == "reglu" else None
    b = (rng.integers(-3, 3, n) + 0.5).astype(dtype)
    w_down = tern((d, n), density)
    A = tern((d, r), 0.1)
    B = tern((r, n), 0.3)
    c = (rng.integers(-12, 2, n) - 0.5).astype(dtype)
    return L(act, w_up, w_gate, b, w_down, A, B, c, rng.random(n))


@pytest.mark.parametrize("act", ["relu", "reglu"])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_integer_exact_bitwise(act, dtype):
    rng = np.random.default_rng(21)
    d, n, r = 512, 2085, 64  # n: 65 words of 32 neurons with a ragged last word
    lay = _integer_layer(rng, d, n, r, act, dtype)
    h = sf.SparseFFN.from_layer(lay, max_batch=5)
    X = rng.integers(-2, 3, (5, d)).astype(dtype)
    for t in range(5):
        ref = oracle.forward(lay, X[t], NTHREADS)
        assert 0.02 * n < ref.mask.sum() < 0.8 * n
        idx, cnt = h.predict(dev(X[t]))
        m = mask_from_idx(idx.cpu().numpy(), cnt.item(), n)
        assert np.array_equal(m, ref.mask)
        y = h.forward(dev(X[t])).cpu().numpy().astype(np.float64)
        assert np.array_equal(y, ref.y)
    Y, bidx, bcnt = h.forward_batch(dev(X), return_sets=True)
    Y = Y.cpu().numpy()
    for t in range(5):
        ref = oracle.forward(lay, X[t], NTHREADS)
        assert np.array_equal(mask_from_idx(bidx[t].cpu().numpy(), bcnt[t].item(), n), ref.mask)
        assert np.array_equal(Y[t].astype(np.float64), ref.y)


@pytest.fixture(scope="module")
def small_layer():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1024, n=3000, r=128)
    return cfg, W.make_layer(cfg, seed=5)


def test_explicit_sets(small_layer):
    cfg, lay = small_layer
    h = sf.SparseFFN.from_layer(lay)
    x = W.make_tokens(cfg, 1, seed=5)[0]
    xd = dev(x)
    g = oracle.preact(x, lay.w_up, None, lay.b, "relu", NTHREADS)
    s_star = np.flatnonzero(g > 0).astype(np.int32)
    dense = oracle.ffn_masked(x, lay.w_up, None, lay.b, lay.w_down, np.ones(cfg.n, np.uint8), "relu")[1]
    # exact set == dense
    y = h.forward(xd, idx=dev(s_star)).cpu().numpy()
    assert oracle.within_tolerance(y, dense)[0]
    # all-ones == dense
    y1 = h.forward(xd, idx=dev(np.arange(cfg.n, dtype=np.int32))).cpu().numpy()
    assert oracle.within_tolerance(y1, dense)[0]
    # shuffled with duplicates == the set
    rng = np.random.default_rng(0)
    dup = np.concatenate([s_star, s_star[: len(s_star) // 2]])
    rng.shuffle(dup)
    y2 = h.forward(xd, idx=dev(dup)).cpu().numpy()
    assert np.array_equal(y2, y)
    # empty set: exact zeros
    y0 = h.forward(xd, idx=dev(np.zeros(4, np.int32)), count=dev(np.zeros(1, np.int32))).cpu().numpy()
    assert not y0.any()
    assert h.get_error() == 0
    # out-of-range entries are skipped and latched
    bad = np.concatenate([s_star, np.array([-1, cfg.n, 10 ** 6], np.int32)])
    y3 = h.forward(xd, idx=dev(bad)).cpu().numpy()
    assert np.array_equal(y3, y)
    assert h.get_error() == 1  # SFNN_ERR_INVALID_ARG latched on the device
    assert h.get_error() == 0  # and cleared by the read


def test_reduced_shapes_parity(small_layer):
    cfg, lay = small_layer
    h = sf.SparseFFN.from_layer(lay)
    X = W.make_tokens(cfg, 16, seed=6)
    for t in range(16):
        idx, cnt = h.predict(dev(X[t]))
        m = mask_from_idx(idx.cpu().numpy(), cnt.item(), cfg.n)
        y = h.forward(dev(X[t])).cpu().numpy()
        check_token(lay, X[t], y, m, f"token {t}")


def test_determinism_and_hotness_invariance(small_layer):
    """The storage order (hotness dealt to the tiles, hot-packed-first, or the original
    order without a profile) changes no set and y only within rounding, on the fused
    single-token kernel, the few-token kernel and the tensor-core batch path."""
    cfg, lay = small_layer
    hs = {"dealt": sf.SparseFFN.from_layer(lay, use_hotness=True, max_batch=4),
          "packed": sf.SparseFFN.from_layer(lay, use_hotness=True, max_batch=4, order="packed"),
          "identity": sf.SparseFFN.from_layer(lay, use_hotness=False, max_batch=4)}
    X = W.make_tokens(cfg, 4, seed=7)
    for t in range(4):
        xd = dev(X[t])
        a = hs["dealt"].forward(xd).cpu().numpy()
        assert np.array_equal(a, hs["dealt"].forward(xd).cpu().numpy())
        sets = {}
        for name, h in hs.items():
            y, m = fused_step(h, xd)
            assert oracle.within_tolerance(y, a.astype(np.float64))[0], name
            check_token(lay, X[t], y, m, f"{name} t={t}")
            sets[name] = m
        assert np.array_equal(sets["dealt"], sets["packed"]) and np.array_equal(sets["dealt"], sets["identity"])
    for path in (sf.BATCH_FUSED, sf.BATCH_TENSOR_CORE):
        Ys = {}
        for name, h in hs.items():
            try:
                h.set_batch_path(path)
            except sf.SfnnError:  # a layer this path cannot serve
                continue
            Y, idx, cnt = h.forward_batch(dev(X), return_sets=True)
            Ys[name] = Y.cpu().numpy()
            for t in range(4):
                check_token(lay, X[t], Ys[name][t], mask_from_idx(idx[t].cpu().numpy(), cnt[t].item(), cfg.n),
                            f"{name} path {path} t={t}")
        for name in Ys:
            assert oracle.within_tolerance(Ys[name], Ys["dealt"].astype(np.float64))[0]


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_reduced_batch_rows_match_single(act):
    base = W.CONFIGS["70b_reglu" if act == "reglu" else "opt30b_relu"]
    cfg = W.small_config(base, d=1024, n=4000, r=128)
    lay = W.make_layer(cfg, seed=8)
    h = sf.SparseFFN.from_layer(lay, max_batch=32)
    for b in (2, 7, 32):
        X = W.make_tokens(cfg, b, seed=9, stream_key=b)
        Y, idx, cnt = h.forward_batch(dev(X), return_sets=True)
        Y = Y.cpu().numpy()
        idx = idx.cpu().numpy()
        for t in range(b):
            m = mask_from_idx(idx[t], cnt[t].item(), cfg.n)
            check_token(lay, X[t], Y[t], m, f"b={b} t={t}")
            ys = h.forward(dev(X[t])).cpu().numpy()
            assert oracle.within_tolerance(Y[t], ys.astype(np.float64))[0]


def test_misaligned_input_is_rejected(small_layer):
    cfg, lay = small_layer
    h = sf.SparseFFN.from_layer(lay, max_batch=2)
    buf = torch.zeros(cfg.d + 8, dtype=torch.float16, device="cuda")
    x_bad = buf[1:1 + cfg.d]  # 2-byte offset
    with pytest.raises(sf.SfnnError) as e:
        h.forward(x_bad)
    assert e.value.status == 1
    with pytest.raises(sf.SfnnError):
        h.predict(x_bad)
    X = torch.zeros(2 * cfg.d + 8, dtype=torch.float16, device="cuda")[4:4 + 2 * cfg.d].view(2, cfg.d)
    with pytest.raises(sf.SfnnError):
        h.forward_batch(X)
    assert h.get_error() == 0
