"""Degenerate cases of the method on every path (fused single token, fused few-token,
tensor-core and CUDA-core batches, residual stack):

* a predictor that switches every neuron off: empty sets, y exactly zero, and the
  stack's output exactly its input;
* a predictor that switches every neuron on: the dense FFN;
* fewer neurons than SMs (n = 37 and n = 1: tiles of one neuron, empty tiles of work);
* the smallest d the fp16 layout allows (d = 16, r = 8) and a tensor-core layer with
  a single 128-column tile (d = 128);
* a layer larger than the device's memory: sfnn_create returns SFNN_ERR_OOM (its
  first allocation fails before any input is read) and the context stays usable.
"""
import ctypes

import numpy as np
import pytest
import torch

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import NTHREADS, check_token, dev, fused_step, mask_from_idx

pytestmark = pytest.mark.gpu


def layer(base, d, n, r, seed, c_value=None):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=seed)
    if c_value is not None:
        lay.c = np.full(cfg.n, c_value, dtype=lay.c.dtype)
    return cfg, lay


def all_paths(cfg, lay, X, max_batch=4):
    """{path: (y of every token, the sets that path used)} for the fused path and both
    batch paths (each batch path reports its own predictor's sets)."""
    h = sf.SparseFFN.from_layer(lay, max_batch=max_batch)
    ys, sets = [], []
    for x in X:  # the fused kernel, with the set it used
        y, m = fused_step(h, dev(x))
        ys.append(y)
        sets.append(m)
    out = {"fused": (np.stack(ys), sets)}
    for name, path in (("cuda-core", sf.BATCH_CUDA_CORE), ("tensor-core", sf.BATCH_TENSOR_CORE),
                       ("fused-multi", sf.BATCH_FUSED)):
        try:
            h.set_batch_path(path)
        except sf.SfnnError:
            continue
        Y, idx, cnt = h.forward_batch(dev(X), return_sets=True)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        out[name] = (Y.cpu().numpy(), [mask_from_idx(idx[t], cnt[t], cfg.n) for t in range(len(X))])
    assert h.get_error() == 0
    return out


@pytest.mark.parametrize("base", ["opt6.7b_relu", "70b_reglu"])
def test_all_neurons_off(base):
    cfg, lay = layer(base, 1024, 3001, 128, seed=61, c_value=-1.0e4)
    X = W.make_tokens(cfg, 3, seed=62)
    out = all_paths(cfg, lay, X)
    for name, (Y, sets) in out.items():
        assert all(m.sum() == 0 for m in sets), name
        assert not Y.any(), name
    lays = [lay, layer(base, 1024, 3001, 128, seed=63, c_value=-1.0e4)[1]]
    hs = [sf.SparseFFN.from_layer(l) for l in lays]
    x0 = X[0].astype(np.float32)
    xl = sf.forward_stack(hs, dev(x0)).cpu().numpy()
    assert np.array_equal(xl, x0)


@pytest.mark.parametrize("base", ["opt6.7b_relu", "70b_reglu"])
def test_all_neurons_on(base):
    cfg, lay = layer(base, 1024, 3001, 128, seed=64, c_value=1.0e4)
    X = W.make_tokens(cfg, 3, seed=65)
    out = all_paths(cfg, lay, X)
    for t in range(3):
        dense = oracle.ffn_masked(X[t], lay.w_up, lay.w_gate, lay.b, lay.w_down, np.ones(cfg.n, np.uint8),
                                  lay.cfg.act, NTHREADS)[1]
        for name, (Y, sets) in out.items():
            assert sets[t].sum() == cfg.n, name
            assert oracle.within_tolerance(Y[t], dense)[0], name


@pytest.mark.parametrize("base,d,n,r", [
    ("opt6.7b_relu", 1024, 37, 64),
    ("70b_reglu", 1024, 1, 64),
    ("opt6.7b_relu", 16, 300, 8),
    ("70b_reglu", 128, 700, 64),
])
def test_small_shapes(base, d, n, r):
    cfg, lay = layer(base, d, n, r, seed=66)
    X = W.make_tokens(cfg, 4, seed=67)
    out = all_paths(cfg, lay, X)
    for name, (Y, sets) in out.items():
        for t in range(4):
            check_token(lay, X[t], Y[t], sets[t], f"{name} d={d} n={n} t={t}")


def test_layer_beyond_device_memory_is_oom():
    # fp16 ReLU rows of d = 65536, n = 2^20 need 2 * 2^20 * 65536 * 2 bytes = 256 GiB;
    # the library allocates before it reads any input, so small stand-ins suffice
    lib = sf.load_library()
    tiny = torch.zeros(64, dtype=torch.float16, device="cuda")
    p = tiny.data_ptr()
    desc = sf.LayerDesc(65536, 1 << 20, 8, 1, sf.RELU, sf.F16, p, None, p, p, p, p, p, None, 0)
    hdl = ctypes.c_void_p()
    st = lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(hdl))
    assert st == sf.STATUS_CODES["SFNN_ERR_OOM"] and not hdl.value
    cfg, lay = layer("opt6.7b_relu", 256, 700, 64, seed=90)  # the device still serves a layer
    h = sf.SparseFFN.from_layer(lay)
    x = W.make_tokens(cfg, 1, seed=91)[0]
    y, m = fused_step(h, dev(x))
    check_token(lay, x, y, m, "after a failed create")
