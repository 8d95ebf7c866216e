"""The allocation-free predictor against the oracle and the handle-based one, on two
calls in a row.

sfnn_predict_noalloc serves callers that cannot call cudaMalloc (graph capture in
progress, pool-owned device memory, no allocation after start-up): it needs no
handle and keeps its scratch in a static device array.  Its set must equal the
oracle's predictor set and sfnn_predict's for the same token, with the rule the
parity tests use: neurons whose oracle logit lies within 1e-3 of the threshold may
go either way.  The Python wrapper is run too, captured in a CUDA graph after a
first eager call, and it refuses buffers too small for the call.  The file is
collected last so that a run stopping at the first failure has run every other
test; it passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import NTHREADS, dev, mask_from_idx

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,shape", [("opt6.7b_relu", None), ("tiny_relu_f32", None),
                                        ("70b_reglu", (1024, 5003, 256))])
def test_noalloc_predictor_matches_handle_predictor(name, shape):
    cfg = W.CONFIGS[name]
    if shape:
        cfg = W.small_config(cfg, d=shape[0], n=shape[1], r=shape[2])
    lay = W.make_layer(cfg, seed=31)
    h = sf.SparseFFN.from_layer(lay)
    A, B, c = dev(lay.A), dev(lay.B), dev(lay.c)
    lib = sf.load_library()
    X = W.make_tokens(cfg, 2, seed=32)
    idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    for t in range(2):  # two calls in a row share the static scratch
        xd = dev(X[t])
        st = lib.sfnn_predict_noalloc(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(A.data_ptr()),
                                      ctypes.c_void_p(B.data_ptr()), ctypes.c_void_p(c.data_ptr()),
                                      cfg.d, cfg.r, cfg.n, sf.F16 if cfg.dtype == "f16" else sf.F32,
                                      ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0
        got = idx.cpu().numpy()
        k = int(cnt.item())
        assert np.all(np.diff(got[:k]) > 0), "indices not ascending"
        m_noalloc = mask_from_idx(got, k, cfg.n)
        _, z_ref, m_ref = oracle.predictor(X[t], lay.A, lay.B, lay.c, NTHREADS)
        _, mism = oracle.arbitrate(z_ref, m_ref, m_noalloc)
        assert mism.size == 0, f"token {t}: sets differ from the oracle's outside the band at {mism[:8]}"
        ref_idx, ref_cnt = h.predict(xd)
        m_handle = mask_from_idx(ref_idx.cpu().numpy(), ref_cnt.item(), cfg.n)
        _, mism = oracle.arbitrate(z_ref, m_handle, m_noalloc)
        assert mism.size == 0, f"token {t}: sets differ from sfnn_predict's outside the band at {mism[:8]}"
        band = int((np.abs(z_ref) < oracle.ARBITRATION_BAND).sum())
        assert abs(k - int(m_ref.sum())) <= band


def test_noalloc_rejects_sizes_beyond_its_scratch():
    d, r, n = 64, 64, 600_000  # the decision mask alone would need 75 KB
    x = torch.zeros(d, dtype=torch.float16, device="cuda")
    A = torch.zeros((d, r), dtype=torch.float16, device="cuda")
    B = torch.zeros((r, 8), dtype=torch.float16, device="cuda")  # never read: the call is refused first
    c = torch.zeros(8, dtype=torch.float16, device="cuda")
    lib = sf.load_library()
    idx = torch.empty(8, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    st = lib.sfnn_predict_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(A.data_ptr()),
                                  ctypes.c_void_p(B.data_ptr()), ctypes.c_void_p(c.data_ptr()), d, r, n, sf.F16,
                                  ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()), None)
    assert st == sf.STATUS_CODES["SFNN_ERR_UNSUPPORTED"]


def test_noalloc_wrapper_captured_in_a_graph():
    """The wrapper's call captured in a CUDA graph (after one eager call, which looks up
    the scratch address) and replayed for two tokens."""
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1024, n=3001, r=128)
    lay = W.make_layer(cfg, seed=33)
    A, B, c = dev(lay.A), dev(lay.B), dev(lay.c)
    X = W.make_tokens(cfg, 3, seed=34)
    xs = dev(X[0])
    idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sf.predict_noalloc(xs, A, B, c, idx, cnt, stream=s)  # eager first call
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sf.predict_noalloc(xs, A, B, c, idx, cnt, stream=s)
    for t in (1, 2):
        xs.copy_(dev(X[t]))
        g.replay()
        torch.cuda.synchronize()
        k = int(cnt.item())
        m = mask_from_idx(idx.cpu().numpy(), k, cfg.n)
        _, z_ref, m_ref = oracle.predictor(X[t], lay.A, lay.B, lay.c, NTHREADS)
        _, mism = oracle.arbitrate(z_ref, m_ref, m)
        assert mism.size == 0, f"replay for token {t}: sets differ at {mism[:8]}"
    del g


def test_noalloc_wrapper_refuses_short_buffers():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=256, n=1000, r=64)
    lay = W.make_layer(cfg, seed=35)
    A, B, c = dev(lay.A), dev(lay.B), dev(lay.c)
    x = dev(W.make_tokens(cfg, 1, seed=36)[0])
    with pytest.raises(ValueError):
        sf.predict_noalloc(x, A, B, c, idx=torch.empty(cfg.n - 1, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError):
        sf.predict_noalloc(x[:-8], A, B, c)
    with pytest.raises(ValueError):
        sf.predict_noalloc(x, A, B, c[:-1])
    with pytest.raises(ValueError):
        sf.predict_noalloc(x, A, B, c, idx=torch.empty(cfg.n, dtype=torch.int64, device="cuda"))
