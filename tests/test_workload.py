"""The synthetic workloads reproduce the statistics the pages and the workload definitions fix.

* power law: the hottest 26% (OPT-30B shape) / 43% (70B ReGLU shape) of the
  neurons carry 80% of the expected activations (hexiedandong.com PowerInfer
  news page, the paragraph on figure (a));
* OPT-6.7B shape: mean activation 0.10, i.e. about 90% activation sparsity
  (53ai.com page, section "激活稀疏的可行性", ReLU sparsity above 90%);
* the realised activation frequency of the FFN and of the calibrated predictor
  match the configured mean; the union of b tokens' predicted sets matches
  E|U|/n = mean_i 1-(1-p_i)^b (why sparsity decays with batch size: 53ai.com
  page, section "工程效果");
* generation is deterministic and independent of the thread count.
"""
import numpy as np
import pytest

import oracle
import workload as W


@pytest.mark.parametrize("name", W.CONFIG_ORDER)
def test_profile_mean_and_clip(name):
    cfg = W.CONFIGS[name]
    p = W.zipf_profile(cfg.n, W.config_alpha(cfg), cfg.mean_p, cfg.p_max)
    assert abs(p.mean() - cfg.mean_p) < 1e-9
    assert p.max() <= cfg.p_max and np.all(np.diff(p) <= 0)


def test_power_law_shares():
    c4, c5 = W.CONFIGS["opt30b_relu"], W.CONFIGS["70b_reglu"]
    p4 = W.zipf_profile(c4.n, W.config_alpha(c4), c4.mean_p)
    p5 = W.zipf_profile(c5.n, W.config_alpha(c5), c5.mean_p)
    assert abs(W.top_share(p4, 0.26) - 0.80) < 0.01
    assert abs(W.top_share(p5, 0.43) - 0.80) < 0.01
    assert abs(W.config_alpha(c4) - 1.253) < 0.01
    assert abs(W.config_alpha(c5) - 0.931) < 0.01


def test_union_density_closed_form_values():
    c4 = W.CONFIGS["opt30b_relu"]
    p4 = W.zipf_profile(c4.n, W.config_alpha(c4), c4.mean_p)
    got = [W.expected_union_density(p4, b) for b in (1, 2, 4, 8)]
    assert np.allclose(got, [0.1, 0.151, 0.227, 0.338], atol=2e-3)


def test_realised_activation_and_prediction_rates():
    cfg = W.CONFIGS["tiny_relu_f32"]
    L = W.make_layer(cfg, seed=0)
    X = W.make_tokens(cfg, 64, seed=0)
    act = np.zeros(cfg.n)
    pred = np.zeros(cfg.n)
    for t in range(64):
        g = oracle.preact(X[t], L.w_up, None, L.b, "relu", nthreads=4)
        act += g > 0
        _, _, m = oracle.predictor(X[t], L.A, L.B, L.c, nthreads=4)
        pred += m
    act /= 64
    pred /= 64
    assert abs(act.mean() - cfg.mean_p) < 0.01
    assert abs(pred.mean() - cfg.mean_p) < 0.02
    # the predictor's per-neuron frequency follows the hotness profile
    assert np.corrcoef(pred, L.p)[0, 1] > 0.9


def test_union_density_of_predicted_sets():
    cfg = W.CONFIGS["tiny_relu_f32"]
    L = W.make_layer(cfg, seed=0)
    X = W.make_tokens(cfg, 64, seed=0, stream_key=5)
    masks = np.array([oracle.predictor(X[t], L.A, L.B, L.c, nthreads=4)[2] for t in range(64)], bool)
    for b in (2, 4, 8):
        u = np.mean([masks[i:i + b].any(axis=0).mean() for i in range(0, 64, b)])
        assert abs(u - W.expected_union_density(L.p, b)) < 0.03, b


def test_generation_is_deterministic_and_thread_independent(monkeypatch):
    cfg = W.small_config(W.CONFIGS["70b_reglu"], d=1024, n=4096, r=64)
    L1 = W.make_layer(cfg, seed=3)
    monkeypatch.setattr(W, "_POOL_THREADS", 1)
    L2 = W.make_layer(cfg, seed=3)
    for k in ("w_up", "w_gate", "w_down", "b", "A", "B", "c"):
        assert np.array_equal(getattr(L1, k), getattr(L2, k)), k
    assert L1.w_up.dtype == np.float16 and L1.w_up.shape == (4096, 1024)
    assert L1.w_down.shape == (1024, 4096) and L1.A.shape == (1024, 64) and L1.B.shape == (64, 4096)
    L3 = W.make_layer(cfg, seed=4)
    assert not np.array_equal(L1.w_up, L3.w_up)


def test_weight_scales():
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=2048, n=1024, r=256)
    L = W.make_layer(cfg, seed=0)
    assert abs(L.w_up.astype(np.float64).std() * np.sqrt(cfg.d) - 1) < 0.01
    assert abs(L.B.astype(np.float64).std() * np.sqrt(cfg.r) - 1) < 0.01
    X = W.make_tokens(cfg, 8)
    assert abs(X.astype(np.float64).std() - 1) < 0.02
