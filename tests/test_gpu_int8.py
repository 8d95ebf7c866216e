"""Weight-only int8 and int4 rows (the FFN's up, gate and down rows as codes with one
fp32 scale per neuron and projection; the predictor, biases, x and all arithmetic
unchanged).

* the library's quantization follows the oracle's rule (fp32 scale = absmax / qmax,
  qmax 127 or 7, codes rounded to nearest even): every token agrees with the oracle's
  quantized step (sets exact outside the arbitration band, y within the tolerance) for
  ReLU and ReGLU, d up to 8192, ragged n, and the full OPT-6.7B- and 70B-shaped layers;
* results are bitwise reproducible; the rows cost a half (int8) or a quarter (int4) of
  the bytes of fp16 rows;
* only the fused single-token path serves such a layer (also at b = 1 through
  forward_batch, which returns the set the kernel used: that set is the one checked);
  batches, explicit sets and the multi-kernel path are refused with
  SFNN_ERR_UNSUPPORTED, the predictor works.
"""
import numpy as np
import pytest

import activation_sparse_ffn_threshold_b200 as sf
import oracle
import workload as W
from parity_util import NTHREADS, REL_TOL, dev, fused_step

pytestmark = pytest.mark.gpu


def check_token_q(lay, qr, x, y_gpu, mask_gpu, what=""):
    ref = oracle.forward_q(lay, qr, x, NTHREADS)
    use, mism = oracle.arbitrate(ref.z, ref.mask, mask_gpu)
    assert mism.size == 0, f"{what}: sets differ outside the arbitration band at {mism[:10]}"
    y_ref = ref.y if np.array_equal(use, ref.mask) else oracle.forward_q_with_mask(lay, qr, x, use, NTHREADS)
    ok, ratio = oracle.within_tolerance(y_gpu, y_ref, REL_TOL)
    assert ok, f"{what}: max|dy|/max|y_ref| = {ratio:.3e} > {REL_TOL}"


BITS = {"int8": 8, "int4": 4}


def run_tokens(cfg, lay, h, count, seed, rows):
    qr = oracle.quantize_layer(lay, bits=BITS[rows])
    X = W.make_tokens(cfg, count, seed=seed)
    for t in range(count):
        xd = dev(X[t])
        y, m = fused_step(h, xd)
        check_token_q(lay, qr, X[t], y, m, f"{cfg.name} t={t}")
        assert np.array_equal(h.forward(xd).cpu().numpy(), y)


@pytest.mark.parametrize("rows", ["int8", "int4"])
@pytest.mark.parametrize("base,d,n,r", [
    ("opt6.7b_relu", 1024, 3001, 128),
    ("70b_reglu", 2048, 5003, 256),
    ("opt30b_relu", 7168, 4099, 1024),
    ("70b_reglu", 8192, 1500, 1024),
])
def test_quantized_rows_match_oracle(base, d, n, r, rows):
    cfg = W.small_config(W.CONFIGS[base], d=d, n=n, r=r)
    lay = W.make_layer(cfg, seed=51)
    h = sf.SparseFFN.from_layer(lay, rows=rows)
    run_tokens(cfg, lay, h, 4, seed=52, rows=rows)
    assert h.get_error() == 0


@pytest.mark.parametrize("rows", ["int8", "int4"])
@pytest.mark.parametrize("name", ["opt6.7b_relu", "70b_reglu"])
def test_quantized_rows_full_size(name, rows):
    cfg = W.CONFIGS[name]
    lay = W.make_layer(cfg, seed=0)
    h = sf.SparseFFN.from_layer(lay, rows=rows)
    run_tokens(cfg, lay, h, 2, seed=53, rows=rows)
    h16 = sf.SparseFFN.from_layer(lay)
    iq, i16 = h.info(), h16.info()
    share = 0.51 if rows == "int8" else 0.26
    assert iq["row_bytes_per_neuron"] < share * i16["row_bytes_per_neuron"]


@pytest.mark.parametrize("rows", ["int8", "int4"])
def test_quantized_rows_refuse_other_paths(rows):
    cfg = W.small_config(W.CONFIGS["opt6.7b_relu"], d=1024, n=3001, r=128)
    lay = W.make_layer(cfg, seed=54)
    h = sf.SparseFFN.from_layer(lay, rows=rows, max_batch=4)
    X = W.make_tokens(cfg, 2, seed=55)
    with pytest.raises(sf.SfnnError) as e:
        h.forward_batch(dev(X))
    assert e.value.status == 4
    idx, cnt = h.predict(dev(X[0]))
    with pytest.raises(sf.SfnnError) as e:
        h.forward(dev(X[0]), idx=idx[:cnt.item()])
    assert e.value.status == 4
    with pytest.raises(sf.SfnnError) as e:
        h.set_fused_decode(False)
    assert e.value.status == 4
    assert h.forward(dev(X[0])).shape[0] == cfg.d
    assert h.get_error() == 0
