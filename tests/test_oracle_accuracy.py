"""End-to-end accuracy of the quantized linear against the exact product
(information only: the pages give no worked example or error bound, so this
is not a parity pin).  It reports the relative Frobenius error of
Y = dequant(Q(X P) Q(P^-1 W^T)) against X W^T in float64, with and without the
Kronecker transform, on activations with two x50 outlier channels, and checks
the premise the transform is there for: it lowers the error."""
import numpy as np

from int4_linear_b200 import synth
from oracle import fq_oracle as O


def _rel_err(d, transform):
    x, w = d["x"], d["w"]
    y_ref = x.astype(np.float64) @ w.astype(np.float64).T
    if transform:
        qw, sw, _ = O.quant_weight(w, O.ROW, 1.0, d["p1_inv"], d["p2_inv"])
        y = O.linear(x, qw, sw, O.ROW, 1.0, d["p1"], d["p2"])
    else:
        qw, sw, _ = O.quant_weight(w, O.ROW, 1.0)
        y = O.linear(x, qw, sw, O.ROW, 1.0)
    y = np.asarray(y, np.float64)
    return float(np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref))


def test_transform_lowers_the_quantization_error():
    d = synth.prefill_linear(4096, 256, m=64, seed=3)
    e_plain = _rel_err(d, False)
    e_kron = _rel_err(d, True)
    print(f"relative Frobenius error, W4A4 per-token x per-channel, M=64 K=4096 N=256: "
          f"no transform {e_plain:.4f}, Kronecker (64, 64) {e_kron:.4f}")
    assert np.isfinite(e_plain) and np.isfinite(e_kron)
    assert e_kron < e_plain
