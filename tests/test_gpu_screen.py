"""The large-batch router's screening bound, measured (needs a B200).

Above 256 tokens the router screens with a tensor-core GEMM on a two-term fp16
split of W and keeps every expert whose approximate logit a_e is within
2 eps of the k-th largest; the candidates are then recomputed exactly.  The
picks are exact only if |a_e - l_e| <= eps for the exact fixed-order logits
l_e; the bound carries a safety factor of 2, so the measured error must stay
within eps / 2.  Measured at the prefill chunk size (T = 8192) on the
Flash-Next-shaped layer and on an adversarial layer whose router weights and
token entries span many binades (fp16 subnormals in the split, large
cancellation in the sums).  The worst ratio is printed (run with -s).
"""
import dataclasses

import numpy as np
import pytest

import gen
import oracle
from tests.gpu_util import THREADS, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import quantized_expert_ffn_04_b200 as qe  # noqa: E402


def adversarial(layer, T, seed):
    """Router weights with magnitudes log-uniform over 2^-30 .. 2^2 and token
    entries log-uniform over 2^-20 .. 2^15, random signs."""
    rng = np.random.default_rng(seed)
    E, H = layer.router_w.shape
    W = (2.0 ** rng.uniform(-30, 2, size=(E, H)) * rng.choice([-1.0, 1.0], size=(E, H)))
    x = (2.0 ** rng.uniform(-20, 15, size=(T, H)) * rng.choice([-1.0, 1.0], size=(T, H)))
    lay = dataclasses.replace(layer, router_w=W.astype(np.float32))
    return lay, gen.f32_to_bf16_bits(x.astype(np.float32))


@pytest.mark.parametrize("kind", ["flash2", "adversarial"])
def test_screen_error_within_half_bound(kind):
    shape, T = gen.FLASH2, 8192
    layer = gen.layer_weights(shape, seed=0)
    if kind == "flash2":
        x = gen.hidden(T, shape.hidden, seed=21)
    else:
        layer, x = adversarial(layer, T, seed=22)
    L = qe.Layer(layer, max_tokens=T)
    a = np.empty((T, shape.n_experts), dtype=np.float32)
    eps = np.empty(T, dtype=np.float32)
    qe.strata_moe_debug_screen(L.handle, to_dev_bf16(x).data_ptr(), T, a.ctypes.data,
                               eps.ctypes.data)
    L.close()
    exact = oracle.router_logits(x, layer.router_w, layer.router_b, threads=THREADS)
    cov = eps > 0
    assert cov.mean() > 0.99, f"only {cov.mean():.3f} of the tokens are covered by the bound"
    err = np.abs(a[cov].astype(np.float64) - exact[cov].astype(np.float64))
    ratio = (err / eps[cov, None].astype(np.float64)).max()
    print(f"\nscreen {kind}: worst |a - l| / eps = {ratio:.3e} over {cov.sum()} tokens")
    assert ratio <= 0.5, f"{kind}: screening error {ratio:.3f} eps exceeds eps / 2"
