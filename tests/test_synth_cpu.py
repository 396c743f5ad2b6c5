"""The seeded input generator gives the distributions its workloads are named for, as
the oracle measures them: the sweep's weight mixtures give 30%, 50% and 70% zero codes
under absmean ternarisation, and the activation generator scales the stated number of
outlier channels."""
import numpy as np
import pytest

import oracle
from ternary_weight_bit_absmean_b200 import synth

pytestmark = pytest.mark.cpu


@pytest.mark.parametrize("zeros", sorted(synth.SWEEP_SMALL_FRAC))
def test_sweep_mixture_zero_share(orc, zeros):
    W = synth.weight(1024, 1024, seed=zeros, small_frac=synth.SWEEP_SMALL_FRAC[zeros])
    _, codes, _ = orc.quantize_weights(W.numpy(), 1e-5)
    assert abs(float(np.mean(codes == 0)) - zeros / 100.0) < 0.015  # a plain Gaussian gives ~31%


@pytest.mark.parametrize("frac", synth.SWEEP_OUTLIER_FRACS)
def test_outlier_channel_count(frac):
    K = 4096
    X = synth.activations(64, K, seed=3, outlier_frac=frac, outlier_scale=synth.SWEEP_OUTLIER_SCALE).float()
    # outlier channels have a column RMS near the scale; the others near 1
    rms = X.pow(2).mean(0).sqrt().numpy()
    assert int((rms > 10).sum()) == max(1, int(round(frac * K)))
