"""How often the lazy rescale fires on the benchmark inputs.

The forward kernel moves its running maximum only when a 64-key tile's maximum exceeds it
by more than 8 in log2 units (the rescaling rule of the page "FlashAttention 4:
Praxisleitfaden ...", section "Intelligenteres Online-Softmax-Rescaling in FA4"), and only
then rescales the accumulator.  This test applies the same rule, in fp32 like the kernel's
scores, to sampled query rows of the workloads and reports the fraction of tiles after
the first that trigger a rescale.  The result is exact for any threshold (the pins of
the tiled restatement show that); the rate measures how much work the rule saves.
"""
import numpy as np
import pytest
import torch

from workloads import WORKLOADS, make_inputs

THRESHOLD = 8.0
BN = 64


def rescale_rate(name, rows=128, heads=2, seed=0):
    w = WORKLOADS[name]
    inp = make_inputs(w, Hq=heads, Hkv=heads)
    rng = np.random.default_rng(seed)
    c = np.float32(w.scale * np.log2(np.e))
    fired = tiles = 0
    for h in range(heads):
        k = inp.k[0, h].float().numpy()
        for i in rng.integers(0, w.N, size=rows // heads):
            x = (k @ inp.q[0, h, i].float().numpy()) * c          # fp32 scores, log2 domain
            nkeys = i + 1 if w.causal else w.N
            m = -np.inf
            for j0 in range(0, nkeys, BN):
                xm = float(x[j0:min(j0 + BN, nkeys)].max())
                if xm > m + THRESHOLD:
                    if j0 > 0:
                        fired += 1
                    m = xm
                if j0 > 0:
                    tiles += 1
    return fired / max(tiles, 1), tiles


@pytest.mark.parametrize("name", ["long", "long_causal", "gpt2"])
def test_lazy_rescale_is_rare_on_the_benchmark_inputs(name):
    rate, tiles = rescale_rate(name)
    print("%s: rescales after the first tile: %.4f%% of %d tiles" % (name, 100 * rate, tiles))
    assert tiles > 0 and rate < 0.01
