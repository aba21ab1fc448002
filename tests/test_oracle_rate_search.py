"""The oracle's exact-rate step search (Methodology step 3: the realised rate lands about 0.01 bps
from any target).  Pins: on Gaussian RHT input the search ends within 0.005 bps of every target
it can reach, from a good and from a far first probe; an unreachable target ends at the step
range's end with the probe closest to it; the bracket result against a brute-force scan of the rate
over a grid of steps."""
import numpy as np
import pytest

import oracle
from post_quantization_tile_b200 import workloads as W


@pytest.mark.parametrize("lattice,n,target", [(oracle.E8, 128, 2.0), (oracle.E8, 128, 4.0), (oracle.E8, 64, 5.5),
                                              (oracle.D4, 128, 3.0), (oracle.A2, 256, 4.0), (oracle.Z, 128, 1.5)])
def test_search_lands_within_tolerance(lattice, n, target):
    x = W.gaussian_bf16(64, 1024, seed=21)
    N = x.size
    for step0 in (0.3, 2.0 ** -8):   # a first probe near the answer, and one at the range's end
        step, probes, bits = oracle.step_search(x, n, lattice, target, seed=5, step0=step0)
        assert abs(bits / N - target) <= 0.005 + 1e-12, (step0, bits / N)
        assert probes <= 16
        # the reported bits are the payload of encoding at the reported step
        assert oracle.encode(x, n, lattice, step, 5).payload_bits() == bits


def test_unreachable_target_ends_at_the_range_end():
    x = np.zeros((32, 256), dtype=np.uint16)    # zero tiles: k = 0, one bit per scalar at any step
    step, probes, bits = oracle.step_search(x, 128, oracle.D4, 4.0, step0=0.25)
    assert bits == x.size                       # 1 bps whatever the step
    assert step == np.float32(0.25)             # every probe is equally far: the first is kept
    assert probes <= 3


def test_search_is_at_least_as_close_as_a_grid_scan():
    # the rate is not monotone in the step (the Rice parameter k switches in steps), so the scan
    # looks at every grid point: the search must land at least as close to the target as the
    # best of 81 steps spread over the same range, with far fewer encodes
    x = W.gaussian_bf16(32, 512, seed=4)
    N = x.size
    grid = np.float32(2.0) ** np.linspace(-4, 1, 81).astype(np.float32)
    rates = np.array([oracle.encode(x, 128, oracle.E8, float(b), 1).payload_bits() / N for b in grid])
    assert np.max(np.diff(rates)) > 0           # the sawtooth is real
    for target in (2.2, 3.3, 4.4):
        step, probes, bits = oracle.step_search(x, 128, oracle.E8, target, seed=1, step0=0.5)
        assert abs(bits / N - target) <= max(0.005, np.min(np.abs(rates - target)))
        assert probes < 12
