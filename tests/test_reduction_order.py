"""The shared-set gather and window decode reduce a row group's partial dots
over its lanes with a transposing reduction; the per-head gather uses a
butterfly.  The kernels rely on both giving the same fp32 bits (their outputs
are compared bit for bit on the GPU).  This checks the claim on the host with
float32 arithmetic that follows the two shuffle schedules step by step."""
import numpy as np
import pytest


def butterfly(x):
    """x: [lanes][values] float32; every lane ends with every total."""
    lanes = x.shape[0]
    x = x.copy()
    o = lanes // 2
    while o > 0:
        x = (x + x[np.arange(lanes) ^ o]).astype(np.float32)
        o //= 2
    return x[0]


def transposing(x):
    """Lane l keeps half of its values at each level (the upper half when bit
    o of l is set) and adds its partner's copy; ends with totals l*HV + i."""
    lanes, nv = x.shape
    v = [list(row) for row in x.astype(np.float32)]
    o, half = lanes // 2, nv // 2
    while o > 0:
        new = []
        for l in range(lanes):
            p = l ^ o
            upper = (l & o) != 0
            row = []
            for i in range(half):
                keep = v[l][half + i] if upper else v[l][i]
                # the partner (its bit o the other way) sends its copy of the
                # half this lane keeps
                recv = v[p][half + i] if upper else v[p][i]
                row.append(np.float32(keep + recv))
            new.append(row)
        v = new
        o //= 2
        half //= 2
    hv = nv // lanes
    out = np.zeros(nv, np.float32)
    for l in range(lanes):
        for i in range(hv):
            out[l * hv + i] = v[l][i]
    return out


@pytest.mark.parametrize("lanes,nv", [(16, 16), (8, 16), (8, 8)])
def test_transposing_reduction_gives_the_butterfly_bits(lanes, nv):
    rng = np.random.default_rng(lanes * 100 + nv)
    for _ in range(200):
        x = (rng.standard_normal((lanes, nv)) * rng.choice([1e-3, 1.0, 1e3])).astype(np.float32)
        assert np.array_equal(butterfly(x).view(np.uint32), transposing(x).view(np.uint32))
