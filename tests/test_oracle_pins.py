"""The CPU oracle against its pins (no GPU needed)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_out_hw_rejects_malformed(orc):
    import ctypes
    for bad in [dict(C=10, G=3), dict(N=0), dict(H=1, kh=5)]:
        kw = dict(N=1, H=8, W=8, C=8, G=2, kh=3, kw=3)
        kw.update(bad)
        p = orc.problem(kw["N"], kw["H"], kw["W"], kw["C"], kw["G"], kw["kh"], kw["kw"],
                        pad=(0, 0))
        with pytest.raises(ValueError):
            orc.out_hw(p)
    assert orc.lib.orc_out_hw(None, None, None) == -1
    assert ctypes is not None


def test_thread_count_does_not_change_results(orc):
    """The timing knob set_threads: forward, backward and MSDCN forward on one
    thread equal the default run bit for bit (the parallel loops write
    disjoint outputs)."""
    import numpy as np
    rng = np.random.default_rng(5)
    p = orc.problem(3, 7, 9, 16, 2)
    x = rng.standard_normal((3, 7, 9, 16)).astype(np.float32)
    ow = (rng.standard_normal((3, 7, 9, 2, 9, 3)) * 2).astype(np.float32)
    go = rng.standard_normal((3, 7, 9, 16)).astype(np.float32)
    raw = rng.standard_normal((3, 7, 9, 2)).astype(np.float32)
    s0 = np.array([1.0, 2.0], np.float32)
    ref = (orc.forward(p, x, ow), *orc.backward(p, x, ow, go),
           orc.msdcn_forward(p, x, ow, raw, s0, 8.0))
    orc.set_threads(1)
    try:
        got = (orc.forward(p, x, ow), *orc.backward(p, x, ow, go),
               orc.msdcn_forward(p, x, ow, raw, s0, 8.0))
    finally:
        import os
        orc.set_threads(len(os.sched_getaffinity(0)))
    for a, b in zip(ref, got):
        assert np.array_equal(a, b)
