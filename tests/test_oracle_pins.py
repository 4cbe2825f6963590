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
