"""The host oracle against what the pages and mathematics fix (CPU only)."""
import pytest

import oracle as O
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O.load())


def test_thread_count_independent():
    """Each output sums in k order on one thread: 1 thread and all threads agree."""
    import torch
    from group_wise_affine_dequant_b200 import workloads as W
    w, x = W.tiny_inputs()
    lib = O.load()
    c, s, b = O.quantize_affine(w, 64, 4)
    n0 = O.threads()
    try:
        O.set_threads(1)
        y1, a1 = O.qmm(x, c, s, b, 64, 4)
        c1, _, _ = O.quantize_affine(w, 64, 4)
    finally:
        O.set_threads(n0)
    y2, a2 = O.qmm(x, c, s, b, 64, 4)
    assert torch.equal(y1, y2) and torch.equal(a1, a2) and torch.equal(c1, c)
    assert lib is O.load()
