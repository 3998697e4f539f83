"""Host-side logic of the binding that needs no GPU: the slice count of the
host pipeline (moe.choose_chunks)."""
import pytest

from dropless_top_mixture_b200.workloads import WORKLOADS


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _args(name):
    w = WORKLOADS[name]
    es = 4 if w.dtype == "f32" else 2
    return w.T, w.d, es, 3 * w.E * w.F * w.d * (1 if w.mxfp8 else es)


@pytest.mark.parametrize("name,chunks", [("olmoe_1b7b", 4), ("mxfp8_e128", 3),
                                         ("fine_grained_e384", 1), ("sweep_e128", 2),
                                         ("sweep_e8", 5), ("sweep_e32", 3)])
def test_choose_chunks_on_the_workloads(name, chunks):
    """The slice counts the benchmark's e2e leg uses on each workload."""
    assert _moe().choose_chunks(*_args(name)) == chunks


def test_choose_chunks_minimises_the_stated_cost():
    """c slices cost c*Wt + Ct*h(c), h = 2, 1, 1/(c-1): the choice is the
    least cost over 1..max_chunks, and the limits behave: weights that take
    long to stream give one slice, free weights the most slices."""
    moe = _moe()
    for T, d, wb in ((4096, 2048, 1e9), (16384, 4096, 3e8), (512, 1024, 5e10), (65536, 7168, 2e9)):
        ct = T * d * 2 / (moe.PCIE_GBS * 1e9)
        wt = wb / (moe.HBM_GBS * 1e9)
        cost = lambda c: c * wt + ct * (2.0 if c == 1 else 1.0 if c == 2 else 1.0 / (c - 1))
        best = min(range(1, 9), key=cost)
        assert moe.choose_chunks(T, d, 2, int(wb)) == best
    assert moe.choose_chunks(1024, 1024, 2, 10 ** 12) == 1
    assert moe.choose_chunks(1 << 20, 8192, 2, 1, max_chunks=6) == 6
