"""The measurement probes behind the roofline peaks and the dense kernels'
design run and report plausible rates (needs a B200).  The figures themselves
are recorded by `bench.py --workload mufu` and `bench.py --workload tcprobe`;
these checks only guard the probes (a sensible range, no timed-out wait)."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import differentiable_bcjr_b200 as B
    B.lib()
    return B


def test_xu_probe(B):
    r = B.probe_xu("ex2", 1024)
    assert 4.0 < r["ops_per_clk_per_sm"] <= 16.5


@pytest.mark.parametrize("n", [16, 64, 256])
def test_mma_probe(B, n):
    r = B.probe_mma_tf32(n, 512)
    # a tf32 product of 128 x n x 8 cannot beat 4096 MAC per clock per SM (twice
    # the nominal dense rate) nor take longer than a microsecond at this size
    assert 0 < r["mac_per_clk_per_sm"] <= 4096
    assert 4 < r["clk_per_mma"] < 2000


@pytest.mark.parametrize("chunk", [0, 256, 4096])
def test_dsmem_probe(B, chunk):
    r = B.probe_dsmem(2, 20, chunk=chunk)
    assert 1.0 < r["bytes_per_clk_per_sm"] < 256.0
