"""GPU parity on irreps sets unlike the workloads (the planner's coverage
check runs on the same sets in tests/test_planner.py): multiplicity 1 and 3,
ragged blocks of 17 and 33 channels, a hidden irrep that feeds no output
(its dx columns are zero), odd hidden parities, degree-4 harmonics, output
subsets.  Random ragged graphs, same bar as the other parity tests.  Named
to be collected after them.
"""
import pytest

from tests.test_gpu_parity import check_random_graph
from tests.test_planner import ODD

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    return torch.device("cuda:0")


@pytest.mark.parametrize("spec", ODD, ids=[f"odd{k}" for k in range(len(ODD))])
def test_odd_irreps_random_graph(spec, dev):
    check_random_graph(*spec, dev)
