"""The Python binding has no CPU path: every compute call given host tensors
(not pinned) refuses with an error before anything runs, instead of falling
back to a computation on the CPU.  Runs without a GPU."""
import pytest
import torch


@pytest.fixture(scope="module")
def nq():
    from e8_lattice_vector_nq_b200 import build, nq as nqmod

    build.build()
    return nqmod


def test_every_compute_call_refuses_host_tensors(nq):
    K = torch.zeros(1, 8, 64, 128, dtype=torch.bfloat16)
    ks = nq.PackedStore.empty(1, 8, 64, 3, "cpu")
    vs = nq.PackedStore.empty(1, 8, 64, 2, "cpu")
    scores = torch.zeros(1, 64, dtype=torch.float64)
    tab = torch.zeros(16)
    calls = {
        "nq_score": lambda: nq.nq_score(K, 16),
        "nq_select": lambda: nq.nq_select(scores, 16, 50),
        "nq_encode": lambda: nq.nq_encode(K, K, ks, vs, 64, tab, 64),
        "nq_decode": lambda: nq.nq_decode(ks, vs, 64, K, K, tab, 64),
        "nq_attend": lambda: nq.nq_attend(torch.zeros(1, 32, 128), ks, vs, 64, 4, tab, 64),
        "nq_e8_quantise": lambda: nq.nq_e8_quantise(torch.zeros(4, 8), 3),
        "nq_entropy_encode": lambda: nq.nq_entropy_encode(ks, 64),
        "nq_entropy_decode": lambda: nq.nq_entropy_decode(
            nq.EntropyCoded(torch.zeros(8, dtype=torch.int16), torch.zeros(2, dtype=torch.int32),
                            torch.zeros(1, 8, 8, dtype=torch.int16), 1, 8, 64, 3, True), ks),
    }
    for name, call in calls.items():
        with pytest.raises(ValueError, match="no CPU path"):
            call()
