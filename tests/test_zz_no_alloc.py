"""nq_score_static: key-key scores without any device allocation.

Some callers cannot allocate device memory: code running inside a host
framework that owns all of the GPU's memory (a serving engine that reserved
HBM for its KV pool up front), or a hot loop where cudaMalloc/cudaFree would
block or synchronise.  They cannot hand nq_score a workspace, so the library
offers nq_score_static, whose scratch is a fixed array in the library's own
device memory.  This file checks, through the C ABI, that its scores equal
nq_score's on two calls in a row (the second with different inputs, so stale
scratch from the first call would show), and that sizes beyond its fixed
scratch are refused.  It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from e8_lattice_vector_nq_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from e8_lattice_vector_nq_b200 import build, nq as nqmod

    build.build()
    return nqmod


def cache(wl, units, T):
    Ks = [synth.gen_layer(wl, u, "cuda", tokens=T)[0] for u in range(units)]
    return torch.stack(Ks)


def test_static_scores_match_workspace_scores_twice(nq):
    wl = synth.WORKLOADS["mistral7b_32k"]
    cases = [(cache(wl, 3, 1500), 64), (cache(synth.WORKLOADS["qwen25_7b_64k"], 5, 2100), 128)]
    for K, W in cases:
        ref = nq.nq_score(K, W)
        got = nq.nq_score_static(K, W)
        torch.cuda.synchronize()
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        # the same kernels on the same inputs: the scores must be identical
        # (a stale or aliased scratch entry would show as a difference)
        assert np.array_equal(g, r)


def test_static_scores_refuse_oversized_calls(nq):
    L = nq.lib()
    K = torch.zeros(1, 8, 64, 128, dtype=torch.bfloat16, device="cuda")
    scores = torch.zeros(300, 64, dtype=torch.float64, device="cuda")
    # 300 units x 8 heads > the fixed scratch: refused on the host, nothing launched
    st = L.nq_score_static(ctypes.c_void_p(K.data_ptr()), nq.KVStrides(0, 64 * 128, 128), 300, 8,
                           64, 16, ctypes.c_void_p(scores.data_ptr()), None)
    assert st == nq.NQ_ERR_UNSUPPORTED
    assert "exceeds" in L.nq_last_error().decode()
    torch.cuda.synchronize()
    assert torch.count_nonzero(scores) == 0
