"""GPU E8 step (nq_e8_quantise) against the oracle's E8 step, bit for bit.

The encode kernels decide between the two cosets from the integer coset's
rounding alone whenever the two distances are clearly apart, and fall back
to both full D8 decodes otherwise.  These inputs aim at that boundary: exact
and near ties of the two distances (sum |e| close to 2), errors at or near
0 and 1/2, tiny values, odd sums with tied largest errors, values large
enough to force the full decision, and a ragged group count.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from e8_lattice_vector_nq_b200 import build, nq as nqmod

    build.build()
    return nqmod


def adversarial_groups(seed: int, n: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    f32 = np.float32
    sign = lambda: rng.choice([-1.0, 1.0], (n, 8))
    base = rng.integers(-4, 4, (n, 8)).astype(np.float64)
    sets = [
        rng.normal(0, 1, (n, 8)),
        rng.normal(0, 3.5, (n, 8)),
        rng.uniform(-5.2, 5.2, (n, 8)),
        base + 0.25 * sign(),                                  # sum |e| = 2 exactly: distance tie
        base + (0.25 + rng.normal(0, 1e-6, (n, 8))) * sign(),  # near ties
        base + (0.25 + rng.normal(0, 3e-5, (n, 8))) * sign(),  # around the decision margin
        base + 0.5 * sign(),                                   # |e| = 1/2: rounding ties
        base + rng.normal(0, 1e-6, (n, 8)),                    # |e| near 0
        base + 0.5 + rng.normal(0, 1e-6, (n, 8)),              # near half-integers
        base,                                                  # integers: e = 0
        rng.normal(0, 1, (n, 8)) * 1e-30,                      # tiny
        np.where(rng.random((n, 8)) < 0.5, base, base + 0.5),  # mixed lattice-like
        rng.normal(0, 1, (n, 8)) * 1e4,                        # large: full decision forced
    ]
    y = np.concatenate(sets).astype(f32)
    y[rng.random(y.shape) < 0.01] = -0.0
    return y


@pytest.mark.parametrize("bits", [2, 3])
def test_e8_step_matches_oracle(nq, oq, bits):
    y = adversarial_groups(7 + bits, 40000)
    perm = np.random.default_rng(3).permutation(len(y))
    y = y[perm]  # mix the kinds inside every warp
    ref_codes, ref_coset = oq.e8_codes(y, bits)
    codes, coset = nq.nq_e8_quantise(torch.from_numpy(y).cuda(), bits)
    torch.cuda.synchronize()
    got_codes = codes.cpu().numpy().view(np.uint32)
    got_coset = coset.cpu().numpy().astype(np.int32)
    bad = np.nonzero((got_codes != ref_codes) | (got_coset != ref_coset))[0]
    assert bad.size == 0, (bad.size, y[bad[:3]], got_codes[bad[:3]], ref_codes[bad[:3]])


@pytest.mark.parametrize("groups", [1, 2, 3, 63, 64, 65, 8191])
def test_e8_step_ragged_counts(nq, oq, groups):
    y = adversarial_groups(groups, 1000)[:groups]
    ref_codes, ref_coset = oq.e8_codes(y, 3)
    codes, coset = nq.nq_e8_quantise(torch.from_numpy(np.ascontiguousarray(y)).cuda(), 3)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), ref_codes)
    assert np.array_equal(coset.cpu().numpy().astype(np.int32), ref_coset)


def test_e8_step_rejects_bad_arguments(nq):
    L = nq.lib()
    y = torch.zeros(4, 8, device="cuda")
    c = torch.zeros(4, dtype=torch.int32, device="cuda")
    s = torch.zeros(4, dtype=torch.uint8, device="cuda")
    assert L.nq_e8_quantise(nq._ptr(y), 4, 4, nq._ptr(c), nq._ptr(s), None) == nq.NQ_ERR_INVALID
    assert L.nq_e8_quantise(None, 4, 3, nq._ptr(c), nq._ptr(s), None) == nq.NQ_ERR_INVALID
    assert L.nq_e8_quantise(nq._ptr(y), 0, 3, None, None, None) == 0
