"""Host-side tests of the C ABI (no GPU needed): the library loads and exports
every function include/nq.h declares, argument validation returns the
documented status without launching anything, and the host-built RoPE
tables and count rules agree with the oracle.
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nq():
    from e8_lattice_vector_nq_b200 import build, nq as nqmod

    build.build()
    return nqmod


def header_functions() -> list[str]:
    src = open(os.path.join(ROOT, "include", "nq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(nq):
    names = header_functions()
    assert len(names) >= 12
    L = ctypes.CDLL(nq.SO_PATH)
    for n in names:
        assert hasattr(L, n), f"libnq.so does not export {n}"
    assert set(names) == set(nq.EXPORTS)
    assert nq.lib().nq_version() == 1


def test_packed_sizes_and_counts(nq, oq):
    L = nq.lib()
    assert L.nq_packed_bytes_per_vector(3) == 52
    assert L.nq_packed_bytes_per_vector(2) == 36
    assert L.nq_packed_bytes_per_vector(4) == -1
    rng = np.random.default_rng(0)
    for _ in range(500):
        T = int(rng.integers(1, 200000))
        W = int(rng.integers(0, 300))
        p = int(rng.integers(0, 101))
        assert nq.kept_count(T, W, p) == oq.kept_count(T, W, p)


def test_rope_tables_match_oracle_rule(nq, oq):
    L = nq.lib()
    max_pos = 70000
    nbytes = L.nq_rope_tables_bytes(max_pos)
    na = (max_pos + 255) // 256
    assert nbytes == (na + 256) * 64 * 8
    buf = np.zeros(nbytes // 4, np.float32)
    assert L.nq_rope_tables_fill_host(1e6, max_pos, buf.ctypes.data, nbytes) == 0
    tab = buf.reshape(na + 256, 64, 2)
    rng = np.random.default_rng(1)
    pos = np.concatenate([[0, 1, 255, 256, max_pos - 1], rng.integers(0, max_pos, 300)])
    c_or, s_or = oq.rope_cs(1e6, pos)
    a, b = pos >> 8, pos & 255
    A, B = tab[a], tab[na + b]
    # emulate c = fmaf(cA, cB, -(sA*sB)) in fp64 (the product is exact), fp32 result
    ss = (A[..., 1] * B[..., 1]).astype(np.float32)
    cs = (A[..., 0] * B[..., 1]).astype(np.float32)
    c = (A[..., 0].astype(np.float64) * B[..., 0] - ss).astype(np.float32)
    s = (A[..., 1].astype(np.float64) * B[..., 0] + cs).astype(np.float32)
    assert np.max(np.abs(c - c_or)) <= 1.2e-7 and np.max(np.abs(s - s_or)) <= 1.2e-7
    assert np.mean(c == c_or) > 0.999 and np.mean(s == s_or) > 0.999


def _err(nq):
    return nq.lib().nq_last_error().decode()


def test_validation_rejects_bad_arguments(nq):
    L = nq.lib()
    S = nq.KVStrides
    ok = S(8 * 128 * 64, 128 * 64, 128)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    pk = nq.Packed(0x20000, 0x30000, 64, 64, 3)
    bad_bits = nq.Packed(0x20000, 0x30000, 64, 64, 4)
    # both inputs missing
    assert L.nq_encode(None, ok, None, ok, 1, 8, 64, 64, None, 0, 0, fake, 64, None, None, 0, None) == nq.NQ_ERR_INVALID
    assert "both NULL" in _err(nq)
    # bits must be 2 or 3
    assert L.nq_encode(fake, ok, None, ok, 1, 8, 64, 64, None, 0, 0, fake, 64,
                       ctypes.byref(bad_bits), None, 0, None) == nq.NQ_ERR_INVALID
    assert "bits" in _err(nq)
    # token stride not a multiple of 8
    assert L.nq_encode(fake, S(0, 0, 130), None, ok, 1, 8, 64, 64, None, 0, 0, fake, 64,
                       ctypes.byref(pk), None, 0, None) == nq.NQ_ERR_INVALID
    # misaligned base pointer
    assert L.nq_encode(ctypes.c_void_p(0x10008), ok, None, ok, 1, 8, 64, 64, None, 0, 0, fake, 64,
                       ctypes.byref(pk), None, 0, None) == nq.NQ_ERR_INVALID
    # keys need rope tables and in-range positions
    assert L.nq_encode(fake, ok, None, ok, 1, 8, 64, 64, None, 0, 0, None, 64,
                       ctypes.byref(pk), None, 0, None) == nq.NQ_ERR_INVALID
    assert L.nq_encode(fake, ok, None, ok, 1, 8, 64, 64, None, 0, 10, fake, 64,
                       ctypes.byref(pk), None, 0, None) == nq.NQ_ERR_INVALID
    assert "rope_max_pos" in _err(nq)
    # n beyond T_in without a kept list
    assert L.nq_encode(fake, ok, None, ok, 1, 8, 64, 65, None, 0, 0, fake, 128,
                       ctypes.byref(pk), None, 0, None) == nq.NQ_ERR_INVALID
    # score: window larger than T, small workspace
    assert L.nq_score(fake, ok, 1, 8, 64, 65, fake, fake, 1 << 20, None) == nq.NQ_ERR_INVALID
    assert L.nq_score(fake, ok, 1, 8, 64, 64, fake, fake, 16, None) == nq.NQ_ERR_WORKSPACE
    assert L.nq_score(fake, ok, 1, 129, 64, 64, fake, fake, 1 << 30, None) == nq.NQ_ERR_UNSUPPORTED
    assert L.nq_score_static(fake, ok, 1, 129, 64, 64, fake, None) == nq.NQ_ERR_UNSUPPORTED
    assert L.nq_encode(fake, ok, None, ok, 1 << 20, 8, 1 << 12, 1 << 12, None, 0, 0, fake, 1 << 12,
                       ctypes.byref(pk), None, 0, None) == nq.NQ_ERR_UNSUPPORTED
    assert L.nq_e8_quantise(fake, 4, 5, fake, fake, None) == nq.NQ_ERR_INVALID
    assert L.nq_e8_quantise(fake, -1, 3, fake, fake, None) == nq.NQ_ERR_INVALID
    # select: percentage range, stride, size limit
    assert L.nq_select(fake, 1, 100, 10, 101, fake, 100, None) == nq.NQ_ERR_INVALID
    assert L.nq_select(fake, 1, 100, 10, 50, fake, 10, None) == nq.NQ_ERR_INVALID
    assert L.nq_select(fake, 1, (1 << 20) + 1, 10, 50, fake, 1 << 21, None) == nq.NQ_ERR_UNSUPPORTED
    # decode: both outputs missing, bad packed descriptor
    assert L.nq_decode(None, None, 1, 8, 64, 0, None, 0, 0, fake, 64, None, ok, None, ok, None) == nq.NQ_ERR_INVALID
    assert L.nq_decode(None, ctypes.byref(bad_bits), 1, 8, 64, 0, None, 0, 0, fake, 64, None, ok,
                       fake, ok, None) == nq.NQ_ERR_INVALID
    # entropy stage: shape, flag, capacity and workspace checks
    assert L.nq_entropy_encode(ctypes.byref(pk), 1, 8, 0, 0, 1, fake, fake, fake, 1 << 30, fake,
                               1 << 30, None) == nq.NQ_ERR_INVALID
    assert L.nq_entropy_encode(ctypes.byref(pk), 1, 8, 64, 0, 2, fake, fake, fake, 1 << 30, fake,
                               1 << 30, None) == nq.NQ_ERR_INVALID
    assert L.nq_entropy_encode(ctypes.byref(bad_bits), 1, 8, 64, 0, 1, fake, fake, fake, 1 << 30,
                               fake, 1 << 30, None) == nq.NQ_ERR_INVALID
    cap = L.nq_entropy_max_words(1, 8, 64)
    assert cap == L.nq_entropy_streams(1, 8, 64) * 2050 == 8 * 128 * 2050
    assert L.nq_entropy_encode(ctypes.byref(pk), 1, 8, 64, 0, 1, fake, fake, fake, cap - 1, fake,
                               1 << 30, None) == nq.NQ_ERR_WORKSPACE
    assert L.nq_entropy_encode(ctypes.byref(pk), 1, 8, 64, 0, 1, fake, fake, fake, cap, fake,
                               16, None) == nq.NQ_ERR_WORKSPACE
    assert L.nq_entropy_encode(ctypes.byref(pk), 1 << 12, 1024, 1 << 20, 0, 1, fake, fake, fake,
                               1 << 62, fake, 1 << 62, None) == nq.NQ_ERR_UNSUPPORTED
    assert L.nq_entropy_decode(fake, fake, fake, 1, 8, 1 << 25, 1, ctypes.byref(pk), 0,
                               None) == nq.NQ_ERR_INVALID
    assert L.nq_entropy_decode(None, fake, fake, 1, 8, 64, 1, ctypes.byref(pk), 0,
                               None) == nq.NQ_ERR_INVALID
    # rope table fill: bad theta, small buffer
    buf = np.zeros(16, np.float32)
    assert L.nq_rope_tables_fill_host(0.5, 10, buf.ctypes.data, 64) == nq.NQ_ERR_INVALID
    assert L.nq_rope_tables_fill_host(1e4, 10, buf.ctypes.data, 64) == nq.NQ_ERR_WORKSPACE


def test_empty_work_is_ok_without_device(nq):
    L = nq.lib()
    S = nq.KVStrides(0, 0, 0)
    fake = ctypes.c_void_p(0x10000)
    assert L.nq_encode(fake, S, None, S, 0, 8, 64, 64, None, 0, 0, fake, 64, None, None, 0, None) == 0
    assert L.nq_score(fake, S, 0, 8, 64, 64, fake, fake, 0, None) == 0
    pk = nq.Packed(0x20000, 0x30000, 64, 64, 2)
    assert L.nq_entropy_encode(ctypes.byref(pk), 0, 8, 64, 0, 1, None, None, None, 0, None, 0,
                               None) == 0
    assert L.nq_entropy_decode(None, None, None, 0, 8, 64, 0, ctypes.byref(pk), 0, None) == 0


def test_decode_engine_switch(nq):
    """The decode engine is a process-wide setting: auto by default, each
    documented value accepted and read back, anything else refused."""
    assert nq.get_decode_engine() == nq.DECODE_AUTO
    try:
        for e in (nq.DECODE_TENSOR_CORES, nq.DECODE_CUDA_CORES, nq.DECODE_AUTO):
            nq.set_decode_engine(e)
            assert nq.get_decode_engine() == e
        L = nq.lib()
        assert L.nq_set_decode_engine(3) == nq.NQ_ERR_INVALID
        assert "decode engine" in L.nq_last_error().decode()
        assert nq.get_decode_engine() == nq.DECODE_AUTO
    finally:
        nq.set_decode_engine(nq.DECODE_AUTO)

