"""The host round trip (nq.HostRoundTrip): a cache in pinned host memory is
compressed and reconstructed chunk by chunk on three streams, with the values
either copied or read in place from the pinned host cache by the encode
kernel.  Its host output must equal, bit for bit, the reconstruction of the
same cache through the device calls in one piece, on every run (the second
run checks the cross-run stream ordering on reused buffers)."""
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


@pytest.mark.parametrize("chunk,in_place", [(1, False), (2, False), (5, False), (2, True),
                                            (3, True)])
def test_host_round_trip_equals_device_path(nq, chunk, in_place):
    wl = synth.WORKLOADS["mistral7b_32k"]
    L, H, T = 7, 4, 3000
    layers = [synth.gen_layer(wl, l, "cuda", tokens=T) for l in range(L)]
    K = torch.stack([k[:H] for k, _ in layers])
    V = torch.stack([v[:H] for _, v in layers])
    ref = nq.Codec(L, H, T, wl.theta, 3, 2, wl.window, wl.evict_pct)
    Kr = torch.empty(L, H, ref.n, 128, dtype=torch.bfloat16, device="cuda")
    Vr = torch.empty_like(Kr)
    ref.encode(K, V)
    ref.decode(Kr, Vr)

    codec = nq.Codec(L, H, T, wl.theta, 3, 2, wl.window, wl.evict_pct)
    Kd, Vd = torch.empty_like(K), torch.empty_like(V)
    Ko, Vo = torch.empty_like(Kr), torch.empty_like(Vr)
    rt = nq.HostRoundTrip(codec, Kd, Vd, Ko, Vo, chunk_units=chunk, values_in_place=in_place)
    Kh, Vh = K.cpu().pin_memory(), V.cpu().pin_memory()
    for run in range(2):
        Koh = torch.zeros(Kr.shape, dtype=Kr.dtype).pin_memory()
        Voh = torch.zeros(Vr.shape, dtype=Vr.dtype).pin_memory()
        rt.run(Kh, Vh, Koh, Voh)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(Koh, Kr.cpu()) and torch.equal(Voh, Vr.cpu()), run
        assert torch.equal(codec.kept.cpu(), ref.kept.cpu())
    assert nq.device_error() == 0


@pytest.mark.parametrize("chunk", [1, 2])
def test_host_ring_passes_every_unit_through(nq, chunk):
    """Host buffers of R < units units act as a ring (unit u uses slot u % R):
    with equal inputs in every unit mapped to a slot (no eviction), each slot
    ends holding the reconstruction of its input, and a ring that does not fit
    the chunk, or values read in place, is refused."""
    wl = synth.WORKLOADS["llama3_8b_128k"]
    L, R, H, T = 8, 4, 8, 700
    ring_in = [synth.gen_layer(wl, l, "cuda", tokens=T) for l in range(R)]
    Kr_in = torch.stack([k for k, _ in ring_in])
    Vr_in = torch.stack([v for _, v in ring_in])
    # reference: the R ring layers through the device calls
    ref = nq.Codec(R, H, T, wl.theta, 3, 2, wl.window, 0)
    ref.encode(Kr_in, Vr_in)
    Kref = torch.empty(R, H, ref.n, 128, dtype=torch.bfloat16, device="cuda")
    Vref = torch.empty_like(Kref)
    ref.decode(Kref, Vref)
    codec = nq.Codec(L, H, T, wl.theta, 3, 2, wl.window, 0)
    Kd = torch.empty(L, H, T, 128, dtype=torch.bfloat16, device="cuda")
    Vd = torch.empty_like(Kd)
    Ko = torch.empty(L, H, codec.n, 128, dtype=torch.bfloat16, device="cuda")
    Vo = torch.empty_like(Ko)
    rt = nq.HostRoundTrip(codec, Kd, Vd, Ko, Vo, chunk_units=chunk)
    Kh, Vh = Kr_in.cpu().pin_memory(), Vr_in.cpu().pin_memory()
    Koh = torch.zeros((R,) + tuple(Ko.shape[1:]), dtype=Ko.dtype).pin_memory()
    Voh = torch.zeros_like(Koh).pin_memory()
    rt.run(Kh, Vh, Koh, Voh)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(Koh, Kref.cpu()) and torch.equal(Voh, Vref.cpu())
    assert rt.h2d_bytes(Kh, Vh) == L * 2 * H * T * 128 * 2
    assert rt.d2h_bytes(Koh, Voh) == L * 2 * H * codec.n * 128 * 2
    assert nq.device_error() == 0
    with pytest.raises(ValueError):
        nq.HostRoundTrip(codec, Kd, Vd, Ko, Vo, chunk_units=3).run(Kh, Vh, Koh, Voh)
