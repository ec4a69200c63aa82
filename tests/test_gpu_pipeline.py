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
