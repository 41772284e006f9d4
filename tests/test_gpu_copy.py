"""parallax_copy: the kernel copy between device memory and mapped page-locked
host memory that the end-to-end decode loop uses for its small per-step
transfers. Bytes must arrive unchanged in every direction; pageable host
memory and misaligned pointers are refused on the host."""
import pytest
import torch

from parameterized_local_linear_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 8448, (1 << 20) + 16 * 37])
def test_copy_round_trip(nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
    dev = torch.full((nbytes,), 7, dtype=torch.uint8, device="cuda")
    binding.parallax_copy(dev, src)                       # host -> device
    dev2 = torch.empty_like(dev)
    binding.parallax_copy(dev2, dev)                      # device -> device
    back = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    binding.parallax_copy(back, dev2)                     # device -> host
    torch.cuda.current_stream().synchronize()
    assert torch.equal(dev.cpu(), src)
    assert torch.equal(back, src)


def test_copy_refusals():
    dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    pageable = torch.zeros(64, dtype=torch.uint8)
    with pytest.raises(RuntimeError):
        binding.parallax_copy(dev, pageable)              # not mapped for the device
    pinned = torch.zeros(80, dtype=torch.uint8).pin_memory()
    with pytest.raises(RuntimeError):
        binding.parallax_copy(dev, pinned[8:72])          # 8-byte offset: misaligned
    with pytest.raises(RuntimeError):
        binding.parallax_copy(dev[:40], pinned[:40])      # not a multiple of 16 bytes


def test_copy_in_a_graph_with_a_decode_step():
    """The e2e loop's shape: bytes in, decode, bytes out, captured and replayed."""
    import oracle
    from parameterized_local_linear_b200 import inputs
    w = inputs.custom_workload("copy", B=2, Hq=16, Hkv=8, D=128, Lmax=300, seed=71)
    x = inputs.make_inputs(w, device="cuda")
    host_q = x["q"].cpu().pin_memory()
    out = torch.empty_like(x["q"])
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    ws = binding.Workspace(2, 16, 8, 128, 300)
    q_dev = torch.zeros_like(x["q"])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        binding.parallax_copy(q_dev, host_q, stream=s)
        binding.parallax_decode(q_dev, x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                out=out, workspace=ws, stream=s)
        binding.parallax_copy(host_out, out, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        binding.parallax_copy(q_dev, host_q, stream=s)
        binding.parallax_decode(q_dev, x["r"], x["k"], x["v"], x["seqlens"], scale=x["scale"],
                                out=out, workspace=ws, stream=s)
        binding.parallax_copy(host_out, out, stream=s)
    host_out.zero_()
    g.replay()
    s.synchronize()
    ref = oracle.parallax_decode(x["q"], x["r"], x["k"], x["v"], x["seqlens"], x["scale"])
    err = (host_out.double().numpy() - ref)
    assert float(abs(err).max() / max(1.0, float(abs(ref).max()))) <= 2e-2
    assert torch.equal(host_out, out.cpu())
