"""commvq_copy_async on the GPU: device to device, mapped pinned host memory to device and back,
whole 16-byte pieces and a ragged tail, every byte compared (the copy's only arithmetic is none)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


@pytest.mark.parametrize("nbytes", [16, 1000, 12288, 16384 + 7, 5 << 20])
def test_copy_device_and_mapped_host(api, nbytes):
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(nbytes)
    src_h = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
    # host -> device (mapped loads) when the pinned buffer is mapped, else device -> device only
    mapped = api.host_mapped(src_h)
    src_d = src_h.to(dev)
    mid = torch.zeros(nbytes + 64, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream()
    api.copy_async(mid, src_h if mapped else src_d, stream=s)
    back_d = torch.full((nbytes + 64,), 7, dtype=torch.uint8, device=dev)
    api.copy_async(back_d, mid[:nbytes], stream=s)           # device -> device
    out_h = torch.full((nbytes,), 9, dtype=torch.uint8).pin_memory()
    if api.host_mapped(out_h):
        api.copy_async(out_h, back_d[:nbytes], stream=s)     # device -> host (mapped stores)
    else:
        out_h.copy_(back_d[:nbytes])
    torch.cuda.synchronize()
    assert torch.equal(mid[:nbytes].cpu(), src_h)
    assert torch.equal(mid[nbytes:].cpu(), torch.zeros(64, dtype=torch.uint8))   # nothing past the end
    assert torch.equal(back_d[nbytes:].cpu(), torch.full((64,), 7, dtype=torch.uint8))
    assert torch.equal(out_h, src_h)
