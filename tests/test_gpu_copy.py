"""arkv_copy_async: the kernel copy the decode loop uses for its host inputs and
outputs -- page-locked host memory to device and back, bit for bit, also when
captured into a CUDA graph; pageable host memory is refused before any launch."""
import pytest
import torch

from mixed_precision_kv_arkv_b200 import abi
from mixed_precision_kv_arkv_b200.build import build
from mixed_precision_kv_arkv_b200.cache import stream_ptr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    abi.lib()


def test_copy_host_device_round_trip(cuda):
    g = torch.Generator().manual_seed(7)
    n = (3 << 20) + 48                                      # not a multiple of the block
    host = torch.randint(0, 256, (n,), dtype=torch.uint8, generator=g).pin_memory()
    dev = torch.empty(n, dtype=torch.uint8, device=cuda)
    back = torch.zeros(n, dtype=torch.uint8).pin_memory()
    abi.arkv_copy_async(dev.data_ptr(), host.data_ptr(), n, stream_ptr())
    abi.arkv_copy_async(back.data_ptr(), dev.data_ptr(), n, stream_ptr())
    torch.cuda.synchronize()
    assert torch.equal(dev.cpu(), host)
    assert torch.equal(back, host)


def test_copy_in_a_cuda_graph(cuda):
    n = 1 << 20
    host_in = torch.arange(n // 4, dtype=torch.int32).pin_memory()
    dev = torch.empty(n // 4, dtype=torch.int32, device=cuda)
    host_out = torch.zeros(n // 4, dtype=torch.int32).pin_memory()
    abi.arkv_copy_async(dev.data_ptr(), host_in.data_ptr(), n, stream_ptr())   # first call outside the capture
    abi.arkv_copy_async(host_out.data_ptr(), dev.data_ptr(), n, stream_ptr())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        abi.arkv_copy_async(dev.data_ptr(), host_in.data_ptr(), n, stream_ptr())
        dev.add_(1)
        abi.arkv_copy_async(host_out.data_ptr(), dev.data_ptr(), n, stream_ptr())
    host_in.mul_(3)                                          # the replay reads the buffer as it is now
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(host_out, host_in + 1)
    del graph


def test_copy_refuses_pageable_host_memory(cuda):
    pageable = torch.zeros(1024, dtype=torch.uint8)
    dev = torch.empty(1024, dtype=torch.uint8, device=cuda)
    rc = abi.arkv_copy_async(dev.data_ptr(), pageable.data_ptr(), 1024, stream_ptr(), check=False)
    assert rc == abi.ARKV_EINVAL
    assert "device-addressable" in abi.arkv_last_error_string()
    torch.cuda.synchronize()
