"""GPU: the host-buffer entry point (chunks of heads, copies overlapped with
kernels) gives exactly the device path's output: every stage is per (batch,
head), so a chunk of heads computes the same bits as the whole problem."""

import pytest
import torch

from mixed_precision_block_b200.synth import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from mixed_precision_block_b200 import da2


def _device_path(wl, q, k, v):
    p = da2.Problem.from_workload(wl)
    ws = da2.workspace(p)
    out = torch.empty_like(q)
    da2.attention(p, q, k, v, ws, out)
    torch.cuda.synchronize()
    assert da2.da2_check_status(p, ws) == 0
    return p, out.cpu()


@pytest.mark.parametrize("name,G", [("mid", 1), ("mid", 5), ("mid", 12), ("tiny", 3)])
def test_host_path_equals_device_path(name, G):
    wl = WORKLOADS[name]
    q, k, v = make_qkv(wl, "cuda")
    p, want = _device_path(wl, q, k, v)
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    hout = torch.full(q.shape, float("nan"), dtype=q.dtype).pin_memory()
    dev = da2.host_buffer(p, G)
    da2.da2_forward_host(p, hq, hk, hv, hout, dev, G)
    assert torch.equal(hout, want)
    # a second call on the same buffer gives the same bits
    hout2 = torch.zeros_like(hout).pin_memory()
    da2.da2_forward_host(p, hq, hk, hv, hout2, dev, G)
    assert torch.equal(hout2, want)


def test_host_path_ragged_padded_batch2():
    wl = WORKLOADS["mid"].with_(B=2, H=3, Hh=20, Ww=28, d=64)
    q, k, v = make_qkv(wl, "cuda")
    p, want = _device_path(wl, q, k, v)
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    dev = da2.host_buffer(p, 4)  # chunks of 4 and 2 (batch, head) slices
    da2.da2_forward_host(p, hq, hk, hv, hout, dev, 4)
    assert torch.equal(hout, want)
