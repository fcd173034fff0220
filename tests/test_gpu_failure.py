"""GPU: the attention kernel's bounded waits end in an error status, not a hang.

The test makes one wait run out without faulting anything: through
``da2_attention_wait_test`` one CTA never issues its first key-tile load, and
every wait is limited to a few thousand polls.  The CTA's MMA issuer and
softmax warps then give up, raise the workspace status word, stop issuing,
let their copies in flight land and release their tensor memory; the host
reads DA2_ERR_TIMEOUT through ``da2_check_status``.  The next ordinary call on
the same workspace must report DA2_OK and reproduce the output bit for bit.
"""

import pytest
import torch

from mixed_precision_block_b200.synth import Workload, make_qkv

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from mixed_precision_block_b200 import da2


@pytest.mark.parametrize("d", [128, 64])
def test_withheld_load_times_out_and_the_next_call_is_clean(d):
    wl = Workload("fail", 1, 2, 3, 16, 24, d, 0.5, (40.0, 20.0, 20.0, 20.0), seed=12)
    q, k, v = make_qkv(wl, "cuda")
    p = da2.Problem.from_workload(wl)
    ws = da2.workspace(p)
    want = torch.empty_like(q)
    da2.attention(p, q, k, v, ws, want)
    assert da2.da2_check_status(p, ws) == da2.DA2_OK

    out = torch.zeros_like(q)
    rc = da2.da2_attention_wait_test(p, q, k, v, ws, out, withheld_cta=0, wait_polls=1 << 12)
    assert rc == da2.DA2_OK  # the launch itself succeeds
    assert da2.da2_check_status(p, ws) == da2.DA2_ERR_TIMEOUT
    torch.cuda.synchronize()  # the context is still usable

    again = torch.empty_like(q)
    da2.da2_attention(p, q, k, v, ws, again)
    assert da2.da2_check_status(p, ws) == da2.DA2_OK
    assert torch.equal(again, want)


def test_wait_bound_alone_does_not_trip_a_normal_call():
    wl = Workload("fail", 1, 2, 3, 16, 24, 128, 0.5, (40.0, 20.0, 20.0, 20.0), seed=12)
    q, k, v = make_qkv(wl, "cuda")
    p = da2.Problem.from_workload(wl)
    ws = da2.workspace(p)
    want = torch.empty_like(q)
    da2.attention(p, q, k, v, ws, want)
    out = torch.empty_like(q)
    assert da2.da2_attention_wait_test(p, q, k, v, ws, out, withheld_cta=-1, wait_polls=1 << 20) == da2.DA2_OK
    assert da2.da2_check_status(p, ws) == da2.DA2_OK
    assert torch.equal(out, want)


def test_dense_status_reads_ok_after_a_dense_call():
    g = torch.Generator(device="cuda").manual_seed(3)
    q, k, v = (torch.randn((1, 2, 300, 128), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    out = torch.empty_like(q)
    da2.da2_dense_attention(q, k, v, out)
    assert da2.da2_dense_check_status() == da2.DA2_OK
