"""Failure detection on the GPU without a fault: a bounded device wait that is
made to run out reports PISA_ERR_DEVICE_TIMEOUT through the device status word,
the status clears once read, and the context stays usable (the next attention
call is still correct).  Nothing here traps, faults or hangs: the wait is
bounded by a cycle limit of about a millisecond."""
import pytest
import torch

import block_sparse_taylor_b200 as pisa
import oracle
import parity
import pisa_synth

pytestmark = pytest.mark.gpu


def _clear_status():
    try:
        pisa.pisa_poll_device_status()
    except pisa.PisaError:
        pass


def test_bounded_wait_reports_a_timeout_and_the_context_survives():
    _clear_status()
    pisa.pisa_selftest_wait_timeout(2_000_000)
    with pytest.raises(pisa.PisaError) as err:
        pisa.pisa_poll_device_status()
    assert err.value.status == pisa.PISA_ERR_DEVICE_TIMEOUT
    pisa.pisa_poll_device_status()  # the status word was cleared by the read
    q, k, v = pisa_synth.random_qkv(31, 2, 512, 64, scale=2.0, dtype="bf16")
    dev = [torch.from_numpy(x).to("cuda").to(torch.bfloat16) for x in (q, k, v)]
    out = pisa.pisa_attention(*dev, 64, 2, 1)
    pisa.pisa_poll_device_status()
    parity.check(out.float().cpu().numpy(), oracle.pisa_attention(q, k, v, 64, 2, 1), "bf16", "after timeout")


def test_timeout_on_a_side_stream_is_seen_by_its_poll():
    s = torch.cuda.Stream()
    _clear_status()
    pisa.pisa_selftest_wait_timeout(1_000_000, stream=s)
    with pytest.raises(pisa.PisaError) as err:
        pisa.pisa_poll_device_status(stream=s)
    assert err.value.status == pisa.PISA_ERR_DEVICE_TIMEOUT
    pisa.pisa_poll_device_status(stream=s)
