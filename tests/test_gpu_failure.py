"""The bounded-wait failure path on the GPU: waits that nothing completes
expire, set the device error word, and leave the context usable."""

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import _lib, synth
from oracle import ns_oracle as O

from helpers import TOL_BF16, rel_fro, to_np

pytestmark = pytest.mark.gpu


def test_expired_waits_report_timeout_and_context_survives():
    msb.sync_status()  # start clean
    msb.selftest_timeout(50_000_000)  # an mbarrier wait and a counter wait, 50 ms each
    with pytest.raises(msb.MsignError) as e:
        msb.sync_status()
    assert e.value.status == _lib.ERR_TIMEOUT
    msb.sync_status()  # reading the status cleared the word
    # the same context keeps working
    x = torch.from_numpy(synth.gaussian((256, 512), seed=3)).cuda().to(torch.bfloat16)
    y = msb.msign_ns(x)
    msb.sync_status()
    assert rel_fro(to_np(y), O.msign_ns(to_np(x), input_cast="bf16")) < TOL_BF16
