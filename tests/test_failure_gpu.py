"""The device-timeout path end to end, without a fault: a kernel's bounded
wait on an mbarrier that nothing arrives at gives up after the library's
limit, the host reads QLORA_ERR_DEVICE_TIMEOUT once, and the context keeps
working (a quantization right after is bit-exact against the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import bit_nf4_quantized_quantize_b200 as q
from bit_nf4_quantized_quantize_b200 import synth

pytestmark = pytest.mark.gpu

QLORA_ERR_DEVICE_TIMEOUT = -4


def test_expired_wait_is_reported_and_the_context_survives():
    assert q.qlora_device_status() == 0
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    q.qlora_selftest_device_timeout(waited)
    assert q.qlora_device_status() == QLORA_ERR_DEVICE_TIMEOUT
    assert q.qlora_device_status() == 0                  # the flag was cleared by the read
    ns = int(waited.item())
    assert 2.0e9 <= ns < 3.0e9, ns                        # the limit is 2 s of %globaltimer
    W = synth.weight(1, 0, 256, 256)
    codes, q8, s2 = q.qlora_quantize_nf4_dq(torch.from_numpy(W).cuda())
    rc, rq, rs, _ = oracle.quantize_nf4_dq(W.reshape(-1))
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(q8.cpu().numpy(), rq)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert q.qlora_device_status() == 0
