"""After the GPU parity suite: no bounded wait inside a decode kernel gave up
and no merge ticket was found above its count (kvq_decode_status).  The
parity tests would also see such events as NaN outputs; this reads the
counters the kernels keep for them."""
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq

pytestmark = pytest.mark.gpu


def test_no_expired_waits_or_bad_tickets():
    torch.cuda.synchronize()
    timeouts, bad = kvq.kvq_decode_status()
    assert timeouts == 0
    assert bad == 0


def test_status_clear():
    kvq.kvq_decode_status(clear=True)
    assert kvq.kvq_decode_status() == (0, 0)
