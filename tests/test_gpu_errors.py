"""Failure detection on the GPU without faulting it: a bounded device wait on
a flag nothing sets must give up, record BQ_ERR_TIMEOUT and leave the context
usable; argument errors leave outputs untouched."""
import numpy as np
import pytest

import ternary_g128_weight_b200 as bq
from gpu_util import cuda

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import torch
    cuda()
    assert bq.bq_check() == bq.BQ_OK
    assert bq.bq_debug_wait_timeout(2000) == bq.BQ_OK      # launch ok
    assert bq.bq_check() == bq.BQ_ERR_TIMEOUT               # the wait gave up
    assert bq.bq_check() == bq.BQ_OK                        # flag cleared
    a = torch.arange(10, device="cuda")
    assert int(a.sum()) == 45                               # context still usable


def test_argument_error_writes_nothing():
    import torch
    dev = cuda()
    y = torch.full((1, 4), 3.0, dtype=torch.float32, device=dev)
    x = torch.zeros((1, 100), dtype=torch.bfloat16, device=dev)
    c = torch.zeros(64, dtype=torch.uint8, device=dev)
    s = torch.zeros(8, dtype=torch.int16, device=dev)
    with pytest.raises(bq.BQError) as ei:
        bq.bq_gemv("q1g128", c, s, 4, 100, x, y=y, y_dtype=bq.BQ_F32)
    assert ei.value.status == bq.BQ_ERR_SHAPE
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)
    with pytest.raises(bq.BQError) as ei:
        bq.bq_gemv("q1g128", c[1:], s, 4, 128, torch.zeros((1, 128), dtype=torch.bfloat16, device=dev),
                   y=y, y_dtype=bq.BQ_F32)
    assert ei.value.status == bq.BQ_ERR_ALIGN
    assert torch.all(y == 3.0)
