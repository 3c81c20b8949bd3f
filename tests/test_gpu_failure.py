"""GPU test of failure detection: a device-side wait that runs out is reported
and leaves the context usable (no fault, no hang).

sa_self_test_timeout makes one bounded mbarrier wait run out on purpose (an
mbarrier that nothing arrives on, a limit of about a millisecond), through the
same wait the attention kernels use.  The error word must then read
SA_ERR_TIMEOUT once, be cleared by that read, and the next real call must run
and match the oracle.
"""
import time

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import masked_attention
from _parity import check_o, check_lse

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def test_bounded_wait_timeout_is_reported_then_cleared(lib):
    stream = torch.cuda.current_stream()
    ops.sa_get_device_status(stream)                       # start from a clean error word
    t0 = time.perf_counter()
    assert lib.sa_self_test_timeout(1_000_000, stream.cuda_stream) == ops.SA_OK
    assert lib.sa_get_device_status(stream.cuda_stream) == ops.SA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert elapsed < 2.0, f"the 1 ms wait took {elapsed:.3f} s"
    assert lib.sa_get_device_status(stream.cuda_stream) == ops.SA_OK   # the read cleared it
    # the context is still usable: a normal call runs and is right
    B, H, N, d, block = 1, 2, 640, 128, 128
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=61)
    lse = torch.empty(B, H, N, device="cuda")
    o = ops.sa_sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), block, lse=lse)
    assert lib.sa_get_device_status(stream.cuda_stream) == ops.SA_OK
    Or, Lr = masked_attention(q, k, v, block, np.ones((N // block, N // block), dtype=np.uint8))
    check_o(o.cpu(), Or, "after the timeout self-test")
    check_lse(lse.cpu(), Lr, "after the timeout self-test")


def test_timeout_reported_through_the_binding(lib):
    ops.sa_self_test_timeout(200_000)
    with pytest.raises(ops.SparseAttnError) as e:
        ops.sa_get_device_status()
    assert e.value.status == ops.SA_ERR_TIMEOUT
    ops.sa_get_device_status()                              # cleared: no error now
