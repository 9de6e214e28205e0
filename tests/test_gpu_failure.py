"""Device-side failure path of the kernels, exercised without any fault.

Every wait of a kernel on a pipeline barrier is bounded: when one runs out, the kernel records
SEP_ERR_TIMEOUT in the sticky device error word, lets the copies and tensor-core work it issued
finish, frees its tensor memory and returns. Here a forward launch is given a pipeline-wait
limit of a few nanoseconds, so its waits give up part-way through a normal launch; the test
checks that the call returns, that the error word reports the timeout, and that the next call
on the same device, with the default limit, runs normally and matches the fp64 oracle (so no
tensor memory, barrier or copy was left behind).
"""

import pytest

from gpu_common import check_lse, check_out, f64
from oracle import sepattn_ref as R

pytestmark = pytest.mark.gpu

SEP_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


@pytest.mark.parametrize("d", [64, 128])
def test_forward_wait_runs_out_then_device_recovers(S, d):
    import torch
    import workloads
    B, L, Hq, Hkv, a, n = 1, 2048, 8, 2, 4, 64
    inp = workloads.small_attn_inputs(31 + d, B, L, Hq, Hkv, d, p=0.1)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    mask = S.sep_mask_build(dev["sep"], a, n)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    S.sep_set_wait_limit_ns(2)
    try:
        S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
        torch.cuda.synchronize()
        status = S.sep_last_device_error()
    finally:
        S.sep_set_wait_limit_ns(0)
    assert status == SEP_ERR_TIMEOUT
    assert S.sep_last_device_error() == 0  # the word was cleared by the read
    # the same launch again, default limit: complete and correct
    for _ in range(2):
        o, lse = S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
        torch.cuda.synchronize()
        assert S.sep_last_device_error() == 0
    Or, LSEr = R.attn_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), inp["sep"].numpy(), a, n,
                          d ** -0.5)
    check_out(f64(o), Or, "O after recovery")
    check_lse(f64(lse), LSEr, "LSE after recovery")
