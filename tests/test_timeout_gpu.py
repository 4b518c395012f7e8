"""Failure detection without a GPU fault: a test hook makes one CTA skip one
arrival, so one of the kernel's bounded waits (about two seconds) runs out.
The kernel must report FA_ERR_DEVICE_TIMEOUT through the status word, leave
the context usable, and the next call must be correct again."""
import math

import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [1, 2], ids=["two_tile", "one_tile"])
def test_bounded_wait_runs_out_and_is_reported(which, force_kernel):
    fa_build.build()
    lib = fa.library()
    force_kernel(which)
    q, k, v = (x.cuda() for x in W.random_qkv(1, 2, 512, 128, torch.bfloat16, seed=71))
    fa.check_device_status()  # start clean
    assert lib.fa_test_skip_one_arrival() == fa.FA_OK
    o, lse = fa.forward(q, k, v, causal=True)
    with pytest.raises(fa.FaError) as e:
        fa.check_device_status()
    assert e.value.status == fa.FA_ERR_DEVICE_TIMEOUT
    # the status was cleared, the context still works, and results are right again
    fa.check_device_status()
    o, lse = fa.forward(q, k, v, causal=True)
    fa.check_device_status()
    o_ref, lse_ref = oracle.attention_fwd(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                          v.float().cpu().numpy(), 1 / math.sqrt(128), True)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 1e-2
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-3
