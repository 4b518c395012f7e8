"""The forward kernels' clock record (`fa_clock_record`): every CTA of a bf16
or E4M3 forward launch adds its SM cycles, its timer nanoseconds and itself
to three counters; the no-alloc forward adds nothing.  Checked by counting
CTAs against the persistent grid (one CTA per 256-row unit, at most one per
SM) and by the clock lying in the range any B200 runs at."""
import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _grid(B, H, N, rows):
    units = B * H * ((N + rows - 1) // rows)
    return min(units, torch.cuda.get_device_properties(0).multi_processor_count)


@pytest.mark.parametrize("which,rows", [(1, 256), (2, 128)], ids=["two_tile", "one_tile"])
def test_clock_record_counts_every_cta(which, rows, force_kernel):
    fa_build.build()
    force_kernel(which)
    B, H, N, d = 1, 4, 1000, 128  # a grid smaller than the SM count
    q, k, v = (x.cuda() for x in W.random_qkv(B, H, N, d, torch.bfloat16, seed=5))
    fa.clock_record(reset=True)
    for _ in range(3):
        fa.forward(q, k, v, causal=True)
    rec = fa.clock_record(reset=True)
    assert rec["ctas"] == 3 * _grid(B, H, N, rows)
    assert rec["cycles"] > 0 and rec["ns"] > 0
    assert 200.0 < rec["sm_mhz"] < 2500.0
    assert fa.clock_record(reset=False)["ctas"] == 0  # cleared by the reset


def test_clock_record_full_grid_and_fp8_and_noalloc():
    fa_build.build()
    B, H, N, d = 2, 32, 2048, 128  # 512 two-tile units: one CTA per SM
    q, k, v = (x.cuda() for x in W.random_qkv(B, H, N, d, torch.bfloat16, seed=6))
    fa.clock_record(reset=True)
    fa.forward(q, k, v, causal=False)
    rec = fa.clock_record(reset=True)
    assert rec["ctas"] == _grid(B, H, N, 256)
    # every CTA runs from the first unit to the queue's end: its cycles are
    # close to the launch's, so the per-CTA figure and the clock agree
    assert rec["cycles_per_cta"] > 0
    assert 200.0 < rec["sm_mhz"] < 2500.0

    q8, k8, v8 = (x.to(torch.float8_e4m3fn) for x in (q, k, v))
    fa.forward_fp8(q8, k8, v8, causal=True)
    assert fa.clock_record(reset=True)["ctas"] == _grid(B, H, N, 256)

    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    s = torch.cuda.current_stream().cuda_stream
    rc = fa.library().fa_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                     B, H, N, d, d ** -0.5, 1, fa.FA_DTYPE_BF16, s)
    assert rc == fa.FA_OK
    assert fa.clock_record(reset=True)["ctas"] == 0
    assert fa.library().fa_noalloc_check_status(s) == fa.FA_OK
