"""The kernels' failure path, driven without faulting, trapping or hanging
the GPU (B200).

Every pipeline wait in the attention kernels is bounded.  The test hook
tf_testing_paged_attn (include/tf_paged_testing.h) gives a call a short wait
limit (about 10 ms) and makes CTA 0 withhold one arrival that no copy or MMA
completes: the softmax warps' "P is written" arrival of their first tile on
the tensor-core kernels (whose ring is filled by TMA, or gathered row by row
for pages that are not a multiple of 128), the release of the first ring
stage on the CUDA-core kernel.  The wait on it must run out: the call returns, its status word holds
TF_DEV_TIMEOUT and a wait-site bit, and the next ordinary call on the same
stream and workspace matches the oracle with a clean status word.
"""
import time

import pytest
import torch

import oracle
import synth
from gpu_cases import TOL, DeviceCase, max_abs

pytestmark = pytest.mark.gpu

SHORT_LIMIT = 20_000_000   # SM cycles: about 10 ms at B200 clocks


@pytest.mark.parametrize("name,d,G,P,W,lens", [
    ("decode, position-major kernel (two issuers)", 128, 4, 512, 1, [60000, 3000]),
    ("verify, position-major kernel (64-row blocks)", 128, 8, 512, 8, [60000, 3000]),
    ("head dim 512 verify, position-major kernel (one issuer)", 512, 8, 512, 4, [30000, 3000]),
    ("prompt chunk, row-major kernel", 128, 4, 512, 200, [60000, 3000]),
    ("pages of 64, position-major kernel (tiles gathered across pages)", 128, 4, 64, 1,
     [60000, 3000]),
    ("head dim 512 decode, CUDA-core kernel", 512, 4, 512, 1, [60000, 3000]),
])
def test_a_withheld_arrival_times_out_and_the_next_call_is_clean(name, d, G, P, W, lens):
    import verify_paged_gqa_b200 as tf
    w = synth.Workload("fail", 0, 1, G, d, P, W, seed=13000 + d + G + P + W)
    case = synth.make_case(w, lens=lens, rows=W)
    dc = DeviceCase(case)
    ws = dc.workspace(W)
    assert tf.tf_workspace_status(ws) == 0
    out = torch.zeros(dc.q.shape, dtype=torch.float32, device="cuda")
    t0 = time.monotonic()
    tf.tf_testing_paged_attn(dc.k_pool, dc.v_pool, dc.table, dc.lens, dc.q, w.scale, out, ws,
                             dc.max_len, SHORT_LIMIT, 1)
    torch.cuda.synchronize()
    took = time.monotonic() - t0
    site = int(ws[4:8].view(torch.int32).item())
    ws[4:8].zero_()
    flags = tf.tf_workspace_status(ws)
    assert flags & tf.TF_DEV_TIMEOUT, (name, flags)
    assert site != 0, name
    assert took < 10.0, (name, took)
    # the same call with nothing withheld and the short limit runs clean
    tf.tf_testing_paged_attn(dc.k_pool, dc.v_pool, dc.table, dc.lens, dc.q, w.scale, out, ws,
                             dc.max_len, SHORT_LIMIT, 0)
    torch.cuda.synchronize()
    assert tf.tf_workspace_status(ws) == 0, name
    # and so does the next library call on the same stream and workspace
    got = dc.attend(ws=ws)
    torch.cuda.synchronize()
    assert tf.tf_workspace_status(ws) == 0, name
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, w.group, w.scale,
                        threads=8)
    assert max_abs(got, ref) <= TOL, name
    assert max_abs(out, ref) <= TOL, name


def test_testing_hook_refuses_settings_out_of_range():
    import verify_paged_gqa_b200 as tf
    w = synth.Workload("fail", 0, 1, 4, 128, 512, 1, seed=13100)
    dc = DeviceCase(synth.make_case(w, lens=[1000]))
    ws = dc.workspace(1)
    out = torch.empty(dc.q.shape, dtype=torch.float32, device="cuda")
    for limit, withhold in ((10, 0), (8_000_000_000, 0), (SHORT_LIMIT, 2)):
        with pytest.raises(tf.TFError):
            tf.tf_testing_paged_attn(dc.k_pool, dc.v_pool, dc.table, dc.lens, dc.q, w.scale,
                                     out, ws, dc.max_len, limit, withhold)
