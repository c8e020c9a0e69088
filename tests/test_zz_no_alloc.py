"""tf_paged_attn_decode_noalloc: the decode entry point that allocates nothing.

Callers that cannot allocate device memory (a plug-in that only receives its
input and output buffers from the engine hosting it, or a serving loop that
must not call cudaMalloc once running) use this call; its split-context
scratch is a static array inside the library.  This file runs last, so a
failure here leaves every other test already run.  It checks, through the C
ABI, that two calls in a row give the workspace entry point's output byte
for byte (both run the same plan and kernels) and match the fp64 oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import TOL, DeviceCase, max_abs

pytestmark = pytest.mark.gpu


def _fn(tf):
    from verify_paged_gqa_b200 import _abi
    fn = tf.raw.tf_paged_attn_decode_noalloc
    fn.argtypes = [ctypes.POINTER(_abi.tf_kv_pool), ctypes.POINTER(_abi.tf_streams),
                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p,
                   ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _noalloc(tf, dc, q, out):
    from verify_paged_gqa_b200 import _abi
    pool = _abi.tf_kv_pool(dc.k_pool.data_ptr(), dc.v_pool.data_ptr(), *dc.k_pool.shape)
    st = _abi.tf_streams(dc.table.data_ptr(), dc.table.shape[1], dc.lens.data_ptr(),
                         dc.table.shape[0], dc.max_len)
    return _fn(tf)(ctypes.byref(pool), ctypes.byref(st), q.data_ptr(), q.shape[2],
                   float(dc.w.scale), out.data_ptr(),
                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("d,G,lens", [(128, 4, [40960, 9000, 513]), (512, 8, [3000, 9216])])
def test_noalloc_decode_matches_workspace_decode_twice(d, G, lens):
    import verify_paged_gqa_b200 as tf
    w = synth.Workload("noalloc", 0, 2, G, d, 512, 1, seed=8000 + d)
    case = synth.make_case(w, lens=lens)
    dc = DeviceCase(case)
    ref = dc.attend(kind="decode")
    exact = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, 1, w.group, w.scale,
                          threads=8)
    for _ in range(2):
        out = torch.full(dc.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(tf, dc, dc.q, out) == tf.TF_OK
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)
        assert max_abs(out, exact) <= TOL


def test_noalloc_call_without_streams_takes_null_buffers():
    """As with tf_paged_attn_decode, a call with no streams reads and writes
    nothing: null table, lens, query and output are accepted."""
    import verify_paged_gqa_b200 as tf
    from verify_paged_gqa_b200 import _abi
    k_pool = torch.zeros((2, 1, 512, 128), dtype=torch.bfloat16, device="cuda")
    pool = _abi.tf_kv_pool(k_pool.data_ptr(), k_pool.data_ptr(), 2, 1, 512, 128)
    st = _abi.tf_streams(None, 1, None, 0, 512)
    rc = _fn(tf)(ctypes.byref(pool), ctypes.byref(st), None, 4, 0.088, None,
                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == tf.TF_OK


def test_noalloc_refuses_a_plan_beyond_its_scratch():
    import verify_paged_gqa_b200 as tf
    # 64 query heads on one KV head at head dim 512: two row blocks of 32 rows,
    # and two partial slots of 32 x 514 floats per CTA -- more than 8 MiB
    w = synth.Workload("noalloc_big", 0, 1, 64, 512, 512, 1, seed=8100)
    S, L = 4, 4096
    k_pool = torch.empty((S * L // 512, 1, 512, 512), dtype=torch.bfloat16, device="cuda")
    table = torch.arange(S * L // 512, dtype=torch.int32, device="cuda").view(S, L // 512)
    lens = torch.full((S,), L, dtype=torch.int32, device="cuda")
    q = torch.zeros((S, 1, 64, 512), dtype=torch.bfloat16, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")

    class _DC:
        pass
    dc = _DC()
    dc.k_pool = dc.v_pool = k_pool
    dc.table, dc.lens, dc.max_len, dc.w = table, lens, L, w
    need = tf.tf_paged_attn_workspace_bytes(k_pool, k_pool, table, lens, 64, 1, L)
    assert need > (8 << 20)
    assert _noalloc(tf, dc, q, out) == tf.TF_ENOSPACE
