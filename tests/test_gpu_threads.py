"""Two host threads making their first calls at once (B200).

The library caches a few things per device on first use (the SM count, the
driver's tensor-map encoder, each kernel's shared-memory attribute).  In a
fresh process, two threads start at a barrier and each make their first
attention calls together, on streams of their own, for kernels that no call
in the process has launched yet; their outputs must equal those of a later
serial run byte for byte.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = textwrap.dedent('''
    import sys, threading
    sys.path[:0] = [{root!r}, {tests!r}]
    import torch
    import synth
    from gpu_cases import DeviceCase
    import verify_paged_gqa_b200 as tf

    # decode on the position-major kernel, head dim 512 decode on the CUDA-core
    # kernel, and a prompt chunk on the row-major kernel: one case per thread
    # pair, set up before any attention call (the row writes only)
    specs = [(128, 4, 1, [3000, 700]), (512, 4, 1, [2100, 900]), (128, 4, 100, [1300, 600])]
    cases = []
    for i, (d, G, W, lens) in enumerate(specs):
        w = synth.Workload("threads", 0, 2, G, d, 512, W, seed=12000 + i)
        cases.append(DeviceCase(synth.make_case(w, lens=lens, rows=W)))
    torch.cuda.synchronize()
    outs = {{}}
    errors = []
    gate = threading.Barrier(2)

    def worker(k):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                bufs = [(dc.workspace(dc.q.shape[1]),
                         torch.empty(dc.q.shape, dtype=torch.float32, device="cuda"))
                        for dc in cases]
                s.synchronize()
                gate.wait()
                for i, dc in enumerate(cases):
                    outs[(k, i)] = dc.attend(ws=bufs[i][0], out=bufs[i][1])
                s.synchronize()
        except Exception as e:  # reported by the main thread
            errors.append(repr(e))

    ts = [threading.Thread(target=worker, args=(k,)) for k in range(2)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    for i, dc in enumerate(cases):
        ref = dc.attend()
        torch.cuda.synchronize()
        for k in range(2):
            assert torch.equal(outs[(k, i)], ref), (k, i)
    print("threads ok")
''')


def test_two_threads_make_their_first_calls_at_once():
    script = _SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "threads ok" in r.stdout
