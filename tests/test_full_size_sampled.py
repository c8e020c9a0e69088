"""Every benchmarked workload at its full size, in the launch configuration
bench.py times (its device set-up, its step), checked against the fp64 oracle
on sampled output rows the oracle computes one by one (B200).

The oracle's inputs are the seeded generator's values for the sampled streams,
drawn again here; nothing is read back from the pools the CUDA path wrote."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import TOL

pytestmark = pytest.mark.gpu

WORKLOADS = ["decode_12x40k", "verify_4x131k", "hd512_verify", "prompt_9216", "gqa12_verify",
             "gqa16_hd512_decode", "hd256_verify", "tree_verify_4x131k", "decode_12x40k_p37"]


@pytest.mark.parametrize("name", WORKLOADS)
def test_full_size_sampled_rows(name):
    import bench
    wl = bench.Workload(name, "cuda:0")
    wl.step()
    torch.cuda.synchronize()
    wl.check_flags()
    w = wl.w
    out = wl.out.cpu().numpy().astype(np.float64)
    q_all = synth.to_bits(wl.q)                    # [S][W][Hq][d] (the prompt: [1][L][Hq][d])
    S, W, Hq = q_all.shape[:3]
    rng = np.random.default_rng(abs(hash(name)) % (2**32))
    streams = sorted(set(int(x) for x in rng.choice(S, size=min(2, S), replace=False)))
    if w.prompt_len:
        # rows of the first and the last chunk
        rows = sorted(set(int(x) for x in rng.choice(w.rows, 3, replace=False)) |
                      set(int(x) for x in W - w.rows + rng.choice(w.rows, 3, replace=False)))
    else:
        rows = sorted(set(int(x) for x in rng.choice(W, size=min(3, W), replace=False)))
    heads = sorted(set(int(x) for x in rng.choice(Hq, size=min(4, Hq), replace=False)))
    tree = getattr(wl, "tree_np", None)
    worst = 0.0
    for s in streams:
        n = int(wl.lens_np[s])
        k, v = synth.kv_rows_torch(w, s, n, "cuda")
        k_lin, v_lin = synth.to_bits(k), synth.to_bits(v)
        del k, v
        units = np.array([(0, r, h) for r in rows for h in heads], dtype=np.int32)
        ref = oracle.attend(q_all[s:s + 1], [k_lin], [v_lin], [n], W, w.group, w.scale,
                            units=units, threads=8,
                            tree=None if tree is None else tree[s:s + 1])
        got = np.stack([out[s, r, h] for r in rows for h in heads])
        assert np.isfinite(got).all()
        worst = max(worst, float(np.abs(got - ref).max()))
    print(f"{name}: {len(streams)} streams x {len(rows)} rows x {len(heads)} heads sampled, "
          f"max-abs {worst:.2e}")
    assert 0.0 < worst <= TOL, (name, worst)
