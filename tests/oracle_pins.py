"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an optional compiled oracle library (``lib``) so
the same checks can be run against copies of the oracle with a planted
mistake (see test_oracle_planted.py).  A pin raises AssertionError (or the
oracle's ValueError) when it fails.

What pins what:
  * hand-derived worked examples (tests/golden/hand_examples.json): exact
    fractions for two keys, a two-row causal window, grouped heads;
  * brute force on tiny inputs: a separate pure-Python formulation (full
    score matrix, explicit mask, no max subtraction, math.fsum);
  * a library routine: torch's scaled_dot_product_attention in fp64 with its
    grouped-query option and an explicit window mask;
  * closed forms: constant values, one visible key, zero query, a dominant
    key;
  * invariants: causality, verify row == decode at that position, thread
    count does not change a bit;
  * the row write: per-element brute force on a tiny pool, untouched bytes;
  * tree masks: a hand-derived tree with siblings, brute force and torch's
    attention with the explicit mask, every tree row equal (to the bit) to a
    decode over the keys on its path, and chain masks equal to the causal
    window;
  * the state copy: per-element brute force over tiny pools with different
    page sizes (untouched bytes included), a round trip through a linear
    buffer checked against numpy gathers, and agreement with the row write
    putting the same rows into the same pages.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf(x):
    return synth.bf16_from_f32(np.asarray(x, dtype=np.float32))


def _f64(b):
    return synth.f32_from_bf16(b).astype(np.float64)


def _random_case(rng, S, W, Hkv, G, d, lens, sigma=1.0):
    q = _bf(rng.standard_normal((S, W, Hkv * G, d)))
    k = [_bf(sigma * rng.standard_normal((n, Hkv, d))) for n in lens]
    v = [_bf(sigma * rng.standard_normal((n, Hkv, d))) for n in lens]
    return q, k, v


def pin_hand_examples(lib=None):
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        data = json.load(f)
    scales = {"ln2": math.log(2.0), "ln3": math.log(3.0), "1": 1.0}
    for ex in data["examples"]:
        q = _bf(ex["q"])
        k = [_bf(x) for x in ex["k"]]
        v = [_bf(x) for x in ex["v"]]
        tree = np.array(ex["tree"], dtype=np.uint8) if "tree" in ex else None
        out = oracle.attend(q, k, v, ex["lens"], ex["W"], ex["G"], scales[ex["scale"]], lib=lib,
                            tree=tree)
        np.testing.assert_allclose(out, np.array(ex["out"]), rtol=0, atol=1e-13,
                                   err_msg=ex["name"])


def brute_force(q, k, v, lens, W, G, scale, tree=None):
    """Pure-Python attention: full score matrix, explicit mask, no max shift."""
    S, _, Hq, d = q.shape
    qf = _f64(q)
    out = np.zeros(q.shape, dtype=np.float64)
    for s in range(S):
        kf, vf = _f64(k[s]), _f64(v[s])
        n = lens[s]
        for r in range(W):
            for h in range(Hq):
                g = h // G
                e = []
                for j in range(n):
                    if tree is None:
                        visible = j <= n - W + r
                    else:
                        visible = j < n - W or (int(tree[s][r]) >> (j - (n - W))) & 1 == 1
                    if visible:
                        x = scale * math.fsum(qf[s, r, h, i] * kf[j, g, i] for i in range(d))
                        e.append((j, math.exp(x)))
                z = math.fsum(w for _, w in e)
                for i in range(d):
                    out[s, r, h, i] = math.fsum(w * vf[j, g, i] for j, w in e) / z
    return out


def pin_brute_force(lib=None):
    rng = np.random.default_rng(11)
    for (S, W, Hkv, G, d, lens) in [(1, 1, 1, 1, 4, [1]), (2, 3, 2, 2, 4, [3, 6]),
                                    (2, 2, 1, 4, 8, [5, 2]), (1, 3, 2, 1, 3, [4])]:
        q, k, v = _random_case(rng, S, W, Hkv, G, d, lens)
        scale = 1.0 / math.sqrt(d)
        got = oracle.attend(q, k, v, lens, W, G, scale, lib=lib)
        want = brute_force(q, k, v, lens, W, G, scale)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def pin_sdpa(lib=None):
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(12)
    for (S, W, Hkv, G, d, lens) in [(3, 4, 2, 4, 16, [4, 37, 9]), (2, 8, 1, 8, 32, [8, 70]),
                                    (1, 1, 3, 2, 8, [50])]:
        q, k, v = _random_case(rng, S, W, Hkv, G, d, lens)
        scale = 1.0 / math.sqrt(d)
        got = oracle.attend(q, k, v, lens, W, G, scale, lib=lib)
        for s in range(S):
            n = lens[s]
            qt = torch.from_numpy(_f64(q[s])).permute(1, 0, 2)[None]          # [1,Hq,W,d]
            kt = torch.from_numpy(_f64(k[s])).permute(1, 0, 2)[None]          # [1,Hkv,n,d]
            vt = torch.from_numpy(_f64(v[s])).permute(1, 0, 2)[None]
            pos = torch.arange(n)[None, :]
            rowpos = (n - W + torch.arange(W))[:, None]
            mask = pos <= rowpos                                              # [W, n]
            ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                                 enable_gqa=True)
            np.testing.assert_allclose(got[s], ref[0].permute(1, 0, 2).numpy(), rtol=0,
                                       atol=1e-12)


def pin_closed_forms(lib=None):
    rng = np.random.default_rng(13)
    S, W, Hkv, G, d = 2, 3, 2, 4, 16
    lens = [7, 3]
    q, k, v = _random_case(rng, S, W, Hkv, G, d, lens)
    scale = 1.0 / math.sqrt(d)
    # constant values: the output is that constant whatever the weights
    vc = [np.full_like(x, _bf([1.5])[0]) for x in v]
    out = oracle.attend(q, k, vc, lens, W, G, scale, lib=lib)
    np.testing.assert_allclose(out, 1.5, rtol=0, atol=1e-14)
    # one visible key (len == W == 1): the output is that key's value
    q1, k1, v1 = _random_case(rng, 2, 1, Hkv, G, d, [1, 1])
    out = oracle.attend(q1, k1, v1, [1, 1], 1, G, scale, lib=lib)
    for s in range(2):
        for h in range(Hkv * G):
            np.testing.assert_allclose(out[s, 0, h], _f64(v1[s][0, h // G]), rtol=0, atol=0)
    # zero query: uniform weights, the output is the mean of the visible values
    q0 = np.zeros_like(q)
    out = oracle.attend(q0, k, v, lens, W, G, scale, lib=lib)
    for s in range(S):
        for r in range(W):
            t = lens[s] - W + r
            for h in range(Hkv * G):
                want = _f64(v[s][: t + 1, h // G]).mean(axis=0)
                np.testing.assert_allclose(out[s, r, h], want, rtol=0, atol=1e-13)
    # a dominant key: one visible key's score sits 40 above the rest -> its value
    d2 = 8
    n = 6
    qd = np.zeros((1, 1, 1, d2), dtype=np.uint16)
    qd[0, 0, 0, 0] = _bf([1.0])[0]
    kd = np.zeros((n, 1, d2), dtype=np.uint16)
    kd[3, 0, 0] = _bf([40.0])[0]
    vd = _bf(rng.standard_normal((n, 1, d2)))
    out = oracle.attend(qd, [kd], [vd], [n], 1, 1, 1.0, lib=lib)
    np.testing.assert_allclose(out[0, 0, 0], _f64(vd[3, 0]), rtol=0, atol=1e-15 + 12 * math.exp(-40) * 8)


def pin_invariants(lib=None):
    rng = np.random.default_rng(14)
    S, W, Hkv, G, d = 2, 4, 2, 2, 16
    lens = [9, 20]
    q, k, v = _random_case(rng, S, W, Hkv, G, d, lens)
    scale = 0.25
    base = oracle.attend(q, k, v, lens, W, G, scale, lib=lib)
    # causality: changing K/V at positions after row r leaves row r unchanged, and
    # changing the position of row r itself changes it
    for s in range(S):
        for r in range(W):
            t = lens[s] - W + r
            k2 = [x.copy() for x in k]
            v2 = [x.copy() for x in v]
            k2[s][t + 1:] = _bf(rng.standard_normal(k2[s][t + 1:].shape))
            v2[s][t + 1:] = _bf(rng.standard_normal(v2[s][t + 1:].shape))
            out = oracle.attend(q, k2, v2, lens, W, G, scale, lib=lib)
            np.testing.assert_array_equal(out[s, r], base[s, r])
            v3 = [x.copy() for x in v]
            v3[s][t] = _bf(_f64(v3[s][t]) + 3.0)
            out = oracle.attend(q, k, v3, lens, W, G, scale, lib=lib)
            assert np.abs(out[s, r] - base[s, r]).max() > 1e-6
    # verify row r == decode of that row alone with len' = len - W + r + 1
    for r in range(W):
        lens_r = [n - W + r + 1 for n in lens]
        out = oracle.attend(q[:, r:r + 1].copy(), [x[:n] for x, n in zip(k, lens_r)],
                            [x[:n] for x, n in zip(v, lens_r)], lens_r, 1, G, scale, lib=lib)
        np.testing.assert_allclose(out[:, 0], base[:, r], rtol=0, atol=1e-14)
    # the thread count changes no bit
    out4 = oracle.attend(q, k, v, lens, W, G, scale, threads=4, lib=lib)
    np.testing.assert_array_equal(out4, base)


def pin_put_rows(lib=None):
    rng = np.random.default_rng(15)
    n_pages, Hkv, P, d = 7, 2, 4, 3
    lens = np.array([6, 9], dtype=np.int32)
    W = 3
    table = np.array([[5, 1, 6], [0, 3, 2]], dtype=np.int32)
    kp = np.full((n_pages, Hkv, P, d), synth.BF16_NAN, dtype=np.uint16)
    vp = kp.copy()
    kr = rng.integers(0, 0x7F00, size=(2, W, Hkv, d)).astype(np.uint16)
    vr = rng.integers(0, 0x7F00, size=(2, W, Hkv, d)).astype(np.uint16)
    oracle.put_rows(kp, vp, table, lens, kr, vr, lib=lib)
    want_k = np.full_like(kp, synth.BF16_NAN)
    want_v = want_k.copy()
    for s in range(2):
        for r in range(W):
            pos = int(lens[s]) - W + r
            for h in range(Hkv):
                for i in range(d):
                    want_k[table[s][pos // P], h, pos % P, i] = kr[s, r, h, i]
                    want_v[table[s][pos // P], h, pos % P, i] = vr[s, r, h, i]
    np.testing.assert_array_equal(kp, want_k)
    np.testing.assert_array_equal(vp, want_v)


def _tree_case(rng, S, W, Hkv, G, d, lens, key):
    q, k, v = _random_case(rng, S, W, Hkv, G, d, lens)
    return q, k, v, synth.tree_masks(key, S, W)


def _visible(n, W, mask):
    return [j for j in range(n) if j < n - W or (int(mask) >> (j - (n - W))) & 1]


def pin_tree_brute_force(lib=None):
    rng = np.random.default_rng(16)
    for i, (S, W, Hkv, G, d, lens) in enumerate([(2, 4, 1, 2, 4, [5, 4]), (1, 8, 2, 1, 4, [11]),
                                                  (3, 3, 1, 3, 3, [3, 7, 4])]):
        q, k, v, tree = _tree_case(rng, S, W, Hkv, G, d, lens, (99, i))
        scale = 1.0 / math.sqrt(d)
        got = oracle.attend(q, k, v, lens, W, G, scale, lib=lib, tree=tree)
        want = brute_force(q, k, v, lens, W, G, scale, tree=tree)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def pin_tree_sdpa(lib=None):
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(17)
    for i, (S, W, Hkv, G, d, lens) in enumerate([(3, 8, 2, 4, 16, [8, 40, 19]),
                                                  (2, 5, 1, 8, 32, [9, 70])]):
        q, k, v, tree = _tree_case(rng, S, W, Hkv, G, d, lens, (98, i))
        scale = 1.0 / math.sqrt(d)
        got = oracle.attend(q, k, v, lens, W, G, scale, lib=lib, tree=tree)
        for s in range(S):
            n = lens[s]
            qt = torch.from_numpy(_f64(q[s])).permute(1, 0, 2)[None]
            kt = torch.from_numpy(_f64(k[s])).permute(1, 0, 2)[None]
            vt = torch.from_numpy(_f64(v[s])).permute(1, 0, 2)[None]
            mask = torch.zeros((W, n), dtype=torch.bool)
            for r in range(W):
                mask[r, _visible(n, W, tree[s][r])] = True
            ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                                 enable_gqa=True)
            np.testing.assert_allclose(got[s], ref[0].permute(1, 0, 2).numpy(), rtol=0,
                                       atol=1e-12)


def pin_tree_paths(lib=None):
    # a tree row attends exactly to the keys on its root path: the same as one
    # decode row over a cache holding only those keys, in order (to the bit)
    rng = np.random.default_rng(18)
    S, W, Hkv, G, d = 3, 8, 2, 2, 8
    lens = [8, 21, 13]
    q, k, v, tree = _tree_case(rng, S, W, Hkv, G, d, lens, (97, 0))
    scale = 0.3
    got = oracle.attend(q, k, v, lens, W, G, scale, lib=lib, tree=tree)
    for s in range(S):
        for r in range(W):
            vis = _visible(lens[s], W, tree[s][r])
            out = oracle.attend(q[s:s + 1, r:r + 1].copy(), [k[s][vis]], [v[s][vis]], [len(vis)],
                                1, G, scale, lib=lib)
            np.testing.assert_array_equal(out[0, 0], got[s, r])
    # chain masks are the causal window, to the bit
    base = oracle.attend(q, k, v, lens, W, G, scale, lib=lib)
    chain = oracle.attend(q, k, v, lens, W, G, scale, lib=lib, tree=synth.chain_masks(S, W))
    np.testing.assert_array_equal(chain, base)
    # and a tree with a branch differs from it
    assert np.abs(got - base).max() > 1e-3


def _state_pool(rng, n_pages, Hkv, P, d, fill=None):
    if fill is not None:
        k = np.full((n_pages, Hkv, P, d), fill, dtype=np.uint16)
        return k, k.copy()
    return (rng.integers(0, 0x7F7F, size=(n_pages, Hkv, P, d)).astype(np.uint16),
            rng.integers(0, 0x7F7F, size=(n_pages, Hkv, P, d)).astype(np.uint16))


def _gather_linear(pool, table, n):
    """Stream positions 0..n-1 of one table row, by numpy indexing: [n][Hkv][d]."""
    P = pool.shape[2]
    pages = np.asarray(table)[np.arange(n) // P]
    return pool[pages, :, np.arange(n) % P, :]


def pin_copy_state_brute(lib=None):
    rng = np.random.default_rng(19)
    Hkv, d = 2, 3
    lens = np.array([7, 4, 0], dtype=np.int32)
    sk, sv = _state_pool(rng, 9, Hkv, 3, d)
    st = np.array([[4, 0, 7], [8, 2, 5], [1, 3, 6]], dtype=np.int32)
    dk, dv = _state_pool(rng, 6, Hkv, 5, d, fill=synth.BF16_NAN)
    dt = np.array([[3, 1], [0, 5], [2, 4]], dtype=np.int32)
    oracle.copy_state(sk, sv, st, dk, dv, dt, lens, lib=lib)
    want_k = np.full_like(dk, synth.BF16_NAN)
    want_v = want_k.copy()
    for s in range(3):
        for j in range(int(lens[s])):
            for h in range(Hkv):
                for i in range(d):
                    want_k[dt[s][j // 5], h, j % 5, i] = sk[st[s][j // 3], h, j % 3, i]
                    want_v[dt[s][j // 5], h, j % 5, i] = sv[st[s][j // 3], h, j % 3, i]
    np.testing.assert_array_equal(dk, want_k)
    np.testing.assert_array_equal(dv, want_v)


def pin_copy_state_round_trip(lib=None):
    # pages of 4 -> a linear buffer (one page of 16 per stream) -> pages of 7
    rng = np.random.default_rng(20)
    Hkv, d = 3, 4
    lens = np.array([13, 16, 1], dtype=np.int32)
    sk, sv = _state_pool(rng, 14, Hkv, 4, d)
    st = rng.permutation(14)[:12].reshape(3, 4).astype(np.int32)
    lk, lv = _state_pool(rng, 3, Hkv, 16, d, fill=synth.BF16_NAN)
    lt = np.array([[2], [0], [1]], dtype=np.int32)
    oracle.copy_state(sk, sv, st, lk, lv, lt, lens, lib=lib)
    for s in range(3):
        n = int(lens[s])
        np.testing.assert_array_equal(lk[lt[s][0], :, :n].transpose(1, 0, 2),
                                      _gather_linear(sk, st[s], n))
        np.testing.assert_array_equal(lv[lt[s][0], :, :n].transpose(1, 0, 2),
                                      _gather_linear(sv, st[s], n))
        assert (lk[lt[s][0], :, n:] == synth.BF16_NAN).all()
    dk, dv = _state_pool(rng, 10, Hkv, 7, d, fill=synth.BF16_NAN)
    dt = rng.permutation(10)[:9].reshape(3, 3).astype(np.int32)
    oracle.copy_state(lk, lv, lt, dk, dv, dt, lens, lib=lib)
    for s in range(3):
        n = int(lens[s])
        np.testing.assert_array_equal(_gather_linear(dk, dt[s], n), _gather_linear(sk, st[s], n))
        np.testing.assert_array_equal(_gather_linear(dv, dt[s], n), _gather_linear(sv, st[s], n))


def pin_copy_state_matches_put_rows(lib=None):
    # resuming a linear state into pages is the row write of all its rows
    rng = np.random.default_rng(21)
    Hkv, d, P = 2, 5, 3
    lens = np.array([8, 8], dtype=np.int32)
    lk, lv = _state_pool(rng, 2, Hkv, 8, d)
    lt = np.array([[1], [0]], dtype=np.int32)
    dt = np.array([[5, 0, 3], [2, 6, 4]], dtype=np.int32)
    ak, av = _state_pool(rng, 7, Hkv, P, d, fill=synth.BF16_NAN)
    oracle.copy_state(lk, lv, lt, ak, av, dt, lens, lib=lib)
    bk, bv = _state_pool(rng, 7, Hkv, P, d, fill=synth.BF16_NAN)
    rows_k = np.stack([lk[lt[s][0]].transpose(1, 0, 2) for s in range(2)])   # [S][8][Hkv][d]
    rows_v = np.stack([lv[lt[s][0]].transpose(1, 0, 2) for s in range(2)])
    oracle.put_rows(bk, bv, dt, lens, rows_k, rows_v, lib=lib)
    np.testing.assert_array_equal(ak, bk)
    np.testing.assert_array_equal(av, bv)


ALL_PINS = [pin_hand_examples, pin_brute_force, pin_sdpa, pin_closed_forms, pin_invariants,
            pin_put_rows, pin_tree_brute_force, pin_tree_sdpa, pin_tree_paths,
            pin_copy_state_brute, pin_copy_state_round_trip, pin_copy_state_matches_put_rows]
