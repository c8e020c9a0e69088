"""The CUDA path against the fp64 oracle, and its byte-level guarantees (B200)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import TOL, DeviceCase, bf16_tensor, max_abs, nan_pool

pytestmark = pytest.mark.gpu


def small_workload(d, G, P, W, Hkv=2, seed=100, sigma=1.0):
    return synth.Workload("sweep", 0, Hkv, G, d, P, W, seed=seed, kv_sigma=sigma)


def run_parity(w, lens, rows, table=None, n_pages=None):
    import verify_paged_gqa_b200 as tf
    case = synth.make_case(w, lens=lens, rows=rows, table=table, n_pages=n_pages)
    dc = DeviceCase(case)
    ws = dc.workspace(rows)
    out = dc.attend(ws=ws)
    torch.cuda.synchronize()
    # a clean call: no timeout, no bad length or page (a wait that ran out
    # leaves rows unwritten, which the comparison below would also catch)
    status = tf.tf_workspace_status(ws)
    assert status == 0, hex(status)
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, rows, w.group, w.scale,
                        threads=8)
    assert torch.isfinite(out).all()
    err = max_abs(out, ref)
    assert err <= TOL, err
    return case, dc, out


def test_parity_small_workload():
    w = synth.WORKLOADS["parity_small"]
    run_parity(w, None, 1)


@pytest.mark.parametrize("d", [128, 256, 512])
@pytest.mark.parametrize("G", [4, 8])
@pytest.mark.parametrize("W", [1, 2, 3, 4, 8])
def test_parity_sweep_page512(d, G, W):
    w = small_workload(d, G, 512, W, seed=1000 + d + 10 * G + W)
    # lengths on both sides of page boundaries: len % 512 in {0, 1, 511} and a short one
    run_parity(w, [1024, 1537, 1023, max(W, 37)], W)


@pytest.mark.parametrize("d", [128, 512])
@pytest.mark.parametrize("W", [1, 5])
def test_parity_page64(d, W):
    w = small_workload(d, 4, 64, W, seed=2000 + d + W)
    run_parity(w, [64 * 7, 64 * 3 + 1, 63 + W, 1000], W)


@pytest.mark.parametrize("W", [16, 100, 512])
def test_parity_prompt_chunks(W):
    w = small_workload(128, 4, 512, W, seed=3000 + W)
    run_parity(w, [W, W + 700, 1536], W)


def test_paged_equals_identity_table_bytes():
    w = small_workload(128, 4, 512, 4, seed=4000)
    lens = [2000, 513, 4096]
    case = synth.make_case(w, lens=lens)
    a = DeviceCase(case).attend()
    table, n_pages = synth.identity_table(case.lens, w.page_size)
    b = DeviceCase(case, table=table, n_pages=n_pages).attend()
    assert torch.equal(a, b)
    # a second shuffle of the same pool contents
    w2 = synth.Workload("sweep", 0, 2, 4, 128, 512, 4, seed=4001)
    t2, n2, _ = synth.page_table(w2, case.lens)
    c = DeviceCase(case, table=t2, n_pages=n2).attend()
    assert torch.equal(a, c)


def test_repeat_runs_are_bitwise_equal():
    w = small_workload(512, 8, 512, 4, seed=4100, sigma=0.5)
    case = synth.make_case(w, lens=[3000, 700, 9000])
    dc = DeviceCase(case)
    a = dc.attend()
    b = dc.attend()
    assert torch.equal(a, b)


def test_nan_never_reaches_output_and_negative_control_goes_red():
    w = small_workload(128, 4, 512, 2, seed=4200)
    lens = [1300, 600]
    case, dc, out = run_parity(w, lens, 2)
    # spare pages and unused slots are NaN (the pool was NaN-filled); output finite.
    assert torch.isfinite(out).all()
    # negative control: point stream 0's first page at a NaN spare page -> must go red
    t = case.table.copy()
    _, _, spares = synth.page_table(w, case.lens)
    t[0, 0] = spares[0]
    bad = DeviceCase(case)
    bad.table.copy_(torch.from_numpy(t).cuda())
    out_bad = bad.attend()
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, 2, w.group, w.scale)
    assert not (torch.isfinite(out_bad).all() and max_abs(out_bad, ref) <= TOL)


@pytest.mark.parametrize("d,G,P,W,lens,tree", [
    (128, 4, 512, 1, [1300, 600, 2049], False),     # decode, short contexts: CUDA-core kernel
    (128, 4, 512, 1, [7000, 600, 2049], False),     # decode, position-major kernel
    (128, 8, 512, 8, [1300, 600, 2049], False),     # verify, position-major kernel
    (512, 4, 512, 1, [1300, 600, 2049], False),     # head dim 512 decode, CUDA-core kernel
    (256, 8, 512, 4, [1300, 600, 2049], False),     # head dim 256 verify
    (128, 4, 512, 100, [1300, 600, 2049], False),   # prompt chunk, row-major kernel
    (128, 4, 37, 4, [1300, 600, 2049], False),      # pages of 37, tiles from page pieces
    (128, 4, 37, 1, [1300, 600, 2049], False),      # pages of 37, CUDA-core decode
    (128, 8, 512, 5, [1300, 600, 2049], True),      # tree masks
])
def test_fill_of_unused_slots_changes_no_output_bit(d, G, P, W, lens, tree):
    """Spare pages, the slots past each stream's length and the table entries
    past its pages filled with NaN, with zeros and with random bits (NaN and
    infinity patterns included): the outputs are equal byte for byte."""
    w = small_workload(d, G, P, W, seed=4300 + d + G + P + W)
    case = synth.make_case(w, lens=lens, rows=W)
    masks = synth.tree_masks((4301, d, G, W), len(lens), W) if tree else None
    outs = []
    for fill in ("nan", "zero", "random"):
        dc = DeviceCase(case, fill=fill)
        outs.append(dc.attend(tree=masks))
    torch.cuda.synchronize()
    assert torch.isfinite(outs[0]).all()
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[0], outs[2])
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, w.group, w.scale,
                        threads=8, tree=masks)
    assert max_abs(outs[0], ref) <= TOL


def test_put_rows_bit_exact_against_host_scatter():
    rng = np.random.default_rng(5)
    import verify_paged_gqa_b200 as tf
    for d, P, W in [(128, 512, 1), (128, 64, 8), (512, 512, 3), (512, 64, 5)]:
        w = synth.Workload("put", 3, 2, 4, d, P, W, seed=6000 + d + P + W)
        lens = np.array([W, P + 3, 3 * P], dtype=np.int32)
        table, n_pages, _ = synth.page_table(w, lens)
        host_k = rng.integers(0, 0x7F7F, size=(n_pages, 2, P, d)).astype(np.uint16)
        host_v = rng.integers(0, 0x7F7F, size=(n_pages, 2, P, d)).astype(np.uint16)
        kp, vp = bf16_tensor(host_k), bf16_tensor(host_v)
        kr = rng.integers(0, 0xFFFF, size=(3, W, 2, d)).astype(np.uint16)
        vr = rng.integers(0, 0xFFFF, size=(3, W, 2, d)).astype(np.uint16)
        tf.tf_kv_put_rows(kp, vp, torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda(),
                          bf16_tensor(kr), bf16_tensor(vr), max_len=int(lens.max()))
        oracle.put_rows(host_k, host_v, table, lens, kr, vr)
        got_k = kp.view(torch.int16).cpu().numpy().view(np.uint16)
        got_v = vp.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got_k, host_k)
        assert np.array_equal(got_v, host_v)


def test_status_flags_bad_len_and_bad_page():
    import verify_paged_gqa_b200 as tf
    w = small_workload(128, 4, 512, 1, seed=7000)
    case = synth.make_case(w, lens=[1000, 1500])
    dc = DeviceCase(case)
    ws = dc.workspace(1)
    tf.tf_workspace_status(ws)  # clear
    lens = torch.tensor([1000, 1500], dtype=torch.int32, device="cuda")
    out = dc.attend(lens=lens, max_len=1200, ws=ws)   # stream 1 longer than max_len
    flags = tf.tf_workspace_status(ws)
    assert flags & tf.TF_DEV_BAD_LEN
    assert torch.isnan(out[1]).all()
    ref = oracle.attend(case.q[:1], case.k_lin[:1], case.v_lin[:1], case.lens[:1], 1, 4, w.scale)
    assert max_abs(out[:1], ref) <= TOL
    # a page id outside the pool is never read and is reported
    dc.table[0, 1] = dc.k_pool.shape[0] + 5
    dc.attend(ws=ws)
    assert tf.tf_workspace_status(ws) & tf.TF_DEV_BAD_PAGE
    assert tf.tf_workspace_status(ws) == 0


def test_workspace_too_small_is_refused():
    import verify_paged_gqa_b200 as tf
    w = small_workload(128, 4, 512, 1, seed=7100)
    case = synth.make_case(w, lens=[40000, 30000])
    dc = DeviceCase(case)
    need = dc.workspace(1).numel()
    with pytest.raises(tf.TFError) as e:
        dc.attend(ws=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == tf.TF_ENOSPACE


@pytest.mark.parametrize("d,G,W", [(128, 8, 8), (128, 4, 3), (512, 8, 4), (512, 4, 8),
                                   (256, 8, 4), (128, 4, 1), (128, 4, 100)])
def test_parity_growing_scores(d, G, W):
    """K rows scaled up along the context: every row's max keeps growing past
    the kernels' rescale margin, so running maxima move and O is rescaled
    many times inside one chunk."""
    w = small_workload(d, G, 512, W, seed=8000 + d + 10 * G + W)
    case = synth.make_case(w, lens=[3000, 1300 + W], rows=W)
    for s, n in enumerate(case.lens):
        ramp = (1.0 + 14.0 * np.arange(n) / n).astype(np.float32)[:, None, None]
        k = synth.f32_from_bf16(case.k_lin[s]) * ramp
        case.k_lin[s] = synth.bf16_from_f32(k)
    dc = DeviceCase(case)
    out = dc.attend()
    torch.cuda.synchronize()
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, w.group, w.scale,
                        threads=8)
    assert torch.isfinite(out).all()
    assert max_abs(out, ref) <= TOL


# --- the stream-K split: every CTA gets an equal run of 128-position tiles
# across the call's (stream, KV head, row block) units; these cases put the
# split's corners under the oracle.

@pytest.mark.parametrize("d,G,W", [(128, 4, 1), (128, 8, 8), (512, 8, 4), (128, 4, 64)])
def test_split_fewer_tiles_than_ctas(d, G, W):
    """A handful of one-tile units: most CTAs get an empty range."""
    w = small_workload(d, G, 512, W, seed=9000 + d + G + W)
    run_parity(w, [W + 5, 100, 127, 128], W)


@pytest.mark.parametrize("d,G,W", [(128, 4, 1), (128, 8, 8), (512, 8, 4), (128, 4, 128)])
def test_split_one_long_stream(d, G, W):
    """One stream and one KV head: its units are split over every CTA, and the
    merge combines about one segment per CTA."""
    w = synth.Workload("one", 0, 1, G, d, 512, W, seed=9100 + d + G + W)
    run_parity(w, [40000 if d == 128 else 12000], W)


def test_split_many_short_streams():
    """Many short streams: a CTA's range runs over many whole units."""
    rng = np.random.default_rng(9200)
    lens = [int(x) for x in rng.integers(8, 700, size=60)] + [5000, 8, 1]
    w = small_workload(128, 8, 512, 1, Hkv=2, seed=9201)
    run_parity(w, lens, 1)


@pytest.mark.parametrize("d,top", [(128, 700), (512, 300)])
def test_page37_many_short_segments(d, top):
    """Decode blocks of 4 rows over pages of 37 on the CUDA-core kernel, which
    arms straddling tiles four ring stages at a time and starts every segment
    on a fresh quad: many short streams (segments of 1 to a few tiles, quads
    with unused slots, tile ends on and beside page ends) match the oracle,
    twice byte for byte, and the same streams with pages laid out in order
    give the same bytes."""
    rng = np.random.default_rng(9400 + d)
    edges = [1, 7, 8, 9, 31, 32, 33, 36, 37, 38, 74, 127, 128, 129]
    lens = [int(x) for x in rng.integers(1, top, size=40)] + edges
    w = small_workload(d, 4, 37, 1, Hkv=2, seed=9401 + d)
    case, dc, out = run_parity(w, lens, 1)
    again = dc.attend()
    assert torch.equal(out, again)
    table, n_pages = synth.identity_table(case.lens, w.page_size)
    inorder = DeviceCase(case, table=table, n_pages=n_pages).attend()
    assert torch.equal(out, inorder)


def test_split_skips_out_of_range_stream():
    """A stream longer than max_len in the middle of the call: its rows are NaN
    and flagged, and the split over the other streams is unaffected."""
    import verify_paged_gqa_b200 as tf
    w = small_workload(128, 8, 512, 4, seed=9300)
    case = synth.make_case(w, lens=[3000, 2500, 4000], rows=4)
    dc = DeviceCase(case)
    ws = dc.workspace(4)
    lens = torch.tensor([3000, 2500, 4000], dtype=torch.int32, device="cuda")
    out = dc.attend(lens=lens, max_len=3500, ws=ws)
    assert tf.tf_workspace_status(ws) & tf.TF_DEV_BAD_LEN
    assert torch.isnan(out[2]).all()
    keep = [0, 1]
    ref = oracle.attend(case.q[keep], [case.k_lin[i] for i in keep], [case.v_lin[i] for i in keep],
                        case.lens[keep], 4, w.group, w.scale, threads=8)
    assert max_abs(out[keep], ref) <= TOL


def test_split_prompt_kernel_more_units_than_ctas():
    """Prompt rows on more (stream, KV head, row block) units than there are
    CTAs: the prompt kernel runs the work split with partials and the merge
    (with fewer units it takes one unit per CTA whole)."""
    rng = np.random.default_rng(9400)
    lens = [int(x) for x in rng.integers(64, 900, size=40)]
    w = small_workload(128, 4, 512, 64, Hkv=2, seed=9401)
    run_parity(w, lens, 64)


# --- shape variants the pages mention: GQA 12 (48 query / 4 KV heads), GQA 16
# at head dim 512 (16 query / 1 KV head), head dim 256

@pytest.mark.parametrize("W", [1, 4, 8])
def test_parity_gqa12(W):
    w = synth.Workload("gqa12", 0, 4, 12, 128, 512, W, seed=9500 + W)
    run_parity(w, [3000, 1025, W + 3], W)


@pytest.mark.parametrize("W", [1, 4, 8])
def test_parity_gqa16_hd512(W):
    w = synth.Workload("gqa16", 0, 1, 16, 512, 512, W, seed=9600 + W)
    run_parity(w, [5000, 700, W], W)


@pytest.mark.parametrize("P", [64, 37, 1, 100])
@pytest.mark.parametrize("W", [1, 4])
def test_hd256_any_page_size(P, W):
    """Head dim 256 over pages that are not a multiple of 128: the tiles that
    straddle pages are gathered row by row."""
    w = small_workload(256, 4, P, W, seed=9700 + P + W)
    lens = [P * 5 + 3, W + 1, 700] if P > 1 else [300, W + 1, 129]
    run_parity(w, lens, W)


@pytest.mark.parametrize("d,G,W", [(128, 4, 1), (128, 8, 8), (256, 8, 4), (512, 8, 4),
                                   (512, 4, 1), (128, 4, 100)])
def test_page_size_changes_no_output_bit(d, G, W):
    """The same streams in pools of pages of 512, 128, 37 and 1 positions:
    whole 128-row boxes or tiles assembled from page pieces, the outputs of
    one kernel are equal byte for byte (the arithmetic depends on positions,
    never on the pages).  A single 4-row block at head dim 128 runs on the
    CUDA-core kernel over pages below 128 that are not a multiple of 64, so
    there the pairs (512, 128) and (37, 1) are compared."""
    lens = [1300, W + 2, 777]
    outs = {}
    for P in (512, 128, 37, 1):
        w = small_workload(d, G, P, W, seed=9800 + d + G + W)   # same seed: same K, V, q
        case = synth.make_case(w, lens=lens, rows=W)
        outs[P] = DeviceCase(case).attend()
    torch.cuda.synchronize()
    assert torch.equal(outs[512], outs[128])
    assert torch.equal(outs[37], outs[1])
    if not (d == 128 and G * W <= 4):
        assert torch.equal(outs[512], outs[37])
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, w.group, w.scale,
                        threads=8)
    for o in outs.values():
        assert max_abs(o, ref) <= TOL


# --- tree-mask verify: each window row sees the positions before the window
# and the window rows its mask names (its ancestors in a draft tree)

def run_tree_parity(w, lens, rows, tree, table=None, n_pages=None):
    case = synth.make_case(w, lens=lens, rows=rows, table=table, n_pages=n_pages)
    dc = DeviceCase(case)
    out = dc.attend(tree=tree)
    torch.cuda.synchronize()
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, rows, w.group, w.scale,
                        threads=8, tree=tree)
    assert torch.isfinite(out).all()
    err = max_abs(out, ref)
    assert err <= TOL, err
    return case, dc, out


@pytest.mark.parametrize("d,G", [(128, 4), (128, 8), (128, 12), (128, 16), (256, 8), (512, 8),
                                 (512, 16)])
@pytest.mark.parametrize("W", [2, 5, 8])
def test_tree_parity_sweep(d, G, W):
    w = small_workload(d, G, 512, W, seed=10000 + d + 10 * G + W)
    lens = [1024, 1537, 1023, W, W + 130]
    tree = synth.tree_masks((10001, d, G, W), len(lens), W)
    run_tree_parity(w, lens, W, tree)


def test_tree_chain_masks_match_the_causal_window():
    w = small_workload(128, 8, 512, 8, seed=10100)
    lens = [3000, 900]
    case, dc, out = run_tree_parity(w, lens, 8, synth.chain_masks(2, 8))
    causal = dc.attend()
    assert (out - causal).abs().max().item() <= TOL


def test_tree_masks_naming_later_rows():
    """Masks are read as given: a row may also name rows after it."""
    rng = np.random.default_rng(10200)
    W = 6
    lens = [W, 700, 2049]
    tree = rng.integers(0, 256, size=(3, W)).astype(np.uint8)
    for r in range(W):
        tree[:, r] |= np.uint8(1 << r)
    w = small_workload(128, 4, 512, W, seed=10201)
    run_tree_parity(w, lens, W, tree)


def test_tree_paged_equals_identity_table_bytes_and_repeats():
    w = small_workload(512, 8, 512, 4, seed=10300, sigma=0.5)
    lens = [2000, 513, 4096]
    tree = synth.tree_masks((10301,), 3, 4)
    case = synth.make_case(w, lens=lens)
    dc = DeviceCase(case)
    a = dc.attend(tree=tree)
    b = dc.attend(tree=tree)
    assert torch.equal(a, b)
    table, n_pages = synth.identity_table(case.lens, w.page_size)
    c = DeviceCase(case, table=table, n_pages=n_pages).attend(tree=tree)
    assert torch.equal(a, c)


@pytest.mark.parametrize("d,G,W", [(128, 8, 8), (512, 8, 4)])
def test_tree_split_one_long_stream(d, G, W):
    w = synth.Workload("one", 0, 1, G, d, 512, W, seed=10400 + d + W)
    tree = synth.tree_masks((10401, d), 1, W)
    run_tree_parity(w, [40000 if d == 128 else 12000], W, tree)


def test_tree_growing_scores():
    W = 8
    w = small_workload(128, 8, 512, W, seed=10500)
    case = synth.make_case(w, lens=[3000, 1300 + W], rows=W)
    for s, n in enumerate(case.lens):
        ramp = (1.0 + 14.0 * np.arange(n) / n).astype(np.float32)[:, None, None]
        case.k_lin[s] = synth.bf16_from_f32(synth.f32_from_bf16(case.k_lin[s]) * ramp)
    tree = synth.tree_masks((10501,), 2, W)
    dc = DeviceCase(case)
    out = dc.attend(tree=tree)
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, w.group, w.scale,
                        threads=8, tree=tree)
    assert torch.isfinite(out).all()
    assert max_abs(out, ref) <= TOL


@pytest.mark.parametrize("P", [64, 37])
@pytest.mark.parametrize("d,G,W", [(128, 4, 4), (128, 8, 8), (512, 8, 3)])
def test_tree_any_page_size(P, d, G, W):
    """Pages that are not a multiple of 128 take tree calls on the CUDA-core kernel."""
    w = small_workload(d, G, P, W, seed=10600 + P + d + G + W)
    lens = [P * 5 + 3, W, 700]
    run_tree_parity(w, lens, W, synth.tree_masks((10601, P, d, G, W), len(lens), W))


# --- any page size (the pages check the paged prompt kernel over pages of 37):
# tiles of the CUDA-core kernel straddle pages, one bulk copy per page piece

@pytest.mark.parametrize("P", [37, 1, 3, 100, 509])
@pytest.mark.parametrize("d", [128, 512])
@pytest.mark.parametrize("W", [1, 4, 8])
def test_parity_any_page_size(P, d, W):
    w = small_workload(d, 4, P, W, seed=11000 + P + d + W)
    lens = [P * 7, P * 3 + 1, W + 2, 1000] if P > 1 else [40, 9, W, 300]
    run_parity(w, lens, W)


@pytest.mark.parametrize("W", [16, 100])
def test_parity_prompt_page37(W):
    w = small_workload(128, 4, 37, W, seed=11100 + W)
    run_parity(w, [W, W + 300, 700], W)


def test_page37_paged_equals_identity_table_and_put_rows_bit_exact():
    w = small_workload(128, 8, 37, 2, seed=11200)
    lens = [2000, 37, 38, 75]
    case = synth.make_case(w, lens=lens)
    a = DeviceCase(case).attend()
    table, n_pages = synth.identity_table(case.lens, w.page_size)
    b = DeviceCase(case, table=table, n_pages=n_pages).attend()
    assert torch.equal(a, b)
    # the row write over pages of 37 and of 1
    import verify_paged_gqa_b200 as tf
    rng = np.random.default_rng(11201)
    for P in (37, 1):
        wp = synth.Workload("put", 3, 2, 4, 128, P, 3, seed=11202 + P)
        lens = np.array([3, P + 3, 5 * P + 2], dtype=np.int32)
        table, n_pages, _ = synth.page_table(wp, lens)
        host_k = rng.integers(0, 0x7F7F, size=(n_pages, 2, P, 128)).astype(np.uint16)
        host_v = host_k[::-1].copy()
        kp, vp = bf16_tensor(host_k), bf16_tensor(host_v)
        kr = rng.integers(0, 0xFFFF, size=(3, 3, 2, 128)).astype(np.uint16)
        vr = rng.integers(0, 0xFFFF, size=(3, 3, 2, 128)).astype(np.uint16)
        tf.tf_kv_put_rows(kp, vp, torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda(),
                          bf16_tensor(kr), bf16_tensor(vr), max_len=int(lens.max()))
        oracle.put_rows(host_k, host_v, table, lens, kr, vr)
        assert np.array_equal(kp.view(torch.int16).cpu().numpy().view(np.uint16), host_k)
        assert np.array_equal(vp.view(torch.int16).cpu().numpy().view(np.uint16), host_v)


def test_page37_bad_page_is_flagged_and_shapes_refused():
    import verify_paged_gqa_b200 as tf
    w = small_workload(128, 4, 37, 1, seed=11300)
    case = synth.make_case(w, lens=[500, 90])
    dc = DeviceCase(case)
    ws = dc.workspace(1)
    tf.tf_workspace_status(ws)
    dc.table[0, 3] = dc.k_pool.shape[0] + 2      # a page in the middle of a straddling tile
    dc.attend(ws=ws)
    assert tf.tf_workspace_status(ws) & tf.TF_DEV_BAD_PAGE
    # a page id past the pool on the tensor-core kernels' gathered tiles
    for d, W in ((128, 8), (256, 4), (512, 4)):
        w3 = small_workload(d, 8, 37, W, seed=11303 + d)
        dc3 = DeviceCase(synth.make_case(w3, lens=[900, 300], rows=W))
        ws3 = dc3.workspace(W)
        tf.tf_workspace_status(ws3)
        dc3.table[1, 2] = -7
        out = dc3.attend(ws=ws3)
        assert tf.tf_workspace_status(ws3) & tf.TF_DEV_BAD_PAGE
        ref = oracle.attend(dc3.case.q[:1], dc3.case.k_lin[:1], dc3.case.v_lin[:1],
                            dc3.case.lens[:1], W, 8, w3.scale)
        assert max_abs(out[:1], ref) <= TOL              # the other stream is untouched
    # head dim 256 over pages of 37, with and without tree masks
    w2 = small_workload(256, 4, 37, 4, seed=11301)
    case2 = synth.make_case(w2, lens=[300, 41], rows=4)
    dc2 = DeviceCase(case2)
    for tree in (None, synth.tree_masks((11302,), 2, 4)):
        out = dc2.attend(tree=tree)
        ref = oracle.attend(case2.q, case2.k_lin, case2.v_lin, case2.lens, 4, 4, w2.scale,
                            threads=8, tree=tree)
        assert max_abs(out, ref) <= TOL


# --- the state copy: a stream's K/V walked from one set of pages to another

def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("sP,dP", [(512, 512), (512, 37), (37, 64), (64, 1), (1, 512), (128, 100)])
@pytest.mark.parametrize("d", [128, 512])
def test_copy_state_bit_exact(sP, dP, d):
    import verify_paged_gqa_b200 as tf
    rng = np.random.default_rng(12000 + sP + dP + d)
    Hkv = 2
    lens = np.array([700, 0, 1, 1537], dtype=np.int32)
    ws = synth.Workload("copy", 4, Hkv, 4, d, sP, 1, seed=12001 + sP)
    wd = synth.Workload("copy", 4, Hkv, 4, d, dP, 1, seed=12002 + dP)
    st, sn, _ = synth.page_table(ws, np.maximum(lens, 1))
    dt, dn, _ = synth.page_table(wd, np.maximum(lens, 1))
    sk = rng.integers(0, 0xFFFF, size=(sn, Hkv, sP, d)).astype(np.uint16)
    sv = rng.integers(0, 0xFFFF, size=(sn, Hkv, sP, d)).astype(np.uint16)
    dk = np.full((dn, Hkv, dP, d), synth.BF16_NAN, dtype=np.uint16)
    dv = dk.copy()
    gk, gv = bf16_tensor(dk), bf16_tensor(dv)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tf.tf_kv_copy_state(bf16_tensor(sk), bf16_tensor(sv), torch.from_numpy(st).cuda(),
                        torch.from_numpy(lens).cuda(), gk, gv, torch.from_numpy(dt).cuda(),
                        max_len=int(lens.max()), status=status)
    oracle.copy_state(sk, sv, st, dk, dv, dt, lens)
    assert np.array_equal(_u16(gk), dk)
    assert np.array_equal(_u16(gv), dv)
    assert int(status.item()) == 0


def test_copy_state_keep_and_resume_give_the_same_attention():
    """Keep every stream's state in a linear buffer (one page per stream), resume
    it into other shuffled pages of the same pool's spare room, and attend: the
    output is byte-equal to attending over the original pages."""
    import verify_paged_gqa_b200 as tf
    W = 4
    w = small_workload(128, 8, 512, W, seed=12100)
    lens = [3000, 513, 2048]
    case = synth.make_case(w, lens=lens)
    a_dc = DeviceCase(case)
    a = a_dc.attend()
    L = int(max(lens))
    lin_k = torch.full((3, 2, L, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin_v = lin_k.clone()
    lin_t = torch.arange(3, dtype=torch.int32, device="cuda")[:, None].contiguous()
    tf.tf_kv_copy_state(a_dc.k_pool, a_dc.v_pool, a_dc.table, a_dc.lens, lin_k, lin_v, lin_t,
                        max_len=L)
    # the linear state holds the stream's rows in order
    for s in range(3):
        n = lens[s]
        assert np.array_equal(_u16(lin_k[s, :, :n].transpose(0, 1).contiguous()), case.k_lin[s])
    w2 = synth.Workload("sweep", 0, 2, 8, 128, 512, W, seed=12101)
    t2, n2, _ = synth.page_table(w2, case.lens)
    b_dc = DeviceCase(case, table=t2, n_pages=n2)
    b_dc.k_pool.fill_(float("nan"))
    b_dc.v_pool.fill_(float("nan"))
    tf.tf_kv_copy_state(lin_k, lin_v, lin_t, a_dc.lens, b_dc.k_pool, b_dc.v_pool, b_dc.table,
                        max_len=L)
    b = b_dc.attend()
    assert torch.equal(a, b)


def test_copy_state_flags_bad_pages_and_lengths():
    import verify_paged_gqa_b200 as tf
    Hkv, d, P = 2, 128, 64
    sk = torch.randn(6, Hkv, P, d, device="cuda").to(torch.bfloat16)
    sv = torch.randn(6, Hkv, P, d, device="cuda").to(torch.bfloat16)
    dk = torch.zeros(6, Hkv, P, d, dtype=torch.bfloat16, device="cuda")
    dv = dk.clone()
    st = torch.tensor([[0, 1, 2], [3, 4, 5]], dtype=torch.int32, device="cuda")
    dt = torch.tensor([[5, 4, 3], [2, 1, 99]], dtype=torch.int32, device="cuda")  # 99: bad
    lens = torch.tensor([150, 140], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tf.tf_kv_copy_state(sk, sv, st, lens, dk, dv, dt, max_len=192, status=status)
    assert int(status.item()) & tf.TF_DEV_BAD_PAGE
    # stream 0 was copied whole; stream 1's good pages too
    assert torch.equal(dk[5], sk[0]) and torch.equal(dk[4], sk[1])
    assert torch.equal(dk[3, :, :150 - 128], sk[2, :, :150 - 128])
    assert torch.equal(dv[2], sv[3]) and torch.equal(dv[1], sv[4])
    status.zero_()
    lens2 = torch.tensor([150, 300], dtype=torch.int32, device="cuda")   # past max_len
    tf.tf_kv_copy_state(sk, sv, st, lens2, dk, dv, st, max_len=192, status=status)
    assert int(status.item()) & tf.TF_DEV_BAD_LEN


# --- edge cases: odd shapes, boundary lengths, empty calls, the largest chunk

@pytest.mark.parametrize("d", [128, 512])
@pytest.mark.parametrize("G,W", [(1, 1), (3, 5), (5, 3), (1, 8), (2, 7), (7, 2)])
def test_parity_odd_group_and_rows(d, G, W):
    """GQA ratios outside 4/8 and odd row counts: odd rows per KV head (partial
    slots of odd size), row blocks that end mid-window."""
    w = small_workload(d, G, 512, W, Hkv=3, seed=13000 + d + 10 * G + W)
    run_parity(w, [1537, W, 512, 2 * W + 1], W)


@pytest.mark.parametrize("d,G,W", [(128, 4, 1), (128, 8, 8), (512, 8, 4), (128, 4, 100)])
def test_parity_lengths_at_the_table_bound(d, G, W):
    """Streams exactly as long as their table can hold (len == stride * page
    size), next to one that is a window and nothing more (len == rows)."""
    w = small_workload(d, G, 512, W, seed=13100 + d + G + W)
    case = synth.make_case(w, lens=[2048, W, 1024], rows=W)
    assert case.table.shape[1] * w.page_size == 2048
    dc = DeviceCase(case)
    out = dc.attend()
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, G, w.scale, threads=8)
    assert torch.isfinite(out).all()
    assert max_abs(out, ref) <= TOL


def test_calls_with_no_streams_do_nothing():
    import verify_paged_gqa_b200 as tf
    w = small_workload(128, 4, 512, 2, seed=13200)
    case = synth.make_case(w, lens=[600])
    dc = DeviceCase(case)
    empty_t = dc.table[:0].contiguous()
    empty_l = dc.lens[:0].contiguous()
    q0 = dc.q[:0].contiguous()
    out0 = torch.empty(q0.shape, dtype=torch.float32, device="cuda")
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    for fn in (tf.tf_paged_attn_verify, tf.tf_paged_attn_prompt):
        fn(dc.k_pool, dc.v_pool, empty_t, empty_l, q0, w.scale, out0, ws, 600)
    tf.tf_paged_attn_verify_tree(dc.k_pool, dc.v_pool, empty_t, empty_l, q0,
                                 torch.zeros((0, 2), dtype=torch.uint8, device="cuda"), w.scale,
                                 out0, ws, 600)
    tf.tf_kv_put_rows(dc.k_pool, dc.v_pool, empty_t, empty_l,
                      torch.zeros((0, 2, 2, 128), dtype=torch.bfloat16, device="cuda"),
                      torch.zeros((0, 2, 2, 128), dtype=torch.bfloat16, device="cuda"), max_len=600)
    tf.tf_kv_copy_state(dc.k_pool, dc.v_pool, empty_t, empty_l, dc.k_pool, dc.v_pool, empty_t,
                        max_len=600)
    torch.cuda.synchronize()
    assert tf.tf_workspace_status(ws) == 0


def test_largest_prompt_chunk_sampled():
    """A 4,096-row chunk (the largest the prompt call takes) over 4,096 + 500
    positions, checked on sampled rows."""
    W = 4096
    w = small_workload(128, 4, 512, W, Hkv=2, seed=13300)
    case = synth.make_case(w, lens=[W + 500], rows=W)
    out = DeviceCase(case).attend().cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(13301)
    rows = sorted(set(int(x) for x in rng.choice(W, 24, replace=False)) | {0, W - 1})
    units = np.array([(0, r, h) for r in rows for h in (0, 5)], dtype=np.int32)
    ref = oracle.attend(case.q, case.k_lin, case.v_lin, case.lens, W, w.group, w.scale,
                        units=units, threads=8)
    got = np.stack([out[0, r, h] for r in rows for h in (0, 5)])
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL
