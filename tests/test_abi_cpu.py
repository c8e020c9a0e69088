"""The C-ABI library without a GPU: it builds for sm_100a, loads, exports every
entry point the header declares, and rejects bad host arguments before it
touches the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_symbols():
    """Every entry point that a header under include/ declares."""
    names = []
    for h in HEADERS:
        names += re.findall(r"TF_API\s+[\w\s\*]+?\b(tf_\w+)\s*\(", open(h).read())
    return names


@pytest.fixture(scope="module")
def lib():
    from verify_paged_gqa_b200 import build
    path = build.build()
    import verify_paged_gqa_b200 as t
    if not os.environ.get("TFPAGED_LIBRARY"):   # else: another build, e.g. a sanitizer build
        assert os.path.samefile(path, t.library_path)
    from verify_paged_gqa_b200 import _abi
    return _abi


def test_header_declares_the_entry_points():
    names = set(declared_symbols())
    assert {"tf_kv_put_rows", "tf_paged_attn_workspace_bytes", "tf_paged_attn_decode",
            "tf_paged_attn_verify", "tf_paged_attn_prompt", "tf_workspace_status",
            "tf_status_str"} <= names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, re.M))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(ctypes.CDLL(lib.library_path), name)


def test_library_is_built_for_sm100a(lib):
    from verify_paged_gqa_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.ARCH


def _pool(lib, **kw):
    base = dict(k_pool=16, v_pool=16, n_pages=8, n_kv_heads=2, page_size=512, head_dim=128)
    base.update(kw)
    return lib.tf_kv_pool(**base)


def _streams(lib, **kw):
    base = dict(table=16, table_stride=4, lens=16, n_streams=2, max_len=2048)
    base.update(kw)
    return lib.tf_streams(**base)


@pytest.mark.parametrize("pool_kw,streams_kw,hq,rows,want", [
    ({"head_dim": 64}, {}, 8, 1, "TF_EUNSUPPORTED"),
    ({"page_size": 0}, {}, 8, 1, "TF_EINVAL"),
    ({"n_pages": 0}, {}, 8, 1, "TF_EINVAL"),
    ({}, {"max_len": 2049}, 8, 1, "TF_EINVAL"),          # past table_stride * page_size
    ({}, {}, 7, 1, "TF_EINVAL"),                          # query heads not a multiple
    ({}, {}, 8, 0, "TF_EINVAL"),                          # no rows
    ({}, {"max_len": 3}, 8, 4, "TF_EINVAL"),              # window longer than the context
    ({"k_pool": 17}, {}, 8, 1, "TF_EINVAL"),              # unaligned pool
    ({}, {"table": 0}, 8, 1, "TF_EINVAL"),                # NULL table
])
def test_bad_host_arguments_are_rejected(lib, pool_kw, streams_kw, hq, rows, want):
    pool, st = _pool(lib, **pool_kw), _streams(lib, **streams_kw)
    rc = lib.raw.tf_paged_attn_verify(ctypes.byref(pool), ctypes.byref(st), 16, hq, rows, 0.1,
                                      16, 16, 1 << 30, None)
    assert rc == getattr(lib, want)
    assert lib.raw.tf_paged_attn_workspace_bytes(ctypes.byref(pool), ctypes.byref(st), hq,
                                                 rows) == 0


def test_verify_rows_limit_and_null_pointers(lib):
    pool, st = _pool(lib), _streams(lib)
    assert lib.raw.tf_paged_attn_verify(ctypes.byref(pool), ctypes.byref(st), 16, 8, 9, 0.1, 16,
                                        16, 1 << 30, None) == lib.TF_EINVAL
    assert lib.raw.tf_paged_attn_decode(None, ctypes.byref(st), 16, 8, 0.1, 16, 16, 1 << 30,
                                        None) == lib.TF_EINVAL
    assert lib.raw.tf_kv_put_rows(ctypes.byref(pool), ctypes.byref(st), 16, 16, 0,
                                  None) == lib.TF_EINVAL
    assert lib.raw.tf_workspace_status(None, None, None) == lib.TF_EINVAL
    assert lib.tf_status_str(lib.TF_ENOSPACE).startswith("TF_ENOSPACE")


def test_tree_verify_host_checks(lib):
    pool, st = _pool(lib), _streams(lib)
    # no mask array
    assert lib.raw.tf_paged_attn_verify_tree(ctypes.byref(pool), ctypes.byref(st), 16, 8, 4, None,
                                             0.1, 16, 16, 1 << 30, None) == lib.TF_EINVAL
    # more rows than a mask byte holds
    assert lib.raw.tf_paged_attn_verify_tree(ctypes.byref(pool), ctypes.byref(st), 16, 8, 9, 16,
                                             0.1, 16, 16, 1 << 30, None) == lib.TF_EINVAL


def test_copy_state_host_checks(lib):
    src, st = _pool(lib), _streams(lib)
    dst = _pool(lib, page_size=37)
    # mismatched head dim or KV heads
    for bad in (_pool(lib, head_dim=512), _pool(lib, n_kv_heads=3)):
        assert lib.raw.tf_kv_copy_state(ctypes.byref(src), ctypes.byref(st), ctypes.byref(bad), 16,
                                        64, None, None) == lib.TF_EINVAL
    # destination table too short for max_len (2048 > 50 * 37)
    assert lib.raw.tf_kv_copy_state(ctypes.byref(src), ctypes.byref(st), ctypes.byref(dst), 16, 50,
                                    None, None) == lib.TF_EINVAL
    # no destination table, an unaligned status word
    assert lib.raw.tf_kv_copy_state(ctypes.byref(src), ctypes.byref(st), ctypes.byref(dst), None,
                                    64, None, None) == lib.TF_EINVAL
    assert lib.raw.tf_kv_copy_state(ctypes.byref(src), ctypes.byref(st), ctypes.byref(dst), 16, 64,
                                    18, None) == lib.TF_EINVAL
