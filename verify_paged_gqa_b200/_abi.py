"""ctypes marshalling for libtfpaged.so.

Each ``tf_*`` function here has the name of the C entry point it calls and
takes torch tensors in the layouts ``include/tf_paged.h`` documents:

    k_pool, v_pool  bf16  [n_pages][n_kv_heads][page_size][head_dim]  (CUDA)
    table           int32 [n_streams][table_stride]                   (CUDA)
    lens            int32 [n_streams]                                  (CUDA)
    q               bf16  [n_streams][rows][n_q_heads][head_dim]       (CUDA)
    out             fp32  [n_streams][rows][n_q_heads][head_dim]       (CUDA)
    k_rows, v_rows  bf16  [n_streams][rows][n_kv_heads][head_dim]      (CUDA)
    workspace       any dtype, tf_paged_attn_workspace_bytes bytes     (CUDA)

``max_len`` is the host upper bound on lens (the launch is sized from it).
Calls are asynchronous on ``stream`` (default: torch's current stream).  A
non-zero status raises TFError.  ``raw`` is the loaded ctypes library, for
callers that hold plain device pointers.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# TFPAGED_LIBRARY names another build of the library (a sanitizer build, for
# instance); by default the one built in place is loaded.
library_path = os.environ.get("TFPAGED_LIBRARY") or os.path.join(_HERE, "libtfpaged.so")


def _header_value(name: str) -> int:
    hdr = os.path.join(os.path.dirname(_HERE), "include", "tf_paged.h")
    if os.path.exists(hdr):
        m = re.search(rf"#define\s+{name}\s+(\d+)", open(hdr).read())
        if m:
            return int(m.group(1))
    return {"TF_OK": 0, "TF_EINVAL": 1, "TF_EUNSUPPORTED": 2, "TF_ENOSPACE": 3,
            "TF_ECUDA": 4, "TF_DEV_BAD_LEN": 1, "TF_DEV_BAD_PAGE": 2, "TF_DEV_TIMEOUT": 4}[name]


TF_OK = _header_value("TF_OK")
TF_EINVAL = _header_value("TF_EINVAL")
TF_EUNSUPPORTED = _header_value("TF_EUNSUPPORTED")
TF_ENOSPACE = _header_value("TF_ENOSPACE")
TF_ECUDA = _header_value("TF_ECUDA")
TF_DEV_BAD_LEN = _header_value("TF_DEV_BAD_LEN")
TF_DEV_BAD_PAGE = _header_value("TF_DEV_BAD_PAGE")
TF_DEV_TIMEOUT = _header_value("TF_DEV_TIMEOUT")

if not os.path.exists(library_path):
    raise ImportError(
        f"{library_path} is missing: build it with `python -m verify_paged_gqa_b200.build` "
        "(there is no fallback path)")


class tf_kv_pool(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("n_pages", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class tf_streams(ctypes.Structure):
    _fields_ = [("table", ctypes.c_void_p), ("table_stride", ctypes.c_int32),
                ("lens", ctypes.c_void_p), ("n_streams", ctypes.c_int32),
                ("max_len", ctypes.c_int32)]


raw = ctypes.CDLL(library_path)
_P = ctypes.POINTER
_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
raw.tf_kv_put_rows.argtypes = [_P(tf_kv_pool), _P(tf_streams), _vp, _vp, _i32, _vp]
raw.tf_kv_put_rows.restype = ctypes.c_int
raw.tf_paged_attn_workspace_bytes.argtypes = [_P(tf_kv_pool), _P(tf_streams), _i32, _i32]
raw.tf_paged_attn_workspace_bytes.restype = _sz
raw.tf_paged_attn_decode.argtypes = [_P(tf_kv_pool), _P(tf_streams), _vp, _i32, _f32,
                                     _vp, _vp, _sz, _vp]
raw.tf_paged_attn_decode.restype = ctypes.c_int
for _name in ("tf_paged_attn_verify", "tf_paged_attn_prompt"):
    getattr(raw, _name).argtypes = [_P(tf_kv_pool), _P(tf_streams), _vp, _i32, _i32, _f32,
                                    _vp, _vp, _sz, _vp]
    getattr(raw, _name).restype = ctypes.c_int
raw.tf_paged_attn_verify_tree.argtypes = [_P(tf_kv_pool), _P(tf_streams), _vp, _i32, _i32, _vp,
                                          _f32, _vp, _vp, _sz, _vp]
raw.tf_paged_attn_verify_tree.restype = ctypes.c_int
raw.tf_kv_copy_state.argtypes = [_P(tf_kv_pool), _P(tf_streams), _P(tf_kv_pool), _vp, _i32, _vp,
                                 _vp]
raw.tf_kv_copy_state.restype = ctypes.c_int
raw.tf_testing_paged_attn.argtypes = [_P(tf_kv_pool), _P(tf_streams), _vp, _i32, _i32, _f32,
                                      _vp, _vp, _sz, ctypes.c_int64, _i32, _vp]
raw.tf_testing_paged_attn.restype = ctypes.c_int
raw.tf_workspace_status.argtypes = [_vp, _P(ctypes.c_uint32), _vp]
raw.tf_workspace_status.restype = ctypes.c_int
raw.tf_status_str.argtypes = [ctypes.c_int]
raw.tf_status_str.restype = ctypes.c_char_p


class TFError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {tf_status_str(status)}")
        self.status = status


def tf_status_str(status: int) -> str:
    return raw.tf_status_str(int(status)).decode()


def _check(status: int, what: str):
    if status != TF_OK:
        raise TFError(status, what)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t, dtype, ndim, name):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != ndim:
        raise TypeError(f"{name} must be a {dtype} tensor with {ndim} dims")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _pool(k_pool, v_pool):
    _need(k_pool, torch.bfloat16, 4, "k_pool")
    _need(v_pool, torch.bfloat16, 4, "v_pool")
    if k_pool.shape != v_pool.shape:
        raise ValueError("k_pool and v_pool differ in shape")
    n_pages, hkv, page, d = k_pool.shape
    return tf_kv_pool(k_pool.data_ptr(), v_pool.data_ptr(), n_pages, hkv, page, d)


def _streams(table, lens, max_len):
    _need(table, torch.int32, 2, "table")
    _need(lens, torch.int32, 1, "lens")
    if lens.shape[0] != table.shape[0]:
        raise ValueError("lens and table disagree on the number of streams")
    return tf_streams(table.data_ptr(), table.shape[1], lens.data_ptr(), table.shape[0],
                      int(max_len))


def tf_kv_put_rows(k_pool, v_pool, table, lens, k_rows, v_rows, max_len, stream=None):
    """Write rows [S][W][Hkv][d] at positions lens[s] - W + r (see tf_kv_put_rows in the header)."""
    _need(k_rows, torch.bfloat16, 4, "k_rows")
    _need(v_rows, torch.bfloat16, 4, "v_rows")
    pool, st = _pool(k_pool, v_pool), _streams(table, lens, max_len)
    _check(raw.tf_kv_put_rows(ctypes.byref(pool), ctypes.byref(st), k_rows.data_ptr(),
                              v_rows.data_ptr(), k_rows.shape[1], _stream(stream)),
           "tf_kv_put_rows")


def tf_kv_copy_state(src_k, src_v, src_table, lens, dst_k, dst_v, dst_table, max_len,
                     status=None, stream=None):
    """Copies every stream's positions [0, lens[s]) of K and V from the source
    pools' pages (src_table) to the destination pools' pages (dst_table).
    status: optional uint32-viewable int32 device tensor of one element that
    collects TF_DEV_* bits."""
    src_pool, st = _pool(src_k, src_v), _streams(src_table, lens, max_len)
    dst_pool = _pool(dst_k, dst_v)
    _need(dst_table, torch.int32, 2, "dst_table")
    if dst_table.shape[0] != lens.shape[0]:
        raise ValueError("dst_table must have one row per stream")
    sp = 0
    if status is not None:
        if status.dtype != torch.int32 or status.numel() < 1:
            raise TypeError("status must be an int32 tensor")
        sp = status.data_ptr()
    _check(raw.tf_kv_copy_state(ctypes.byref(src_pool), ctypes.byref(st), ctypes.byref(dst_pool),
                                dst_table.data_ptr(), dst_table.shape[1], sp or None,
                                _stream(stream)), "tf_kv_copy_state")


def tf_paged_attn_workspace_bytes(k_pool, v_pool, table, lens, n_q_heads, rows, max_len) -> int:
    pool, st = _pool(k_pool, v_pool), _streams(table, lens, max_len)
    n = raw.tf_paged_attn_workspace_bytes(ctypes.byref(pool), ctypes.byref(st), n_q_heads, rows)
    if n == 0:
        raise TFError(TF_EINVAL, "tf_paged_attn_workspace_bytes")
    return int(n)


def _attn(fn, name, k_pool, v_pool, table, lens, q, scale, out, workspace, max_len, stream,
          with_rows, tree=None):
    _need(q, torch.bfloat16, 4, "q")
    _need(out, torch.float32, 4, "out")
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    if not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    pool, st = _pool(k_pool, v_pool), _streams(table, lens, max_len)
    ws_bytes = workspace.numel() * workspace.element_size()
    args = [ctypes.byref(pool), ctypes.byref(st), q.data_ptr(), q.shape[2]]
    if with_rows:
        args.append(q.shape[1])
    if tree is not None:
        args.append(tree.data_ptr())
    args += [float(scale), out.data_ptr(), workspace.data_ptr(), ws_bytes, _stream(stream)]
    _check(fn(*args), name)
    return out


def tf_paged_attn_decode(k_pool, v_pool, table, lens, q, scale, out, workspace, max_len,
                         stream=None):
    """One query row per stream (q [S][1][Hq][d])."""
    if q.shape[1] != 1:
        raise ValueError("decode takes one row per stream")
    return _attn(raw.tf_paged_attn_decode, "tf_paged_attn_decode", k_pool, v_pool, table, lens,
                 q, scale, out, workspace, max_len, stream, with_rows=False)


def tf_paged_attn_verify(k_pool, v_pool, table, lens, q, scale, out, workspace, max_len,
                         stream=None):
    """A causal window of q.shape[1] <= 8 rows per stream."""
    return _attn(raw.tf_paged_attn_verify, "tf_paged_attn_verify", k_pool, v_pool, table, lens,
                 q, scale, out, workspace, max_len, stream, with_rows=True)


def tf_paged_attn_verify_tree(k_pool, v_pool, table, lens, q, tree, scale, out, workspace,
                              max_len, stream=None):
    """A window of q.shape[1] <= 8 rows per stream under draft-tree masks:
    tree is a uint8 [S][rows] device tensor, bit c of tree[s][r] set when row r
    sees window row c (positions before the window are seen by every row)."""
    _need(tree, torch.uint8, 2, "tree")
    if tuple(tree.shape) != (q.shape[0], q.shape[1]):
        raise ValueError("tree must be [S][rows]")
    return _attn(raw.tf_paged_attn_verify_tree, "tf_paged_attn_verify_tree", k_pool, v_pool,
                 table, lens, q, scale, out, workspace, max_len, stream, with_rows=True,
                 tree=tree)


def tf_paged_attn_prompt(k_pool, v_pool, table, lens, q, scale, out, workspace, max_len,
                         stream=None):
    """A causal chunk of q.shape[1] prompt rows per stream (the last rows of each stream)."""
    return _attn(raw.tf_paged_attn_prompt, "tf_paged_attn_prompt", k_pool, v_pool, table, lens,
                 q, scale, out, workspace, max_len, stream, with_rows=True)


def tf_testing_paged_attn(k_pool, v_pool, table, lens, q, scale, out, workspace, max_len,
                          wait_limit_cycles, withhold, stream=None):
    """The test hook of include/tf_paged_testing.h: a causal attention call of
    q.shape[1] rows per stream with a shorter wait limit and, with
    ``withhold=1``, one arrival withheld in CTA 0 so that a wait runs out."""
    _need(q, torch.bfloat16, 4, "q")
    _need(out, torch.float32, 4, "out")
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    pool, st = _pool(k_pool, v_pool), _streams(table, lens, max_len)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(raw.tf_testing_paged_attn(ctypes.byref(pool), ctypes.byref(st), q.data_ptr(),
                                     q.shape[2], q.shape[1], float(scale), out.data_ptr(),
                                     workspace.data_ptr(), ws_bytes, int(wait_limit_cycles),
                                     int(withhold), _stream(stream)),
           "tf_testing_paged_attn")
    return out


def tf_workspace_status(workspace, stream=None) -> int:
    """Reads and clears the device status word (TF_DEV_* bits); synchronises the stream."""
    flags = ctypes.c_uint32(0)
    _check(raw.tf_workspace_status(workspace.data_ptr(), ctypes.byref(flags), _stream(stream)),
           "tf_workspace_status")
    return int(flags.value)
