"""fp64 CPU oracle for attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``verify_paged_gqa_b200``) never imports it and shares no code with it.

The arithmetic lives in ``tf_oracle.c`` (plain C, fp64, single pass per
output row, straight from the definition of softmax attention); this module
only compiles it with gcc and marshals numpy arrays.  Inputs are raw bf16
bit patterns (``numpy.uint16``); outputs are ``float64``.

Sources for what is computed:
  * TensorFold pull request #1620 (Kolibri-1 full layers in pages of the core
    pool), opening comment, Writes / Reads bullets and the kernel-contract
    bullet: rows are written into pages, then decode / verify / prompt rows
    attend over them; paged results must equal linear caches.
  * TensorFold pull request #2730 (eight-row verify window), "What this
    changes" and the checklist: a window is the pending token plus drafts,
    and drafted output equals undrafted output (causal inside the window).
  * TensorFold pull request #1620, opening comment, "Kept states" bullet: a
    kept state is copied by walking the slot's pages (``copy_state``).
  * TensorFold pull request #1620, opening comment, first bullet and Reads
    bullet: the verify kernels are "tree attention" over key groups of one
    page.  The pages give no mask; the reading is a per-row bitmask over the
    window's rows (its ancestors in the draft tree and itself), with every
    position before the window visible (``attend(..., tree=...)``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tf_oracle.c")
_LIB = os.path.join(_HERE, "libtforacle.so")
_lock = threading.Lock()
_lib = None


SANITIZE_FLAGS = ["-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
                  "-fno-omit-frame-pointer", "-g"]


def compile_source(src: str, out: str, sanitize: bool = False) -> str:
    """Compile one C source of the oracle into a shared library (gcc, -O2, no
    fast-math); ``sanitize`` adds AddressSanitizer and UndefinedBehaviorSanitizer
    (the process that loads it must preload libasan)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-Wall", "-Wextra",
         "-fno-fast-math", "-ffp-contract=off", *(SANITIZE_FLAGS if sanitize else []),
         src, "-o", tmp, "-lm", "-lpthread"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile tf_oracle.c into libtforacle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def open_library(path: str):
    """Load a compiled oracle (the default one, or a copy built from an edited source)."""
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    lib.tfo_attend_units.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, f64,
                                     p, i64, p, i32]
    lib.tfo_attend_units.restype = ctypes.c_int
    lib.tfo_attend_units_tree.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, f64,
                                          p, p, i64, p, i32]
    lib.tfo_attend_units_tree.restype = ctypes.c_int
    lib.tfo_put_rows.argtypes = [p, p, i32, i32, i32, i32, p, i32, p, i32, p, p, i32]
    lib.tfo_put_rows.restype = ctypes.c_int
    lib.tfo_copy_state.argtypes = [p, p, i32, i32, p, i32, p, p, i32, i32, p, i32, i32, i32, p,
                                   i32]
    lib.tfo_copy_state.restype = ctypes.c_int
    return lib


def _load():
    """The oracle library: TF_ORACLE_LIB names another build of tf_oracle.c (a
    sanitizer build, for instance), else the default one is built and used."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = open_library(os.environ.get("TF_ORACLE_LIB") or build())
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _pack_linear(caches):
    """Concatenate per-stream linear caches; returns (flat uint16, int64 offsets)."""
    offs = np.zeros(len(caches), dtype=np.int64)
    total = 0
    for s, c in enumerate(caches):
        offs[s] = total
        total += c.size
    flat = np.empty(total, dtype=np.uint16)
    for s, c in enumerate(caches):
        flat[offs[s]:offs[s] + c.size] = np.ascontiguousarray(c, dtype=np.uint16).ravel()
    return flat, offs


def attend(q, k_lin, v_lin, lens, rows, group, scale, units=None, threads=1, lib=None,
           tree=None):
    """Softmax attention over linear caches, in fp64.

    q      : uint16 (bf16 bits) [S][rows][Hq][d]
    k_lin  : list of S uint16 arrays [len_s][Hkv][d] (V likewise)
    lens   : int sequence [S], positions held AFTER this step's rows
    rows   : window rows W; row r sits at position len_s - W + r and sees 0..that
    group  : query heads per KV head G (query head h reads KV head h // G)
    units  : optional int array [n][3] of (s, r, h); then returns [n][d]
    lib    : optional library from ``open_library`` (default: the built oracle)
    tree   : optional uint8 [S][rows] row masks (rows <= 8): bit c of tree[s][r]
             set means row r sees window row c; positions before the window
             are seen by every row.  None is the causal window.
    Returns float64 [S][rows][Hq][d] (or [n][d] for ``units``).
    """
    lib = lib or _load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    S, W, Hq, d = q.shape
    assert W == rows and Hq % group == 0
    Hkv = Hq // group
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    assert lens.shape == (S,)
    for s in range(S):
        assert k_lin[s].shape == (lens[s], Hkv, d) and v_lin[s].shape == (lens[s], Hkv, d)
    kf, offs = _pack_linear(k_lin)
    vf, _ = _pack_linear(v_lin)
    full = units is None
    if full:
        units = np.stack(np.meshgrid(np.arange(S), np.arange(W), np.arange(Hq),
                                     indexing="ij"), axis=-1).reshape(-1, 3)
    units = np.ascontiguousarray(units, dtype=np.int32)
    out = np.zeros((units.shape[0], d), dtype=np.float64)
    if tree is None:
        st = lib.tfo_attend_units(_ptr(q), _ptr(kf), _ptr(vf), _ptr(offs), _ptr(lens), S, W,
                                  Hkv, group, d, float(scale), _ptr(units), units.shape[0],
                                  _ptr(out), int(threads))
    else:
        tree = np.ascontiguousarray(tree, dtype=np.uint8)
        assert tree.shape == (S, W)
        st = lib.tfo_attend_units_tree(_ptr(q), _ptr(kf), _ptr(vf), _ptr(offs), _ptr(lens), S,
                                       W, Hkv, group, d, float(scale), _ptr(tree), _ptr(units),
                                       units.shape[0], _ptr(out), int(threads))
    if st != 0:
        raise ValueError(f"oracle attend refused its arguments (status {st})")
    return out.reshape(S, W, Hq, d) if full else out


def put_rows(k_pool, v_pool, table, lens, k_rows, v_rows, lib=None):
    """Host scatter of new rows into a host copy of the pools (in place, bitwise).

    pools  : uint16 [n_pages][Hkv][P][d];  table: int32 [S][stride]
    rows   : uint16 [S][W][Hkv][d]; row r goes to position lens[s] - W + r.
    """
    lib = lib or _load()
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    n_pages, Hkv, P, d = k_pool.shape
    table = np.ascontiguousarray(table, dtype=np.int32)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    k_rows = np.ascontiguousarray(k_rows, dtype=np.uint16)
    v_rows = np.ascontiguousarray(v_rows, dtype=np.uint16)
    S, W = k_rows.shape[:2]
    st = lib.tfo_put_rows(_ptr(k_pool), _ptr(v_pool), n_pages, Hkv, P, d, _ptr(table),
                          table.shape[1], _ptr(lens), S, _ptr(k_rows), _ptr(v_rows), W)
    if st != 0:
        raise ValueError(f"oracle put_rows refused its arguments (status {st})")


def copy_state(src_k, src_v, src_table, dst_k, dst_v, dst_table, lens, lib=None):
    """Host copy of every stream's positions [0, lens[s]) from the source pools'
    pages to the destination pools' pages (in place in dst, bitwise).

    pools : uint16 [n_pages][Hkv][P][d] (source and destination may differ in
            n_pages and P);  tables: int32 [S][stride] each.
    """
    lib = lib or _load()
    for a in (src_k, src_v, dst_k, dst_v):
        assert a.flags.c_contiguous and a.dtype == np.uint16
    sn, Hkv, sP, d = src_k.shape
    dn, Hkv2, dP, d2 = dst_k.shape
    assert (Hkv, d) == (Hkv2, d2)
    src_table = np.ascontiguousarray(src_table, dtype=np.int32)
    dst_table = np.ascontiguousarray(dst_table, dtype=np.int32)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    st = lib.tfo_copy_state(_ptr(src_k), _ptr(src_v), sn, sP, _ptr(src_table),
                            src_table.shape[1], _ptr(dst_k), _ptr(dst_v), dn, dP,
                            _ptr(dst_table), dst_table.shape[1], Hkv, d, _ptr(lens), len(lens))
    if st != 0:
        raise ValueError(f"oracle copy_state refused its arguments (status {st})")
