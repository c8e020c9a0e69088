"""Device-side set-up shared by the GPU tests: a synthetic case uploaded into a
NaN-filled paged pool through the library's own row write."""
from __future__ import annotations

import numpy as np
import torch

import synth

TOL = 2e-3   # max-abs against the fp64 oracle on fp32 outputs (bf16 in, fp32 accumulate)


def bf16_tensor(u16, device="cuda"):
    a = np.ascontiguousarray(u16, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def nan_pool(n_pages, w, fill="nan"):
    """K and V pools whose every slot holds NaN (``fill="nan"``), zero or
    random bits (``"random"``: NaN and infinity patterns included), before the
    streams' rows are written."""
    shape = (n_pages, w.n_kv_heads, w.page_size, w.head_dim)
    if fill == "random":
        g = torch.Generator(device="cuda")
        g.manual_seed(n_pages * 1000 + w.head_dim)
        return tuple(torch.randint(-2**15, 2**15, shape, dtype=torch.int16, device="cuda",
                                   generator=g).view(torch.bfloat16) for _ in range(2))
    value = float("nan") if fill == "nan" else 0.0
    return (torch.full(shape, value, dtype=torch.bfloat16, device="cuda"),
            torch.full(shape, value, dtype=torch.bfloat16, device="cuda"))


class DeviceCase:
    """Pools, table and lens on the GPU for one synth.Case.  Every stream's rows
    are written with tf_kv_put_rows (one call per stream, all its positions)."""

    def __init__(self, case: synth.Case, table=None, n_pages=None, fill="nan"):
        import verify_paged_gqa_b200 as tf
        self.tf = tf
        self.case = case
        w = case.w
        self.w = w
        table = case.table if table is None else table
        n_pages = case.n_pages if n_pages is None else n_pages
        self.k_pool, self.v_pool = nan_pool(n_pages, w, fill)
        self.table = torch.from_numpy(np.ascontiguousarray(table, dtype=np.int32)).cuda()
        self.lens = torch.from_numpy(np.ascontiguousarray(case.lens, dtype=np.int32)).cuda()
        self.max_len = int(case.lens.max())
        for s in range(len(case.lens)):
            n = int(case.lens[s])
            if n == 0 or case.k_lin[s].shape[0] != n:
                continue
            tf.tf_kv_put_rows(self.k_pool, self.v_pool, self.table[s:s + 1], self.lens[s:s + 1],
                              bf16_tensor(case.k_lin[s][None]), bf16_tensor(case.v_lin[s][None]),
                              max_len=n)
        self.q = bf16_tensor(case.q)

    def workspace(self, rows):
        n = self.tf.tf_paged_attn_workspace_bytes(self.k_pool, self.v_pool, self.table, self.lens,
                                                  self.w.n_q_heads, rows, self.max_len)
        return torch.zeros(n, dtype=torch.uint8, device="cuda")

    def attend(self, q=None, lens=None, max_len=None, ws=None, out=None, kind=None, tree=None):
        q = self.q if q is None else q
        lens = self.lens if lens is None else lens
        max_len = self.max_len if max_len is None else max_len
        W = q.shape[1]
        ws = self.workspace(W) if ws is None else ws
        out = torch.empty(q.shape, dtype=torch.float32, device="cuda") if out is None else out
        if tree is not None:
            t = torch.from_numpy(np.ascontiguousarray(tree, dtype=np.uint8)).cuda()
            self.tf.tf_paged_attn_verify_tree(self.k_pool, self.v_pool, self.table, lens, q, t,
                                              self.w.scale, out, ws, max_len)
            return out
        if kind is None:
            kind = "decode" if W == 1 else "verify" if W <= 8 else "prompt"
        fn = {"decode": self.tf.tf_paged_attn_decode, "verify": self.tf.tf_paged_attn_verify,
              "prompt": self.tf.tf_paged_attn_prompt}[kind]
        fn(self.k_pool, self.v_pool, self.table, lens, q, self.w.scale, out, ws, max_len)
        return out


def max_abs(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.detach().cpu().numpy().astype(np.float64)
    return float(np.abs(g - ref).max())
