"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and lays out tables; it holds none of the
attention arithmetic and none of the row-write addressing.  Both the oracle
and the CUDA path receive what it returns:

  * the oracle gets per-stream LINEAR caches ``[len_s][Hkv][d]`` and the query
    rows;
  * the CUDA path gets the same rows and writes them into its pages itself
    (through its own row write), guided by the page table built here.

Values are drawn as float32 from numpy's PCG64 (one independent SeedSequence
per stream and tensor, so one stream can be regenerated alone for sampled
checks at full size) and rounded to bf16 with round-to-nearest-even.  bf16 is
handled as raw ``uint16`` bit patterns everywhere.

Workloads (synthetic stand-ins for the pages' served runs):
  * ``parity_small``   one stream, 1 KV head, GQA 4, d 128, 1,037 positions in
    pages of 512 (last one partial) in a pool of 8, one decode row;
  * ``decode_12x40k``  12 streams at 40,960, 8 KV / 32 query heads, d 128,
    pool 1.2x the pages needed, one row per stream (TensorFold #1620's
    ``--parallel 12 --context 40960`` cells);
  * ``verify_4x131k``  4 streams at 131,072, 4 KV / 32 query heads (GQA 8),
    d 128, 8-row causal windows (TensorFold #2730: eight rows, 131,072 context,
    four streams);
  * ``hd512_verify``   16 streams, lengths uniform in [2,048, 9,216], 2 KV / 16
    query heads, d 512, 4-row windows, K/V ~ N(0, 0.5^2) (TensorFold #1620's
    head dim 512 global layer, four-row cells);
  * ``prompt_9216``    one 9,216-token prompt written into shuffled pages, then
    attended in causal chunks of 512 rows, 8 KV / 32 query heads, d 128;
  * ``decode_12x40k_p37`` the decode workload in pages of 37 positions
    (TensorFold #1620, Checks: the paged prompt kernel over pages of 37);
  * ``tree_verify_4x131k`` the verify workload with every stream's window a
    random draft tree (TensorFold #1620 calls the verify kernels "tree
    attention"; each row sees its ancestors and itself).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BF16_NAN = np.uint16(0x7FC0)


def bf16_from_f32(x) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = BF16_NAN
    return out


def _seed_int(*key: int) -> int:
    """A 63-bit seed for torch's generator, mixed from an int tuple."""
    return int(np.random.SeedSequence([int(k) for k in key]).generate_state(2, np.uint64)[0]
               >> np.uint64(1))


def normal_bf16_torch(key, shape, sigma: float = 1.0, device="cuda"):
    """Like normal_bf16 but drawn by torch's generator on ``device`` (fast for the
    full-size workloads); a different stream of numbers than the numpy one.
    Returns a torch.bfloat16 tensor (rounded to nearest even by torch)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(_seed_int(*key))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16)


def to_bits(t) -> np.ndarray:
    """bf16 torch tensor -> host uint16 bit patterns."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_from_bf16(b) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def normal_bf16(key, shape, sigma: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0, sigma^2) samples of the given shape, seeded by the int tuple ``key``."""
    x = _rng(*key).standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return bf16_from_f32(x)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_streams: int
    n_kv_heads: int
    group: int                 # query heads per KV head
    head_dim: int
    page_size: int
    rows: int                  # window rows W (decode 1, verify <= 8, prompt chunk)
    seed: int
    kv_sigma: float = 1.0
    q_sigma: float = 1.0
    lens: tuple = ()           # fixed per-stream lengths, or () with len_range
    len_range: tuple = ()      # (lo, hi) inclusive uniform integer lengths
    pool_factor: float = 1.2
    n_pages: int = 0           # fixed pool size (0: ceil(pool_factor * needed) + 1)
    prompt_len: int = 0        # >0: one prompt attended in chunks of ``rows``
    tree: bool = False         # verify windows under random draft-tree masks

    @property
    def n_q_heads(self) -> int:
        return self.n_kv_heads * self.group

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    "parity_small": Workload("parity_small", 1, 1, 4, 128, 512, 1, seed=1, lens=(1037,),
                             n_pages=8),
    "decode_12x40k": Workload("decode_12x40k", 12, 8, 4, 128, 512, 1, seed=2,
                              lens=(40960,) * 12),
    "verify_4x131k": Workload("verify_4x131k", 4, 4, 8, 128, 512, 8, seed=3,
                              lens=(131072,) * 4),
    "hd512_verify": Workload("hd512_verify", 16, 2, 8, 512, 512, 4, seed=4, kv_sigma=0.5,
                             len_range=(2048, 9216)),
    "prompt_9216": Workload("prompt_9216", 1, 8, 4, 128, 512, 512, seed=5, lens=(9216,),
                            prompt_len=9216),
    # shape variants the pages mention: GQA 12 (48 query / 4 KV heads), GQA 16
    # at head dim 512 (16 query / 1 KV head), head dim 256
    "gqa12_verify": Workload("gqa12_verify", 4, 4, 12, 128, 512, 8, seed=8, lens=(32768,) * 4),
    "gqa16_hd512_decode": Workload("gqa16_hd512_decode", 16, 1, 16, 512, 512, 1, seed=9,
                                   lens=(16384,) * 16),
    "hd256_verify": Workload("hd256_verify", 16, 2, 8, 256, 512, 4, seed=10,
                             len_range=(2048, 9216)),
    # the verify workload with each stream's 8 rows a random draft tree
    "tree_verify_4x131k": Workload("tree_verify_4x131k", 4, 4, 8, 128, 512, 8, seed=11,
                                   lens=(131072,) * 4, tree=True),
    # the decode workload in pages of 37 positions (tiles straddle pages)
    "decode_12x40k_p37": Workload("decode_12x40k_p37", 12, 8, 4, 128, 37, 1, seed=12,
                                  lens=(40960,) * 12),
    # many short streams (a serving batch early in its contexts): 64 x 2,048
    # and 256 x 512 positions, the decode workload's heads
    "decode_64x2k": Workload("decode_64x2k", 64, 8, 4, 128, 512, 1, seed=14, lens=(2048,) * 64),
    "decode_256x512": Workload("decode_256x512", 256, 8, 4, 128, 512, 1, seed=15,
                               lens=(512,) * 256),
    # smaller copies of the decode and verify workloads for profiler captures
    # (still larger than the 126 MB L2)
    "decode_12x8k": Workload("decode_12x8k", 12, 8, 4, 128, 512, 1, seed=6, lens=(8192,) * 12),
    "decode_12x8k_p37": Workload("decode_12x8k_p37", 12, 8, 4, 128, 37, 1, seed=13,
                                 lens=(8192,) * 12),
    "verify_4x16k": Workload("verify_4x16k", 4, 4, 8, 128, 512, 8, seed=7, lens=(16384,) * 4),
    # the verify copy in pages of 64 (tensor-core tiles assembled from page pieces)
    "verify_4x16k_p64": Workload("verify_4x16k_p64", 4, 4, 8, 128, 64, 8, seed=16,
                                 lens=(16384,) * 4),
}


def tree_masks(key, n_streams: int, rows: int) -> np.ndarray:
    """Random draft trees, one per stream: row 0 is the root and row r > 0 hangs
    under a parent drawn uniformly from rows 0 .. r - 1.  Returns uint8
    [S][rows] with bit c of [s][r] set when window row c is row r or one of its
    ancestors (the mask a tree-verify call takes)."""
    assert 1 <= rows <= 8
    rng = _rng(*key)
    out = np.zeros((n_streams, rows), dtype=np.uint8)
    for s in range(n_streams):
        for r in range(rows):
            parent_mask = int(out[s, int(rng.integers(0, r))]) if r > 0 else 0
            out[s, r] = parent_mask | (1 << r)
    return out


def chain_masks(n_streams: int, rows: int) -> np.ndarray:
    """The causal window as tree masks: row r sees rows 0 .. r."""
    return np.tile(np.array([(1 << (r + 1)) - 1 for r in range(rows)], dtype=np.uint8),
                   (n_streams, 1))


def workload_tree(w: Workload, n_streams: int | None = None, rows: int | None = None):
    """The tree masks of a tree workload (None for a causal one)."""
    if not w.tree:
        return None
    return tree_masks((w.seed, 11), w.n_streams if n_streams is None else n_streams,
                      w.rows if rows is None else rows)


def stream_lens(w: Workload) -> np.ndarray:
    if w.lens:
        return np.array(w.lens, dtype=np.int32)
    lo, hi = w.len_range
    return _rng(w.seed, 0).integers(lo, hi + 1, size=w.n_streams).astype(np.int32)


def pages_needed(lens, page_size: int) -> np.ndarray:
    return (np.asarray(lens, dtype=np.int64) + page_size - 1) // page_size


def page_table(w: Workload, lens, spare_fill: bool = True):
    """Seeded shuffled page table.

    Returns (table int32 [S][stride], n_pages, spare_ids).  Stream s owns
    ``ceil(len_s / P)`` distinct pool pages drawn from one seeded permutation
    of the pool; entries past a stream's pages point at spare (NaN-filled)
    pages, so a kernel that reads past a stream's end would read NaN.
    """
    P = w.page_size
    need = pages_needed(lens, P)
    stride = int(need.max())
    total = int(need.sum())
    n_pages = w.n_pages or int(math.ceil(w.pool_factor * total)) + 1
    assert n_pages > total, "the pool needs at least one spare page"
    perm = _rng(w.seed, 7).permutation(n_pages).astype(np.int32)
    spare = perm[total:]
    table = np.empty((len(lens), stride), dtype=np.int32)
    off = 0
    for s, n in enumerate(need):
        table[s, :n] = perm[off:off + n]
        table[s, n:] = spare[(s + np.arange(stride - n)) % len(spare)] if spare_fill else -1
        off += n
    return table, n_pages, spare


def identity_table(lens, page_size: int):
    """Pages laid out in order: stream 0's pages first, then stream 1's, ... (no shuffle)."""
    need = pages_needed(lens, page_size)
    stride = int(need.max())
    total = int(need.sum())
    table = np.full((len(lens), stride), total, dtype=np.int32)   # page `total` is the spare
    off = 0
    for s, n in enumerate(need):
        table[s, :n] = np.arange(off, off + n, dtype=np.int32)
        off += n
    return table, total + 1


def kv_rows(w: Workload, s: int, length: int):
    """Linear K and V of stream s: two uint16 arrays [length][Hkv][d] (bf16 bits)."""
    shape = (length, w.n_kv_heads, w.head_dim)
    return (normal_bf16((w.seed, 1, s), shape, w.kv_sigma),
            normal_bf16((w.seed, 2, s), shape, w.kv_sigma))


def kv_rows_torch(w: Workload, s: int, length: int, device="cuda"):
    """Linear K and V of stream s drawn on the device: two bf16 tensors [length][Hkv][d]."""
    shape = (length, w.n_kv_heads, w.head_dim)
    return (normal_bf16_torch((w.seed, 11, s), shape, w.kv_sigma, device),
            normal_bf16_torch((w.seed, 12, s), shape, w.kv_sigma, device))


def q_rows_torch(w: Workload, n_streams: int, rows: int, tag: int = 0, device="cuda"):
    """Query rows [S][W][Hq][d] drawn on the device (bf16 tensor)."""
    return normal_bf16_torch((w.seed, 13, tag), (n_streams, rows, w.n_q_heads, w.head_dim),
                             w.q_sigma, device)


def q_rows(w: Workload, rows: int | None = None, tag: int = 0):
    """Query rows [S][W][Hq][d] (bf16 bits)."""
    W = w.rows if rows is None else rows
    return normal_bf16((w.seed, 3, tag), (w.n_streams, W, w.n_q_heads, w.head_dim), w.q_sigma)


@dataclasses.dataclass
class Case:
    """One attention call's inputs, in both views."""
    w: Workload
    lens: np.ndarray            # int32 [S], positions after this step's rows
    rows: int                   # W
    q: np.ndarray               # uint16 [S][W][Hq][d]
    k_lin: list                 # S x uint16 [len_s][Hkv][d]
    v_lin: list
    table: np.ndarray           # int32 [S][stride]
    n_pages: int

    @property
    def new_k(self) -> np.ndarray:
        """This step's rows [S][W][Hkv][d]: the last W positions of each stream."""
        return np.stack([k[len(k) - self.rows:] for k in self.k_lin])

    @property
    def new_v(self) -> np.ndarray:
        return np.stack([v[len(v) - self.rows:] for v in self.v_lin])


def make_case(w: Workload, lens=None, rows: int | None = None, table=None, n_pages=None,
              streams=None) -> Case:
    """Build a call's inputs.  ``streams`` restricts K/V generation to some streams
    (others get empty caches; for sampled checks at full size)."""
    lens = stream_lens(w) if lens is None else np.asarray(lens, dtype=np.int32)
    W = w.rows if rows is None else rows
    if table is None:
        table, n_pages, _ = page_table(w, lens)
    k_lin, v_lin = [], []
    for s in range(len(lens)):
        if streams is None or s in streams:
            k, v = kv_rows(w, s, int(lens[s]))
        else:
            k = v = np.zeros((0, w.n_kv_heads, w.head_dim), dtype=np.uint16)
        k_lin.append(k)
        v_lin.append(v)
    wq = dataclasses.replace(w, n_streams=len(lens))
    return Case(w, lens, W, q_rows(wq, W), k_lin, v_lin, table, n_pages)
