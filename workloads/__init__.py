"""Seeded synthetic inputs for PISA pyramid block-sparse attention.

This module is the only code shared by the CPU oracle and the CUDA path. It
draws the Q/K/V tensors of the five benchmark workloads and rounds them to
bf16 (round to nearest even). It holds none of the method's arithmetic: no
pooling, no selection, no attention.

Every (tensor, batch, head, row-chunk) slice is drawn from its own PCG64
stream keyed by ``SeedSequence([seed, tensor, b, h, chunk])``. A slice can
therefore be regenerated on its own (the oracle checks sampled slices of the
full-size workloads) and whole tensors can be drawn by many threads with a
result that does not depend on the thread count.

Workloads (the pages name no dataset for PISA; these synthetic sets stand in
for long-context prefill and decode):

* ``tiny``      B1 H2 N4096 D64, block 64, factor 4, K 8, non-causal, iid N(0,1)
* ``causal32k`` B1 H16 N32768 D128, block 64, factor 4, K 32, causal, clustered keys
* ``gqa128k``   B1 Hq32/Hkv8 N131072 D128, block 64, factor 4, K 64, causal,
                iid N(0,1) plus 16 planted needle blocks per KV head
* ``decode128k`` 64 sequences x 1 query token, KV 131072, Hq32/Hkv8, D128,
                block 64, factor 4, K 64, clustered keys
* ``long1m``    B1 H8 N1048576 D128, block 128, factor 8, K 128, causal, clustered keys
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK_ROWS = 4096          # rows per independently seeded slice
N_CENTROIDS = 64           # clusters per (batch, KV head) for clustered keys
CLUSTER_NOISE_STD = 0.3    # "N(0,0.3)" read as standard deviation 0.3
N_NEEDLES = 16             # planted needle blocks per KV head (gqa128k)
NEEDLE_COS = 0.9           # cosine between a needle key and its target direction

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "centroid": 4, "qcid": 5, "kcid": 6, "needle": 7, "needle_w": 8}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seq_q: int
    seq_kv: int
    head_dim: int
    block: int
    factor: int
    topk: int
    causal: int
    keys: str            # "iid" | "clustered" | "needle"
    seed: int

    @property
    def group(self) -> int:
        return self.heads_q // self.heads_kv

    @property
    def n_blocks(self) -> int:
        return self.seq_kv // self.block

    @property
    def decode(self) -> bool:
        return self.seq_q == 1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 4096, 4096, 64, 64, 4, 8, 0, "iid", 1001),
    "causal32k": Workload("causal32k", 1, 16, 16, 32768, 32768, 128, 64, 4, 32, 1, "clustered", 1002),
    "gqa128k": Workload("gqa128k", 1, 32, 8, 131072, 131072, 128, 64, 4, 64, 1, "needle", 1003),
    "decode128k": Workload("decode128k", 64, 32, 8, 1, 131072, 128, 64, 4, 64, 0, "clustered", 1004),
    "long1m": Workload("long1m", 1, 8, 8, 1048576, 1048576, 128, 128, 8, 128, 1, "clustered", 1005),
}


# ----------------------------------------------------------------------------- bf16 marshalling

def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even. Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the fp32 values they represent (exact)."""
    return (np.ascontiguousarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------- seeded streams

def _rng(w: Workload, tensor: str, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence([w.seed, _TENSOR_IDS[tensor], *[int(k) for k in key]])
    return np.random.Generator(np.random.PCG64(ss))


def _rows(w: Workload, tensor: str) -> int:
    return w.seq_q if tensor == "q" else w.seq_kv


def _centroids(w: Workload, b: int, kvh: int) -> np.ndarray:
    return _rng(w, "centroid", b, kvh).standard_normal((N_CENTROIDS, w.head_dim), dtype=np.float32)


def _key_block_cluster(w: Workload, b: int, kvh: int) -> np.ndarray:
    return _rng(w, "kcid", b, kvh).integers(0, N_CENTROIDS, size=w.n_blocks)


def _query_cluster(w: Workload, b: int, h: int) -> np.ndarray:
    """Cluster id per query block (prefill) or for the single decode token."""
    n = 1 if w.decode else w.seq_q // w.block
    return _rng(w, "qcid", b, h).integers(0, N_CENTROIDS, size=n)


def needles(w: Workload, b: int, kvh: int) -> list[tuple[int, int]]:
    """(target query block i, needle key block j) pairs planted in one KV head.

    i is uniform in [128, nb-1], j uniform in [0, i-2], needle blocks distinct per head.
    """
    g = _rng(w, "needle", b, kvh)
    nb = w.n_blocks
    lo = min(128, nb - 1)
    out, used = [], set()
    while len(out) < N_NEEDLES:
        i = int(g.integers(max(lo, 2), nb))
        j = int(g.integers(0, i - 1))
        if j in used:
            continue
        used.add(j)
        out.append((i, j))
    return out


def _base_chunk(w: Workload, tensor: str, b: int, h: int, c: int) -> np.ndarray:
    """fp32 values (before bf16 rounding) of rows [c*CHUNK_ROWS, ...) of plane (b, h)."""
    rows = _rows(w, tensor)
    r0, r1 = c * CHUNK_ROWS, min((c + 1) * CHUNK_ROWS, rows)
    g = _rng(w, tensor, b, h, c)
    x = g.standard_normal((r1 - r0, w.head_dim), dtype=np.float32)
    if w.keys == "clustered" and tensor in ("k", "q"):
        kvh = h if tensor == "k" else h // w.group
        cent = _centroids(w, b, kvh)
        if tensor == "k":
            cid = np.repeat(_key_block_cluster(w, b, kvh), w.block)[r0:r1]
        elif w.decode:
            cid = np.repeat(_query_cluster(w, b, h), r1 - r0)
        else:
            cid = np.repeat(_query_cluster(w, b, h), w.block)[r0:r1]
        x = cent[cid] + np.float32(CLUSTER_NOISE_STD) * x
    return x


def _query_block_rows(w: Workload, b: int, kvh: int, i: int) -> np.ndarray:
    """bf16-exact fp32 query rows of block i for the g query heads of KV head kvh: [g*block, D]."""
    rows = []
    r0 = i * w.block
    c = r0 // CHUNK_ROWS
    off = r0 - c * CHUNK_ROWS
    for hh in range(kvh * w.group, (kvh + 1) * w.group):
        x = bf16_to_f32(round_bf16(_base_chunk(w, "q", b, hh, c)))
        rows.append(x[off:off + w.block])
    return np.concatenate(rows, axis=0)


def _plant_needles(w: Workload, x: np.ndarray, b: int, kvh: int, c: int) -> None:
    """Replace each key k of a needle block by |k| (0.9 u + sqrt(0.19) w), w a random unit vector orthogonal to u."""
    r0, r1 = c * CHUNK_ROWS, c * CHUNK_ROWS + x.shape[0]
    for n, (i, j) in enumerate(needles(w, b, kvh)):
        j0 = j * w.block
        if not (r0 <= j0 < r1):
            continue
        d = _query_block_rows(w, b, kvh, i).astype(np.float64).sum(axis=0)
        u = d / np.linalg.norm(d)
        z = _rng(w, "needle_w", b, kvh, n).standard_normal((w.block, w.head_dim))
        z -= np.outer(z @ u, u)
        z /= np.linalg.norm(z, axis=1, keepdims=True)
        blk = x[j0 - r0:j0 - r0 + w.block].astype(np.float64)
        norm = np.linalg.norm(blk, axis=1, keepdims=True)
        s = np.sqrt(1.0 - NEEDLE_COS ** 2)
        x[j0 - r0:j0 - r0 + w.block] = (norm * (NEEDLE_COS * u[None, :] + s * z)).astype(np.float32)


def chunk_bf16(w: Workload, tensor: str, b: int, h: int, c: int) -> np.ndarray:
    """bf16 bit patterns (uint16) of one seeded slice [rows, D]."""
    x = _base_chunk(w, tensor, b, h, c)
    if w.keys == "needle" and tensor == "k":
        _plant_needles(w, x, b, h, c)
    return round_bf16(x)


def plane_bf16(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    """bf16 bits of one (batch, head) plane: [rows, D]."""
    rows = _rows(w, tensor)
    n_chunks = (rows + CHUNK_ROWS - 1) // CHUNK_ROWS
    return np.concatenate([chunk_bf16(w, tensor, b, h, c) for c in range(n_chunks)], axis=0)


def plane_f32(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    return bf16_to_f32(plane_bf16(w, tensor, b, h))


def tensor_bf16(w: Workload, tensor: str, out: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """Whole tensor [B, H, rows, D] as bf16 bits (uint16), drawn by a thread pool."""
    heads = w.heads_q if tensor == "q" else w.heads_kv
    rows = _rows(w, tensor)
    if out is None:
        out = np.empty((w.batch, heads, rows, w.head_dim), dtype=np.uint16)
    n_chunks = (rows + CHUNK_ROWS - 1) // CHUNK_ROWS
    jobs = [(b, h, c) for b in range(w.batch) for h in range(heads) for c in range(n_chunks)]

    def run(job):
        b, h, c = job
        out[b, h, c * CHUNK_ROWS:min((c + 1) * CHUNK_ROWS, rows)] = chunk_bf16(w, tensor, b, h, c)

    threads = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, jobs))
    return out


def qkv_f32(w: Workload) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Small workloads only: Q, K, V as bf16-exact fp32 arrays [B, H, rows, D]."""
    return tuple(bf16_to_f32(tensor_bf16(w, t)) for t in ("q", "k", "v"))


def device_tensor(w: Workload, tensor: str, device):
    """bf16 torch tensor [B, H, rows, D] on `device`, drawn batch by batch (bounded host memory)."""
    import torch
    heads = w.heads_q if tensor == "q" else w.heads_kv
    rows = _rows(w, tensor)
    out = torch.empty((w.batch, heads, rows, w.head_dim), dtype=torch.bfloat16, device=device)
    n_chunks = (rows + CHUNK_ROWS - 1) // CHUNK_ROWS
    host = np.empty((heads, rows, w.head_dim), dtype=np.uint16)
    threads = min(32, os.cpu_count() or 1)
    for b in range(w.batch):
        def run(job, b=b):
            h, c = job
            r0 = c * CHUNK_ROWS
            host[h, r0:min(r0 + CHUNK_ROWS, rows)] = chunk_bf16(w, tensor, b, h, c)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, [(h, c) for h in range(heads) for c in range(n_chunks)]))
        out[b].copy_(torch.from_numpy(host.view(np.int16)).view(torch.bfloat16))
    return out
