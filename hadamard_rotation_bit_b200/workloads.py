"""Seeded synthetic activations shaped like the pages' Llama-class workloads.

This module holds input recipes only -- no rotation or quantization
arithmetic -- so both the CUDA path and the float64 oracle can consume the
same bit patterns.  Every tensor is generated in chunks of ``CHUNK_ROWS``
rows from a counter-keyed numpy ``PCG64`` stream, so any row range can be
regenerated on its own (row sampling for the oracle, per-rank shards) and
gives the same bits as the whole tensor.

Recipes (seed 0 everywhere; an "outlier set" is the first k entries of a
permutation drawn from a ``seed + 1`` stream):

* ``c1``  64 x 1024 fp32 ~ N(0, 1); full 1024-point rotation; int4, group 128.
* ``c2``  R1 residual stream: 4096 tokens x 4096 bf16 ~ N(0, 1), 41 outlier
  channels (1 %) scaled x50; full 4096-point rotation; int4, group 128.
* ``c3``  R4 down_proj input: 8192 x 14336 bf16 = SiLU(a) * b with a, b ~
  N(0, 1), 72 outlier channels (0.5 %) scaled x30; block 128; int8 per token.
* ``c4q`` / ``c4k``  R3 Q and K after RoPE: [16, 32, 4096, 128] bf16 ~ N(0, 1),
  two outlier dims per head (per-head seeded choice) scaled x20 before RoPE
  (rotate-half pairing (i, i + 64), theta_i = 10000^(-i/64), position = s);
  per-head 128-point rotation; Q -> bf16, K -> int4 group 128.
* ``c5``  65536 x 8192 bf16 Student-t(3); full 8192-point rotation; MXFP4.
* ``c2n`` / ``c5n``  the ``c2`` / ``c5`` input quantized to NVFP4 (E4M3 scale
  per 16 elements, per-tensor scale 1) instead.
* ``c2r`` / ``c2rb``  the ``c2`` input and quantizer with a random Hadamard
  rotation ("Rotation Transform", section 1.5): signs after (the random
  Hadamard matrix) or before (its transpose); the b signs are Rademacher
  draws (``generate_signs``), int8 +/-1.
* ``c3rb`` / ``c5rb``  the ``c3`` / ``c5`` input and quantizer with signs
  before the rotation (block 128 / full 8192).
* ``c2p`` / ``c2q``  the ``c2`` input through orbitquant's RPBH rotation (a
  seeded random permutation of the 4096 columns and 4096 Rademacher signs,
  ``generate_rpbh``, then the full 4096-point rotation), quantized to int4 g128
  (``c2p``) or by the per-token norm and the 4-bit unit-sphere Lloyd-Max
  codebook (``c2q``, "orbitquant 0.2.0", Method Conformance).
* ``pl256`` / ``pl1024``  per-Linear shapes of "Rotation Transform" section 2
  on the butterfly kernels: the ``c5`` input with block 256 and int4 g128;
  131072 x 1024 bf16 ~ N(0, 1) with 1 % of the channels x50, rotated in full
  to MXFP4.
* ``c3k`` / ``c3km``  the ``c3`` input rotated in full instead of by blocks
  of 128: the 14336-point rotation of a non-power-of-2 size ("Rotation
  Transform", section 1.5: 14336 = 28 * 2^9, a base matrix of order 28 with a
  Sylvester block); int8 per token / MXFP4.

Values are drawn in float64, rounded to float32 (nearest even) and, for
bf16 tensors, to bfloat16 (nearest even).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

CHUNK_ROWS = 1024
SEED = 0


@dataclass(frozen=True)
class Workload:
    key: str
    name: str
    rows: int
    n: int
    block: int          # applied rotation block; == n for a full rotation
    x_dtype: str        # "f32" | "bf16"
    fmt: str | None     # "int4" | "int8" | "mxfp4" | None (rotation only)
    group: int          # quant group (0 = per token for int8)
    out_dtype: str | None = None   # rotation-only output dtype
    signs: str | None = None       # random Hadamard: "after" | "before" | None (deterministic)
    base: str | None = None        # input recipe of another workload (same bits)
    rpbh: bool = False             # RPBH: a column permutation and n signs ahead of the block rotation

    @property
    def in_bytes(self) -> int:
        return self.rows * self.n * (4 if self.x_dtype == "f32" else 2)

    @property
    def out_bytes(self) -> int:
        r, n = self.rows, self.n
        if self.fmt is None:
            return r * n * (4 if self.out_dtype == "f32" else 2)
        if self.fmt == "int4":
            return r * n // 2 + r * (n // self.group) * 2
        if self.fmt == "int8":
            return r * n + r * 4
        if self.fmt == "mxfp4":
            return r * n // 2 + r * (n // 32)
        if self.fmt == "nvfp4":
            return r * n // 2 + r * (n // 16)
        if self.fmt == "codebook":       # group = bits per code; one fp32 norm per row
            return r * n * self.group // 8 + r * 4
        raise ValueError(self.fmt)

    @property
    def algorithmic_bytes(self) -> int:
        """Input read once plus outputs written once."""
        return self.in_bytes + self.out_bytes


WORKLOADS = {
    "c1": Workload("c1", "64x1024 fp32, full 1024-point Hadamard, int4 sym g128 fp16 scales",
                   64, 1024, 1024, "f32", "int4", 128),
    "c2": Workload("c2", "R1 4096 tokens x hidden 4096 bf16, full 4096-point Hadamard, int4 sym g128 fp16 scales",
                   4096, 4096, 4096, "bf16", "int4", 128),
    "c3": Workload("c3", "R4 8192 tokens x intermediate 14336 bf16, block 128 (112 blocks), int8 per token",
                   8192, 14336, 128, "bf16", "int8", 0),
    "c4q": Workload("c4q", "R3 Q [16,32,4096,128] bf16 after RoPE, per-head 128-point Hadamard -> bf16",
                    16 * 32 * 4096, 128, 128, "bf16", None, 0, "bf16"),
    "c4k": Workload("c4k", "R3 K [16,32,4096,128] bf16 after RoPE, per-head 128-point Hadamard, int4 g128",
                    16 * 32 * 4096, 128, 128, "bf16", "int4", 128),
    "c5": Workload("c5", "large R1 65536 tokens x hidden 8192 bf16 Student-t(3), full 8192-point Hadamard, MXFP4",
                   65536, 8192, 8192, "bf16", "mxfp4", 32),
    "c2n": Workload("c2n", "R1 4096 tokens x hidden 4096 bf16, full 4096-point Hadamard, NVFP4 (E4M3 scale per 16)",
                    4096, 4096, 4096, "bf16", "nvfp4", 16, base="c2"),
    "c5n": Workload("c5n", "large R1 65536 tokens x hidden 8192 bf16 Student-t(3), full 8192-point Hadamard, NVFP4 "
                    "(E4M3 scale per 16)", 65536, 8192, 8192, "bf16", "nvfp4", 16, base="c5"),
    "c2r": Workload("c2r", "R1 4096 tokens x hidden 4096 bf16, full 4096-point random Hadamard (signs after), "
                    "int4 sym g128 fp16 scales", 4096, 4096, 4096, "bf16", "int4", 128, signs="after", base="c2"),
    "c2rb": Workload("c2rb", "R1 4096 tokens x hidden 4096 bf16, full 4096-point random Hadamard transpose "
                     "(signs before), int4 sym g128 fp16 scales", 4096, 4096, 4096, "bf16", "int4", 128,
                     signs="before", base="c2"),
    "c3k": Workload("c3k", "R4 8192 tokens x intermediate 14336 bf16, full 14336-point Hadamard (K = 28 base "
                    "(x) 512-point Sylvester), int8 per token", 8192, 14336, 14336, "bf16", "int8", 0, base="c3"),
    "c3km": Workload("c3km", "R4 8192 tokens x intermediate 14336 bf16, full 14336-point Hadamard (K = 28 base "
                     "(x) 512-point Sylvester), MXFP4", 8192, 14336, 14336, "bf16", "mxfp4", 32, base="c3"),
    "c3rb": Workload("c3rb", "R4 8192 tokens x intermediate 14336 bf16, block 128 random Hadamard transpose "
                     "(signs before), int8 per token", 8192, 14336, 128, "bf16", "int8", 0, signs="before", base="c3"),
    "c2p": Workload("c2p", "R1 4096 tokens x hidden 4096 bf16, RPBH (random column permutation, n signs, full "
                    "4096-point Hadamard), int4 sym g128 fp16 scales", 4096, 4096, 4096, "bf16", "int4", 128,
                    base="c2", rpbh=True),
    "c2q": Workload("c2q", "R1 4096 tokens x hidden 4096 bf16, RPBH (full 4096-point), per-token norm + 4-bit "
                    "unit-sphere Lloyd-Max codebook", 4096, 4096, 4096, "bf16", "codebook", 4, base="c2", rpbh=True),
    "pl256": Workload("pl256", "per-Linear block-diagonal: 65536 tokens x 8192 bf16 Student-t(3), block 256, int4 sym "
                      "g128", 65536, 8192, 256, "bf16", "int4", 128, base="c5"),
    "pl1024": Workload("pl1024", "per-Linear full 1024: 131072 tokens x 1024 bf16 ~ N(0,1), 1 % channels x50, full "
                       "1024-point Hadamard, MXFP4", 131072, 1024, 1024, "bf16", "mxfp4", 32),
    "c5rb": Workload("c5rb", "large R1 65536 tokens x hidden 8192 bf16 Student-t(3), full 8192-point random Hadamard "
                     "transpose (signs before), MXFP4", 65536, 8192, 8192, "bf16", "mxfp4", 32, signs="before",
                     base="c5"),
}

_STREAM = {"c1": 1, "c2": 2, "c3": 3, "c4q": 4, "c4k": 5, "c5": 6, "pl1024": 7}
_SIGN_STREAM = 100


def generate_signs(key: str, seed: int = SEED) -> np.ndarray:
    """The b int8 Rademacher signs (+/-1) of a random Hadamard workload."""
    w = WORKLOADS[key]
    if w.signs is None:
        raise ValueError(f"{key} has no random Hadamard signs")
    g = _rng(seed, _SIGN_STREAM, _STREAM[w.base or key])
    return np.where(g.random(w.block) < 0.5, -1, 1).astype(np.int8)


_RPBH_STREAM = 200


def generate_rpbh(key: str, seed: int = SEED):
    """The RPBH permutation (int32, a shuffle of the n columns) and its n int8
    Rademacher signs for an RPBH workload."""
    w = WORKLOADS[key]
    if not w.rpbh:
        raise ValueError(f"{key} has no RPBH permutation")
    g = _rng(seed, _RPBH_STREAM, _STREAM[w.base or key])
    perm = g.permutation(w.n).astype(np.int32)
    signs = np.where(g.random(w.n) < 0.5, -1, 1).astype(np.int8)
    return perm, signs


def _rng(seed: int, stream: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=(stream, chunk))))


def _outlier_set(seed: int, stream: int, n: int, k: int) -> np.ndarray:
    return _rng(seed + 1, stream, 0).permutation(n)[:k]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round half to even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bits_to_float64(x: np.ndarray, x_dtype: str) -> np.ndarray:
    """Exact float64 value of stored fp32 values or bf16 bit patterns."""
    if x_dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if x_dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(x_dtype)


def _chunk_values(key: str, chunk: int, seed: int) -> np.ndarray:
    key = WORKLOADS[key].base or key
    w = WORKLOADS[key]
    r0 = chunk * CHUNK_ROWS
    nr = min(CHUNK_ROWS, w.rows - r0)
    g = _rng(seed, _STREAM[key], chunk)
    if key == "c1":
        return g.standard_normal((nr, w.n))
    if key == "c2":
        v = g.standard_normal((nr, w.n))
        v[:, _outlier_set(seed, _STREAM[key], w.n, round(0.01 * w.n))] *= 50.0
        return v
    if key == "c3":
        a = g.standard_normal((nr, w.n))
        b = g.standard_normal((nr, w.n))
        v = a / (1.0 + np.exp(-a)) * b
        v[:, _outlier_set(seed, _STREAM[key], w.n, round(0.005 * w.n))] *= 30.0
        return v
    if key in ("c4q", "c4k"):
        seq, heads, d = 4096, 32, 128
        rows = np.arange(r0, r0 + nr)
        head = (rows // seq) % heads
        pos = (rows % seq).astype(np.float64)
        v = g.standard_normal((nr, d))
        for h in np.unique(head):
            dims = _rng(seed + 1, _STREAM[key], 1000 + int(h)).choice(d, 2, replace=False)
            sel = head == h
            v[np.ix_(sel, dims)] *= 20.0
        half = d // 2
        theta = 10000.0 ** (-np.arange(half) / half)
        ang = pos[:, None] * theta[None, :]
        c, s = np.cos(ang), np.sin(ang)
        x1, x2 = v[:, :half], v[:, half:]
        return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)
    if key == "c5":
        return g.standard_t(3, (nr, w.n))
    if key == "pl1024":
        v = g.standard_normal((nr, w.n))
        v[:, _outlier_set(seed, _STREAM[key], w.n, round(0.01 * w.n))] *= 50.0
        return v
    raise KeyError(key)


def _chunk_stored(key: str, chunk: int, seed: int) -> np.ndarray:
    vals = _chunk_values(key, chunk, seed).astype(np.float32)
    return vals if WORKLOADS[key].x_dtype == "f32" else f32_to_bf16_bits(vals)


def generate(key: str, rows: slice | None = None, seed: int = SEED, workers: int = 1) -> np.ndarray:
    """Stored input for rows ``rows`` of workload ``key``.

    Returns float32 values for fp32 workloads and uint16 bf16 bit patterns for
    bf16 workloads, shape (len(rows), n), row-major.  ``workers > 1``
    generates the chunks in a pool of spawned processes (spawned, not forked,
    so it is safe after CUDA has been initialised); the bits do not depend on
    the worker count.
    """
    w = WORKLOADS[key]
    r = range(w.rows)[rows if rows is not None else slice(None)]
    if r.step != 1:
        raise ValueError("row ranges must be contiguous")
    out = np.empty((len(r), w.n), dtype=np.float32 if w.x_dtype == "f32" else np.uint16)
    if len(r) == 0:
        return out
    chunks = list(range(r.start // CHUNK_ROWS, (r.stop - 1) // CHUNK_ROWS + 1))

    def place(c, stored):
        lo = max(r.start, c * CHUNK_ROWS)
        hi = min(r.stop, c * CHUNK_ROWS + stored.shape[0])
        out[lo - r.start: hi - r.start] = stored[lo - c * CHUNK_ROWS: hi - c * CHUNK_ROWS]

    if workers > 1 and len(chunks) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(max_workers=min(workers, len(chunks)), mp_context=mp.get_context("spawn")) as ex:
            for c, stored in zip(chunks, ex.map(_chunk_stored, [key] * len(chunks), chunks, [seed] * len(chunks))):
                place(c, stored)
    else:
        for c in chunks:
            place(c, _chunk_stored(key, c, seed))
    return out


def generate_rows(key: str, row_ids, seed: int = SEED) -> np.ndarray:
    """Stored input for an arbitrary set of rows (sorted or not)."""
    row_ids = np.asarray(row_ids, dtype=np.int64)
    w = WORKLOADS[key]
    out = np.empty((len(row_ids), w.n), dtype=np.float32 if w.x_dtype == "f32" else np.uint16)
    for c in np.unique(row_ids // CHUNK_ROWS):
        sel = np.nonzero(row_ids // CHUNK_ROWS == c)[0]
        block = generate(key, slice(int(c) * CHUNK_ROWS, min(w.rows, (int(c) + 1) * CHUNK_ROWS)), seed)
        out[sel] = block[row_ids[sel] - int(c) * CHUNK_ROWS]
    return out


def rank_seed(rank: int, seed: int = SEED) -> int:
    """Seed of the batch a rank owns when every rank processes its own full
    batch of the workload (weak scaling: per-GPU work fixed, no exchange)."""
    if rank < 0:
        raise ValueError("rank must be >= 0")
    return seed + 7919 * rank
