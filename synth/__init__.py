"""Seeded synthetic inputs for the Q4_0 decode path.

This module only *produces* input bytes: random nibbles, random block scales,
bf16 activation rows, and K/V caches quantised from normal samples.  It holds
none of the arithmetic the decode path computes (no dequantisation, no dot
product, no softmax).  Both the CPU oracle (through the tests) and the CUDA
path consume what it writes; neither of them is imported here.

Storage layout written here (the library's documented layout):

* Q4_0 block: 32 weights, one fp16 scale ``d`` and 16 bytes of nibbles; byte
  ``j`` holds element ``j`` in its low nibble and element ``j + 16`` in its
  high nibble; the weight is ``d * (q - 8)``.
* super-block: 256 consecutive elements (8 blocks) in 144 bytes -- the 8
  blocks' 16-byte nibble arrays first (bytes ``16*b .. 16*b+15``), then the 8
  fp16 scales (bytes ``128 + 2*b``, little endian).
* a weight matrix [N][K] is stored super-block-column-major: K/256 columns,
  column s holding super-block s of rows 0..N-1, so super-block (n, s) sits at
  byte (s*N + n)*144.  A K/V cache row (one token of one KV head, head_dim
  256) is one super-block, tokens of a head consecutive.

Recipes (the workloads of the decode path):

* weights: ``q ~ U{0..15}``, ``d = fp16(|N(0,1)| * 0.02)`` per block, drawn in
  that order (all q of the matrix, then all d);
* activations: ``x = bf16(N(0,1))`` rows, one independent row per draft row;
* K/V caches: ``N(0,1)`` values quantised per 32-block with ``amax`` = the
  signed element of largest magnitude, ``d = fp16(amax / -8)``,
  ``q = clamp(floor(v / d + 8.5), 0, 15)`` (``d = 0`` gives ``q = 8``);
* queries: ``bf16(N(0,1) / 16)``;
* Q8_0 K/V caches (the 8-bit cache variant): one 272-byte super-block per
  token: 256 int8 values (element ``j`` of block ``b`` at byte ``32*b + j``,
  two's complement), then the 8 fp16 scales (bytes ``256 + 2*b``); the value
  is ``d * q``.  Recipe: ``N(0,1)`` values per 32-block, ``d = fp16(amax/127)``
  with ``amax`` the largest magnitude, ``q = clamp(rint(v / d), -127, 127)``
  (``d = 0`` gives ``q = 0``).

Host generation uses ``numpy.random.default_rng(seed)`` (PCG64).  The large
workloads (gigabytes) are generated directly on the GPU with a seeded
``torch.Generator`` (Philox) following the same recipe; their values differ
from the host ones for the same seed, and checks against the oracle copy the
sampled device bytes back to the host.
"""
from __future__ import annotations

import numpy as np

SUPERBLOCK_ELEMS = 256
SUPERBLOCK_BYTES = 144
BLOCK_ELEMS = 32
BLOCKS_PER_SUPERBLOCK = 8


# --------------------------------------------------------------------------
# rounding helpers (fp32 -> bf16 / fp16 bit patterns, round-to-nearest-even)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = (u + 0x7FFF + lsb) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(np.asarray(v, dtype=np.float32))
    if nan.any():
        out[nan] = 0x7FC0
    return out


def f32_to_f16_bits(v: np.ndarray) -> np.ndarray:
    """Round float32 values to IEEE fp16 (numpy's RNE cast); return uint16 bits."""
    return np.asarray(v, dtype=np.float32).astype(np.float16).view(np.uint16)


# --------------------------------------------------------------------------
# packing into the super-block layout
# --------------------------------------------------------------------------
def pack_superblocks(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """Pack nibbles ``q[rows][K]`` (0..15) and scale bits ``d_bits[rows][K/32]``
    into ``rows * K/256`` super-blocks of 144 bytes (flat uint8 array)."""
    q = np.asarray(q, dtype=np.uint8)
    rows, K = q.shape
    if K % SUPERBLOCK_ELEMS:
        raise ValueError("K must be a multiple of 256")
    nsb = K // SUPERBLOCK_ELEMS
    d_bits = np.asarray(d_bits, dtype=np.uint16).reshape(rows, nsb, BLOCKS_PER_SUPERBLOCK)
    qb = q.reshape(rows, nsb, BLOCKS_PER_SUPERBLOCK, 2, 16)  # [.., half, j]
    nib = (qb[..., 0, :] | (qb[..., 1, :] << 4)).astype(np.uint8)  # [rows,nsb,8,16]
    out = np.empty((rows, nsb, SUPERBLOCK_BYTES), dtype=np.uint8)
    out[:, :, :128] = nib.reshape(rows, nsb, 128)
    out[:, :, 128:] = d_bits.astype("<u2").view(np.uint8).reshape(rows, nsb, 16)
    return out.reshape(-1)


def quantize_blocks(v: np.ndarray):
    """Quantise float values ``v[rows][K]`` per 32-block (recipe in the module
    docstring).  Returns ``(q uint8[rows][K], d_bits uint16[rows][K/32])``."""
    v = np.asarray(v, dtype=np.float32)
    rows, K = v.shape
    vb = v.reshape(rows, K // BLOCK_ELEMS, BLOCK_ELEMS)
    idx = np.abs(vb).argmax(axis=-1)
    amax = np.take_along_axis(vb, idx[..., None], axis=-1)[..., 0]
    d16 = (amax / np.float32(-8.0)).astype(np.float16)
    d16[d16 == 0] = 0  # an all-zero block stores d = +0
    d32 = d16.astype(np.float32)
    safe = np.where(d32 == 0, np.float32(1.0), d32)
    qf = np.floor(vb / safe[..., None] + np.float32(8.5))
    q = np.clip(qf, 0, 15).astype(np.uint8)
    q[d32 == 0] = 8
    return q.reshape(rows, K), d16.view(np.uint16)


# --------------------------------------------------------------------------
# host generators (numpy PCG64)
# --------------------------------------------------------------------------
def column_major(rows_buf: np.ndarray, N: int, K: int) -> np.ndarray:
    """Reorder super-blocks of a row-ordered matrix ([N][K/256]) into the
    weight layout ([K/256][N]), flat bytes."""
    nsb = K // SUPERBLOCK_ELEMS
    return np.ascontiguousarray(
        np.asarray(rows_buf, dtype=np.uint8).reshape(N, nsb, SUPERBLOCK_BYTES).transpose(1, 0, 2)
    ).reshape(-1)


def q4_0_weights(seed: int, N: int, K: int) -> np.ndarray:
    """Random Q4_0 weight matrix [N][K] in the weight layout (flat uint8)."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    d = np.abs(rng.standard_normal(size=(N, K // BLOCK_ELEMS))) * 0.02
    return column_major(pack_superblocks(q, f32_to_f16_bits(d.astype(np.float32))), N, K)


def bf16_normal(seed: int, shape, scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns of ``N(0,1) * scale`` (uint16 array of ``shape``)."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(size=shape) * scale
    return f32_to_bf16_bits(v.astype(np.float32))


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """M independent bf16 N(0,1) activation rows, uint16 bits [M][K]."""
    return bf16_normal(seed, (M, K))


def q4_0_kv_cache(seed: int, n_kv_heads: int, ctx: int, head_dim: int = 256) -> np.ndarray:
    """One K (or V) cache: N(0,1) values quantised per block, laid out as
    ``[n_kv_heads][ctx]`` super-blocks (flat uint8)."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(size=(n_kv_heads * ctx, head_dim)).astype(np.float32)
    q, d = quantize_blocks(v)
    return pack_superblocks(q, d)


Q8_SUPERBLOCK_BYTES = 272


def quantize_q8_blocks(v: np.ndarray):
    """Quantise float values ``v[rows][K]`` per 32-block to 8 bits (Q8_0 recipe
    in the module docstring).  Returns ``(q int8[rows][K], d_bits uint16[rows][K/32])``."""
    v = np.asarray(v, dtype=np.float32)
    rows, K = v.shape
    vb = v.reshape(rows, K // BLOCK_ELEMS, BLOCK_ELEMS)
    amax = np.abs(vb).max(axis=-1)
    d16 = (amax / np.float32(127.0)).astype(np.float16)
    d32 = d16.astype(np.float32)
    safe = np.where(d32 == 0, np.float32(1.0), d32)
    q = np.clip(np.rint(vb / safe[..., None]), -127, 127).astype(np.int8)
    q[d32 == 0] = 0
    return q.reshape(rows, K), d16.view(np.uint16)


def pack_q8_superblocks(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """int8 ``q[rows][K]`` and fp16 scale bits ``d_bits[rows][K/32]`` -> flat
    uint8 of ``rows * K/256`` Q8_0 super-blocks in row order."""
    rows, K = q.shape
    nsb = K // SUPERBLOCK_ELEMS
    out = np.empty((rows, nsb, Q8_SUPERBLOCK_BYTES), dtype=np.uint8)
    out[:, :, :256] = np.asarray(q, dtype=np.int8).view(np.uint8).reshape(rows, nsb, 256)
    out[:, :, 256:] = (np.asarray(d_bits, dtype=np.uint16).reshape(rows, nsb, 8)
                       .view(np.uint8).reshape(rows, nsb, 16))
    return out.reshape(-1)


def q8_0_kv_cache(seed: int, n_kv_heads: int, ctx: int, head_dim: int = 256) -> np.ndarray:
    """One Q8_0 K (or V) cache: N(0,1) values quantised per block, laid out as
    ``[n_kv_heads][ctx]`` 272-byte super-blocks (flat uint8)."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(size=(n_kv_heads * ctx, head_dim)).astype(np.float32)
    q, d = quantize_q8_blocks(v)
    return pack_q8_superblocks(q, d)


def queries(seed: int, M: int, n_q_heads: int, head_dim: int = 256) -> np.ndarray:
    """bf16 bits of ``N(0,1)/16`` queries, shape [M][n_q_heads][head_dim]."""
    return bf16_normal(seed, (M, n_q_heads, head_dim), scale=1.0 / 16.0)


def from_parts(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Pack explicit nibbles and float scales (rounded to fp16) row after row
    -- the K/V cache layout; hand-made cases (all q = 8, powers of two ...)."""
    return pack_superblocks(q, f32_to_f16_bits(np.asarray(d, dtype=np.float32)))


def weights_from_parts(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Like ``from_parts`` but in the weight layout (column-major super-blocks)."""
    q = np.asarray(q, dtype=np.uint8)
    return column_major(from_parts(q, d), q.shape[0], q.shape[1])


# --------------------------------------------------------------------------
# device generators (torch, seeded Philox) for the multi-gigabyte workloads
# --------------------------------------------------------------------------
def _torch():
    import torch  # local import: host-only users need no torch

    return torch


def device_q4_0_weights(seed: int, N: int, K: int, device="cuda"):
    """Random Q4_0 weight matrix [N][K] generated on ``device``; returns a
    flat uint8 tensor in the weight layout (same recipe as ``q4_0_weights``)."""
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    nsb = K // SUPERBLOCK_ELEMS
    out = torch.empty((nsb, N, SUPERBLOCK_BYTES), dtype=torch.uint8, device=device)
    # q: two uniform nibbles per byte == one uniform byte
    out[:, :, :128] = torch.randint(0, 256, (nsb, N, 128), generator=g, device=device,
                                    dtype=torch.int32).to(torch.uint8)
    d = (torch.randn((nsb, N, 8), generator=g, device=device).abs() * 0.02).to(torch.float16)
    out[:, :, 128:] = d.view(torch.uint8).reshape(nsb, N, 16)
    return out.reshape(-1)


def device_bf16_normal(seed: int, shape, scale: float = 1.0, device="cuda"):
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=device) * scale).to(torch.bfloat16)


def device_q4_0_kv_cache(seed: int, n_kv_heads: int, ctx: int, head_dim: int = 256,
                         device="cuda", chunk_tokens: int = 1 << 16):
    """K (or V) cache of N(0,1) values quantised per block, generated on the
    device in chunks; flat uint8 tensor ``[n_kv_heads][ctx]`` super-blocks."""
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    rows = n_kv_heads * ctx
    nsb = head_dim // SUPERBLOCK_ELEMS
    out = torch.empty((rows, nsb, SUPERBLOCK_BYTES), dtype=torch.uint8, device=device)
    for r0 in range(0, rows, chunk_tokens):
        r1 = min(rows, r0 + chunk_tokens)
        v = torch.randn((r1 - r0, head_dim), generator=g, device=device)
        vb = v.reshape(r1 - r0, head_dim // BLOCK_ELEMS, BLOCK_ELEMS)
        idx = vb.abs().argmax(dim=-1, keepdim=True)
        amax = torch.gather(vb, -1, idx)[..., 0]
        d16 = (amax / -8.0).to(torch.float16)
        d16[d16 == 0] = 0  # an all-zero block stores d = +0
        d32 = d16.to(torch.float32)
        safe = torch.where(d32 == 0, torch.ones_like(d32), d32)
        q = torch.floor(vb / safe[..., None] + 8.5).clamp_(0, 15).to(torch.uint8)
        q[d32 == 0] = 8
        q = q.reshape(r1 - r0, nsb, 8, 2, 16)
        nib = q[..., 0, :] | (q[..., 1, :] << 4)
        out[r0:r1, :, :128] = nib.reshape(r1 - r0, nsb, 128)
        out[r0:r1, :, 128:] = d16.view(torch.uint8).reshape(r1 - r0, nsb, 16)
    return out.reshape(-1)


def device_q8_0_kv_cache(seed: int, n_kv_heads: int, ctx: int, head_dim: int = 256,
                         device="cuda", chunk_tokens: int = 1 << 16):
    """Q8_0 K (or V) cache of N(0,1) values quantised per block, generated on
    the device in chunks; flat uint8 tensor ``[n_kv_heads][ctx]`` super-blocks."""
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    rows = n_kv_heads * ctx
    nsb = head_dim // SUPERBLOCK_ELEMS
    out = torch.empty((rows, nsb, Q8_SUPERBLOCK_BYTES), dtype=torch.uint8, device=device)
    for r0 in range(0, rows, chunk_tokens):
        r1 = min(rows, r0 + chunk_tokens)
        v = torch.randn((r1 - r0, head_dim), generator=g, device=device)
        vb = v.reshape(r1 - r0, head_dim // BLOCK_ELEMS, BLOCK_ELEMS)
        d16 = (vb.abs().amax(dim=-1) / 127.0).to(torch.float16)
        d32 = d16.to(torch.float32)
        safe = torch.where(d32 == 0, torch.ones_like(d32), d32)
        q = torch.round(vb / safe[..., None]).clamp_(-127, 127).to(torch.int8)
        q[d32 == 0] = 0
        out[r0:r1, :, :256] = q.view(torch.uint8).reshape(r1 - r0, nsb, 256)
        out[r0:r1, :, 256:] = d16.view(torch.uint8).reshape(r1 - r0, nsb, 16)
    return out.reshape(-1)
