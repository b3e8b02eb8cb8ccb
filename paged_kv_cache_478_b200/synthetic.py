"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws inputs: context lengths, block placements, query and
KV values.  It computes nothing of the method itself (no slot arithmetic, no
attention, no block management); the CUDA path and the CPU oracle each do
that on their own.

Workload shapes follow the pages' GPT-style setting ("Atención paginada en
modelos de lenguaje grandes (LLM)", 7minutos.es, section 1: 32 layers, 32
heads, head_dim 128, fp16, 16-token pages; maximum length 2048 and mean
response about 500 tokens; 10 to 200 concurrent requests).

Conventions:
  pools are [num_blocks, heads, block_size, head_dim];
  block_tables are int32 [num_seqs, max_blocks] with -1 past a sequence's
  last block; context_lens are the lengths AFTER the new token is appended,
  so the new token sits at position context_len - 1.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK_SIZE = 16


def _normal(rng, shape, dtype):
    """N(0,1) drawn in fp32 and rounded to dtype (round to nearest even)."""
    return rng.standard_normal(shape, dtype=np.float32).astype(dtype)


def _blocks_for(lengths, block_size=BLOCK_SIZE):
    return [int(math.ceil(int(n) / block_size)) for n in lengths]


def random_tables(rng, lengths, num_pool_blocks, max_blocks, block_size=BLOCK_SIZE):
    """Give each sequence's logical blocks distinct physical ids drawn from a
    seeded random permutation of the pool, consumed in sequence order."""
    need = _blocks_for(lengths, block_size)
    total = sum(need)
    if total > num_pool_blocks:
        raise ValueError("pool too small for the requested lengths")
    perm = rng.permutation(num_pool_blocks).astype(np.int32)
    tables = np.full((len(lengths), max_blocks), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    return tables


def decode_case(seed, lengths, heads, head_dim, dtype, num_pool_blocks=None, max_blocks=None,
                block_size=BLOCK_SIZE, pool_fill="normal"):
    """A one-step decode problem with host (numpy) arrays.

    lengths are post-append context lengths.  The pool is filled entirely
    with N(0,1) values (pool_fill="normal"), or with NaN (pool_fill="nan"), in
    which case the caller writes the cached tokens itself and anything read
    outside them poisons the output.
    Returns a dict with q, k_new, v_new [S,H,D]; k_pool, v_pool; block_tables;
    context_lens; scale = 1/sqrt(head_dim).
    """
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int32)
    S = len(lengths)
    need = _blocks_for(lengths, block_size)
    if num_pool_blocks is None:
        num_pool_blocks = max(1, sum(need))
    if max_blocks is None:
        max_blocks = max(1, max(need) if need else 1)
    tables = random_tables(rng, lengths, num_pool_blocks, max_blocks, block_size)
    shape = (num_pool_blocks, heads, block_size, head_dim)
    if pool_fill == "nan":
        k_pool = np.full(shape, np.nan, dtype=dtype)
        v_pool = np.full(shape, np.nan, dtype=dtype)
    else:
        k_pool = _normal(rng, shape, dtype)
        v_pool = _normal(rng, shape, dtype)
    q = _normal(rng, (S, heads, head_dim), dtype)
    k_new = _normal(rng, (S, heads, head_dim), dtype)
    v_new = _normal(rng, (S, heads, head_dim), dtype)
    return dict(q=q, k_new=k_new, v_new=v_new, k_pool=k_pool, v_pool=v_pool,
                block_tables=tables, context_lens=lengths, scale=1.0 / math.sqrt(head_dim),
                block_size=block_size)


# ---- the five workloads -------------------------------------------------------------

def tiny_case(seed=0):
    """4 sequences with lengths {1,15,16,33}, 2 heads, head_dim 64, fp32,
    pool of 16 blocks placed by a seeded permutation, scale 1/8."""
    return decode_case(seed, [1, 15, 16, 33], heads=2, head_dim=64, dtype=np.float32,
                       num_pool_blocks=16)


def single_layer_lengths(seed=0, num_seqs=64, max_len=2048):
    """Context lengths uniform in [1, max_len]."""
    return np.random.default_rng(seed).integers(1, max_len + 1, size=num_seqs).astype(np.int32)


def single_layer_case(seed=0, num_seqs=64, heads=32, head_dim=128, max_len=2048):
    """One layer of GPT-style decode: 64 sequences, lengths uniform in
    [1,2048], fp16, pool sized to exactly the used blocks."""
    lengths = single_layer_lengths(seed, num_seqs, max_len)
    return decode_case(seed + 1, lengths, heads, head_dim, np.float16,
                       max_blocks=int(math.ceil(max_len / BLOCK_SIZE)))


def full_step_lengths(seed=0, num_seqs=200, max_len=2048, mean=500.0):
    """Context lengths min(max_len, 1 + floor(Exponential(mean)))."""
    rng = np.random.default_rng(seed)
    e = np.floor(rng.exponential(mean, size=num_seqs)).astype(np.int64)
    return np.minimum(max_len, 1 + e).astype(np.int32)


def full_step_tables(seed, lengths, max_len=2048):
    """Random placement of every sequence's blocks in one shared pool of
    exactly the used blocks (one block-id space shared by all layers)."""
    rng = np.random.default_rng(seed + 7)
    total = sum(_blocks_for(lengths))
    tables = random_tables(rng, lengths, total, int(math.ceil(max_len / BLOCK_SIZE)))
    return tables, total


def long_context_tables(seed=0, num_seqs=8, context=32768):
    lengths = np.full(num_seqs, context, dtype=np.int32)
    rng = np.random.default_rng(seed)
    total = num_seqs * (context // BLOCK_SIZE)
    tables = random_tables(rng, lengths, total, context // BLOCK_SIZE)
    return lengths, tables, total


def shared_prefix_case(seed=0, num_seqs=128, heads=32, head_dim=128, prefix_len=1000,
                       max_suffix=512, dtype=np.float16):
    """A common system prefix of prefix_len tokens held by num_seqs
    sequences, then a per-sequence suffix of uniform [1, max_suffix] tokens.

    Returns token data only: prefix K/V [prefix_len, H, D], suffix K/V as a
    list of [n_s, H, D] arrays, q [S, H, D].  Block management (sharing,
    copy-on-write, slots) is left to whoever consumes the case.
    """
    rng = np.random.default_rng(seed)
    suffix = rng.integers(1, max_suffix + 1, size=num_seqs).astype(np.int32)
    k_prefix = _normal(rng, (prefix_len, heads, head_dim), dtype)
    v_prefix = _normal(rng, (prefix_len, heads, head_dim), dtype)
    k_suffix = [_normal(rng, (int(n), heads, head_dim), dtype) for n in suffix]
    v_suffix = [_normal(rng, (int(n), heads, head_dim), dtype) for n in suffix]
    q = _normal(rng, (num_seqs, heads, head_dim), dtype)
    return dict(prefix_len=prefix_len, suffix_lens=suffix, k_prefix=k_prefix, v_prefix=v_prefix,
                k_suffix=k_suffix, v_suffix=v_suffix, q=q, scale=1.0 / math.sqrt(head_dim),
                heads=heads, head_dim=head_dim, block_size=BLOCK_SIZE)


# ---- device-side fills for pools too large to draw on the host ----------------------

def fill_normal_device(tensor, seed):
    """Fill a CUDA tensor in place with seeded N(0,1) values (torch's Philox
    generator), for pools of tens of GB."""
    import torch

    g = torch.Generator(device=tensor.device)
    g.manual_seed(int(seed))
    tensor.normal_(0.0, 1.0, generator=g)
    return tensor
