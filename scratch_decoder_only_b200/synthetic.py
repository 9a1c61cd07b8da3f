"""Seeded synthetic inputs (token ids, targets, segment ids, prompts).

This module holds no arithmetic of the model; it only draws integer inputs
with numpy's PCG64 generator, so that the same arrays can be handed to the
CUDA library and to the CPU oracle.  The corpora the pages train on are not
available; these draws stand in for them with the shapes and distributions
the workloads state.

Recipes:
* uniform bytes: ids i.i.d. uniform over 0..256 inclusive (257 values);
* Zipf(s) over V ids: P(id = k) proportional to (k+1)^-s, sampled by inverse CDF;
* skewed bytes: weight 20*u_b for printable b in 32..126, u_b otherwise
  (u_b ~ U(0.5, 1.5)) for b in 0..255, and 0 for id 256;
* packing: documents of length ~ U[16, 512] are laid end to end in a row of
  T+1 tokens until it is full (the last one truncated); seg_ids number the
  documents of a row from 0.

Targets are the input shifted by one; in a packed row a position whose next
token belongs to another document gets target -1 (ignored).
"""
from __future__ import annotations

import numpy as np


def zipf_ids(rng, n, vocab, s):
    k = np.arange(vocab, dtype=np.float64)
    w = (k + 1.0) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1).astype(np.int64)


def skewed_byte_ids(rng, n):
    u = rng.uniform(0.5, 1.5, size=256)
    w = u.copy()
    w[32:127] *= 20.0
    w = np.concatenate([w, [0.0]])
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    return np.minimum(np.searchsorted(cdf, rng.random(n), side="right"), 255).astype(np.int64)


def packed_segments(rng, rows, length, lo=16, hi=512):
    seg = np.zeros((rows, length), dtype=np.int64)
    for r in range(rows):
        t, doc = 0, 0
        while t < length:
            L = int(rng.integers(lo, hi + 1))
            L = min(L, length - t)
            seg[r, t:t + L] = doc
            t += L
            doc += 1
    return seg


def shift_targets(x, seg=None):
    """inputs = x[:, :T], targets = x[:, 1:T+1] (-1 across a document boundary)."""
    tokens = x[:, :-1].copy()
    targets = x[:, 1:].copy()
    if seg is not None:
        cross = seg[:, 1:] != seg[:, :-1]
        targets[cross] = -1
    return tokens, targets


def make_batch(workload, batch=None, seq=None, seed=None):
    """(tokens, targets, seg_ids or None) as int32 arrays for a workload."""
    B = batch or workload.batch
    T = seq or workload.seq
    rng = np.random.default_rng(workload.data_seed if seed is None else seed)
    V = workload.model.vocab
    name = workload.name
    seg = None
    if name.startswith("tiny-byte"):
        x = rng.integers(0, 257, size=(B, T + 1))
    elif name.startswith("packed"):
        seg_full = packed_segments(rng, B, T + 1)
        x = zipf_ids(rng, B * (T + 1), V, 1.1).reshape(B, T + 1)
        seg = seg_full
    elif name.startswith("byte30m"):
        x = skewed_byte_ids(rng, B * (T + 1)).reshape(B, T + 1)
    elif name.startswith("gpt2-124m-v"):
        x = zipf_ids(rng, B * (T + 1), V, 1.0).reshape(B, T + 1)
    else:
        x = rng.integers(0, V, size=(B, T + 1))
    tokens, targets = shift_targets(x, seg)
    seg_in = None if seg is None else seg[:, :T].astype(np.int32)
    return tokens.astype(np.int32), targets.astype(np.int32), seg_in


def make_prompts(workload, batch, prompt_len=128, seed=None):
    rng = np.random.default_rng(workload.data_seed if seed is None else seed)
    return rng.integers(0, workload.model.vocab, size=(batch, prompt_len)).astype(np.int32)


def random_tokens(rng, B, T, V):
    x = rng.integers(0, V, size=(B, T + 1))
    t, y = shift_targets(x)
    return t.astype(np.int32), y.astype(np.int32)
