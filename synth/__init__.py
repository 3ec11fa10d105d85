"""Seeded synthetic inputs for MoE expert-parallel token routing.

This module only *draws inputs*: router outputs (top-K expert ids and their gate
weights), hidden rows, and the inputs of the logical->physical mapping op (an
eplb_table, pruning thresholds, an active mask). It computes nothing of the routing
method itself (no histogram, no placement, no mapping, no dispatch or combine), so
both the oracle under ``oracle/`` and the CUDA path can consume the same inputs
without sharing any of the method's arithmetic.

Workload shapes follow the pages:
  * MoonEP benchmark defaults (twodots.gr article on MoonEP, "public benchmark"
    paragraph): S=8192 tokens per rank, E=384 experts, H=7168, K=8, EP=8.
  * aclnnMoeUpdateExpert (gitcode ops-transformer doc, "参数说明" / "约束说明"):
    eplb_table of shape (moeExpertNum, F), column 0 = instance count, columns
    1..count = distinct instance ids in [0, world_size*place_per_rank);
    expert_scales descending per token; pruning_threshold of shape (K,);
    active_mask with every True before every False.

Randomness: numpy's PCG64 generator, seeded through ``SeedSequence([seed, tag,
chunk])`` so that every array is reproducible and independent of thread count.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

# Distinct stream tags, one per kind of draw.
_TAG_LOGITS = 1
_TAG_PERM = 2
_TAG_HIDDEN = 3
_TAG_OUTLIER = 4
_TAG_TABLE = 5
_TAG_THR = 6
_TAG_Y = 7

_ROWS_PER_CHUNK = 2048


@dataclasses.dataclass(frozen=True)
class Workload:
    """One routing workload: R simulated EP ranks of S tokens, K of E experts each."""

    name: str
    R: int                 # simulated expert-parallel ranks (partitions of one GPU's HBM)
    E: int                 # logical experts, E % R == 0, home(e) = e // (E // R)
    S: int                 # tokens per rank
    K: int                 # experts per token
    H: int                 # hidden size (bf16 elements per row)
    zipf_s: float          # exponent of the per-expert Zipf bias on router logits
    permute: bool          # shuffle which expert gets which Zipf rank
    seed: int
    quant: int = 0         # 0: bf16 dispatch, 1: per-token dynamic int8 dispatch
    outlier_frac: float = 0.0   # fraction of hidden rows scaled by outlier_scale
    outlier_scale: float = 1.0
    force_expert0: bool = False  # expert 0 joins every token's top-K
    # Logical->physical mapping op (aclnnMoeUpdateExpert) parameters
    mapping: bool = False
    place_per_rank: int = 0
    F: int = 0
    n_hot: int = 0          # experts that get a second instance
    n_active: int = 0       # tokens per rank with active_mask = True

    @property
    def T(self) -> int:
        return self.R * self.S

    @property
    def N(self) -> int:
        return self.R * self.S * self.K


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_r4_e16_s128_k2_h256", R=4, E=16, S=128, K=2, H=256,
                 zipf_s=1.2, permute=False, seed=0),
        Workload("r8_e64_s4096_k8_h7168", R=8, E=64, S=4096, K=8, H=7168,
                 zipf_s=1.0, permute=True, seed=1),
        Workload("map_ws8_bs256_k8_e256_ppr34_h4096", R=8, E=256, S=256, K=8, H=4096,
                 zipf_s=1.0, permute=True, seed=2, mapping=True, place_per_rank=34,
                 F=3, n_hot=16, n_active=200),
        Workload("int8_r32_e256_s8192_k8_h7168", R=32, E=256, S=8192, K=8, H=7168,
                 zipf_s=1.1, permute=True, seed=3, quant=1, outlier_frac=0.01,
                 outlier_scale=20.0),
        Workload("skew_r64_e512_s2048_k8_h4096", R=64, E=512, S=2048, K=8, H=4096,
                 zipf_s=1.5, permute=True, seed=4, force_expert0=True),
    ]
}

# Short aliases, in the order the five workloads are listed.
ALIASES = {
    "tiny": "tiny_r4_e16_s128_k2_h256",
    "r8": "r8_e64_s4096_k8_h7168",
    "map": "map_ws8_bs256_k8_e256_ppr34_h4096",
    "int8": "int8_r32_e256_s8192_k8_h7168",
    "skew": "skew_r64_e512_s2048_k8_h4096",
}


def get(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields replaced (e.g. a smaller S for a fast case)."""
    return dataclasses.replace(w, **changes)


def _rng(seed: int, tag: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, chunk])))


def zipf_bias(w: Workload) -> np.ndarray:
    """Per-expert additive logit bias ln((rank+1)^-s), rank = Zipf rank of the expert."""
    if w.permute:
        rank = _rng(w.seed, _TAG_PERM).permutation(w.E)
    else:
        rank = np.arange(w.E)
    return -w.zipf_s * np.log(rank.astype(np.float64) + 1.0), rank


def _topk_rows(z: np.ndarray, K: int) -> np.ndarray:
    """Columns of the K largest entries per row, largest first, ties to the lower column."""
    order = np.argsort(-z, axis=1, kind="stable")
    return order[:, :K]


def router(w: Workload, threads: int = 8):
    """Top-K expert ids (int32 [T,K]) and gates (fp32 [T,K]) of a synthetic router.

    Logits z = N(0,1) + Zipf bias; ids = the K largest z per token, in descending z;
    gates = softmax of the chosen logits (computed in float64, stored as fp32), so
    gates are descending within a token and sum to 1 up to fp32 rounding.
    With ``force_expert0`` the token's set is expert 0 plus the K-1 largest of experts
    1..E-1, ordered by z like the rest.
    """
    bias, _ = zipf_bias(w)
    T, E, K = w.T, w.E, w.K
    ids = np.empty((T, K), np.int32)
    gates = np.empty((T, K), np.float32)
    nchunks = (T + _ROWS_PER_CHUNK - 1) // _ROWS_PER_CHUNK

    def work(c):
        lo, hi = c * _ROWS_PER_CHUNK, min(T, (c + 1) * _ROWS_PER_CHUNK)
        z = _rng(w.seed, _TAG_LOGITS, c).standard_normal((hi - lo, E)) + bias[None, :]
        if w.force_expert0:
            rest = _topk_rows(z[:, 1:], K - 1) + 1
            cand = np.concatenate([np.zeros((hi - lo, 1), np.int64), rest], axis=1)
            zc = np.take_along_axis(z, cand, axis=1)
            # order the K candidates by z descending, ties to the lower expert id
            o = np.lexsort((cand, -zc), axis=1)
            sel = np.take_along_axis(cand, o, axis=1)
        else:
            sel = _topk_rows(z, K)
        zs = np.take_along_axis(z, sel, axis=1)
        ez = np.exp(zs - zs[:, :1])
        g = ez / ez.sum(axis=1, keepdims=True)
        ids[lo:hi] = sel.astype(np.int32)
        gates[lo:hi] = g.astype(np.float32)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(nchunks)))
    return ids, gates


def hidden(w: Workload, threads: int = 8, rows: Optional[int] = None, tag: int = _TAG_HIDDEN):
    """bf16 hidden rows ~ N(0,1), as a torch.bfloat16 CPU tensor of shape [rows, H].

    ``rows`` defaults to T. A fraction ``outlier_frac`` of rows (seeded choice) is
    multiplied by ``outlier_scale`` in fp32 before the round-to-nearest-even
    conversion to bf16.
    """
    import torch

    T = w.T if rows is None else rows
    H = w.H
    out = torch.empty((T, H), dtype=torch.bfloat16)
    scale = np.ones(T, np.float32)
    if w.outlier_frac > 0 and tag == _TAG_HIDDEN:
        n_out = max(1, int(round(w.outlier_frac * T)))
        scale[_rng(w.seed, _TAG_OUTLIER).choice(T, size=n_out, replace=False)] = w.outlier_scale
    nchunks = (T + _ROWS_PER_CHUNK - 1) // _ROWS_PER_CHUNK

    def work(c):
        lo, hi = c * _ROWS_PER_CHUNK, min(T, (c + 1) * _ROWS_PER_CHUNK)
        f = _rng(w.seed, tag, c).standard_normal((hi - lo, H), dtype=np.float32)
        f *= scale[lo:hi, None]
        out[lo:hi] = torch.from_numpy(f).to(torch.bfloat16)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(nchunks)))
    return out


def expert_outputs(w: Workload, rows: int, threads: int = 8):
    """Arbitrary bf16 rows ~ N(0,1) [rows, H] standing in for expert outputs.

    Used to test combine on rows that are not copies of the token's own hidden row.
    """
    return hidden(w, threads=threads, rows=rows, tag=_TAG_Y)


def mapping_inputs(w: Workload):
    """Inputs of the logical->physical mapping op for every simulated rank.

    Returns (eplb_table int32 [E, F], pruning_threshold fp32 [K], active_mask bool [T]).

    eplb_table: the ``n_hot`` experts with the largest Zipf bias get two instances,
    every other expert one; instance ids are a seeded permutation of
    [0, R*place_per_rank) dealt in expert order (first instance, then the replica).
    Column 0 holds the count, columns 1..count the ids, unused columns hold -1.
    The physical rank of an instance id is id // place_per_rank, so every rank holds
    exactly place_per_rank instances.
    pruning_threshold[k] ~ U[0, 0.1). active_mask: the first ``n_active`` of each
    rank's S tokens are True, the rest False.
    """
    assert w.mapping
    _, zrank = zipf_bias(w)
    hot = zrank < w.n_hot
    n_inst = w.E + int(hot.sum())
    assert n_inst == w.R * w.place_per_rank, (n_inst, w.R * w.place_per_rank)
    assert w.F >= 3 or w.n_hot == 0
    perm = _rng(w.seed, _TAG_TABLE).permutation(n_inst).astype(np.int32)
    table = np.full((w.E, w.F), -1, np.int32)
    j = 0
    for e in range(w.E):
        c = 2 if hot[e] else 1
        table[e, 0] = c
        table[e, 1:1 + c] = perm[j:j + c]
        j += c
    thr = (_rng(w.seed, _TAG_THR).random(w.K) * 0.1).astype(np.float32)
    active = np.zeros((w.R, w.S), bool)
    active[:, : w.n_active] = True
    return table, thr, active.reshape(-1)
