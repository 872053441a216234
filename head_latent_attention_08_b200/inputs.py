"""Seeded synthetic inputs shared by the CUDA path's tests, the oracle's tests and the benchmark.

This module only draws random numbers and casts them to the storage dtype. It does none of the
method's arithmetic: no normalisation, no rotation, no projection, no softmax. Both sides of every
parity check receive the very same arrays from here.

Distributions (the workloads of the absorbed-decode configurations):

* activations, latent rows ``c_t`` and rotary parts ``q_pe`` / ``k_pe``: N(0, 1);
* weights: N(0, 1/fan_in), where fan_in is the width the weight contracts over when applied;
* bf16 workloads: every value is rounded once (round-to-nearest-even) to bf16 and stored as the
  float32 number it represents, so the oracle and the GPU read identical values.

Two readings are built in here, stated where they apply:

* A RoPE rotation is orthogonal, so a rotated N(0, 1) pair is again N(0, 1). Drawing ``q_pe`` and
  ``k_pe`` as N(0, 1) therefore gives exactly the distribution of "N(0, 1) rotated at its position".
* An RMS-normalised N(0, 1) row of width d has RMS exactly 1; a raw N(0, 1) row has RMS
  1 +- O(1/sqrt(d)). Cache rows are drawn raw; the normalisation itself is exercised by the append
  step (its RMSNorm flag), which every decode step applies to the freshly appended row.
"""
from __future__ import annotations

import dataclasses
import numpy as np
import torch

__all__ = [
    "DecodeProblem",
    "GatedProblem",
    "ProjectionWeights",
    "NotebookProblem",
    "round_to",
    "decode_problem",
    "gated_problem",
    "projection_weights",
    "notebook_problem",
    "ragged_seqlens",
    "CONFIG_SEEDS",
]

# seed of configuration k (1-based) is 1000 + k; a second seed (7) is used by the CI-sized cases
CONFIG_SEEDS = {k: 1000 + k for k in range(1, 6)}


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round ``x`` to the storage dtype ('f32', 'bf16' or 'e4m3') and return it as float32 values.
    'e4m3' saturates at +-448 (the format's largest finite value) before torch's cast."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    if dtype == "e4m3":
        return torch.from_numpy(np.clip(x, -448.0, 448.0)).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def ragged_seqlens(batch: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Integer context lengths drawn uniformly in [lo, hi] (both ends included)."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=batch, dtype=np.int64)


@dataclasses.dataclass
class DecodeProblem:
    """One absorbed-decode step: the inputs of append, query absorption, decode and projection.

    Shapes (N_q = batch * n_q):
      q_nope [N_q, H, qk_nope], q_pe [N_q, H, rope_dim], w_uk [H, qk_nope, d_c],
      w_uv [H, v_head, d_c], w_o [d_model, H * v_head],
      cache [sum(seqlens), d_c + rope_dim] (sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]),
      c_new [N_q, d_c] and kpe_new [N_q, rope_dim]: the raw (un-normed, un-rotated) latent of the
      n_q newest tokens of each sequence, appended at rows row_idx with RoPE positions positions.
    """

    dtype: str
    n_heads: int
    kv_lora_rank: int
    rope_dim: int
    qk_nope: int
    v_head: int
    d_model: int
    n_q: int
    seqlens: np.ndarray
    cu_seqlens: np.ndarray
    q_nope: np.ndarray
    q_pe: np.ndarray
    w_uk: np.ndarray
    w_uv: np.ndarray
    w_o: np.ndarray
    cache: np.ndarray
    c_new: np.ndarray
    kpe_new: np.ndarray
    row_idx: np.ndarray
    positions: np.ndarray

    @property
    def batch(self) -> int:
        return int(self.seqlens.shape[0])

    @property
    def width(self) -> int:
        return self.kv_lora_rank + self.rope_dim

    @property
    def kq_scale(self) -> float:
        return 1.0 / float(np.sqrt(self.qk_nope + self.rope_dim))


def decode_problem(*, batch: int, n_heads: int, kv_lora_rank: int, rope_dim: int, qk_nope: int,
                   v_head: int, d_model: int, seqlens, n_q: int = 1, dtype: str = "f32",
                   seed: int = 7, with_weights: bool = True, cache_dtype: str = "") -> DecodeProblem:
    seqlens = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    if seqlens.shape[0] != batch:
        raise ValueError("seqlens must have one entry per sequence")
    if np.any(seqlens < n_q):
        raise ValueError("every sequence must hold at least its n_q query tokens")
    rng = np.random.default_rng(seed)
    H, dc, dr, n, dv, D = n_heads, kv_lora_rank, rope_dim, qk_nope, v_head, d_model
    nq_tot = batch * n_q
    cu = np.zeros(batch + 1, dtype=np.int64)
    cu[1:] = np.cumsum(seqlens)
    total = int(cu[-1])
    q_nope = round_to(_normal(rng, (nq_tot, H, n)), dtype)
    q_pe = round_to(_normal(rng, (nq_tot, H, dr)), dtype)
    if with_weights:
        w_uk = round_to(_normal(rng, (H, n, dc), 1.0 / np.sqrt(n)), dtype)
        w_uv = round_to(_normal(rng, (H, dv, dc), 1.0 / np.sqrt(dc)), dtype)
        w_o = round_to(_normal(rng, (D, H * dv), 1.0 / np.sqrt(H * dv)), dtype)
    else:
        w_uk = np.zeros((0,), np.float32)
        w_uv = np.zeros((0,), np.float32)
        w_o = np.zeros((0,), np.float32)
    cache = round_to(_normal(rng, (total, dc + dr)), cache_dtype or dtype)
    c_new = _normal(rng, (nq_tot, dc))
    kpe_new = _normal(rng, (nq_tot, dr))
    # the n_q newest tokens of sequence b sit at its last n_q rows, at positions T_b - n_q .. T_b - 1
    row_idx = np.concatenate([np.arange(cu[b + 1] - n_q, cu[b + 1]) for b in range(batch)]).astype(np.int64)
    positions = np.concatenate([np.arange(seqlens[b] - n_q, seqlens[b]) for b in range(batch)]).astype(np.int32)
    return DecodeProblem(dtype, H, dc, dr, n, dv, D, n_q, seqlens, cu, q_nope, q_pe, w_uk, w_uv, w_o,
                         cache, c_new, kpe_new, row_idx, positions)


@dataclasses.dataclass
class ProjectionWeights:
    """Hidden states and the input-projection weights of one decode step, PyTorch Linear
    convention (weight = [out, in]):

      x [N, d_model]; w_cq [q_rank, d_model] (the query down-projection);
      w_qc [H * qk_nope, q_rank] and w_qr [H * rope_dim, q_rank] (head h owns rows h*qk_nope.. and
      h*rope_dim..); w_dkv [d_c + rope_dim, d_model]: the latent rows first, then the rotary-key rows.
    """

    x: np.ndarray
    w_cq: np.ndarray
    w_qc: np.ndarray
    w_qr: np.ndarray
    w_dkv: np.ndarray


def projection_weights(*, n_tokens: int, d_model: int, q_rank: int, n_heads: int, qk_nope: int,
                       rope_dim: int, kv_lora_rank: int, dtype: str = "f32",
                       seed: int = 7) -> ProjectionWeights:
    rng = np.random.default_rng(seed)
    H, D = n_heads, d_model
    x = round_to(_normal(rng, (n_tokens, D)), dtype)
    w_cq = round_to(_normal(rng, (q_rank, D), 1.0 / np.sqrt(D)), dtype)
    w_qc = round_to(_normal(rng, (H * qk_nope, q_rank), 1.0 / np.sqrt(q_rank)), dtype)
    w_qr = round_to(_normal(rng, (H * rope_dim, q_rank), 1.0 / np.sqrt(q_rank)), dtype)
    w_dkv = round_to(_normal(rng, (kv_lora_rank + rope_dim, D), 1.0 / np.sqrt(D)), dtype)
    return ProjectionWeights(x, w_cq, w_qc, w_qr, w_dkv)


@dataclasses.dataclass
class GatedProblem:
    """Gated MLA prefill inputs in the PyTorch Linear convention (weight = [out, in])."""

    dtype: str
    num_heads: int
    causal: bool
    x: np.ndarray      # [B, S, D]
    wq: np.ndarray     # [D, D]
    wc: np.ndarray     # [L, D]
    wk: np.ndarray     # [D, L]
    wv: np.ndarray     # [D, L]
    wg: np.ndarray     # [D, D]
    wo: np.ndarray     # [D, D]


def gated_problem(*, batch: int, seq: int, d_model: int, num_heads: int, latent: int,
                  causal: bool = True, dtype: str = "bf16", seed: int = 7) -> GatedProblem:
    rng = np.random.default_rng(seed)
    B, S, D, L = batch, seq, d_model, latent
    x = round_to(_normal(rng, (B, S, D)), dtype)
    wq = round_to(_normal(rng, (D, D), 1.0 / np.sqrt(D)), dtype)
    wc = round_to(_normal(rng, (L, D), 1.0 / np.sqrt(D)), dtype)
    wk = round_to(_normal(rng, (D, L), 1.0 / np.sqrt(L)), dtype)
    wv = round_to(_normal(rng, (D, L), 1.0 / np.sqrt(L)), dtype)
    wg = round_to(_normal(rng, (D, D), 1.0 / np.sqrt(D)), dtype)
    wo = round_to(_normal(rng, (D, D), 1.0 / np.sqrt(D)), dtype)
    return GatedProblem(dtype, num_heads, causal, x, wq, wc, wk, wv, wg, wo)


@dataclasses.dataclass
class NotebookProblem:
    """RoPE-less notebook inputs, row-vector convention (y = x @ W)."""

    h: int
    x: np.ndarray      # [1, d_1]
    w_dq: np.ndarray   # [d_1, d_2]
    w_dkv: np.ndarray  # [d_1, d_2]
    w_uq: np.ndarray   # [d_2, d_3]
    w_uk: np.ndarray   # [d_2, d_3]
    w_uv: np.ndarray   # [d_2, d_3]
    w_o: np.ndarray    # [d_3, d_1]
    c_kv: np.ndarray   # [existing, d_2]


def notebook_problem(*, d_1: int = 100, d_2: int = 20, d_3: int = 60, h: int = 3,
                     existing: int = 5, seed: int = 1001) -> NotebookProblem:
    rng = np.random.default_rng(seed)
    x = _normal(rng, (1, d_1))
    w_dq = _normal(rng, (d_1, d_2))
    w_dkv = _normal(rng, (d_1, d_2))
    w_uq = _normal(rng, (d_2, d_3))
    w_uk = _normal(rng, (d_2, d_3))
    w_uv = _normal(rng, (d_2, d_3))
    w_o = _normal(rng, (d_3, d_1))
    c_kv = _normal(rng, (existing, d_2))
    return NotebookProblem(h, x, w_dq, w_dkv, w_uq, w_uk, w_uv, w_o, c_kv)
