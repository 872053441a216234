"""Plain CPU oracle for absorbed Multi-head Latent Attention (MLA) decode.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute this module:
only the test suite, the smoke check of ``__graft_entry__`` and the CPU-baseline leg of the
benchmark use it. It shares no code with the CUDA library and never imports it.

Every function is a direct restatement, in float64 numpy, of what the pages define. A library
matmul (``@`` / ``einsum``) serves as a step where the definition is a matrix product; there is no
blocking, fusion or reordering beyond the definitions. Storing into a bf16 cache rounds once,
round-to-nearest-even, through torch's CPU cast.

Sources (cited by page title and section):

* [nb]  "MLA_RoPE-less.ipynb" (gist notebook), its single code cell: head splitting, matrix
        absorption, cache update, attention part, value part, the adding trick.
* [rs]  "ferrox-core 0.23.0 src/mla_absorbed.rs": the module docs ("What it is": the score,
        out_lat and v formulas and the kq_scale paragraph), the doc comment and body of
        ``causal_mla_absorbed_attention``, and the unit test
        ``absorbed_equals_naive_for_the_same_kv_b``.
* [lab] "Lab 01 - Ejercicio matematico de MLA" (lynx-cortex): Bloque A (KV-cache size per
        token, steps 1-4), Bloque B (the matmul identity), Bloque C (parameter counts).
* [gm]  "Gated MLA" (tensortonic, Kimi K3 step 2 of 11): the problem equations, Examples,
        Hints, Requirements.
* [fm]  "preacher-1/MLA_tutorial formula.md", Part 3: the training-form equation and the
        inference-form equation (the latent is the value, queries absorb W_kc).

Pins (what fixes each function independently of this file; see tests/test_oracle_pins.py):

* absorb_query / decode_absorbed / value_project: equal to decode_unabsorbed (the plain,
  un-absorbed definition); equal to torch's scaled_dot_product_attention in float64 as a
  multi-query attention; closed forms at T = 1 (output = c_0) and zero query (output = mean of
  the rows); the [rs] test's wrong-scale check; invariances (score shift, permutation).
* append_latent: exact row placement; RMS of a normed row is 1; RoPE keeps pair norms and
  composes as a rotation by the position difference.
* fold_qk / fold_vo / notebook_forward: the printed notebook shapes; absorbed == unabsorbed;
  the linear form against the notebook's cell restated with torch matmuls; the softmax form
  against torch scaled_dot_product_attention (its default scale, 1/sqrt(head width)) on
  explicit per-head Q, K, V, at the notebook's sizes and at sizes where d_2 != d_h.
* rope_interleaved: relativity and composition, and hand-computed angles (tests/golden/
  rope_frequencies.json: pair i of a d-wide row at position p turns by p * theta^(-2i/d)).
* gated_mla: the worked example (output 1.0, latent_cache 2.0) and the shape examples; causal
  first query equals the first value row; gated_mla_absorbed equals gated_mla.
* kv_values_per_token_*: the worked table of [lab] Bloque A, filled by hand in the tests.
* out_project / linear: equal to torch.nn.functional.linear in float64.
* project_inputs: with absorb_query and the append's rotation, its scores equal those of [fm]
  Part 3's training-form equation (per-head keys c_i W_kc^(s) and x_i W_kr R_i, rotations built
  as explicit block-diagonal matrices in torch), at sizes where d = d_c' = d_c so that feeding the
  wrong latent to a weight still runs.
* store_e4m3: hand-worked e4m3 roundings (tests/golden/e4m3_rounding.json: ties to even at several
  binades, subnormals, saturation), and a planted round-toward-zero must fail them.
No function here is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np
import torch

F64 = np.float64


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=F64)


def store_e4m3(x: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """Value an fp8 (e4m3) latent-cache element stands for, as float64: the e4m3 value nearest to
    fp32(x) / scale (an fp32 division; ties to the even code), saturated at +-448, times scale.

    The pages fix no fp8 format (the lab's "<5 GB at 128k" needs at most one byte per value); the
    reading taken is E4M3 as published for 8-bit floating point (bias 7, 3 mantissa bits, no
    infinities, largest finite value 448) with one scale per cache. The code is decided in fp32,
    the precision the append kernel decides it in; torch's cast serves as the rounding step.
    """
    v = _f64(x).astype(np.float32) / np.float32(scale)
    v = np.clip(v, -448.0, 448.0).astype(np.float32)
    code = torch.from_numpy(np.ascontiguousarray(v)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    return code * float(scale)


def store_as(x: np.ndarray, dtype: str) -> np.ndarray:
    """Value a tensor holds after being stored in ``dtype`` ('f32' or 'bf16'), as float64."""
    x = _f64(x)
    if dtype == "f64":
        return x
    if dtype == "f32":
        return x.astype(np.float32).astype(F64)
    if dtype == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------------------------
# append step (latent cache update)
# --------------------------------------------------------------------------------------------

def rms_norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Row-wise RMS normalisation with unit weight: x / sqrt(mean(x^2) + eps).

    [rs] module docs: the cached compressed KV is "RMS-normed"; no weight or eps is printed, so
    unit weight and eps = 1e-6 are the reading taken.
    """
    x = _f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_interleaved(x: np.ndarray, positions: np.ndarray, theta: float = 10000.0) -> np.ndarray:
    """Rotary embedding R_i of [fm] (inference form, k = [c, x W_kr R_i]).

    The pages name the rotation R_i but print no convention; the reading taken is the RoFormer
    interleaved form: the pair (2i, 2i+1) of a d-wide row at position p turns by the angle
    p * theta^(-2i/d).
    """
    x = _f64(x)
    d = x.shape[-1]
    if d % 2:
        raise ValueError("rotary width must be even")
    pos = _f64(positions).reshape(-1, 1)
    i = np.arange(d // 2, dtype=F64)
    ang = pos * theta ** (-2.0 * i / d)
    cos, sin = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


def append_latent(cache: np.ndarray, row_idx: np.ndarray, c_new: np.ndarray, kpe_new: np.ndarray,
                  positions: np.ndarray, *, norm: bool, rope: bool, eps: float = 1e-6,
                  theta: float = 10000.0, dtype: str = "f32") -> np.ndarray:
    """Return a copy of ``cache`` with row ``row_idx[k]`` = concat(c_new[k], kpe_new[k]).

    [nb] "update cache": the new latent is stacked onto the cache BEFORE attention runs, so the
    query attends to itself. [rs] fn docs: a cache row is the normed compressed KV followed by
    the roped k_pe (concat(kv_cmpr, k_pe) order). The row is computed in float64 and stored in
    the cache dtype.
    """
    out = _f64(cache).copy()
    c = _f64(c_new)
    k = _f64(kpe_new)
    if norm:
        c = rms_norm(c, eps)
    if rope and k.shape[-1] > 0:
        k = rope_interleaved(k, positions, theta)
    rows = np.concatenate([c, k], axis=-1)
    out[np.asarray(row_idx, dtype=np.int64)] = store_as(rows, dtype)
    return out


# --------------------------------------------------------------------------------------------
# query absorption and weight folding
# --------------------------------------------------------------------------------------------

def absorb_query(q_nope: np.ndarray, q_pe: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """q_abs[t, h] = concat(W_UK[h]^T q_nope[t, h], q_pe[t, h]).

    [rs] module docs: the query is pushed into the latent, q_nope_absorbed[h] = wk_b[h] . q_nope[h]
    (kv_lora_rank wide), and the absorbed query is followed by the roped q_pe. [lab] Bloque B:
    q^T W_UK c = (W_UK^T q)^T c. W_UK is [H, qk_nope, kv_lora_rank] (the k rows of kv_b).
    """
    q_nope, q_pe, w_uk = _f64(q_nope), _f64(q_pe), _f64(w_uk)
    q_lat = np.einsum("thi,hij->thj", q_nope, w_uk)
    return np.concatenate([q_lat, q_pe], axis=-1)


def fold_qk(w_uq_heads: np.ndarray, w_uk_heads: np.ndarray) -> np.ndarray:
    """W_aQK[h] = W_uQ[h] @ W_uK[h]^T, each head [d_2, d_h] -> [d_2, d_2].   [nb] matrix absorption."""
    a, b = _f64(w_uq_heads), _f64(w_uk_heads)
    return a @ np.transpose(b, (0, 2, 1))


def fold_vo(w_uv_heads: np.ndarray, w_o_heads: np.ndarray) -> np.ndarray:
    """W_aVO[h] = W_uV[h] @ W_O[h], [d_2, d_h] @ [d_h, d_1] -> [d_2, d_1].   [nb] matrix absorption."""
    return _f64(w_uv_heads) @ _f64(w_o_heads)


# --------------------------------------------------------------------------------------------
# attention over the latent cache
# --------------------------------------------------------------------------------------------

def attended_count(T: int, n_q: int, j: int, causal: bool) -> int:
    """How many cache positions query j (of the n_q newest tokens of a T-long sequence) sees.

    The query tokens are the last n_q positions (they were appended before attention, [nb]
    "update cache"); under the causal mask query j sits at position T - n_q + j and sees
    positions 0 .. T - n_q + j ([gm]: the mask removes later positions). Without the mask it
    sees all T.
    """
    return (T - n_q + j + 1) if causal else T


def softmax_attend(scores: np.ndarray, values: np.ndarray):
    """softmax over the last axis, then the weighted sum of ``values`` rows.

    [rs] fn body: subtract the row max, exponentiate, sum, divide only when the sum is positive
    (an empty row gives a zero output). Returns (output, lse) with lse = max + log(sum).
    """
    if scores.shape[-1] == 0:
        out = np.zeros(scores.shape[:-1] + (values.shape[-1],), dtype=F64)
        return out, np.full(scores.shape[:-1], -np.inf)
    m = np.max(scores, axis=-1, keepdims=True)
    e = np.exp(scores - m)
    z = np.sum(e, axis=-1, keepdims=True)
    p = np.where(z > 0, e / np.where(z > 0, z, 1.0), e)
    return p @ values, (m + np.log(z))[..., 0]


def decode_absorbed(q_abs: np.ndarray, cache: np.ndarray, cu_seqlens: np.ndarray, n_q: int,
                    kv_lora_rank: int, scale: float, causal: bool = True):
    """Absorbed attention of every query over its sequence's latent cache.

    [rs] module docs and fn: score[h][t] = (q_abs[h] . c[t] + q_pe[h] . k_pe[t]) * kq_scale,
    out_lat[h] = sum_t softmax(score[h])[t] * c[t] (kv_lora_rank wide, before wv_b). One cache row
    is the shared key of every head and its first kv_lora_rank entries are the shared value
    ([fm] inference form: the value is c_i). Query row b*n_q + j belongs to sequence b.

    q_abs [N_q, H, d_c + d_r], cache [sum T_b, d_c + d_r] -> out_lat [N_q, H, d_c], lse [N_q, H].
    """
    q_abs, cache = _f64(q_abs), _f64(cache)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    n_seq = cu.shape[0] - 1
    NQ, H, W = q_abs.shape
    out = np.zeros((NQ, H, kv_lora_rank))
    lse = np.full((NQ, H), -np.inf)
    for b in range(n_seq):
        K = cache[cu[b]:cu[b + 1]]
        T = K.shape[0]
        for j in range(n_q):
            r = b * n_q + j
            cnt = attended_count(T, n_q, j, causal)
            s = (q_abs[r] @ K[:cnt].T) * scale               # [H, cnt]
            out[r], lse[r] = softmax_attend(s, K[:cnt, :kv_lora_rank])
    return out, lse


def value_project(out_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """v[t, h] = W_UV[h] out_lat[t, h].   [rs] module docs: v[h] = wv_b[h] . out_lat[h]."""
    return np.einsum("hij,thj->thi", _f64(w_uv), _f64(out_lat))


def decode_unabsorbed(q_nope: np.ndarray, q_pe: np.ndarray, cache: np.ndarray,
                      cu_seqlens: np.ndarray, n_q: int, w_uk: np.ndarray, w_uv: np.ndarray,
                      scale: float, causal: bool = True) -> np.ndarray:
    """The plain (naive) MLA definition: expand every position into per-head K and V.

    [rs] unit test: k_h[t] = concat(W_UK[h] c_t, k_pe_t) and v_h[t] = W_UV[h] c_t, then per-head
    softmax attention with the naive head width's scale. [fm] training form: o^(s) is the
    softmax-weighted sum of v^(s) with k^(s) = [c W_kc, x W_kr R] (k_pe shared by every head).
    Returns v [N_q, H, d_v] (heads not yet concatenated or projected by W_O).
    """
    q_nope, q_pe, cache = _f64(q_nope), _f64(q_pe), _f64(cache)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    H, n, dc = w_uk.shape
    dv = w_uv.shape[1]
    NQ = q_nope.shape[0]
    out = np.zeros((NQ, H, dv))
    for b in range(cu.shape[0] - 1):
        rows = cache[cu[b]:cu[b + 1]]
        T = rows.shape[0]
        c, kpe = rows[:, :dc], rows[:, dc:]
        for h in range(H):
            k_h = np.concatenate([c @ w_uk[h].T, kpe], axis=-1)   # [T, n + d_r]
            v_h = c @ w_uv[h].T                                    # [T, d_v]
            for j in range(n_q):
                r = b * n_q + j
                cnt = attended_count(T, n_q, j, causal)
                q = np.concatenate([q_nope[r, h], q_pe[r, h]])
                s = (k_h[:cnt] @ q) * scale
                out[r, h], _ = softmax_attend(s[None, :], v_h[:cnt])
    return out


def out_project(out_lat: np.ndarray, w_uv: np.ndarray, w_o: np.ndarray,
                gate: np.ndarray | None = None) -> np.ndarray:
    """y[t] = W_O concat_h(gate[t] * v[t, h]) with v = W_UV out_lat.

    [fm] inference form: o_t = [o^(1) W_v^(1), ..., o^(h) W_v^(h)] then the output projection;
    [nb] "adding trick": sum over heads of out_h W_O[h] is the same product. [gm]: the optional
    channel gate multiplies the concatenated head contexts before W_o.
    """
    v = value_project(out_lat, w_uv)
    flat = v.reshape(v.shape[0], -1)
    if gate is not None:
        flat = flat * _f64(gate)
    return flat @ _f64(w_o).T


def sigmoid(x: np.ndarray) -> np.ndarray:
    x = _f64(x)
    return 1.0 / (1.0 + np.exp(-x))


def linear(x: np.ndarray, w: np.ndarray, *, sigmoid_out: bool = False) -> np.ndarray:
    """Y = X W^T (PyTorch Linear convention, W = [out, in]).   [gm] problem equations."""
    y = _f64(x) @ _f64(w).T
    return sigmoid(y) if sigmoid_out else y


# --------------------------------------------------------------------------------------------
# input projections: the low-rank query chain and the KV down-projection
# --------------------------------------------------------------------------------------------

def project_inputs(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta: float = 10000.0):
    """The parts of [fm] Part 3's inference-form equation computed from the hidden states x_i.

    In the page's row-vector notation (x [N, d]; W'_c [d, d_c']; W_qc [H, d_c', d_k];
    W_qr [H, d_c', d_r]; W_c [d, d_c]; W_kr [d, d_r]):

      c'_i        = x_i W'_c                      (the query latent, d_c' = 1536 on the page)
      q_nope[i,s] = c'_i W_qc^(s)                 (absorbed afterwards by W_kc^(s)^T: absorb_query)
      q_pe[i,s]   = c'_i W_qr^(s) R_i             (rotated at the token's position)
      c_i         = x_i W_c                       (the latent, i.e. the cached key and value)
      k_r[i]      = x_i W_kr                      (one rotary key shared by all heads, made from
                                                   x_i and not from c_i: the page's note on the
                                                   second term of k says so)

    Returns (q_nope [N, H, d_k], q_pe [N, H, d_r], c [N, d_c], k_r [N, d_r]). k_r is returned
    before its rotation R_i and c before any normalisation: both belong to the cache append
    (append_latent), which writes the row concat(c_i, k_r[i] R_i).
    """
    x = _f64(x)
    c_q = x @ _f64(w_cq)
    q_nope = np.einsum("nq,hqk->nhk", c_q, _f64(w_qc))
    q_r = np.einsum("nq,hqr->hnr", c_q, _f64(w_qr))          # heads first: one rotation per token
    q_pe = rope_interleaved(q_r, positions, theta).transpose(1, 0, 2)
    c = x @ _f64(w_c)
    k_r = x @ _f64(w_kr)
    return q_nope, q_pe, c, k_r


# --------------------------------------------------------------------------------------------
# the RoPE-less notebook
# --------------------------------------------------------------------------------------------

def notebook_split_heads(w_uq, w_uk, w_uv, w_o, h: int):
    """[nb] head splitting: (d_2, d_3) -> (h, d_2, d_h); W_O (d_3, d_1) -> (h, d_h, d_1)."""
    d_2, d_3 = np.shape(w_uq)
    d_h = d_3 // h

    def split(w):
        return _f64(w).reshape(d_2, h, d_h).transpose(1, 0, 2)

    return split(w_uq), split(w_uk), split(w_uv), _f64(w_o).reshape(h, d_h, -1)


def notebook_kq_scale(d_h: int) -> float:
    """Score scale of the notebook's softmax form: 1/sqrt(d_h), d_h = d_3 / h the width of one
    un-absorbed head ([rs] kq_scale paragraph: the scale of the naive head width, kept after the
    absorption widens the dot product)."""
    return 1.0 / math.sqrt(d_h)


def notebook_attention_weights(s: np.ndarray, scale: float, form: str) -> np.ndarray:
    """Attention weights of the notebook step over the last axis of the raw scores ``s``.

    ``form='linear'``: the notebook literally, attn = C_Q C_KV^T with no softmax and no scale.
    ``form='softmax'``: softmax of the scaled scores (scale inside the exponent, row max
    subtracted first, [rs] fn body).
    """
    if form == "linear":
        return s
    m = np.max(s * scale, axis=-1, keepdims=True)
    e = np.exp(s * scale - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def notebook_forward(x, w_dq, w_dkv, w_uq, w_uk, w_uv, w_o, c_kv, h: int, *,
                     form: str = "softmax", route: str = "absorbed"):
    """One decode step of the notebook's RoPE-less MLA (row-vector convention, y = x W).

    [nb]: split heads, absorb W_aQK = W_uQ W_uK^T and W_aVO = W_uV W_O, append new_CV = X W_dKV
    to C_KV, C_Q = X W_dQ W_aQK, attn = C_Q C_KV^T, out = attn (C_KV W_aVO), summed over heads.

    ``form='linear'`` is the notebook literally (no softmax, no scale). ``form='softmax'`` applies
    the method's softmax with scale 1/sqrt(d_h) (the un-absorbed head width, [rs] kq_scale
    paragraph), which the pages' other definitions ([rs], [gm]) use. ``route='unabsorbed'``
    computes the same result with explicit per-head Q, K, V. Returns a dict of every printed
    quantity: C_Q, C_KV, W_aQK, W_aVO and the output.
    """
    uq, uk, uv, o = notebook_split_heads(w_uq, w_uk, w_uv, w_o, h)
    d_h = uq.shape[2]
    w_aqk = fold_qk(uq, uk)
    w_avo = fold_vo(uv, o)
    x = _f64(x)
    new_cv = x @ _f64(w_dkv)
    ckv = np.vstack((_f64(c_kv), new_cv))
    cq_lat = x @ _f64(w_dq)                                  # [1, d_2]
    scale = notebook_kq_scale(d_h)

    def weights(s):
        return notebook_attention_weights(s, scale, form)

    if route == "absorbed":
        c_q = cq_lat @ w_aqk                                 # [h, 1, d_2]
        attn = weights(c_q @ ckv.T)                          # [h, 1, T]
        out_heads = attn @ (ckv @ w_avo)                     # [h, 1, d_1]
    elif route == "unabsorbed":
        q = cq_lat @ uq                                      # [h, 1, d_h]
        k = ckv @ uk                                         # [h, T, d_h]
        v = ckv @ uv                                         # [h, T, d_h]
        attn = weights(q @ np.transpose(k, (0, 2, 1)))
        out_heads = (attn @ v) @ o                           # [h, 1, d_1]
        c_q = cq_lat @ w_aqk
    else:
        raise ValueError(route)
    return {"C_Q": c_q, "C_KV": ckv, "W_aQK": w_aqk, "W_aVO": w_avo,
            "output": out_heads.sum(axis=0)}


# --------------------------------------------------------------------------------------------
# gated MLA (causal prefill, no positional encoding)
# --------------------------------------------------------------------------------------------

def gated_mla(x, wq, wc, wk, wv, wg, wo, num_heads: int, causal: bool):
    """[gm] problem equations, literally: Q = X Wq^T, C = X Wc^T, K = C Wk^T, V = C Wv^T; split into
    H heads of width D_h (channel h*D_h + d, Hint 1); A = softmax(Q K^T / sqrt(D_h) + M) with M
    removing later positions when causal (Hint 2); concatenate head contexts (Hint 3);
    Y = [sigmoid(X Wg^T) * O] Wo^T. Returns (output [B,S,D], latent_cache [B,S,L])."""
    x = _f64(x)
    B, S, D = x.shape
    H = num_heads
    if D % H:
        raise ValueError("model width must be divisible by the head count")
    Dh = D // H
    Q = x @ _f64(wq).T
    C = x @ _f64(wc).T
    K = C @ _f64(wk).T
    V = C @ _f64(wv).T

    def heads(t):
        return t.reshape(B, S, H, Dh).transpose(0, 2, 1, 3)   # [B, H, S, Dh]

    Qh, Kh, Vh = heads(Q), heads(K), heads(V)
    s = Qh @ Kh.transpose(0, 1, 3, 2) / math.sqrt(Dh)
    if causal:
        mask = np.triu(np.ones((S, S), dtype=bool), k=1)     # above the main diagonal
        s = np.where(mask, -np.inf, s)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    A = e / np.sum(e, axis=-1, keepdims=True)
    O = (A @ Vh).transpose(0, 2, 1, 3).reshape(B, S, D)
    Y = (sigmoid(x @ _f64(wg).T) * O) @ _f64(wo).T
    return Y, C


def gated_mla_absorbed(x, wq, wc, wk, wv, wg, wo, num_heads: int, causal: bool):
    """The same gated MLA computed through the absorbed route: per head q_abs = Wk_h^T q_h
    ([lab] Bloque B identity with W_UK = Wk_h, the rows h*D_h .. of Wk), attention over the latent
    C (value = C, [fm] inference form), then Wv_h lifts the latent output ([rs] v = wv_b out_lat)."""
    x = _f64(x)
    B, S, D = x.shape
    H = num_heads
    Dh = D // H
    Q = x @ _f64(wq).T
    C = x @ _f64(wc).T
    L = C.shape[-1]
    w_uk = _f64(wk).reshape(H, Dh, L)
    w_uv = _f64(wv).reshape(H, Dh, L)
    gate = sigmoid(x @ _f64(wg).T)
    Y = np.zeros((B, S, D))
    for b in range(B):
        q_abs = absorb_query(Q[b].reshape(S, H, Dh), np.zeros((S, H, 0)), w_uk)
        cu = np.array([0, S])
        out_lat, _ = decode_absorbed(q_abs, C[b], cu, S, L, 1.0 / math.sqrt(Dh), causal)
        Y[b] = out_project(out_lat, w_uv, _f64(wo), gate=gate[b])
    return Y, C


# --------------------------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------------------------

def kv_values_per_token_mha(n_layers: int, n_heads: int, d_head: int) -> int:
    """[lab] Bloque A step 1: standard MHA caches K and V per layer and head: 2 L H d_head values."""
    return 2 * n_layers * n_heads * d_head


def kv_values_per_token_mla(n_layers: int, d_c: int, d_rope: int = 0) -> int:
    """[lab] Bloque A steps 2-3: MLA caches c_t (d_c) plus the decoupled k^rope (d_h^R) per layer."""
    return n_layers * (d_c + d_rope)


def kv_ratio(n_heads: int, d_head: int, d_c: int, d_rope: int) -> float:
    """[lab] Bloque A step 4: M_MHA / M_MLA = 2 H d_head / (d_c + d_h^R) (L cancels)."""
    return 2.0 * n_heads * d_head / float(d_c + d_rope)
