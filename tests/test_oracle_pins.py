"""Pins of the CPU oracle to things other than itself: printed values and shapes from the pages,
closed forms, special cases that reduce to a library routine (torch SDPA / F.linear in float64),
invariances, and brute force on tiny inputs. The last block plants plausible mistakes in the
oracle (on the CPU) and checks that a pin catches each one."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import mla_oracle as O
from head_latent_attention_08_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def t64(x):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float64)))


# ------------------------------------------------------------------------------------------
# library-routine references (torch, float64)
# ------------------------------------------------------------------------------------------

def sdpa_mqa(q_abs, cache, cu, n_q, d_c, scale, causal):
    """Multi-query attention via torch SDPA: every head shares key = cache row, value = c part."""
    q_abs = t64(q_abs)
    cache = t64(cache)
    NQ, H, W = q_abs.shape
    out = torch.zeros(NQ, H, d_c, dtype=torch.float64)
    for b in range(len(cu) - 1):
        K = cache[cu[b]:cu[b + 1]]
        T = K.shape[0]
        q = q_abs[b * n_q:(b + 1) * n_q].permute(1, 0, 2)            # [H, n_q, W]
        k = K.unsqueeze(0).expand(H, T, W)
        v = K[:, :d_c].unsqueeze(0).expand(H, T, d_c)
        if causal and n_q == T:
            o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
        elif causal:
            # each query token j sees the prefix ending at its own position (T - n_q + j):
            # attend with SDPA on that prefix alone
            o = torch.cat([F.scaled_dot_product_attention(q[:, j:j + 1], k[:, :T - n_q + j + 1],
                                                          v[:, :T - n_q + j + 1], scale=scale)
                           for j in range(n_q)], dim=1)
        else:
            o = F.scaled_dot_product_attention(q, k, v, scale=scale)
        out[b * n_q:(b + 1) * n_q] = o.permute(1, 0, 2)
    return out.numpy()


def sdpa_unabsorbed(q_nope, q_pe, cache, cu, n_q, w_uk, w_uv, scale):
    """Plain MHA via SDPA over explicitly expanded per-head K and V (non-causal, one seq block)."""
    H, n, dc = w_uk.shape
    outs = []
    for b in range(len(cu) - 1):
        rows = t64(cache[cu[b]:cu[b + 1]])
        c, kpe = rows[:, :dc], rows[:, dc:]
        K = torch.stack([torch.cat([F.linear(c, t64(w_uk[h])), kpe], -1) for h in range(H)])
        V = torch.stack([F.linear(c, t64(w_uv[h])) for h in range(H)])
        q = torch.cat([t64(q_nope[b * n_q:(b + 1) * n_q]), t64(q_pe[b * n_q:(b + 1) * n_q])], -1)
        o = F.scaled_dot_product_attention(q.permute(1, 0, 2), K, V, scale=scale)
        outs.append(o.permute(1, 0, 2))
    return torch.cat(outs).numpy()


def rel_err(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def small_problem(seed=7, batch=3, H=4, dc=16, dr=8, n=8, dv=8, D=24, seqlens=(5, 9, 13), n_q=1):
    return I.decode_problem(batch=batch, n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=n,
                            v_head=dv, d_model=D, seqlens=list(seqlens), n_q=n_q, dtype="f32",
                            seed=seed)


# ------------------------------------------------------------------------------------------
# printed values and shapes
# ------------------------------------------------------------------------------------------

def test_notebook_printed_shapes(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "notebook_shapes.json")))
    d = g["dims"]
    p = I.notebook_problem(d_1=d["d_1"], d_2=d["d_2"], d_3=d["d_3"], h=d["h"],
                           existing=d["existing_cache"])
    r = O.notebook_forward(p.x, p.w_dq, p.w_dkv, p.w_uq, p.w_uk, p.w_uv, p.w_o, p.c_kv, p.h,
                           form="linear")
    s = g["shapes"]
    assert list(p.x.shape) == s["input"]
    assert list(r["C_Q"].shape) == s["latent_query"]
    assert list(r["C_KV"].shape) == s["latent_kv_cache"]
    assert list(r["W_aQK"].shape) == s["absorbed_qk_kernel"]
    assert list(r["W_aVO"].shape) == s["absorbed_vo_kernel"]
    assert list(r["output"].shape) == s["final_output"]


@pytest.mark.parametrize("form", ["linear", "softmax"])
def test_notebook_absorbed_equals_unabsorbed(form):
    p = I.notebook_problem()
    args = (p.x, p.w_dq, p.w_dkv, p.w_uq, p.w_uk, p.w_uv, p.w_o, p.c_kv, p.h)
    a = O.notebook_forward(*args, form=form, route="absorbed")["output"]
    b = O.notebook_forward(*args, form=form, route="unabsorbed")["output"]
    assert rel_err(a, b) < 1e-12


def test_notebook_linear_form_literal_with_torch():
    # the notebook's cell, restated with torch float64 matmuls in its own operand order
    p = I.notebook_problem()
    h, d_2, d_3 = p.h, p.w_uq.shape[0], p.w_uq.shape[1]
    d_h = d_3 // h
    uq = t64(p.w_uq).reshape(d_2, h, d_h).permute(1, 0, 2)
    uk = t64(p.w_uk).reshape(d_2, h, d_h).permute(1, 0, 2)
    uv = t64(p.w_uv).reshape(d_2, h, d_h).permute(1, 0, 2)
    wo = t64(p.w_o).reshape(h, d_h, -1)
    X = t64(p.x)
    ckv = torch.cat([t64(p.c_kv), X @ t64(p.w_dkv)])
    out = ((X @ t64(p.w_dq) @ torch.bmm(uq, uk.transpose(1, 2))) @ ckv.T
           @ (ckv @ torch.bmm(uv, wo))).sum(0)
    r = O.notebook_forward(p.x, p.w_dq, p.w_dkv, p.w_uq, p.w_uk, p.w_uv, p.w_o, p.c_kv, p.h,
                           form="linear")["output"]
    assert rel_err(r, out.numpy()) < 1e-12


def sdpa_notebook_softmax(p):
    """The notebook step with the method's softmax, built from explicit per-head Q, K, V with torch
    (row-vector convention) and attended by scaled_dot_product_attention at its default scale,
    1/sqrt(q.shape[-1]) = 1/sqrt(d_h); heads are summed after W_O[h] ([nb] adding trick)."""
    h, d_2, d_3 = p.h, p.w_uq.shape[0], p.w_uq.shape[1]
    d_h = d_3 // h
    X = t64(p.x)
    ckv = torch.cat([t64(p.c_kv), X @ t64(p.w_dkv)])
    out = torch.zeros(1, p.w_o.shape[1], dtype=torch.float64)
    for k in range(h):
        cols = slice(k * d_h, (k + 1) * d_h)
        q = X @ t64(p.w_dq) @ t64(p.w_uq)[:, cols]                # [1, d_h]
        K = ckv @ t64(p.w_uk)[:, cols]                            # [T, d_h]
        V = ckv @ t64(p.w_uv)[:, cols]
        o = F.scaled_dot_product_attention(q[None], K[None], V[None])[0]
        out += o @ t64(p.w_o)[cols, :]
    return out.numpy()


NOTEBOOK_SIZES = [dict(), dict(d_1=30, d_2=12, d_3=24, h=3, existing=4, seed=77)]


def _notebook_softmax_pin_passes():
    for kw in NOTEBOOK_SIZES:
        p = I.notebook_problem(**kw)
        ref = sdpa_notebook_softmax(p)
        for route in ("absorbed", "unabsorbed"):
            r = O.notebook_forward(p.x, p.w_dq, p.w_dkv, p.w_uq, p.w_uk, p.w_uv, p.w_o, p.c_kv, p.h,
                                   form="softmax", route=route)["output"]
            if not rel_err(r, ref) < 1e-12:
                return False
    return True


def test_notebook_softmax_form_matches_torch_sdpa():
    # the second size has d_2 = 12 != d_h = 8, so a scale taken from the latent width would differ
    assert _notebook_softmax_pin_passes()


def test_planted_notebook_scale_from_latent_width(monkeypatch):
    # 1/sqrt(d_2) instead of 1/sqrt(d_h): identical at the notebook's own sizes (d_2 = d_h = 20),
    # caught at the second size
    monkeypatch.setattr(O, "notebook_kq_scale", lambda d_h: 1.0 / math.sqrt(12.0 if d_h == 8 else d_h))
    assert not _notebook_softmax_pin_passes()


def test_planted_notebook_scale_after_softmax(monkeypatch):
    def bad(s, scale, form):
        e = np.exp(s - np.max(s, axis=-1, keepdims=True))
        return scale * e / np.sum(e, axis=-1, keepdims=True)
    monkeypatch.setattr(O, "notebook_attention_weights", bad)
    assert not _notebook_softmax_pin_passes()


def _rope_golden_passes(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "rope_frequencies.json")))
    for case in g["cases"]:
        d = case["d"]
        for i, ang in case["angles"].items():
            i = int(i)
            e = np.zeros((1, d))
            e[0, 2 * i] = 1.0                      # unit vector on the first entry of pair i
            r = O.rope_interleaved(e, [case["position"]], case["theta"])[0]
            want = np.zeros(d)
            want[2 * i], want[2 * i + 1] = math.cos(ang), math.sin(ang)
            if not np.allclose(r, want, rtol=0, atol=1e-12):
                return False
    return True


def test_rope_frequencies_golden(golden_dir):
    assert _rope_golden_passes(golden_dir)


def test_planted_rope_frequency_exponent(monkeypatch, golden_dir):
    # theta^(-i/d) instead of theta^(-2i/d): relativity, composition and "pair 0 turns by p" all
    # still hold, the hand-computed angles do not
    def bad(x, positions, theta=10000.0):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        ang = np.asarray(positions, np.float64).reshape(-1, 1) * theta ** (-np.arange(d // 2) / d)
        out = np.empty_like(x)
        out[..., 0::2] = x[..., 0::2] * np.cos(ang) - x[..., 1::2] * np.sin(ang)
        out[..., 1::2] = x[..., 0::2] * np.sin(ang) + x[..., 1::2] * np.cos(ang)
        return out
    monkeypatch.setattr(O, "rope_interleaved", bad)
    assert not _rope_golden_passes(golden_dir)


def test_gated_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "gated_examples.json")))["worked_example"]
    for fn in (O.gated_mla, O.gated_mla_absorbed):
        y, c = fn(np.array(g["hidden_states"]), np.array(g["query_projection"]),
                  np.array(g["latent_down_projection"]), np.array(g["key_up_projection"]),
                  np.array(g["value_up_projection"]), np.array(g["output_gate_projection"]),
                  np.array(g["output_projection"]), g["num_heads"], g["causal"])
        assert y.tolist() == g["output"]
        assert c.tolist() == g["latent_cache"]


def test_gated_shape_examples(golden_dir):
    for ex in json.load(open(os.path.join(golden_dir, "gated_examples.json")))["shape_examples"]:
        B, S, D = ex["hidden_shape"]
        L = ex["latent"]
        p = I.gated_problem(batch=B, seq=S, d_model=D, num_heads=ex["num_heads"], latent=L,
                            causal=ex["causal"], dtype="f32", seed=3)
        y, c = O.gated_mla(p.x, p.wq, p.wc, p.wk, p.wv, p.wg, p.wo, ex["num_heads"], ex["causal"])
        assert list(y.shape) == ex["output_shape"]
        assert list(c.shape) == ex["latent_cache_shape"]
        y2, c2 = O.gated_mla_absorbed(p.x, p.wq, p.wc, p.wk, p.wv, p.wg, p.wo, ex["num_heads"],
                                      ex["causal"])
        assert rel_err(y2, y) < 1e-12 and np.array_equal(c, c2)


def test_kv_cache_closed_forms(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "kv_cache_table.json")))
    for row in g["rows"]:
        mha = O.kv_values_per_token_mha(row["L"], row["H"], row["d_head"])
        mla = O.kv_values_per_token_mla(row["L"], row["d_c"], row["d_r"])
        assert mha == row["mha"] and mla == row["mla"]
        assert Fraction(mha, mla) == Fraction(row["ratio"])
        assert math.isclose(O.kv_ratio(row["H"], row["d_head"], row["d_c"], row["d_r"]),
                            float(Fraction(row["ratio"])), rel_tol=1e-15)
    # forgetting the decoupled rope term gives the over-optimistic ratio the lab warns about
    assert O.kv_ratio(128, 128, 512, 0) == 64.0


# ------------------------------------------------------------------------------------------
# decode: library routine, un-absorbed definition, closed forms, invariances
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("n_q,causal", [(1, False), (1, True), (3, True), (3, False)])
def test_decode_absorbed_matches_sdpa(n_q, causal):
    p = small_problem(n_q=n_q)
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, n_q, p.kv_lora_rank, p.kq_scale,
                                 causal)
    ref = sdpa_mqa(q_abs, p.cache, p.cu_seqlens, n_q, p.kv_lora_rank, p.kq_scale, causal)
    assert rel_err(out, ref) < 1e-13


def test_decode_prefill_causal_matches_sdpa_is_causal():
    p = small_problem(batch=1, seqlens=(11,), n_q=11)
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, _ = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 11, p.kv_lora_rank, p.kq_scale, True)
    ref = sdpa_mqa(q_abs, p.cache, p.cu_seqlens, 11, p.kv_lora_rank, p.kq_scale, True)
    assert rel_err(out, ref) < 1e-13
    # the first query sees only its own row: its output is that row's latent, exactly
    np.testing.assert_array_equal(out[0], np.broadcast_to(p.cache[0, :p.kv_lora_rank], out[0].shape))


def test_absorbed_equals_unabsorbed_definition():
    p = small_problem(n_q=2)
    for causal in (True, False):
        q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
        out_lat, _ = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 2, p.kv_lora_rank,
                                       p.kq_scale, causal)
        v_abs = O.value_project(out_lat, p.w_uv)
        v_naive = O.decode_unabsorbed(p.q_nope, p.q_pe, p.cache, p.cu_seqlens, 2, p.w_uk, p.w_uv,
                                      p.kq_scale, causal)
        assert rel_err(v_abs, v_naive) < 1e-12


def test_unabsorbed_matches_sdpa_mha():
    p = small_problem(n_q=2)
    v_naive = O.decode_unabsorbed(p.q_nope, p.q_pe, p.cache, p.cu_seqlens, 2, p.w_uk, p.w_uv,
                                  p.kq_scale, causal=False)
    ref = sdpa_unabsorbed(p.q_nope, p.q_pe, p.cache, p.cu_seqlens, 2, p.w_uk, p.w_uv, p.kq_scale)
    assert rel_err(v_naive, ref) < 1e-13


def _xorshift_uniform(n, state=0x9E37):
    """Uniform values in [-0.5, 0.5) from a 32-bit xorshift (shifts 13, 17, 5), the generator
    the ferrox-core unit test draws from."""
    out = np.empty(n)
    s = state
    for i in range(n):
        s ^= (s << 13) & 0xFFFFFFFF
        s ^= s >> 17
        s ^= (s << 5) & 0xFFFFFFFF
        out[i] = s / 4294967295.0 - 0.5
    return out


def test_ferrox_unit_test_shapes_absorbed_equals_naive_and_scale_matters():
    # ferrox-core mla_absorbed.rs, unit test absorbed_equals_naive_for_the_same_kv_b: shapes
    # (heads 3, nope 4, rope 2, v 5, kv_lora 6, seq 7); absorbed == naive within 1e-5; the
    # latent-width scale 1/sqrt(kv_lora + rope) gives a different result somewhere (> 1e-4).
    H, nope, rope, dv, dc, T = 3, 4, 2, 5, 6, 7
    vals = _xorshift_uniform(H * (nope + dv) * dc + T * (dc + rope) + H * (nope + rope))
    o = 0
    kv_b = vals[o:o + H * (nope + dv) * dc].reshape(H, nope + dv, dc); o += H * (nope + dv) * dc
    latent = vals[o:o + T * (dc + rope)].reshape(T, dc + rope); o += T * (dc + rope)
    q = vals[o:].reshape(1, H, nope + rope)
    w_uk, w_uv = kv_b[:, :nope], kv_b[:, nope:]
    cu = np.array([0, T])
    scale = 1.0 / math.sqrt(nope + rope)
    q_abs = O.absorb_query(q[..., :nope], q[..., nope:], w_uk)
    out_lat, _ = O.decode_absorbed(q_abs, latent, cu, 1, dc, scale, causal=False)
    absorbed = O.value_project(out_lat, w_uv)
    naive = O.decode_unabsorbed(q[..., :nope], q[..., nope:], latent, cu, 1, w_uk, w_uv, scale,
                                causal=False)
    assert np.max(np.abs(absorbed - naive)) < 1e-5
    wrong, _ = O.decode_absorbed(q_abs, latent, cu, 1, dc, 1.0 / math.sqrt(dc + rope), causal=False)
    assert np.any(np.abs(wrong - out_lat) > 1e-4)


def test_single_position_returns_that_row():
    p = small_problem(batch=2, seqlens=(1, 1))
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, p.kv_lora_rank, p.kq_scale)
    for b in range(2):
        np.testing.assert_array_equal(out[b], np.broadcast_to(p.cache[b, :p.kv_lora_rank],
                                                               out[b].shape))
        np.testing.assert_allclose(lse[b], (q_abs[b] @ p.cache[b]) * p.kq_scale, rtol=1e-14)


def test_zero_query_gives_mean_of_rows():
    p = small_problem()
    q_abs = np.zeros((p.batch, p.n_heads, p.width))
    out, lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, p.kv_lora_rank, p.kq_scale,
                                 causal=False)
    for b in range(p.batch):
        rows = p.cache[p.cu_seqlens[b]:p.cu_seqlens[b + 1], :p.kv_lora_rank].astype(np.float64)
        np.testing.assert_allclose(out[b], np.broadcast_to(rows.mean(0), out[b].shape), rtol=1e-13,
                                   atol=1e-15)
        np.testing.assert_allclose(lse[b], math.log(p.seqlens[b]), rtol=1e-14)


def test_empty_context_gives_zero_and_minus_inf():
    q_abs = np.ones((1, 2, 5))
    out, lse = O.decode_absorbed(q_abs, np.zeros((0, 5)), np.array([0, 0]), 1, 3, 0.5, causal=False)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_score_shift_invariance():
    # an extra rotary column with k_pe = 1 on every row and q_pe = 7 shifts every score of a head
    # by the same constant: the softmax output must not move
    p = small_problem()
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, p.kv_lora_rank, 0.3, False)
    q2 = np.concatenate([q_abs, np.full(q_abs.shape[:2] + (1,), 7.0)], -1)
    c2 = np.concatenate([p.cache, np.ones((p.cache.shape[0], 1))], -1)
    out2, lse2 = O.decode_absorbed(q2, c2, p.cu_seqlens, 1, p.kv_lora_rank, 0.3, False)
    assert rel_err(out2, out) < 1e-13
    np.testing.assert_allclose(lse2, lse + 0.3 * 7.0, rtol=1e-13)


def test_permutation_invariance_without_mask():
    p = small_problem(batch=1, seqlens=(17,))
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, _ = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, p.kv_lora_rank, p.kq_scale, False)
    perm = np.random.default_rng(0).permutation(17)
    out2, _ = O.decode_absorbed(q_abs, p.cache[perm], p.cu_seqlens, 1, p.kv_lora_rank,
                                p.kq_scale, False)
    assert rel_err(out2, out) < 1e-13


def test_split_combine_invariance():
    # softmax over a union of chunks equals the LSE-weighted merge of per-chunk softmaxes
    p = small_problem(batch=1, seqlens=(23,))
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    full, full_lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, p.kv_lora_rank,
                                       p.kq_scale, False)
    parts = []
    for lo, hi in [(0, 6), (6, 7), (7, 23)]:
        o, l = O.decode_absorbed(q_abs, p.cache[lo:hi], np.array([0, hi - lo]), 1,
                                 p.kv_lora_rank, p.kq_scale, False)
        parts.append((o, l))
    L = np.stack([l for _, l in parts])
    m = L.max(0)
    w = np.exp(L - m)
    merged = sum(w[i][..., None] * parts[i][0] for i in range(3)) / w.sum(0)[..., None]
    assert rel_err(merged, full) < 1e-13
    np.testing.assert_allclose(m + np.log(w.sum(0)), full_lse, rtol=1e-14)


def test_brute_force_tiny_pure_python():
    # two heads, three positions, width 3 (d_c 2, d_r 1): every step written out as scalar loops
    p = small_problem(batch=1, H=2, dc=2, dr=1, n=2, dv=2, D=4, seqlens=(3,))
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, _ = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, 2, 0.7, causal=False)
    for h in range(2):
        qa = [sum(float(p.w_uk[h][i][j]) * float(p.q_nope[0][h][i]) for i in range(2))
              for j in range(2)] + [float(p.q_pe[0][h][0])]
        s = [0.7 * sum(qa[d] * float(p.cache[t][d]) for d in range(3)) for t in range(3)]
        e = [math.exp(x - max(s)) for x in s]
        z = sum(e)
        for d in range(2):
            ref = sum(e[t] / z * float(p.cache[t][d]) for t in range(3))
            assert abs(out[0][h][d] - ref) < 1e-14


# ------------------------------------------------------------------------------------------
# append, projections, gated MLA against library routines
# ------------------------------------------------------------------------------------------

def test_append_places_rows_and_norm_rope_properties():
    rng = np.random.default_rng(5)
    cache = rng.standard_normal((10, 12))
    c_new = rng.standard_normal((3, 8)) * 3.0
    kpe = rng.standard_normal((3, 4))
    rows = np.array([9, 0, 4])
    pos = np.array([100, 0, 7])
    out = O.append_latent(cache, rows, c_new, kpe, pos, norm=False, rope=False, dtype="f64")
    untouched = [i for i in range(10) if i not in rows]
    np.testing.assert_array_equal(out[untouched], cache[untouched])
    np.testing.assert_array_equal(out[rows], np.concatenate([c_new, kpe], -1))
    out = O.append_latent(cache, rows, c_new, kpe, pos, norm=True, rope=True, dtype="f64")
    rms = np.sqrt(np.mean(out[rows, :8] ** 2, -1))
    np.testing.assert_allclose(rms, 1.0, rtol=1e-6)
    # rotation keeps every pair's norm; position 0 is the identity
    r = out[rows, 8:]
    np.testing.assert_allclose(r[:, 0::2] ** 2 + r[:, 1::2] ** 2, kpe[:, 0::2] ** 2 + kpe[:, 1::2] ** 2,
                               rtol=1e-13)
    np.testing.assert_allclose(r[1], kpe[1], rtol=0, atol=0)


def test_rope_is_relative():
    # <R_a q, R_b k> depends only on a - b, and R_a R_b = R_(a+b)
    rng = np.random.default_rng(6)
    q, k = rng.standard_normal((1, 16)), rng.standard_normal((1, 16))
    d1 = float(O.rope_interleaved(q, [9])[0] @ O.rope_interleaved(k, [4])[0])
    d2 = float(O.rope_interleaved(q, [25])[0] @ O.rope_interleaved(k, [20])[0])
    assert abs(d1 - d2) < 1e-12
    ab = O.rope_interleaved(O.rope_interleaved(q, [3]), [11])
    np.testing.assert_allclose(ab, O.rope_interleaved(q, [14]), rtol=1e-12, atol=1e-13)
    # first pair turns by exactly the position (theta^0 = 1)
    e0 = np.zeros((1, 4)); e0[0, 0] = 1.0
    np.testing.assert_allclose(O.rope_interleaved(e0, [0.5])[0, :2], [math.cos(0.5), math.sin(0.5)])


def test_store_bf16_is_round_to_nearest_even():
    # 1 + 2^-8 is half way between bf16 neighbours 1 and 1 + 2^-7: ties go to the even mantissa
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9])
    np.testing.assert_array_equal(O.store_as(x, "bf16"), [1.0, 1.0 + 2.0 ** -6, 1.0])


def test_out_project_and_linear_match_torch():
    p = small_problem(n_q=2)
    rng = np.random.default_rng(9)
    out_lat = rng.standard_normal((p.batch * 2, p.n_heads, p.kv_lora_rank))
    gate = rng.random((p.batch * 2, p.n_heads * p.v_head))
    y = O.out_project(out_lat, p.w_uv, p.w_o, gate)
    v = torch.einsum("hij,thj->thi", t64(p.w_uv), t64(out_lat)).reshape(p.batch * 2, -1)
    ref = F.linear(v * t64(gate), t64(p.w_o))
    assert rel_err(y, ref.numpy()) < 1e-13
    x = rng.standard_normal((5, 7))
    w = rng.standard_normal((3, 7))
    assert rel_err(O.linear(x, w), F.linear(t64(x), t64(w)).numpy()) < 1e-14
    assert rel_err(O.linear(x, w, sigmoid_out=True),
                   torch.sigmoid(F.linear(t64(x), t64(w))).numpy()) < 1e-14


@pytest.mark.parametrize("causal", [True, False])
def test_gated_mla_matches_torch_sdpa(causal):
    p = I.gated_problem(batch=2, seq=9, d_model=12, num_heads=3, latent=5, causal=causal,
                        dtype="f32", seed=11)
    y, c = O.gated_mla(p.x, p.wq, p.wc, p.wk, p.wv, p.wg, p.wo, 3, causal)
    X = t64(p.x)
    C = F.linear(X, t64(p.wc))
    Q, K, V = F.linear(X, t64(p.wq)), F.linear(C, t64(p.wk)), F.linear(C, t64(p.wv))

    def heads(t):
        return t.reshape(2, 9, 3, 4).transpose(1, 2)

    o = F.scaled_dot_product_attention(heads(Q), heads(K), heads(V), is_causal=causal)
    o = o.transpose(1, 2).reshape(2, 9, 12)
    ref = F.linear(torch.sigmoid(F.linear(X, t64(p.wg))) * o, t64(p.wo))
    assert rel_err(y, ref.numpy()) < 1e-13
    assert rel_err(c, C.numpy()) < 1e-15
    y2, _ = O.gated_mla_absorbed(p.x, p.wq, p.wc, p.wk, p.wv, p.wg, p.wo, 3, causal)
    assert rel_err(y2, y) < 1e-12


# ------------------------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# ------------------------------------------------------------------------------------------

def _decode_pins_pass():
    try:
        for n_q, causal in [(1, False), (3, True)]:
            test_decode_absorbed_matches_sdpa(n_q, causal)
        test_absorbed_equals_unabsorbed_definition()
        test_ferrox_unit_test_shapes_absorbed_equals_naive_and_scale_matters()
    except AssertionError:
        return False
    return True


def test_pins_pass_unmodified():
    assert _decode_pins_pass()


def test_planted_dropped_rope_term(monkeypatch):
    orig = O.absorb_query
    monkeypatch.setattr(O, "absorb_query", lambda qn, qp, w: np.concatenate(
        [orig(qn, qp, w)[..., :w.shape[2]], np.zeros(np.shape(qp))], -1))
    assert not _decode_pins_pass()


def test_planted_wrong_head_index(monkeypatch):
    orig = O.absorb_query
    monkeypatch.setattr(O, "absorb_query", lambda qn, qp, w: orig(qn, qp, np.asarray(w)[::-1]))
    assert not _decode_pins_pass()


def test_planted_causal_off_by_one(monkeypatch):
    monkeypatch.setattr(O, "attended_count", lambda T, n_q, j, causal: (T - n_q + j) if causal else T)
    assert not _decode_pins_pass()


def test_planted_softmax_missing_normalisation(monkeypatch):
    # a softmax that forgets to divide by the sum
    def bad(scores, values):
        m = np.max(scores, axis=-1, keepdims=True)
        e = np.exp(scores - m)
        return e @ values, (m + np.log(np.sum(e, -1, keepdims=True)))[..., 0]
    monkeypatch.setattr(O, "softmax_attend", bad)
    assert not _decode_pins_pass()


# ------------------------------------------------------------------------------------------
# input projections: the inference form ("formula.md", Part 3) against its training form
# ------------------------------------------------------------------------------------------

# the first size has d = d_c' = d_c, so a latent handed to the wrong weight still runs (and must be
# caught by value, not by a shape error); the second has every width different
PROJ_SIZES = [
    dict(N=5, d=16, dcq=16, dc=16, H=3, dk=8, dr=6, positions=[3, 17, 0, 250, 9], seed=31),
    dict(N=4, d=20, dcq=12, dc=10, H=2, dk=6, dr=4, positions=[1, 2, 40, 7], seed=32),
]


def rotation_matrix(p, d, theta=10000.0):
    """R_p as an explicit d x d block-diagonal matrix acting on row vectors (x R_p): the pair
    (2i, 2i+1) turns by p * theta^(-2i/d), the angles fixed by tests/golden/rope_frequencies.json."""
    R = torch.zeros(d, d, dtype=torch.float64)
    for i in range(d // 2):
        a = p * theta ** (-2.0 * i / d)
        R[2 * i, 2 * i], R[2 * i, 2 * i + 1] = math.cos(a), math.sin(a)
        R[2 * i + 1, 2 * i], R[2 * i + 1, 2 * i + 1] = -math.sin(a), math.cos(a)
    return R


def projection_case(sz):
    rng = np.random.default_rng(sz["seed"])
    N, d, dcq, dc, H, dk, dr = (sz[k] for k in ("N", "d", "dcq", "dc", "H", "dk", "dr"))
    return dict(x=rng.standard_normal((N, d)), w_cq=rng.standard_normal((d, dcq)),
                w_qc=rng.standard_normal((H, dcq, dk)), w_qr=rng.standard_normal((H, dcq, dr)),
                w_c=rng.standard_normal((d, dc)), w_kr=rng.standard_normal((d, dr)),
                w_kc=rng.standard_normal((H, dc, dk)), positions=np.asarray(sz["positions"]))


def training_form_scores(c):
    """Scores q_t^(s) . k_i^(s) of the training-form equation, head by head, in torch:
    q^(s) = [c' W_qc^(s), c' W_qr^(s) R_t], k^(s) = [c W_kc^(s), x W_kr R_i], c' = x W'_c, c = x W_c."""
    X = t64(c["x"])
    cq, lat = X @ t64(c["w_cq"]), X @ t64(c["w_c"])
    pos = [int(p) for p in c["positions"]]
    dr = c["w_kr"].shape[1]
    k_rot = torch.stack([X[i] @ t64(c["w_kr"]) @ rotation_matrix(p, dr) for i, p in enumerate(pos)])
    out = []
    for s in range(c["w_qc"].shape[0]):
        q_n = cq @ t64(c["w_qc"][s])
        q_r = torch.stack([cq[t] @ t64(c["w_qr"][s]) @ rotation_matrix(p, dr) for t, p in enumerate(pos)])
        out.append(q_n @ (lat @ t64(c["w_kc"][s])).T + q_r @ k_rot.T)
    return torch.stack(out).numpy()                       # [H, N (query), N (key)]


def inference_form_scores(c):
    """The same scores through the oracle: project_inputs, the append (rotation of k_r), then the
    absorbed query q_abs[t, s] = [q_nope W_kc^(s)^T, q_pe] against the cache row [c, k_r R]."""
    q_nope, q_pe, lat, k_r = O.project_inputs(c["x"], c["w_cq"], c["w_qc"], c["w_qr"], c["w_c"],
                                              c["w_kr"], c["positions"])
    N = lat.shape[0]
    rows = O.append_latent(np.zeros((N, lat.shape[1] + k_r.shape[1])), np.arange(N), lat, k_r,
                           c["positions"], norm=False, rope=True, dtype="f64")
    q_abs = O.absorb_query(q_nope, q_pe, np.transpose(c["w_kc"], (0, 2, 1)))
    return np.einsum("ths,is->hti", q_abs, rows)


def _projection_pin_passes():
    for sz in PROJ_SIZES:
        c = projection_case(sz)
        want = training_form_scores(c)
        got = inference_form_scores(c)
        if not np.allclose(got, want, rtol=1e-11, atol=1e-11 * np.max(np.abs(want))):
            return False
    return True


def test_project_inputs_matches_training_form():
    assert _projection_pin_passes()


def _plant_projection(monkeypatch, fn):
    monkeypatch.setattr(O, "project_inputs", fn)


def test_planted_rotary_key_from_latent(monkeypatch):
    # k_r = c W_kr instead of x W_kr (runs at the first size, where d_c = d)
    orig = O.project_inputs

    def bad(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta=10000.0):
        q_nope, q_pe, lat, _ = orig(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta)
        return q_nope, q_pe, lat, lat @ np.asarray(w_kr)
    _plant_projection(monkeypatch, bad)
    assert not _projection_pin_passes()


def test_planted_latent_from_query_latent(monkeypatch):
    # c = c' W_c instead of x W_c (runs at the first size, where d_c' = d)
    orig = O.project_inputs

    def bad(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta=10000.0):
        q_nope, q_pe, _, k_r = orig(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta)
        return q_nope, q_pe, (np.asarray(x) @ np.asarray(w_cq)) @ np.asarray(w_c), k_r
    _plant_projection(monkeypatch, bad)
    assert not _projection_pin_passes()


def test_planted_query_from_hidden_state(monkeypatch):
    # q_nope = x W_qc, skipping the query latent (runs at the first size, where d = d_c')
    orig = O.project_inputs

    def bad(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta=10000.0):
        _, q_pe, lat, k_r = orig(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta)
        return np.einsum("nq,hqk->nhk", np.asarray(x), np.asarray(w_qc)), q_pe, lat, k_r
    _plant_projection(monkeypatch, bad)
    assert not _projection_pin_passes()


def test_planted_unrotated_query(monkeypatch):
    orig = O.project_inputs

    def bad(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta=10000.0):
        q_nope, _, lat, k_r = orig(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta)
        c_q = np.asarray(x) @ np.asarray(w_cq)
        return q_nope, np.einsum("nq,hqr->nhr", c_q, np.asarray(w_qr)), lat, k_r
    _plant_projection(monkeypatch, bad)
    assert not _projection_pin_passes()


def test_planted_query_rotated_one_position_late(monkeypatch):
    orig = O.project_inputs

    def bad(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta=10000.0):
        return orig(x, w_cq, w_qc, w_qr, w_c, w_kr, np.asarray(positions) + 1, theta)[:2] + \
            orig(x, w_cq, w_qc, w_qr, w_c, w_kr, positions, theta)[2:]
    _plant_projection(monkeypatch, bad)
    assert not _projection_pin_passes()


# ------------------------------------------------------------------------------------------
# fp8 (e4m3) cache values
# ------------------------------------------------------------------------------------------

def _e4m3_golden_passes(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "e4m3_rounding.json")))
    for x, want, _ in g["cases"]:
        if O.store_e4m3(np.array([x]))[0] != want:
            return False
    for x, scale, want, _ in g["scaled_cases"]:
        if O.store_e4m3(np.array([x]), scale)[0] != want:
            return False
    return True


def test_e4m3_rounding_golden(golden_dir):
    assert _e4m3_golden_passes(golden_dir)


def test_planted_e4m3_round_toward_zero(monkeypatch, golden_dir):
    # every finite e4m3 magnitude, then the largest one not above |x| (truncation instead of nearest)
    mags = sorted({m * 2.0 ** -9 for m in range(8)} |
                  {(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if (e, m) != (15, 7)})

    def bad(x, scale=1.0):
        v = np.asarray(x, np.float64) / scale
        out = np.array([math.copysign(max(m for m in mags if m <= min(abs(t), 448.0)), t) for t in v.ravel()])
        return out.reshape(v.shape) * scale
    monkeypatch.setattr(O, "store_e4m3", bad)
    assert not _e4m3_golden_passes(golden_dir)
