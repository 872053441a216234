"""GPU parity: the CUDA path through the C ABI against the float64 oracle on identical seeded inputs.

Small cases compare every element and span several tiles plus a ragged tail; full-size cases run
the same launch configuration as the benchmark and compare sampled sequences the oracle computes
one by one. Tolerance: max |gpu - ref| <= tol * max |ref|, tol = 1e-4 (fp32), 2e-2 (bf16)."""
import math

import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import mla as M
from head_latent_attention_08_b200 import inputs as I
from oracle import mla_oracle as O
from gpu_helpers import (GpuDecode, TOL, assert_close, assert_lse_close, dev, host, mla_dims_of, oracle_seq,
                         rel_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_08_b200 import build
    build.build()
    M.lib()


# ------------------------------------------------------------------------------------------
# append
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("flags", [0, M.MLA_APPEND_NORM, M.MLA_APPEND_NORM | M.MLA_APPEND_ROPE])
def test_append_latent(dtype, flags):
    p = I.decode_problem(batch=3, n_heads=2, kv_lora_rank=512, rope_dim=64, qk_nope=8, v_head=8,
                         d_model=8, seqlens=[5, 40000, 9], n_q=2, dtype=dtype, seed=21,
                         with_weights=False)
    cache = dev(p.cache, dtype)
    before = cache.clone()
    M.mla_append_latent(mla_dims_of(p), cache, torch.from_numpy(p.row_idx).cuda(), dev(p.c_new),
                        dev(p.kpe_new), torch.from_numpy(p.positions).cuda(), flags)
    torch.cuda.synchronize()
    ref = O.append_latent(p.cache, p.row_idx, p.c_new, p.kpe_new, p.positions,
                          norm=bool(flags & M.MLA_APPEND_NORM), rope=bool(flags & M.MLA_APPEND_ROPE),
                          dtype=dtype)
    got = host(cache)
    untouched = np.setdiff1d(np.arange(p.cache.shape[0]), p.row_idx)
    assert torch.equal(cache[torch.from_numpy(untouched).cuda()], before[torch.from_numpy(untouched).cuda()])
    # fp32: same value up to the last bit of the float32 normalisation; bf16: at most one ulp apart
    tol = 1e-6 if dtype == "f32" else 2.0 ** -7
    np.testing.assert_allclose(got[p.row_idx], ref[p.row_idx], rtol=tol, atol=1e-6)


# ------------------------------------------------------------------------------------------
# absorption and folding
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,H,dc,dr,n,rows", [
    ("f32", 16, 128, 32, 64, 4), ("f32", 3, 20, 0, 20, 1),
    ("bf16", 128, 512, 64, 128, 64), ("bf16", 128, 512, 64, 128, 7), ("bf16", 16, 512, 0, 128, 200)])
def test_absorb_query(dtype, H, dc, dr, n, rows):
    p = I.decode_problem(batch=rows, n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=n, v_head=8,
                         d_model=8, seqlens=[1] * rows, dtype=dtype, seed=22)
    out = torch.empty(rows, H, dc + dr, dtype=dev(p.q_nope, dtype).dtype, device="cuda")
    M.mla_absorb_weights(mla_dims_of(p), M.MLA_ABSORB_QUERY, dev(p.q_nope, dtype),
                         dev(p.q_pe, dtype) if dr else None, dev(p.w_uk, dtype), rows, out)
    torch.cuda.synchronize()
    ref = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    assert_close(host(out), ref, dtype, "q_abs")
    # the rotary tail is copied, bit for bit
    if dr:
        assert np.array_equal(host(out)[..., dc:], p.q_pe.astype(np.float64))


def test_notebook_config_end_to_end():
    """RoPE-less notebook (d_1 100, d_2 20, d_3 60, h 3, 5 cached rows + 1 appended), fp32: fold the
    weights, append X W_dKV, absorb, attend (softmax, scale 1/sqrt(d_h)), project by W_aVO."""
    p = I.notebook_problem()
    h, d_2, d_3, d_1 = p.h, p.w_uq.shape[0], p.w_uq.shape[1], p.x.shape[1]
    d_h = d_3 // h
    uq, uk, uv, wo = O.notebook_split_heads(p.w_uq, p.w_uk, p.w_uv, p.w_o, h)   # layout only
    d = M.dims(h, d_2, 0, d_h, d_h, d_1, 1.0 / math.sqrt(d_h))
    w_aqk = torch.empty(h, d_2, d_2, device="cuda")
    w_avo = torch.empty(h, d_2, d_1, device="cuda")
    M.mla_absorb_weights(d, M.MLA_FOLD_QK, dev(uq), None, dev(uk), d_2, w_aqk)
    M.mla_absorb_weights(d, M.MLA_FOLD_VO, dev(uv), None, dev(wo), d_2, w_avo)
    x = dev(p.x)
    cq = torch.empty(1, d_2, device="cuda")
    cnew = torch.empty(1, d_2, device="cuda")
    M.mla_linear(x, dev(p.w_dq), 1, d_2, d_1, M.MLA_LINEAR_W_KN, cq)
    M.mla_linear(x, dev(p.w_dkv), 1, d_2, d_1, M.MLA_LINEAR_W_KN, cnew)
    cache = torch.zeros(6, d_2, device="cuda")
    cache[:5] = dev(p.c_kv)
    M.mla_append_latent(d, cache, torch.tensor([5], device="cuda"), cnew, None, None, 0)
    q_abs = torch.empty(1, h, d_2, device="cuda")
    d_q = M.dims(h, d_2, 0, d_2, d_h, d_1, 1.0 / math.sqrt(d_h))   # W_aQK acts on the d_2-wide C_Q
    M.mla_absorb_weights(d_q, M.MLA_ABSORB_QUERY, cq.expand(h, d_2).contiguous().reshape(1, h, d_2),
                         None, w_aqk, 1, q_abs)
    out_lat = torch.empty(1, h, d_2, device="cuda")
    cu = torch.tensor([0, 6], dtype=torch.int32, device="cuda")
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.float32, 1, 1, 6, 6, M.MLA_DECODE_CAUSAL), "cuda")
    M.mla_decode_absorbed(d, q_abs, cache, cu, 1, 1, 6, M.MLA_DECODE_CAUSAL, out_lat, None, ws)
    y = torch.empty(1, d_1, device="cuda")
    M.mla_linear(out_lat.reshape(1, h * d_2), w_avo.reshape(h * d_2, d_1), 1, d_1, h * d_2,
                 M.MLA_LINEAR_W_KN, y)
    torch.cuda.synchronize()
    ref = O.notebook_forward(p.x, p.w_dq, p.w_dkv, p.w_uq, p.w_uk, p.w_uv, p.w_o, p.c_kv, h,
                             form="softmax", route="unabsorbed")
    assert tuple(y.shape) == (1, 100) and tuple(w_aqk.shape) == (3, 20, 20) and tuple(w_avo.shape) == (3, 20, 100)
    assert_close(host(w_aqk), ref["W_aQK"], "f32", "W_aQK")
    assert_close(host(w_avo), ref["W_aVO"], "f32", "W_aVO")
    assert_close(host(cache), ref["C_KV"], "f32", "C_KV")
    assert_close(host(q_abs).reshape(h, 1, d_2), ref["C_Q"], "f32", "C_Q")
    assert_close(host(y), ref["output"], "f32", "output")


# ------------------------------------------------------------------------------------------
# decode: small cases, every element
# ------------------------------------------------------------------------------------------

SMALL = [
    # dtype, H, dc, dr, n, dv, D, seqlens, n_q, causal
    ("f32", 16, 128, 32, 64, 64, 96, [1, 77, 300], 1, True),
    ("f32", 3, 20, 0, 20, 20, 12, [6, 2], 2, True),
    ("f32", 16, 128, 32, 64, 64, 96, [4, 37], 4, True),
    ("bf16", 128, 512, 64, 128, 128, 256, [1, 63, 64, 65, 200, 1000], 1, True),
    ("bf16", 128, 512, 64, 128, 128, 256, [4, 5, 64, 67, 300], 4, True),
    ("bf16", 128, 512, 64, 128, 128, 256, [129, 3, 700], 1, False),
    ("bf16", 16, 512, 0, 128, 128, 128, [100, 257], 100, True),
    ("bf16", 16, 512, 0, 128, 128, 128, [9, 40], 9, False),
]


def _check_decode_case(case):
    dtype, H, dc, dr, n, dv, D, seqlens, n_q, causal = case
    p = I.decode_problem(batch=len(seqlens), n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=n,
                         v_head=dv, d_model=D, seqlens=seqlens, n_q=n_q, dtype=dtype, seed=23)
    g = GpuDecode(p, causal=causal, append=True)
    y = host(g.run())
    out_lat, lse = host(g.step.out_lat), host(g.step.lse)
    for b in range(p.batch):
        _, ref_lat, ref_lse, ref_y, ref_cache = oracle_seq(p, b, causal=causal)
        rows = slice(b * n_q, (b + 1) * n_q)
        assert_close(out_lat[rows], ref_lat, dtype, f"out_lat b={b}")
        assert_close(y[rows], ref_y, dtype, f"y b={b}")
        assert_lse_close(lse[rows], ref_lse, dtype, f"lse b={b}")


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}-H{c[1]}-dc{c[2]}-dr{c[3]}-T{c[7]}-nq{c[8]}-c{int(c[9])}")
def test_decode_small(case):
    _check_decode_case(case)


@pytest.mark.parametrize("clusters", [1, 2, 3])
@pytest.mark.parametrize("case", [SMALL[3], SMALL[6]], ids=["dr64-ragged-nq1", "dr0-causal-nq100"])
def test_decode_many_segments_per_cluster(case, clusters):
    """One to three clusters for all the work: every CTA pair crosses many blocks (whole blocks and
    split ones), so each block boundary's query hand-over, epilogue and cache-stage release runs
    many times per CTA, next to the combine of split blocks."""
    M.mla_set_decode_clusters(clusters)
    try:
        _check_decode_case(case)
    finally:
        M.mla_set_decode_clusters(0)


def test_decode_empty_and_zero_length_sequences():
    p = I.decode_problem(batch=3, n_heads=16, kv_lora_rank=128, rope_dim=32, qk_nope=64, v_head=64,
                         d_model=64, seqlens=[1, 1, 1], dtype="f32", seed=24)
    d = mla_dims_of(p)
    cache = dev(p.cache[:2])           # sequence 1 has no rows at all
    cu = torch.tensor([0, 1, 1, 2], dtype=torch.int32, device="cuda")
    q = torch.randn(3, 16, 160, device="cuda")
    out = torch.full((3, 16, 128), 7.0, device="cuda")
    lse = torch.zeros(3, 16, device="cuda")
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.float32, 3, 1, 1, 2, 0), "cuda")
    M.mla_decode_absorbed(d, q, cache, cu, 3, 1, 1, 0, out, lse, ws)
    torch.cuda.synchronize()
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    assert torch.allclose(out[0], cache[0, :128].expand(16, 128))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_does_not_modify_inputs(dtype):
    p = I.decode_problem(batch=2, n_heads=128 if dtype == "bf16" else 16,
                         kv_lora_rank=512 if dtype == "bf16" else 128, rope_dim=64 if dtype == "bf16" else 32,
                         qk_nope=128, v_head=128, d_model=128, seqlens=[70, 130], dtype=dtype, seed=25)
    g = GpuDecode(p, causal=True, append=False)
    snaps = [t.clone() for t in (g.cache, g.q_nope, g.q_pe, g.w_uk, g.w_uv, g.w_o, g.cu)]
    g.run()
    for a, b in zip(snaps, (g.cache, g.q_nope, g.q_pe, g.w_uk, g.w_uv, g.w_o, g.cu)):
        assert torch.equal(a, b)


# ------------------------------------------------------------------------------------------
# the five workloads at full size (sampled sequences)
# ------------------------------------------------------------------------------------------

def test_config2_fp32_full():
    p = I.decode_problem(batch=4, n_heads=16, kv_lora_rank=128, rope_dim=32, qk_nope=64, v_head=64,
                         d_model=1024, seqlens=[1024] * 4, dtype="f32", seed=I.CONFIG_SEEDS[2])
    g = GpuDecode(p)
    y = host(g.run())
    out_lat = host(g.step.out_lat)
    for b in range(4):
        _, ref_lat, _, ref_y, _ = oracle_seq(p, b)
        assert_close(out_lat[b:b + 1], ref_lat, "f32", f"out_lat b={b}")
        assert_close(y[b:b + 1], ref_y, "f32", f"y b={b}")


def test_config3_deepseek_scale_full_sampled():
    p = I.decode_problem(batch=64, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=5120, seqlens=[4096] * 64, dtype="bf16", seed=I.CONFIG_SEEDS[3])
    g = GpuDecode(p)
    y = host(g.run())
    out_lat = host(g.step.out_lat)
    for b in (0, 17, 38, 63):
        _, ref_lat, _, ref_y, _ = oracle_seq(p, b)
        assert_close(out_lat[b:b + 1], ref_lat, "bf16", f"out_lat b={b}")
        assert_close(y[b:b + 1], ref_y, "bf16", f"y b={b}")


@pytest.mark.parametrize("n_q", [1, 4])
def test_config4_ragged_long_context_sampled(n_q):
    seqlens = I.ragged_seqlens(16, 1024, 32768, I.CONFIG_SEEDS[4])
    p = I.decode_problem(batch=16, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=5120, seqlens=seqlens, n_q=n_q, dtype="bf16", seed=I.CONFIG_SEEDS[4])
    g = GpuDecode(p)
    y = host(g.run())
    out_lat = host(g.step.out_lat)
    longest, shortest = int(np.argmax(seqlens)), int(np.argmin(seqlens))
    for b in sorted({longest, shortest, 5}):
        _, ref_lat, _, ref_y, _ = oracle_seq(p, b)
        rows = slice(b * n_q, (b + 1) * n_q)
        assert_close(out_lat[rows], ref_lat, "bf16", f"out_lat b={b}")
        assert_close(y[rows], ref_y, "bf16", f"y b={b}")


@pytest.mark.parametrize("route", ["unabsorbed", "absorbed"])
def test_config5_gated_prefill_full_sampled(route):
    gp = I.gated_problem(batch=4, seq=2048, d_model=2048, num_heads=16, latent=512, causal=True,
                         dtype="bf16", seed=I.CONFIG_SEEDS[5])
    args = [dev(a, "bf16") for a in (gp.x, gp.wq, gp.wc, gp.wk, gp.wv, gp.wg, gp.wo)]
    x_before = args[0].clone()
    r = M.gated_mla(*args, num_heads=16, causal=True, route=route)
    torch.cuda.synchronize()
    assert set(r) == {"output", "latent_cache"}
    assert r["output"].shape == (4, 2048, 2048) and r["output"].dtype == torch.bfloat16
    assert r["latent_cache"].shape == (4, 2048, 512) and r["latent_cache"].dtype == torch.bfloat16
    assert torch.equal(args[0], x_before)
    b = 2
    y_ref, c_ref = O.gated_mla(gp.x[b:b + 1], gp.wq, gp.wc, gp.wk, gp.wv, gp.wg, gp.wo, 16, True)
    assert_close(host(r["latent_cache"][b:b + 1]), c_ref, "bf16", "latent_cache")
    assert_close(host(r["output"][b:b + 1]), y_ref, "bf16", "output")


def test_gated_worked_example_on_gpu():
    one = torch.ones(1, 1, dtype=torch.float32, device="cuda")
    x = torch.full((1, 1, 1), 2.0, device="cuda")
    r = M.gated_mla(x, one, one, one, one, torch.zeros_like(one), one, num_heads=1, causal=True)
    torch.cuda.synchronize()
    assert r["output"].item() == 1.0 and r["latent_cache"].item() == 2.0


@pytest.mark.parametrize("shape,L,H,causal", [((1, 2, 2), 1, 1, True), ((1, 3, 2), 1, 2, False)])
def test_gated_shape_examples_on_gpu(shape, L, H, causal):
    gp = I.gated_problem(batch=shape[0], seq=shape[1], d_model=shape[2], num_heads=H, latent=L,
                         causal=causal, dtype="f32", seed=26)
    r = M.gated_mla(*[dev(a) for a in (gp.x, gp.wq, gp.wc, gp.wk, gp.wv, gp.wg, gp.wo)], num_heads=H,
                    causal=causal)
    torch.cuda.synchronize()
    y_ref, c_ref = O.gated_mla(gp.x, gp.wq, gp.wc, gp.wk, gp.wv, gp.wg, gp.wo, H, causal)
    assert tuple(r["output"].shape) == shape and tuple(r["latent_cache"].shape) == (shape[0], shape[1], L)
    assert_close(host(r["output"]), y_ref, "f32", "output")


@pytest.mark.parametrize("dtype,m,n,k,flags", [
    ("bf16", 7, 128, 64, 0), ("bf16", 300, 256, 192, M.MLA_LINEAR_SIGMOID), ("bf16", 64, 5120, 1024, 0),
    ("bf16", 513, 512, 2048, 0), ("f32", 5, 33, 17, M.MLA_LINEAR_SIGMOID), ("bf16", 3, 40, 24, 0)])
def test_linear(dtype, m, n, k, flags):
    rng = np.random.default_rng(m * 1000 + n)
    x = I.round_to(rng.standard_normal((m, k)).astype(np.float32), dtype)
    w = I.round_to((rng.standard_normal((n, k)) / math.sqrt(k)).astype(np.float32), dtype)
    y = torch.empty(m, n, dtype=dev(x, dtype).dtype, device="cuda")
    M.mla_linear(dev(x, dtype), dev(w, dtype), m, n, k, flags, y)
    torch.cuda.synchronize()
    ref = O.linear(x, w, sigmoid_out=bool(flags & M.MLA_LINEAR_SIGMOID))
    assert_close(host(y), ref, dtype, "linear")


@pytest.mark.parametrize("rows,D", [(64, 5120), (5, 256), (130, 1024)])
def test_out_project_bf16(rows, D):
    H, dc, dv = 128, 512, 128
    rng = np.random.default_rng(rows + D)
    out_lat = rng.standard_normal((rows, H, dc)).astype(np.float32)
    w_uv = I.round_to((rng.standard_normal((H, dv, dc)) / math.sqrt(dc)).astype(np.float32), "bf16")
    w_o = I.round_to((rng.standard_normal((D, H * dv)) / math.sqrt(H * dv)).astype(np.float32), "bf16")
    gate = I.round_to(rng.random((rows, H * dv)).astype(np.float32), "bf16")
    d = M.dims(H, dc, 64, 128, dv, D)
    for g in (None, gate):
        y = torch.empty(rows, D, dtype=torch.bfloat16, device="cuda")
        ws = M.workspace(M.mla_out_project_workspace_size(d, torch.bfloat16, rows), "cuda")
        M.mla_out_project(d, dev(out_lat), dev(w_uv, "bf16"), dev(w_o, "bf16"),
                          None if g is None else dev(g, "bf16"), rows, y, ws)
        torch.cuda.synchronize()
        ref = O.out_project(out_lat, w_uv, w_o, g)
        assert_close(host(y), ref, "bf16", "y")
