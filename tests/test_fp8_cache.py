"""GPU parity of the fp8 (e4m3) latent cache: the append stores the e4m3 code of each row value (the
code is decided in fp32 on both sides; one scale per cache), and the decode over an e4m3 cache with a
bf16 or fp32 query matches the oracle's decode over the same values."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import inputs as I
from head_latent_attention_08_b200 import mla as M
from oracle import mla_oracle as O

from gpu_helpers import FLAGS_APPEND, assert_close, assert_lse_close, dev, host

pytestmark = pytest.mark.gpu


def e4m3_values(cache_u8: torch.Tensor) -> np.ndarray:
    return cache_u8.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("scale", [1.0, 0.03125, 0.37])
@pytest.mark.parametrize("flags", [FLAGS_APPEND, 0], ids=["norm_rope", "plain"])
def test_append_latent_fp8(scale, flags):
    H, dc, dr, N, rows = 4, 512, 64, 37, 100
    rng = np.random.default_rng(11)
    c_new = (3 * rng.standard_normal((N, dc))).astype(np.float32)
    kpe = (3 * rng.standard_normal((N, dr))).astype(np.float32)
    row_idx = rng.permutation(rows)[:N].astype(np.int64)
    positions = rng.integers(0, 30000, size=N).astype(np.int32)
    init = torch.randint(0, 120, (rows, dc + dr), dtype=torch.uint8)      # finite codes
    cache = init.clone().cuda()
    d = M.dims(H, dc, dr, 64, 64, 64)
    M.mla_append_latent_fp8(d, cache, torch.from_numpy(row_idx).cuda(), dev(c_new), dev(kpe),
                            torch.from_numpy(positions).cuda(), flags, cache_scale=scale)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    got = e4m3_values(cache)[row_idx] * scale
    c, k = c_new.astype(np.float64), kpe.astype(np.float64)
    if flags & M.MLA_APPEND_NORM:
        c = O.rms_norm(c)
    if flags & M.MLA_APPEND_ROPE:
        k = O.rope_interleaved(k, positions)
    want = O.store_e4m3(np.concatenate([c, k], -1), scale)
    # the code is decided in fp32 on both sides; the GPU's fp32 norm and rotation may land one fp32
    # unit away from the oracle's rounded float64 value, which can move a value sitting on a rounding
    # boundary by one e4m3 step: such values must be rare and one step apart
    diff = got != want
    assert diff.mean() < 1e-3
    if diff.any():
        step = np.abs(want[diff]) * 2.0 ** -3 + 1e-30
        assert np.all(np.abs(got[diff] - want[diff]) <= step * 1.01 + 2.0 ** -9 * scale)
    untouched = np.setdiff1d(np.arange(rows), row_idx)
    assert torch.equal(cache.cpu()[untouched], init[untouched])


CASES = [
    # q dtype, H, dc, dr, seqlens, n_q, causal. A bf16 query at H 128, d_c 512 runs on the tensor cores
    # (QK^T as e4m3 MMAs against the query split into e4m3 high and low parts, P.C in f16 over the
    # codes converted exactly); the rest on CUDA cores in fp32.
    ("bf16", 128, 512, 64, [1, 63, 300, 1000], 1, True),
    ("bf16", 128, 512, 64, [4, 67, 300], 4, True),
    ("bf16", 128, 512, 0, [5, 256, 257, 900], 2, True),
    ("bf16", 128, 512, 64, [700, 1500], 3, False),
    ("f32", 16, 128, 32, [5, 64, 65, 200], 3, False),
]


def tensor_core_route(qdt, H, dc):
    return qdt == "bf16" and dc == 512


def run_fp8(p, q_dev, codes, scale, causal, clusters=0):
    H, dc, dr, n_q = p.n_heads, p.kv_lora_rank, p.rope_dim, p.n_q
    d = M.dims(H, dc, dr, p.qk_nope, p.v_head, p.d_model)
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    nq = p.batch * n_q
    out = torch.empty(nq, H, dc, dtype=torch.float32, device="cuda")
    lse = torch.empty(nq, H, dtype=torch.float32, device="cuda")
    flags = M.MLA_DECODE_CAUSAL if causal else 0
    tmax = int(p.seqlens.max())
    M.mla_set_decode_clusters(clusters)
    try:
        ws = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, p.batch, n_q, tmax,
                                                     codes.shape[0], flags), "cuda")
        M.mla_decode_absorbed_fp8(d, q_dev, codes, scale, cu, p.batch, n_q, tmax, flags, out, lse, ws)
        torch.cuda.synchronize()
    finally:
        M.mla_set_decode_clusters(0)
    assert M.mla_check_status() == M.MLA_OK
    return host(out), host(lse)


def to_codes(values):
    """e4m3-representable float64 values -> the device byte tensor of their codes."""
    return torch.from_numpy(np.ascontiguousarray(values)).to(torch.float8_e4m3fn).view(torch.uint8).cuda()


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-H{c[1]}-dr{c[3]}-T{c[4]}-nq{c[5]}-c{int(c[6])}")
def test_decode_absorbed_fp8(case):
    qdt, H, dc, dr, seqlens, n_q, causal = case
    p = I.decode_problem(batch=len(seqlens), n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=64, v_head=64,
                         d_model=64, seqlens=seqlens, n_q=n_q, dtype=qdt, seed=90, cache_dtype="e4m3")
    scale = 0.5
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, lse = run_fp8(p, dev(q_abs, qdt), to_codes(p.cache), scale, causal)
    ref, ref_lse = O.decode_absorbed(O.store_as(q_abs, qdt), p.cache.astype(np.float64) * scale, p.cu_seqlens,
                                     n_q, dc, p.kq_scale, causal)
    # the CUDA-core route keeps fp32 arithmetic over the same e4m3 values; the tensor-core route rounds
    # P to f16 and carries the query to about 2^-8: the bf16 rule
    tol = "bf16" if tensor_core_route(qdt, H, dc) else "f32"
    assert_close(out, ref, tol, "out_lat")
    assert_lse_close(lse, ref_lse, tol, "lse")


@pytest.mark.parametrize("clusters", [1, 3])
def test_decode_fp8_split_blocks(clusters):
    """One or three clusters for all blocks: segments cross block boundaries (query reload, staging
    ring across blocks) and split blocks leave partials, scaled by cache_scale, for the combine."""
    p = I.decode_problem(batch=3, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=64, v_head=64,
                         d_model=64, seqlens=[1300, 90, 2049], n_q=2, dtype="bf16", seed=93, cache_dtype="e4m3")
    scale = 0.0625
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    out, lse = run_fp8(p, dev(q_abs, "bf16"), to_codes(p.cache), scale, True, clusters)
    ref, ref_lse = O.decode_absorbed(O.store_as(q_abs, "bf16"), p.cache.astype(np.float64) * scale,
                                     p.cu_seqlens, 2, 512, p.kq_scale, True)
    assert_close(out, ref, "bf16", "out_lat")
    assert_lse_close(lse, ref_lse, "bf16", "lse")


def test_decode_fp8_peaked_and_scaled_queries():
    """Keys planted along some heads' queries (logits 20..100 after kq_scale, at later tiles, so the
    reference maximum moves and the output is rescaled), then every query x16: a nearly one-hot
    softmax, where the two-part query and the e4m3 keys decide the winner."""
    seqlens = [4096, 1500, 700]
    p = I.decode_problem(batch=3, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=64, seqlens=seqlens, dtype="bf16", seed=94, cache_dtype="e4m3")
    q_abs = O.store_as(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), "bf16")
    cache = p.cache.astype(np.float64).copy()
    heads, logits = [0, 17, 64, 127, 99, 33], [20.0, 40.0, 60.0, 80.0, 100.0, 30.0]
    for b in range(p.batch):
        lo, T = int(p.cu_seqlens[b]), int(p.seqlens[b])
        for j, (h, L) in enumerate(zip(heads, logits)):
            t = 128 + (j + 1) * (T - 128) // (len(heads) + 1)
            q = q_abs[b, h]
            cache[lo + t] = (L / p.kq_scale) * q / float(q @ q)
    scale = float(np.max(np.abs(cache))) / 448.0
    stored = O.store_e4m3(cache, scale)          # what the append would have stored (value = code * scale)
    codes = to_codes(stored / scale)
    for mult in (1.0, 16.0):
        q = O.store_as(mult * q_abs, "bf16")
        out, lse = run_fp8(p, dev(q, "bf16"), codes, scale, True)
        ref, ref_lse = O.decode_absorbed(q, stored, p.cu_seqlens, 1, 512, p.kq_scale, True)
        assert_close(out, ref, "bf16", f"out_lat x{mult}")
        assert_lse_close(lse, ref_lse, "bf16", f"lse x{mult}")


def test_decode_fp8_deepseek_scale_sampled():
    """The benchmark's decode shape (64 sequences of 4096 positions, H 128) over an e4m3 cache, in the
    launch configuration the benchmark uses; four sequences checked against the oracle."""
    B, T = 64, 4096
    rng = np.random.default_rng(95)
    vals = torch.from_numpy(rng.standard_normal((B * T, 576)).astype(np.float32)).to(torch.float8_e4m3fn)
    codes = vals.view(torch.uint8).cuda()
    q = O.store_as(rng.standard_normal((B, 128, 576)), "bf16")
    cu = np.arange(0, (B + 1) * T, T)
    scale, kq = 0.25, 1.0 / np.sqrt(192.0)
    d = M.dims(128, 512, 64, 128, 128, 64)
    out = torch.empty(B, 128, 512, device="cuda")
    lse = torch.empty(B, 128, device="cuda")
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, B, 1, T, B * T, M.MLA_DECODE_CAUSAL), "cuda")
    M.mla_decode_absorbed_fp8(d, dev(q, "bf16"), codes, scale, torch.from_numpy(cu.astype(np.int32)).cuda(), B, 1, T,
                              M.MLA_DECODE_CAUSAL, out, lse, ws)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    out, lse = host(out), host(lse)
    for b in (0, 21, 42, 63):
        rows = vals[b * T:(b + 1) * T].float().numpy().astype(np.float64) * scale
        ref, ref_lse = O.decode_absorbed(q[b:b + 1], rows, np.array([0, T]), 1, 512, kq, True)
        assert_close(out[b:b + 1], ref, "bf16", f"out_lat b={b}")
        assert_lse_close(lse[b:b + 1], ref_lse, "bf16", f"lse b={b}")


def test_decode_fp8_empty_and_short_sequences():
    """Tensor-core route over an e4m3 cache with an empty sequence (zeros and -inf lse), a one-position
    sequence and one that ends one position into a second tile (ragged: plan and combine run)."""
    p = I.decode_problem(batch=3, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=64, v_head=64,
                         d_model=64, seqlens=[1, 257, 40], n_q=1, dtype="bf16", seed=96, cache_dtype="e4m3")
    rng = np.random.default_rng(96)
    q_abs = O.store_as(np.concatenate([rng.standard_normal((1, 128, 576)),
                                       O.absorb_query(p.q_nope, p.q_pe, p.w_uk)]), "bf16")
    cu = np.concatenate([[0], p.cu_seqlens]).astype(np.int64)          # sequence 0 holds no positions
    d = M.dims(128, 512, 64, 64, 64, 64)
    out = torch.empty(4, 128, 512, device="cuda")
    lse = torch.empty(4, 128, device="cuda")
    codes = to_codes(p.cache)
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, 4, 1, 257, codes.shape[0], 0), "cuda")
    M.mla_decode_absorbed_fp8(d, dev(q_abs, "bf16"), codes, 2.0, torch.from_numpy(cu.astype(np.int32)).cuda(), 4, 1,
                              257, 0, out, lse, ws)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    out, lse = host(out), host(lse)
    ref, ref_lse = O.decode_absorbed(q_abs, p.cache.astype(np.float64) * 2.0, cu, 1, 512, p.kq_scale, False)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert_close(out, ref, "bf16", "out_lat")
    assert_lse_close(lse, ref_lse, "bf16", "lse")
