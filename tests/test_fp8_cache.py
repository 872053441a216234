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
    # q dtype, H, dc, dr, seqlens, n_q, causal
    ("bf16", 128, 512, 64, [1, 63, 300, 1000], 1, True),
    ("bf16", 128, 512, 64, [4, 67, 300], 4, True),
    ("f32", 16, 128, 32, [5, 64, 65, 200], 3, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-H{c[1]}-T{c[4]}-nq{c[5]}-c{int(c[6])}")
def test_decode_absorbed_fp8(case):
    qdt, H, dc, dr, seqlens, n_q, causal = case
    p = I.decode_problem(batch=len(seqlens), n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=64, v_head=64,
                         d_model=64, seqlens=seqlens, n_q=n_q, dtype=qdt, seed=90, cache_dtype="e4m3")
    scale = 0.5
    d = M.dims(H, dc, dr, 64, 64, 64)
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    q_dev = dev(q_abs, qdt)
    q_used = O.store_as(q_abs, qdt)
    codes = torch.from_numpy(p.cache).to(torch.float8_e4m3fn).view(torch.uint8).cuda()
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    nq = p.batch * n_q
    out = torch.empty(nq, H, dc, dtype=torch.float32, device="cuda")
    lse = torch.empty(nq, H, dtype=torch.float32, device="cuda")
    flags = M.MLA_DECODE_CAUSAL if causal else 0
    tmax = int(p.seqlens.max())
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, p.batch, n_q, tmax,
                                                 codes.shape[0], flags), "cuda")
    M.mla_decode_absorbed_fp8(d, q_dev, codes, scale, cu, p.batch, n_q, tmax, flags, out, lse, ws)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    ref, ref_lse = O.decode_absorbed(q_used, p.cache.astype(np.float64) * scale, p.cu_seqlens, n_q, dc,
                                     p.kq_scale, causal)
    assert_close(host(out), ref, "f32", "out_lat")        # fp32 arithmetic over the same e4m3 values
    assert_lse_close(host(lse), ref_lse, "f32", "lse")
