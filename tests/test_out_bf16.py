"""The decode's bf16 out_lat (MLA_DECODE_OUT_BF16) and the output projection that reads it
(mla_out_project_bf16), on the tensor-core route: the bf16 result is the fp32 result rounded to
nearest even, bit for bit (same arithmetic, rounded once at the store), for whole blocks and for
blocks split over clusters (combine); the projection of it equals the fp32 route's projection bit for
bit (that route rounds out_lat the same way before its W_UV product); and both meet the oracle."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import inputs as I
from head_latent_attention_08_b200 import mla as M
from oracle import mla_oracle as O

from gpu_helpers import assert_close, dev, host, mla_dims_of

pytestmark = pytest.mark.gpu


def _decode(p, q, cache, cu, flags, out, fp8_scale=None, clusters=0):
    d = mla_dims_of(p)
    tmax = int(p.seqlens.max())
    M.mla_set_decode_clusters(clusters)
    try:
        if fp8_scale is None:
            ws = M.workspace(M.mla_decode_workspace_size(d, torch.bfloat16, p.batch, p.n_q, tmax, cache.shape[0],
                                                         flags), "cuda")
            M.mla_decode_absorbed(d, q, cache, cu, p.batch, p.n_q, tmax, flags, out, None, ws)
        else:
            ws = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, p.batch, p.n_q, tmax, cache.shape[0],
                                                         flags), "cuda")
            M.mla_decode_absorbed_fp8(d, q, cache, fp8_scale, cu, p.batch, p.n_q, tmax, flags, out, None, ws)
        torch.cuda.synchronize()
    finally:
        M.mla_set_decode_clusters(0)
    assert M.mla_check_status() == M.MLA_OK


@pytest.mark.parametrize("clusters", [0, 3])
@pytest.mark.parametrize("cache_kind", ["bf16", "e4m3"])
def test_decode_out_bf16_is_the_rounded_fp32_result(clusters, cache_kind):
    p = I.decode_problem(batch=3, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=256, seqlens=[1500, 90, 2049], n_q=2, dtype="bf16", seed=97,
                         cache_dtype="e4m3" if cache_kind == "e4m3" else "")
    q_abs = O.store_as(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), "bf16")
    q = dev(q_abs, "bf16")
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    scale = 0.25 if cache_kind == "e4m3" else None
    cache = (torch.from_numpy(p.cache).to(torch.float8_e4m3fn).view(torch.uint8).cuda() if scale
             else dev(p.cache, "bf16"))
    nq = p.batch * p.n_q
    out32 = torch.empty(nq, 128, 512, device="cuda")
    out16 = torch.full((nq, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    flags = M.MLA_DECODE_CAUSAL
    _decode(p, q, cache, cu, flags, out32, scale, clusters)
    _decode(p, q, cache, cu, flags | M.MLA_DECODE_OUT_BF16, out16, scale, clusters)
    assert torch.equal(out16, out32.to(torch.bfloat16))
    values = p.cache.astype(np.float64) * (scale if scale else 1.0)
    ref, _ = O.decode_absorbed(q_abs, values, p.cu_seqlens, p.n_q, 512, p.kq_scale, True)
    assert_close(host(out16.float()), ref, "bf16", "out_lat bf16")
    # the projection of the bf16 out_lat equals the fp32 route's projection, bit for bit
    d = mla_dims_of(p)
    w_uv, w_o = dev(p.w_uv, "bf16"), dev(p.w_o, "bf16")
    ws = M.workspace(M.mla_out_project_workspace_size(d, torch.bfloat16, nq), "cuda")
    y32 = torch.empty(nq, p.d_model, dtype=torch.bfloat16, device="cuda")
    y16 = torch.empty_like(y32)
    M.mla_out_project(d, out32, w_uv, w_o, None, nq, y32, ws)
    M.mla_out_project_bf16(d, out16, w_uv, w_o, None, nq, y16, ws)
    torch.cuda.synchronize()
    assert torch.equal(y16, y32)
    assert_close(host(y16.float()), O.out_project(ref, p.w_uv, p.w_o), "bf16", "y")


def test_out_bf16_refused_off_the_tensor_core_route():
    p = I.decode_problem(batch=2, n_heads=16, kv_lora_rank=128, rope_dim=32, qk_nope=64, v_head=64, d_model=64,
                         seqlens=[10, 20], dtype="f32", seed=98)
    d = mla_dims_of(p)
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    out = torch.empty(2, 16, 128, dtype=torch.bfloat16, device="cuda")
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.float32, 2, 1, 20, 30, 0), "cuda")
    with pytest.raises(M.MLAError):
        M.mla_decode_absorbed(d, dev(np.zeros((2, 16, 160))), dev(p.cache), cu, 2, 1, 20, M.MLA_DECODE_OUT_BF16,
                              out, None, ws)
