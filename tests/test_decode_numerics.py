"""Absorbed decode where its numerics are stressed, on the tensor-core path (H 128, d_c 512, d_r 64,
bf16), against the oracle on identical inputs. Both sides read the same bf16 q_abs and cache, so the
differences are those of the kernel's arithmetic alone:

* peaked attention: for several heads a key is planted along that head's query so that its logit
  (after kq_scale) is 20 to 100, at positions in later tiles: each such row moves its reference
  maximum in the middle of the sequence, and the rescale of the accumulated output runs;
* the same with the blocks split over clusters (partials merged by the combine);
* every query scaled x16 (logits of tens, the softmax nearly one-hot);
* every query scaled x1024: raw scores (before kq_scale) up to about 10^5, beyond the fp16 range.

The rule is max|gpu - ref| <= 2e-2 max|ref| for out_lat and for y = W_O (W_UV out_lat); lse must meet
the same rule and an absolute bound in nats.

Pages: "ferrox-core 0.23.0 src/mla_absorbed.rs", module docs "What it is" (score, softmax,
out_lat, v) and the kq_scale paragraph."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import mla as M
from head_latent_attention_08_b200 import inputs as I
from oracle import mla_oracle as O
from gpu_helpers import assert_close, assert_lse_close, dev, host, mla_dims_of

pytestmark = pytest.mark.gpu

H, DC, DR = 128, 512, 64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_08_b200 import build
    build.build()
    M.lib()
    assert M.mla_check_status() == M.MLA_OK


def _problem(seqlens, seed):
    return I.decode_problem(batch=len(seqlens), n_heads=H, kv_lora_rank=DC, rope_dim=DR, qk_nope=128,
                            v_head=128, d_model=256, seqlens=seqlens, dtype="bf16", seed=seed)


def _bf16(x):
    return O.store_as(x, "bf16")


def _q_abs(p, mult=1.0):
    return _bf16(mult * O.absorb_query(p.q_nope, p.q_pe, p.w_uk))


def _plant(p, q_abs, heads, logits):
    """Cache rows k_j = (L_j / kq_scale) q_abs[b, h_j] / |q_abs[b, h_j]|^2 at positions spread over
    each sequence (past the first tile), so that head h_j scores about L_j there."""
    cache = p.cache.astype(np.float64).copy()
    for b in range(p.batch):
        lo, T = int(p.cu_seqlens[b]), int(p.seqlens[b])
        for j, (h, L) in enumerate(zip(heads, logits)):
            t = 128 + (j + 1) * (T - 128) // (len(heads) + 1)
            q = q_abs[b, h]
            cache[lo + t] = (L / p.kq_scale) * q / float(q @ q)
    return _bf16(cache)


def _run(p, q_abs, cache, clusters=0):
    d = mla_dims_of(p)
    nq = p.batch
    q = dev(q_abs, "bf16")
    c = dev(cache, "bf16")
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    out = torch.empty(nq, H, DC, device="cuda")
    lse = torch.empty(nq, H, device="cuda")
    tmax = int(p.seqlens.max())
    M.mla_set_decode_clusters(clusters)
    try:
        ws = M.workspace(M.mla_decode_workspace_size(d, torch.bfloat16, p.batch, 1, tmax, int(p.cu_seqlens[-1]),
                                                     M.MLA_DECODE_CAUSAL), "cuda")
        M.mla_decode_absorbed(d, q, c, cu, p.batch, 1, tmax, M.MLA_DECODE_CAUSAL, out, lse, ws)
        w_uv, w_o = dev(p.w_uv, "bf16"), dev(p.w_o, "bf16")
        y = torch.empty(nq, p.d_model, dtype=torch.bfloat16, device="cuda")
        wso = M.workspace(M.mla_out_project_workspace_size(d, torch.bfloat16, nq), "cuda")
        M.mla_out_project(d, out, w_uv, w_o, None, nq, y, wso)
        torch.cuda.synchronize()
        assert M.mla_check_status() == M.MLA_OK
    finally:
        M.mla_set_decode_clusters(0)
    return host(out), host(lse), host(y)


def _check(p, q_abs, cache, clusters=0, lse_atol=None):
    out, lse, y = _run(p, q_abs, cache, clusters)
    ref_lat, ref_lse = O.decode_absorbed(q_abs, cache, p.cu_seqlens, 1, DC, p.kq_scale, True)
    ref_y = O.out_project(ref_lat, p.w_uv, p.w_o)
    for b in range(p.batch):
        assert_close(out[b:b + 1], ref_lat[b:b + 1], "bf16", f"out_lat b={b}")
        assert_close(y[b:b + 1], ref_y[b:b + 1], "bf16", f"y b={b}")
    assert_lse_close(lse, ref_lse, "bf16", atol=lse_atol)
    return ref_lat, ref_lse


PLANTED_HEADS = [0, 17, 64, 127, 5, 99, 33, 80]
PLANTED_LOGITS = [20.0, 40.0, 60.0, 80.0, 100.0, 100.0, 30.0, 50.0]


@pytest.mark.parametrize("clusters", [0, 3])
def test_peaked_attention_planted_keys(clusters):
    p = _problem([4096, 1500, 700, 3001], seed=41)
    q_abs = _q_abs(p)
    cache = _plant(p, q_abs, PLANTED_HEADS, PLANTED_LOGITS)
    ref_lat, _ = _check(p, q_abs, cache, clusters)
    # the planted rows dominate their heads: the case is as peaked as intended
    for b in range(p.batch):
        lo, T = int(p.cu_seqlens[b]), int(p.seqlens[b])
        t = 128 + 6 * (T - 128) // (len(PLANTED_HEADS) + 1)        # head 99 (j = 5): logit 100
        np.testing.assert_allclose(ref_lat[b, 99], cache[lo + t, :DC], rtol=1e-6, atol=1e-6)


def test_queries_scaled_by_16():
    p = _problem([4096, 2000, 333], seed=42)
    q_abs = _q_abs(p, 16.0)
    _check(p, q_abs, p.cache)


def test_raw_scores_beyond_fp16_range():
    p = _problem([2048, 777], seed=43)
    q_abs = _q_abs(p, 1024.0)
    raw = max(float(np.max(np.abs(q_abs[b] @ p.cache[int(p.cu_seqlens[b]):int(p.cu_seqlens[b + 1])].T)))
              for b in range(p.batch))
    assert raw > 65504.0
    # logits of thousands: lse is checked against the rule and to 1e-4 of its size (fp32 scores)
    _, ref_lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, 1, DC, p.kq_scale, True)
    _check(p, q_abs, p.cache, lse_atol=1e-4 * float(np.max(np.abs(ref_lse))))
