"""Failure detection without a GPU fault: every device-side wait of the tensor-core kernels is bounded
by a global-timer limit. A wait that runs out sets MLA_ERR_TIMEOUT in the status word, its kernel
abandons its work after its own copies and MMAs in flight have ended, and the context stays usable.
The deterministic case waits on a barrier nothing completes; the decode case cuts the limit to 1 ns,
so whichever of its waits is not already satisfied gives up, and the next call must be correct."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import mla as M
from head_latent_attention_08_b200 import inputs as I
from oracle import mla_oracle as O
from gpu_helpers import assert_close, dev, host, mla_dims_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_08_b200 import build
    build.build()
    M.lib()


def _small_decode_is_correct():
    p = I.decode_problem(batch=2, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=128, seqlens=[200, 65], dtype="bf16", seed=33)
    d = mla_dims_of(p)
    q_abs = dev(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), "bf16")
    cache = dev(p.cache, "bf16")
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    out = torch.empty(2, 128, 512, device="cuda")
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.bfloat16, 2, 1, 200, cache.shape[0], 1), "cuda")
    M.mla_decode_absorbed(d, q_abs, cache, cu, 2, 1, 200, M.MLA_DECODE_CAUSAL, out, None, ws)
    assert M.mla_check_status() == M.MLA_OK
    ref, _ = O.decode_absorbed(O.store_as(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), "bf16"), p.cache,
                               p.cu_seqlens, 1, 512, p.kq_scale, True)
    assert_close(host(out), ref, "bf16", "out_lat")


def test_wait_on_a_barrier_nothing_completes_runs_out():
    assert M.mla_check_status() == M.MLA_OK
    limit_ns = 2_000_000
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        M.mla_set_wait_limit(limit_ns)
        ev0.record()
        M.mla_wait_selftest()
        ev1.record()
        torch.cuda.synchronize()
    finally:
        M.mla_set_wait_limit(0)
    assert M.mla_check_status() == M.MLA_ERR_TIMEOUT
    assert M.mla_check_status() == M.MLA_OK          # reading the status clears it
    ms = ev0.elapsed_time(ev1)
    assert limit_ns * 1e-6 <= ms < 1000.0, ms         # it waited its limit, and no longer than bounded
    _small_decode_is_correct()


def test_negative_wait_limit_is_rejected():
    with pytest.raises(M.MLAError):
        M.mla_set_wait_limit(-1)


def test_decode_with_a_tiny_wait_limit_abandons_cleanly():
    p = I.decode_problem(batch=4, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=128, seqlens=[300, 65, 1000, 7], dtype="bf16", seed=31)
    d = mla_dims_of(p)
    q_abs = dev(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), "bf16")
    cache = dev(p.cache, "bf16")
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    out = torch.empty(4, 128, 512, device="cuda")
    ws = M.workspace(M.mla_decode_workspace_size(d, torch.bfloat16, 4, 1, 1000, cache.shape[0], 1), "cuda")
    assert M.mla_check_status() == M.MLA_OK
    try:
        M.mla_set_wait_limit(1)
        M.mla_decode_absorbed(d, q_abs, cache, cu, 4, 1, 1000, M.MLA_DECODE_CAUSAL, out, None, ws)
        torch.cuda.synchronize()
        # every wait that was not satisfied at its first poll gives up; the status says whether any did
        status = M.mla_check_status()
    finally:
        M.mla_set_wait_limit(0)
    assert status in (M.MLA_OK, M.MLA_ERR_TIMEOUT)
    print(f"decode with a 1 ns wait limit: status {status}")
    # the status word was cleared by the read, the context is usable and the result correct again
    M.mla_decode_absorbed(d, q_abs, cache, cu, 4, 1, 1000, M.MLA_DECODE_CAUSAL, out, None, ws)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    ref, _ = O.decode_absorbed(O.store_as(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), "bf16"), p.cache,
                               p.cu_seqlens, 1, 512, p.kq_scale, True)
    assert_close(host(out), ref, "bf16", "out_lat after recovery")


def test_out_of_range_append_row_is_skipped_and_reported():
    p = I.decode_problem(batch=1, n_heads=2, kv_lora_rank=16, rope_dim=8, qk_nope=8, v_head=8, d_model=8,
                         seqlens=[4], dtype="f32", seed=32, with_weights=False)
    cache = dev(p.cache)
    before = cache.clone()
    rows = torch.tensor([4], dtype=torch.int64, device="cuda")      # one past the end
    M.mla_append_latent(mla_dims_of(p), cache, rows, dev(p.c_new), dev(p.kpe_new),
                        torch.from_numpy(p.positions).cuda(), 0)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_ERR_SHAPE
    assert torch.equal(cache, before)


def _with_tiny_wait_limit(fn):
    """Run fn with a 1 ns wait limit; return the status word it left (MLA_OK or MLA_ERR_TIMEOUT)."""
    assert M.mla_check_status() == M.MLA_OK
    try:
        M.mla_set_wait_limit(1)
        fn()
        torch.cuda.synchronize()
        status = M.mla_check_status()
    finally:
        M.mla_set_wait_limit(0)
    assert status in (M.MLA_OK, M.MLA_ERR_TIMEOUT)
    return status


def test_prefill_attention_with_a_tiny_wait_limit_abandons_cleanly():
    # the un-absorbed prefill kernel: producer, MMA issuer and eight softmax warps in pairs that share
    # their rows at a barrier; every path out of an abandoned CTA must meet the same barriers
    B, S, H, Dh = 2, 640, 2, 128
    rng = np.random.default_rng(3)
    q, k, v = (I.round_to(rng.standard_normal((B * S, H * Dh)).astype(np.float32), "bf16") for _ in range(3))
    out = torch.empty(B * S, H * Dh, dtype=torch.bfloat16, device="cuda")
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    status = _with_tiny_wait_limit(
        lambda: M.mla_prefill_attention(qd, kd, vd, None, B, S, H, Dh, 0.0, M.MLA_DECODE_CAUSAL, out))
    print(f"prefill with a 1 ns wait limit: status {status}")
    M.mla_prefill_attention(qd, kd, vd, None, B, S, H, Dh, 0.0, M.MLA_DECODE_CAUSAL, out)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    x = np.asarray(q, np.float64).reshape(B, S, H, Dh)
    kk = np.asarray(k, np.float64).reshape(B, S, H, Dh)
    vv = np.asarray(v, np.float64).reshape(B, S, H, Dh)
    ref = np.zeros((B, S, H, Dh))
    for b in range(B):
        for h in range(H):
            sc = x[b, :, h] @ kk[b, :, h].T / np.sqrt(Dh)
            for i in range(S):
                ref[b, i, h], _ = O.softmax_attend(sc[i, :i + 1], vv[b, :i + 1, h])
    assert_close(host(out), ref.reshape(B * S, H * Dh), "bf16", "attention after recovery")


@pytest.mark.parametrize("m,n,k", [(4096, 2048, 2048), (64, 9728, 1024)], ids=["persistent", "one-tile"])
def test_linear_with_a_tiny_wait_limit_abandons_cleanly(m, n, k):
    # (4096 tokens x 2048 outputs, K 2048: more tiles than SMs and long K, the persistent GEMM with
    # its epilogue warps; 64 tokens x 9728 outputs: 76 one-tile CTAs without a K split)
    rng = np.random.default_rng(4)
    x = I.round_to(rng.standard_normal((m, k)).astype(np.float32), "bf16")
    w = I.round_to((rng.standard_normal((n, k)) / np.sqrt(k)).astype(np.float32), "bf16")
    xd, wd = dev(x, "bf16"), dev(w, "bf16")
    y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    status = _with_tiny_wait_limit(lambda: M.mla_linear(xd, wd, m, n, k, 0, y))
    print(f"linear {m}x{n}x{k} with a 1 ns wait limit: status {status}")
    M.mla_linear(xd, wd, m, n, k, 0, y)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    assert_close(host(y), O.linear(x, w), "bf16", "linear after recovery")
