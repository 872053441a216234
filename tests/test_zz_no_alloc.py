"""mla_decode_absorbed_noalloc (scratch in the library's fixed device array) against
mla_decode_absorbed (caller workspace) on the same inputs: two calls in a row, each bit-identical to
the workspace entry point, on the tensor-core path (ragged lengths, so split partials live in the
scratch) and on the CUDA-core fp32 path. Collected last on purpose: it must pass alone and after
every other test."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import mla as M
from head_latent_attention_08_b200 import inputs as I
from oracle import mla_oracle as O
from gpu_helpers import dev, mla_dims_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_08_b200 import build
    build.build()
    M.lib()
    M.mla_set_decode_clusters(0)
    assert M.mla_check_status() == M.MLA_OK


def _case(dtype, seqlens, seed, n_q=1):
    if dtype == "bf16":
        p = I.decode_problem(batch=len(seqlens), n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128,
                             v_head=128, d_model=128, seqlens=seqlens, n_q=n_q, dtype="bf16", seed=seed)
    else:
        p = I.decode_problem(batch=len(seqlens), n_heads=16, kv_lora_rank=128, rope_dim=32, qk_nope=64,
                             v_head=64, d_model=64, seqlens=seqlens, n_q=n_q, dtype="f32", seed=seed)
    d = mla_dims_of(p)
    q_abs = dev(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), dtype)
    cache = dev(p.cache, dtype)
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
    rows = p.batch * n_q
    return dict(p=p, d=d, q_abs=q_abs, cache=cache, cu=cu, n_q=n_q, T=int(max(seqlens)),
                out=torch.empty(rows, p.n_heads, p.kv_lora_rank, device="cuda"),
                lse=torch.empty(rows, p.n_heads, device="cuda"))


def _with_workspace(c):
    p = c["p"]
    out, lse = torch.full_like(c["out"], 5.0), torch.full_like(c["lse"], 5.0)
    ws = M.workspace(M.mla_decode_workspace_size(c["d"], c["q_abs"].dtype, p.batch, c["n_q"], c["T"],
                                                 c["cache"].shape[0], M.MLA_DECODE_CAUSAL), "cuda")
    M.mla_decode_absorbed(c["d"], c["q_abs"], c["cache"], c["cu"], p.batch, c["n_q"], c["T"],
                          M.MLA_DECODE_CAUSAL, out, lse, ws)
    return out, lse


def _no_alloc(c):
    p = c["p"]
    c["out"].fill_(7.0)
    c["lse"].fill_(7.0)
    M.mla_decode_absorbed_noalloc(c["d"], c["q_abs"], c["cache"], c["cu"], p.batch, c["n_q"], c["T"],
                                  M.MLA_DECODE_CAUSAL, c["out"], c["lse"])
    return c["out"], c["lse"]


@pytest.mark.parametrize("dtype,first,second", [
    ("bf16", [300, 65, 4000, 7, 1200], [64, 1, 2500]),
    ("f32", [1, 77, 300], [500, 33]),
])
def test_two_calls_in_a_row_match_the_workspace_entry_point(dtype, first, second):
    a, b = _case(dtype, first, 41), _case(dtype, second, 42)
    ref_a, ref_b = _with_workspace(a), _with_workspace(b)
    got_a = _no_alloc(a)
    got_b = _no_alloc(b)              # reuses the scratch the first call left behind
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    for got, ref in ((got_a, ref_a), (got_b, ref_b)):
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1], ref[1])


def test_repeated_calls_take_no_device_memory():
    c = _case("bf16", [300, 65, 4000], 43)
    _no_alloc(c)                      # first use on this device: the library's module is resident
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        _no_alloc(c)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_problem_beyond_the_fixed_scratch_is_rejected():
    c = _case("bf16", [4096] * 16, 44)
    p = c["p"]
    M.mla_set_decode_clusters(200)    # 400 partial slots of 256 KiB: more than the fixed array holds
    try:
        need = M.mla_decode_workspace_size(c["d"], torch.bfloat16, p.batch, 1, 4096, c["cache"].shape[0],
                                           M.MLA_DECODE_CAUSAL)
        assert need > M.MLA_DECODE_NOALLOC_MAX_BYTES
        with pytest.raises(M.MLAError) as e:
            _no_alloc(c)
        assert e.value.status == 5   # MLA_ERR_WORKSPACE
    finally:
        M.mla_set_decode_clusters(0)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
