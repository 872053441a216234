"""Context-parallel decode on one GPU: the ranks are emulated one after another (each rank's slice of
the cache decoded by the library with the rank's causal rule, into its own buffers, no rank waiting on
another), then the library's log-sum-exp merge reads every rank's partials. The merged result must
match the oracle's decode over the whole sequences within the usual tolerance."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import context_parallel as CP
from head_latent_attention_08_b200 import inputs as I
from head_latent_attention_08_b200 import mla as M
from oracle import mla_oracle as O

from gpu_helpers import TORCH_DT, assert_close, assert_lse_close, dev, host

pytestmark = pytest.mark.gpu


def emulate(p, world, causal, dtype):
    """Every rank's decode of its slice; returns the per-rank (out_lat, lse) device tensors."""
    d = M.dims(p.n_heads, p.kv_lora_rank, p.rope_dim, p.qk_nope, p.v_head, p.d_model)
    q_abs = dev(O.absorb_query(p.q_nope, p.q_pe, p.w_uk), dtype)
    nq = p.batch * p.n_q
    parts = []
    for rank in range(world):
        lo, hi, lens, last = CP.local_slice(p.seqlens, p.n_q, world, rank)
        rows = np.concatenate([np.arange(p.cu_seqlens[b] + lo[b], p.cu_seqlens[b] + hi[b]) for b in range(p.batch)])
        cache = dev(p.cache[rows.astype(np.int64)], dtype) if rows.size else \
            torch.zeros(0, p.width, dtype=TORCH_DT[dtype], device="cuda")
        cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).cuda()
        flags = M.MLA_DECODE_CAUSAL if (causal and last) else 0
        o = torch.empty(nq, p.n_heads, p.kv_lora_rank, dtype=torch.float32, device="cuda")
        l = torch.empty(nq, p.n_heads, dtype=torch.float32, device="cuda")
        tmax = int(lens.max())
        ws = M.workspace(M.mla_decode_workspace_size(d, TORCH_DT[dtype], p.batch, p.n_q, tmax, cache.shape[0], flags),
                         "cuda")
        M.mla_decode_absorbed(d, q_abs, cache, cu, p.batch, p.n_q, tmax, flags, o, l, ws)
        parts.append((o, l))
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    return d, parts


CASES = {
    # tensor-core decode: ragged lengths, one shorter than the world size, n_q 1 and 4 (causal)
    "bf16_nq1": ("bf16", 128, 512, 64, [3, 70, 300, 1000], 1, True),
    "bf16_nq4": ("bf16", 128, 512, 64, [4, 70, 517, 900], 4, True),
    # CUDA-core decode, non-causal multi-query
    "f32_nq3": ("f32", 16, 128, 32, [5, 64, 65, 200], 3, False),
    # latent widths the merge takes by its other routes: float4 columns not a multiple of 128, and more
    # than 512 columns
    "f32_dc96": ("f32", 8, 96, 16, [5, 40, 90], 2, True),
    "f32_dc1024": ("f32", 4, 1024, 16, [7, 33, 60], 1, False),
    # rows that are not a whole number of 16-byte chunks: the element-wise route
    "f32_dc42": ("f32", 4, 42, 16, [5, 40, 61], 1, True),
}


@pytest.mark.parametrize("world", [2, 3, 4, 6])
@pytest.mark.parametrize("name", list(CASES))
def test_context_parallel_decode(name, world):
    dtype, H, dc, dr, seqlens, n_q, causal = CASES[name]
    p = I.decode_problem(batch=len(seqlens), n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=64, v_head=64,
                         d_model=64, seqlens=seqlens, n_q=n_q, dtype=dtype, seed=70 + world)
    d, parts = emulate(p, world, causal, dtype)
    nq = p.batch * n_q
    out = torch.empty(nq, H, dc, dtype=torch.float32, device="cuda")
    lse = torch.empty(nq, H, dtype=torch.float32, device="cuda")
    M.mla_lse_merge(d, [o for o, _ in parts], [l for _, l in parts], 0, nq, out, lse)
    torch.cuda.synchronize()
    q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
    if dtype == "bf16":
        q_abs = O.store_as(q_abs, "bf16")          # the GPU reads the absorbed query in bf16
    ref, ref_lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, n_q, dc, p.kq_scale, causal)
    assert_close(host(out), ref, dtype, "merged out_lat")
    assert_lse_close(host(lse), ref_lse, dtype, "merged lse")


def test_merge_of_one_part_is_exact_and_row_ranges_agree():
    p = I.decode_problem(batch=3, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=64, v_head=64, d_model=64,
                         seqlens=[9, 130, 257], n_q=1, dtype="bf16", seed=77)
    d, parts = emulate(p, 1, True, "bf16")
    o, l = parts[0]
    out = torch.empty_like(o)
    lse = torch.empty_like(l)
    M.mla_lse_merge(d, [o], [l], 0, 3, out, lse)
    torch.cuda.synchronize()
    assert torch.equal(out, o) and torch.equal(lse, l)      # w = 1: a copy, bit for bit
    # merging rows 1..2 alone gives rows 1..2 of the full merge
    d2, parts2 = emulate(p, 3, True, "bf16")
    full = torch.empty_like(o)
    full_l = torch.empty_like(l)
    M.mla_lse_merge(d2, [x for x, _ in parts2], [y for _, y in parts2], 0, 3, full, full_l)
    sub = torch.empty(2, 128, 512, dtype=torch.float32, device="cuda")
    sub_l = torch.empty(2, 128, dtype=torch.float32, device="cuda")
    M.mla_lse_merge(d2, [x for x, _ in parts2], [y for _, y in parts2], 1, 2, sub, sub_l)
    torch.cuda.synchronize()
    assert torch.equal(sub, full[1:]) and torch.equal(sub_l, full_l[1:])


def test_merge_rejects_bad_arguments():
    d = M.dims(4, 16, 0, 8, 8, 8)
    o = torch.zeros(2, 4, 16, device="cuda")
    l = torch.zeros(2, 4, device="cuda")
    with pytest.raises(M.MLAError):
        M.mla_lse_merge(d, [o] * 17, [l] * 17, 0, 2, o.clone(), l.clone())
    with pytest.raises(M.MLAError):
        M.mla_lse_merge(d, [], [], 0, 2, o.clone(), l.clone())
    # a part that does not start on a 16-byte boundary
    shifted = torch.zeros(o.numel() + 1, device="cuda")[1:].view_as(o)
    with pytest.raises(M.MLAError):
        M.mla_lse_merge(d, [o, shifted], [l, l], 0, 2, o.clone(), l.clone())
