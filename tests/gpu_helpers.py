"""Shared helpers of the GPU parity tests: device copies of the seeded inputs, oracle-side
reference steps and the tolerance rule (max |gpu - ref| <= tol * max |ref|)."""
import numpy as np
import torch

from head_latent_attention_08_b200 import mla as M
from head_latent_attention_08_b200 import inputs as I
from oracle import mla_oracle as O

TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}
FLAGS_APPEND = M.MLA_APPEND_NORM | M.MLA_APPEND_ROPE


def dev(x, dtype="f32", device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=TORCH_DT[dtype])


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    return float(np.max(np.abs(gpu - ref))) / scale


def assert_close(gpu, ref, dtype, what=""):
    e = rel_err(gpu, ref)
    assert e <= TOL[dtype], f"{what}: max|gpu-ref|/max|ref| = {e:.3e} > {TOL[dtype]}"
    return e


# lse is a log-sum-exp in nats: besides the rule above (relative to max|lse_ref|), its absolute error
# is bounded by the arithmetic. On the bf16 path P is rounded to bf16 (relative error below 2^-9 per
# term, numerator and row sum share it), so the row sum is off by less than 2^-8 relative: 4e-3 nats;
# 1e-2 leaves room for the fp32 score accumulation. The fp32 path has no such rounding.
LSE_ATOL = {"f32": 1e-4, "bf16": 1e-2}


def assert_lse_close(gpu, ref, dtype, what="lse", atol=None):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(gpu), empty), f"{what}: -inf rows differ"
    if np.all(empty):
        return 0.0
    d = float(np.max(np.abs(gpu[~empty] - ref[~empty])))
    scale = float(np.max(np.abs(ref[~empty])))
    assert d <= TOL[dtype] * scale, f"{what}: max|gpu-ref| = {d:.3e} > {TOL[dtype]} * {scale:.3e}"
    a = LSE_ATOL[dtype] if atol is None else atol
    assert d <= a, f"{what}: max|gpu-ref| = {d:.3e} nats > {a}"
    return d


def mla_dims_of(p: I.DecodeProblem):
    return M.dims(p.n_heads, p.kv_lora_rank, p.rope_dim, p.qk_nope, p.v_head, p.d_model)


class GpuDecode:
    """The device copies of a DecodeProblem and one full step through the C ABI."""

    def __init__(self, p: I.DecodeProblem, causal=True, append=True):
        self.p = p
        dt = p.dtype
        self.cache = dev(p.cache, dt)
        self.cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
        self.q_nope, self.q_pe = dev(p.q_nope, dt), dev(p.q_pe, dt)
        self.w_uk, self.w_uv, self.w_o = dev(p.w_uk, dt), dev(p.w_uv, dt), dev(p.w_o, dt)
        self.c_new, self.kpe_new = dev(p.c_new), dev(p.kpe_new)
        self.row_idx = torch.from_numpy(p.row_idx).cuda()
        self.positions = torch.from_numpy(p.positions).cuda()
        self.step = M.DecodeStep(mla_dims_of(p), TORCH_DT[dt], p.batch, p.n_q, int(p.seqlens.max()),
                                 self.cache, self.cu, self.w_uk, self.w_uv, self.w_o, causal=causal,
                                 append_flags=FLAGS_APPEND if append else 0)
        self.append = append

    def run(self):
        if self.append:
            y = self.step(self.q_nope, self.q_pe, self.c_new, self.kpe_new, self.row_idx,
                          self.positions)
        else:
            d = self.step.d
            nq = self.p.batch * self.p.n_q
            M.mla_absorb_weights(d, M.MLA_ABSORB_QUERY, self.q_nope, self.q_pe if d.rope_dim else None,
                                 self.w_uk, nq, self.step.q_abs)
            M.mla_decode_absorbed(d, self.step.q_abs, self.cache, self.cu, self.p.batch, self.p.n_q,
                                  self.step.max_seqlen, self.step.flags, self.step.out_lat,
                                  self.step.lse, self.step.ws_dec)
            M.mla_out_project(d, self.step.out_lat, self.w_uv, self.w_o, None, nq, self.step.y,
                              self.step.ws_out)
            y = self.step.y
        torch.cuda.synchronize()
        assert M.mla_check_status() == M.MLA_OK
        return y


def oracle_seq(p: I.DecodeProblem, b: int, causal=True, append=True):
    """Oracle reference for sequence b alone: (q_abs, out_lat, lse, y) of its n_q query rows."""
    lo, hi = int(p.cu_seqlens[b]), int(p.cu_seqlens[b + 1])
    rows = slice(b * p.n_q, (b + 1) * p.n_q)
    cache = p.cache[lo:hi].astype(np.float64)
    if append:
        cache = O.append_latent(cache, p.row_idx[rows] - lo, p.c_new[rows], p.kpe_new[rows],
                                p.positions[rows], norm=True, rope=True, dtype=p.dtype)
    q_abs = O.absorb_query(p.q_nope[rows], p.q_pe[rows], p.w_uk)
    out_lat, lse = O.decode_absorbed(q_abs, cache, np.array([0, hi - lo]), p.n_q, p.kv_lora_rank,
                                     p.kq_scale, causal)
    y = O.out_project(out_lat, p.w_uv, p.w_o)
    return q_abs, out_lat, lse, y, cache
