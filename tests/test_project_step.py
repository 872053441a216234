"""GPU parity of the input projections (mla_project_inputs) and of the whole decode step from hidden
states (mla_decode_step, device and host io) against the oracle: the query latent chain and the KV
down-projection of "preacher-1/MLA_tutorial formula.md", Part 3 (inference form), followed by the
append, absorption, decode and output projection already checked one by one elsewhere.

Tolerance: max|gpu - ref| <= tol * max|ref| with tol 1e-4 (fp32) and 2e-2 (bf16); the bf16 path
rounds c' once to bf16 as the operand of the next product, which the fp64 oracle does not."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import inputs as I
from head_latent_attention_08_b200 import mla as M
from oracle import mla_oracle as O

from gpu_helpers import FLAGS_APPEND, TORCH_DT, assert_close, dev, host

pytestmark = pytest.mark.gpu


def page_weights(w: I.ProjectionWeights, H, n, dr, dc):
    """The Linear-convention weights in the page's row-vector layout (a reshape / transpose only)."""
    q_rank = w.w_cq.shape[0]
    return dict(w_cq=w.w_cq.T,
                w_qc=w.w_qc.reshape(H, n, q_rank).transpose(0, 2, 1),
                w_qr=w.w_qr.reshape(H, dr, q_rank).transpose(0, 2, 1),
                w_c=w.w_dkv[:dc].T, w_kr=w.w_dkv[dc:].T)


class Projection:
    def __init__(self, N, D, q_rank, H, n, dr, dc, dtype, seed, cache_rows=None, flags=FLAGS_APPEND):
        self.w = I.projection_weights(n_tokens=N, d_model=D, q_rank=q_rank, n_heads=H, qk_nope=n, rope_dim=dr,
                                      kv_lora_rank=dc, dtype=dtype, seed=seed)
        rng = np.random.default_rng(seed + 1)
        self.rows_total = cache_rows if cache_rows is not None else 2 * N + 3
        self.cache0 = I.round_to(rng.standard_normal((self.rows_total, dc + dr)).astype(np.float32), dtype)
        self.row_idx = rng.permutation(self.rows_total)[:N].astype(np.int64)
        self.positions = rng.integers(0, 40000, size=N).astype(np.int32)
        self.N, self.D, self.q_rank, self.H, self.n, self.dr, self.dc = N, D, q_rank, H, n, dr, dc
        self.dtype, self.flags = dtype, flags

    def gpu(self):
        dt = self.dtype
        d = M.dims(self.H, self.dc, self.dr, self.n, self.n, self.D)
        cache = dev(self.cache0, dt)
        q_nope = torch.empty(self.N, self.H, self.n, dtype=TORCH_DT[dt], device="cuda")
        q_pe = torch.empty(self.N, self.H, self.dr, dtype=TORCH_DT[dt], device="cuda")
        ws = M.workspace(M.mla_project_workspace_size(d, TORCH_DT[dt], self.q_rank, self.N), "cuda")
        w = self.w
        M.mla_project_inputs(d, self.q_rank, dev(w.x, dt), dev(w.w_cq, dt), dev(w.w_qc, dt),
                             dev(w.w_qr, dt) if self.dr else None, dev(w.w_dkv, dt),
                             torch.from_numpy(self.positions).cuda(), q_nope, q_pe if self.dr else None, cache,
                             torch.from_numpy(self.row_idx).cuda(), self.flags, ws)
        torch.cuda.synchronize()
        assert M.mla_check_status() == M.MLA_OK
        return host(q_nope), host(q_pe), host(cache)

    def oracle(self):
        pw = page_weights(self.w, self.H, self.n, self.dr, self.dc)
        rope = bool(self.flags & M.MLA_APPEND_ROPE)
        pos = self.positions if rope else np.zeros_like(self.positions)   # position 0: no rotation
        q_nope, q_pe, c, k_r = O.project_inputs(self.w.x, pw["w_cq"], pw["w_qc"], pw["w_qr"], pw["w_c"],
                                                pw["w_kr"], pos)
        cache = O.append_latent(self.cache0, self.row_idx, c, k_r, self.positions,
                                norm=bool(self.flags & M.MLA_APPEND_NORM), rope=rope, dtype=self.dtype)
        return q_nope, q_pe, cache

    def check(self):
        g_qn, g_qp, g_cache = self.gpu()
        r_qn, r_qp, r_cache = self.oracle()
        assert_close(g_qn, r_qn, self.dtype, "q_nope")
        if self.dr:
            assert_close(g_qp, r_qp, self.dtype, "q_pe")
        assert_close(g_cache[self.row_idx], r_cache[self.row_idx], self.dtype, "appended rows")
        untouched = np.setdiff1d(np.arange(self.rows_total), self.row_idx)
        np.testing.assert_array_equal(g_cache[untouched], np.asarray(self.cache0, np.float64)[untouched])


# (N tokens, d_model, q_rank, H, qk_nope, rope_dim, d_c, dtype). The bf16 cases take the tensor-core
# path: products of 160, 16 and 72 output rows end inside a 128-row tile, 70 tokens leave a ragged
# token tile. The fp32 cases take the CUDA-core path, one of them without a rotary part.
CASES = [
    (70, 256, 128, 4, 64, 32, 128, "bf16"),
    (5, 320, 192, 2, 64, 8, 64, "bf16"),
    (7, 96, 40, 3, 16, 8, 24, "f32"),
    (4, 64, 32, 2, 16, 0, 20, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("flags", [FLAGS_APPEND, 0], ids=["norm_rope", "plain"])
def test_project_inputs(case, flags):
    N, D, q_rank, H, n, dr, dc, dtype = case
    Projection(N, D, q_rank, H, n, dr, dc, dtype, seed=50 + N, flags=flags).check()


def test_project_inputs_deepseek_scale_full():
    # the full query chain and KV down-projection of 64 tokens at DeepSeek-V2 scale: d_model 5120,
    # q_rank 1536, 128 heads of 128 + 64, latent 512 (every output compared)
    Projection(64, 5120, 1536, 128, 128, 64, 512, "bf16", seed=1003, cache_rows=8192).check()


def test_project_inputs_zero_rows():
    d = M.dims(4, 128, 32, 64, 64, 256)
    ws = M.workspace(256, "cuda")
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(8, 160, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(1024, 256, dtype=torch.bfloat16, device="cuda")
    M.mla_project_inputs(d, 128, x, w, w, w, w, None, torch.empty(0, 4, 64, dtype=torch.bfloat16, device="cuda"),
                         None, cache, torch.empty(0, dtype=torch.int64, device="cuda"), 0, ws)
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(cache)) == 0


# ------------------------------------------------------------------------------------------
# the whole step from x
# ------------------------------------------------------------------------------------------

class Step:
    def __init__(self, dtype, H, dc, dr, n, dv, D, q_rank, seqlens, seed):
        self.p = I.decode_problem(batch=len(seqlens), n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=n,
                                  v_head=dv, d_model=D, seqlens=seqlens, n_q=1, dtype=dtype, seed=seed)
        self.w = I.projection_weights(n_tokens=len(seqlens), d_model=D, q_rank=q_rank, n_heads=H, qk_nope=n,
                                      rope_dim=dr, kv_lora_rank=dc, dtype=dtype, seed=seed + 100)
        self.q_rank, self.dtype = q_rank, dtype

    def layer(self):
        p, w, dt = self.p, self.w, self.dtype
        self.cache = dev(p.cache, dt)
        cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).cuda()
        d = M.dims(p.n_heads, p.kv_lora_rank, p.rope_dim, p.qk_nope, p.v_head, p.d_model)
        return M.DecodeLayerStep(d, self.q_rank, p.batch, int(p.seqlens.max()), self.cache, cu, dev(w.w_cq, dt),
                                 dev(w.w_qc, dt), dev(w.w_qr, dt) if p.rope_dim else None, dev(w.w_dkv, dt),
                                 dev(p.w_uk, dt), dev(p.w_uv, dt), dev(p.w_o, dt))

    def run(self, io=M.MLA_IO_DEVICE):
        layer = self.layer()
        p, dt = self.p, self.dtype
        if io == M.MLA_IO_DEVICE:
            y = layer(dev(self.w.x, dt), torch.from_numpy(p.row_idx).cuda(), torch.from_numpy(p.positions).cuda())
        else:
            y = torch.empty(p.batch, p.d_model, dtype=TORCH_DT[dt]).pin_memory()
            layer(torch.from_numpy(self.w.x).to(TORCH_DT[dt]).pin_memory(), torch.from_numpy(p.row_idx).pin_memory(),
                  torch.from_numpy(p.positions).pin_memory(), y=y, io=M.MLA_IO_HOST)
        torch.cuda.synchronize()
        assert M.mla_check_status() == M.MLA_OK
        return host(y), host(self.cache)

    def oracle(self, seqs):
        """y rows and appended cache rows of the sampled sequences, each sequence on its own."""
        p, w = self.p, self.w
        pw = page_weights(w, p.n_heads, p.qk_nope, p.rope_dim, p.kv_lora_rank)
        q_nope, q_pe, c, k_r = O.project_inputs(w.x[seqs], pw["w_cq"], pw["w_qc"], pw["w_qr"], pw["w_c"],
                                                pw["w_kr"], p.positions[seqs])
        lat, rows = [], []
        for k, b in enumerate(seqs):
            lo, hi = int(p.cu_seqlens[b]), int(p.cu_seqlens[b + 1])
            cache = O.append_latent(p.cache[lo:hi], [int(p.row_idx[b]) - lo], c[k:k + 1], k_r[k:k + 1],
                                    p.positions[b:b + 1], norm=True, rope=True, dtype=p.dtype)
            q_abs = O.absorb_query(q_nope[k:k + 1], q_pe[k:k + 1], p.w_uk)
            out_lat, _ = O.decode_absorbed(q_abs, cache, np.array([0, hi - lo]), 1, p.kv_lora_rank, p.kq_scale,
                                           True)
            lat.append(out_lat)
            rows.append(cache[int(p.row_idx[b]) - lo])
        return O.out_project(np.concatenate(lat), p.w_uv, p.w_o), np.stack(rows)

    def check(self, seqs):
        y, cache = self.run()
        y_ref, rows_ref = self.oracle(seqs)
        assert_close(y[seqs], y_ref, self.dtype, "y")
        assert_close(cache[self.p.row_idx[seqs]], rows_ref, self.dtype, "appended rows")
        return y


STEP_CASES = {
    # tensor-core path everywhere: 128 heads, latent 512 + 64, sequences of 1, 70 and 300 positions
    "bf16_tc": ("bf16", 128, 512, 64, 128, 128, 256, 256, [1, 70, 300], 61),
    # CUDA-core path: the fp32 decode-config widths, short sequences across a tile edge
    "f32": ("f32", 16, 128, 32, 64, 64, 128, 96, [5, 64, 65], 62),
}


@pytest.mark.parametrize("name", list(STEP_CASES))
def test_decode_step_from_x(name):
    s = Step(*STEP_CASES[name])
    s.check(list(range(s.p.batch)))


def test_decode_step_host_io_equals_device_io():
    s = Step(*STEP_CASES["bf16_tc"])
    y_dev, cache_dev = s.run(M.MLA_IO_DEVICE)
    y_host, cache_host = s.run(M.MLA_IO_HOST)
    np.testing.assert_array_equal(y_host, y_dev)
    np.testing.assert_array_equal(cache_host, cache_dev)


def test_decode_step_host_io_captured_in_a_cuda_graph():
    # the whole step from host buffers, captured once and replayed: a replay reads x, the index arrays
    # and writes y as they are at replay time, like a direct call with the same buffers
    s = Step(*STEP_CASES["bf16_tc"])
    layer = s.layer()
    p, dt = s.p, s.dtype
    x_h = torch.from_numpy(s.w.x).to(TORCH_DT[dt]).pin_memory()
    rows_h = torch.from_numpy(p.row_idx).pin_memory()
    pos_h = torch.from_numpy(p.positions).pin_memory()
    y_h = torch.empty(p.batch, p.d_model, dtype=TORCH_DT[dt]).pin_memory()
    layer(x_h, rows_h, pos_h, y=y_h, io=M.MLA_IO_HOST)       # first call: one-time set-up outside capture
    torch.cuda.synchronize()
    y_first = y_h.clone()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=side):
        layer(x_h, rows_h, pos_h, y=y_h, io=M.MLA_IO_HOST)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_first)
    # new inputs in the same host buffers: the replay must see them
    x_h.copy_(torch.from_numpy(s.w.x[::-1].copy()).to(TORCH_DT[dt]))
    pos_h.add_(3)
    g.replay()
    torch.cuda.synchronize()
    y_replay = y_h.clone()
    assert not torch.equal(y_replay, y_first)
    layer(x_h, rows_h, pos_h, y=y_h, io=M.MLA_IO_HOST)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    assert torch.equal(y_replay, y_h)
    del g


@pytest.mark.parametrize("n_seq", [240, 241])
def test_decode_step_host_io_many_sequences(n_seq):
    # 240 sequences: the most the index arrays' launch-parameter route takes; 241: they are copied
    rng = np.random.default_rng(64)
    s = Step("bf16", 128, 512, 64, 128, 128, 256, 256, [int(t) for t in rng.integers(1, 40, n_seq)], 63)
    y_dev, cache_dev = s.run(M.MLA_IO_DEVICE)
    y_host, cache_host = s.run(M.MLA_IO_HOST)
    np.testing.assert_array_equal(y_host, y_dev)
    np.testing.assert_array_equal(cache_host, cache_dev)


def test_decode_step_deepseek_scale_sampled():
    # the benchmark's workload: 64 sequences of 4096 positions, d_model 5120, q_rank 1536; four
    # sequences computed by the oracle
    s = Step("bf16", 128, 512, 64, 128, 128, 5120, 1536, [4096] * 64, 1003)
    s.check([0, 21, 42, 63])
