"""The host logic of the context-parallel decode on CPU, as gloo ranks (world size 2 and 3): the
position split, the causal rule per rank, the exchange and the order of the parts. Each rank decodes
its slice with the oracle and the test merges the gathered parts by their log-sum-exp (restated
here); the result must equal the oracle's decode over the whole sequences. The device side of the
same path (the library's decode on every slice and its merge kernel) is tests/test_context_parallel.py."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (seqlens, n_q, causal): one sequence shorter than the world (empty slices), one of exactly n_q
CASES = [
    ([9, 2, 17, 1], 1, True),
    ([11, 4, 16], 4, True),
    ([11, 5, 16], 3, False),
]


def lse_merge(o_parts, l_parts):
    L = np.stack(l_parts)                         # [R, rows, H]
    m = L.max(0)
    safe = np.where(np.isneginf(m), 0.0, m)
    w = np.where(np.isneginf(L), 0.0, np.exp(L - safe))
    s = w.sum(0)
    o = sum(w[r][..., None] * o_parts[r] for r in range(len(o_parts)))
    out = np.where(s[..., None] > 0, o / np.where(s > 0, s, 1.0)[..., None], 0.0)
    return out, np.where(s > 0, safe + np.log(np.where(s > 0, s, 1.0)), -np.inf)


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from head_latent_attention_08_b200 import context_parallel as CP
    from head_latent_attention_08_b200 import inputs as I
    from head_latent_attention_08_b200 import mla as M
    from oracle import mla_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for k, (seqlens, n_q, causal) in enumerate(CASES):
            p = I.decode_problem(batch=len(seqlens), n_heads=3, kv_lora_rank=16, rope_dim=8, qk_nope=8, v_head=8,
                                 d_model=24, seqlens=seqlens, n_q=n_q, dtype="f32", seed=40 + k)
            q_abs = O.absorb_query(p.q_nope, p.q_pe, p.w_uk)
            lo, hi, lens, last = CP.local_slice(seqlens, n_q, world, rank)
            rows = np.concatenate([np.arange(p.cu_seqlens[b] + lo[b], p.cu_seqlens[b] + hi[b])
                                   for b in range(p.batch)]).astype(np.int64)
            cache_slice = torch.from_numpy(p.cache[rows].astype(np.float32))

            class OracleRank(CP.ContextParallelDecode):
                def decode_slice(self, q):
                    cu = np.concatenate([[0], np.cumsum(self.lens)])
                    o, l = O.decode_absorbed(q, self.cache.numpy(), cu, n_q, p.kv_lora_rank, p.kq_scale,
                                             bool(self.flags & M.MLA_DECODE_CAUSAL))
                    self.o_part.copy_(torch.from_numpy(o))
                    self.l_part.copy_(torch.from_numpy(l))

                def merge(self, o_parts, l_parts, out_lat, lse):
                    o, l = lse_merge([t.numpy().astype(np.float64) for t in o_parts],
                                     [t.numpy().astype(np.float64) for t in l_parts])
                    out_lat.copy_(torch.from_numpy(o))
                    lse.copy_(torch.from_numpy(l))

            d = M.dims(3, 16, 8, 8, 8, 24)
            cp = OracleRank(d, p.batch, n_q, seqlens, cache_slice, causal=causal)
            out = torch.empty(p.batch * n_q, 3, 16, dtype=torch.float32)
            lse = torch.empty(p.batch * n_q, 3, dtype=torch.float32)
            cp(q_abs, out, lse)
            ref, ref_lse = O.decode_absorbed(q_abs, p.cache, p.cu_seqlens, n_q, p.kv_lora_rank, p.kq_scale, causal)
            err = float(np.max(np.abs(out.numpy() - ref))) / float(np.max(np.abs(ref)))
            finite = np.isfinite(ref_lse)
            lerr = float(np.max(np.abs(lse.numpy()[finite] - ref_lse[finite])))
            q.put((rank, k, err, lerr, bool(np.array_equal(np.isneginf(lse.numpy()), np.isneginf(ref_lse))),
                   int(cp.flags)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_host_logic(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + world * 17 + os.getpid() % 500
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
        assert p.exitcode == 0
    got = [q.get(timeout=5) for _ in range(world * len(CASES))]
    for rank, k, err, lerr, same_empty, flags in got:
        assert err < 1e-5, (rank, k, err)          # fp32 partials, fp64 merge
        assert lerr < 1e-5, (rank, k, lerr)
        assert same_empty
        causal = CASES[k][2]
        assert flags == (1 if (causal and rank == world - 1) else 0)


def test_slice_bounds_cover_and_keep_queries_on_last_rank():
    sys.path.insert(0, ROOT)
    from head_latent_attention_08_b200 import context_parallel as CP
    rng = np.random.default_rng(3)
    for world in (1, 2, 3, 5, 8):
        for n_q in (1, 2, 4):
            T = rng.integers(n_q, 60, size=7)
            b = CP.slice_bounds(T, n_q, world)
            assert np.all(b[0] == 0) and np.array_equal(b[-1], T)
            assert np.all(np.diff(b, axis=0) >= 0)
            assert np.all(b[-1] - b[-2] >= n_q)                  # the queries' own positions
            assert np.all(b[-2] <= T - n_q)
