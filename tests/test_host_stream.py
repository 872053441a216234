"""HostStream: decode steps fed from pinned host memory with the transfers overlapped with the
compute must give, step by step, exactly what the same DecodeStep gives on device inputs."""
import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import mla as M
from head_latent_attention_08_b200 import inputs as I
from gpu_helpers import GpuDecode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_08_b200 import build
    build.build()
    M.lib()


def test_pipelined_steps_match_direct_steps():
    p = I.decode_problem(batch=3, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                         d_model=256, seqlens=[70, 300, 129], dtype="bf16", seed=51)
    g = GpuDecode(p, causal=True, append=True)
    ref = g.run().clone()                      # one direct step (appends the new rows)
    hs = M.HostStream(g.step)
    host = dict(q_nope=g.q_nope.cpu().pin_memory(), q_pe=g.q_pe.cpu().pin_memory(),
                c_new=g.c_new.cpu().pin_memory(), kpe_new=g.kpe_new.cpu().pin_memory())
    outs = [torch.empty(ref.shape, dtype=ref.dtype).pin_memory() for _ in range(5)]
    for h_y in outs:                           # the append rewrites the same rows with the same values
        hs.submit(host["q_nope"], host["q_pe"], host["c_new"], host["kpe_new"], g.row_idx, g.positions, h_y)
    hs.wait()
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    for h_y in outs:
        assert torch.equal(h_y, ref.cpu())
