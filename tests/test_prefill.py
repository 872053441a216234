"""GPU parity of the un-absorbed prefill attention (mla_prefill_attention: tcgen05, bf16, head width
128) against the oracle's softmax, head by head, and of the gated MLA prefill through that route
against the oracle's literal gated_mla ("Gated MLA", the problem equations)."""
import math

import numpy as np
import pytest
import torch

from head_latent_attention_08_b200 import inputs as I
from head_latent_attention_08_b200 import mla as M
from oracle import mla_oracle as O

from gpu_helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu


def oracle_attention(q, k, v, gate, B, S, H, Dh, causal):
    """softmax(Q_h K_h^T / sqrt(D_h)) V_h per sequence and head, each query through the oracle's
    softmax over the positions it may see (attended_count), times the gate."""
    q, k, v = (np.asarray(t, np.float64).reshape(B, S, H, Dh) for t in (q, k, v))
    out = np.zeros((B, S, H, Dh))
    for b in range(B):
        for h in range(H):
            s = (q[b, :, h] @ k[b, :, h].T) / math.sqrt(Dh)
            for i in range(S):
                cnt = O.attended_count(S, S, i, causal)
                out[b, i, h], _ = O.softmax_attend(s[i, :cnt], v[b, :cnt, h])
    out = out.reshape(B * S, H * Dh)
    return out if gate is None else out * np.asarray(gate, np.float64)


# (B, S, H, causal, gate): one tile, a ragged last tile, several tiles with the diagonal inside
CASES = [
    (1, 128, 1, True, False),
    (2, 300, 2, True, True),
    (2, 300, 2, False, False),
    (1, 1000, 2, True, False),
    (3, 77, 3, False, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-S{c[1]}-H{c[2]}-c{int(c[3])}-g{int(c[4])}")
def test_prefill_attention(case):
    B, S, H, causal, with_gate = case
    Dh = 128
    rng = np.random.default_rng(100 + S)
    q, k, v = (I.round_to(rng.standard_normal((B * S, H * Dh)).astype(np.float32), "bf16") for _ in range(3))
    gate = I.round_to(rng.random((B * S, H * Dh)).astype(np.float32), "bf16") if with_gate else None
    out = torch.empty(B * S, H * Dh, dtype=torch.bfloat16, device="cuda")
    M.mla_prefill_attention(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(gate, "bf16") if with_gate else None,
                            B, S, H, Dh, 0.0, M.MLA_DECODE_CAUSAL if causal else 0, out)
    torch.cuda.synchronize()
    assert M.mla_check_status() == M.MLA_OK
    assert_close(host(out), oracle_attention(q, k, v, gate, B, S, H, Dh, causal), "bf16", "attention")


def test_prefill_attention_peaked_scores():
    # queries scaled up 16x: most rows put nearly all weight on one or two keys, and the row maxima
    # move between key tiles, so the reference-maximum rescaling of O runs
    B, S, H, Dh = 1, 640, 2, 128
    rng = np.random.default_rng(5)
    q = I.round_to(16 * rng.standard_normal((B * S, H * Dh)).astype(np.float32), "bf16")
    k, v = (I.round_to(rng.standard_normal((B * S, H * Dh)).astype(np.float32), "bf16") for _ in range(2))
    out = torch.empty(B * S, H * Dh, dtype=torch.bfloat16, device="cuda")
    M.mla_prefill_attention(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), None, B, S, H, Dh, 0.0,
                            M.MLA_DECODE_CAUSAL, out)
    torch.cuda.synchronize()
    assert_close(host(out), oracle_attention(q, k, v, None, B, S, H, Dh, True), "bf16", "attention")


def test_prefill_attention_rejects_unsupported():
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MLAError) as e:
        M.mla_prefill_attention(x, x, x, None, 1, 64, 1, 64, 0.0, 0, x)
    assert e.value.status == 8        # MLA_ERR_UNSUPPORTED: head width 64
    xf = torch.zeros(128, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MLAError):
        M.mla_prefill_attention(xf, xf, xf, None, 1, 128, 1, 128, 0.0, 0, xf)


@pytest.mark.parametrize("causal", [True, False])
def test_gated_mla_unabsorbed_route(causal):
    gp = I.gated_problem(batch=2, seq=384, d_model=512, num_heads=4, latent=128, causal=causal, dtype="bf16",
                         seed=81)
    args = [dev(a, "bf16") for a in (gp.x, gp.wq, gp.wc, gp.wk, gp.wv, gp.wg, gp.wo)]
    r = M.gated_mla(*args, num_heads=4, causal=causal, route="unabsorbed")
    torch.cuda.synchronize()
    y_ref, c_ref = O.gated_mla(gp.x, gp.wq, gp.wc, gp.wk, gp.wv, gp.wg, gp.wo, 4, causal)
    assert_close(host(r["latent_cache"]), c_ref, "bf16", "latent_cache")
    assert_close(host(r["output"]), y_ref, "bf16", "output")
