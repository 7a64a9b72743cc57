"""kda_chunk_bwd_recorded on the GPU: after a bf16 forward (or a forward prep with the per-head
gate scale) wrote its records into the backward's workspace, the backward that skips its own
prep gives kda_chunk_bwd's gradients bit for bit."""
import numpy as np
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,H,D,with_A", [(1, 200, 2, 128, False), (2, 150, 3, 64, True), (1, 1, 1, 128, False),
                                            (2, 333, 2, 128, True)])
def test_recorded_backward_equals_backward_bitwise(B, T, H, D, with_A):
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1700 + T, s0_std=0.1)
    rng = np.random.default_rng(1701 + T)
    d = {n: x[n].cuda() for n in NAMES}
    dO = torch.from_numpy(rng.normal(size=(B, T, H, D)).astype(np.float32)).to(torch.bfloat16).cuda()
    dST = torch.from_numpy((rng.normal(size=(B, H, D, D)) * 0.5).astype(np.float32)).cuda()
    S0 = x["S0"].cuda()
    A = torch.from_numpy((rng.normal(size=H) * 0.5).astype(np.float32)).cuda() if with_A else None
    g1 = kda.kda_chunk_bwd(*(d[n] for n in NAMES), dO, G_MIN, S0=S0, dS_T=dST, A_log=A)
    ws = torch.empty(kda.kda_chunk_bwd_workspace(B, T, H, D, D), dtype=torch.uint8, device="cuda")
    ws.fill_(0xAB)  # nothing of the backward's own prep may be left to read
    if with_A:
        kda.kda_chunk_fwd_prep(*(d[n] for n in NAMES), ws, G_MIN, A_log=A)
    else:
        kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN, S0=S0, workspace=ws)
    g2 = kda.kda_chunk_bwd_recorded(*(d[n] for n in NAMES), dO, ws, G_MIN, S0=S0, dS_T=dST, A_log=A)
    g3 = kda.kda_chunk_bwd_recorded(*(d[n] for n in NAMES), dO, ws, G_MIN, S0=S0, dS_T=dST, A_log=A)  # again
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    for n, t in g1.items():
        if t is not None:
            assert torch.equal(t, g2[n]), n
            assert torch.equal(t, g3[n]), n
