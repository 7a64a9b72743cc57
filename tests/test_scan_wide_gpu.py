"""The forward scan with two value blocks per CTA.  kda_chunk_fwd takes it when one block per
CTA would need more CTAs than the GPU has SMs (one scan CTA fills an SM), so that every state
chain runs in one wave.  Checked against the fp64 oracle, and bit for bit against the
one-block scan on the same heads (calls small enough to take that path)."""
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES, TOL_BF16_O, TOL_BF16_S, err_o, err_s, oracle_run, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,H,D", [(1, 200, 40, 128), (2, 130, 40, 64), (1, 65, 80, 64)])
def test_two_block_scan_matches_oracle_and_one_block_scan(B, T, H, D):
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    assert B * H * (D // 32) > nsm  # this call takes the two-block scan
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1500 + T + H, s0_std=0.1)
    d = to_dev(x)
    o, ST = kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN, S0=d["S0"])
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    o_ref, S_ref = oracle_run(x, x["S0"])
    eo, es = err_o(o.float().cpu().numpy(), o_ref), err_s(ST.cpu().numpy(), S_ref)
    assert eo <= TOL_BF16_O and es <= TOL_BF16_S, (eo, es)
    # the same heads in groups that fit one wave of one-block CTAs
    hg = nsm // (B * (D // 32))
    for h0 in range(0, H, hg):
        sl = slice(h0, min(H, h0 + hg))
        xs = {n: d[n][:, :, sl].contiguous() for n in NAMES}
        o1, S1 = kda.kda_chunk_fwd(*(xs[n] for n in NAMES), G_MIN, S0=d["S0"][:, sl].contiguous())
        torch.cuda.synchronize()
        assert kda.kda_device_status() == 0
        assert torch.equal(o1, o[:, :, sl]), h0
        assert torch.equal(S1, ST[:, sl]), h0
