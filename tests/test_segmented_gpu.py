"""kda_chunk_fwd_segmented on the GPU: the whole problem taken a stretch at a time, the prep of
each stretch overlapping the scan of the one before, must equal kda_chunk_fwd on the whole
problem bit for bit (stretches are whole 64-token chunks; the state is carried in float32)."""
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES, TOL_BF16_O, TOL_BF16_S, err_o, err_s, oracle_run, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,H,D,seg", [(1, 1000, 3, 128, 256), (2, 700, 2, 64, 128), (1, 200, 2, 128, 256),
                                         (1, 32768, 16, 128, 4096), (3, 130, 1, 128, 64)])
def test_segmented_equals_one_call_bitwise(B, T, H, D, seg):
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1600 + T + seg, s0_std=0.1)
    d = to_dev(x)
    o1, S1 = kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN, S0=d["S0"])
    o2, S2 = kda.kda_chunk_fwd_segmented(*(d[n] for n in NAMES), seg, G_MIN, S0=d["S0"])
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_segmented_in_place_state_and_zero_start_match_the_oracle():
    B, T, H, D, seg = 1, 450, 2, 128, 128
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1650, s0_std=0.1)
    d = to_dev(x)
    S = d["S0"].clone()
    o, S_T = kda.kda_chunk_fwd_segmented(*(d[n] for n in NAMES), seg, G_MIN, S0=S, S_T=S)  # in place
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0 and S_T.data_ptr() == S.data_ptr()
    o_ref, S_ref = oracle_run(x, x["S0"])
    assert err_o(o.float().cpu().numpy(), o_ref) <= TOL_BF16_O
    assert err_s(S.cpu().numpy(), S_ref) <= TOL_BF16_S
    o0, S0r = kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN)               # S0 = NULL: zeros
    o0s, S0s = kda.kda_chunk_fwd_segmented(*(d[n] for n in NAMES), seg, G_MIN)
    torch.cuda.synchronize()
    assert torch.equal(o0, o0s) and torch.equal(S0r, S0s)


def test_segmented_orders_later_work_on_the_stream():
    """Work queued on the caller's stream after the call sees the last stretch's output and
    state (the scans run on the library's own stream)."""
    B, T, H, D, seg = 1, 2048, 4, 128, 256
    x = synth.make_inputs(B, T, H, D, D, "bf16", seed=1660, s0_std=0.1)
    d = to_dev(x)
    ref_o, ref_S = kda.kda_chunk_fwd(*(d[n] for n in NAMES), G_MIN, S0=d["S0"])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, S_T = kda.kda_chunk_fwd_segmented(*(d[n] for n in NAMES), seg, G_MIN, S0=d["S0"])
        o_copy, S_copy = o.clone(), S_T.clone()   # queued on s right behind the call
    s.synchronize()
    assert torch.equal(o_copy, ref_o) and torch.equal(S_copy, ref_S)
