"""GPU parity of gdn_decode_multi (M tokens per sequence, a state checkpoint
after each) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_12_b200 import gdn, inputs
from tests.gpu_util import O_TOL, S_TOL, o_err, s_err

pytestmark = pytest.mark.gpu


def _run(B, M, H_qk, H_v, dtype, seed, s=0):
    dc = inputs.make_decode(B, H_qk, H_v, 128, seed=seed)
    win = dc.window(s, M, dtype)
    dev = [x.cuda() for x in win]
    S_in = dc.S0.cuda()
    o, S_steps = gdn.decode_multi(*dev, S_in)
    torch.cuda.synchronize()
    assert gdn.last_device_error() == gdn.GDN_OK
    assert torch.equal(S_in.cpu(), dc.S0)  # the input state is read only
    return dc, win, o, S_steps


@pytest.mark.parametrize("M", [2, 3, 4, 8])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_multi_small(M, dtype):
    B, H_qk, H_v = 5, 2, 6
    dc, win, o, S_steps = _run(B, M, H_qk, H_v, dtype, seed=31 + M)
    o_ref, S_ref = oracle.decode_multi(*win, dc.S0)
    for j in range(M):
        assert o_err(o[:, j], o_ref[:, j]) <= O_TOL, j
        assert s_err(S_steps[:, j], S_ref[:, j]) <= S_TOL, j


def test_one_token_in_place_is_a_decode_step():
    B, H_qk, H_v = 6, 2, 6
    dc = inputs.make_decode(B, H_qk, H_v, 128, seed=41)
    q, k, v, la, be = (x.cuda() for x in dc.window(0, 1))
    S = dc.S0.cuda()
    o, S_steps = gdn.decode_multi(q, k, v, la, be, S, S_steps=S.view(B, 1, H_v, 128, 128))
    S2 = dc.S0.cuda()
    o2 = gdn.decode_step(q[:, 0].contiguous(), k[:, 0].contiguous(), v[:, 0].contiguous(),
                         la[:, 0].contiguous(), be[:, 0].contiguous(), S2)
    torch.cuda.synchronize()
    assert torch.equal(o[:, 0], o2)
    assert torch.equal(S, S2)


def test_checkpoints_equal_chained_single_steps():
    # the multi-token kernel against M launches of the single-step kernel
    B, H_qk, H_v, M = 8, 2, 6, 4
    dc, win, o, S_steps = _run(B, M, H_qk, H_v, torch.bfloat16, seed=42)
    S = dc.S0.cuda()
    for j in range(M):
        q, k, v, la, be = (x[:, j].contiguous().cuda() for x in win)
        oj = gdn.decode_step(q, k, v, la, be, S)
        torch.cuda.synchronize()
        assert (o[:, j].float() - oj.float()).abs().max().item() <= 2e-2 * oj.float().abs().max().item()
        rel = ((S_steps[:, j] - S).norm() / S.norm()).item()
        assert rel <= 1e-5, (j, rel)


def test_decode_multi_256_sequences_48_heads_sampled():
    # the serving shape: 256 sequences x 48 V heads, M = 4 (three drafted tokens)
    B, H_qk, H_v, M = 256, 16, 48, 4
    dc, win, o, S_steps = _run(B, M, H_qk, H_v, torch.bfloat16, seed=4, s=100)
    rows = np.array([0, 1, 77, 128, 200, 255])
    sub = [x[rows] for x in win]
    o_ref, S_ref = oracle.decode_multi(*sub, dc.S0[rows])
    ridx = torch.from_numpy(rows).cuda()
    for j in range(M):
        assert o_err(o[ridx, j], o_ref[:, j]) <= O_TOL, j
        assert s_err(S_steps[ridx, j], S_ref[:, j]) <= S_TOL, j
    assert torch.isfinite(S_steps).all() and torch.isfinite(o.float()).all()
