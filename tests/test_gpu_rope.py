"""Rotary position embedding with per-document positions (thd_rope_apply) against the
fp64 oracle, on layouts whose positions reach 65535."""
import numpy as np
import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import synthetic as syn
from oracle import rope as R
from gpu_util import assert_bf16_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,heads,dim,rot", [([65536, 512, 96], 2, 128, 128), ([3000, 17, 1024], 4, 192, 64),
                                                 ([2], 1, 64, 64)])
def test_rope_matches_oracle(lens, heads, dim, rot):
    cu = syn.cu_seqlens_of(lens)
    T = int(cu[-1])
    pos = thd.thd_position_ids(cu)
    g = torch.Generator(device="cpu").manual_seed(T + dim)
    x = torch.randn(T, heads, dim, generator=g).to(torch.bfloat16)
    xd = x.to("cuda")
    thd.thd_rope_apply(xd, torch.from_numpy(pos).to("cuda"), rot_dim=rot, base=10000.0)
    torch.cuda.synchronize()
    want = R.rope(x.float().numpy(), pos, rot, 10000.0)
    got = xd.float().cpu().numpy()
    assert_bf16_close(got, want, "rope")
    assert np.abs(got - want).mean() <= 2e-3
    assert torch.equal(xd[:, :, rot:].cpu(), x[:, :, rot:])


def test_rope_rejects_bad_arguments():
    x = torch.zeros(4, 1, 8, dtype=torch.float32, device="cuda")
    p = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(thd.ThdError) as e:
        thd.thd_rope_apply(x, p)
    assert e.value.kind == "UNSUPPORTED"
    with pytest.raises(thd.ThdError) as e:
        thd.thd_rope_apply(x.to(torch.bfloat16), p, rot_dim=7)
    assert e.value.kind == "INVALID_ARG"
