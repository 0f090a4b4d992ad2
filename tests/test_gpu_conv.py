"""Standalone causal depthwise conv1d + SiLU against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_34_b200 as ssm
from selective_state_space_34_b200 import workloads as wl
from gpu_helpers import TOL, assert_close, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Bt,Dn,L,K", [(2, 33, 100, 4), (1, 4, 3, 4), (1, 5, 9, 1), (3, 7, 64, 2),
                                       (1, 3, 1, 3),
                                       # rows of whole 16-byte vectors: the vector path
                                       (2, 9, 8, 4), (1, 6, 16, 3), (2, 5, 256, 1), (1, 3, 256, 2),
                                       (2, 7, 24, 4)])
@pytest.mark.parametrize("dtype,odt", [("bf16", "f32"), ("bf16", "bf16"), ("f32", "f32")])
def test_conv1d_silu(Bt, Dn, L, K, dtype, odt):
    w = wl.shaped("mamba130m_fwd", Bt=Bt, Dn=Dn, L=L, K=K, in_dtype=dtype)
    a = wl.generate(w)
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(a["x"]).to("cuda", act)
    cw = torch.from_numpy(a["conv_w"]).cuda()
    cb = torch.from_numpy(np.linspace(-0.5, 0.5, Dn).astype(np.float32)).cuda()
    u = ssm.ssm_conv1d_silu(x, cw, cb, out_dtype=torch.bfloat16 if odt == "bf16" else torch.float32)
    ref = oracle.conv1d_silu(a["x"], a["conv_w"], np.linspace(-0.5, 0.5, Dn).astype(np.float32))
    assert_close("u", to_np(u), ref, *TOL[(dtype, odt)])


def test_conv_without_bias_and_full_size():
    w = wl.WORKLOADS["mamba130m_fwd"]
    a = wl.generate(w)
    x = torch.from_numpy(a["x"]).to("cuda", torch.bfloat16)
    u = ssm.ssm_conv1d_silu(x, torch.from_numpy(a["conv_w"]).cuda(), None, out_dtype=torch.float32)
    got = to_np(u)
    for b, d in wl.sample_channels(w.Bt, w.Dn, 16):
        ref = oracle.conv1d_silu(a["x"][b:b + 1, d:d + 1], a["conv_w"][d:d + 1])
        assert_close("u", got[b:b + 1, d:d + 1], ref, *TOL[("bf16", "f32")])
