"""qmoe_forward_static (library-owned scratch, no allocation) against the
workspace entry point qmoe_forward and against the fp64 oracle, through the
C ABI.

Collected after the other test files on purpose: the static scratch is
resolved on its first use, and these tests must pass both alone and after
everything else has run in the same process.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import synth
from cases import MAX_ERR_RMS, REL_L2, MoECase, bf16_dev_to_f64, small_cfg, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qm():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from skinny_gemm_top_b200 import qmoe
    return qmoe


CFGS = {
    "tiny": synth.TINY,
    # routed + shared experts, INT4 both layers (the decode workload's structure)
    "shared": small_cfg(synth.V2LITE, H=512, I=384, E=16),
}


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 8), ("tiny", 24), ("shared", 1), ("shared", 5)])
def test_static_matches_workspace_forward_twice(qm, name, T):
    import torch
    cfg = CFGS[name]
    case = MoECase(cfg, seed=11)
    layer = case.layer()
    x = to_dev(synth.tokens(cfg.H, 11, T))
    lg = torch.from_numpy(np.ascontiguousarray(synth.router_logits(cfg, 11, T))).cuda()
    ws = torch.empty(qm.workspace_size(layer, T), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    qm.forward(layer, x, lg, y_ref, ws)
    torch.cuda.synchronize()
    ref = bf16_dev_to_f64(y_ref)
    assert np.all(np.isfinite(ref))
    x_bits = synth.tokens(cfg.H, 11, T)
    oracle = Q.moe_forward(Q.bf16_bits_to_f64(x_bits), synth.router_logits(cfg, 11, T), cfg.k, case.bank)
    assert Q.rel_l2(ref, oracle) <= REL_L2 and Q.max_err_over_rms(ref, oracle) <= MAX_ERR_RMS, (name, T)
    for call in range(2):  # two calls in a row on the same static scratch
        y = torch.full((T, cfg.H), -1, dtype=torch.int16, device="cuda")
        qm.forward_static(layer, x, lg, y)
        torch.cuda.synchronize()
        got = bf16_dev_to_f64(y)
        for what, want in (("workspace forward", ref), ("oracle", oracle)):
            assert Q.rel_l2(got, want) <= REL_L2, (name, T, call, what)
            assert Q.max_err_over_rms(got, want) <= MAX_ERR_RMS, (name, T, call, what)
    assert qm.get_stats().device_status == 0


def test_static_rejects_requests_beyond_the_array(qm):
    import torch
    cfg = synth.TINY
    case = MoECase(cfg, seed=11)
    layer = case.layer()
    T = 64
    while qm.workspace_size(layer, T) <= qm.STATIC_SCRATCH_BYTES:
        T *= 2
    x = torch.zeros((T, cfg.H), dtype=torch.int16, device="cuda")
    lg = torch.zeros((T, cfg.E), dtype=torch.float32, device="cuda")
    y = torch.zeros((T, cfg.H), dtype=torch.int16, device="cuda")
    with pytest.raises(qm.QmoeError) as e:
        qm.forward_static(layer, x, lg, y)
    assert e.value.status == qm.ERR_STATIC_SCRATCH
    assert "static scratch" in qm.status_str(qm.ERR_STATIC_SCRATCH)
    torch.cuda.synchronize()
    assert int(y.abs().sum().item()) == 0  # nothing was launched
