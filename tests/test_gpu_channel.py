"""GPU parity of the top-k channel-selective layer (qmoe_chan_forward)
against the fp64 oracle (oracle/channel_select.py).

* scores: within 1e-3 relative (plus 2e-5 of the token's largest score);
* selection: bit-exact top-n_keep of the device's own fp32 scores (ranked on
  the host), a valid top-n_keep of the oracle's scores within the score
  tolerance, and the oracle's exact set wherever the oracle's scores leave a
  gap wider than that tolerance at the boundary (n_keep is chosen so from the
  oracle's scores alone);
* y: rel-L2 5e-3 and max |err| 3e-2 * rms(ref), as the MoE layer."""
import numpy as np
import pytest

from oracle import channel_select as CS
from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import synth

from cases import MAX_ERR_RMS, REL_L2, ChanCase, small_cfg

pytestmark = pytest.mark.gpu

SMALL = synth.MoEConfig("chan_small", H=512, I=256, E=16, k=4, n_shared=1, fc1_fmt="int4", fc2_fmt="int4",
                        block=64, hot_experts=3, hot_boost=1.5)


@pytest.fixture(scope="module")
def qm(cuda_ok):
    from skinny_gemm_top_b200 import qmoe
    qmoe.clear_status()
    yield qmoe
    assert qmoe.get_stats().device_status == 0


_CASES = {}


def _case(cfg, seed=1):
    key = (cfg, seed)
    if key not in _CASES:
        _CASES[key] = ChanCase(cfg, seed)
    return _CASES[key]


def _tol(ref_t):
    return 1e-3 * np.abs(ref_t) + 2e-5 * np.abs(ref_t).max()


def _gaps(ref_scores, nk):
    """Per token: the oracle's gap at the n_keep boundary in units of twice the score tolerance."""
    g = []
    for t in range(ref_scores.shape[0]):
        s = np.sort(ref_scores[t])[::-1]
        tol = 1e-3 * s[nk - 1] + 2e-5 * s[0]
        g.append((s[nk - 1] - s[nk]) / (2 * tol) if nk < s.size else np.inf)
    return np.array(g)


def _gap_n_keep(ref_scores, target, spread=64):
    """An n_keep near `target` (from the oracle's scores alone) that leaves the
    most tokens, and then the widest smallest gap, clear of the tolerance."""
    n = ref_scores.shape[1]
    best, key = None, None
    for nk in range(max(1, target - spread), min(n - 1, target + spread) + 1):
        g = _gaps(ref_scores, nk)
        k = ((g > 1.0).sum(), g.min())
        if key is None or k > key:
            best, key = nk, k
    clear = _gaps(ref_scores, best) > 1.0
    assert clear.sum() >= max(1, (clear.size + 1) // 2), "too few tokens with a clear boundary"
    return best, clear


def _check_scores_and_selection(sc_dev, sel_dev, ref_scores, ref_sel, n_keep, clear):
    T = ref_scores.shape[0]
    for t in range(T):
        d, r = sc_dev[t].astype(np.float64), ref_scores[t]
        tol = _tol(r)
        bad = np.abs(d - r) > tol
        assert not bad.any(), f"token {t}: {bad.sum()} scores off, worst {np.max(np.abs(d - r) - tol):.3g}"
        # the device's selection is exactly the top-n_keep of its own fp32 scores
        assert np.array_equal(sel_dev[t], CS.select_top(d, n_keep))
        # ... a valid top-n_keep of the oracle's scores within the tolerance ...
        if n_keep:
            theta = np.sort(r)[::-1][n_keep - 1]
            assert np.all(r[sel_dev[t]] >= theta - tol[sel_dev[t]])
        # ... and the oracle's own set where the oracle's boundary is clear
        if clear[t]:
            assert np.array_equal(sel_dev[t], ref_sel[t])


def _close(got, ref, what=""):
    r, m = Q.rel_l2(got, ref), Q.max_err_over_rms(got, ref)
    assert r <= REL_L2 and m <= MAX_ERR_RMS, f"{what}: rel_l2={r:.3g} max_err/rms={m:.3g}"


@pytest.mark.parametrize("f1,f2,block,T,budget,H", [
    ("int4", "int4", 64, 1, 0.18, 512), ("int4", "int4", 64, 3, 0.13, 512), ("int2", "int4", 128, 1, 0.18, 512),
    ("int2", "int2", 64, 8, 0.18, 512), ("int4", "int2", 128, 2, 0.5, 512), ("int4", "int4", 128, 5, 0.18, 1024),
    ("int2", "int4", 64, 1, 0.13, 1024)])
def test_channel_layer_small(qm, f1, f2, block, T, budget, H):
    cfg = small_cfg(SMALL, fc1_fmt=f1, fc2_fmt=f2, block=block, H=H)
    case = _case(cfg)
    x = synth.tokens(cfg.H, 5, T)
    lg = synth.router_logits(cfg, 5, T)
    xd = Q.bf16_bits_to_f64(x)
    _, _, ref_scores = CS.channel_scores(xd, lg, cfg.k, case.bank)
    n_keep, clear = _gap_n_keep(ref_scores, int(budget * cfg.k * cfg.I))
    y_ref, sel_ref, _ = CS.channel_forward(xd, lg, cfg.k, case.bank, n_keep)
    y, sel, sc = case.run(x, lg, n_keep)
    _check_scores_and_selection(sc, sel, ref_scores, sel_ref, n_keep, clear)
    _close(y[clear], y_ref[clear], f"{f1}/{f2} T={T} n_keep={n_keep}")


def test_channel_layer_full_and_empty_budget(qm):
    cfg = SMALL
    case = _case(cfg)
    T = 2
    x = synth.tokens(cfg.H, 7, T)
    lg = synth.router_logits(cfg, 7, T)
    xd = Q.bf16_bits_to_f64(x)
    full = cfg.k * cfg.I
    y_ref, sel_ref, _ = CS.channel_forward(xd, lg, cfg.k, case.bank, full)
    y, sel, sc = case.run(x, lg, full)
    assert np.array_equal(sel, sel_ref)
    _, _, ref_scores = CS.channel_scores(xd, lg, cfg.k, case.bank)
    _check_scores_and_selection(sc, sel, ref_scores, sel_ref, full, np.ones(T, dtype=bool))
    _close(y, y_ref, "full budget")
    y0_ref, _, _ = CS.channel_forward(xd, lg, cfg.k, case.bank, 0)
    y0, _, _ = case.run(x, lg, 0)
    _close(y0, y0_ref, "no budget")


def test_channel_layer_without_shared_experts_and_repeat_calls(qm):
    cfg = small_cfg(SMALL, n_shared=0, E=8, k=2)
    case = _case(cfg)
    x = synth.tokens(cfg.H, 9, 1)
    lg = synth.router_logits(cfg, 9, 1)
    xd = Q.bf16_bits_to_f64(x)
    _, _, ref_scores = CS.channel_scores(xd, lg, cfg.k, case.bank)
    n_keep, clear = _gap_n_keep(ref_scores, 100)
    assert clear.all()
    y_ref, _, _ = CS.channel_forward(xd, lg, cfg.k, case.bank, n_keep)
    outs = [case.run(x, lg, n_keep)[0] for _ in range(3)]
    for y in outs:
        _close(y, y_ref, "repeat")
    y0, _, _ = case.run(x, lg, 0)
    assert not y0.any()  # no shared expert, no channel: y = 0


def test_channel_layer_v2lite_full_size(qm):
    """The decode workload: V2-Lite shapes, one token, 18% of the routed channels."""
    cfg = synth.V2LITE
    case = _case(cfg, 3)
    x = synth.tokens(cfg.H, 11, 1)
    lg = synth.router_logits(cfg, 11, 1)
    xd = Q.bf16_bits_to_f64(x)
    _, _, ref_scores = CS.channel_scores(xd, lg, cfg.k, case.bank)
    n_keep, clear = _gap_n_keep(ref_scores, int(0.18 * cfg.k * cfg.I))
    assert clear.all()
    y_ref, sel_ref, _ = CS.channel_forward(xd, lg, cfg.k, case.bank, n_keep)
    y, sel, sc = case.run(x, lg, n_keep)
    _check_scores_and_selection(sc, sel, ref_scores, sel_ref, n_keep, clear)
    _close(y, y_ref, f"v2lite n_keep={n_keep}")


def test_channel_layer_rejects_bad_arguments(qm):
    import torch
    case = _case(SMALL)
    c = SMALL
    x = torch.zeros((1, c.H), dtype=torch.int16, device="cuda")
    lg = torch.zeros((1, c.E), dtype=torch.float32, device="cuda")
    y = torch.zeros((1, c.H), dtype=torch.int16, device="cuda")
    need = qm.chan_workspace_size(case.layer, 1, 10)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(qm.QmoeError) as ei:
        qm.chan_forward(case.layer, x, lg, 10, y, ws, ws_bytes=need - 256)
    assert ei.value.status == qm.ERR_SCRATCH
    with pytest.raises(qm.QmoeError) as ei:
        qm.chan_forward(case.layer, x, lg, c.k * c.I + 1, y, ws)
    assert ei.value.status == qm.ERR_INVALID_ARG
    x9 = torch.zeros((9, c.H), dtype=torch.int16, device="cuda")
    with pytest.raises(qm.QmoeError) as ei:
        qm.chan_forward(case.layer, x9, lg, 10, y, ws)
    assert ei.value.status == qm.ERR_INVALID_ARG


def test_channel_wait_expiry_leaves_y_and_recovers(qm):
    """The exact-read kernel's bounded wait driven to expiry by the test hook
    (every block waits 1 ms on a barrier nothing arrives at): the timeout flag
    is set, y keeps its contents, and the next call (hook off) is correct."""
    import torch
    cfg = SMALL
    case = _case(cfg)
    x_bits = synth.tokens(cfg.H, 13, 1)
    lg_np = synth.router_logits(cfg, 13, 1)
    xd = Q.bf16_bits_to_f64(x_bits)
    _, _, ref_scores = CS.channel_scores(xd, lg_np, cfg.k, case.bank)
    n_keep, clear = _gap_n_keep(ref_scores, 150)
    assert clear.all()
    y_ref, _, _ = CS.channel_forward(xd, lg_np, cfg.k, case.bank, n_keep)
    ws = torch.empty(qm.chan_workspace_size(case.layer, 1, n_keep), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    lg = torch.from_numpy(np.ascontiguousarray(lg_np, dtype=np.float32)).cuda()
    y = torch.full((1, cfg.H), 0x3F80, dtype=torch.int16, device="cuda")  # bf16 1.0 everywhere
    try:
        qm.test_set_fault(1, 1_000_000)
        qm.clear_status()
        qm.chan_forward(case.layer, x, lg, n_keep, y, ws)
        torch.cuda.synchronize()
        assert qm.get_stats().device_status & qm.DEVICE_TIMEOUT
        assert bool((y == 0x3F80).all()), "y was written although a block gave up"
    finally:
        qm.test_set_fault(0, 0)
        qm.clear_status()
    qm.chan_forward(case.layer, x, lg, n_keep, y, ws)
    torch.cuda.synchronize()
    assert qm.get_stats().device_status == 0
    from cases import bf16_dev_to_f64
    _close(bf16_dev_to_f64(y), y_ref, "channel layer after an expired wait")
