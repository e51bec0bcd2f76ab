"""1-bit LAMB on the GPU (ob_set_layerwise) against the CPU oracle's
1-bit LAMB (OracleRun(lamb=True)), through the C ABI, in both readings.

The readings (the 1-bit LAMB review page prints no rule): each tensor's
step is scaled by its trust ratio ||p|| / ||u||, u being Adam's direction
in the warmup and, in the compression phase, the decoded compressed
momentum over the frozen d ("step": the ratio recomputed every step) or
the ratio of the last warmup step kept from the freeze on ("frozen").  The trust ratios are floats rounded from fp64 sums of
squares that the GPU adds in its own order, so they are compared at 1e-6
relative; whenever they are equal the state that depends on them
(parameters) is compared bit for bit, otherwise within rounding.  The
Adam moments and the frozen d do not depend on the ratios and are compared
bit for bit at every warmup step.
"""
import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.distributed import LocalRanks
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
from gpu_harness import Pair

pytestmark = pytest.mark.gpu

RATIO_RTOL = 1e-6
PARAM_TOL = 1e-5

CASES = {
    "flat-4097-W4": WL.Workload("lamb-flat", ((4097,),), 4, 3, 4, seed=61),
    "encoder-2L-W8": WL.Workload("lamb-encoder", WL.encoder_shapes(2, 128, 512, 1000, 64), 8, 3, 4,
                                 seed=62, fan_in_scaling=True),
    "ragged-W6": WL.Workload("lamb-ragged", ((100_003,), (31,), (0,), (4097,), (70_000,), (1,)), 6,
                             3, 4, seed=63, zero_fraction=0.2),
    "many-workers-W16": WL.Workload("lamb-w16", ((8192 * 3 + 5,), (300,)), 16, 2, 3, seed=64),
}


MODES = ["step", "frozen"]


def _run(wl, synced, mode="step"):
    pr = Pair(wl, lamb=mode)
    exact = True
    for _ in range(wl.warmup_steps):
        pr.warmup_step()
        ratio = pr.gpu.read(B.OB_STATE_RATIO)
        np.testing.assert_allclose(ratio, pr.orc.ratio, rtol=RATIO_RTOL, atol=0)
        exact = exact and np.array_equal(ratio, pr.orc.ratio)
        # the moments depend on the gradients only, never on the ratios
        for kind, ref in ((B.OB_STATE_M, pr.orc.m), (B.OB_STATE_V, pr.orc.v)):
            got = pr.read_tensors(kind)
            for t in range(len(ref)):
                assert np.array_equal(got[t].view(np.uint32), ref[t].view(np.uint32)), (kind, t)
        if exact:
            pr.check_warmup_exact()
        else:
            assert pr.params_rel_l2() <= 1e-6
    pr.freeze()
    pr.check_freeze_exact()
    history = exact
    for _ in range(wl.compressed_steps):
        if synced:
            pr.sync_into_gpu()
        pr.compressed_step()
        ratio = pr.gpu.read(B.OB_STATE_RATIO)
        np.testing.assert_allclose(ratio, pr.orc.ratio, rtol=RATIO_RTOL, atol=0)
        same_ratio = np.array_equal(ratio, pr.orc.ratio)
        scales = pr.check_compressed(history_exact=history or synced,
                                     exact_state=synced and same_ratio)
        history = history and scales and same_ratio
    return pr


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(CASES))
def test_lamb_resynced_steps_match_the_oracle(name, mode):
    """Every compressed step starts from the oracle's state (written into
    the GPU, which makes it recompute ||p||^2 and D_j; in the frozen mode
    the kept ratios too): words, scales, ratios, errors, momentum and
    parameters as the oracle's."""
    pr = _run(CASES[name], synced=True, mode=mode)
    pr.close()


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", list(CASES))
def test_lamb_free_running_steps_track_the_oracle(name, mode):
    pr = _run(CASES[name], synced=False, mode=mode)
    try:
        assert pr.params_rel_l2() <= PARAM_TOL
    finally:
        pr.close()


@pytest.mark.parametrize("mode", MODES)
def test_lamb_with_unit_ratios_is_one_bit_adam(mode):
    """Parameters held at 0 (learning rate 0) make every trust ratio 1: the
    LAMB context then takes 1-bit Adam's steps bit for bit."""
    wl = WL.Workload("lamb-unit", ((5000,), (129,), (0,)), 4, 2, 3, seed=65)
    offs, n_pad = B.ob_layout(wl.numels)
    scale = WL.grad_scale_vector(wl, offs, n_pad, device="cuda")
    hp = dict(WL.HYPER, lr=0.0)
    a = OneBitAdam(wl.numels, wl.W, **hp)
    b = OneBitAdam(wl.numels, wl.W, layerwise=mode, **hp)
    g = torch.empty((wl.W, n_pad), device="cuda")
    try:
        for step in range(5):
            WL.fill_grads(wl, step, scale, g)
            for o in (a, b):
                if step < 2:
                    o.warmup_step(g)
                else:
                    if step == 2:
                        o.freeze()
                    o.step(g)
            assert np.all(b.read(B.OB_STATE_RATIO) == 1.0)
        for kind in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_D, B.OB_STATE_E_SERVER,
                     B.OB_STATE_BITS_SERVER, B.OB_STATE_S_SERVER):
            np.testing.assert_array_equal(a.read(kind), b.read(kind), err_msg=str(kind))
    finally:
        a.close()
        b.close()


def _lamb_pair_steps(opts, wl, steps, warmup=2):
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offs, n_pad, device="cuda")
    for o in opts:
        o.params.copy_(params)
    g = torch.empty((wl.W, n_pad), device="cuda")
    for step in range(steps):
        WL.fill_grads(wl, step, scale, g)
        for o in opts:
            if step < warmup:
                o.warmup_step(g)
            else:
                if step == warmup:
                    o.freeze()
                o.step(g)
    torch.cuda.synchronize()


@pytest.mark.parametrize("mode", MODES)
def test_lamb_graph_mode_equals_direct_launches(mode):
    wl = WL.Workload("lamb-graph", ((70_000,), (33,), (4096 * 3,)), 4, 2, 4, seed=66)
    a = OneBitAdam(wl.numels, wl.W, layerwise=mode, **WL.HYPER)
    b = OneBitAdam(wl.numels, wl.W, layerwise=mode, **WL.HYPER)
    a.graph(False)
    b.graph(True)
    try:
        _lamb_pair_steps([a, b], wl, 7)
        for kind in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_RATIO, B.OB_STATE_S_SERVER):
            np.testing.assert_array_equal(a.read(kind), b.read(kind), err_msg=str(kind))
    finally:
        a.close()
        b.close()


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("peer_words", [False, True], ids=["exchange", "peer-words"])
@pytest.mark.parametrize("G", [2, 4])
def test_lamb_split_step_equals_one_context(G, peer_words, mode):
    """The split step with layerwise rates: every rank updates all
    parameters with the same ratios, bit for bit one LAMB context."""
    sizes, W = ((100_003,), (31,), (4097,), (70_000,)), 8
    wl = WL.Workload("lamb-split", sizes, W, 2, 4, seed=67)
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offs, n_pad, device="cuda")
    ref = OneBitAdam(wl.numels, W, params=params.clone(), layerwise=mode, **WL.HYPER)
    ranks = LocalRanks(wl.numels, W, G, layerwise=mode, peer_words=peer_words, **WL.HYPER)
    try:
        for r in ranks.ranks:
            r.params.copy_(params)
        g = torch.empty((W, n_pad), device="cuda")
        for step in range(6):
            WL.fill_grads(wl, step, scale, g)
            if step < 2:
                ref.warmup_step(g)
                ranks.warmup_step(g)
            else:
                if step == 2:
                    ref.freeze()
                    ranks.freeze()
                ref.step(g)
                ranks.step(g)
        torch.cuda.synchronize()
        for r in ranks.ranks:
            for kind in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_RATIO, B.OB_STATE_S_SERVER):
                np.testing.assert_array_equal(r.read(kind), ref.read(kind), err_msg=str(kind))
    finally:
        ref.close()
        ranks.close()


def test_layerwise_switch_only_before_the_first_step():
    o = OneBitAdam([1000], 2, **WL.HYPER)
    try:
        B.ob_set_layerwise(o.ctx, True)
        B.ob_set_layerwise(o.ctx, False)
        assert np.all(o.read(B.OB_STATE_RATIO) == 1.0)
        o.warmup_step(torch.zeros((2, 1024), device="cuda"))
        with pytest.raises(B.OnebitError) as e:
            B.ob_set_layerwise(o.ctx, True)
        assert e.value.status == B.OB_ERR_PHASE
        with pytest.raises(B.OnebitError) as e:     # read only
            o.write(B.OB_STATE_RATIO, 0, np.ones(1, np.float32))
        assert e.value.status == B.OB_ERR_INVALID_ARG
    finally:
        o.close()


def test_frozen_ratios_are_the_last_warmup_steps():
    """In the frozen mode the ratios read after every compressed step are
    those of the last warmup step, bit for bit; in the per-step mode they
    change with the steps."""
    wl = WL.Workload("lamb-kept", ((30_000,), (4_097,), (77,)), 4, 3, 3, seed=68)
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offs, n_pad, device="cuda")
    hp = dict(WL.HYPER, lr=0.05)
    runs = {m: OneBitAdam(wl.numels, wl.W, params=params.clone(), layerwise=m, **hp) for m in MODES}
    g = torch.empty((wl.W, n_pad), device="cuda")
    try:
        kept = {}
        for step in range(6):
            WL.fill_grads(wl, step, scale, g)
            for m, o in runs.items():
                if step < 3:
                    o.warmup_step(g)
                else:
                    if step == 3:
                        o.freeze()
                        kept[m] = o.read(B.OB_STATE_RATIO)
                    o.step(g)
        np.testing.assert_array_equal(kept["step"], kept["frozen"])   # the same warmup
        np.testing.assert_array_equal(runs["frozen"].read(B.OB_STATE_RATIO), kept["frozen"])
        assert not np.array_equal(runs["step"].read(B.OB_STATE_RATIO), kept["step"])
    finally:
        for o in runs.values():
            o.close()


def test_frozen_ratios_are_state():
    """In the frozen mode the kept ratios can be written (resume): a ratio of
    0 leaves that tensor's parameters unchanged by a compressed step, a
    ratio of 1 gives 1-bit Adam's step, bit for bit.  In the per-step mode
    the ratios stay read only, and a mode outside the three is refused."""
    wl = WL.Workload("lamb-state", ((20_000,), (4_097,)), 4, 2, 2, seed=69)
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offs, n_pad, device="cuda")
    adam = OneBitAdam(wl.numels, wl.W, params=params.clone(), **WL.HYPER)
    lamb = OneBitAdam(wl.numels, wl.W, params=params.clone(), layerwise="frozen", **WL.HYPER)
    g = torch.empty((wl.W, n_pad), device="cuda")
    try:
        for step in range(2):
            WL.fill_grads(wl, step, scale, g)
            adam.warmup_step(g)
            lamb.warmup_step(g)
        adam.freeze()
        lamb.freeze()
        # the same state entering the compressed step, and ratios (0, 1)
        for kind in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_D):
            lamb.write(kind, 0, adam.read(kind))
        lamb.write(B.OB_STATE_RATIO, 0, np.array([0.0, 1.0], np.float32))
        before = lamb.read(B.OB_STATE_P)
        WL.fill_grads(wl, 2, scale, g)
        adam.step(g)
        lamb.step(g)
        got, want = lamb.read(B.OB_STATE_P), adam.read(B.OB_STATE_P)
        a, n0 = offs[0], wl.numels[0]
        b, n1 = offs[1], wl.numels[1]
        assert np.array_equal(got[a:a + n0].view(np.uint32), before[a:a + n0].view(np.uint32))
        assert np.array_equal(got[b:b + n1].view(np.uint32), want[b:b + n1].view(np.uint32))
        assert not np.array_equal(want[a:a + n0], before[a:a + n0])
        np.testing.assert_array_equal(lamb.read(B.OB_STATE_RATIO), [0.0, 1.0])
    finally:
        adam.close()
        lamb.close()
    o = OneBitAdam([1000], 2, **WL.HYPER)
    try:
        with pytest.raises(B.OnebitError) as e:
            B.ob_set_layerwise(o.ctx, 3)
        assert e.value.status == B.OB_ERR_INVALID_ARG
    finally:
        o.close()
