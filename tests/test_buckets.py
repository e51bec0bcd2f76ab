"""Bucketed steps (one context per bucket, each on its own stream)."""
import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.buckets import BucketedOneBitAdam, split_buckets
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
import oracle


def test_split_buckets_keeps_order_and_sizes():
    assert split_buckets([5, 5, 5, 20, 1, 1], 10) == [[0, 1], [2], [3], [4, 5]]
    assert split_buckets([3], 1) == [[0]]
    assert split_buckets([], 10) == []
    sizes = [4096, 100, 7, 30000, 5, 5, 5]
    b = split_buckets(sizes, 5000)
    assert [t for x in b for t in x] == list(range(len(sizes)))


@pytest.mark.gpu
def test_bucketed_steps_equal_one_context():
    """Tensors are independent problems, so stepping buckets on their own
    streams, each after an event of the producer stream, gives bit for bit
    what one context over the whole list gives; and both follow the CPU
    oracle over the same list (sign words and warmup state bit for bit,
    scales within 1e-6, parameters within 1e-5 relative L2)."""
    wl = WL.Workload("buckets", WL.encoder_shapes(2, 64, 256, 1000, 64), 4, 2, 3, seed=41,
                     fan_in_scaling=True)
    dev = torch.device("cuda")
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device=dev)
    scale = WL.grad_scale_vector(wl, offs, n_pad, device=dev)
    grads = torch.empty((wl.W, n_pad), device=dev)
    whole = OneBitAdam(wl.numels, wl.W, params=params.clone(), **WL.HYPER)
    buckets = split_buckets(wl.numels, 40_000)
    assert len(buckets) > 2
    bk = BucketedOneBitAdam(wl.numels, wl.W, buckets, graph=True, **WL.HYPER)
    b_offs = [bk.layout(b)[0] for b in range(len(buckets))]
    for b, ts in enumerate(buckets):            # same initial parameters
        for t, o in zip(ts, b_offs[b]):
            bk.params(b)[o:o + wl.numels[t]].copy_(params[offs[t]:offs[t] + wl.numels[t]])
    bgrads = [torch.empty((wl.W, bk.layout(b)[1]), device=dev) for b in range(len(buckets))]
    orc = oracle.OracleRun(WL.split(params.cpu().numpy(), offs, wl.numels), wl.W, WL.HYPER)

    def bucket_grads(step):
        WL.fill_grads(wl, step, scale, grads)
        for b, ts in enumerate(buckets):
            bgrads[b].zero_()
            for t, o in zip(ts, b_offs[b]):
                bgrads[b][:, o:o + wl.numels[t]].copy_(grads[:, offs[t]:offs[t] + wl.numels[t]])
        ev = torch.cuda.Event()
        ev.record()
        host = grads.cpu().numpy()
        return ev, [WL.split(host[w], offs, wl.numels) for w in range(wl.W)]

    for step in range(5):
        ev, host_g = bucket_grads(step)
        for b in reversed(range(len(buckets))):  # backward order
            (bk.warmup_step if step < 2 else bk.step)(b, bgrads[b], ev)
        if step == 1:
            bk.wait()
            bk.freeze()
        (whole.warmup_step if step < 2 else whole.step)(grads)
        (orc.warmup_step if step < 2 else orc.compressed_step)(host_g)
        if step == 1:
            whole.freeze()
            orc.freeze()
        bk.wait()
    torch.cuda.synchronize()
    p_whole = whole.read(B.OB_STATE_P)
    sw_whole = whole.read(B.OB_STATE_S_SERVER)
    for b, ts in enumerate(buckets):
        p_b = bk.opts[b].read(B.OB_STATE_P)
        sw_b = bk.opts[b].read(B.OB_STATE_S_SERVER)
        for i, (t, o) in enumerate(zip(ts, b_offs[b])):
            a = p_whole[offs[t]:offs[t] + wl.numels[t]]
            c = p_b[o:o + wl.numels[t]]
            assert np.array_equal(a.view(np.uint32), c.view(np.uint32)), (b, t)
            assert np.array_equal(sw_whole[t], sw_b[i])
            np.testing.assert_allclose(sw_b[i], orc.s_srv[t], rtol=1e-6, err_msg=f"tensor {t}")
        words_b = bk.opts[b].read(B.OB_STATE_BITS_SERVER)
        for t, o in zip(ts, b_offs[b]):
            nw = (wl.numels[t] + 31) // 32
            got_w = words_b[o // 32:o // 32 + nw]
            # bit for bit unless a scale rounded differently (the fp64 sums
            # of squares are added in different orders): then at most 1e-3
            # of the signs may differ
            diff = int(np.unpackbits((got_w ^ orc.sbits[t]).view(np.uint8)).sum())
            assert diff == 0 or (not np.array_equal(sw_whole, orc.s_srv)
                                 and diff <= max(1, 1e-3 * 32 * nw)), (b, t, diff)
    got = np.concatenate(WL.split(p_whole, offs, wl.numels)).astype(np.float64)
    want = np.concatenate(orc.p).astype(np.float64)
    assert np.linalg.norm(got - want) <= 1e-5 * np.linalg.norm(want)
    whole.close()
    bk.close()
