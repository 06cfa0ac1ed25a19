"""The attention kernel's timeout path, run on purpose and without a fault.

Every device-side wait of the tcgen05 kernels is bounded; when one runs out the
kernel latches VSA_ERR_DEVICE_TIMEOUT, lets its own copies and tensor-core work
finish, frees its tensor memory and returns ("From 650 s to 72 s", "What
transfers": fail loudly, never hang). Here a short limit and the plan's test hold
(the softmax warps wait, after their first block of scores, on a barrier nothing
arrives on) make every CTA take that path with copies and MMAs in flight. The
status must reach the host, and the context must stay usable: the next launch on
the same plan, with the hold off, must match the oracle.
"""
import numpy as np
import pytest

import oracle.vsa_oracle as O
import tile_sparse_video_pack_b200 as T
from gpu_util import LayerRun, bf16_to_f64, check_close, oracle_inputs_f64, ragged_gpu_config
from vsa_synth import get_config

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "ragged128"])
def test_wait_limit_runs_out_and_the_plan_recovers(name):
    import torch
    cfg = get_config("tiny") if name == "tiny" else ragged_gpu_config(128)
    r = LayerRun(cfg, 0.5).run(fused=True)           # a normal run first: selection and packed tiles
    b, p = r.bufs, r.plan
    good = bf16_to_f64(b["op"])
    p.set_wait_limit(20_000_000)                      # 20 ms
    p.set_test_hold(True)
    b["op"].zero_()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], b["lse"])
    t1.record()
    with pytest.raises(T.VsaError) as e:
        p.check()
    assert e.value.status == 4                        # VSA_ERR_DEVICE_TIMEOUT
    assert t0.elapsed_time(t1) < 2000.0               # ended near the short limit, not the default
    # the check cleared the latched error; the context still works
    p.set_test_hold(False)
    p.set_wait_limit(0)
    p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], b["lse"])
    p.check()
    assert np.array_equal(bf16_to_f64(b["op"]), good)
    p.tile_unpack(b["op"], r.out)
    p.check()
    q, k, v = oracle_inputs_f64(r.inp)
    kept = {(bb, h): r.kept(bb, h) for bb in range(cfg.batch) for h in range(cfg.heads)}
    res = O.run_layer(cfg, q, k, v, r.k, gate=r.inp.gate, w_q=r.inp.w_q, w_k=r.inp.w_k, kept=kept)
    check_close(bf16_to_f64(r.out), res.out)


def test_wait_limit_bounds():
    r = LayerRun(get_config("tiny"), 0.5)
    for bad in (1, 999, 60_000_000_001):
        with pytest.raises(T.VsaError):
            r.plan.set_wait_limit(bad)
    r.plan.set_wait_limit(1000)
    r.plan.set_wait_limit(0)
    assert T.vsa.library().vsa_plan_set_test_hold(r.plan._h, 2) == 1   # only 0 or 1
