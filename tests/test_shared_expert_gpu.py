"""Shared expert (a dense SwiGLU MLP with LoRA on every token, added to the routed
experts' output) through the C ABI against the fp64 oracle.

The shared expert is the layer with one expert, k = 1 and routing weight 1
(softmax over a single picked logit), run by shared_expert_step.  Checked element
by element against the oracle, and in combination with a routed layer: the sum of
the two outputs and of the two dX against the oracle's sum.
"""
import numpy as np
import pytest

import mixture_experts_lora_b200 as ml
import oracle.moe_lora_oracle as O
from moe_inputs import small_config

from gpu_common import TOL, check_full_parity, ensure_built, inputs_on, oracle_full, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def _shared(cfg, seed):
    inp, cpu = inputs_on(cfg, seed=seed)
    buf = ml.alloc_buffers(cfg.T, cfg.m, cfg.n, 1, 1, cfg.r, cfg.scale)
    ml.shared_expert_step(inp, cfg.scale, buf)
    assert ml.moe_get_device_error() == ml.MOE_OK
    return inp, cpu, buf


@pytest.mark.parametrize("cfg", [small_config(T=300, m=128, n=64, E=1, k=1, r=16, alpha=32),
                                 small_config(T=77, m=144, n=80, E=1, k=1, r=8, alpha=16)],
                         ids=["dense", "ragged"])
def test_shared_expert_full_parity(cfg):
    inp, cpu, buf = _shared(cfg, seed=4)
    errs = check_full_parity(buf, cpu, cfg)
    print(errs)
    # every token's single weight is exactly one
    assert np.all(to_np(buf.w) == 1.0)


def test_routed_plus_shared_layer():
    routed = small_config(T=200, m=128, n=64, E=8, k=2, r=8, alpha=16)
    shared = small_config(T=200, m=128, n=64, E=1, k=1, r=8, alpha=16)
    inp_r, cpu_r = inputs_on(routed, seed=1)
    inp_s, cpu_s, buf_s = _shared(shared, seed=2)
    inp_s["X"].copy_(inp_r["X"])            # the same tokens go through both
    inp_s["dY"].copy_(inp_r["dY"])
    cpu_s["X"], cpu_s["dY"] = cpu_r["X"], cpu_r["dY"]
    ml.shared_expert_step(inp_s, shared.scale, buf_s)
    buf_r = ml.alloc_buffers(routed.T, routed.m, routed.n, routed.E, routed.k, routed.r, routed.scale)
    ml.layer_step(inp_r, routed.k, routed.scale, buf_r)
    assert ml.moe_get_device_error() == ml.MOE_OK
    Yr, _, gr = oracle_full(cpu_r, routed)
    Ys, _, gs = oracle_full(cpu_s, shared)
    Y = to_np(buf_r.Y) + to_np(buf_s.Y)
    dX = to_np(buf_r.dX) + to_np(buf_s.dX)
    assert rel_err(Y, Yr + Ys) <= TOL
    assert rel_err(dX, gr["dX"] + gs["dX"]) <= TOL


def test_routed_and_shared_on_two_streams_match_their_solo_runs():
    # a model runs the shared expert beside the routed layer: the two share no
    # library state but the status word, so concurrent calls give the solo bits
    import torch
    rcfg = small_config(T=512, m=256, n=128, E=8, k=2, r=16, alpha=16)
    scfg = small_config(T=512, m=256, n=128, E=1, k=1, r=16, alpha=16)
    rinp, _ = inputs_on(rcfg, seed=5)
    sinp, _ = inputs_on(scfg, seed=6)
    names = ("Y", "dX", "dA_gu", "dB_gu", "dA_d", "dB_d")

    def solo():
        rb = ml.alloc_buffers(rcfg.T, rcfg.m, rcfg.n, rcfg.E, rcfg.k, rcfg.r, rcfg.scale)
        sb = ml.alloc_buffers(scfg.T, scfg.m, scfg.n, 1, 1, scfg.r, scfg.scale)
        ml.layer_step(rinp, rcfg.k, rcfg.scale, rb)
        ml.shared_expert_step(sinp, scfg.scale, sb)
        torch.cuda.synchronize()
        return rb, sb

    ref_r, ref_s = solo()
    rb = ml.alloc_buffers(rcfg.T, rcfg.m, rcfg.n, rcfg.E, rcfg.k, rcfg.r, rcfg.scale)
    sb = ml.alloc_buffers(scfg.T, scfg.m, scfg.n, 1, 1, scfg.r, scfg.scale)
    side = torch.cuda.Stream()
    for _ in range(3):
        main = torch.cuda.current_stream()
        side.wait_stream(main)
        ml.layer_step(rinp, rcfg.k, rcfg.scale, rb)
        with torch.cuda.stream(side):
            ml.shared_expert_step(sinp, scfg.scale, sb)
        main.wait_stream(side)
        torch.cuda.synchronize()
        assert ml.moe_get_device_error() == ml.MOE_OK
        for n in names:
            assert torch.equal(getattr(rb, n), getattr(ref_r, n)), ("routed", n)
            assert torch.equal(getattr(sb, n), getattr(ref_s, n)), ("shared", n)
