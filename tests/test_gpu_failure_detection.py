"""Failure detection in the tensor-core GEMMs, without a GPU fault.

Every pipeline wait inside the GEMMs is bounded in time.  The test makes one
run out on purpose: with the test switch of moe_debug_set_pipeline the TMA
producer issues nothing, so the MMA issuer waits for a stage that never
fills.  After the (short) limit the kernel must record MOE_DEV_PIPELINE_TIMEOUT
in the workspace status word, drain and return -- the context stays usable --
and the next call on the same stream and workspace must be correct against the
fp64 oracle.
"""
import time

import numpy as np
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu

# A small bf16 layer on the tensor-core expert path (d, I multiples of 64).
CFG = C.MoEConfig("timeout_bf16_T64_d256_N8_Z4_K3_I128", T=64, d=256, N=8, Z=4, K=3, I=128,
                  dtype="bf16", w_std=0.05, bias_kind="zero")


@pytest.fixture
def routed():
    L = IN.make_layer_inputs(CFG, device="cuda")
    shape = B.shape_of(CFG)
    buf = B.LayerBuffers(shape)
    B.route(shape, L["x"], L["w_router"], L["bias"], buf.ws, buf.topk_idx, buf.topk_gate,
            buf.counts, buf.n_ffn)
    B.permute(shape, L["x"], buf.topk_idx, buf.counts, buf.offsets, buf.row_token,
              buf.slot_pos, buf.x_perm, buf.ws)
    torch.cuda.synchronize()
    assert B.device_status(buf.ws) == 0
    yield shape, L, buf
    B.set_pipeline_wait(0, False)


def _check_experts(L, buf):
    R = int(buf.offsets[-1])
    off = buf.offsets.cpu().numpy()
    rows = P.to_f64(L["x"])[buf.row_token[:R].cpu().numpy()]
    want = orc.grouped_ffn(rows, off, L["w1"], L["w3"], L["w2"], decode=P.to_f64)
    P.assert_close(P.to_f64(buf.y_perm[:R]), want, "bf16", "y_perm after recovery")


def test_pipeline_wait_that_runs_out_is_reported_and_the_next_call_is_correct(routed):
    shape, L, buf = routed
    limit_ns = 20_000_000  # 20 ms
    B.set_pipeline_wait(limit_ns, stall_first_fill=True)
    try:
        t0 = time.perf_counter()
        B.expert_gate_up(shape, buf.x_perm, L["w1"], L["w3"], buf.offsets, buf.h, buf.ws)
    finally:
        B.set_pipeline_wait(0, False)
    status = B.device_status(buf.ws)  # synchronises
    waited = time.perf_counter() - t0
    assert status & B.DEV_PIPELINE_TIMEOUT, hex(status)
    # it gave up after the short limit, not the 4 s default
    assert waited < 2.0, waited
    # the same stream and workspace: a normal pass is correct and reports nothing
    B.expert_gate_up(shape, buf.x_perm, L["w1"], L["w3"], buf.offsets, buf.h, buf.ws)
    B.expert_down(shape, buf.h, L["w2"], buf.offsets, buf.y_perm, buf.ws)
    torch.cuda.synchronize()
    assert B.device_status(buf.ws) == 0
    _check_experts(L, buf)


def test_short_wait_limit_leaves_normal_calls_unchanged(routed):
    shape, L, buf = routed
    B.expert_ffn(shape, buf.x_perm, L["w1"], L["w3"], L["w2"], buf.offsets, buf.y_perm, buf.ws)
    torch.cuda.synchronize()
    ref = buf.y_perm.clone()
    B.set_pipeline_wait(1_000_000_000)  # 1 s: every wait of a healthy pipeline is far shorter
    try:
        B.expert_ffn(shape, buf.x_perm, L["w1"], L["w3"], L["w2"], buf.offsets, buf.y_perm,
                     buf.ws)
        torch.cuda.synchronize()
    finally:
        B.set_pipeline_wait(0, False)
    assert B.device_status(buf.ws) == 0
    R = int(buf.offsets[-1])
    assert torch.equal(buf.y_perm[:R], ref[:R])
    _check_experts(L, buf)
