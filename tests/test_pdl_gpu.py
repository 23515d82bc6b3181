"""Programmatic dependent launch of the one-token decode kernel (MOE_LAUNCH_PDL,
MOE_LAUNCH_EARLY_WEIGHTS): results match the oracle when the inputs the flags do
not vouch for are written by the kernel right before the call on the same stream.

* With "pdl" the ids and x come from a torch kernel launched just before; the
  kernel must wait for it before reading either.
* With "early_weights" the ids were ready before that kernel began (the promise the
  flag makes) but x is its output; the weights stream early, x is read after.
* The gate/up + down sequence of a decode step, both flags, inside a CUDA graph.
"""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import TORCH_OUT, check_full
from workloads import config_problem
from workloads.torch_io import to_device

pytestmark = pytest.mark.gpu


def _call(P, dev, x, ids, out, ws, launch):
    return M.qmm_id(x, ids, dev["packed"], dev["scales"], dev["aux"], n=P.n, group_size=P.group_size,
                    bits=P.bits, fmt=P.fmt, num_experts=P.num_experts, out=out,
                    out_dtype=TORCH_OUT[P.out_dtype], workspace=ws, launch=launch)


@pytest.mark.parametrize("launch", ["pdl", "early_weights"])
@pytest.mark.parametrize("name", ["decode_gate_up", "decode_down"])
def test_inputs_written_just_before(name, launch):
    P = config_problem(name)
    dev = to_device(P)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    x_src = dev["x"].clone()
    ids_src = dev["ids"].clone()
    x = torch.full_like(x_src, float("nan"))
    ids = ids_src.clone() if launch == "early_weights" else torch.zeros_like(ids_src)
    out = torch.full((P.m, P.n_expert_used, P.n), float("nan"), device="cuda")
    torch.cuda.synchronize()
    for _ in range(3):
        # a long-running kernel ahead, then the kernel that produces this call's inputs
        big = torch.empty(64 << 20, dtype=torch.float32, device="cuda").normal_()
        big.mul_(1.0001)
        torch.mul(x_src, 1.0, out=x)
        if launch == "pdl":
            torch.add(ids_src, 0, out=ids)
        _call(P, dev, x, ids, out, ws, launch)
        torch.cuda.synchronize()
        assert M.poll_error(ws) == 0
        nviol, ratio, info = check_full(P, out)
        assert nviol == 0, f"{name}/{launch}: {nviol} outside tolerance ({ratio:.3g}, {info})"
        x.fill_(float("nan"))
        out.fill_(float("nan"))
        if launch == "pdl":
            ids.zero_()


def test_decode_step_in_a_graph():
    Ps = [config_problem("decode_gate_up"), config_problem("decode_down")]
    devs = [to_device(P) for P in Ps]
    wss = [M.new_workspace(1, 8, P.num_experts) for P in Ps]
    outs = [torch.empty((1, 8, P.n), dtype=torch.float32, device="cuda") for P in Ps]
    launches = ("pdl", "early_weights")
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for i in range(2):
            _call(Ps[i], devs[i], devs[i]["x"], devs[i]["ids"], outs[i], wss[i], launches[i])
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(4):
            for i in range(2):
                _call(Ps[i], devs[i], devs[i]["x"], devs[i]["ids"], outs[i], wss[i], launches[i])
    for o in outs:
        o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for i, P in enumerate(Ps):
        assert M.poll_error(wss[i]) == 0
        nviol, ratio, info = check_full(P, outs[i])
        assert nviol == 0, f"{P.name}: {nviol} outside tolerance ({ratio:.3g}, {info})"
    del g
    _ = np
