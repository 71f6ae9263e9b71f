"""The C-ABI host pipeline (ulysses_host_pipeline_*, through HostPipeline:
inputs and results in pinned host memory, copies of neighbouring steps
overlapping the kernels on the library's three streams) against the plain
device-resident layer: several different steps submitted back to back must
each give exactly the results of running that step alone, which catches a
step reading or overwriting the other buffer set too early. With the
one-pass backward, dQ is summed by fp32 reductions in a timing-dependent
order, so it is compared to one bf16 step; everything else bit for bit."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _host_shards(a, P):
    n = a.shape[0] // P
    return [torch.from_numpy(a[p * n:(p + 1) * n].view(np.int16)).view(torch.bfloat16).pin_memory()
            for p in range(P)]


@pytest.mark.parametrize("backward,deterministic", [(True, True), (False, True), (True, False)])
def test_pipelined_steps_equal_single_steps(backward, deterministic):
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d = 1024, 4, 8, 4, 128
    cu = torch.tensor([0, 300, 301, 1024], dtype=torch.int32, device="cuda")
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=cu, backward=backward, deterministic=deterministic)
    steps = []
    for seed in range(5):
        rng = np.random.Generator(np.random.PCG64(100 + seed))
        mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
        arrs = {"q": mk((N, H, d)), "k": mk((N, H_kv, d)), "v": mk((N, H_kv, d))}
        if backward:
            arrs["do"] = mk((N, H, d))
        steps.append(arrs)
    hp = U.HostPipeline(layer)
    outs = []
    for arrs in steps:
        host_in = {k: _host_shards(a, P) for k, a in arrs.items()}
        host_out = {"o": [torch.empty_like(x).pin_memory() for x in host_in["q"]]}
        if backward:
            host_out.update(dq=[torch.empty_like(x).pin_memory() for x in host_in["q"]],
                            dk=[torch.empty_like(x).pin_memory() for x in host_in["k"]],
                            dv=[torch.empty_like(x).pin_memory() for x in host_in["v"]])
        hp.submit(host_in, host_out)
        outs.append(host_out)
    hp.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    for arrs, got in zip(steps, outs):
        dev = {k: [x.cuda() for x in _host_shards(a, P)] for k, a in arrs.items()}
        o = layer.forward(dev["q"], dev["k"], dev["v"])
        ref = {"o": o}
        if backward:
            ref["dq"], ref["dk"], ref["dv"] = layer.backward(dev["do"])
        torch.cuda.synchronize()
        for name, ts in ref.items():
            for r, (a, b) in enumerate(zip(got[name], ts)):
                if name == "dq" and not deterministic:
                    bf = b.cpu().float()
                    step = torch.clamp(bf.abs(), min=2.0 ** -126) * 2.0 ** -7   # one bf16 step (upper bound)
                    assert ((a.float() - bf).abs() <= step).all(), (name, r)
                else:
                    assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16)), (name, r)
    hp.close()
