"""The allocation-free backward entry point (ulysses_attn_bwd_noalloc), for
callers that cannot allocate device memory themselves -- for example a plugin
inside another runtime that owns every allocation, or a loop where a
cudaMalloc (which can synchronise the device) is not allowed.

Called straight through the C ABI, twice in a row with different inputs, and
compared bit for bit with the workspace-taking ulysses_attn_bwd on the same
inputs: both run the same deterministic kernels, so any difference would be a
scratch-aliasing or stale-contents fault in the shared array. This file is
collected last so a failure here comes after every other test ran."""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import f64, shards_to_dev

pytestmark = pytest.mark.gpu


def _arr(ts):
    a = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))


def _draw(shape, seed):
    import workloads
    rng = np.random.Generator(np.random.PCG64(seed))
    return workloads.round_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def test_noalloc_backward_matches_workspace_backward_twice():
    import ulysses_sequence_parallelism_b200 as U
    L = U.lib()
    N, P, H, H_kv, d = 1024, 4, 16, 4, 128
    cu_np = np.array([0, 300, 301, 777, 1024], dtype=np.int32)
    cu = torch.tensor(cu_np, device="cuda")
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=cu)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((101, 202)):
        q, k, v, do = (shards_to_dev(_draw(s, seed + i), P) for i, s in
                       enumerate([(N, H, d), (N, H_kv, d), (N, H_kv, d), (N, H, d)]))
        layer.forward(q, k, v)
        U.ulysses_a2a_seq_to_head(do, None, None, layer.do_h, None, None, N, P, H, H_kv, d)
        # reference: the entry point that takes a caller-owned workspace
        U.ulysses_attn_bwd(layer.q_h, layer.k_h, layer.v_h, layer.o_h, layer.lse, layer.do_h, layer.dq_h,
                           layer.dk_h, layer.dv_h, N, P, H, H_kv, d, layer.workspace, cu, deterministic=True)
        ref = [f64(torch.cat(x, 0)) for x in (layer.dq_h, layer.dk_h, layer.dv_h)]
        dq = [torch.full_like(x, float("nan")) for x in layer.dq_h]
        dk = [torch.full_like(x, float("nan")) for x in layer.dk_h]
        dv = [torch.full_like(x, float("nan")) for x in layer.dv_h]
        fp = [ctypes.cast((ctypes.c_void_p * P)(*[t.data_ptr() for t in layer.lse]), ctypes.POINTER(ctypes.c_void_p))]
        code = L.ulysses_attn_bwd_noalloc(
            _arr(layer.q_h), _arr(layer.k_h), _arr(layer.v_h), _arr(layer.o_h), fp[0], _arr(layer.do_h),
            _arr(dq), _arr(dk), _arr(dv), N, P, H, H_kv, d, ctypes.c_void_p(cu.data_ptr()), len(cu_np) - 1, 0,
            0.0, 0, P, stream)
        assert code == 0, f"call {call}: status {code}"
        torch.cuda.synchronize()
        assert U.ulysses_get_device_status() == (0, 0)
        for name, got, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            g = f64(torch.cat(got, 0))
            assert np.all(np.isfinite(g)), (call, name)
            assert np.array_equal(g, r), f"call {call} {name}: differs from the workspace call"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import ulysses_sequence_parallelism_b200 as U
    L = U.lib()
    P = 4
    fake = (ctypes.c_void_p * P)(*([0x10000] * P))
    pp = ctypes.cast(fake, ctypes.POINTER(ctypes.c_void_p))
    # H * padded N = 32 * 262144 > 4,194,304: rejected before any launch
    code = L.ulysses_attn_bwd_noalloc(pp, pp, pp, pp, pp, pp, pp, pp, pp, 262144, P, 32, 8, 128, None, 0, 0,
                                      0.0, 0, P, None)
    assert code == 2

