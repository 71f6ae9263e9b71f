"""NEXT-4: the QKV and output projections with the all-to-alls folded into the
GEMMs, against the fp64 oracle: the QKV GEMM's head-shard outputs equal the
oracle's projection followed by its seq->head all-to-all, the output GEMM
reading head shards equals the oracle's head->seq all-to-all followed by its
projection, and the projected forward block matches the oracle chain."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import f64, assert_close, err_stats

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


SHAPES = [
    # N,    P, H, H_kv, d,  hidden
    (1024, 2, 8, 2, 128, 1024),
    (1024, 4, 8, 4, 64, 512),
    (384, 1, 4, 4, 64, 256),      # P = 1, three 128-row tiles, one 256-column tile per tensor group
    (9216, 2, 4, 4, 64, 256),     # weight gradients over 3 token chunks (4096, 4096, 1024) added in fp32
    (1024, 4, 32, 8, 128, 4096),  # the Llama-3-8B layer at the hidden size the bench times (H d = 4096)
]


@pytest.mark.parametrize("N,P,H,H_kv,d,hidden", SHAPES)
def test_qkv_projection_into_head_shards(N, P, H, H_kv, d, hidden):
    import ulysses_sequence_parallelism_b200 as U
    x, w_qkv, _ = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=N + hidden)
    x_seq = [_dev(s) for s in workloads.seq_shards(x, P)]
    mk = lambda hx: [torch.empty(N, hx // P, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    qh, kh, vh = mk(H), mk(H_kv), mk(H_kv)
    U.ulysses_qkv_proj_seq_to_head(x_seq, _dev(w_qkv), qh, kh, vh, N, P, H, H_kv, d, hidden)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    q_s, k_s, v_s = oracle.qkv_projection(workloads.seq_shards(w(x), P), w(w_qkv), H, H_kv, d)
    for name, got, ref in (("Q", qh, q_s), ("K", kh, k_s), ("V", vh, v_s)):
        refh = oracle.seq_to_head(ref)
        for r in range(P):
            assert_close(f"{name} rank {r}", f64(got[r]), refh[r])


@pytest.mark.parametrize("N,P,H,H_kv,d,hidden", SHAPES)
def test_out_projection_from_head_shards(N, P, H, H_kv, d, hidden):
    import ulysses_sequence_parallelism_b200 as U
    _, _, w_o = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=7)
    rng = np.random.Generator(np.random.PCG64(N + P))
    o = workloads.round_to_bf16_bits(rng.standard_normal((N, H, d), dtype=np.float32))
    o_head = oracle.seq_to_head(workloads.seq_shards(o, P))                   # bit patterns, head layout
    oh = [_dev(t) for t in o_head]
    y = [torch.empty(N // P, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    U.ulysses_out_proj_head_to_seq(oh, _dev(w_o), y, N, P, H, H_kv, d, hidden)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    ref = oracle.out_projection(workloads.seq_shards(w(o), P), w(w_o))
    for p in range(P):
        assert_close(f"Y shard {p}", f64(y[p]), ref[p])


def test_projected_forward_block_matches_oracle():
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d, hidden = 1024, 2, 8, 2, 128, 1024
    cu = [0, 300, 301, 1024]
    x, w_qkv, w_o = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=3)
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=torch.tensor(cu, dtype=torch.int32, device="cuda"),
                           backward=False)
    y = layer.forward_projected([_dev(s) for s in workloads.seq_shards(x, P)], _dev(w_qkv), _dev(w_o))
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    q_s, k_s, v_s = oracle.qkv_projection(workloads.seq_shards(w(x), P), w(w_qkv), H, H_kv, d)
    o_s, _ = oracle.ulysses_layer_forward(q_s, k_s, v_s, cu)
    ref = oracle.out_projection(o_s, w(w_o))
    for p in range(P):
        assert_close(f"Y shard {p}", f64(y[p]), ref[p])


@pytest.mark.parametrize("N,P,H,H_kv,d,hidden", SHAPES)
def test_out_projection_backward(N, P, H, H_kv, d, hidden):
    """dO into the head shards and dW_o (reduction over every token of every
    shard, O read from the head shards) against the oracle."""
    import ulysses_sequence_parallelism_b200 as U
    _, _, w_o = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=11)
    rng = np.random.Generator(np.random.PCG64(N + 5))
    mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
    o, dy = mk((N, H, d)), mk((N, hidden))
    oh = [_dev(t) for t in oracle.seq_to_head(workloads.seq_shards(o, P))]
    dys = [_dev(t) for t in workloads.seq_shards(dy, P)]
    doh = [torch.empty(N, H // P, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    dwo = torch.empty(hidden, H * d, dtype=torch.float32, device="cuda")
    U.ulysses_out_proj_bwd(oh, _dev(w_o), dys, doh, dwo, N, P, H, H_kv, d, hidden)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    do_ref, dw_ref = oracle.out_projection_backward(workloads.seq_shards(w(o), P), w(w_o),
                                                    workloads.seq_shards(w(dy), P))
    do_ref_h = oracle.seq_to_head(do_ref)
    for r in range(P):
        assert_close(f"dO rank {r}", f64(doh[r]), do_ref_h[r])
    assert_close("dW_o", f64(dwo), dw_ref)


@pytest.mark.parametrize("N,P,H,H_kv,d,hidden", SHAPES)
def test_qkv_projection_backward(N, P, H, H_kv, d, hidden):
    """dX gathered from the dQ/dK/dV head shards into the sequence shards, and
    dW_qkv (head shards read feature-major) against the oracle."""
    import ulysses_sequence_parallelism_b200 as U
    x, w_qkv, _ = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=13)
    rng = np.random.Generator(np.random.PCG64(N + 9))
    mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
    dq, dk, dv = mk((N, H, d)), mk((N, H_kv, d)), mk((N, H_kv, d))
    heads = lambda a: [_dev(t) for t in oracle.seq_to_head(workloads.seq_shards(a, P))]
    dqh, dkh, dvh = heads(dq), heads(dk), heads(dv)
    xs = [_dev(t) for t in workloads.seq_shards(x, P)]
    dxs = [torch.empty(N // P, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    dw = torch.empty((H + 2 * H_kv) * d, hidden, dtype=torch.float32, device="cuda")
    U.ulysses_qkv_proj_bwd(xs, _dev(w_qkv), dqh, dkh, dvh, dxs, dw, N, P, H, H_kv, d, hidden)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    sh = lambda a: workloads.seq_shards(w(a), P)
    dx_ref, dw_ref = oracle.qkv_projection_backward(sh(x), w(w_qkv), sh(dq), sh(dk), sh(dv))
    for p in range(P):
        assert_close(f"dX shard {p}", f64(dxs[p]), dx_ref[p])
    assert_close("dW_qkv", f64(dw), dw_ref)


def test_projected_block_backward_matches_oracle():
    """forward_projected + backward_projected (QKV projection, attention, output
    projection and their gradients; no permute launches) against the oracle."""
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d, hidden = 1024, 2, 8, 2, 128, 1024
    cu = [0, 300, 301, 1024]
    x, w_qkv, w_o = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=17)
    rng = np.random.Generator(np.random.PCG64(19))
    dy = workloads.round_to_bf16_bits(rng.standard_normal((N, hidden), dtype=np.float32))
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=torch.tensor(cu, dtype=torch.int32, device="cuda"),
                           deterministic=True)
    xs = [_dev(s) for s in workloads.seq_shards(x, P)]
    wq, wo = _dev(w_qkv), _dev(w_o)
    layer.forward_projected(xs, wq, wo)
    dx, dwq, dwo = layer.backward_projected([_dev(s) for s in workloads.seq_shards(dy, P)], xs, wq, wo)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    sh = lambda a: workloads.seq_shards(w(a), P)
    q_s, k_s, v_s = oracle.qkv_projection(sh(x), w(w_qkv), H, H_kv, d)
    o_s, _ = oracle.ulysses_layer_forward(q_s, k_s, v_s, cu)
    do_s, dwo_ref = oracle.out_projection_backward(o_s, w(w_o), sh(dy))
    dq_s, dk_s, dv_s = oracle.ulysses_layer_backward(q_s, k_s, v_s, do_s, cu)
    dx_ref, dwq_ref = oracle.qkv_projection_backward(sh(x), w(w_qkv), dq_s, dk_s, dv_s)
    # The whole chain rounds to bf16 three times on the way to dX and the
    # weight gradients (dO of the output projection, dQ/dK/dV of the attention
    # backward, then the GEMM's own output), against an fp64 chain with no
    # rounding in between; the weight gradients also sum over all N tokens
    # (values here reach ~40). Measured on dX: 0.021 at |ref| = 2.0. So the
    # bar for the chained block is relative: rel RMS <= 1e-2, max error <= 1%
    # of max|ref|. Each stage alone meets the absolute bar (the tests above).
    for name, got, ref in ([(f"dX shard {p}", dx[p], dx_ref[p]) for p in range(P)] +
                           [("dW_qkv", dwq, dwq_ref), ("dW_o", dwo, dwo_ref)]):
        ma, rr = err_stats(f64(got), ref)
        assert rr <= 1e-2 and ma <= 1e-2 * np.abs(ref).max(), (name, ma, rr, np.abs(ref).max())
