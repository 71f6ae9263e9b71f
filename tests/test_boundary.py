"""C-ABI library: it loads, exports every symbol include/ulysses.h declares, and
its host-side validation rejects bad arguments before any launch. No compute
call is made here (these run without a GPU: validation returns before the
CUDA runtime is touched)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ulysses.h")


@pytest.fixture(scope="module")
def L():
    from ulysses_sequence_parallelism_b200 import build
    build.build()
    from ulysses_sequence_parallelism_b200 import _lib
    return _lib.lib()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"ULY_API\s+[\w\s\*]+?\b(ulysses_\w+)\s*\(", txt)))


def test_header_declares_the_four_layer_entry_points():
    syms = declared_symbols()
    for s in ("ulysses_a2a_seq_to_head", "ulysses_a2a_head_to_seq", "ulysses_attn_fwd", "ulysses_attn_bwd"):
        assert s in syms


def test_library_exports_every_declared_symbol(L):
    from ulysses_sequence_parallelism_b200 import _lib
    for s in declared_symbols():
        assert hasattr(L, s), s
    assert set(declared_symbols()) <= set(_lib.exported_symbols()) | set(declared_symbols())
    assert set(_lib.exported_symbols()) <= set(declared_symbols())


def test_status_strings(L):
    assert L.ulysses_status_string(0) == b"ok"
    assert L.ulysses_status_string(1) == b"invalid argument"
    assert L.ulysses_status_string(4) == b"bounded device wait timed out"


def _arr(vals):
    a = (ctypes.c_void_p * len(vals))(*vals)
    return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))


GOOD = 0x10000   # a 16-byte aligned fake device address: never dereferenced (validation fails first)


def _fwd(L, N=256, P=2, H=8, H_kv=8, d=64, ptr=GOOD, causal=1, lo=0, hi=None, cu=None, ns=0, lse_ptr=GOOD):
    p = _arr([ptr] * P)
    lp = _arr([lse_ptr] * P)
    return L.ulysses_attn_fwd(p, p, p, p, lp, N, P, H, H_kv, d, cu, ns, 0, 0.0, causal, lo,
                              P if hi is None else hi, None)


@pytest.mark.parametrize("kw,code", [
    (dict(P=0), 1), (dict(N=0), 1), (dict(N=255), 1),             # N % P
    (dict(H=8, H_kv=3, P=1), 1),                                   # H % H_kv
    (dict(P=16, N=256, H=8, H_kv=8), 1),                           # fewer heads than ranks
    (dict(H=8, H_kv=2, P=4), 1),                                   # H_kv % P: kv heads must split too
    (dict(P=17, N=17 * 16, H=17, H_kv=17), 2),                     # more ranks than supported
    (dict(d=96), 2), (dict(d=256), 2),                             # head dims not built
    (dict(causal=0), 2),                                           # non-causal not built
    (dict(lo=1, hi=1), 1), (dict(lo=-1), 1), (dict(hi=3), 1),      # rank range
    (dict(ptr=0), 1), (dict(ptr=GOOD + 8), 1), (dict(lse_ptr=GOOD + 4), 1),   # null / misaligned
    (dict(cu=ctypes.c_void_p(GOOD), ns=0), 1),                     # cu_seqlens with no documents
])
def test_attn_fwd_validation(L, kw, code):
    assert _fwd(L, **kw) == code


def test_a2a_validation(L):
    P = 2
    p = _arr([GOOD] * P)
    bad = _arr([GOOD, GOOD + 2])
    # slot 1/2 must be given on both sides or neither
    assert L.ulysses_a2a_seq_to_head(p, p, None, p, None, None, 256, P, 8, 8, 64, None, 0, 0, P, None) == 1
    assert L.ulysses_a2a_seq_to_head(bad, None, None, p, None, None, 256, P, 8, 8, 64, None, 0, 0, P, None) == 1
    assert L.ulysses_a2a_head_to_seq(p, None, None, bad, None, None, 256, P, 8, 8, 64, None, 0, 0, P, None) == 1
    assert L.ulysses_a2a_seq_to_head(p, None, None, p, None, None, 256, P, 8, 8, 48, None, 0, 0, P, None) == 2
    # a NULL head-side buffer of a rank inside the range is rejected
    half = _arr([GOOD, 0])
    assert L.ulysses_a2a_seq_to_head(p, None, None, half, None, None, 256, P, 8, 8, 64, None, 0, 0, P, None) == 1


def test_bwd_validation_and_workspace_size(L):
    ws = L.ulysses_attn_bwd_workspace_size(8192, 4, 32, 8, 128, 1)
    assert ws == 2 * 4 * 8 * 8192 * 4          # lse*log2(e) and D_i per (rank, head, row)
    # one pass (d = 128): plus the fp32 dQ accumulator, N x H x d floats
    assert L.ulysses_attn_bwd_workspace_size(8192, 4, 32, 8, 128, 0) == ws + 8192 * 32 * 128 * 4
    # d = 64 always runs the two-pass kernels: no accumulator
    assert L.ulysses_attn_bwd_workspace_size(8192, 4, 32, 8, 64, 0) == ws
    # rows are padded to a multiple of 128
    assert L.ulysses_attn_bwd_workspace_size(200, 2, 8, 8, 128, 0) == 2 * 2 * 4 * 256 * 4 + 256 * 8 * 128 * 4
    assert L.ulysses_attn_bwd_workspace_size(8192, 3, 32, 8, 128, 0) == 0     # invalid shape -> 0
    P = 2
    p = _arr([GOOD] * P)
    for det in (0, 1):
        # workspace too small / misaligned
        assert L.ulysses_attn_bwd(p, p, p, p, p, p, p, p, p, 256, P, 8, 8, 128, None, 0, 0, 0.0, det,
                                  ctypes.c_void_p(GOOD), 16, 0, P, None) == 1
        need = L.ulysses_attn_bwd_workspace_size(256, P, 8, 8, 128, det)
        assert L.ulysses_attn_bwd(p, p, p, p, p, p, p, p, p, 256, P, 8, 8, 128, None, 0, 0, 0.0, det,
                                  ctypes.c_void_p(GOOD + 16), need, 0, P, None) == 1
    # a workspace sized for the two-pass path is too small for the one-pass path
    need1 = L.ulysses_attn_bwd_workspace_size(256, P, 8, 8, 128, 1)
    assert L.ulysses_attn_bwd(p, p, p, p, p, p, p, p, p, 256, P, 8, 8, 128, None, 0, 0, 0.0, 0,
                              ctypes.c_void_p(GOOD), need1, 0, P, None) == 1


def test_fused_entry_points_need_shards_of_128_tokens(L):
    P = 2
    p = _arr([GOOD] * P)
    # N/P = 100: a 128-token tile would straddle two shards
    assert L.ulysses_attn_fwd_seq(p, p, p, p, p, 200, P, 8, 8, 64, None, 0, 0, 0.0, 1, 0, P, None) == 2
    assert L.ulysses_attn_bwd_seq(p, p, p, p, p, p, p, p, p, 200, P, 8, 8, 64, None, 0, 0, 0.0, 1,
                                  ctypes.c_void_p(GOOD), 1 << 20, 0, P, None) == 2
    # every sequence shard must be given, even for a partial rank range
    half = _arr([GOOD, 0])
    assert L.ulysses_attn_fwd_seq(half, p, p, p, p, 256, P, 8, 8, 64, None, 0, 0, 0.0, 1, 0, 1, None) == 1


def test_fragment_entry_points_validate_before_launch(L):
    """Head fragments must be whole GQA groups inside one rank's heads; NULL
    pairing of the k/v slots must match; anything else is rejected with
    nothing launched (fake, never-dereferenced pointers)."""
    P = 2
    p = _arr([GOOD] * P)
    f = ctypes.c_void_p(GOOD)
    N, H, H_kv, d = 256, 8, 2, 128              # g = 4, 4 query heads per rank
    ok_args = (N, P, H, H_kv, d)
    # not whole groups
    assert L.ulysses_a2a_seq_to_head_frag(p, p, p, f, f, f, *ok_args, 2, 4, None) == 1
    assert L.ulysses_a2a_seq_to_head_frag(p, p, p, f, f, f, *ok_args, 0, 2, None) == 1
    # crosses from rank 0's heads into rank 1's
    assert L.ulysses_a2a_seq_to_head_frag(p, p, p, f, f, f, N, P, 8, 8, d, 2, 4, None) == 1
    # out of range, empty
    assert L.ulysses_a2a_seq_to_head_frag(p, p, p, f, f, f, *ok_args, 8, 4, None) == 1
    assert L.ulysses_a2a_head_to_seq_frag(f, f, f, p, p, p, *ok_args, 0, 0, None) == 1
    # k slot given on one side only; misaligned fragment pointer
    assert L.ulysses_a2a_seq_to_head_frag(p, p, None, f, f, f, *ok_args, 0, 4, None) == 1
    assert L.ulysses_a2a_head_to_seq_frag(ctypes.c_void_p(GOOD + 8), None, None, p, None, None, *ok_args, 4, 4,
                                          None) == 1
    # unsupported head dim
    assert L.ulysses_a2a_seq_to_head_frag(p, None, None, f, None, None, N, P, H, H_kv, 96, 0, 4, None) == 2


def test_projection_entry_points_validate_before_launch(L):
    P = 2
    p = _arr([GOOD] * P)
    w = ctypes.c_void_p(GOOD)
    # hidden not a multiple of 256, rows per shard not a multiple of 128: unsupported
    assert L.ulysses_qkv_proj_seq_to_head(p, w, p, p, p, 512, P, 8, 2, 128, 1000, None) == 2
    assert L.ulysses_qkv_proj_seq_to_head(p, w, p, p, p, 400, P, 8, 2, 128, 1024, None) == 2
    assert L.ulysses_out_proj_head_to_seq(p, w, p, 400, P, 8, 2, 128, 1024, None) == 2
    # (H + 2 H_kv) d not a multiple of 256
    assert L.ulysses_qkv_proj_seq_to_head(p, w, p, p, p, 512, P, 2, 2, 64, 1024, None) == 2
    # misaligned weight, missing shard pointer, bad hidden
    assert L.ulysses_qkv_proj_seq_to_head(p, ctypes.c_void_p(GOOD + 2), p, p, p, 512, P, 8, 2, 128, 1024,
                                          None) == 1
    assert L.ulysses_out_proj_head_to_seq(_arr([GOOD, 0]), w, p, 512, P, 8, 2, 128, 1024, None) == 1
    assert L.ulysses_out_proj_head_to_seq(p, w, p, 512, P, 8, 2, 128, 0, None) == 1


@pytest.mark.parametrize("kw", [dict(d=96), dict(d=256), dict(P=17, N=17 * 64, H=17, H_kv=17), dict(N=1023),
                                dict(H_kv=3), dict(lo=2, hi=2)])
def test_noalloc_returns_the_same_status_as_the_workspace_call(L, kw):
    """Shapes the backward rejects get the same status from both entry points
    (nothing is launched: validation fails first)."""
    a = dict(N=1024, P=4, H=16, H_kv=4, d=128, lo=0, hi=None)
    a.update(kw)
    P = a["P"]
    hi = P if a["hi"] is None else a["hi"]
    fake = (ctypes.c_void_p * P)(*([0x10000] * P))
    pp = ctypes.cast(fake, ctypes.POINTER(ctypes.c_void_p))
    ws = ctypes.c_void_p(0x10000)
    ref = L.ulysses_attn_bwd(pp, pp, pp, pp, pp, pp, pp, pp, pp, a["N"], P, a["H"], a["H_kv"], a["d"], None, 0, 0,
                             0.0, 1, ws, 1 << 40, a["lo"], hi, None)
    got = L.ulysses_attn_bwd_noalloc(pp, pp, pp, pp, pp, pp, pp, pp, pp, a["N"], P, a["H"], a["H_kv"], a["d"], None,
                                     0, 0, 0.0, a["lo"], hi, None)
    assert ref != 0
    assert got == ref, (kw, got, ref)


def test_onepass_backward_selection_rule(L):
    """The backward picks the one-pass kernel only when its shared-memory
    layout fits at the dynamic shared-memory offset the device gives it (else
    it runs the two-pass kernels). Offsets at a 1024-byte boundary fit (the
    case on sm_100: 1 KB reserved, no static shared memory); an offset just
    past a boundary leaves the layout short by up to 1008 bytes and does not."""
    f = L.ulysses_attn_bwd_onepass_layout_fits
    assert f(0) == 1 and f(1024) == 1 and f(2048) == 1
    assert f(1024 + 16) == 0 and f(1024 + 64) == 0
    assert f(1024 - 16) == 1                      # 16 bytes of padding: fits
    fits = [o for o in range(0, 2048, 16) if f(o)]
    # the fitting offsets are those within a fixed distance below each boundary
    pads = sorted({(1024 - o % 1024) % 1024 for o in fits})
    assert pads == list(range(0, pads[-1] + 1, 16)) and pads[-1] < 1024


def test_host_pipeline_scratch_size_and_validation(L):
    """The host-to-host pipeline's scratch size is the sum of its parts (two
    sets of sequence-side shards, the head-side shards, the LSE and the
    backward workspace, each rounded up to 256 bytes), unsupported shapes give
    0, and create/submit reject bad arguments before touching CUDA."""
    import ctypes
    N, P, H, H_kv, d = 1024, 4, 8, 4, 128
    rnd = lambda x: (x + 255) // 256 * 256
    q = N // P * H * d * 2
    kv = N // P * H_kv * d * 2
    lse = H // P * N * 4
    for bwd, det in ((0, 0), (1, 0), (1, 1)):
        ins = [q, kv, kv] + ([q] if bwd else [])
        outs = [q] + ([q, kv, kv] if bwd else [])
        heads = [q, kv, kv, q] + ([q, q, kv, kv] if bwd else [])
        want = 2 * P * sum(rnd(x) for x in ins + outs) + P * sum(rnd(x) for x in heads) + P * rnd(lse)
        if bwd:
            want += rnd(L.ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, det))
        assert L.ulysses_host_pipeline_scratch_bytes(N, P, H, H_kv, d, bwd, det) == want, (bwd, det)
    assert L.ulysses_host_pipeline_scratch_bytes(N, P, H, H_kv, 96, 1, 0) == 0
    assert L.ulysses_host_pipeline_scratch_bytes(N + 1, P, H, H_kv, d, 1, 0) == 0
    h = ctypes.c_void_p()
    n = L.ulysses_host_pipeline_scratch_bytes(N, P, H, H_kv, d, 1, 0)
    assert L.ulysses_host_pipeline_create(N, P, H, H_kv, d, 1, 0, None, n, ctypes.byref(h)) == 1
    assert L.ulysses_host_pipeline_create(N, P, H, H_kv, d, 1, 0, 1 << 40, n - 1, ctypes.byref(h)) == 1
    assert L.ulysses_host_pipeline_create(N, P, H, H_kv, d, 1, 0, (1 << 40) + 16, n, ctypes.byref(h)) == 1
    assert L.ulysses_host_pipeline_create(N, P, H, H_kv, 96, 1, 0, 1 << 40, n, ctypes.byref(h)) == 2
    assert L.ulysses_host_pipeline_create(N, P, H, H_kv, d, 1, 0, 1 << 40, n, None) == 1
    assert not h.value
    assert L.ulysses_host_pipeline_submit(None, None, None, None, None, None, None, None, None, None, 0, 0.0,
                                          None, None) == 1
    assert L.ulysses_host_pipeline_synchronize(None) == 1
    assert L.ulysses_host_pipeline_destroy(None) == 0


def test_seq_backward_workspace_size(L):
    """The sequence-layout backward's larger workspace (room to stage Q and dO
    in head shards) exists only for the one-pass mode: 2 * P * N * (H/P) * d
    bf16 more than the plain backward's; otherwise the two sizes agree."""
    N, P, H, H_kv = 8192, 4, 32, 8
    for d, det in ((128, 0), (128, 1), (64, 0)):
        base = L.ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, det)
        seq = L.ulysses_attn_bwd_seq_workspace_size(N, P, H, H_kv, d, det)
        extra = 2 * P * N * (H // P) * d * 2 if (d == 128 and det == 0) else 0
        assert base > 0 and seq == base + extra, (d, det)
    assert L.ulysses_attn_bwd_seq_workspace_size(N, P, H, H_kv, 96, 0) == 0
