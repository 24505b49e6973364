"""The C ABI on the CPU host: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch.

The argument checks below pass fake (never dereferenced) device pointers, so
they only run where no GPU is present: a check that wrongly let one through
must not reach a real device.
"""
import ctypes
import os
import re

import pytest
import torch

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "ulysses.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ulysses_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import ulysses_head_attention_b200 as uly
    names = header_functions()
    assert names == sorted(uly.EXPORTS)
    for n in names:
        assert hasattr(uly.lib, n), n


def test_status_strings():
    import ulysses_head_attention_b200 as uly
    for code in range(7):
        assert uly.status_string(code) and uly.status_string(code) != "unknown status"
    assert uly.status_string(99) == "unknown status"


no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake-pointer checks run only without a GPU")
F = 0x100000          # fake, 256-byte aligned "device" addresses, never dereferenced
INVALID, UNSUPPORTED, CUDA, WORKSPACE = 1, 2, 3, 4


@no_gpu
@pytest.mark.parametrize("args,want", [
    ((F, F + 1 << 30, 1, 100, 32, 128, 8), INVALID),        # n % P != 0 (padding rule)
    ((F, F + 1 << 30, 1, 64, 12, 128, 8), INVALID),         # H % P != 0 (head rule)
    ((F, F + 1 << 30, 1, 64, 32, 128, 0), INVALID),         # P < 1
    ((0, F + 1 << 30, 1, 64, 32, 128, 4), INVALID),         # null input
    ((F + 8, F + 1 << 30, 1, 64, 32, 128, 4), INVALID),     # misaligned
    ((F, F + 1024, 1, 64, 32, 128, 4), INVALID),            # overlapping buffers
    ((F, F + (1 << 30), 1, 0, 32, 128, 4), INVALID),        # empty sequence
    ((F, F + (1 << 30), 0, 64, 32, 128, 4), INVALID),       # no batch rows
    ((F, F + (1 << 30), 1, 64, 32, 0, 4), INVALID),         # empty head dimension
])
def test_relayout_rejects(args, want):
    import ulysses_head_attention_b200 as uly
    src, dst, b, n, H, d, P = args
    for fn in (uly.lib.ulysses_seq_to_head, uly.lib.ulysses_head_to_seq):
        assert fn(src, dst, b, n, H, d, P, 0, None) == want


@no_gpu
def test_relayout_rejects_unknown_dtype():
    import ulysses_head_attention_b200 as uly
    for fn in (uly.lib.ulysses_seq_to_head, uly.lib.ulysses_head_to_seq, uly.lib.ulysses_kv_seq_to_head,
               uly.lib.ulysses_kv_head_to_seq):
        assert fn(F, F + (1 << 30), 1, 64, 32, 128, 4, 7, None) == INVALID


def shape(b=1, n=1024, hq=32, hkv=8, d=128, P=4):
    import ulysses_head_attention_b200 as uly
    return uly.make_shape(b, n, hq, hkv, d, P)


@no_gpu
@pytest.mark.parametrize("kw,rank,want", [
    (dict(n=1000, P=16), -1, INVALID),       # n % P
    (dict(hkv=6, P=4, hq=24), -1, INVALID),  # H_kv neither a multiple nor a divisor of P
    (dict(hkv=3, P=4, hq=12), -1, INVALID),  # H_kv < P but does not divide P
    (dict(hq=12, hkv=8, P=4), -1, INVALID),  # H_q % H_kv
    (dict(P=0), -1, INVALID),
    ({}, 4, INVALID),                        # rank out of range
    ({}, -2, INVALID),
    (dict(d=96), -1, UNSUPPORTED),           # head dim not implemented
    (dict(n=0), -1, INVALID),                # empty sequence
    (dict(b=0), -1, INVALID),                # no batch rows
    (dict(hq=0), -1, INVALID),
    (dict(n=1 << 31, P=4), -1, UNSUPPORTED),  # beyond the int32 TMA coordinates
])
def test_attention_rejects_shapes(kw, rank, want):
    import ulysses_head_attention_b200 as uly
    s = shape(**kw)
    G = 1 << 30
    ws_bytes = 1 << 24
    st = uly.lib.ulysses_attn_fwd(F, F + G, F + 2 * G, F + 3 * G, ctypes.byref(s), rank, 0.0, F + 4 * G, 1,
                                  F + 5 * G, F + 6 * G, ws_bytes, None)
    assert st == want
    st = uly.lib.ulysses_attn_bwd(F, F + G, F + 2 * G, F + 3 * G, 1, F + 4 * G, F + 5 * G, F + 6 * G,
                                  ctypes.byref(s), rank, 0.0, F + 7 * G, F + 8 * G, F + 9 * G, 1,
                                  F + 10 * G, ws_bytes, None)
    assert st == want


@no_gpu
def test_attention_rejects_workspace():
    import ulysses_head_attention_b200 as uly
    s = shape()
    need = uly.ulysses_attn_fwd_workspace(s)
    assert need > 0
    G = 1 << 30
    for ws, nbytes in ((0, need), (F + 6 * G, need - 1), (F + 6 * G + 16, need)):
        st = uly.lib.ulysses_attn_fwd(F, F + G, F + 2 * G, F + 3 * G, ctypes.byref(s), -1, 0.0, F + 4 * G, 1,
                                      F + 5 * G, ws, nbytes, None)
        assert st == WORKSPACE


def test_workspace_queries_reject_bad_shapes():
    import ulysses_head_attention_b200 as uly
    assert uly.ulysses_attn_fwd_workspace(shape(n=1001)) == 0
    assert uly.ulysses_attn_bwd_workspace(shape(P=3), 1) == 0
    assert uly.ulysses_attn_fwd_workspace(shape()) >= 256 + 2 * 4 * 1024


def test_timed_backward_rejects_missing_events():
    """The event array is checked before anything else: null array or null handle."""
    import ulysses_head_attention_b200 as uly
    s = shape()
    G = 1 << 30
    args = (F, F + G, F + 2 * G, F + 3 * G, 1, F + 4 * G, F + 5 * G, F + 6 * G, ctypes.byref(s), -1, 0.0,
            F + 7 * G, F + 8 * G, F + 9 * G, 1, F + 10 * G, 1 << 24, None)
    assert uly.lib.ulysses_attn_bwd_timed(*args, None) == INVALID
    events = (ctypes.c_void_p * 5)(1, 2, 0, 4, 5)
    assert uly.lib.ulysses_attn_bwd_timed(*args, events) == INVALID


@no_gpu
@pytest.mark.parametrize("b,n,P,want", [
    (1, 64, 0, INVALID),        # P < 1
    (1, 64, 2048, INVALID),     # P > 1024
    (1, 100, 8, INVALID),       # n % P
    (0, 64, 4, INVALID),        # b < 1
])
def test_loss_aggregate_rejects_shapes(b, n, P, want):
    import ulysses_head_attention_b200 as uly
    G = 1 << 30
    st = uly.lib.ulysses_sp_loss_aggregate(F, F + G, b, n, P, -100, F + 2 * G, F + 3 * G, F + 4 * G, None)
    assert st == want


@no_gpu
def test_loss_aggregate_rejects_pointers():
    import ulysses_head_attention_b200 as uly
    G = 1 << 30
    ok = [F, F + G, F + 2 * G, F + 3 * G, F + 4 * G]
    for i, bad in ((0, 0), (1, F + G + 4), (3, F + 3 * G + 4), (4, F + G)):   # null, misaligned, overlap
        args = list(ok)
        args[i] = bad
        st = uly.lib.ulysses_sp_loss_aggregate(args[0], args[1], 1, 64, 4, -100, args[2], args[3], args[4], None)
        assert st == INVALID


@no_gpu
@pytest.mark.parametrize("H,P,want", [
    (3, 4, INVALID),      # neither a multiple nor a divisor of P
    (6, 4, INVALID),
    (2, 0, INVALID),
])
def test_kv_relayout_rejects(H, P, want):
    import ulysses_head_attention_b200 as uly
    for fn in (uly.lib.ulysses_kv_seq_to_head, uly.lib.ulysses_kv_head_to_seq):
        assert fn(F, F + (1 << 30), 1, 64, H, 128, P, 0, None) == want


@no_gpu
def test_kv_relayout_rejects_unsupported_row_and_overlap():
    import ulysses_head_attention_b200 as uly
    for fn in (uly.lib.ulysses_kv_seq_to_head, uly.lib.ulysses_kv_head_to_seq):
        assert fn(F, F + (1 << 30), 1, 64, 2, 4, 4, 0, None) == UNSUPPORTED      # d * 2 bytes not a multiple of 16
        assert fn(F, F + 1024, 1, 64, 2, 128, 4, 0, None) == INVALID            # overlapping buffers


@no_gpu
def test_ring_entries_reject_bad_ranges_and_parts():
    import ulysses_head_attention_b200 as uly
    s = shape()
    G = 1 << 30
    for lo, hi in ((-1, 10), (10, 10), (0, 1025), (20, 5)):
        st = uly.lib.ulysses_attn_fwd_kv_range(F, F + G, F + 2 * G, F + 3 * G, ctypes.byref(s), -1, 0.0, lo, hi,
                                               F + 4 * G, 1, F + 5 * G, F + 6 * G, 1 << 24, None)
        assert st == INVALID
        st = uly.lib.ulysses_attn_bwd_kv_range(F, F + G, F + 2 * G, F + 3 * G, 1, F + 4 * G, F + 5 * G, F + 6 * G,
                                               ctypes.byref(s), -1, 0.0, lo, hi, F + 7 * G, F + 8 * G, F + 9 * G, 1,
                                               F + 10 * G, 1 << 26, None)
        assert st == INVALID
    for nparts in (0, 33):
        assert uly.lib.ulysses_attn_lse_merge(F, F + G, nparts, ctypes.byref(s), F + 2 * G, 1, F + 3 * G,
                                              None) == INVALID
    assert uly.lib.ulysses_attn_lse_merge(F, F + G, 2, ctypes.byref(shape(d=96)), F + 2 * G, 1, F + 3 * G,
                                          None) == UNSUPPORTED


@no_gpu
def test_transpose_rejects():
    import ulysses_head_attention_b200 as uly
    G = 1 << 30
    assert uly.lib.ulysses_transpose_runs(0, F, 2, 2, 16, None) == INVALID
    assert uly.lib.ulysses_transpose_runs(F, F + G, 0, 2, 16, None) == INVALID
    assert uly.lib.ulysses_transpose_runs(F, F + G, 2, 2, 0, None) == INVALID
    assert uly.lib.ulysses_transpose_runs(F, F + 32, 2, 2, 16, None) == INVALID   # overlap


def _attn_tensors(P=2, b=1, n=8, hq=2, hkv=1, d=4, o=torch.float32, g=torch.float32):
    """Host tensors with the layouts of one attention call (never launched)."""
    bf = torch.bfloat16
    return dict(q_head=torch.zeros(P, b, n, hq, d, dtype=bf), k_head=torch.zeros(P, b, n, hkv, d, dtype=bf),
                v_head=torch.zeros(P, b, n, hkv, d, dtype=bf), position_ids=torch.zeros(b, n, dtype=torch.int64),
                o_head=torch.zeros(P, b, n, hq, d, dtype=o), lse=torch.zeros(P, b, hq, n),
                do_head=torch.zeros(P, b, n, hq, d, dtype=bf), dq_head=torch.zeros(P, b, n, hq, d, dtype=g),
                dk_head=torch.zeros(P, b, n, hkv, d, dtype=g), dv_head=torch.zeros(P, b, n, hkv, d, dtype=g),
                ws=torch.zeros(256, dtype=torch.uint8))


FWD_ARGS = ("q_head", "k_head", "v_head", "position_ids", "o_head", "lse", "ws")
BWD_ARGS = ("q_head", "k_head", "v_head", "o_head", "lse", "do_head", "position_ids", "dq_head", "dk_head",
            "dv_head", "ws")


@pytest.mark.parametrize("name,bad,exc", [
    ("v_head", torch.zeros(2, 1, 8, 2, 4, dtype=torch.bfloat16), ValueError),   # v heads differ from k
    ("position_ids", torch.zeros(8, dtype=torch.int64), ValueError),            # not [b][n]
    ("position_ids", torch.zeros(1, 8, dtype=torch.int32), TypeError),
    ("o_head", torch.zeros(2, 1, 4, 2, 4), ValueError),                         # too few rows
    ("o_head", torch.zeros(2, 1, 8, 2, 4, dtype=torch.float16), TypeError),
    ("lse", torch.zeros(2, 1, 8, 2), ValueError),                               # [P][b][n][h], transposed
    ("q_head", torch.zeros(2, 1, 8, 2, 4), TypeError),                          # fp32 q
])
def test_binding_checks_forward_layouts_before_launch(name, bad, exc):
    """A mis-sized or mistyped tensor is refused by the binding, before any
    pointer reaches the library (these are host tensors: nothing launches)."""
    import ulysses_head_attention_b200 as uly
    t = _attn_tensors()
    t[name] = bad
    args = [t[a] for a in FWD_ARGS]
    for fn in (uly.ulysses_attn_fwd, lambda *a: uly.ulysses_attn_fwd_kv_range(*a, k_lo=0, k_hi=8)):
        with pytest.raises(exc, match=name):
            fn(*args)
    with pytest.raises(exc, match=name):
        uly.ulysses_attn_fwd_noalloc(*args[:-1])


@pytest.mark.parametrize("name,bad,exc", [
    ("do_head", torch.zeros(2, 1, 8, 2, 4), TypeError),                          # dO must be bf16
    ("dq_head", torch.zeros(2, 1, 8, 1, 4), ValueError),
    ("dk_head", torch.zeros(2, 1, 8, 1, 4, dtype=torch.bfloat16), TypeError),    # dtype differs from dq
    ("dv_head", torch.zeros(2, 1, 8, 2, 4), ValueError),
])
def test_binding_checks_backward_layouts_before_launch(name, bad, exc):
    import ulysses_head_attention_b200 as uly
    t = _attn_tensors()
    t[name] = bad
    args = [t[a] for a in BWD_ARGS]
    with pytest.raises(exc, match=name):
        uly.ulysses_attn_bwd(*args)
    with pytest.raises(exc, match=name):
        uly.ulysses_attn_bwd_kv_range(*args, k_lo=0, k_hi=8)
    with pytest.raises(exc, match=name):
        uly.ulysses_attn_bwd_timed(*args, events=[None] * 5)


def test_binding_refuses_host_tensors():
    """Well-formed layouts on the host still never reach the library."""
    import ulysses_head_attention_b200 as uly
    t = _attn_tensors()
    with pytest.raises(ValueError, match="CUDA tensor"):
        uly.ulysses_attn_fwd(*[t[a] for a in FWD_ARGS])
    with pytest.raises(ValueError, match="CUDA tensor"):
        uly.ulysses_attn_bwd(*[t[a] for a in BWD_ARGS])


def test_binding_checks_merge_layouts():
    import ulysses_head_attention_b200 as uly
    o_parts, lse_parts = torch.zeros(3, 2, 1, 8, 2, 4), torch.zeros(3, 2, 1, 2, 8)
    o_head, lse = torch.zeros(2, 1, 8, 2, 4), torch.zeros(2, 1, 2, 8)
    with pytest.raises(ValueError, match="lse_parts"):
        uly.ulysses_attn_lse_merge(o_parts, lse_parts[:2], o_head, lse, h_kv=2)
    with pytest.raises(ValueError, match="lse"):
        uly.ulysses_attn_lse_merge(o_parts, lse_parts, o_head, lse[:, :, :1], h_kv=2)
    with pytest.raises(ValueError, match="o_head"):
        uly.ulysses_attn_lse_merge(o_parts, lse_parts, o_head[:1], lse, h_kv=2)
    with pytest.raises(ValueError, match="CUDA tensor"):
        uly.ulysses_attn_lse_merge(o_parts, lse_parts, o_head, lse, h_kv=2)


@no_gpu
def test_noalloc_forward_refuses_before_touching_the_device():
    """Bad shapes and shapes beyond the fixed scratch (b * n > 524288 tokens)
    are refused on the host, before the scratch lookup or any launch."""
    import ulysses_head_attention_b200 as uly
    G = 1 << 30

    def call(s, rank=-1):
        return uly.lib.ulysses_attn_fwd_noalloc(F, F + G, F + 2 * G, F + 3 * G, ctypes.byref(s), rank, 0.0,
                                                F + 4 * G, 1, F + 5 * G, None)
    assert call(shape(n=1000, P=16)) == INVALID
    assert call(shape(b=1, n=1 << 20)) == WORKSPACE
    assert call(shape(b=2, n=1 << 19)) == WORKSPACE
    # the largest accepted size passes the size check and stops at the device
    # lookup, which has no device to find here
    assert call(shape(b=1, n=1 << 19)) == CUDA


@no_gpu
def test_noalloc_status_refuses_a_null_code():
    import ulysses_head_attention_b200 as uly
    assert uly.lib.ulysses_attn_fwd_noalloc_status(None, None) == INVALID
    # a valid request stops at the device lookup, which has no device to find here
    code = ctypes.c_int32(-1)
    assert uly.lib.ulysses_attn_fwd_noalloc_status(None, ctypes.byref(code)) == CUDA


@no_gpu
def test_selftest_wait_timeout_rejects():
    import ulysses_head_attention_b200 as uly
    f = uly.lib.ulysses_selftest_wait_timeout
    assert f(None, 4096, 1000000, None) == WORKSPACE                 # no workspace
    assert f(F + 16, 4096, 1000000, None) == WORKSPACE               # not 256-byte aligned
    assert f(F, 1024, 1000000, None) == WORKSPACE                    # below 256 + 1024 bytes
    assert f(F, 4096, 999, None) == INVALID                          # limit below 1 us
    assert f(F, 4096, 5000000001, None) == INVALID                   # limit above 5 s


@no_gpu
def test_push_and_wait_reject():
    import ulysses_head_attention_b200 as uly
    P = 4
    dst = (ctypes.c_void_p * P)(*[F + (i + 1) * (1 << 30) for i in range(P)])
    flg = (ctypes.c_void_p * P)(*[F + (i + 9) * (1 << 30) for i in range(P)])
    ws = F + (20 << 30)
    push = uly.lib.ulysses_seq_to_head_push
    ok_args = (F, dst, flg, 0, 1, 4096, 32, 128, P, 0, 1, ws, 4096, None)

    def call(**kw):
        names = ("src", "dst", "flags", "rank", "b", "n", "H", "d", "P", "dt", "epoch", "ws", "ws_bytes", "stream")
        a = dict(zip(names, ok_args))
        a.update(kw)
        return push(*[a[k] for k in names])

    assert call(rank=4) == INVALID                      # rank outside [0, P)
    assert call(rank=-1) == INVALID
    assert call(n=4095) == INVALID                      # n % P
    assert call(H=30) == INVALID                        # H % P
    assert call(epoch=0) == INVALID                     # 0 means "nothing yet"
    assert call(P=65, rank=0) == INVALID                # more ranks than the kernel carries
    assert call(ws=None) == WORKSPACE
    assert call(ws_bytes=8) == WORKSPACE                # below 4 P bytes
    assert call(src=F + 8) == INVALID                   # misaligned source
    assert call(src=F + (1 << 30)) == INVALID           # source overlaps this rank's own destination
    assert call(d=4, dt=0, H=4) == UNSUPPORTED          # a run of 2 bytes: not a 16-byte multiple
    bad = (ctypes.c_void_p * P)(*([0] + [F] * (P - 1)))
    assert call(dst=bad) == INVALID                     # a null destination
    wait = uly.lib.ulysses_wait_flags
    assert wait(F, 0, 1, 10**6, ws, None) == INVALID    # no flags
    assert wait(F, 4, 0, 10**6, ws, None) == INVALID    # epoch 0
    assert wait(F, 4, 1, 10, ws, None) == INVALID       # limit below 1 us
    assert wait(F, 4, 1, 10**6, None, None) == WORKSPACE
    assert uly.lib.ulysses_ipc_handle(None, None) == INVALID
    assert uly.lib.ulysses_ipc_open(None, None) == INVALID
    assert uly.lib.ulysses_ipc_close(None) == INVALID


def test_release_build_has_no_bounds_checks():
    import ulysses_head_attention_b200 as uly
    code = ctypes.c_int32(-1)
    if uly.DEBUG_BUILD:
        pytest.skip("the debug build is loaded")
    assert uly.lib.ulysses_debug_status(None, ctypes.byref(code)) == UNSUPPORTED and code.value == 0


def test_debug_build_exports_the_same_symbols():
    """libulysses_debug.so (built with ULY_DEBUG_BOUNDS) loads and exports what the header declares."""
    lib = os.path.join(ROOT, "ulysses_head_attention_b200", "libulysses_debug.so")
    if not os.path.exists(lib):
        pytest.fail("libulysses_debug.so is missing: build it with `python ulysses_head_attention_b200/build.py --debug`")
    d = ctypes.CDLL(lib)
    for n in header_functions():
        assert hasattr(d, n), n


@no_gpu
def test_layer_step_host_rejects():
    import ulysses_head_attention_b200 as uly
    f = uly.lib.ulysses_layer_step_host
    s = shape()
    need = uly.lib.ulysses_layer_step_host_bytes(ctypes.byref(s))
    assert need > 0 and uly.lib.ulysses_layer_step_host_bytes(ctypes.byref(shape(n=1001))) == 0
    ev = (ctypes.c_void_p * 3)(F, F + 64, F + 128)
    host = [F + (i + 1) * (1 << 30) for i in range(9)]

    def call(dev=F + (20 << 30), dev_bytes=need, events=ev, sh=s):
        return f(*host[:5], ctypes.byref(sh), 0.0, *host[5:], dev, dev_bytes, None, None, None, events)
    assert call(dev_bytes=need - 1) == WORKSPACE            # device buffer too small
    assert call(dev=F + (20 << 30) + 16) == WORKSPACE       # not 256-byte aligned
    assert call(events=None) == INVALID                      # no ordering events
    assert call(events=(ctypes.c_void_p * 3)(F, 0, F)) == INVALID
    assert call(sh=shape(n=1001)) == INVALID                 # n % P


@no_gpu
def test_block_calls_and_accumulate_reject():
    import ulysses_head_attention_b200 as uly
    G = 1 << 30
    s = shape(b=1, n=4096, hq=8, hkv=2, d=128, P=1)
    ws = uly.lib.ulysses_attn_fwd_workspace(ctypes.byref(s))
    fb = uly.lib.ulysses_attn_fwd_block

    def fwd(q_base, q_rows, k_base, k_rows):
        return fb(F, F + G, F + 2 * G, F + 3 * G, ctypes.byref(s), q_base, q_rows, k_base, k_rows, 0.0,
                  F + 4 * G, 1, F + 5 * G, F + 6 * G, ws, None)
    assert fwd(64, 128, 0, 128) == INVALID         # query block off a tile edge
    assert fwd(0, 128, 100, 128) == INVALID        # key block off a tile edge
    assert fwd(4096, 128, 0, 128) == INVALID       # query block past the sequence
    assert fwd(0, 128, 3968, 256) == INVALID       # key block past the sequence
    assert fwd(0, 0, 0, 128) == INVALID            # empty block
    acc = uly.lib.ulysses_accumulate
    assert acc(F, F + G, 6, None) == INVALID       # not a multiple of 4
    assert acc(F, F + 64, 1024, None) == INVALID   # overlapping, not identical
    assert acc(F + 4, F + G, 8, None) == INVALID   # misaligned

