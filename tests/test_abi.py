"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point its header declares, builds the random table bit for bit
like the oracle's independent generator, and rejects invalid arguments on
the host before touching the device."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from block_sparse_long_bwd_b200 import binding as bb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f)
           for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def _declared():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(bb_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = bb.lib()
    names = _declared()
    assert "bb_attn_fwd" in names and "bb_attn_bwd" in names
    for name in names:
        assert hasattr(lib, name), name
    assert bb.bb_abi_version() == 5


@pytest.mark.parametrize("seed,H,nb,r", [
    (0, 12, 64, 3), (0, 16, 64, 3), (0, 12, 256, 3), (0, 2, 16, 3),
    (123456789, 3, 32, 6), ((1 << 64) - 1, 2, 8, 6), (7, 4, 5, 1),
    (9, 1, 4, 3), (9, 1, 1, 2), (5, 12, 1024, 6), (2, 3, 33, 0),
])
def test_rand_table_bit_exact_vs_oracle(seed, H, nb, r):
    got = bb.bb_rand_attn_build(seed, H, nb, r).numpy()
    want = oracle.rand_table(seed, H, nb, r)
    assert got.dtype == np.int32
    assert np.array_equal(got, want)


@pytest.mark.parametrize("seed,H,nb,r,mx,last", [
    (0, 12, 16, 3, 64, 16), (3, 12, 32, 3, 64, 16), (11, 12, 64, 3, 64, 16),
    (5, 4, 40, 6, 41, 0), (7, 4, 33, 9, 0, 12), (2**64 - 1, 2, 8, 3, 8, 3),
    (1, 3, 1, 3, 5, 0), (1, 3, 3, 2, 64, 0)])
def test_rand_table_layer_options_bit_exact_vs_oracle(seed, H, nb, r, mx, last):
    got = bb.bb_rand_attn_build_ex(seed, H, nb, r, mx, last).numpy()
    want = oracle.rand_table(seed, H, nb, r, max_blocks=mx, last_block=last)
    assert np.array_equal(got, want)


def test_rand_table_layer_options_off_equal_the_base_call():
    assert np.array_equal(bb.bb_rand_attn_build_ex(4, 3, 48, 3, 0, 0).numpy(),
                          bb.bb_rand_attn_build(4, 3, 48, 3).numpy())
    lib = bb.lib()
    buf = (ctypes.c_int32 * 64)()
    assert lib.bb_rand_attn_build_ex(0, 1, 32, 2, 16, 0, buf) == -1  # mx < nb
    assert lib.bb_rand_attn_build_ex(0, 1, 32, 2, 0, -1, buf) == -1
    assert lib.bb_rand_attn_build_ex(0, 1, 32, 2, -1, 0, buf) == -1
    assert lib.bb_rand_attn_build_ex(0, 1, 32, 2, 64, 16, None) == -1
    assert lib.bb_rand_attn_build_ex(0, 0, 32, 2, 64, 16, None) == 0  # empty


def test_binding_table_options_in_tokens():
    """The binding's table helper takes the pages' options in tokens: a
    4096-token table with random blocks before token 1024, layer 7, used at
    L = 2048 with block 64."""
    got = bb.make_table(7, 12, 2048, 64, 3, max_rand_mask_length=4096,
                        last_idx=1024).numpy()
    assert np.array_equal(got, oracle.rand_table(7, 12, 32, 3, 64, 16))
    assert np.array_equal(bb.make_table(7, 12, 2048, 64, 3).numpy(),
                          oracle.rand_table(7, 12, 32, 3))
    with pytest.raises(bb.BBError):
        bb.make_table(7, 12, 2048, 64, 3, max_rand_mask_length=1024)


def test_wait_probe_rejects_bad_arguments_on_host():
    """Invalid arguments are refused before any launch (fake pointers)."""
    lib = bb.lib()
    good = 1 << 20
    assert lib.bb_debug_wait_probe(None, 256, 1, None) == -1
    assert lib.bb_debug_wait_probe(good + 4, 256, 1, None) == -1
    assert lib.bb_debug_wait_probe(good, 255, 1, None) == -1
    assert lib.bb_debug_wait_probe(good, 256, 2, None) == -1


def test_rand_table_errors():
    lib = bb.lib()
    assert lib.bb_rand_attn_build(0, -1, 4, 3, None) == -1
    assert lib.bb_rand_attn_build(0, 2, 4, 3, None) == -1
    assert lib.bb_rand_attn_build(0, 0, 4, 3, None) == 0   # empty table


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, 42):
        assert isinstance(bb.bb_status_str(code), str)


def _desc(**kw):
    base = dict(B=2, H=3, L=512, d=64, block_size=64, r=3, dtype=bb.BB_BF16)
    base.update(kw)
    return bb.make_desc(**base)


def test_workspace_size_and_validation():
    n0 = bb.bb_attn_workspace_size(_desc(), 0)
    n1 = bb.bb_attn_workspace_size(_desc(), 1)
    assert n0 > 0 and n1 > n0
    bad = [
        (dict(L=500), -1), (dict(B=0), -1), (dict(r=-1), -1),
        (dict(dtype=7), -1), (dict(d=128), -2), (dict(block_size=16), -2),
        (dict(r=33), -2), (dict(L=64 * 8193), -2),
        # dropout outside [0, 1), NaN, or a rate that rounds to 1 (256/256)
        (dict(dropout=1.0), -1), (dict(dropout=-0.1), -1),
        (dict(dropout=float("nan")), -1), (dict(dropout=255.6 / 256), -1),
        (dict(mask_queries=2), -1), (dict(mask_queries=-1), -1),
        (dict(grad_fp32=2), -1), (dict(grad_fp32=-1), -1),
    ]
    lib = bb.lib()
    for kw, code in bad:
        n = ctypes.c_size_t(0)
        got = lib.bb_attn_workspace_size(ctypes.byref(_desc(**kw)), 0,
                                         ctypes.byref(n))
        assert got == code, (kw, got)
    # fp32 gradient outputs change nothing in the workspace
    assert bb.bb_attn_workspace_size(_desc(grad_fp32=1), 1) == n1
    for rate in (0.1, 0.5, 255.4 / 256):  # valid rates, any seed
        assert bb.bb_attn_workspace_size(
            _desc(dropout=rate, dropout_seed=2**64 - 1), 1) == n1
    n = ctypes.c_size_t(0)
    assert lib.bb_attn_workspace_size(None, 0, ctypes.byref(n)) == -1
    assert lib.bb_attn_workspace_size(ctypes.byref(_desc()), 2,
                                      ctypes.byref(n)) == -1


def _keep_slots(nb, r):
    # One slot per attended (query block, key block) pair: nb for each
    # global query block, 5 + r for each middle one.
    return 1 if nb == 1 else 2 * nb + (nb - 2) * (5 + r)


@pytest.mark.parametrize("L,bs,r", [
    (512, 64, 3), (4096, 64, 3), (1024, 32, 6), (2048, 128, 0), (64, 64, 3),
    (128, 64, 2), (4096 * 4, 64, 3),
])
def test_dropout_bits_size(L, bs, r):
    nb = L // bs
    d = _desc(L=L, block_size=bs, r=r, dropout=0.1)
    want = 2 * 3 * _keep_slots(nb, r) * bs * bs // 8
    assert bb.bb_attn_dropout_bits_size(d) == want
    # room for every attended pair of a drawn table
    table = oracle.rand_table(0, 3, nb, r)
    for h in range(3):
        assert oracle.pair_count(nb, table[h]) <= _keep_slots(nb, r)
    # no dropout (or a rate that rounds to 0): no buffer
    assert bb.bb_attn_dropout_bits_size(_desc(L=L, block_size=bs, r=r)) == 0
    assert bb.bb_attn_dropout_bits_size(
        _desc(L=L, block_size=bs, r=r, dropout=0.001)) == 0


def test_dropout_bits_pointer_validation():
    lib = bb.lib()
    d = _desc(dropout=0.1)
    d.dropout_bits = 8  # misaligned (never dereferenced)
    n = ctypes.c_size_t(0)
    assert lib.bb_attn_dropout_bits_size(ctypes.byref(d), ctypes.byref(n)) == -1
    assert lib.bb_attn_workspace_size(ctypes.byref(d), 0, ctypes.byref(n)) == -1
    d.dropout_bits = 1 << 20  # aligned: accepted, sizes unchanged
    assert bb.bb_attn_workspace_size(d, 0) == bb.bb_attn_workspace_size(
        _desc(dropout=0.1), 0)
    assert lib.bb_attn_dropout_bits_size(None, ctypes.byref(n)) == -1
    assert lib.bb_attn_dropout_bits_size(ctypes.byref(d), None) == -1


def test_compute_calls_reject_bad_arguments_on_host():
    """Fake (never dereferenced) pointers: every case fails validation before
    any CUDA call is made."""
    lib = bb.lib()
    d = _desc()
    good = 1 << 20  # 16-byte aligned fake address
    ws_n = bb.bb_attn_workspace_size(d, 0)
    args = [good] * 8
    # NULL q
    assert lib.bb_attn_fwd(ctypes.byref(d), None, *args[1:], ws_n, None) == -1
    # misaligned v
    a = list(args)
    a[2] = good + 2
    assert lib.bb_attn_fwd(ctypes.byref(d), *a, ws_n, None) == -1
    # workspace too small / missing
    assert lib.bb_attn_fwd(ctypes.byref(d), *args, ws_n - 1, None) == -4
    a = list(args)
    a[7] = None
    assert lib.bb_attn_fwd(ctypes.byref(d), *a, ws_n, None) == -4
    # unsupported desc
    assert lib.bb_attn_fwd(ctypes.byref(_desc(d=32)), *args, ws_n, None) == -2
    # r > 0 with no table
    a = list(args)
    a[4] = None
    assert lib.bb_attn_fwd(ctypes.byref(d), *a, ws_n, None) == -1
    ws_b = bb.bb_attn_workspace_size(d, 1)
    bargs = [good] * 12
    assert lib.bb_attn_bwd(ctypes.byref(d), *bargs, ws_b - 16, None) == -4
    b = list(bargs)
    b[9] = None  # dk
    assert lib.bb_attn_bwd(ctypes.byref(d), *b, ws_b, None) == -1
    assert lib.bb_attn_bwd(None, *bargs, ws_b, None) == -1


def _names(desc, pass_):
    return [bb.bb_attn_launch_name(desc, pass_, i)
            for i in range(bb.bb_attn_launch_count(desc, pass_))]


def test_launch_lists_follow_the_dispatch():
    """The launch list a pass reports (what event timing is keyed by): the
    tensor-core path for bf16 shapes (backward plans in one launch while a
    head's transposed adjacency fits in shared memory), one dK/dV launch
    below 16384 tokens and two from there (global key blocks with the hi/lo
    split on their own), merge launches only where global rows are split
    into chunks, the CUDA-core path for fp32."""
    import torch
    short = bb.make_desc(2, 4, 4096, 64, 64, 3, torch.bfloat16)
    assert _names(short, 0) == ["plan", "tc_fwd", "fwd_combine"]
    assert _names(short, 1) == ["plan", "tc_dq", "tc_dkdv", "bwd_finish"]
    # dropout and the query mask change the kernels' variants, not the list
    opt = bb.make_desc(2, 4, 4096, 64, 64, 3, torch.bfloat16, dropout=0.1,
                       dropout_seed=3, mask_queries=1)
    assert _names(opt, 0) == _names(short, 0)
    assert _names(opt, 1) == _names(short, 1)
    for bs in (32, 64, 128):
        long_ = bb.make_desc(1, 2, 16384, 64, bs, 3, torch.bfloat16)
        assert _names(long_, 0) == ["plan", "tc_fwd", "fwd_combine"], bs
        assert _names(long_, 1) == ["plan", "tc_dq", "tc_dkdv", "tc_dkdv", "bwd_finish"], bs
    # Enough work that a global row's 64 tiles run as one item: no chunk
    # partials, so no merge launches (the BigBird-large and -base shapes).
    for B, H in ((4, 16), (8, 12)):
        for bs in (32, 64, 128):
            whole = bb.make_desc(B, H, 4096, 64, bs, 3, torch.bfloat16)
            assert _names(whole, 0) == ["plan", "tc_fwd"], (B, H, bs)
            assert _names(whole, 1) == ["plan", "tc_dq", "tc_dkdv"], (B, H, bs)
    f32 = bb.make_desc(1, 2, 1024, 64, 64, 3, torch.float32)
    assert _names(f32, 0) == ["simt_fwd"]
    assert _names(f32, 1) == ["bwd_pre", "csr_build", "simt_dq", "simt_dkdv"]
    # bf16 shapes outside the tensor-core bounds: L not a multiple of 64,
    # r past the planner bound (27 at block 64, 11 at blocks 32 and 128).
    for B, H, L, bs, r in ((1, 2, 96, 32, 2), (1, 1, 1024, 64, 28),
                           (1, 1, 1024, 32, 12), (1, 1, 1024, 128, 12)):
        d_ = bb.make_desc(B, H, L, 64, bs, r, torch.bfloat16)
        assert _names(d_, 0) == ["simt_fwd"], (L, bs, r)
        assert _names(d_, 1) == ["bwd_pre", "csr_build", "simt_dq",
                                 "simt_dkdv"], (L, bs, r)
    for bs, r in ((64, 27), (32, 11), (128, 11)):  # the largest on the tensor cores
        d_ = bb.make_desc(1, 1, 1024, 64, bs, r, torch.bfloat16)
        assert _names(d_, 0) == ["plan", "tc_fwd", "fwd_combine"], (bs, r)
    # A head's adjacency too large for shared memory: CSR built separately.
    huge = bb.make_desc(1, 1, 131072, 64, 32, 3, torch.bfloat16)
    assert _names(huge, 1)[:2] == ["csr_build", "plan"]


def test_host_calls_are_reentrant_across_threads():
    """The host-only entry points called concurrently from several threads
    (ctypes releases the GIL during the call) give the single-thread
    results: the table builder, workspace sizing and the launch-name
    lookup (thread-local name buffer)."""
    import threading

    import torch
    want_t = bb.bb_rand_attn_build_ex(123, 4, 256, 6, 300, 100).numpy()
    d_short = bb.make_desc(2, 4, 4096, 64, 64, 3, torch.bfloat16)
    d_f32 = bb.make_desc(1, 2, 1024, 64, 64, 3, torch.float32)
    want_n = (_names(d_short, 1), _names(d_f32, 1))
    want_w = bb.bb_attn_workspace_size(d_short, 1)
    errors = []

    def worker(i):
        try:
            for _ in range(20):
                t = bb.bb_rand_attn_build_ex(123, 4, 256, 6, 300, 100).numpy()
                assert np.array_equal(t, want_t)
                d = d_short if i % 2 else d_f32
                names = [bb.bb_attn_launch_name(d, 1, k)
                         for k in range(bb.bb_attn_launch_count(d, 1))]
                assert names == want_n[0 if i % 2 else 1]
                assert bb.bb_attn_workspace_size(d_short, 1) == want_w
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors


def test_projection_argument_checks_without_a_gpu():
    """The projection entry points validate before touching any pointer or
    calling CUDA: NULL or misaligned pointers, sizes the tiles do not cover,
    a missing or short workspace."""
    lib = bb.lib()
    P = 1 << 20  # a fake 16-byte aligned address, never dereferenced
    ws = P
    # NULL input / misaligned pointer
    assert lib.bb_qkv_proj(1, 128, 768, 12, None, P, None, P, P, P, ws, 256, None) == -1
    assert lib.bb_qkv_proj(1, 128, 768, 12, P + 2, P, None, P, P, P, ws, 256, None) == -1
    assert lib.bb_out_proj(1, 128, 12, 768, None, P, None, P, ws, 256, None) == -1
    # shapes: L % 128, hidden % 64, H % 4 (QKV); hidden % 256 (output)
    assert lib.bb_qkv_proj(1, 100, 768, 12, P, P, None, P, P, P, ws, 256, None) == -2
    assert lib.bb_qkv_proj(1, 128, 770, 12, P, P, None, P, P, P, ws, 256, None) == -2
    assert lib.bb_qkv_proj(1, 128, 768, 6, P, P, None, P, P, P, ws, 256, None) == -2
    assert lib.bb_out_proj(1, 128, 12, 640, P, P, None, P, ws, 256, None) == -2
    assert lib.bb_qkv_proj(0, 128, 768, 12, P, P, None, P, P, P, ws, 256, None) == -1
    # workspace
    assert lib.bb_qkv_proj(1, 128, 768, 12, P, P, None, P, P, P, None, 256, None) == -4
    assert lib.bb_out_proj(1, 128, 12, 768, P, P, None, P, ws, 64, None) == -4
