"""The C-ABI library loads without a GPU, exports every symbol its header declares,
and rejects bad arguments on the host (no device work is launched)."""
import ctypes
import math
import os
import re

import pytest

from free_block_sparse_mean_b200 import _lib
from free_block_sparse_mean_b200._lib import SaShape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_attn.h")


@pytest.fixture(scope="module")
def lib():
    from free_block_sparse_mean_b200 import build
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sparse_attn_\w+)\s*\(", src)))


def test_header_matches_binding_list():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(6):
        s = lib.sparse_attn_status_string(code).decode()
        assert s.startswith(_lib.STATUS_NAMES[code])
    assert lib.sparse_attn_status_string(99).decode() == "unknown sa_status"


def test_workspace_and_tiles(lib):
    s = SaShape(1, 40, 75600, 128, 64)
    Nb = math.ceil(75600 / 64)
    al = lambda x: (x + 255) // 256 * 256

    def strips(BH, Nb):   # score strips of 128 rows of ceil(Nb/32)*32 floats, at most 64 MiB of them
        sb = 128 * ((Nb + 31) // 32 * 32) * 4
        return al(max(1, min(BH * math.ceil(Nb / 128), (64 << 20) // sb)) * sb)

    W = (Nb + 31) // 32
    # pooled Q and K, sort keys and bitsets (1182 blocks per head: the pairing keeps
    # its copy of the bitsets in shared memory), then the score strips
    expect = 2 * al(40 * Nb * 128 * 4) + al(40 * Nb * 8) + al(40 * Nb * W * 4) + strips(40, Nb)
    assert lib.sparse_attn_plan_workspace_size(s) == expect
    big = SaShape(1, 24, 118800, 128, 64)                         # 1857 blocks: a global copy too
    Nb2 = math.ceil(118800 / 64)
    W2 = (Nb2 + 31) // 32
    assert lib.sparse_attn_plan_workspace_size(big) == (2 * al(24 * Nb2 * 128 * 4) + al(24 * Nb2 * 8)
                                                        + 2 * al(24 * Nb2 * W2 * 4) + strips(24, Nb2))
    tiny = SaShape(1, 1, 1000, 64, 64)                            # one strip of one head
    Nb3 = math.ceil(1000 / 64)
    assert lib.sparse_attn_plan_workspace_size(tiny) == (2 * al(Nb3 * 64 * 4) + al(Nb3 * 8) + al(Nb3 * 4)
                                                         + al(128 * 32 * 4))
    assert lib.sparse_attn_num_tiles(s) == 40 * ((Nb + 1) // 2)
    assert lib.sparse_attn_num_tiles(SaShape(2, 3, 1, 64, 64)) == 6
    for bad in (SaShape(1, 1, 64, 96, 64), SaShape(1, 1, 64, 128, 32), SaShape(0, 1, 64, 128, 64),
                SaShape(1, 1, 0, 128, 64), SaShape(1, 1, 64 * 4097, 128, 64)):
        assert lib.sparse_attn_plan_workspace_size(bad) == 0
        assert lib.sparse_attn_num_tiles(bad) == 0


FAKE = ctypes.c_void_p(0x10000)       # never dereferenced: checks fail before any launch
FAKE_ODD = ctypes.c_void_p(0x10008)


def _plan(lib, Q=FAKE, K=FAKE, s=SaShape(1, 2, 128, 128, 64), tau=0.9, scale=0.1, mask=FAKE, count=FAKE,
          ws=FAKE, ws_bytes=1 << 30):
    return lib.sparse_attn_plan(Q, K, s, tau, scale, 0, mask, count, None, None, ws, ws_bytes, None)


def test_plan_argument_errors(lib):
    E = _lib
    assert _plan(lib, Q=None) == 1
    assert _plan(lib, mask=None) == 1
    assert _plan(lib, count=None) == 1
    assert _plan(lib, tau=0.0) == 1
    assert _plan(lib, tau=1.5) == 1
    assert _plan(lib, tau=float("nan")) == 1
    assert _plan(lib, scale=float("inf")) == 1
    assert _plan(lib, scale=-1.0) == 1
    assert _plan(lib, Q=FAKE_ODD) == 1
    assert _plan(lib, s=SaShape(1, 2, 128, 96, 64)) == 2
    assert _plan(lib, s=SaShape(1, 2, 128, 128, 128)) == 2
    assert _plan(lib, s=SaShape(1, 1, 64 * 5000, 128, 64)) == 2
    assert _plan(lib, s=SaShape(1, 2, 0, 128, 64)) == 1
    assert _plan(lib, ws=None) == 3
    assert _plan(lib, ws_bytes=10) == 3
    assert _plan(lib, ws=ctypes.c_void_p(0x10010)) == 3     # not 256-byte aligned


def _fwd(lib, Q=FAKE, K=FAKE, V=FAKE, s=SaShape(1, 2, 128, 128, 64), mask=FAKE, lam=-math.inf, scale=0.1,
         O=FAKE, stats=None):
    return lib.sparse_attn_fwd(Q, K, V, s, mask, None, lam, scale, 0, O, stats, None)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, V=None) == 1
    assert _fwd(lib, mask=None) == 1
    assert _fwd(lib, O=None) == 1
    assert _fwd(lib, lam=float("nan")) == 1
    assert _fwd(lib, lam=float("inf")) == 1
    assert _fwd(lib, scale=0.0) == 1
    assert _fwd(lib, O=FAKE_ODD) == 1
    assert _fwd(lib, stats=ctypes.c_void_p(0x10004)) == 1
    assert _fwd(lib, s=SaShape(1, 2, 128, 32, 64)) == 2
    assert _fwd(lib, s=SaShape(70000, 1, 128, 128, 64)) == 2


def test_q8_entry_points_reject_bad_arguments(lib):
    s, s64 = SaShape(1, 2, 128, 128, 64), SaShape(1, 2, 128, 64, 64)
    ws = ctypes.c_void_p(0x100000)

    def plan(s=s, Q8=FAKE, qs=FAKE, tau=0.9):
        return lib.sparse_attn_plan_q8(FAKE, FAKE, s, tau, 0.1, 0, FAKE, FAKE, None, None, Q8, FAKE, qs, FAKE,
                                       ws, 1 << 30, None)

    def fwd(s=s, K8=FAKE, ks=FAKE, lam=-math.inf):
        return lib.sparse_attn_fwd_q8(FAKE, K8, FAKE, ks, FAKE, s, FAKE, None, lam, 0.1, 0, FAKE, None, None)

    assert plan(Q8=None) == 1 and plan(qs=None) == 1
    assert plan(qs=ctypes.c_void_p(0x10002)) == 1                    # scales must be 4-byte aligned
    assert plan(Q8=FAKE_ODD) == 1 and plan(tau=1.5) == 1
    assert plan(s=s64) == 2                                         # d = 128 only
    assert fwd(K8=None) == 1 and fwd(ks=None) == 1 and fwd(lam=float("nan")) == 1
    assert fwd(s=s64) == 2


def test_recall_forward_rejects_bad_arguments(lib):
    s = SaShape(1, 2, 128, 128, 64)

    def fwd(s=s, K=FAKE, O=FAKE, recall=0.95, stats=None):
        return lib.sparse_attn_fwd_recall(FAKE, K, FAKE, s, FAKE, None, recall, 0.1, 0, O, stats, None)

    assert fwd(K=None) == 1 and fwd(O=None) == 1
    for bad in (0.0, -0.5, 1.0001, float("nan"), float("inf")):
        assert fwd(recall=bad) == 1, bad
    assert fwd(stats=ctypes.c_void_p(0x10004)) == 1                 # stats must be 8-byte aligned
    assert fwd(K=FAKE_ODD) == 1
    assert fwd(s=SaShape(1, 2, 128, 96, 64)) == 2                   # d in {64, 128}


def test_cluster_entry_points_reject_bad_arguments(lib):
    s = SaShape(1, 2, 1000, 128, 64)
    ws_need = int(lib.sparse_attn_cluster_workspace_size(s))
    assert ws_need > 0 and lib.sparse_attn_cluster_workspace_size(SaShape(1, 2, 1000, 96, 64)) == 0
    ws = ctypes.c_void_p(0x100000)

    def cl(X=FAKE, perm=FAKE, iters=2, ws=ws, nbytes=ws_need, s=s):
        return lib.sparse_attn_cluster(X, FAKE, s, iters, None, perm, None, ws, nbytes, None)

    assert cl(X=None) == 1 and cl(perm=None) == 1 and cl(X=FAKE_ODD) == 1
    assert cl(iters=-1) == 1 and cl(iters=65) == 1
    assert cl(ws=None) == 3 and cl(nbytes=ws_need - 1) == 3 and cl(ws=ctypes.c_void_p(0x100010)) == 3
    assert cl(s=SaShape(1, 2, 1000, 96, 64)) == 2

    def pr(src=FAKE, dst=ctypes.c_void_p(0x20000), perm=FAKE, s=s):
        return lib.sparse_attn_permute_rows(src, perm, s, 0, dst, None)

    assert pr(src=None) == 1 and pr(perm=None) == 1 and pr(dst=FAKE) == 1     # dst must differ from src
    assert pr(src=FAKE_ODD) == 1 and pr(perm=ctypes.c_void_p(0x10002)) == 1
    assert pr(s=SaShape(1, 2, 1000, 128, 32)) == 2


def test_device_error_needs_output_pointer(lib):
    assert lib.sparse_attn_device_error(None, None) == 1


def test_selftest_rejects_bad_limits(lib):
    # checked on the host: nothing is launched
    assert lib.sparse_attn_selftest_wait_timeout(0, None) == 1
    assert lib.sparse_attn_selftest_wait_timeout(4000001, None) == 1


def test_plan_heads_rejects_bad_arguments(lib):
    s = SaShape(1, 2, 128, 128, 64)
    fake = ctypes.c_void_p(256)       # never dereferenced: the checks run first
    ws = int(lib.sparse_attn_plan_workspace_size(s))
    # no tau array
    assert lib.sparse_attn_plan_heads(fake, fake, s, None, 0.1, 0, fake, fake, None, None, fake, ws, None) == 1
    # misaligned tau array
    assert lib.sparse_attn_plan_heads(fake, fake, s, ctypes.c_void_p(258), 0.1, 0, fake, fake, None, None,
                                      fake, ws, None) == 1
    # bad scale, bad shape, missing workspace
    assert lib.sparse_attn_plan_heads(fake, fake, s, fake, 0.0, 0, fake, fake, None, None, fake, ws, None) == 1
    assert lib.sparse_attn_plan_heads(fake, fake, SaShape(1, 2, 128, 96, 64), fake, 0.1, 0, fake, fake, None,
                                      None, fake, ws, None) == 2
    assert lib.sparse_attn_plan_heads(fake, fake, s, fake, 0.1, 0, fake, fake, None, None, None, ws, None) == 3


def test_decisions_forward_rejects_bad_arguments(lib):
    s = SaShape(1, 2, 128, 128, 64)

    def fwd(s=s, filt=0, value=-12.0, dec=FAKE, O=FAKE):
        return lib.sparse_attn_fwd_decisions(FAKE, FAKE, FAKE, s, FAKE, None, filt, value, 0.1, 0, O, None, dec,
                                             None)

    assert fwd(dec=None) == 1 and fwd(O=None) == 1
    assert fwd(filt=2) == 1 and fwd(filt=-1) == 1                   # unknown filter
    assert fwd(value=float("nan")) == 1 and fwd(value=float("inf")) == 1
    assert fwd(filt=1, value=0.0) == 1 and fwd(filt=1, value=1.5) == 1
    assert fwd(s=SaShape(1, 2, 128, 96, 64)) == 2


def test_host_call_rejects_bad_arguments(lib):
    s = SaShape(1, 2, 128, 128, 64)
    need = lib.sparse_attn_host_workspace_size(s, 2, 0)
    assert need > 4 * 2 * 128 * 128 * 2                              # the four device copies at least
    assert lib.sparse_attn_host_workspace_size(s, 0, 0) == 0         # chunks >= 1
    assert lib.sparse_attn_host_workspace_size(s, 2, 1) > need       # FP8 codes and scales on top
    ws = ctypes.c_void_p(0x100000)

    def call(s=s, Qh=FAKE, tau=0.9, tau_heads=None, filt=0, value=-12.0, flags=0, ws=ws, nbytes=need, chunks=2):
        return lib.sparse_attn_host(Qh, FAKE, FAKE, s, tau, tau_heads, filt, value, 0.1, 0, flags, FAKE, ws,
                                    nbytes, chunks, None, None, None)

    assert call(Qh=None) == 1
    assert call(tau=0.0) == 1 and call(tau=float("nan")) == 1
    assert call(tau_heads=ctypes.c_void_p(0x10002)) == 1             # per-head taus must be 4-byte aligned
    assert call(filt=3) == 1 and call(value=float("nan")) == 1
    assert call(filt=1, value=0.9, flags=1) == 1                     # recall with FP8 scores: not combined
    assert call(flags=4) == 1 and call(chunks=0) == 1
    assert call(flags=1, s=SaShape(1, 2, 128, 64, 64)) == 2           # FP8 scores: d = 128
    assert call(ws=None) == 3 and call(nbytes=need - 1) == 3
    assert call(ws=ctypes.c_void_p(0x100010)) == 3                   # workspace 256-byte aligned


def test_int8_entry_points_reject_bad_arguments(lib):
    s, s64 = SaShape(1, 2, 128, 128, 64), SaShape(1, 2, 128, 64, 64)
    ws = ctypes.c_void_p(0x100000)

    def plan(s=s, Q8=FAKE, qs=FAKE, tau=0.9):
        return lib.sparse_attn_plan_i8(FAKE, FAKE, s, tau, 0.1, 0, FAKE, FAKE, None, None, Q8, FAKE, qs, FAKE,
                                       ws, 1 << 30, None)

    def fwd(s=s, K8=FAKE, ks=FAKE, lam=-math.inf):
        return lib.sparse_attn_fwd_i8(FAKE, K8, FAKE, ks, FAKE, s, FAKE, None, lam, 0.1, 0, FAKE, None, None)

    assert plan(Q8=None) == 1 and plan(qs=None) == 1
    assert plan(qs=ctypes.c_void_p(0x10002)) == 1
    assert plan(Q8=FAKE_ODD) == 1 and plan(tau=1.5) == 1
    assert plan(s=s64) == 2
    assert fwd(K8=None) == 1 and fwd(ks=None) == 1 and fwd(lam=float("nan")) == 1
    assert fwd(s=s64) == 2
    # the host call: the two score flags exclude each other, and INT8 needs d = 128
    need = lib.sparse_attn_host_workspace_size(s, 2, 2)
    assert need == lib.sparse_attn_host_workspace_size(s, 2, 1)
    call = lambda flags, shape=s: lib.sparse_attn_host(FAKE, FAKE, FAKE, shape, 0.9, None, 0, -12.0, 0.1, 0,
                                                       flags, FAKE, ws, need, 2, None, None, None)
    assert call(3) == 1 and call(2, s64) == 2
