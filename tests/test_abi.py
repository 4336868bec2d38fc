"""The C-ABI library loads and exports every entry point include/sru.h declares,
and its host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sru.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sru_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib_path():
    from parallelizable_recurrence_b200 import build
    return build.build()


@pytest.fixture(scope="module")
def lib(lib_path):
    import parallelizable_recurrence_b200 as m
    return m.load_library(lib_path)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sru_project", "sru_project_backward", "sru_forward", "sru_backward",
                     "sru_workspace_bytes", "sru_sync_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib_path, lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (sru_[a-z_0-9]+)\b", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_binding_lists_every_declared_symbol():
    import parallelizable_recurrence_b200 as m
    assert sorted(m.EXPORTED) == declared_functions()


def test_status_strings_and_version(lib):
    assert lib.sru_status_string(0) == b"SRU_OK"
    assert b"TIMEOUT" in lib.sru_status_string(3)
    assert lib.sru_version() >= 100


def test_workspace_size_is_host_arithmetic(lib):
    # checkpoints (ceil(L/16) * B * n_dir * d floats) + partial sums (B * n_dir * 4 * d doubles)
    n = lib.sru_workspace_bytes(1024, 16, 2048, 0, 0)
    assert n >= 64 * 16 * 2048 * 4 + 16 * 4 * 2048 * 8
    assert lib.sru_workspace_bytes(1024, 16, 2048, 1, 0) > n
    assert lib.sru_workspace_bytes(10, 2, 12, 0, 0) == 0      # d % 8 != 0 is unsupported


def test_invalid_arguments_return_before_any_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)
    # d not a multiple of 8
    st = lib.sru_forward(fake, 1, fake, fake, fake, None, None, 4, 2, 12, 1.0, 0, 0, fake, fake, None, 0, None)
    assert st == 4
    # negative sizes
    st = lib.sru_forward(fake, 1, fake, fake, fake, None, None, -1, 2, 16, 1.0, 0, 0, fake, fake, None, 0, None)
    assert st == 1
    # unknown U dtype
    st = lib.sru_forward(fake, 7, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, fake, fake, None, 0, None)
    assert st == 1
    # null outputs
    st = lib.sru_forward(fake, 1, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, None, None, None, 0, None)
    assert st == 1
    # misaligned pointer
    st = lib.sru_project(vp(0x1001), 1, fake, 1, fake, 1, 64, 64, 64, None)
    assert st == 1
    # unsupported type combination
    st = lib.sru_project(fake, 0, fake, 1, fake, 1, 64, 64, 64, None)
    assert st == 1
    # backward without a workspace
    st = lib.sru_backward(fake, 1, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, fake, None, None, 0,
                          fake, 1, fake, fake, fake, fake, None)
    assert st == 1
    # a workspace smaller than sru_workspace_bytes reports
    need = lib.sru_workspace_bytes(4, 2, 16, 0, 0)
    st = lib.sru_backward(fake, 1, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, fake, None, fake, need - 1,
                          fake, 1, fake, fake, fake, fake, None)
    assert st == 1
    st = lib.sru_forward(fake, 1, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, fake, fake, fake, need - 1, None)
    assert st == 1
    # the scan regions: always with SRU_FLAG_V_ZERO; without it only where the
    # backward would take the scan (a small batch*width); not for a wide layer
    assert lib.sru_workspace_bytes(4096, 64, 4096, 0, 1) > lib.sru_workspace_bytes(4096, 64, 4096, 0, 0)
    small = lib.sru_workspace_bytes(4096, 2, 64, 0, 0)
    assert small >= 4096 // 64 * 2 * (4 + 3 * 64 * 4)
    st = lib.sru_forward(fake, 1, fake, fake, fake, None, None, 4096, 2, 64, 1.0, 0, 1 | 2, fake, fake, None, 0, None)
    assert st == 1


def test_decode_step_checks_arguments_before_any_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)
    args = [fake] * 7
    assert lib.sru_decode_step(*args, 0, 64, 1.0, None, 0, None) == 0          # B = 0: nothing to do
    assert lib.sru_decode_step(*args, 2, 12, 1.0, None, 0, None) == 4          # d % 8 != 0
    assert lib.sru_decode_step(*args, -1, 64, 1.0, None, 0, None) == 1         # negative B
    assert lib.sru_decode_step(None, *args[1:], 2, 64, 1.0, None, 0, None) == 1  # null X_t
    assert lib.sru_decode_step(vp(0x1008), *args[1:], 2, 64, 1.0, None, 0, None) == 1  # misaligned X_t
    assert lib.sru_decode_step(*args, 1, 1 << 25, 1.0, None, 0, None) == 4     # d beyond the size limit
    # the batched tensor-core path: its workspace size, and a short workspace rejected
    assert lib.sru_decode_workspace_bytes(4, 64) == 0
    assert lib.sru_decode_workspace_bytes(21, 64) == 0                # not a multiple of 8
    need = lib.sru_decode_workspace_bytes(16, 64)
    assert need >= 3 * 64 * 16 * 4
    assert lib.sru_decode_step(*args, 16, 64, 1.0, fake, need - 256, None) == 1


def test_per_channel_vectors_must_be_pair_aligned(lib):
    """v, b, c0, c_T (and dc_T, dv, db, dc0) are read and written as 8-byte channel
    pairs: a pointer off an 8-byte boundary is rejected before any launch."""
    vp = ctypes.c_void_p
    fake, odd = vp(0x1000), vp(0x1004)
    for pos in (3, 4, 5, 14):  # v, b, c0, c_T
        args = [fake, 1, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, fake, fake, None, 0, None]
        args[pos] = odd
        assert lib.sru_forward(*args) == 1, pos
    need = lib.sru_workspace_bytes(4, 2, 16, 0, 0)
    for pos in (3, 4, 14, 20, 21, 22):  # v, b, dc_T, dv, db, dc0
        args = [fake, 1, fake, fake, fake, None, None, 4, 2, 16, 1.0, 0, 0, fake, fake, fake, need,
                fake, 1, fake, fake, fake, fake, None]
        args[pos] = odd
        assert lib.sru_backward(*args) == 1, pos
    for pos in (3, 4, 12):  # b, c0, c_T
        args = [fake, 1, fake, fake, fake, None, 4, 2, 64, 1.0, 0, fake, fake, None]
        args[pos] = odd
        assert lib.sru_forward_scan_noalloc(*args) == 1, pos


def test_attention_backward_checks_arguments_before_any_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)
    L, B, d, dp, N = 64, 2, 128, 32, 384
    fneed = lib.sru_attention_workspace_bytes(L, B, dp)
    need = lib.sru_attention_backward_workspace_bytes(L, B, d, dp, N)
    # per group: scores or their gradient (fp32), P and dS (bf16) of each batch row
    assert need >= B * L * L * 8 + L * B * dp * (4 + 4 + 2 + 4 + 2)
    assert lib.sru_attention_backward_workspace_bytes(60, B, d, dp, N) == 0      # L % 8 != 0
    assert lib.sru_attention_backward_workspace_bytes(L, B, d, 12, N) == 0       # d' % 8 != 0
    assert lib.sru_attention_backward_workspace_bytes(L, B, 100, dp, N) == 0     # d % 8 != 0

    def call(**kw):
        a = dict(dU=fake, X=fake, Wq=fake, Wkv=fake, Wo=fake, alpha=0.5, g=None, b=None, causal=1, fws=fake,
                 fwsb=fneed, dX=fake, acc=0, dWq=fake, dWkv=fake, dWo=fake, dg=None, db=None, L=L, B=B, d=d, dp=dp,
                 N=N, ws=fake, wsb=need, st=None)
        a.update(kw)
        return lib.sru_attention_project_backward(*a.values())

    assert call(dU=None) == 1                       # null input
    assert call(dWkv=None) == 1                     # null output
    assert call(dX=vp(0x1008)) == 1                 # misaligned output
    assert call(fwsb=fneed - 256) == 1              # short forward workspace
    assert call(wsb=need - 256) == 1                # short workspace
    assert call(g=fake) == 1                        # gamma without beta
    assert call(g=fake, b=fake) == 1                # the norm without its gradient outputs
    assert call(g=vp(0x1004), b=fake, dg=fake, db=fake) == 1   # gamma off a 16-byte boundary
    assert call(d=100) == 4                         # d % 8 != 0
    assert call(L=0) == 1                           # no tokens
