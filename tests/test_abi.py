"""The C ABI without a GPU: the library builds and loads, exports every
function include/mglu.h declares, and rejects bad arguments with the
documented status before touching the device."""
import ctypes
import os
import subprocess

import pytest

from masked_glu_b200 import build as mbuild
from masked_glu_b200 import mglu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    mbuild.build()
    return mglu.lib()


def test_exports_every_declared_symbol(L):
    names = mglu.header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", mglu.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert f" T {n}" in out, n


def test_kernel_launch_counter_counts_only_launches(L):
    """The counter moves only when a kernel was launched: calls rejected on
    the host (here: bad arguments, or no device at all) leave it as it was."""
    before = mglu.kernel_launches()
    assert before >= 0
    assert L.mglu_forward(None, 1, 64, None, 64, None, 4, 0, 0, None, None, 0, None) != 0
    assert mglu.kernel_launches() == before


def test_status_strings(L):
    for s in (0, -1, -2, -3, -4, -5):
        assert mglu.status_string(s) and mglu.status_string(s) != "unknown status"
    assert mglu.status_string(7) == "unknown status"


def test_sizes(L):
    assert mglu.packed_bytes(8, 4096, 14336) == 4096 * 14336
    assert mglu.packed_bytes(4, 2048, 8192) == 2048 * 8192 // 2
    assert mglu.packed_bytes(1, 8, 3) == 3
    assert mglu.packed_bytes(3, 8, 3) == 0
    assert mglu.workspace_bytes(16, 4096, 14336, 8) == 16 * 14336 * 2 + L.mglu_scratch_bytes(14336)
    assert L.mglu_workspace_bytes(3, 64, 100, 8, 1) == (3 * 100 * 4 + 255) // 256 * 256 + L.mglu_scratch_bytes(100)


def test_path_choice(L):
    prev = mglu.set_decode_max_tokens(16)
    try:
        assert mglu.forward_path(1) == mglu.PATH_DECODE
        assert mglu.forward_path(16) == mglu.PATH_DECODE
        assert mglu.forward_path(17) == mglu.PATH_PREFILL
        assert L.mglu_forward_path(3, 1) == mglu.PATH_F32
        assert mglu.set_decode_max_tokens(0) == 16
        assert mglu.forward_path(1) == mglu.PATH_PREFILL
        assert L.mglu_set_decode_max_tokens(17) == mglu.ERR_INVALID
        assert L.mglu_set_decode_max_tokens(-1) == mglu.ERR_INVALID
    finally:
        mglu.set_decode_max_tokens(prev)


A = 0x10000  # a 16-byte-aligned fake device address: never dereferenced, every call below fails validation


def fwd(L, x=A, T=1, d=128, W=A, h=16, pk=A, n_m=8, act=0, dtype=0, out=A, ws=A, wsb=1 << 30):
    return L.mglu_forward(x, T, d, W, h, pk, n_m, act, dtype, out, ws, wsb, None)


def test_forward_rejects_bad_arguments(L):
    assert fwd(L, n_m=3) == mglu.ERR_UNSUPPORTED
    assert fwd(L, n_m=0) == mglu.ERR_UNSUPPORTED
    assert fwd(L, n_m=16) == mglu.ERR_UNSUPPORTED
    assert fwd(L, x=None) == mglu.ERR_INVALID
    assert fwd(L, W=None) == mglu.ERR_INVALID
    assert fwd(L, pk=None) == mglu.ERR_INVALID
    assert fwd(L, out=None) == mglu.ERR_INVALID
    assert fwd(L, act=3) == mglu.ERR_INVALID
    assert fwd(L, dtype=2) == mglu.ERR_INVALID
    assert fwd(L, T=-1) == mglu.ERR_INVALID
    assert fwd(L, d=0) == mglu.ERR_INVALID
    assert fwd(L, h=0) == mglu.ERR_INVALID
    assert fwd(L, d=1 << 31) == mglu.ERR_INVALID
    # bf16 alignment rules
    assert fwd(L, x=A + 8) == mglu.ERR_ALIGN
    assert fwd(L, W=A + 2) == mglu.ERR_ALIGN
    assert fwd(L, pk=A + 4) == mglu.ERR_ALIGN
    assert fwd(L, out=A + 8) == mglu.ERR_ALIGN
    assert fwd(L, d=100) == mglu.ERR_ALIGN             # d % 8
    assert fwd(L, d=4) == mglu.ERR_ALIGN
    assert fwd(L, d=1026, n_m=1) == mglu.ERR_ALIGN
    # fp32 path: 4-byte alignment only
    assert fwd(L, dtype=1, x=A + 2) == mglu.ERR_ALIGN
    # decode scratch: required (and sized for h) on the decode path only
    need = L.mglu_scratch_bytes(16)
    assert need > 0
    assert fwd(L, ws=None) == mglu.ERR_INVALID
    assert fwd(L, wsb=need - 1) == mglu.ERR_INVALID
    assert fwd(L, ws=A + 8, wsb=need) == mglu.ERR_ALIGN
    # two partial slots per CTA of the grid, whatever the number of rows
    assert L.mglu_scratch_bytes(14336) == L.mglu_scratch_bytes(16)


def routed(L, x=A, T=1, d=128, W=A, h=16, pk=A, n_m=8, Wr=A, k=2, mode=0, act=0, dtype=0, w=A, sc=A, out=A, ws=A,
           wsb=1 << 30):
    return L.mglu_forward_routed(x, T, d, W, h, pk, n_m, Wr, k, mode, act, dtype, w, sc, out, ws, wsb, None)


def test_forward_routed_rejects_bad_arguments(L):
    """Every call below fails validation before any launch."""
    assert routed(L, n_m=3) == mglu.ERR_UNSUPPORTED
    assert routed(L, mode=2) == mglu.ERR_INVALID
    assert routed(L, k=9) == mglu.ERR_INVALID
    assert routed(L, k=-1) == mglu.ERR_INVALID
    assert routed(L, Wr=None) == mglu.ERR_INVALID
    assert routed(L, w=None) == mglu.ERR_INVALID
    assert routed(L, x=None) == mglu.ERR_INVALID
    assert routed(L, Wr=A + 1) == mglu.ERR_ALIGN
    assert routed(L, w=A + 2) == mglu.ERR_ALIGN
    assert routed(L, sc=A + 2) == mglu.ERR_ALIGN
    assert routed(L, ws=None) == mglu.ERR_INVALID   # the decode path needs its scratch
    assert routed(L, T=0) == mglu.OK                # nothing to do


def test_forward_zero_tokens_is_a_noop(L):
    # T == 0 returns before any device work, even with no x / out
    assert fwd(L, T=0, x=None, out=None) == mglu.OK


def test_down_and_block_reject_bad_arguments(L):
    big = 1 << 30
    assert L.mglu_down_proj(A, 1, 100, A, 64, 0, A, A, big, None) == mglu.ERR_ALIGN  # h % 8
    assert L.mglu_down_proj(A, 1, 12, A, 64, 0, A, A, big, None) == mglu.ERR_ALIGN
    assert L.mglu_down_proj(None, 1, 128, A, 64, 0, A, A, big, None) == mglu.ERR_INVALID
    assert L.mglu_down_proj(A, 1, 128, A, 64, 5, A, A, big, None) == mglu.ERR_INVALID
    assert L.mglu_down_proj(A, 1, 128, A, 64, 0, A, None, 0, None) == mglu.ERR_INVALID  # decode needs scratch
    assert L.mglu_down_proj(A, 0, 128, A, 64, 0, None, None, 0, None) == mglu.OK
    need = L.mglu_workspace_bytes(4, 128, 64, 8, 0)
    args = lambda ws, wsb: L.mglu_forward_down(A, 4, 128, A, 64, A, 8, 0, 0, A, ws, wsb, A, None)
    assert args(A, need - 1) == mglu.ERR_INVALID
    assert args(None, need) == mglu.ERR_INVALID
    assert L.mglu_forward_down(A, 4, 128, A, 64, A, 8, 0, 0, None, A, need, A, None) == mglu.ERR_INVALID


def test_pack_rejects_bad_arguments(L):
    assert L.mglu_pack_masks(A, 3, 8, 8, A, None) == mglu.ERR_UNSUPPORTED
    assert L.mglu_pack_masks(None, 8, 8, 8, A, None) == mglu.ERR_INVALID
    assert L.mglu_pack_masks(A, 8, 8, 8, A + 1, None) == mglu.ERR_ALIGN
    assert L.mglu_unpack_masks(A + 4, 8, 8, 8, A, None) == mglu.ERR_ALIGN
    assert L.mglu_pack_masks(A, 8, 0, 8, A, None) == mglu.ERR_INVALID


def test_mask_expansion_host_check(tmp_path):
    """The bit -> bf16x2 lane-mask helper the kernels use, compiled for the
    host (with an emulation of prmt) and checked against the packed-format
    definition for every n_m, register and mask."""
    exe = tmp_path / "pair_mask_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "masked_glu_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "native", "pair_mask_check.cpp")], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout


def test_sign_flip_host_check(tmp_path):
    """The decode kernel's sign-flip operand construction (group_bits and
    flip_pair in csrc/common.cuh), compiled for the host and checked against
    the packed-format definition for every n_m, group, pair and mask."""
    exe = tmp_path / "flip_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "masked_glu_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "native", "flip_check.cpp")], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout


def test_logit_bit_rule_on_every_fp16_pattern(tmp_path):
    """The mask-logit bit rule (logit_bit in csrc/common.cuh), compiled for
    the host and evaluated on all 65536 binary16 patterns, equals numpy's
    IEEE comparison logit > 0 (so +-0 and NaN give 0, +inf and positive
    subnormals give 1)."""
    import numpy as np
    exe = tmp_path / "logit_bit_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "masked_glu_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "native", "logit_bit_check.cpp")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.strip()
    got = np.frombuffer(out.encode(), dtype=np.uint8) - ord("0")
    with np.errstate(invalid="ignore"):
        want = (np.arange(65536, dtype=np.uint16).view(np.float16) > 0).astype(np.uint8)
    assert got.shape == want.shape and np.array_equal(got, want)


def test_decode_schedule_host_check(tmp_path):
    """The decode kernel's work split (csrc/sched.cuh), compiled for the host:
    every (row block, k-stage) unit done once, split row blocks' contributor
    counts and scratch slots consistent, over many shapes and grid sizes."""
    exe = tmp_path / "sched_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "masked_glu_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "native", "sched_check.cpp")], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout


def test_forward_host_rejects_before_any_copy():
    """Argument errors of the host-buffer entry point come back before any
    copy or launch is queued (no device is touched)."""
    L = mglu.lib()
    p = ctypes.c_void_p(1 << 20)
    need = L.mglu_host_workspace_bytes(2, 128, 64, 4, 0, 0)
    assert need > 0
    assert L.mglu_host_workspace_bytes(2, 128, 64, 4, 0, 1) > need   # the block also stages the hidden
    args = lambda xh, ws, wsb, rh: L.mglu_forward_host(xh, 2, 128, p, 64, p, 4, 0, 0, None, ws, wsb, rh, None)
    assert args(None, p, need, p) == -1                  # no host input
    assert args(p, p, need, None) == -1                  # no host result
    assert args(p, None, need, p) == -1                  # no workspace
    assert args(p, p, need - 1, p) == -1                 # workspace too small
    assert args(p, ctypes.c_void_p((1 << 20) + 16), need, p) == -3   # workspace not 256-byte aligned
    assert L.mglu_forward_host(p, 0, 128, p, 64, p, 4, 0, 0, None, p, need, p, None) == 0   # T == 0: no-op


C_CALLER = r"""
/* A plain C99 caller of the library: no CUDA headers, only mglu.h. */
#include <stdio.h>
#include <stdint.h>
#include <stdlib.h>
#include "mglu.h"

int main(void)
{
    /* malloc gives 16-byte aligned blocks on this platform, as the bf16 path requires */
    uint16_t *x = malloc(128 * 2), *W = malloc(128 * 4 * 2), *out = malloc(4 * 2);
    uint8_t *packed = malloc(256);
    if (!x || !W || !out || !packed || ((uintptr_t)W | (uintptr_t)packed | (uintptr_t)x | (uintptr_t)out) % 16)
        return 2;
    /* host-side size queries */
    printf("packed %zu\n", mglu_packed_bytes(4, 128, 4));
    printf("scratch_nonzero %d\n", mglu_scratch_bytes(4) > 0);
    printf("path %d %d\n", mglu_forward_path(1, MGLU_BF16), mglu_forward_path(64, MGLU_BF16));
    /* rejected before any device work: unsupported n_m, bad act, d % 8 */
    printf("nm3 %d\n", mglu_forward(x, 1, 128, W, 4, packed, 3, MGLU_ACT_SWISH, MGLU_BF16, out, 0, 0, 0));
    printf("act9 %d\n", mglu_forward(x, 1, 128, W, 4, packed, 4, 9, MGLU_BF16, out, 0, 0, 0));
    printf("d60 %d\n", mglu_forward(x, 1, 60, W, 4, packed, 4, MGLU_ACT_GELU, MGLU_BF16, out, 0, 0, 0));
    printf("zeroT %d\n", mglu_forward(x, 0, 128, W, 4, packed, 4, MGLU_ACT_RELU, MGLU_BF16, out, 0, 0, 0));
    printf("msg %s\n", mglu_status_string(MGLU_ERR_ALIGN));
    printf("f32path %d\n", mglu_forward_path(1, MGLU_F32));
    free(x), free(W), free(out), free(packed);
    return 0;
}
"""


def test_header_serves_a_plain_c99_caller(tmp_path):
    """include/mglu.h compiles as strict C99 and a C program links against
    libmglu.so and gets the documented host-side answers (no GPU needed)."""
    mbuild.build()
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    lib_dir = os.path.dirname(mglu.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), f"-L{lib_dir}", "-l:libmglu.so", f"-Wl,-rpath,{lib_dir}"],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(line.split(" ", 1) for line in out if line)
    assert got["packed"] == str(128 * 4 * 4 // 8)
    assert got["scratch_nonzero"] == "1"
    assert got["path"] == "0 1" and got["f32path"] == "2"  # decode for 1 token, prefill for 64; fp32 path
    assert got["nm3"] == "-2" and got["act9"] == "-1" and got["d60"] == "-3" and got["zeroT"] == "0"
    assert got["msg"] == "alignment requirement not met"
