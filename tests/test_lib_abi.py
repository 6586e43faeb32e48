"""The C-ABI library loads without a GPU and exports every symbol the header
declares; host-side checks return before any CUDA call (CPU only)."""
import ctypes
import os
import re

import pytest

from combine_top_route_counting_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from combine_top_route_counting_b200 import build
    build.build()
    return moe.load()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe.h but not exported"
    assert sorted(moe.exported_symbols()) == names, "binding covers exactly the header's functions"


def test_host_only_queries(lib):
    sh = moe.shape(8, 7168, 384, 8, 7168, 2048)
    # rows_max = P*N*k + E*(pad-1) rounded up to 256
    assert moe.rows_max(sh) == (8 * 7168 * 8 + 384 * 255 + 255) // 256 * 256
    # [P][blocks of 2048 routes][E] counters, then a 64-byte line for the grid
    # barrier and the [E][P] totals the one-launch schedule accumulates
    assert moe.schedule_workspace_bytes(sh) == (8 * 28 * 384 + 16 + 384 * 8) * 4
    ws = moe.layer_workspace_bytes(sh)
    rm = moe.rows_max(sh)
    assert ws >= rm * (7168 * 2 + 2048 * 2 + 7168 * 4)  # xg, h and y
    assert moe.layer_host_workspace_bytes(sh) > ws
    assert moe.status_string(0) == "MOE_OK" and moe.status_string(3) == "MOE_WORKSPACE_TOO_SMALL"
    assert moe.status_from_device_flags(0) == 0
    assert moe.status_from_device_flags(moe.DEV_BAD_EXPERT_ID) == 6
    assert moe.status_from_device_flags(moe.DEV_TIMEOUT | moe.DEV_BAD_EXPERT_ID) == 5


@pytest.mark.parametrize("bad", [dict(P=0), dict(P=65), dict(E=0), dict(E=1025), dict(k=0),
                                 dict(k=17), dict(k=9, E=8), dict(N=-1), dict(pad=0)])
def test_shape_limits(lib, bad):
    args = dict(P=2, N=16, E=8, k=2, H=256, I=128, pad=256)
    args.update(bad)
    sh = moe.shape(**args)
    assert moe.rows_max(sh) == -1
    assert moe.layer_workspace_bytes(sh) == 0


@pytest.mark.parametrize("H,I,pad", [(128, 128, 256), (384, 128, 256), (256, 64, 256),
                                     (256, 128, 64)])
def test_ffn_shape_limits(lib, H, I, pad):
    sh = moe.shape(2, 16, 8, 2, H, I, pad)
    assert moe.layer_workspace_bytes(sh) == 0


def test_argument_errors_return_before_cuda(lib):
    sh = moe.shape(1, 16, 8, 2, 256, 128)
    L = lib
    assert L.moe_route_topk(None, None, None, ctypes.byref(sh), None) == 1
    assert L.moe_route_topk(None, None, None, None, None) == 1
    assert L.moe_schedule(None, None, None, None, None, None, 0, None, ctypes.byref(sh), None) == 1
    assert L.moe_expert_ffn(*([None] * 9), ctypes.byref(sh), None) == 1
    assert L.moe_layer_forward(*([None] * 6), 0, None, 0, None, ctypes.byref(sh), None, None) == 1
    assert L.moe_selftest_bounded_wait(None, 1000, None) == 1
    # misaligned pointers are rejected
    assert L.moe_combine(ctypes.c_void_p(8), ctypes.c_void_p(16), ctypes.c_void_p(16),
                         ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.byref(sh), None) == 1
    # negative minibatch
    p = ctypes.c_void_p(256)
    assert L.moe_layer_forward(p, p, p, p, p, p, -1, p, 1 << 40, p, ctypes.byref(sh), None,
                               None) == 1
    # workspace too small
    assert L.moe_layer_forward(p, p, p, p, p, p, 0, p, 16, p, ctypes.byref(sh), None, None) == 3


def test_backward_shape_limits_and_workspace(lib):
    kimi = moe.shape(8, 7168, 384, 8, 7168, 2048)
    rm = moe.rows_max(kimi)
    tw = moe.train_workspace_bytes(kimi)
    # forward buffers + ab, dys, dab, hg (dxg reuses y)
    assert tw >= moe.layer_workspace_bytes(kimi) + rm * (2048 * 4 + 7168 * 2 + 2048 * 4 + 2048 * 2)
    # the backward runs 256x256 pair tiles only: I % 256 and pad % 256
    assert moe.train_workspace_bytes(moe.shape(1, 512, 8, 2, 256, 128)) == 0
    assert moe.train_workspace_bytes(moe.shape(1, 512, 8, 2, 256, 256, pad=128)) == 0
    assert moe.train_workspace_bytes(moe.shape(1, 512, 8, 2, 256, 256)) > 0


def test_backward_argument_errors_return_before_cuda(lib):
    L = lib
    sh = moe.shape(1, 16, 8, 2, 256, 256)
    S = ctypes.byref(sh)
    assert L.moe_layer_forward_train(*([None] * 7), 0, None, S, None, None) == 1
    assert L.moe_expert_ffn_train(*([None] * 10), S, None) == 1
    assert L.moe_reverse_combine(*([None] * 8), S, None) == 1
    assert L.moe_expert_ffn_dgrad(*([None] * 14), S, None) == 1
    assert L.moe_reverse_dispatch(*([None] * 4), S, None) == 1
    assert L.moe_router_backward(*([None] * 6), S, None) == 1
    assert L.moe_expert_ffn_wgrad(*([None] * 10), S, None) == 1
    assert L.moe_layer_backward(*([None] * 10), 0, None, S, None, None) == 1
    p = ctypes.c_void_p(256)
    # I = 128: unsupported by the backward
    sh128 = moe.shape(1, 16, 8, 2, 256, 128)
    assert L.moe_layer_backward(*([p] * 10), 1 << 40, p, ctypes.byref(sh128), None, None) == 2
    assert L.moe_expert_ffn_wgrad(*([p] * 10), ctypes.byref(sh128), None) == 2
    # workspace too small; misaligned (16- but not 32-byte) workspace
    assert L.moe_layer_backward(*([p] * 10), 16, p, S, None, None) == 3
    assert L.moe_layer_forward_train(*([p] * 6), ctypes.c_void_p(272), 1 << 40, p, S, None,
                                     None) == 1


def test_host_async_entry_needs_an_event(lib):
    sh = moe.shape(1, 16, 8, 2, 256, 128)
    p = ctypes.c_void_p(256)
    args = [p] * 6 + [0, p, 1 << 40, p, ctypes.byref(sh), None]
    assert lib.moe_layer_forward_host_async(*args, None) == 1
    assert lib.moe_layer_forward_host_async(*args[:8], 16, p, ctypes.byref(sh), None, p) == 3


def test_mx_entry_points_argument_errors(lib):
    L = lib
    p = ctypes.c_void_p(256)
    assert L.moe_mx_quantize_rows(p, 4, 48, p, p, None) == 1       # K % 32 != 0
    assert L.moe_mx_quantize_rows(p, -1, 64, p, p, None) == 1      # negative rows
    assert L.moe_mx_quantize_rows(None, 4, 64, p, p, None) == 1    # null source
    assert L.moe_mx_quantize_rows(ctypes.c_void_p(264), 4, 64, p, p, None) == 1  # misaligned
    assert L.moe_mx_quantize_rows(None, 0, 64, None, None, None) == 0            # nothing to do
    sh = moe.shape(1, 16, 8, 2, 48, 128)                           # H % 32 != 0
    assert L.moe_dispatch_mxfp8(p, p, p, p, p, p, ctypes.byref(sh), None) == 2
    sh = moe.shape(1, 16, 8, 2, 256, 128)
    assert L.moe_dispatch_mxfp8(p, None, p, p, p, p, ctypes.byref(sh), None) == 1


def test_mx_ffn_entry_points_argument_errors(lib):
    L = lib
    p = ctypes.c_void_p(256)
    # weight quantisation: K and N multiples of 128, non-negative E, aligned pointers
    assert L.moe_mx_quantize_weights(p, 2, 192, 256, p, p, None) == 1     # K % 128
    assert L.moe_mx_quantize_weights(p, 2, 256, 64, p, p, None) == 1      # N % 128
    assert L.moe_mx_quantize_weights(p, -1, 256, 256, p, p, None) == 1
    assert L.moe_mx_quantize_weights(None, 2, 256, 256, p, p, None) == 1
    assert L.moe_mx_quantize_weights(ctypes.c_void_p(264), 2, 256, 256, p, p, None) == 1
    assert L.moe_mx_quantize_weights(p, 1 << 20, 1 << 12, 1 << 12, p, p, None) == 2  # too large
    assert L.moe_mx_quantize_weights(None, 0, 256, 256, None, None, None) == 0       # nothing to do
    # tiled dispatch: H % 128
    sh = moe.shape(1, 16, 8, 2, 96, 128)
    assert L.moe_dispatch_mxfp8_tiled(p, p, p, p, p, p, ctypes.byref(sh), None) == 2
    sh = moe.shape(1, 16, 8, 2, 256, 128)
    assert L.moe_dispatch_mxfp8_tiled(p, None, p, p, p, p, ctypes.byref(sh), None) == 1
    # block-scaled FFN: CTA-pair tiles need pad % 256; 32-byte aligned hq and y
    ok = moe.shape(2, 256, 8, 2, 256, 256)
    pad128 = moe.shape(2, 256, 8, 2, 256, 256, pad=128)
    args = [p] * 14 + [ctypes.byref(ok), None]
    assert L.moe_expert_ffn_mxfp8(*[p] * 14, ctypes.byref(pad128), None) == 2
    bad_h = moe.shape(2, 256, 8, 2, 384, 256)                             # H % 256
    assert L.moe_expert_ffn_mxfp8(*[p] * 14, ctypes.byref(bad_h), None) == 2
    for i in range(14):
        if i == 9:
            continue                                                      # counts may be null
        a = list(args)
        a[i] = None
        assert L.moe_expert_ffn_mxfp8(*a) == 1, i
    a = list(args)
    a[10] = ctypes.c_void_p(256 + 16)                                     # hq not 32-byte aligned
    assert L.moe_expert_ffn_mxfp8(*a) == 1
    # the layer: same limits; the bf16 layer's workspace without a shared
    # expert, the larger MXFP8 one with it
    need = moe.layer_workspace_bytes(ok)
    need_sh = moe.layer_mxfp8_workspace_bytes(ok)
    assert need_sh > need
    lay = [p] * 8 + [None] * 3 + [p, p] + [need - 1, p, ctypes.byref(ok), None, None]
    assert L.moe_layer_forward_mxfp8(*lay) == 3
    lay[13] = need
    lay[12] = ctypes.c_void_p(256 + 16)                                   # ws not 32-byte aligned
    assert L.moe_layer_forward_mxfp8(*lay) == 1
    lay[12] = p
    lay[15] = ctypes.byref(pad128)
    assert L.moe_layer_forward_mxfp8(*lay) == 2
    lay[15] = ctypes.byref(ok)
    lay[2] = None                                                         # W1q
    assert L.moe_layer_forward_mxfp8(*lay) == 1
    lay[2] = p
    lay[8] = p                                                            # Ws1 without Ws3, Ws2
    assert L.moe_layer_forward_mxfp8(*lay) == 1
    lay[9] = lay[10] = p                                                  # a shared expert needs
    assert L.moe_layer_forward_mxfp8(*lay) == 3                           # the larger workspace
    assert moe.layer_mxfp8_workspace_bytes(pad128) == 0


def test_size_queries_hold_their_invariants_on_random_shapes(lib):
    """Host-only size queries over random shapes (hypothesis): no crash, -1/0 for
    unsupported shapes, and rows_max / workspace bounds where supported."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=300, deadline=None)
    @given(P=st.integers(-2, 70), N=st.integers(-5, 20000), E=st.integers(-1, 1100),
           k=st.integers(-1, 20), H=st.sampled_from([0, 128, 256, 300, 512, 7168]),
           I=st.sampled_from([0, 64, 128, 256, 384, 2048]), pad=st.sampled_from([0, 1, 64, 128, 256, 512]))
    def check(P, N, E, k, H, I, pad):
        sh = moe.shape(P, N, E, k, H, I, pad)
        rm = moe.rows_max(sh)
        ok = 1 <= P <= 64 and N >= 0 and 1 <= E <= 1024 and 1 <= k <= min(E, 16) and 1 <= pad <= 65536
        if not ok:
            assert rm == -1 and moe.layer_workspace_bytes(sh) == 0
            return
        assert rm >= P * N * k and rm % 256 == 0
        assert rm <= P * N * k + E * (pad - 1) + 255
        ffn_ok = H >= 256 and H % 256 == 0 and I >= 128 and I % 128 == 0 and pad % 128 == 0
        ws = moe.layer_workspace_bytes(sh)
        assert (ws > 0) == ffn_ok
        if ffn_ok:
            assert ws >= rm * (H * 2 + I * 2 + H * 4)
            assert moe.layer_host_workspace_bytes(sh) > ws
            tw = moe.train_workspace_bytes(sh)
            assert (tw > 0) == (I % 256 == 0 and pad % 256 == 0)
            if tw:
                assert tw > ws

    check()


@pytest.mark.parametrize("P,N", [(8, 7168), (2, 300)])
def test_mxfp8_layer_workspace_covers_the_shared_expert(lib, P, N):
    """The layer's workspace plus the shared expert's h (bf16) and output (fp32)
    over round_up(P*N, 256) rows, and a padded copy of x when P*N is ragged."""
    H, I = 7168, 2048
    sh = moe.shape(P, N, 384, 8, H, I)
    rows = (P * N + 255) // 256 * 256
    extra = rows * (I * 2 + H * 4) + (rows * H * 2 if (P * N) % 256 else 0)
    assert moe.layer_mxfp8_workspace_bytes(sh) >= moe.layer_workspace_bytes(sh) + extra
    assert moe.layer_mxfp8_workspace_bytes(sh) < moe.layer_workspace_bytes(sh) + extra + 8 * 1024


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/moe.h compiles as C99 with a C compiler, and a C program linked
    against the library calls its host-only entry points (no GPU needed)."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
  moe_shape_t s = {8, 7168, 384, 8, 7168, 2048, 256};
  long long rows = (long long)moe_rows_max(&s);
  if (rows != (8LL * 7168 * 8 + 384 * 255 + 255) / 256 * 256) return 1;
  if (strcmp(moe_status_string(MOE_WORKSPACE_TOO_SMALL), "MOE_WORKSPACE_TOO_SMALL") != 0) return 2;
  if (moe_layer_workspace_bytes(&s) == 0) return 3;
  if (moe_route_topk(NULL, NULL, NULL, &s, NULL) != MOE_INVALID_ARG) return 4;
  s.pad = 0;
  if (moe_rows_max(&s) != -1) return 5;
  printf("ok %lld\n", rows);
  return 0;
}
''')
    lib_dir = os.path.dirname(moe.LIB_PATH)
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic-errors",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", lib_dir, "-l:" + os.path.basename(moe.LIB_PATH),
                        "-Wl,-rpath," + lib_dir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("ok"), (r.returncode, r.stdout, r.stderr)
