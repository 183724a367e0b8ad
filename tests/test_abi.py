"""The C-ABI library loads and exports every symbol include/moe.h declares; the host-side
argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from routed_grouped_gemm_softmax_b200 import api, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return api.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 8, names
    for n in names:
        assert hasattr(L, n), f"{n} declared in moe.h but not exported"
    assert sorted(names) == sorted(api.EXPORTS)


def test_workspace_size_and_tiles(L):
    for (T, H, I, E, k) in [(64, 256, 512, 8, 2), (16, 2048, 512, 256, 8), (4096, 2048, 512, 256, 8),
                            (8192, 4096, 1408, 64, 6)]:
        n = api.moe_workspace_size(T, H, I, E, k)
        A = T * k
        # at least the three activation-sized buffers plus the logits
        assert n >= A * H * 2 * 2 + A * I * 2 + T * E * 4
        assert n % 1024 == 0
        assert api.moe_max_tiles(T, H, I, E, k) == (A + 127) // 128 + min(A, E)
    assert api.moe_workspace_size(64, 100, 512, 8, 2) == 0   # H not a multiple of 64
    assert api.moe_workspace_size(64, 256, 512, 8, 9) == 0   # top_k > E
    assert api.moe_workspace_size(64, 256, 512, 2000, 2) == 0  # too many experts


def test_host_argument_errors(L):
    null = None
    d = api.dims(4, 256, 512, 8, 2)
    # missing inputs are rejected before any device work
    assert L.moe_route(ctypes.byref(d), null, null, null, null, null, null, 0, null) == 1
    assert L.moe_forward(ctypes.byref(d), null, null, null, null, null, null, null, null, 0, null) == 1
    assert L.moe_permute(ctypes.byref(d), null, null, null, null, null, null, null, 0, null) == 1
    bad = api.dims(4, 256, 512, 8, 0)
    assert L.moe_route(ctypes.byref(bad), null, null, null, null, null, null, 0, null) == 1
    wide = api.dims(4, 256, 512, 4096, 2)
    assert L.moe_route(ctypes.byref(wide), null, null, null, null, null, null, 0, null) == 2
    assert L.moe_route(None, null, null, null, null, null, null, 0, null) == 1
    # T == 0 is a no-op
    zero = api.dims(0, 256, 512, 8, 2)
    assert L.moe_forward(ctypes.byref(zero), null, null, null, null, null, null, null, null, 0, null) == 0
    # a workspace that is too small or misaligned
    buf = ctypes.create_string_buffer(4096)
    addr = (ctypes.addressof(buf) + 255) // 256 * 256
    fake = ctypes.c_void_p(addr)
    assert L.moe_route(ctypes.byref(d), fake, fake, null, fake, fake, fake, 16, null) == 3
    assert L.moe_route(ctypes.byref(d), fake, fake, null, fake, fake, ctypes.c_void_p(addr + 8),
                       1 << 30, null) == 3
    assert L.moe_get_device_status(null, null) == 1


def test_shared_expert_host_checks(L):
    null = None
    d = api.dims(64, 256, 512, 8, 2)
    base = api.moe_workspace_size(64, 256, 512, 8, 2)
    # no shared expert: the plain layer's workspace; each I-wide slice adds T rows of h and y
    assert api.moe_workspace_size_shared(64, 256, 512, 8, 2, 0) == base
    two = api.moe_workspace_size_shared(64, 256, 512, 8, 2, 1024)
    assert two >= base + 2 * 64 * (512 + 256) * 2
    assert api.moe_workspace_size_shared(64, 256, 512, 8, 2, 700) == 0   # not a multiple of I
    assert api.moe_workspace_size_shared(64, 256, 512, 8, 2, -512) == 0
    buf = ctypes.create_string_buffer(64)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) // 16 * 16)
    # shared_I not a multiple of I, or missing shared weights: rejected before any device work
    assert L.moe_forward_shared(ctypes.byref(d), p, p, null, p, p, p, 700, p, p, p, p, null, 0, null) == 1
    assert L.moe_forward_shared(ctypes.byref(d), p, p, null, p, p, p, 512, null, p, p, p, null, 0, null) == 1
    # and a workspace sized for the plain layer is too small for a shared expert
    ws = ctypes.create_string_buffer(base + 512)
    wsp = ctypes.c_void_p((ctypes.addressof(ws) + 255) // 256 * 256)
    assert L.moe_forward_shared(ctypes.byref(d), p, p, null, p, p, p, 512, p, p, p, p, wsp, base, null) == 3


def test_workspace_regions_do_not_overlap(L):
    # the routing regions moe_workspace_offsets reports: 1 KiB aligned, inside the
    # workspace, and each at least as large as moe.h documents before the next begins
    for dtype in (api.DTYPE_BF16, api.DTYPE_FP8):
        for (T, H, I, E, k) in [(16, 2048, 512, 256, 8), (4096, 2048, 512, 256, 8), (8192, 4096, 1408, 64, 6),
                                (150, 384, 384, 12, 3), (1, 256, 256, 300, 4)]:
            d = api.dims(T, H, I, E, k)
            size = api.moe_workspace_size(T, H, I, E, k, dtype)
            off = (ctypes.c_size_t * 8)()
            assert L.moe_workspace_offsets(ctypes.byref(d), dtype, off, 8) == 0
            A = T * k
            need = [A * 4, A * 4, (E + 1) * 4, A * 4, A * 4, 3 * api.moe_max_tiles(T, H, I, E, k) * 4, 4, T * E * 4]
            regions = sorted(zip(list(off), need))
            for (o, n), (o2, _) in zip(regions, regions[1:] + [(size, 0)]):
                assert o % 1024 == 0, (dtype, T, o)
                assert o + n <= o2, (dtype, T, o, n, o2)
    bad = api.dims(4, 100, 512, 8, 2)
    assert L.moe_workspace_offsets(ctypes.byref(bad), 0, (ctypes.c_size_t * 8)(), 8) == 1


def test_header_is_plain_c_and_links(L, tmp_path):
    # a C99 program includes moe.h, links the library and calls its host-only entry
    # points (workspace sizing; the argument checks), with warnings as errors
    import subprocess

    lib_dir = os.path.dirname(api.LIB_PATH)
    src = tmp_path / "use_moe.c"
    src.write_text(r"""
#include <stdio.h>
#include "moe.h"
int main(void) {
    moe_dims_t d = {16, 2048, 512, 256, 8};
    size_t ws = moe_workspace_size(&d, MOE_DTYPE_BF16);
    int32_t tiles = moe_max_tiles(&d);
    moe_status_t bad = moe_forward(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
    printf("%zu %d %d\n", ws, (int)tiles, (int)bad);
    return (ws > 0 && tiles == 1 + 128 && bad == MOE_ERR_INVALID_ARG) ? 0 : 1;
}
""")
    exe = tmp_path / "use_moe"
    inc = os.path.dirname(HEADER)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", inc, str(src), "-o", str(exe),
                    "-L", lib_dir, "-lmoe_b200", f"-Wl,-rpath,{lib_dir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert int(r.stdout.split()[0]) == api.moe_workspace_size(16, 2048, 512, 256, 8)


def test_forward_plan_follows_the_tile_table(L):
    # The plan query is host-only: the kernels a forward would launch under the
    # current settings, by the M bucket (average rows per expert) of the batch.
    bf = lambda T, H, I, E, k: api.forward_plan(T, H, I, E, k, api.DTYPE_BF16)
    # gate/up A rows straight from x up to 16 rows per expert, the sorted copy above
    def plan(T, H, I, E, k, dt=api.DTYPE_BF16):
        p = api.forward_plan(T, H, I, E, k, dt)
        return p if p < 0 or dt != api.DTYPE_BF16 else p & ~api.PLAN_DIRECT_A
    for T in (1, 16, 33, 128):
        assert bf(T, 2048, 1024, 64, 8) & api.PLAN_DIRECT_A
    for T in (136, 4096, 8192):   # 17 and more rows per expert
        assert not bf(T, 2048, 1024, 64, 8) & api.PLAN_DIRECT_A
    # decode-sized: the two-kernel router, 128-row tiles, one GEMM launch, combine inside
    assert plan(16, 2048, 512, 256, 8) == api.PLAN_SMALL_ROUTER | api.PLAN_FUSED_COMBINE | api.PLAN_LAYER_GEMM
    # 128 rows per expert: 128-row tiles, one GEMM launch, the combine kernel
    assert plan(4096, 2048, 512, 256, 8) == api.PLAN_LAYER_GEMM
    # 767 rows per expert still 128-row tiles; 768 and up pair tiles
    assert plan(767 * 64 // 8 + 7, 2048, 1024, 64, 8) & api.PLAN_PAIR_TILES == 0
    assert plan(768 * 64 // 8, 2048, 1024, 64, 8) & api.PLAN_PAIR_TILES
    assert plan(8192, 4096, 1408, 64, 6) == api.PLAN_PAIR_TILES | api.PLAN_LAYER_GEMM   # the Skewed workload
    # the combine inside the down GEMM up to 32 tokens
    assert plan(32, 512, 512, 64, 8) & api.PLAN_FUSED_COMBINE
    assert not plan(33, 512, 512, 64, 8) & api.PLAN_FUSED_COMBINE
    # forced settings
    try:
        api.set_pair_mma("never")
        api.set_layer_gemm("never")
        api.set_direct_a("never")
        assert bf(8192, 4096, 1408, 64, 6) == 0
    finally:
        api.set_pair_mma("auto")
        api.set_layer_gemm("auto")
        api.set_direct_a("auto")
    assert plan(64, 100, 512, 8, 2) == -1   # invalid dims
    assert plan(1024, 7168, 2048, 256, 8, api.DTYPE_FP8) == 0
    assert plan(16, 7168, 2048, 256, 8, api.DTYPE_FP8) == api.PLAN_SMALL_ROUTER | api.PLAN_FUSED_COMBINE
