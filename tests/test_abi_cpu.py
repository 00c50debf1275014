"""The C-ABI library on the host, without a GPU: it loads, exports every entry
point that include/gdn.h declares, and rejects bad arguments before enqueuing
anything. Every call here fails a host check on purpose (fake pointer values are
never dereferenced), so the file is safe to run on a machine with a GPU too."""
import ctypes
import os
import re

import numpy as np
import pytest

import gated_delta_rule_102_b200 as gdn
from gated_delta_rule_102_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = open(os.path.join(ROOT, "include", "gdn.h")).read()


@pytest.fixture(scope="module")
def L():
    gdn_build.build()
    return gdn.lib()


def declared_functions():
    body = re.sub(r"/\*.*?\*/", "", HEADER, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_\w+)\s*\(", body)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("gdn_conv_update", "gdn_recurrent_step", "gdn_gated_rmsnorm", "gdn_decode_step"):
        assert f in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {gdn.LIB_PATH}").read()
    exported = set(re.findall(r" T (gdn_\w+)", out))
    assert set(declared_functions()) <= exported
    assert set(gdn._abi.EXPORTS) == set(declared_functions())


def test_abi_version_matches_header(L):
    m = re.search(r"#define GDN_ABI_VERSION \(\((\d+) << 16\) \| (\d+)\)", HEADER)
    assert gdn.abi_version() == (int(m.group(1)) << 16) | int(m.group(2))


def test_status_codes_match_header(L):
    for name in ("GDN_OK", "GDN_ERR_INVALID_ARGUMENT", "GDN_ERR_UNSUPPORTED", "GDN_ERR_MISALIGNED",
                 "GDN_ERR_SLOT_RANGE", "GDN_ERR_CUDA"):
        m = re.search(rf"\b{name} = (\d+)", HEADER)
        assert m and int(m.group(1)) == getattr(gdn, name)
        assert gdn.status_string(getattr(gdn, name))
    for name in ("GDN_DEVICE_ERR_SLOT_RANGE", "GDN_DEVICE_ERR_TIMEOUT", "GDN_DEVICE_ERR_SEQLEN", "GDN_DEVICE_ERR_BATCH"):
        m = re.search(rf"#define {name} (\d+)", HEADER)
        assert int(m.group(1)) == getattr(gdn, name)


def test_check_slots_host(L):
    assert gdn.gdn_check_slots_host([0, 3, 1], 4) == gdn.GDN_OK
    assert gdn.gdn_check_slots_host([], 4) == gdn.GDN_OK
    assert gdn.gdn_check_slots_host([0, 4], 4) == gdn.GDN_ERR_SLOT_RANGE
    assert gdn.gdn_check_slots_host([-1], 4) == gdn.GDN_ERR_SLOT_RANGE
    assert gdn.gdn_check_slots_host([2, 1, 2], 4) == gdn.GDN_ERR_SLOT_RANGE
    assert L.gdn_check_slots_host(None, 3, 4) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert L.gdn_check_slots_host(None, -1, 4) == gdn.GDN_ERR_INVALID_ARGUMENT


FAKE = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced
FAKE_ODD = ctypes.c_void_p((1 << 20) + 2)


def good_cfg(**kw):
    base = dict(num_k_heads=16, num_v_heads=32, head_k_dim=128, head_v_dim=128, conv_width=4)
    base.update(kw)
    return gdn.GdnConfig.make(**base)


def decode(L, cfg, B=4, T=1, ptrs=None, pool=8, out_f32=None, err=None, ws=None):
    p = [FAKE] * 10 if ptrs is None else ptrs
    return L.gdn_decode_step(ctypes.byref(cfg) if cfg is not None else None, B, T, *p, pool, FAKE, FAKE,
                             out_f32, err, ws, None)


@pytest.mark.parametrize("kw,status", [
    (dict(num_k_heads=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(num_v_heads=-2), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(num_v_heads=24, num_k_heads=16), gdn.GDN_ERR_INVALID_ARGUMENT),  # Hv not a multiple of Hk
    (dict(num_v_heads=160, num_k_heads=16), gdn.GDN_ERR_UNSUPPORTED),      # Hv/Hk = 10 > 8
    (dict(head_k_dim=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(head_v_dim=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(head_v_dim=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(conv_width=1), gdn.GDN_ERR_UNSUPPORTED),
    (dict(conv_width=9), gdn.GDN_ERR_UNSUPPORTED),
    (dict(l2_eps=-1.0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(rms_eps=float("nan")), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(q_scale=float("inf")), gdn.GDN_ERR_INVALID_ARGUMENT),
])
def test_decode_rejects_bad_config(L, kw, status):
    assert decode(L, good_cfg(**kw)) == status


def test_decode_rejects_bad_sizes_and_pointers(L):
    cfg = good_cfg()
    assert decode(L, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert decode(L, cfg, B=-1) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert decode(L, cfg, T=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert decode(L, cfg, T=17) == gdn.GDN_ERR_UNSUPPORTED
    assert decode(L, cfg, pool=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    for i in range(10):
        ptrs = [FAKE] * 10
        ptrs[i] = None
        assert decode(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_INVALID_ARGUMENT, i
        ptrs[i] = FAKE_ODD
        assert decode(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_MISALIGNED, i
    assert decode(L, cfg, out_f32=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    assert decode(L, cfg, err=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    assert decode(L, cfg, ws=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    assert gdn.decode_workspace_bytes() % 16 == 0 and gdn.decode_workspace_bytes() >= 8


def static_scratch(L, cfg, B=4, T=1, ptrs=None, pool=8, out_f32=None, err=None):
    p = [FAKE] * 10 if ptrs is None else ptrs
    return L.gdn_decode_step_static_scratch(ctypes.byref(cfg) if cfg is not None else None, B, T, *p, pool, FAKE,
                                            FAKE, out_f32, err, None)


def test_static_scratch_checks_every_argument_before_touching_the_device(L):
    # Without a GPU any CUDA call fails, so a status other than GDN_ERR_CUDA shows that
    # the check ran before the scratch lookup and the memset were enqueued.
    cfg = good_cfg()
    assert static_scratch(L, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert static_scratch(L, good_cfg(head_k_dim=96)) == gdn.GDN_ERR_UNSUPPORTED
    assert static_scratch(L, cfg, T=17) == gdn.GDN_ERR_UNSUPPORTED
    assert static_scratch(L, cfg, B=-1) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert static_scratch(L, cfg, B=0, ptrs=[None] * 10) == gdn.GDN_OK
    for i in range(10):
        ptrs = [FAKE] * 10
        ptrs[i] = None
        assert static_scratch(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_INVALID_ARGUMENT, i
        ptrs[i] = FAKE_ODD
        assert static_scratch(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_MISALIGNED, i
    assert static_scratch(L, cfg, out_f32=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    assert static_scratch(L, cfg, err=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    assert gdn.decode_static_scratch_bytes() >= gdn.decode_workspace_bytes()


def spec_verify(L, cfg, B=4, T=4, ptrs=None, pool=8, out_f32=None, spec=None, err=None):
    p = [FAKE] * 10 if ptrs is None else ptrs
    s = [FAKE] * 3 if spec is None else spec
    return L.gdn_spec_verify(ctypes.byref(cfg) if cfg is not None else None, B, T, *p, pool, FAKE, FAKE, out_f32,
                             *s, err, None)


def spec_commit(L, cfg, B=4, T=4, ptrs=None, pool=8, err=None):
    p = [FAKE] * 8 if ptrs is None else ptrs  # n_accept, qkv, conv_pool, state_pool, slots, k, delta, alpha
    return L.gdn_spec_commit(ctypes.byref(cfg) if cfg is not None else None, B, T, p[0], p[1], p[2], p[3], pool,
                             p[4], p[5], p[6], p[7], err, None)


def test_spec_entry_points_check_every_argument_before_touching_the_device(L):
    cfg = good_cfg()
    for call in (spec_verify, spec_commit):
        assert call(L, None) == gdn.GDN_ERR_INVALID_ARGUMENT
        assert call(L, good_cfg(head_v_dim=48)) == gdn.GDN_ERR_UNSUPPORTED
        assert call(L, cfg, T=0) == gdn.GDN_ERR_INVALID_ARGUMENT
        assert call(L, cfg, T=17) == gdn.GDN_ERR_UNSUPPORTED
        assert call(L, cfg, B=-2) == gdn.GDN_ERR_INVALID_ARGUMENT
        assert call(L, cfg, pool=0) == gdn.GDN_ERR_INVALID_ARGUMENT
        assert call(L, cfg, B=0, ptrs=[None] * (10 if call is spec_verify else 8)) == gdn.GDN_OK
        assert call(L, cfg, err=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    for i in range(3):
        spec = [FAKE] * 3
        spec[i] = None
        assert spec_verify(L, cfg, spec=spec) == gdn.GDN_ERR_INVALID_ARGUMENT, i
        spec[i] = FAKE_ODD
        assert spec_verify(L, cfg, spec=spec) == gdn.GDN_ERR_MISALIGNED, i
    for i in range(10):
        ptrs = [FAKE] * 10
        ptrs[i] = FAKE_ODD
        assert spec_verify(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_MISALIGNED, i
    for i in range(8):
        ptrs = [FAKE] * 8
        ptrs[i] = None
        assert spec_commit(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_INVALID_ARGUMENT, i
        ptrs[i] = FAKE_ODD
        assert spec_commit(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_MISALIGNED, i


def test_device_batch_entry_point_checks_arguments_on_the_host(L):
    cfg = good_cfg()

    def call(bdev=FAKE, B=4, T=1, ptrs=None, ws=None):
        p = [FAKE] * 10 if ptrs is None else ptrs
        return L.gdn_decode_step_device_batch(ctypes.byref(cfg), bdev, B, T, *p, 8, FAKE, FAKE, None, None, ws, None)
    assert call(bdev=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert call(bdev=ctypes.c_void_p((1 << 20) + 2)) == gdn.GDN_ERR_MISALIGNED
    assert call(bdev=ctypes.c_void_p((1 << 20) + 4)) != gdn.GDN_ERR_MISALIGNED  # 4-byte aligned is enough
    assert call(B=0, bdev=None, ptrs=[None] * 10) == gdn.GDN_OK           # B_max = 0: nothing to launch
    assert call(T=17) == gdn.GDN_ERR_UNSUPPORTED
    assert call(ws=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    for i in range(10):
        ptrs = [FAKE] * 10
        ptrs[i] = None
        assert call(ptrs=ptrs) == gdn.GDN_ERR_INVALID_ARGUMENT, i


def test_selftest_checks_arguments_on_the_host(L):
    assert L.gdn_selftest_wait_timeout(1000, None, None, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert L.gdn_selftest_wait_timeout(0, FAKE, None, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert L.gdn_selftest_wait_timeout(1 << 41, FAKE, None, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert L.gdn_selftest_wait_timeout(1000, ctypes.c_void_p((1 << 20) + 2), None, None) == gdn.GDN_ERR_MISALIGNED
    assert L.gdn_selftest_wait_timeout(1000, FAKE, ctypes.c_void_p((1 << 20) + 4), None) == gdn.GDN_ERR_MISALIGNED


def test_empty_batch_is_a_no_op(L):
    # B = 0 returns before any pointer is looked at or any launch is made
    assert decode(L, good_cfg(), B=0, ptrs=[None] * 10) == gdn.GDN_OK
    assert L.gdn_conv_update(ctypes.byref(good_cfg()), 0, 1, *([None] * 3), 4, *([None] * 6)) == gdn.GDN_OK
    assert L.gdn_gated_rmsnorm(ctypes.byref(good_cfg()), 0, *([None] * 5), None) == gdn.GDN_OK


def test_stage_entry_points_check_arguments(L):
    cfg = good_cfg()
    assert L.gdn_conv_update(ctypes.byref(cfg), 2, 1, FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, FAKE, None,
                             None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert L.gdn_conv_update(ctypes.byref(good_cfg(conv_width=12)), 2, 1, *([FAKE] * 3), 4,
                             *([FAKE] * 4), None, None) == gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_recurrent_step(ctypes.byref(cfg), 2, 1, *([FAKE] * 7), FAKE_ODD, 4, FAKE, FAKE, None,
                                None) == gdn.GDN_ERR_MISALIGNED
    assert L.gdn_recurrent_step(ctypes.byref(cfg), 2, 20, *([FAKE] * 8), 4, FAKE, FAKE, None,
                                None) == gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_gated_rmsnorm(ctypes.byref(cfg), -1, *([FAKE] * 4), None, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert L.gdn_gated_rmsnorm(ctypes.byref(cfg), 4, FAKE, FAKE, None, FAKE, None,
                               None) == gdn.GDN_ERR_INVALID_ARGUMENT


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    cfg = good_cfg(num_k_heads=1, num_v_heads=1, head_k_dim=16, head_v_dim=16)
    x = torch.zeros(1, 1, cfg.channels, dtype=torch.bfloat16)
    with pytest.raises((ValueError, TypeError)):
        gdn.gdn_decode_step(cfg, x, x, x, x, x, x, x, x, x, x, x, x)


def varlen(L, cfg, B=4, cu=FAKE, T_max=16, total=40, ptrs=None, pool=8, out_f32=None, err=None):
    # qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool; then slots, out
    p = [FAKE] * 10 if ptrs is None else ptrs
    return L.gdn_decode_step_varlen(ctypes.byref(cfg), B, cu, T_max, total, *p, pool, FAKE, FAKE, out_f32, err,
                                    None)


def test_varlen_checks_its_arguments_on_the_host(L):
    cfg = good_cfg()
    assert varlen(L, good_cfg(head_k_dim=96)) == gdn.GDN_ERR_UNSUPPORTED
    assert varlen(L, cfg, B=-1) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert varlen(L, cfg, T_max=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert varlen(L, cfg, T_max=17) == gdn.GDN_ERR_UNSUPPORTED
    assert varlen(L, cfg, total=-1) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert varlen(L, cfg, cu=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert varlen(L, cfg, cu=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED        # int32 offsets: 4-byte aligned
    assert varlen(L, cfg, pool=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    for i in range(10):
        ptrs = [FAKE] * 10
        ptrs[i] = None
        assert varlen(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_INVALID_ARGUMENT, i
        ptrs[i] = FAKE_ODD
        assert varlen(L, cfg, ptrs=ptrs) == gdn.GDN_ERR_MISALIGNED, i
    assert varlen(L, cfg, out_f32=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED
    assert varlen(L, cfg, err=FAKE_ODD) == gdn.GDN_ERR_MISALIGNED


def test_varlen_without_tokens_is_a_no_op(L):
    # no sequence, or no token at all: returns before any pointer is looked at or any launch
    assert varlen(L, good_cfg(), B=0, cu=None, ptrs=[None] * 10) == gdn.GDN_OK
    assert varlen(L, good_cfg(), total=0, cu=None, ptrs=[None] * 10) == gdn.GDN_OK


def test_a_plain_c_program_builds_against_the_header_and_library(tmp_path, L):
    """The boundary is plain C: a C99 program includes gdn.h, links libgdn.so and calls
    the entry points that need no GPU (status strings, ABI version, host slot check, an
    argument check that fails before any launch)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_gdn.c"
    src.write_text(r'''
#include <stdio.h>
#include "gdn.h"
int main(void) {
    const int32_t slots[3] = {0, 2, 1};
    gdn_config cfg = {16, 32, 128, 128, 4, 1e-6f, 1e-6f, 0.0f};
    if (gdn_abi_version() != GDN_ABI_VERSION) return 1;
    if (gdn_check_slots_host(slots, 3, 3) != GDN_OK) return 2;
    if (gdn_decode_step(&cfg, 2, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 4, 0, 0, 0, 0, 0, 0) !=
        GDN_ERR_INVALID_ARGUMENT) return 3;                    /* T = 0: rejected on the host */
    printf("%s\n", gdn_status_string(GDN_ERR_MISALIGNED));
    return 0;
}
''')
    libdir = os.path.dirname(gdn.LIB_PATH)
    exe = tmp_path / "use_gdn"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, str(src), "-o", str(exe),
                    "-L", libdir, "-lgdn", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip() == gdn.status_string(gdn.GDN_ERR_MISALIGNED)
