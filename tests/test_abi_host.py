"""Host-only checks of the C ABI: the library loads without a GPU, exports every
function ``include/attn.h`` declares, and rejects bad arguments before touching
the device."""

import ctypes
import os
import re

import pytest

import attention_forward_flash_b200 as afb
from attention_forward_flash_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_function():
    L = afb.lib()
    names = _declared_functions()
    assert "attn_forward" in names and "attn_create" in names and "attn_quantize_qk" in names
    for name in names:
        assert hasattr(L, name), name
    assert set(names) <= set(_abi.EXPORTED)


def _params(**kw):
    base = dict(batch=1, n_q_heads=2, n_kv_heads=2, q_len=256, kv_len=256, head_dim=64,
                start_pos=0, causal=0, window_lo=0, scale=0.0, dtype=0, precision=0, num_splits=0)
    base.update(kw)
    return _abi.AttnParams(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(n_q_heads=3, n_kv_heads=2), _abi.ATTN_ERR_INVALID_ARG),
    (dict(batch=0), _abi.ATTN_ERR_INVALID_ARG),
    (dict(q_len=-1), _abi.ATTN_ERR_INVALID_ARG),
    (dict(kv_len=-5), _abi.ATTN_ERR_INVALID_ARG),
    (dict(start_pos=-1), _abi.ATTN_ERR_INVALID_ARG),
    (dict(window_lo=-1), _abi.ATTN_ERR_INVALID_ARG),
    (dict(window_size=-1), _abi.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), _abi.ATTN_ERR_INVALID_ARG),
    (dict(dtype=7), _abi.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _abi.ATTN_ERR_INVALID_ARG),
    (dict(num_splits=-1), _abi.ATTN_ERR_INVALID_ARG),
    (dict(num_splits=100000), _abi.ATTN_ERR_INVALID_ARG),
    (dict(head_dim=96), _abi.ATTN_ERR_UNSUPPORTED),
    (dict(head_dim=256), _abi.ATTN_ERR_UNSUPPORTED),
    (dict(precision=4), _abi.ATTN_ERR_INVALID_ARG),
    (dict(precision=3, head_dim=128), _abi.ATTN_ERR_UNSUPPORTED),   # FP4: head_dim 64 only
    (dict(precision=3, rope_dim=64), _abi.ATTN_ERR_UNSUPPORTED),
    (dict(precision=3, num_splits=2), _abi.ATTN_ERR_INVALID_ARG),    # single-pass modes
    (dict(precision=2, num_splits=2), _abi.ATTN_ERR_INVALID_ARG),
    (dict(precision=2, rope_dim=64), _abi.ATTN_ERR_UNSUPPORTED),
    # size limits: stacked rows and positions below 2^30, 32-bit grid and block counts,
    # and the quantisers' units on gridDim.y
    (dict(n_q_heads=64, n_kv_heads=1, q_len=1 << 25), _abi.ATTN_ERR_UNSUPPORTED),
    (dict(start_pos=(1 << 30) - 100, q_len=101), _abi.ATTN_ERR_UNSUPPORTED),
    (dict(batch=1 << 20, n_q_heads=1 << 11, n_kv_heads=1 << 11, q_len=1),
     _abi.ATTN_ERR_UNSUPPORTED),
    (dict(batch=1 << 16, n_q_heads=1 << 8, n_kv_heads=1 << 8, q_len=1, kv_len=1 << 16),
     _abi.ATTN_ERR_UNSUPPORTED),
    (dict(precision=1, batch=65536, n_q_heads=1, n_kv_heads=1, q_len=16, kv_len=16),
     _abi.ATTN_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_params_before_any_device_call(kw, status):
    L = afb.lib()
    ctx = ctypes.c_void_p(1234)
    p = _params(**kw)
    assert L.attn_create(ctypes.byref(p), ctypes.byref(ctx)) == status
    assert ctx.value is None  # *out is cleared on failure


def test_null_arguments():
    L = afb.lib()
    assert L.attn_create(None, None) == _abi.ATTN_ERR_INVALID_ARG
    p = _params()
    assert L.attn_create(ctypes.byref(p), None) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_forward(None, None, None, None, None, None, None, None) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_quantize_qk(None, None, None, None, None, None) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_forward_host(*([None] * 12), 0, None) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_forward_paged(*([None] * 5), 0, None, None, None) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_get_error(None, None) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_debug_set(None, 0) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_num_splits(None) == 0
    assert L.attn_kernel_path(None) == 0
    assert L.attn_quantize_qk_paged(*([None] * 5), 0, None, None) == _abi.ATTN_ERR_INVALID_ARG
    L.attn_destroy(None)


def test_status_strings():
    for s in range(6):
        assert isinstance(afb.attn_status_string(s), str) and afb.attn_status_string(s)
    assert afb.attn_status_string(99) == "unknown status"


def test_qbufs_sizes():
    p = _params(batch=2, n_q_heads=8, n_kv_heads=2, q_len=300, kv_len=4133, head_dim=128)
    q, k, qs, ks, vt, vs = afb.attn_qbufs_sizes(p)
    assert q == 2 * 8 * 300 * 128 and k == 2 * 2 * 4133 * 128
    assert qs == 2 * 8 * 3 * 4 and ks == 2 * 2 * 33 * 4
    assert vt == 2 * 2 * 128 * 33 * 128 and vs == 2 * 2 * 128 * 4
    with pytest.raises(afb.AttnError):
        afb.attn_qbufs_sizes(_params(head_dim=80))
    # FP4 mode: packed codes, no FP32 Q/K scales, E8M0 chunks per 128 rows (Q's rows
    # stacked per unit and rounded to an even tile count)
    p4 = _params(batch=2, n_q_heads=8, n_kv_heads=2, q_len=300, kv_len=4133, head_dim=64,
                 precision=3)
    q, k, qs, ks, vt, vs = afb.attn_qbufs_sizes(p4)
    assert q == 2 * 8 * 300 * 32 and k == 2 * 2 * 4133 * 32 and qs == ks == 0
    assert vt == 2 * 2 * 64 * 33 * 128 and vs == 2 * 2 * 64 * 4
    from attention_forward_flash_b200 import _abi as abi
    qsf, ksf = abi.attn_qbufs_sf_sizes(p4)
    assert qsf == 4 * (2 * ((4 * 300 + 255) // 256)) * 512 and ksf == 4 * 33 * 512
    assert abi.attn_qbufs_sf_sizes(_params()) == [0, 0]


C_CALLER = r"""
#include <stddef.h>
#include <stdint.h>
#include "attn.h"

/* Every declared function, called with the argument types the header states. */
int main(void) {
  attn_params p = {1, 2, 2, 256, 256, 64, 0, 0, 0, 0.0f, ATTN_BF16, ATTN_EXACT, 0, 0, 0, 0, 0};
  attn_ctx *c = NULL;
  attn_qbufs qb = {0};
  size_t sizes[6];
  unsigned err = 0;
  int32_t table[2] = {0, 1};
  if (attn_create(&p, &c) != ATTN_OK) return 1;
  attn_quantize_qk(c, NULL, NULL, NULL, &qb, NULL);
  attn_forward(c, NULL, NULL, NULL, NULL, NULL, NULL, NULL);
  attn_forward_host(c, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0,
                    NULL);
  attn_forward_paged(c, NULL, NULL, NULL, table, 1, NULL, NULL, NULL);
  attn_get_error(c, NULL);
  attn_qbufs_sizes(&p, sizes);
  attn_qbufs_sf_sizes(&p, sizes);
  attn_num_splits(c);
  if (attn_kernel_path(c) == ATTN_PATH_DECODE) return 2;
  attn_quantize_qk_paged(c, NULL, NULL, NULL, table, 1, &qb, NULL);
  attn_plan plan;
  if (attn_plan_for(&p, 148, &plan) != ATTN_OK || plan.path != ATTN_PATH_SINGLE_PASS) return 3;
  attn_debug_set(c, 0u);
  attn_debug_exp2(NULL, NULL, 0, NULL);
  attn_forward_splitkv_noalloc(&p, NULL, NULL, NULL, NULL, NULL, &err, NULL);
  attn_rope_freq f = {10000.0f, ATTN_ROPE_YARN, 4.0f, 4096, 32.0f, 1.0f};
  float rope[2 * 64];
  attn_rope_table(64, 2, &f, rope);
  attn_set_rope_table(c, NULL, 0);
  attn_rope_apply(c, NULL, NULL, 1, 0, 0, NULL);
  (void)attn_status_string(ATTN_OK);
  attn_destroy(c);
  return 0;
}
"""


def test_header_is_plain_c_and_links_against_the_library(tmp_path):
    """include/attn.h compiles as C99 with warnings as errors, and a C program that
    calls every declared function links against libattn.so (it is not run: that
    needs a GPU)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    called = set(re.findall(r"\b(attn_\w+)\s*\(", C_CALLER))
    assert called >= set(_declared_functions())
    lib_dir = os.path.dirname(afb.lib_path())
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o",
                        str(tmp_path / "caller"), "-L", lib_dir, "-lattn",
                        "-Wl,--unresolved-symbols=ignore-in-shared-libs"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_noalloc_rejects_one_split_before_any_device_call():
    # The split-free entry always splits: num_splits must be 0 (library's choice) or > 1.
    L = afb.lib()
    p = _params(q_len=4, kv_len=4096, num_splits=1)
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: the call returns first
    status = L.attn_forward_splitkv_noalloc(ctypes.byref(p), fake, fake, fake, fake, None, None,
                                            None)
    assert status == _abi.ATTN_ERR_INVALID_ARG


DEVICE_ONCE_TEST = r"""
#include <cstdio>
#include <initializer_list>
#include "device_once.h"

int main() {
  attn::PerDeviceOnce<8> once;
  int calls[8] = {0};
  bool fail_next = true;
  auto setup = [&](int dev) {
    return [&, dev] {
      ++calls[dev];
      if (dev == 3 && fail_next) { fail_next = false; return false; }
      return true;
    };
  };
  // The first use on each device runs the set-up; later uses on that device do not.
  for (int rep = 0; rep < 3; ++rep)
    for (int dev : {0, 1, 0, 2, 1}) if (!once.ensure(dev, setup(dev))) return 10 + dev;
  if (calls[0] != 1 || calls[1] != 1 || calls[2] != 1) return 2;
  // A failed set-up is not remembered: the next use on that device runs it again.
  if (once.ensure(3, setup(3))) return 3;
  if (once.done(3)) return 4;
  if (!once.ensure(3, setup(3)) || calls[3] != 2 || !once.done(3)) return 5;
  // Devices outside the table are refused without running the set-up.
  int outside = 0;
  if (once.ensure(8, [&] { ++outside; return true; }) || outside != 0) return 6;
  if (once.ensure(-1, [&] { ++outside; return true; }) || outside != 0) return 7;
  std::puts("ok");
  return 0;
}
"""


def test_kernel_attributes_are_kept_per_device(tmp_path):
    """The flag behind every kernel's shared-memory attribute is keyed by device
    ordinal: set-up runs once per device, failures are retried, and out-of-range
    devices are refused (host logic, compiled with g++ against the library's header)."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler")
    src = tmp_path / "device_once_test.cc"
    src.write_text(DEVICE_ONCE_TEST)
    exe = tmp_path / "device_once_test"
    csrc = os.path.join(ROOT, "attention_forward_flash_b200", "csrc")
    r = subprocess.run([gxx, "-std=c++17", "-Wall", "-Werror", "-I", csrc, str(src), "-o",
                        str(exe), "-pthread"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout)
    # and the library uses it for every launch that raises the shared-memory limit
    api = open(os.path.join(csrc, "attn_api.cu")).read()
    assert "PerDeviceOnce" in api and "static bool" not in api
