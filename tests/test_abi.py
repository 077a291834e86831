"""The C-ABI library: it loads without a GPU, exports every function the
header declares, its structs match ctypes' view, and host-side validation
rejects bad arguments before anything is launched (no GPU needed)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import long_context_prefill_last_b200 as crisp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "crisp.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from long_context_prefill_last_b200 import build
    build.build()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(crisp_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = header_functions()
    assert sorted(names) == sorted(crisp.SYMBOLS)
    L = crisp.lib()
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", crisp.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(crisp_\w+)", out))
    assert set(names) <= exported


def test_library_has_sm100a_code_and_no_undefined_cuda_driver_link():
    out = subprocess.run(["ldd", crisp.library_path()], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out        # driver entry points are resolved at run time
    assert "libcudart" not in out          # runtime is linked statically


def test_struct_layout_matches_header():
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "crisp.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu\n", sizeof(crisp_cfg), offsetof(crisp_cfg, tau_proxy),
             offsetof(crisp_cfg, workspace), offsetof(crisp_cfg, workspace_bytes), sizeof(crisp_index));
      return 0;
    }"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True).stdout.split()]
    assert vals == [ctypes.sizeof(crisp._Cfg), crisp._Cfg.tau_proxy.offset, crisp._Cfg.workspace.offset,
                    crisp._Cfg.workspace_bytes.offset, ctypes.sizeof(crisp._Index)]


def test_cfg_init_defaults_match_python_config():
    c = crisp._Cfg()
    assert crisp.lib().crisp_cfg_init(ctypes.byref(c), 32768, 32, 8, 128, crisp.BF16) == 0
    py = crisp.Config(n=32768, h_q=32, h_kv=8)._c()
    for f, _ in crisp._Cfg._fields_:
        assert getattr(c, f) == pytest.approx(getattr(py, f)), f


def test_workspace_size_and_dims():
    cfg = crisp.Config(n=524288, h_q=32, h_kv=8)
    nb, w = crisp.index_dims(cfg)
    assert (nb, w) == (4096, 128)
    ws = crisp.workspace_size(cfg)
    # the proxy partials (two floats per proxy row and key tile) and the bf16
    # hi/lo pooled queries dominate; the pooled map itself is never stored
    partials = 2 * 32 * 64 * 4096 * 4
    pooled_q = 2 * 32 * 4096 * 128 * 2
    assert partials + pooled_q < ws < 300 * 2 ** 20


@pytest.mark.parametrize("field,value,code", [
    ("n", 1000, "CRISP_ERR_SHAPE"), ("n", 256, "CRISP_ERR_SHAPE"), ("n", 4095, "CRISP_ERR_SHAPE"),
    ("d", 64, "CRISP_ERR_SHAPE"), ("h_kv", 3, "CRISP_ERR_SHAPE"), ("h_q", 0, "CRISP_ERR_SHAPE"),
    ("dtype", 7, "CRISP_ERR_DTYPE"), ("block", 64, "CRISP_ERR_UNSUPPORTED"),
    ("last_q", 128, "CRISP_ERR_UNSUPPORTED"), ("w_sink", 64, "CRISP_ERR_UNSUPPORTED"),
    ("gamma", 0.0, "CRISP_ERR_INVALID_ARG"), ("gamma", 1.5, "CRISP_ERR_INVALID_ARG"),
    ("alpha", -1.0, "CRISP_ERR_INVALID_ARG"), ("tau_proxy", float("nan"), "CRISP_ERR_INVALID_ARG"),
    ("force_route", 2, "CRISP_ERR_INVALID_ARG"), ("reserved", 1, "CRISP_ERR_INVALID_ARG"),
])
def test_invalid_configs_are_rejected_on_the_host(field, value, code):
    cfg = crisp.Config(n=4096, h_q=4, h_kv=2)
    setattr(cfg, field, value)
    with pytest.raises(crisp.CrispError) as e:
        crisp.workspace_size(cfg)
    assert crisp.STATUS_NAMES[e.value.code] == code


class _FakeTensor:
    def __init__(self, ptr, nbytes=0):
        self.ptr, self.nbytes = ptr, nbytes

    def data_ptr(self):
        return self.ptr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


def test_bad_pointers_and_workspace_fail_before_any_launch():
    L = crisp.lib()
    cfg = crisp.Config(n=4096, h_q=4, h_kv=2)
    c = cfg._c()
    # no workspace
    assert L.crisp_prefill(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(c), None) == 5
    # null tensor
    assert L.crisp_prefill(0, 0x20000, 0x30000, 0x40000, ctypes.byref(c), None) == 1
    # misaligned tensor
    assert L.crisp_dense_attention(0x10008, 0x20000, 0x30000, 0x40000, ctypes.byref(c), None) == 4
    # workspace too small / misaligned
    cfg.workspace = _FakeTensor(0x100000, 1024)
    assert L.crisp_prefill(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(cfg._c()), None) == 5
    cfg.workspace = _FakeTensor(0x100010, 1 << 40)
    assert L.crisp_route(0x10000, 0x20000, ctypes.byref(cfg._c()), 0x5000, 0x6000, None) == 4
    # route outputs missing
    cfg.workspace = _FakeTensor(0x100000, 1 << 40)
    assert L.crisp_route(0x10000, 0x20000, ctypes.byref(cfg._c()), 0, 0x6000, None) == 1
    # select without an index
    assert L.crisp_select(0x10000, 0x20000, ctypes.byref(cfg._c()), None, None) == 1


def test_route_noalloc_rejects_layers_beyond_its_static_scratch_before_any_launch():
    L = crisp.lib()
    big = crisp.Config(n=524288, h_q=32, h_kv=8)._c()
    assert L.crisp_route_noalloc(0x10000, 0x20000, ctypes.byref(big), 0x30000, 0x40000, None) == 11
    assert crisp.STATUS_NAMES[11] == "CRISP_ERR_TOO_LARGE"
    assert "too large" in crisp.status_string(11)
    small = crisp.Config(n=4096, h_q=4, h_kv=2)._c()
    assert L.crisp_route_noalloc(0, 0x20000, ctypes.byref(small), 0x30000, 0x40000, None) == 1
    assert L.crisp_route_noalloc(0x10008, 0x20000, ctypes.byref(small), 0x30000, 0x40000, None) == 4


def test_status_strings():
    assert crisp.status_string(0) == "ok"
    assert "timed out" in crisp.status_string(9)
    assert crisp.lib().crisp_version() >= 100


def test_batch_and_varlen_validation_before_any_launch():
    L = crisp.lib()
    one = crisp.Config(n=4096, h_q=8, h_kv=2)
    # a batch of b sequences needs the workspace of the folded shape
    for b in (1, 2, 3):
        folded = crisp.Config(n=4096, h_q=8 * b, h_kv=2 * b)
        assert crisp.workspace_size_batch(one, b) == crisp.workspace_size(folded)
    out = ctypes.c_size_t(0)
    assert L.crisp_workspace_size_batch(ctypes.byref(one._c()), 0, ctypes.byref(out)) == 1
    assert L.crisp_prefill_batch(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(one._c()), 0, None) == 1
    # the folded shape obeys the single-call limits (h_q <= 1024)
    assert L.crisp_prefill_batch(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(one._c()), 129, None) == 2
    # without a workspace: rejected before anything runs
    assert L.crisp_prefill_batch(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(one._c()), 2, None) == 5

    vp = ctypes.c_void_p
    arr = vp * 2
    q, k, v, o = arr(0x10000, 0x50000), arr(0x20000, 0x60000), arr(0x30000, 0x70000), arr(0x40000, 0x80000)
    cfg = crisp.Config(n=4096, h_q=8, h_kv=2)
    cfg.workspace = _FakeTensor(0x100000, 1 << 40)
    c = cfg._c()
    n_ok = (ctypes.c_int32 * 2)(4096, 2048)
    n_bad = (ctypes.c_int32 * 2)(4096, 1000)       # not a multiple of 128
    fn = L.crisp_prefill_varlen
    assert fn(q, k, v, o, n_ok, 0, ctypes.byref(c), None) == 1            # no sequences
    assert fn(None, k, v, o, n_ok, 2, ctypes.byref(c), None) == 1         # missing array
    assert fn(q, k, v, o, None, 2, ctypes.byref(c), None) == 1            # missing lengths
    assert fn(q, k, v, o, n_bad, 2, ctypes.byref(c), None) == 2           # second length invalid: nothing runs
    q_bad = arr(0x10000, 0x50008)                                         # second q misaligned
    assert fn(q_bad, k, v, o, n_ok, 2, ctypes.byref(c), None) == 4
    small = crisp.Config(n=2048, h_q=8, h_kv=2)
    small.workspace = _FakeTensor(0x100000, crisp.workspace_size(small))  # too small for n=4096
    assert fn(q, k, v, o, n_ok, 2, ctypes.byref(small._c()), None) == 5


def test_host_prefill_workspace_and_validation_before_any_launch():
    L = crisp.lib()
    cfg = crisp.Config(n=4096, h_q=8, h_kv=2)
    group = crisp.Config(n=4096, h_q=4, h_kv=1)
    per_group = lambda nbytes: (nbytes + 255) // 256 * 256
    q_bytes, kv_bytes = 4 * 4096 * 128 * 2, 4096 * 128 * 2
    slots = 2 * (2 * per_group(q_bytes) + 2 * per_group(kv_bytes))
    assert crisp.workspace_size_host(cfg) == per_group(crisp.workspace_size(group)) + slots
    c = cfg._c()
    # no workspace, null host buffer, misaligned host buffer, same stream twice
    assert L.crisp_prefill_host(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(c), None, 0x1) == 5
    assert L.crisp_prefill_host(0, 0x20000, 0x30000, 0x40000, ctypes.byref(c), None, 0x1) == 1
    assert L.crisp_prefill_host(0x10004, 0x20000, 0x30000, 0x40000, ctypes.byref(c), None, 0x1) == 4
    cfg.workspace = _FakeTensor(0x100000, crisp.workspace_size_host(cfg))
    assert L.crisp_prefill_host(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(cfg._c()), 0x7, 0x7) == 1
    cfg.workspace = _FakeTensor(0x100000, crisp.workspace_size_host(cfg) - 256)
    assert L.crisp_prefill_host(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(cfg._c()), None, 0x1) == 5


def test_wait_selftest_validates_before_launch():
    L = crisp.lib()
    assert L.crisp_wait_selftest(10, 0x10000, None) == 1          # limit below 1000 cycles
    assert L.crisp_wait_selftest(5_000_000_000, 0x10000, None) == 1
    assert L.crisp_wait_selftest(1_000_000, 0, None) == 1         # no status buffer
