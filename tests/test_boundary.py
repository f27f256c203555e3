"""The C ABI without a GPU: the library loads, exports every entry point declared in
include/twl.h, sizes workspaces, and rejects bad arguments on the host with the documented status
before launching anything.  Pointers here are fake addresses: every call below fails validation
before any CUDA call, so nothing is dereferenced."""
import ctypes as C
import os
import re
import shutil
import subprocess
import sys

import numpy as np
import pytest

from adaptive_top_sparse_b200 import twl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "twl.h")

A = 1 << 20          # a fake, 256-byte aligned address


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:twl_status|size_t|const char\*|void)\s+(twl_\w+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ["twl_quantize_k", "twl_page_bounds", "twl_select_pages", "twl_estimate",
                 "twl_prune_top_p", "twl_group_union", "twl_sparse_decode", "twl_decode_step",
                 "twl_workspace_bytes", "twl_workspace_init", "twl_device_status",
                 "twl_status_string"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(twl.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing
    # the binding lists exactly the declared entry points and wraps each under the same name
    assert set(declared_symbols()) == set(twl.EXPORTED)
    assert all(callable(getattr(twl, s, None)) for s in declared_symbols())


def test_status_strings():
    for code in range(twl.TWL_ERR_SCRATCH_LIMIT, 1):
        assert twl.twl_status_string(code) != "unknown status"
    assert twl.twl_status_string(-99) == "unknown status"


def test_package_without_the_library_fails_at_import(tmp_path):
    """The Python side has no fallback: a copy of the package without libtwl.so refuses to
    import, both the binding and the layer wrapper built on it."""
    src = os.path.join(ROOT, "adaptive_top_sparse_b200")
    dst = tmp_path / "adaptive_top_sparse_b200"
    dst.mkdir()
    for name in os.listdir(src):
        if name.endswith(".py"):
            shutil.copy(os.path.join(src, name), dst / name)
    for mod in ("twl", "layer"):
        r = subprocess.run([sys.executable, "-c", f"import adaptive_top_sparse_b200.{mod}"],
                           cwd=tmp_path, capture_output=True, text=True, timeout=300,
                           env=dict(os.environ, PYTHONPATH=str(tmp_path)))
        assert r.returncode != 0, mod
        assert "ImportError" in r.stderr and "libtwl.so is missing" in r.stderr, r.stderr[-500:]


def test_package_never_imports_the_oracle():
    """The oracle is test infrastructure: nothing in the package imports or opens it."""
    pkg = os.path.join(ROOT, "adaptive_top_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for name in files:
            if name.endswith((".py", ".cu", ".h", ".cuh")):
                text = open(os.path.join(dirpath, name)).read()
                assert not re.search(r"\boracle\b", text), os.path.join(dirpath, name)


def _kv(**over):
    d = dict(k=A, v=A + 4096, page_table=A + 8192, seq_lens=A + 12288, batch=2, num_kv_heads=8,
             head_dim=128, page_size=16, max_pages=64, num_phys_pages=128)
    d.update(over)
    return twl._PagedKV(d["k"], d["v"], d["page_table"], d["seq_lens"], d["batch"],
                        d["num_kv_heads"], d["head_dim"], d["page_size"], d["max_pages"],
                        d["num_phys_pages"])


def _select(kv=None, hq=32, budget_pages=0, budget_div=4, max_budget=16, ws=A, ws_bytes=1 << 30,
            q=A, bounds=A, sel=A, cnt=A):
    kv = kv or _kv()
    return twl._lib.twl_select_pages(q, hq, C.byref(kv), bounds, budget_pages, budget_div,
                                     max_budget, sel, cnt, None, ws, ws_bytes, None)


@pytest.mark.parametrize("over,code", [
    (dict(head_dim=64), twl.TWL_ERR_UNSUPPORTED),
    (dict(page_size=32), twl.TWL_ERR_UNSUPPORTED),
    (dict(max_pages=40000), twl.TWL_ERR_UNSUPPORTED),
    (dict(batch=0), twl.TWL_ERR_INVALID_ARG),
    (dict(num_kv_heads=0), twl.TWL_ERR_INVALID_ARG),
    (dict(page_table=0), twl.TWL_ERR_INVALID_ARG),
    (dict(seq_lens=0), twl.TWL_ERR_INVALID_ARG),
    (dict(page_table=A + 2), twl.TWL_ERR_INVALID_ARG),
])
def test_select_rejects_bad_cache(over, code):
    assert _select(kv=_kv(**over)) == code


@pytest.mark.parametrize("kw,code", [
    (dict(hq=12), twl.TWL_ERR_UNSUPPORTED),        # group of 12 / 8: not an integer
    (dict(hq=24), twl.TWL_ERR_UNSUPPORTED),        # group 3
    (dict(hq=128), twl.TWL_ERR_UNSUPPORTED),       # group 16
    (dict(q=0), twl.TWL_ERR_INVALID_ARG),
    (dict(q=A + 8), twl.TWL_ERR_INVALID_ARG),      # q must be 16-byte aligned
    (dict(bounds=0), twl.TWL_ERR_INVALID_ARG),
    (dict(sel=0), twl.TWL_ERR_INVALID_ARG),
    (dict(max_budget=15), twl.TWL_ERR_INVALID_ARG),  # ceil(64 / 4) = 16 needed
    (dict(max_budget=65), twl.TWL_ERR_INVALID_ARG),
    (dict(budget_div=0), twl.TWL_ERR_INVALID_ARG),
    (dict(budget_pages=-1), twl.TWL_ERR_INVALID_ARG),
    (dict(budget_pages=8, max_budget=7), twl.TWL_ERR_INVALID_ARG),
    (dict(ws=0), twl.TWL_ERR_WORKSPACE),
    (dict(ws=A + 64), twl.TWL_ERR_WORKSPACE),
    (dict(ws_bytes=1024), twl.TWL_ERR_WORKSPACE),
])
def test_select_rejects_bad_arguments(kw, code):
    if kw.get("hq") == 12:
        assert _select(**kw) == twl.TWL_ERR_INVALID_ARG
        return
    assert _select(**kw) == code


@pytest.mark.parametrize("p,eps", [(0.0, 1e-6), (-0.5, 1e-6), (1.5, 1e-6), (float("nan"), 1e-6),
                                   (0.9, 0.0), (0.9, -1e-6), (0.9, float("inf")),
                                   (0.9, float("nan"))])
def test_prune_rejects_bad_p_eps(p, eps):
    st = twl._lib.twl_prune_top_p(A, None, 4, 1024, p, eps, A, A, None, None, 0, None)
    assert st == twl.TWL_ERR_INVALID_ARG


def test_prune_rejects_null_and_empty_is_ok():
    assert twl._lib.twl_prune_top_p(0, None, 4, 16, 0.9, 1e-6, A, A, None, None, 0, None) == -1
    assert twl._lib.twl_prune_top_p(A, None, 4, 0, 0.9, 1e-6, A, A, None, None, 0, None) == -1
    assert twl._lib.twl_prune_top_p(A, None, -1, 16, 0.9, 1e-6, A, A, None, None, 0, None) == -1
    # zero rows: nothing to do, nothing launched
    assert twl._lib.twl_prune_top_p(A, None, 0, 16, 0.9, 1e-6, A, A, None, None, 0, None) == 0


def test_decode_step_rejects_bad_arguments():
    kv = _kv()
    aux = twl._KAux(A, A, A)
    f = twl._lib.twl_decode_step

    def call(q=A, aux_=aux, p=0.85, eps=1e-6, o=A, lse=A, ws=A, ws_bytes=1 << 40, kvv=kv,
             max_budget=16):
        return f(q, 32, C.byref(kvv), C.byref(aux_), 0, 4, max_budget, p, eps, o, lse, None, ws,
                 ws_bytes, None)

    assert call(p=0.0) == twl.TWL_ERR_INVALID_ARG
    assert call(eps=0.0) == twl.TWL_ERR_INVALID_ARG
    assert call(o=0) == twl.TWL_ERR_INVALID_ARG
    assert call(o=A + 4) == twl.TWL_ERR_INVALID_ARG
    assert call(aux_=twl._KAux(A, 0, A)) == twl.TWL_ERR_INVALID_ARG
    assert call(kvv=_kv(v=0)) == twl.TWL_ERR_INVALID_ARG
    assert call(ws_bytes=100) == twl.TWL_ERR_WORKSPACE
    assert call(max_budget=3) == twl.TWL_ERR_INVALID_ARG
    assert call(kvv=_kv(max_pages=40000)) == twl.TWL_ERR_UNSUPPORTED   # > 512K tokens
    assert call(kvv=_kv(head_dim=64)) == twl.TWL_ERR_UNSUPPORTED


def test_sparse_decode_rejects_bad_arguments():
    kv = _kv()
    f = twl._lib.twl_sparse_decode
    assert f(A, 32, C.byref(kv), A, A, 0, 0.088, A, A, A, 1 << 30, None) == -1   # tok_stride 0
    assert f(A, 32, C.byref(kv), A, A, 64, 0.0, A, A, A, 1 << 30, None) == -1    # sm_scale 0
    assert f(A, 32, C.byref(kv), A, A, 64, 0.088, A, A, A, 16, None) == -5       # workspace


def test_cache_calls_reject_bad_arguments():
    kv = _kv()
    assert twl._lib.twl_page_bounds(C.byref(kv), 0, None, 0, None) == -1
    assert twl._lib.twl_page_bounds(C.byref(kv), A + 2, None, 0, None) == -1
    assert twl._lib.twl_quantize_k(C.byref(kv), A, 0, None, 0, None) == -1
    assert twl._lib.twl_quantize_k(C.byref(_kv(k=0)), A, A, None, 0, None) == -1
    assert twl._lib.twl_page_bounds(C.byref(kv), A, A, 16, None) == -5


def test_estimate_and_union_reject_bad_arguments():
    kv = _kv()
    est = twl._lib.twl_estimate

    def e(q=A, k4=A, sz=A, sel=A, cnt=A, mb=16, w=A, tok=A, cc=A, ws=A, wsb=1 << 30, hq=32,
          kvv=kv):
        return est(q, hq, C.byref(kvv), k4, sz, sel, cnt, mb, w, tok, cc, ws, wsb, None)

    assert e(q=0) == twl.TWL_ERR_INVALID_ARG
    assert e(q=A + 8) == twl.TWL_ERR_INVALID_ARG            # q 16-byte aligned
    assert e(k4=A + 4) == twl.TWL_ERR_INVALID_ARG
    assert e(w=0) == twl.TWL_ERR_INVALID_ARG
    assert e(mb=0) == twl.TWL_ERR_INVALID_ARG
    assert e(mb=65) == twl.TWL_ERR_INVALID_ARG              # above max_pages
    assert e(hq=24) == twl.TWL_ERR_UNSUPPORTED              # group of 3
    assert e(kvv=_kv(page_size=8)) == twl.TWL_ERR_UNSUPPORTED
    assert e(wsb=256) == twl.TWL_ERR_WORKSPACE
    assert e(ws=0) == twl.TWL_ERR_WORKSPACE
    uni = twl._lib.twl_group_union

    def u(tok=A, ki=A, kc=A, cs=16, ut=A, uc=A, ws=None, wsb=0, hq=32):
        return uni(hq, C.byref(kv), tok, ki, kc, cs, ut, uc, ws, wsb, None)

    assert u(tok=0) == twl.TWL_ERR_INVALID_ARG
    assert u(uc=0) == twl.TWL_ERR_INVALID_ARG
    assert u(cs=0) == twl.TWL_ERR_INVALID_ARG
    assert u(hq=12) == twl.TWL_ERR_INVALID_ARG               # not a multiple of the kv-heads
    assert u(ws=A + 64, wsb=1 << 20) == twl.TWL_ERR_WORKSPACE  # misaligned workspace
    assert u(ws=A, wsb=16) == twl.TWL_ERR_WORKSPACE          # smaller than the header


def test_workspace_init_and_status_reject_bad_workspaces():
    flags = C.c_uint32(7)
    assert twl._lib.twl_workspace_init(None, 1 << 20, None) == twl.TWL_ERR_WORKSPACE
    assert twl._lib.twl_workspace_init(A, 100, None) == twl.TWL_ERR_WORKSPACE
    assert twl._lib.twl_workspace_init(A + 16, 1 << 20, None) == twl.TWL_ERR_WORKSPACE
    assert twl._lib.twl_device_status(None, C.byref(flags), 0, None) == twl.TWL_ERR_WORKSPACE
    assert twl._lib.twl_device_status(A + 16, C.byref(flags), 0, None) == twl.TWL_ERR_WORKSPACE


def test_workspace_sizes():
    wb = twl.twl_workspace_bytes
    assert wb(twl.TWL_OP_CACHE) == 256
    assert wb(twl.TWL_OP_PRUNE, 1, 1, 1, 1, 1, 4096, 8192) == 256     # header only, unused
    assert wb(99) == 0
    s1 = wb(twl.TWL_OP_DECODE_STEP, 1, 32, 8, 2048, 512)
    s2 = wb(twl.TWL_OP_DECODE_STEP, 2, 32, 8, 2048, 512)
    assert 256 < s1 < s2
    assert s1 % 256 == 0
    assert wb(twl.TWL_OP_SELECT, 1, 32, 8, 2048) >= 256 + 32 * 2048 * 4
    assert wb(twl.TWL_OP_SPARSE_DECODE, 1, 32, 8, 0, 0, 0, 4096) > 256
    assert wb(twl.TWL_OP_DECODE_STEP, -1, 32, 8, 2048, 512) == 0


def test_layer_rejects_host_and_misshaped_tensors_before_any_call():
    """DecodeLayer checks q (and the appended rows) before handing raw pointers to the library:
    a host tensor, another device, a wrong dtype or shape, or a strided view raises at once.
    The layer here is a bare object whose cache lives on the meta device, so any call that got
    through to the library would fail differently."""
    import torch
    from adaptive_top_sparse_b200.layer import DecodeLayer, Staged, expect_tensor

    layer = DecodeLayer.__new__(DecodeLayer)
    layer.k = torch.empty((4, 2, 16, 128), dtype=torch.float16, device="meta")
    layer.batch, layer.num_q_heads, layer.num_kv_heads = 3, 8, 2
    good = torch.empty((3, 8, 128), dtype=torch.float16, device="meta")
    layer.expect_query(good)
    bad = {
        "host tensor": torch.zeros((3, 8, 128), dtype=torch.float16),
        "dtype": torch.empty((3, 8, 128), dtype=torch.float32, device="meta"),
        "shape": torch.empty((3, 8, 64), dtype=torch.float16, device="meta"),
        "strided": torch.empty((3, 128, 8), dtype=torch.float16, device="meta").transpose(1, 2),
    }
    for what, q in bad.items():
        with pytest.raises(ValueError):
            layer.decode(q)
        stg = Staged.__new__(Staged)
        stg.layer = layer
        with pytest.raises(ValueError):
            stg.decode(q)
    with pytest.raises(TypeError):
        layer.decode(np.zeros((3, 8, 128), np.float16))
    rows = torch.zeros((3, 2, 128), dtype=torch.float16)             # on the host
    with pytest.raises(ValueError):
        layer.append(rows, rows)
    expect_tensor("x", rows, (3, 2, 128), torch.float16, rows.device)


def test_header_compiles_as_c_and_a_c_program_links_and_calls(tmp_path):
    """include/twl.h is plain C: a C99 program includes it, links libtwl.so and calls through the
    ABI (host-side rejections only, so no GPU is needed)."""
    src = tmp_path / "use_twl.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "twl.h"
int main(void) {
  twl_paged_kv kv = {0, 0, 0, 0, 2, 8, 128, 16, 64, 100};
  twl_k_aux aux = {0, 0, 0};
  float o[1], lse[1];
  twl_status st = twl_decode_step(0, 32, &kv, &aux, 0, 4, 16, 0.85f, 1e-6f, o, lse, 0, 0, 0, 0);
  if (st != TWL_ERR_INVALID_ARG) { printf("decode_step %d\n", (int)st); return 1; }
  st = twl_prune_top_p(0, 0, 1, 8, 0.9f, 1e-6f, 0, 0, 0, 0, 0, 0);
  if (st != TWL_ERR_INVALID_ARG) { printf("prune %d\n", (int)st); return 2; }
  if (strcmp(twl_status_string(TWL_OK), "ok") != 0) return 3;
  if (twl_workspace_bytes(TWL_OP_PRUNE, 1, 1, 1, 1, 1, 4, 8) != 256) return 4;
  printf("%s\n", twl_status_string(TWL_ERR_INVALID_ARG));
  return 0;
}
''')
    lib_dir = os.path.dirname(twl.LIB_PATH)
    exe = tmp_path / "use_twl"
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), "-L", lib_dir, "-ltwl",
                        "-Wl,-rpath," + lib_dir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)


def test_readme_c_example_compiles(tmp_path):
    """The C example in README.md compiles and links as written (it is not run: its pointers
    would have to be device memory)."""
    text = open(os.path.join(ROOT, "README.md")).read()
    m = re.search(r"```c\n(.*?)```", text, flags=re.S)
    assert m, "README has a C example"
    cuda_inc = "/usr/local/cuda/include"
    if not os.path.isdir(cuda_inc):
        pytest.skip("no CUDA headers")
    src = tmp_path / "readme_example.c"
    src.write_text(
        "#include <cuda_runtime.h>\n#include \"twl.h\"\n"
        "int example(void* d_k, void* d_v, int32_t* d_page_table, int32_t* d_seq_lens,\n"
        "            void* d_k_int4, void* d_k_scale_zero, void* d_bounds, void* d_q, float* d_o,\n"
        "            float* d_lse, int32_t B, int32_t Hq, int32_t Hkv, int32_t max_pages,\n"
        "            int32_t P, twl_stream_t stream) {\n" + m.group(1) + "  return (int)st;\n}\n")
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(twl.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-shared", "-fPIC",
                        "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src),
                        "-o", str(tmp_path / "libexample.so"), "-L", lib_dir, "-ltwl",
                        "-L", "/usr/local/cuda/lib64", "-lcudart"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
