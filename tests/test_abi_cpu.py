"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every function include/sage_b200.h declares, sizes
workspaces, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import fp8_quantized_exact_b200 as sage

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fp8_quantized_exact_b200 import build
    build.build()
    return sage.lib()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                text = f.read()
            names |= set(re.findall(r"SAGE_API\s+[\w\s\*]+?\b(sage_\w+)\s*\(", text))
    return names


def test_header_declares_the_binding_exports():
    assert declared_functions() == set(sage.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_workspace_sizes(lib):
    # long-context fused config: B1 N37810 H56 D128
    n = sage.sage_workspace_bytes(sage.SAGE_OP_ATTN_FWD, 1, 37810, 56, 128)
    bh, Nq, Nk, T = 56, 37888, 37824, 591
    quant = bh * (Nq * 128 + Nk * 128 + 128 * Nk)
    # the quantised tensors, FP64 K partials per 64-token chunk and channel, and small vectors
    assert quant + bh * T * 128 * 8 < n < quant + bh * T * 128 * 8 + (2 << 20)
    assert sage.sage_workspace_bytes(sage.SAGE_OP_ATTN_FROM_QUANT, 1, 37810, 56, 128) < 4096
    assert sage.sage_workspace_bytes(sage.SAGE_OP_QUANT_QK, 2, 1000, 8, 64) >= 2 * 8 * 16 * 64 * 8
    lay = sage.sage_fwd_workspace_layout(1, 1000, 8, 128)
    offs = [lay[k] for k in ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean", "v_fp8", "v_scale")]
    assert offs == sorted(offs) and all(o % 1024 == 0 for o in offs) and offs[0] >= 256
    assert lay["total"] == sage.sage_workspace_bytes(sage.SAGE_OP_ATTN_FWD, 1, 1000, 8, 128)
    # the host pipeline: two chunk workspaces, each rounded up to 1024 bytes
    one = sage.sage_workspace_bytes(sage.SAGE_OP_ATTN_FWD, 1, 1000, 4, 128)
    assert sage.sage_workspace_bytes(sage.SAGE_OP_ATTN_FWD_HOST, 1, 1000, 4, 128) == 2 * ((one + 1023) // 1024 * 1024)


def test_argument_errors_need_no_device(lib):
    assert sage.sage_strerror(0) == "success"
    n = ctypes.c_size_t()
    assert lib.sage_workspace_bytes(2, 1, 100, 2, 96, ctypes.byref(n)) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_workspace_bytes(2, -1, 100, 2, 64, ctypes.byref(n)) == sage.SAGE_ERR_INVALID_ARG
    assert lib.sage_workspace_bytes(9, 1, 100, 2, 64, ctypes.byref(n)) == sage.SAGE_ERR_INVALID_ARG
    # grid extents: B and H at most 65535 each; B*H at most 2^30; N at most 2^28
    for (B, N, H) in ((65536, 16, 1), (1, 16, 65536), (32768, 16, 32769), (1, (1 << 28) + 1, 1)):
        assert lib.sage_workspace_bytes(2, B, N, H, 64, ctypes.byref(n)) == sage.SAGE_ERR_UNSUPPORTED, (B, N, H)
    assert lib.sage_workspace_bytes(2, 65535, 16, 1, 64, ctypes.byref(n)) == sage.SAGE_OK
    null = sage.sage_view_bf16(None, 0, 0, 0)
    good = sage.sage_view_bf16(4096, 256 * 2 * 128, 2 * 128, 128)
    odd = sage.sage_view_bf16(4096 + 2, 256 * 2 * 128, 2 * 128, 128)
    badstride = sage.sage_view_bf16(4096, 256 * 2 * 128, 2 * 128 + 4, 128)
    fwd = lib.sage_attn_fwd
    # empty problems succeed and launch nothing
    assert fwd(null, null, null, None, 0, 0, 0, 0, 10, 2, 128, 0.0, None, 0, None) == sage.SAGE_OK
    assert fwd(null, null, null, None, 0, 0, 0, 1, 0, 2, 128, 0.0, None, 0, None) == sage.SAGE_OK
    assert fwd(null, good, good, 4096, 0, 0, 0, 1, 10, 2, 128, 0.0, 4096, 1 << 20, None) == sage.SAGE_ERR_INVALID_ARG
    assert fwd(good, good, good, 4096, 0, 0, 0, 1, 10, 2, 100, 0.0, 4096, 1 << 20, None) == sage.SAGE_ERR_UNSUPPORTED
    assert fwd(odd, good, good, 4096, 0, 0, 0, 1, 10, 2, 128, 0.0, 4096, 1 << 20, None) == sage.SAGE_ERR_UNSUPPORTED
    assert fwd(good, badstride, good, 4096, 0, 0, 0, 1, 10, 2, 128, 0.0, 4096, 1 << 20, None) == sage.SAGE_ERR_UNSUPPORTED
    assert fwd(good, good, good, None, 0, 0, 0, 1, 10, 2, 128, 0.0, 4096, 1 << 20, None) == sage.SAGE_ERR_INVALID_ARG
    # workspace missing, misaligned, too small
    assert fwd(good, good, good, 4096, 0, 0, 0, 1, 10, 2, 128, 0.0, None, 1 << 20, None) == sage.SAGE_ERR_WORKSPACE
    assert fwd(good, good, good, 4096, 0, 0, 0, 1, 10, 2, 128, 0.0, 4096 + 16, 1 << 20, None) == sage.SAGE_ERR_WORKSPACE
    assert fwd(good, good, good, 4096, 0, 0, 0, 1, 10, 2, 128, 0.0, 4096, 100, None) == sage.SAGE_ERR_WORKSPACE
    fq = lib.sage_attn_from_quant
    assert fq(None, 4096, 4096, 4096, 4096, 4096, 4096, 0, 0, 0, 1, 10, 2, 64, 0.0, 4096, 4096, None) == sage.SAGE_ERR_INVALID_ARG
    assert fq(4096, 4096, 4096 + 8, 4096, 4096, 4096, 4096, 0, 0, 0, 1, 10, 2, 64, 0.0, 4096, 4096, None) == sage.SAGE_ERR_UNSUPPORTED
    nr = lib.sage_norm_rope_quant_qk
    v4 = sage.sage_view_bf16(4096, 0, 128, 128)
    # (q, k, wq, wk, cos, sin, eps, B, N, H, D, q8, qs, k8, ks, km, ws, ws_bytes, stream)
    assert nr(v4, v4, None, 4096, 4096, 4096, 1e-6, 1, 10, 2, 64, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
              None) == sage.SAGE_ERR_INVALID_ARG
    assert nr(v4, v4, 4096, 4096, 4096, 4096, -1.0, 1, 10, 2, 64, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
              None) == sage.SAGE_ERR_INVALID_ARG
    assert nr(v4, v4, 4096 + 2, 4096, 4096, 4096, 1e-6, 1, 10, 2, 64, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
              None) == sage.SAGE_ERR_UNSUPPORTED
    assert nr(v4, v4, 4096, 4096, 4096, 4096, 1e-6, 1, 10, 2, 96, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
              None) == sage.SAGE_ERR_UNSUPPORTED
    qkv = lib.sage_quant_qkv
    assert qkv(v4, v4, v4, 1, 10, 2, 64, None, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
               None) == sage.SAGE_ERR_INVALID_ARG
    assert qkv(v4, v4, v4, 1, 10, 2, 64, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 100,
               None) == sage.SAGE_ERR_WORKSPACE
    # no work-item limit beyond the common shape limits: a large problem only needs its workspace
    assert qkv(v4, v4, v4, 1, 1 << 24, 1 << 14, 128, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
               None) == sage.SAGE_ERR_WORKSPACE
    assert qkv(v4, v4, v4, 70000, 10, 1, 64, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
               None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_set_mainloop(7) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_set_mainloop(-1) == sage.SAGE_ERR_UNSUPPORTED
    # every declared mainloop value is accepted; the explicit ones read back as set
    for which in (sage.SAGE_MAINLOOP_TCGEN05, sage.SAGE_MAINLOOP_MMA_SYNC, sage.SAGE_MAINLOOP_TCGEN05_F32):
        assert lib.sage_set_mainloop(which) == sage.SAGE_OK
        assert lib.sage_get_mainloop() == which
    assert lib.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT) == sage.SAGE_OK
    dbg = lib.sage_debug_qk_s32
    assert dbg(4096, 4096, 4096, 4096, 4096, 4096, 1, 100, 2, 64, 0, 2, 0, 0, 4096, 4096, 4096,
               None) == sage.SAGE_ERR_INVALID_ARG                     # head 2 of 2
    assert dbg(4096, 4096, 4096, 4096, 4096, 4096, 1, 100, 2, 64, 0, 1, 1, 0, 4096, 4096, 4096,
               None) == sage.SAGE_ERR_INVALID_ARG                     # query tile 1 of 1
    assert dbg(4096, 4096, 4096, 4096, 4096, 4096, 1, 100, 2, 64, 0, 1, 0, 2, 4096, 4096, 4096,
               None) == sage.SAGE_ERR_INVALID_ARG                     # key tile 2 of 2
    assert dbg(4096, None, 4096, 4096, 4096, 4096, 1, 100, 2, 64, 0, 1, 0, 0, 4096, 4096, 4096,
               None) == sage.SAGE_ERR_INVALID_ARG                     # missing scale
    host = lib.sage_attn_fwd_host
    other = sage.sage_view_bf16(8192, 256 * 2 * 128, 2 * 128, 128)
    narrow = sage.sage_view_bf16(4096, 256 * 2 * 128, 32, 128)

    def fh(qh=good, qd=good, out_host=4096, D=128, hpc=4, ws_bytes=1 << 24, ev=4096, N=10):
        # (q/k/v host, q/k/v dev, out host, out dev, out strides, B, N, H, D, sm_scale, heads_per_chunk,
        #  ws, ws bytes, stream, stream_in, stream_out, three events)
        return host(qh, good, good, qd, good, good, out_host, 4096, 0, 256, 128, 1, N, 2, D, 0.0, hpc, 4096,
                    ws_bytes, None, None, None, None, ev, ev, ev)
    assert fh(D=96) == sage.SAGE_ERR_UNSUPPORTED
    assert fh(qd=odd) == sage.SAGE_ERR_UNSUPPORTED
    assert fh(qh=null) == sage.SAGE_ERR_INVALID_ARG
    assert fh(qh=other) == sage.SAGE_ERR_INVALID_ARG          # host and device strides differ
    assert fh(out_host=None) == sage.SAGE_ERR_INVALID_ARG
    assert fh(ev=None) == sage.SAGE_ERR_INVALID_ARG
    assert fh(ws_bytes=100) == sage.SAGE_ERR_WORKSPACE
    assert host(narrow, good, good, narrow, good, good, 4096, 4096, 0, 256, 128, 1, 10, 2, 64, 0.0, 4, 4096,
                1 << 24, None, None, None, None, 4096, 4096, 4096) == sage.SAGE_ERR_UNSUPPORTED  # stride_n < D
    assert fh(N=0) == sage.SAGE_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sage, "_lib", None)
    monkeypatch.setattr(sage, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        sage.lib()


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """The header is plain C: a C99 program that includes it, takes the
    address of every declared function and calls the argument-only entry
    points compiles with -pedantic -Werror, links against the library and
    runs without a GPU."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    names = sorted(declared_functions())
    table = ",\n    ".join(f"(void (*)(void))&{n}" for n in names)
    src = tmp_path / "abi_check.c"
    src.write_text(f"""#include <stdio.h>
#include <string.h>
#include "sage_b200.h"

static void (*const every_entry[])(void) = {{
    {table}
}};

int main(void) {{
  size_t bytes = 0;
  sage_fwd_layout lay;
  unsigned i;
  for (i = 0; i < sizeof every_entry / sizeof every_entry[0]; ++i)
    if (!every_entry[i]) return 10;
  if (sage_workspace_bytes(SAGE_OP_ATTN_FWD, 1, 1000, 8, 128, &bytes) != SAGE_OK || bytes == 0) return 1;
  if (sage_fwd_workspace_layout(1, 1000, 8, 128, &lay) != SAGE_OK || lay.total != bytes) return 2;
  if (sage_workspace_bytes(SAGE_OP_ATTN_FWD, 1, 1000, 8, 96, &bytes) != SAGE_ERR_UNSUPPORTED) return 3;
  if (sage_workspace_bytes(SAGE_OP_ATTN_FWD, 1, 1000, 8, 128, NULL) != SAGE_ERR_INVALID_ARG) return 4;
  if (strcmp(sage_strerror(SAGE_OK), "success") != 0) return 5;
  if (sage_set_mainloop(99) != SAGE_ERR_UNSUPPORTED) return 6;
  printf("%u entry points\\n", i);
  return 0;
}}
""")
    so = os.path.abspath(lib._name)
    exe = tmp_path / "abi_check"
    cc = subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I",
                         os.path.join(ROOT, "include"), str(src), so, f"-Wl,-rpath,{os.path.dirname(so)}",
                         "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.strip() == f"{len(names)} entry points"


def _header_prototypes():
    protos = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        with open(os.path.join(ROOT, "include", fn)) as f:
            text = re.sub(r"/\*.*?\*/", " ", f.read(), flags=re.S)
        for ret, name, params in re.findall(r"SAGE_API\s+([\w\s\*]+?)\s*\b(sage_\w+)\s*\(([^)]*)\)\s*;", text):
            plist = [p.strip() for p in params.split(",")]
            if plist == ["void"]:
                plist = []
            protos[name] = (" ".join(ret.split()), [re.sub(r"\s*\b\w+$", "", p).strip() for p in plist])
    return protos


def test_binding_signatures_match_the_header(lib):
    """Every ctypes prototype the binding sets has the header's parameter
    count and kinds, and the header's return type."""
    scalar = {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "size_t": ctypes.c_size_t,
              "long long": ctypes.c_longlong, "float": ctypes.c_float, "sage_view_bf16": sage.sage_view_bf16}
    protos = _header_prototypes()
    assert set(protos) == set(sage.EXPORTS)
    for name, (ret, params) in protos.items():
        f = getattr(lib, name)
        assert len(f.argtypes) == len(params), (name, len(f.argtypes), params)
        for i, (ctype, decl) in enumerate(zip(f.argtypes, params)):
            if "*" in decl:
                assert ctype is ctypes.c_void_p or issubclass(ctype, ctypes._Pointer), (name, i, decl, ctype)
            else:
                assert ctype is scalar[decl], (name, i, decl, ctype)
        want = ctypes.c_char_p if ret == "const char*" else scalar[ret]
        assert f.restype is want, (name, ret, f.restype)


def test_product_path_does_not_reach_the_oracle(lib):
    """The library and its binding neither import, load nor link anything of
    the oracle; the oracle's C source includes nothing of the library."""
    import subprocess
    pkg = os.path.join(ROOT, "fp8_quantized_exact_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                with open(os.path.join(dirpath, fn)) as f:
                    text = f.read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b|liboracle|sage_oracle|oracle_\w+\(", text, re.M), fn
    needed = subprocess.run(["readelf", "-d", sage.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in needed and "synth" not in needed
    with open(os.path.join(ROOT, "oracle", "sage_oracle.c")) as f:
        src = f.read()
    assert not re.search(r'#include\s+"', src), "the oracle includes a project header"
    assert "sage_b200" not in src and "csrc" not in src


def test_long_context_tile_geometry(lib):
    """The pages' tiling of the 37,810-token workload: 591 key tiles of 64,
    296 query tiles of 128 (the (296, 56, 1) grid) and so 1,182 query groups
    of 32 ("Vortex Exact Attention", section "Authoritative Baseline";
    "architecture_model.json", key "baseline"; "State-Ownership Architecture
    Decision", section "Non-Negotiable Dataflow"); the workspace holds
    those padded buffers."""
    shp = sage.quant_shapes(1, 37810, 56, 128)
    assert shp["k_scale"] == (1, 56, 591) and shp["q_scale"] == (1, 56, 1182)
    assert shp["q_i8"] == (1, 56, 296 * 128, 128) and shp["v_fp8"] == (1, 56, 128, 591 * 64)
    lay = sage.sage_fwd_workspace_layout(1, 37810, 56, 128)
    assert lay["q_scale"] - lay["q_i8"] >= 56 * 296 * 128 * 128
    assert lay["k_scale"] - lay["k_i8"] >= 56 * 591 * 64 * 128
    assert lay["v_scale"] - lay["v_fp8"] >= 56 * 128 * 591 * 64


def test_c_example_compiles(lib, tmp_path):
    """The C example (tests/c_example/attend.c, the code README.md shows)
    compiles as C11 against the header and the CUDA runtime header, and links
    against the library and cudart (it needs a GPU only to run)."""
    import shutil
    import subprocess
    gcc, cuda_inc = shutil.which("gcc"), "/usr/local/cuda/include"
    if gcc is None or not os.path.isdir(cuda_inc):
        pytest.skip("no C compiler or CUDA headers")
    src = os.path.join(ROOT, "tests", "c_example", "attend.c")
    obj = tmp_path / "example.o"
    cc = subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
                         os.path.join(ROOT, "include"), "-isystem", cuda_inc, "-c", str(src), "-o", str(obj)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    so = tmp_path / "example.so"
    ld = subprocess.run([gcc, "-shared", "-o", str(so), str(obj), os.path.abspath(lib._name),
                         "-L/usr/local/cuda/lib64", "-lcudart", "-Wl,--no-undefined"],
                        capture_output=True, text=True)
    assert ld.returncode == 0, ld.stderr


def test_attn_fwd_prepass_choice(lib):
    """sage_attn_fwd's prepass: the single launch below 128 MiB of Q, K and V
    (3*B*H*N*D BF16 values), the six separate kernels from there on."""
    if os.environ.get("SAGE_PREPASS"):
        pytest.skip("SAGE_PREPASS overrides the choice")
    k = sage.sage_attn_fwd_prepass_kernels
    assert k(1, 256, 2, 128) == 1 and k(1, 1000, 8, 128) == 1
    assert k(2, 8192, 32, 128) == 6 and k(1, 37810, 56, 128) == 6 and k(4, 16384, 24, 64) == 6
    assert k(1, 174762, 1, 128) == 1 and k(1, 174763, 1, 128) == 6  # 768 N bytes against 2^27
    assert k(0, 10, 2, 64) == 0
    assert lib.sage_attn_fwd_prepass_kernels(1, 10, 2, 96) == sage.SAGE_ERR_UNSUPPORTED
