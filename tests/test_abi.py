"""The C ABI library loads and exports every entry point the header declares;
host-side validation rejects bad arguments before touching a GPU (no GPU
needed)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


@pytest.fixture(scope="module")
def lib():
    from routing_grouped_gemm_moe_b200 import build
    build.build()
    from routing_grouped_gemm_moe_b200 import _lib
    return _lib.lib()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for must in ["moe_router_topk", "moe_permute_rows", "moe_grouped_gemm", "moe_swiglu",
                 "moe_unpermute_combine", "moe_layer_fwd", "moe_layer_bwd", "mxfp8_quantize"]:
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    from routing_grouped_gemm_moe_b200 import _lib
    names = _declared_functions()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(_lib.SIGNATURES), set(names) - set(_lib.SIGNATURES)


def test_status_strings_and_version(lib):
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(4) == b"MOE_ERR_DEVICE_TIMEOUT"
    assert lib.moe_version() >= 100


def test_host_validation_rejects_bad_arguments(lib):
    from routing_grouped_gemm_moe_b200 import _lib as L
    # null pointers / k > E / misaligned pointer: rejected before any launch
    assert lib.moe_router_topk(None, 10, 8, 2, None, None, None) == 1
    assert lib.moe_router_topk(C.c_void_p(16), 10, 8, 9, C.c_void_p(16), C.c_void_p(16), None) == 1
    assert lib.moe_router_topk(C.c_void_p(18), 10, 8, 2, C.c_void_p(16), C.c_void_p(16), None) == 1
    assert lib.moe_permute_rows(None, None, 4, 12, 4, 1, None, None, None, None, None, None, 0, None) == 1
    args = L.GGArgs(mode=7, dtype=0, E=2, N=8, K=8)
    assert lib.moe_grouped_gemm(C.byref(args), None) == 1
    assert lib.mxfp8_quantize(None, 4, 33, 1, None, 0, None, None, None, None) == 1
    # the MXFP8 dispatch: d must be a multiple of 32, codes / scales given and aligned
    p16, ws = C.c_void_p(16), C.c_void_p(1 << 20)
    base = [p16, p16, 4, 48, 4, 1, p16, p16, p16, p16, p16]
    assert lib.moe_permute_rows_mxfp8(*base, p16, p16, ws, 1 << 16, None) == 1   # d = 48
    base[3] = 64
    assert lib.moe_permute_rows_mxfp8(*base, None, p16, ws, 1 << 16, None) == 1  # no codes
    assert lib.moe_permute_rows_mxfp8(*base, p16, C.c_void_p(24), ws, 1 << 16, None) == 1  # misaligned
    assert lib.moe_permute_rows_mxfp8(*base, p16, p16, ws, 8, None) == 1         # workspace too small
    assert lib.mxfp8_quantize_rowcol(None, 64, 64, None, 1, None, None, None, None, None) == 1
    d = L.LayerDesc(T=4, d=12, E=4, k=2, f=16, dtype=0, router_mode=0)   # d % 8 != 0
    assert lib.moe_layer_fwd(C.byref(d), C.byref(L.LayerParams()), C.byref(L.LayerSaved()),
                             None, None, 0, None) == 1


def test_workspace_sizes(lib):
    from routing_grouped_gemm_moe_b200 import _lib as L
    assert lib.moe_permute_workspace_bytes(128, 8) == 256 + 8 * 4
    assert lib.moe_permute_workspace_bytes(129, 8) == 256 + 2 * 8 * 4
    d = L.LayerDesc(T=256, d=128, E=8, k=2, f=256, dtype=0, router_mode=1)
    ws = lib.moe_layer_workspace_bytes(C.byref(d))
    M = 256 * 2
    assert ws >= 256 + M * 128 * 2 + M * 512 * 2 + 256 * 2 * 4


def test_bf16_gemm_workspace_size(lib):
    """BF16 ragged-M needs no workspace; BF16 ragged-K takes an optional one of
    two 128-byte tensor maps per expert (256-byte rounded)."""
    from routing_grouped_gemm_moe_b200 import _lib as L
    for E in (1, 8, 1024):
        a = L.GGArgs(mode=L.GG_RAGGED_K, dtype=L.DTYPE_BF16, epilogue=L.EPI_NONE, E=E, M_total=1000,
                     M=64, N=128)
        assert lib.moe_grouped_gemm_workspace_bytes(C.byref(a)) == (2 * E * 128 + 255) // 256 * 256
        a.mode = L.GG_RAGGED_M
        a.K = 64
        assert lib.moe_grouped_gemm_workspace_bytes(C.byref(a)) == 0


def test_mxfp8_gemm_workspace_size(lib):
    from routing_grouped_gemm_moe_b200 import _lib as L
    a = L.GGArgs(mode=L.GG_RAGGED_M, dtype=L.DTYPE_MXFP8, epilogue=L.EPI_NONE, E=4, M_total=1000,
                 N=256, K=512)
    # A: (1000 // 128 + 4) row tiles x 4 K-stages; B: 4 experts x 2 row tiles x 4 stages; 512 B atoms
    assert lib.moe_grouped_gemm_workspace_bytes(C.byref(a)) == 11 * 4 * 512 + 4 * 2 * 4 * 512
    a.dtype = L.DTYPE_BF16
    assert lib.moe_grouped_gemm_workspace_bytes(C.byref(a)) == 0


def test_header_is_plain_c(tmp_path):
    """The boundary header is C99 (no C++ or CUDA types): a C program that
    takes the address of every declared entry point compiles without a
    warning and links against the library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    names = _declared_functions()
    src = tmp_path / "use_abi.c"
    body = "\n".join(f"    (entry)&{n}," for n in names)
    src.write_text('#include "moe_b200.h"\n'
                   "typedef void (*entry)(void);\n"
                   f"entry entry_points[] = {{\n{body}\n}};\n"
                   "int main(void) { return entry_points[0] == 0; }\n")
    from routing_grouped_gemm_moe_b200 import build
    build.build()
    libdir = os.path.join(ROOT, "routing_grouped_gemm_moe_b200")
    out = tmp_path / "use_abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(out),
                        "-L", libdir, "-lmoe_b200", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr



def test_binding_matches_the_header(tmp_path):
    """The ctypes binding's structures and constants are the header's: a C
    program prints sizeof / offsetof of every structure and the enum values,
    which must equal what _lib.py declares."""
    import ctypes
    import shutil
    import subprocess
    from routing_grouped_gemm_moe_b200 import _lib as L
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    structs = {"moe_gg_args": L.GGArgs, "moe_layer_desc": L.LayerDesc,
               "moe_layer_params": L.LayerParams, "moe_layer_saved": L.LayerSaved,
               "moe_layer_grads": L.LayerGrads}
    consts = {"MOE_OK": L.MOE_OK, "MOE_DTYPE_BF16": L.DTYPE_BF16, "MOE_DTYPE_MXFP8": L.DTYPE_MXFP8,
              "MOE_GG_RAGGED_M": L.GG_RAGGED_M, "MOE_GG_RAGGED_K": L.GG_RAGGED_K,
              "MOE_EPI_NONE": L.EPI_NONE, "MOE_EPI_SWIGLU": L.EPI_SWIGLU,
              "MOE_EPI_SWIGLU_BWD": L.EPI_SWIGLU_BWD, "MOE_ROUTER_LOGITS": L.ROUTER_LOGITS,
              "MOE_ROUTER_PROJ": L.ROUTER_PROJ, "MOE_FWD_STAGES": L.FWD_STAGES,
              "MOE_BWD_STAGES": L.BWD_STAGES}
    consts.update({f"MOE_ERR_{n[8:]}": v for v, n in L.STATUS_NAMES.items() if n.startswith("MOE_ERR_")})
    consts.update({f"MOE_MX_{n.upper()}": getattr(L, f"MX_{n.upper()}") for n in
                   ("gemm1", "gemm2", "da", "dw2", "dx", "dw13")})
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "moe_b200.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'    printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'    printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    for n in consts:
        lines.append(f'    printf("{n} %d\\n", (int)({n}));')
    lines += ["    return 0;", "}"]
    src, exe = tmp_path / "layout.c", tmp_path / "layout"
    src.write_text("\n".join(lines) + "\n")
    r = subprocess.run([gcc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {" ".join(x.split()[:-1]): int(x.split()[-1]) for x in out if x.strip()}
    for cname, cls in structs.items():
        assert got[f"{cname} sizeof"] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[f"{cname} {fname}"] == getattr(cls, fname).offset, (cname, fname)
    for n, v in consts.items():
        assert got[n] == v, n


def test_binding_rejects_tensors_of_the_wrong_shape_or_type():
    """The Python binding checks every tensor it hands the library as a raw
    pointer (the C side cannot know the buffer sizes)."""
    import torch
    from routing_grouped_gemm_moe_b200 import ops
    ok = torch.zeros(4, 8, dtype=torch.bfloat16)
    assert ops.expect(ok, "x", (4, 8), torch.bfloat16, "cpu") is ok
    for bad in (torch.zeros(8, 4, dtype=torch.bfloat16), torch.zeros(4, 8),
                torch.zeros(8, 4, dtype=torch.bfloat16).t(), None):
        with pytest.raises(ValueError):
            ops.expect(bad, "x", (4, 8), torch.bfloat16)
    with pytest.raises(ValueError):
        ops.expect(ok, "x", (4, 8), torch.bfloat16, "meta")
    m = torch.zeros(4, 8, dtype=torch.bfloat16, device="meta")
    assert ops.expect(m, "x", (4, 8), torch.bfloat16, torch.device("meta")) is m


def test_dispatch_and_quantiser_wrappers_check_index_tensors():
    """An int64 expert index (torch.topk's default) or int64 group offsets
    would be read by the library as pairs of int32 -- routing silently wrong,
    or offsets that go down -- so the wrappers refuse them before any call."""
    import torch
    from routing_grouped_gemm_moe_b200 import ops
    T, d, E, k = 16, 32, 4, 2
    x = torch.zeros(T, d, dtype=torch.bfloat16)
    idx64 = torch.zeros(T, k, dtype=torch.int64)
    for fn in (ops.permute_rows, ops.permute_rows_mxfp8, ops.permute_rows_noalloc):
        with pytest.raises(ValueError, match="idx"):
            fn(x, idx64, E)
        with pytest.raises(ValueError, match="x"):
            fn(x.float(), idx64.int(), E)
    with pytest.raises(ValueError, match="idx"):
        ops.permute_rows(x, torch.zeros(T, k, dtype=torch.int32, device="meta"), E)
    off64 = torch.tensor([0, 8, 16], dtype=torch.int64)
    with pytest.raises(ValueError, match="group_offsets"):
        ops.mxfp8_quantize(x, 0, off64)
    with pytest.raises(ValueError, match="group_offsets"):
        ops.mxfp8_quantize_rowcol(x, off64)
