"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function that
include/moe.h declares, and rejects invalid arguments before launching anything."""
import os
import re

import pytest

import combine_moe_route_10_b200 as pkg
from combine_moe_route_10_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    from combine_moe_route_10_b200 import build
    build.build()
    return pkg.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C11 program that takes the address of every declared function compiles against moe.h with
    warnings as errors and links against libmoe.so: the boundary is usable from plain C."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    body = "\n".join(f"  fns[{i}] = (void (*)(void))&{n};" for i, n in enumerate(names))
    src = tmp_path / "use_moe.c"
    src.write_text(
        '#include "moe.h"\n#include <stdio.h>\n'
        f"int main(void) {{\n  void (*fns[{len(names)}])(void);\n{body}\n"
        '  printf("%d %d\\n", moe_abi_version(), moe_capacity(1.25, 16384, 2, 128));\n'
        "  return fns[0] == 0;\n}\n")
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "use_moe"
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-l:" + os.path.basename(_lib.LIB_PATH), "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == [str(pkg.moe_abi_version()), "320"]


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ["moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(_lib.EXPORTS) == names


def test_abi_version_and_status_strings(lib):
    assert pkg.moe_abi_version() == 1
    for code in range(7):
        assert pkg.status_string(code).startswith("MOE_")
    assert "unknown" in pkg.status_string(99)


def test_capacity_helper(lib):
    assert pkg.moe_capacity(1.0, 65536, 2, 128) == 1024     # printed example
    assert pkg.moe_capacity(1.25, 16384, 2, 128) == 320
    assert pkg.moe_capacity(1.0, 10, 1, 3) == 4
    assert pkg.moe_capacity(0.0, 10, 1, 3) == 0
    assert pkg.moe_capacity(1.0, -1, 1, 3) == -1


FAKE = 1 << 20   # never dereferenced: every call below fails validation first


def test_route_rejects_bad_arguments(lib):
    bad = [dict(T=-1, E=8, k=2), dict(T=4, E=0, k=1), dict(T=4, E=8, k=9), dict(T=4, E=8, k=0),
           dict(T=4, E=2048, k=2), dict(T=4, E=64, k=33)]
    for a in bad:
        st = lib.moe_route(FAKE, a["T"], a["E"], a["k"], 1, FAKE, FAKE, None, None)
        assert st == pkg.MOE_ERR_INVALID_ARG, a
    assert lib.moe_route(None, 4, 8, 2, 1, FAKE, FAKE, None, None) == pkg.MOE_ERR_INVALID_ARG
    assert lib.moe_route(FAKE + 2, 4, 8, 2, 1, FAKE, FAKE, None, None) == pkg.MOE_ERR_INVALID_ARG


def dispatch(lib, **kw):
    a = dict(x=FAKE, T=16, H=256, idx=FAKE, k=2, E=8, R=4, cap=0, payload=0, send=FAKE,
             scales=FAKE, counts=FAKE, offsets=FAKE, rank_offsets=FAKE, slot_row=FAKE,
             row_token=FAKE, ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    return lib.moe_dispatch(a["x"], a["T"], a["H"], a["idx"], a["k"], a["E"], a["R"], a["cap"],
                            a["payload"], a["send"], a["scales"], a["counts"], a["offsets"],
                            a["rank_offsets"], a["slot_row"], a["row_token"], a["ws"],
                            a["ws_bytes"], None)


def test_dispatch_rejects_bad_arguments(lib):
    E = pkg.MOE_ERR_INVALID_ARG
    assert dispatch(lib, R=3) == E                       # E % R != 0
    assert dispatch(lib, k=9) == E                       # k > E
    assert dispatch(lib, cap=-1) == E
    assert dispatch(lib, payload=7) == E
    assert dispatch(lib, x=FAKE + 8) == E                # x not 16-byte aligned
    assert dispatch(lib, send=None) == E
    assert dispatch(lib, payload=1, scales=None) == E    # FP8 needs the scale output
    assert dispatch(lib, H=100) == pkg.MOE_ERR_UNSUPPORTED
    assert dispatch(lib, payload=1, H=320) == pkg.MOE_ERR_UNSUPPORTED
    assert dispatch(lib, ws_bytes=16) == pkg.MOE_ERR_WORKSPACE
    assert dispatch(lib, ws=FAKE + 64) == pkg.MOE_ERR_WORKSPACE


def test_workspace_sizes(lib):
    s1 = pkg.moe_dispatch_workspace_size(16384, 128, 2)     # 16 chunks of 1024 tokens
    assert s1 >= 256 + 16 * 128 * 4 and s1 % 256 == 0
    s8 = pkg.moe_dispatch_workspace_size(4096, 256, 8)      # 16 chunks of 256 tokens
    assert s8 >= 256 + 16 * 256 * 4 and s8 % 256 == 0
    f = pkg.moe_ffn_workspace_size(32768, 256, 7168, 2048, pkg.MOE_PAYLOAD_FP8_E4M3_B128)
    assert f >= 256 + 32768 * 2048 * 2 + 32768 * 7168 * 2
    assert pkg.moe_ffn_workspace_size(100, 8, 256, 512, pkg.MOE_PAYLOAD_BF16) >= 256 + 100 * 512 * 2


@pytest.mark.parametrize("max_rows,E,H,F", [(100, 8, 256, 512), (32768, 256, 7168, 2048),
                                            (1, 1, 128, 64)])
def test_ffn_workspace_layout_matches_the_python_views(lib, max_rows, E, H, F):
    """The binding reads two parts of the FFN workspace directly: h at byte 256 and, for the FP8
    payload, the dequantised bf16 input rows right after h (``MoeShuffle.dequantized_rows``, the
    expert-parallel backward's FFN input rows), and the failure test writes the GEMM-1 counters
    after those.  The library's size is exactly that layout: status | h | (FP8: rows) | counters,
    each part rounded up to 256 bytes."""
    up = lambda b: (b + 255) // 256 * 256  # noqa: E731
    h = up(max_rows * F * 2)
    counters = up((2 * (max_rows // 128 + E + 1) + 4) * 4)
    assert pkg.moe_ffn_workspace_size(max_rows, E, H, F, pkg.MOE_PAYLOAD_BF16) == 256 + h + counters
    assert pkg.moe_ffn_workspace_size(max_rows, E, H, F, pkg.MOE_PAYLOAD_FP8_E4M3_B128) == (
        256 + h + up(max_rows * H * 2) + counters)


@pytest.mark.parametrize("max_rows,T,k,H,F", [(8192, 4096, 2, 4096, 14336), (5, 3, 2, 64, 64),
                                              (0, 0, 1, 128, 128)])
def test_backward_workspace_layout_matches_the_python_views(lib, max_rows, T, k, H, F):
    """``MoeShuffle.backward_intermediate`` reads d_eo, h, dg, du and dx_rows at fixed offsets of
    the backward workspace: status | d_eo [r,H] | h, dg, du [r,F] | dx_rows [r,H] | unit weights
    [T,k] fp32, each part rounded up to 256 bytes (r = max(max_rows, 1)); the expert backward's own
    workspace is status | h, dg, du."""
    up = lambda b: (b + 255) // 256 * 256  # noqa: E731
    r, tk = max(max_rows, 1), max(T, 1) * k
    assert pkg.moe_backward_workspace_size(max_rows, T, k, H, F) == (
        256 + 2 * up(r * H * 2) + 3 * up(r * F * 2) + up(tk * 4))
    assert pkg.moe_expert_backward_workspace_size(max_rows, F) == 256 + 3 * up(r * F * 2)


def test_package_exports_every_binding_function():
    """Every moe_* function of the binding (one per C entry point, moe_status_string aside, which
    the binding wraps as status_string) is part of the package's public names."""
    import inspect
    from combine_moe_route_10_b200 import _lib
    names = {n for n, f in inspect.getmembers(_lib, inspect.isfunction) if n.startswith("moe_")}
    assert names and names <= set(pkg.__all__)
    assert all(hasattr(pkg, n) for n in pkg.__all__)
    consts = {n for n in dir(_lib) if n.startswith("MOE_")}
    assert consts <= set(pkg.__all__)


def test_ffn_and_combine_reject_bad_arguments(lib):
    ffn = lambda **kw: lib.moe_expert_ffn(
        kw.get("send", FAKE), kw.get("scales", None), kw.get("payload", 0), FAKE,
        kw.get("rows", 64), kw.get("E", 8), kw.get("H", 256), kw.get("F", 512), FAKE, FAKE, FAKE,
        FAKE, kw.get("ws", FAKE), kw.get("ws_bytes", 1 << 30), None)
    assert ffn(H=200) == pkg.MOE_ERR_UNSUPPORTED
    assert ffn(F=96) == pkg.MOE_ERR_UNSUPPORTED
    assert ffn(payload=1) == pkg.MOE_ERR_INVALID_ARG       # FP8 without scales
    assert ffn(E=0) == pkg.MOE_ERR_INVALID_ARG
    assert ffn(ws_bytes=100) == pkg.MOE_ERR_WORKSPACE
    assert ffn(send=FAKE + 4) == pkg.MOE_ERR_INVALID_ARG
    comb = lambda **kw: lib.moe_combine(FAKE, 64, FAKE, FAKE, kw.get("T", 4), kw.get("k", 2),
                                        kw.get("H", 256), kw.get("y", FAKE), kw.get("st", None),
                                        None)
    assert comb(k=0) == pkg.MOE_ERR_INVALID_ARG
    assert comb(H=12) == pkg.MOE_ERR_UNSUPPORTED
    assert comb(y=FAKE + 2) == pkg.MOE_ERR_INVALID_ARG
    assert comb(st=FAKE + 2) == pkg.MOE_ERR_INVALID_ARG
    assert lib.moe_sync_status(None, None) == pkg.MOE_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libmoe.so"))
    with pytest.raises(ImportError):
        _lib.load()


def test_weight_list_calls_reject_bad_arguments(lib):
    """The per-expert weight-list entry points validate on the host before touching the GPU."""
    import ctypes
    assert pkg.moe_ffn_weight_list_bytes(8) == 8 * 4 * 128        # four descriptors per expert
    assert pkg.moe_ffn_weight_list_bytes(0) == 0
    assert pkg.moe_ffn_weight_list_bytes(1025) == 0
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    p = ctypes.cast(ptrs, ctypes.c_void_p)
    init = lambda **kw: lib.moe_ffn_weight_list_init(
        kw.get("g", p), p, p, kw.get("E", 2), kw.get("H", 256), kw.get("F", 512),
        kw.get("list", FAKE), None)
    assert init(g=None) == pkg.MOE_ERR_INVALID_ARG
    assert init(H=200) == pkg.MOE_ERR_UNSUPPORTED
    assert init(list=FAKE + 32) == pkg.MOE_ERR_INVALID_ARG          # not 64-byte aligned
    assert init(E=0) == pkg.MOE_ERR_INVALID_ARG
    bad = ctypes.cast((ctypes.c_void_p * 2)(FAKE, FAKE + 8), ctypes.c_void_p)
    assert init(g=bad) == pkg.MOE_ERR_INVALID_ARG                    # a misaligned expert
    ffn = lambda **kw: lib.moe_expert_ffn_list(
        FAKE, None, kw.get("payload", 0), FAKE, 64, 8, kw.get("H", 256), 512,
        kw.get("list", FAKE), FAKE, FAKE, kw.get("ws_bytes", 1 << 30), None)
    assert ffn(list=None) == pkg.MOE_ERR_INVALID_ARG
    assert ffn(list=FAKE + 16) == pkg.MOE_ERR_INVALID_ARG
    assert ffn(H=200) == pkg.MOE_ERR_UNSUPPORTED
    assert ffn(payload=1) == pkg.MOE_ERR_INVALID_ARG                 # FP8 without scales
    assert ffn(ws_bytes=100) == pkg.MOE_ERR_WORKSPACE


def _declared_prototypes():
    """{name: (return type, [parameter types])} of every function declared in include/moe.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"([A-Za-z_][A-Za-z0-9_ \*]*?)\b(moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        if params in ("", "void"):
            types = []
        else:
            types = []
            for p in params.split(","):
                p = " ".join(p.split())
                # drop the parameter name: the last identifier
                t = re.sub(r"\b[A-Za-z_][A-Za-z0-9_]*\s*$", "", p).strip()
                types.append(t)
        out[name] = (ret, types)
    return out


def _ctype_for(c_type: str):
    import ctypes
    if "*" in c_type or c_type == "moe_stream_t":
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "double": ctypes.c_double,
            "moe_payload_t": ctypes.c_int, "moe_status_t": ctypes.c_int}[c_type]


def test_binding_signatures_match_the_header(lib):
    """Every ctypes prototype of the binding has the header's parameter count and kinds: a
    pointer passed where the table says int would be truncated to 32 bits."""
    import ctypes
    protos = _declared_prototypes()
    assert set(protos) == set(declared_functions())
    for name, (ret, types) in protos.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == len(types), (name, len(fn.argtypes), types)
        for i, (got, t) in enumerate(zip(fn.argtypes, types)):
            assert got == _ctype_for(t), (name, i, t, got)
        if ret == "const char*":
            assert fn.restype == ctypes.c_char_p, name
        else:
            assert fn.restype == _ctype_for(ret), (name, ret, fn.restype)
