"""The C ABI on the host (no GPU): the library loads, exports every symbol the header
declares, and rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def _declared():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if fn.endswith(".h"):
            src = open(os.path.join(HEADER_DIR, fn)).read()
            names |= set(re.findall(r"LA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from long_context_attn_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"lightning_attn_prefill", "lightning_attn_prefill_varlen", "lightning_attn_decode_step"} <= names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_binding_names_match_header(lib):
    from long_context_attn_b200 import lightning_attn as la
    assert set(la.EXPORTED) == _declared()
    for n in la.EXPORTED:
        assert callable(getattr(la, n))


def test_status_strings(lib):
    lib.lightning_attn_status_string.restype = ctypes.c_char_p
    assert lib.lightning_attn_status_string(0) == b"LA_OK"
    assert lib.lightning_attn_status_string(4) == b"LA_ERR_TIMEOUT"
    assert lib.lightning_attn_status_string(99) == b"LA_ERR_UNKNOWN"


def test_decode_workspace_size_is_host_only(lib):
    lib.lightning_attn_workspace_size.restype = ctypes.c_size_t
    n = lib.lightning_attn_workspace_size(2, 256, 0, 0, 64, 128, 0, 1, 2)
    # error record + counters + y [B, H, D] fp32 + per-head partial sums
    assert n >= 256 + 256 * 64 * 128 * 4 + 256 * 64 * 4
    assert lib.lightning_attn_workspace_size(2, 0, 0, 0, 64, 128, 0, 1, 2) == 0
    assert lib.lightning_attn_workspace_size(2, 4, 0, 0, 64, 96, 0, 1, 2) == 0  # D not supported


def test_invalid_arguments_rejected_before_launch(lib):
    f = lib.lightning_attn_prefill
    vp = ctypes.c_void_p
    f.argtypes = [vp, vp, vp, vp, vp, vp, vp] + [ctypes.c_int] * 8 + [ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    fake = vp(0x1000)
    odd = vp(0x1008)
    ws = vp(0x100000)
    args = dict(q=fake, k=fake, v=fake, g=fake, out=fake, si=None, so=None, B=1, T=8, H=2, D=128, C=256,
                dt=1, phi=0, mode=2, eps=1e-6, w=None, ws=ws, wsb=1 << 30, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["q"], a["k"], a["v"], a["g"], a["out"], a["si"], a["so"], a["B"], a["T"], a["H"], a["D"],
                 a["C"], a["dt"], a["phi"], a["mode"], a["eps"], a["w"], a["ws"], a["wsb"], a["st"])

    assert call(D=96) == 1          # unsupported head dim
    assert call(q=None) == 1        # missing input
    assert call(g=None) == 1        # gate required in RMSNORM_GATE mode
    assert call(k=odd) == 1         # misaligned
    assert call(dt=7) == 1          # bad enum
    assert call(mode=1, eps=0.0) == 1   # norm needs eps > 0
    assert call(B=0) == 1
    assert call(C=0) == 1
    assert call(H=200) == 1         # H*D > 16384 with a norm mode
    assert call(ws=None) == 1
    assert call(ws=vp(0x100010)) == 1   # workspace not 256-byte aligned

    d = lib.lightning_attn_decode_step
    d.argtypes = [vp, vp, vp, vp, vp, vp] + [ctypes.c_int] * 6 + [ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    assert d(fake, fake, fake, fake, fake, None, 4, 2, 128, 1, 0, 2, ctypes.c_float(1e-6), None, ws, 1 << 20,
             None) == 1  # missing state
    assert d(fake, fake, fake, fake, fake, fake, 4, 2, 128, 1, 0, 2, ctypes.c_float(1e-6), None, ws, 16,
             None) == 1  # workspace too small


def test_mixed_step_host_checks(lib):
    """The mixed step's split and argument checks happen on the host before any launch."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.lightning_attn_mixed_step
    f.argtypes = [vp] * 9 + [i32] * 7 + [ctypes.c_float, vp, vp, ctypes.c_size_t, vp, vp]
    fake, ws = vp(0x1000), vp(0x100000)
    good = (ctypes.c_int * 4)(0, 1, 5, 6)
    bad = (ctypes.c_int * 4)(0, 3, 2, 6)        # decreasing offsets

    def call(host, **kw):
        a = dict(q=fake, k=fake, v=fake, g=fake, out=fake, cu=fake, pool=fake, slot=fake, n=3, H=2, D=128, C=256,
                 dt=1, phi=0, mode=2, ws=ws)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["g"], a["out"], a["cu"], ctypes.cast(host, vp), a["pool"], a["slot"],
                 a["n"], a["H"], a["D"], a["C"], a["dt"], a["phi"], a["mode"], ctypes.c_float(1e-6), None, a["ws"],
                 1 << 30, None, None)

    assert call(bad) == 1                 # host cu_seqlens decrease
    assert call(good, slot=None) == 1     # no slot map
    assert call(good, pool=None) == 1     # no state pool
    assert call(good, g=None) == 1        # gate required
    assert call(good, D=96) == 1
    assert call(good, ws=vp(0x100010)) == 1
    lib.lightning_attn_workspace_size.restype = ctypes.c_size_t
    # LA_OP_MIXED sizes: prefill part for the longest multi-token sequence + decode part for N.
    n3 = lib.lightning_attn_workspace_size(3, 3, 4, 6, 2, 128, 256, 1, 2)
    n_dec_only = lib.lightning_attn_workspace_size(3, 3, 0, 3, 2, 128, 256, 1, 2)
    assert n3 > n_dec_only > 256


def test_backward_host_checks(lib):
    """The backward's argument checks happen on the host before any launch; its workspace
    holds the raw-pass prefill part plus six token buffers and the transposed states."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.lightning_attn_backward
    f.argtypes = [vp] * 14 + [i32] * 8 + [ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    fake, ws = vp(0x1000), vp(0x100000)

    def call(**kw):
        a = dict(q=fake, k=fake, v=fake, g=fake, dout=fake, s0=None, dsT=None, y=None, dq=fake, dk=fake, dv=fake,
                 dg=fake, ds=None, dw=None, B=1, T=64, H=2, D=128, C=256, dt=1, phi=0, mode=2, ws=ws, nbytes=1 << 40)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["g"], a["dout"], a["s0"], a["dsT"], a["y"], a["dq"], a["dk"], a["dv"],
                 a["dg"], a["ds"], a["dw"],
                 a["B"], a["T"], a["H"], a["D"], a["C"], a["dt"], a["phi"], a["mode"], ctypes.c_float(1e-6), None,
                 a["ws"], a["nbytes"], None)

    assert call(dg=None) == 1             # gate mode needs dg
    assert call(dq=None) == 1
    assert call(dout=vp(0x1008)) == 1     # 16-byte alignment
    assert call(D=96) == 1
    assert call(mode=7) == 1
    assert call(ws=vp(0x100010)) == 1     # 256-byte aligned workspace
    assert call(nbytes=1024) == 1         # workspace too small
    assert call(dsT=vp(0x1008)) == 1      # misaligned final-state gradient
    assert call(y=vp(0x1008)) == 1        # misaligned saved output
    assert call(dw=vp(0x1008)) == 1       # misaligned norm-weight gradient
    lib.lightning_attn_workspace_size.restype = ctypes.c_size_t
    fwd = lib.lightning_attn_workspace_size(0, 2, 1000, 0, 8, 128, 256, 1, 0)
    bwd = lib.lightning_attn_workspace_size(4, 2, 1000, 0, 8, 128, 256, 1, 2)
    bwd_var = lib.lightning_attn_workspace_size(5, 2, 1000, 2000, 8, 128, 256, 1, 2)
    assert bwd >= fwd + 6 * 2000 * 8 * 128 * 2 + 2 * 2 * 8 * 128 * 128 * 4
    assert bwd_var == bwd


def test_chunk_state_workspace_and_checks(lib):
    """LA_OP_CHUNK_STATE needs no block size; bad arguments are rejected on the host."""
    lib.lightning_attn_workspace_size.restype = ctypes.c_size_t
    n = lib.lightning_attn_workspace_size(8, 1, 1000, 0, 8, 128, 0, 1, 0)
    assert n > 256
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f = lib.lightning_attn_chunk_state
    f.argtypes = [vp, vp, vp, vp] + [i32] * 6 + [vp, ctypes.c_size_t, vp]
    fake, ws = vp(0x1000), vp(0x100000)
    assert f(fake, fake, None, None, 1, 64, 2, 128, 1, 0, ws, 1 << 30, None) == 1       # no state_out
    assert f(fake, fake, None, fake, 1, 64, 2, 96, 1, 0, ws, 1 << 30, None) == 1        # D
    assert f(fake, vp(0x1008), None, fake, 1, 64, 2, 128, 1, 0, ws, 1 << 30, None) == 1  # alignment
    assert f(fake, fake, None, fake, 1, 64, 2, 128, 1, 0, ws, 16, None) == 1            # workspace too small


def test_header_is_plain_c_and_links(lib, tmp_path):
    """The header compiles as C11 (no C++ in it) and every entry point it declares links
    against the built library from a C program (compiled and linked with gcc, not run)."""
    import subprocess
    names = sorted(_declared())
    src = tmp_path / "use_abi.c"
    body = "\n".join(f"  (void *)&{n}," for n in names)
    src.write_text('#include "lightning_attn.h"\n#include <stdio.h>\n'
                   f"static void *const entry[] = {{\n{body}\n}};\n"
                   "int main(void) { printf(\"%d\\n\", (int)(sizeof(entry) / sizeof(entry[0]))); return 0; }\n")
    so = os.path.join(ROOT, "long_context_attn_b200", "liblightning_attn.so")
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", HEADER_DIR, str(src), so,
                        "-o", str(tmp_path / "use_abi")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_output_transform_backward_host_checks(lib):
    """lightning_attn_output_transform_backward rejects bad arguments on the host; its
    workspace (the norm weight's gradient as partial rows) is sized from the token count."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.lightning_attn_workspace_size.restype = ctypes.c_size_t
    n0 = lib.lightning_attn_workspace_size(9, 0, 0, 0, 8, 128, 0, 1, 2)
    n1 = lib.lightning_attn_workspace_size(9, 100, 0, 0, 8, 128, 0, 1, 2)
    n2 = lib.lightning_attn_workspace_size(9, 100000, 0, 0, 8, 128, 0, 1, 2)
    assert n0 >= 256 and n1 >= 100 * 8 * 128 * 4 and n2 >= 1024 * 8 * 128 * 4 and n2 < 2 * 1024 * 8 * 128 * 4
    assert lib.lightning_attn_workspace_size(9, 100, 0, 0, 8, 96, 0, 1, 2) == 0
    f = lib.lightning_attn_output_transform_backward
    f.argtypes = [vp] * 6 + [i32] * 5 + [ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    y, g, d, dy, dg = (vp(0x1000 * (i + 1)) for i in range(5))
    ws = vp(0x100000)

    def call(**kw):
        a = dict(y=y, g=g, d=d, dy=dy, dg=dg, dw=None, tokens=10, H=8, D=128, dt=1, mode=2, eps=1e-6, w=None, ws=None,
                 nbytes=0)
        a.update(kw)
        return f(a["y"], a["g"], a["d"], a["dy"], a["dg"], a["dw"], a["tokens"], a["H"], a["D"], a["dt"], a["mode"],
                 ctypes.c_float(a["eps"]), a["w"], a["ws"], a["nbytes"], None)

    assert call(dg=None) == 1                     # gate mode needs dg
    assert call(y=None) == 1                      # norm modes need y
    assert call(dy=vp(0x1008)) == 1               # 16-byte alignment
    assert call(dy=d) == 1                        # dy may not be dout
    assert call(dg=dy) == 1                       # dg distinct
    assert call(D=96) == 1
    assert call(H=200) == 1                       # H*D > 16384
    assert call(eps=0.0) == 1
    assert call(mode=5) == 1
    assert call(tokens=-1) == 1
    assert call(dw=vp(0x2000)) == 1               # dw without a workspace
    assert call(dw=vp(0x2000), ws=vp(0x100010), nbytes=1 << 30) == 1   # misaligned workspace
    assert call(dw=vp(0x2000), ws=ws, nbytes=256) == 1                 # workspace too small
    assert call(dw=vp(0x2004), ws=ws, nbytes=1 << 30) == 1             # misaligned dw


def test_binding_constants_match_header_enums(lib):
    """Every LA_* enumerator the header defines has the same value in the Python binding, and
    the binding defines no LA_* status, dtype, mode, feature-map or op constant the header
    lacks."""
    from long_context_attn_b200 import lightning_attn as la
    src = open(os.path.join(HEADER_DIR, "lightning_attn.h")).read()
    enums = {}
    for body in re.findall(r"typedef\s+enum\s*\{(.*?)\}", src, flags=re.S):
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        for name, value in re.findall(r"\b(LA_\w+)\s*=\s*(\d+)", body):
            enums[name] = int(value)
    assert {"LA_OK", "LA_BF16", "LA_OUT_RMSNORM_GATE", "LA_PHI_SILU", "LA_OP_OUTPUT_TRANSFORM_BACKWARD"} <= set(enums)
    for name, value in enums.items():
        if hasattr(la, name):
            assert getattr(la, name) == value, name
    prefixes = ("LA_OK", "LA_ERR_", "LA_F32", "LA_BF16", "LA_OUT_", "LA_PHI_", "LA_OP_")
    py = {n for n in dir(la) if n.startswith(prefixes)}
    assert py <= set(enums), py - set(enums)
    missing = {n for n in enums if n.startswith("LA_OP_")} - py
    assert not missing, missing


def test_binding_argument_counts_match_header(lib):
    """The ctypes argument list the binding sets for each entry point has as many entries as
    the header's declaration has parameters."""
    from long_context_attn_b200 import lightning_attn as la
    src = open(os.path.join(HEADER_DIR, "lightning_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decls = dict(re.findall(r"LA_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)\s*;", src))
    assert len(decls) == len(_declared())
    for name, params in decls.items():
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        argtypes = getattr(la._lib, name).argtypes
        assert argtypes is not None and len(argtypes) == n, (name, n, argtypes)


def test_every_workspace_op_has_a_size(lib):
    """lightning_attn_workspace_size answers every LA_OP_* with a positive size for valid
    arguments and 0 for an invalid head size (host-only query)."""
    from long_context_attn_b200 import lightning_attn as la
    lib.lightning_attn_workspace_size.restype = ctypes.c_size_t
    ops = sorted(getattr(la, n) for n in dir(la) if n.startswith("LA_OP_"))
    assert ops == list(range(len(ops)))
    for op in ops:
        n = lib.lightning_attn_workspace_size(op, 2, 300, 600, 8, 128, 256, la.LA_BF16, la.LA_OUT_RMSNORM_GATE)
        assert n >= 256, op
        assert lib.lightning_attn_workspace_size(op, 2, 300, 600, 8, 100, 256, la.LA_BF16,
                                                 la.LA_OUT_RMSNORM_GATE) == 0, op
