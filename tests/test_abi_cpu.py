"""The C ABI without a GPU: the library loads, exports every entry point that
include/la.h declares, the Python binding's ctypes signatures and structures
match the header's declarations and C layouts, the library sizes its workspace
on the host, and it rejects bad arguments before enqueuing anything (so no
call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

from block_causal_linear_b200 import build as la_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def la():
    la_build.build()
    from block_causal_linear_b200 import la as _la

    return _la


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("la_state_init", "la_block_forward", "la_full_forward", "la_workspace_size",
              "la_status_string", "la_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(la):
    lib = la.lib()
    for n in declared_symbols():
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def _c_kind(decl):
    """The ABI kind of one C parameter or return type of include/la.h."""
    t = " ".join(decl.replace("const", " ").split())
    if "*" in t:
        return "char*" if t.startswith("char") and t.count("*") == 1 and t.split("*")[0].strip() == "char" \
            else "ptr"
    base = t.split()[0] if t else "void"
    return {"size_t": "size_t", "float": "float", "void": "void", "long": "int64"}.get(base, "int")


def _ctypes_kind(t):
    if t is None:
        return "void"
    if t is ctypes.c_char_p:
        return "char*"
    if t is ctypes.c_void_p or isinstance(t, type(ctypes.POINTER(ctypes.c_int))):
        return "ptr"
    return {ctypes.c_size_t: "size_t", ctypes.c_float: "float", ctypes.c_int: "int",
            ctypes.c_longlong: "int64"}.get(t, repr(t))


def test_binding_signatures_match_the_header(la):
    """Every entry point's ctypes argtypes and restype in la.py agree with its
    C declaration: same count, and pointer / int / float / size_t in the same
    places (a drifted signature would pass garbage across the boundary)."""
    text = re.sub(r"/\*.*?\*/", "", "".join(open(os.path.join(ROOT, "include", h)).read()
                                            for h in os.listdir(os.path.join(ROOT, "include")) if h.endswith(".h")),
                  flags=re.S)
    decls = re.findall(r"LA_API\s+([\w\s\*]+?)\b(la_\w+)\s*\(([^)]*)\)\s*;", text)
    assert len(decls) == len(declared_symbols())
    lib = la.lib()
    for ret, name, params in decls:
        params = " ".join(params.split())
        want = [] if params in ("", "void") else [
            _c_kind(re.sub(r"\b\w+$", "", p.strip()) if not p.strip().endswith("*") else p) for p in params.split(",")]
        fn = getattr(lib, name)
        got = [_ctypes_kind(a) for a in (fn.argtypes or [])]
        assert got == want, f"{name}: la.py {got} vs la.h {want}"
        assert _ctypes_kind(fn.restype) == _c_kind(ret), f"{name}: restype"


def test_binding_structs_match_the_header(la, tmp_path):
    """la_rope, la_state and la_state_counters have the same size and field
    offsets in la.py's ctypes structures as the C compiler gives them."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"la_rope": la.la_rope, "la_state": la.la_state, "la_state_counters": la.la_state_counters}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "la.h"', "int main(void) {"]
    for s, py in structs.items():
        lines.append(f'printf("{s} size %zu\\n", sizeof({s}));')
        for f, _ in py._fields_:
            lines.append(f'printf("{s} {f} %zu\\n", offsetof({s}, {f}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    got = {tuple(x.split()[:2]): int(x.split()[2]) for x in out if x.strip()}
    for s, py in structs.items():
        assert got[(s, "size")] == ctypes.sizeof(py), s
        for f, _ in py._fields_:
            assert got[(s, f)] == getattr(py, f).offset, f"{s}.{f}"


def test_status_strings(la):
    for s in range(6):
        assert la.la_status_string(s).startswith("LA_")
    assert "unknown" in la.la_status_string(99)


def test_workspace_size_host_only(la):
    a = la.la_workspace_size(1, 8190, 64, 32, 0)
    assert a > 0 and a % 256 == 0
    # invalid sizes
    assert la.la_workspace_size(0, 10, 1, 32, 0) == 0
    assert la.la_workspace_size(1, 0, 1, 32, 0) == 0
    assert la.la_workspace_size(1, 10, 1, 32, -1) == 0
    # the workspace of a streaming block does not grow with the number of blocks
    # already streamed (it only depends on this block's shape)
    blk = la.la_workspace_size(1, 15600, 64, 32, 15600)
    assert blk == la.la_workspace_size(1, 15600, 64, 32, 0)
    # many blocks in one call need one effective state per block
    assert la.la_workspace_size(1, 24 * 15600, 64, 32, 15600) > blk


FAKE = 1 << 20    # never dereferenced: every call below fails validation first


def _full(la, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, dt=la.LA_BF16, B=1, N=256, H=4, d=32, tpb=0,
             rope=None, eps=1e-6, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return la.la_full_forward(a["q"], a["k"], a["v"], a["out"], a["dt"], a["B"], a["N"], a["H"], a["d"],
                              a["tpb"], a["rope"], a["eps"], a["ws"], a["ws_bytes"], a["stream"])


def test_full_forward_validation(la):
    assert _full(la, q=None) == la.LA_EINVAL
    assert _full(la, out=FAKE + 8) == la.LA_EINVAL              # misaligned
    assert _full(la, d=16) == la.LA_EUNSUPPORTED
    assert _full(la, d=64) == la.LA_EUNSUPPORTED
    assert _full(la, N=0) == la.LA_EINVAL
    assert _full(la, B=-1) == la.LA_EINVAL
    assert _full(la, dt=7) == la.LA_EINVAL
    assert _full(la, eps=float("nan")) == la.LA_EINVAL
    assert _full(la, eps=-1.0) == la.LA_EINVAL
    assert _full(la, tpb=-3) == la.LA_EINVAL
    assert _full(la, ws=None) == la.LA_EWORKSPACE
    assert _full(la, ws_bytes=16) == la.LA_EWORKSPACE
    assert _full(la, ws=FAKE + 16) == la.LA_EWORKSPACE        # not 256-byte aligned
    bad = la.make_rope(Hg=2, Wg=2, dims=(8, 12, 10))            # sections do not sum to d
    assert _full(la, rope=bad) == la.LA_EINVAL
    odd = la.make_rope(Hg=2, Wg=2, dims=(7, 13, 12))
    assert _full(la, rope=odd) == la.LA_EINVAL
    neg = la.make_rope(Hg=2, Wg=2, t_offset=-1)                 # only block_forward may defer t
    assert _full(la, rope=neg) == la.LA_EINVAL
    zero = la.make_rope(Hg=0, Wg=2)
    assert _full(la, rope=zero) == la.LA_EINVAL


def test_block_forward_and_state_validation(la):
    st = la.la_state()
    assert la.la_state_init(st, None, FAKE, 1, 4, 32, None) == la.LA_EINVAL
    assert la.la_state_init(st, FAKE, FAKE, 1, 4, 16, None) == la.LA_EUNSUPPORTED
    # a state that was never bound
    assert la.la_block_forward(FAKE, FAKE, FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, st, 1, None, 1e-6,
                               FAKE, 1 << 30, None) == la.LA_EINVAL
    # a state bound to other sizes
    st.S, st.Z, st.B, st.H, st.d = FAKE, FAKE, 1, 8, 32
    assert la.la_block_forward(FAKE, FAKE, FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, st, 1, None, 1e-6,
                               FAKE, 1 << 30, None) == la.LA_EINVAL
    st.H = 4
    assert la.la_block_forward(FAKE, FAKE, FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, st, 1, None, 1e-6,
                               FAKE, 8, None) == la.LA_EWORKSPACE
    assert st.blocks_committed == 0


def _bwd(la, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, dt=la.LA_BF16, B=1, N=256, H=4,
             d=32, tpb=0, rope=None, eps=1e-6, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return la.la_full_backward(a["q"], a["k"], a["v"], a["dout"], a["dq"], a["dk"], a["dv"], a["dt"], a["B"],
                               a["N"], a["H"], a["d"], a["tpb"], a["rope"], a["eps"], a["ws"], a["ws_bytes"],
                               a["stream"])


def test_full_backward_validation(la):
    for name in ("q", "k", "v", "dout", "dq", "dk", "dv"):
        assert _bwd(la, **{name: None}) == la.LA_EINVAL
        assert _bwd(la, **{name: FAKE + 8}) == la.LA_EINVAL      # misaligned
    assert _bwd(la, d=16) == la.LA_EUNSUPPORTED
    assert _bwd(la, N=0) == la.LA_EINVAL
    assert _bwd(la, dt=7) == la.LA_EINVAL
    assert _bwd(la, tpb=-1) == la.LA_EINVAL
    assert _bwd(la, eps=float("inf")) == la.LA_EINVAL
    assert _bwd(la, ws=None) == la.LA_EWORKSPACE
    assert _bwd(la, ws_bytes=la.la_backward_workspace_size(1, 256, 4, 32, 0) - 1) == la.LA_EWORKSPACE
    assert _bwd(la, rope=la.make_rope(Hg=2, Wg=2, t_offset=-1)) == la.LA_EINVAL


def test_backward_workspace_size(la):
    fwd = la.la_workspace_size(1, 4 * 640, 8, 32, 640)
    bwd = la.la_backward_workspace_size(1, 4 * 640, 8, 32, 640)
    assert bwd > fwd and bwd % 256 == 0
    assert la.la_backward_workspace_size(1, 0, 8, 32, 0) == 0


def test_e4m3_validation(la):
    def full(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, sq=0.01, sk=0.01, sv=0.01, out=FAKE, B=1, N=256, H=4, d=32, tpb=0,
                 rope=None, eps=1e-6, ws=FAKE, ws_bytes=1 << 30, stream=None)
        a.update(kw)
        return la.la_full_forward_e4m3(a["q"], a["k"], a["v"], a["sq"], a["sk"], a["sv"], a["out"], a["B"], a["N"],
                                       a["H"], a["d"], a["tpb"], a["rope"], a["eps"], a["ws"], a["ws_bytes"],
                                       a["stream"])
    assert full(q=None) == la.LA_EINVAL
    assert full(out=FAKE + 4) == la.LA_EINVAL
    assert full(sq=0.0) == la.LA_EINVAL
    assert full(sk=-1.0) == la.LA_EINVAL
    assert full(sv=float("nan")) == la.LA_EINVAL
    assert full(d=16) == la.LA_EUNSUPPORTED
    assert full(H=6) == la.LA_EUNSUPPORTED             # the E4M3 path takes 4-head groups
    # RoPE is checked like the bf16 calls': dims must add up to d, even and >= 0
    assert full(rope=la.make_rope(Hg=3, Wg=5, dims=(8, 12, 10))) in (la.LA_EINVAL, la.LA_EUNSUPPORTED)
    assert full(rope=la.make_rope(Hg=3, Wg=5, t_offset=-1)) in (la.LA_EINVAL, la.LA_EUNSUPPORTED)
    st = la.la_state()
    assert la.la_block_forward_e4m3(FAKE, FAKE, FAKE, 1.0, 1.0, 1.0, FAKE, 1, 64, 4, 32, st, 1, None, 1e-6, FAKE,
                                    1 << 30, None) in (la.LA_EINVAL, la.LA_EUNSUPPORTED)
    assert st.blocks_committed == 0


def test_nvfp4_validation(la):
    def full(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, qs=FAKE, ks=FAKE, vs=FAKE, sq=0.01, sk=0.01, sv=0.01, out=FAKE, B=1, N=256,
                 H=8, d=32, tpb=0, rope=None, eps=1e-6, ws=FAKE, ws_bytes=1 << 30, stream=None)
        a.update(kw)
        return la.la_full_forward_nvfp4(a["q"], a["k"], a["v"], a["qs"], a["ks"], a["vs"], a["sq"], a["sk"], a["sv"],
                                        a["out"], a["B"], a["N"], a["H"], a["d"], a["tpb"], a["rope"], a["eps"],
                                        a["ws"], a["ws_bytes"], a["stream"])
    assert full(k=None) == la.LA_EINVAL
    assert full(vs=None) == la.LA_EINVAL                # a missing block-scale tensor
    assert full(qs=FAKE + 8) == la.LA_EINVAL            # block scales must be 16-byte aligned
    assert full(sk=0.0) == la.LA_EINVAL
    assert full(sv=float("inf")) == la.LA_EINVAL
    assert full(d=64) == la.LA_EUNSUPPORTED
    assert full(H=4) == la.LA_EUNSUPPORTED              # rows of block scales must be whole 16-byte units
    assert full(rope=la.make_rope(Hg=3, Wg=5, dims=(8, 12, 10))) in (la.LA_EINVAL, la.LA_EUNSUPPORTED)
    st = la.la_state()
    assert la.la_block_forward_nvfp4(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1.0, 1.0, 1.0, FAKE, 1, 64, 8, 32, st, 1,
                                     None, 1e-6, FAKE, 1 << 30, None) in (la.LA_EINVAL, la.LA_EUNSUPPORTED)
    assert st.blocks_committed == 0


def test_e4m3_quantiser_round_trip():
    import torch
    from block_causal_linear_b200 import synth

    x = torch.randn(3, 100, 2, 32, generator=torch.Generator().manual_seed(5))
    codes, s = synth.to_e4m3(x)
    assert codes.dtype == torch.uint8 and codes.shape == x.shape and s > 0
    back = codes.view(torch.float8_e4m3fn).to(torch.float32) * s
    # E4M3 keeps 4 significant bits: relative error <= 2^-4 for normal values
    big = x.abs() > 2.0 ** -6 * s
    assert bool(((back - x).abs() <= 2.0 ** -4 * x.abs() + 1e-30)[big].all())
    # amax scaling: the largest magnitude lands on the largest code, 448
    assert float(codes.view(torch.float8_e4m3fn).to(torch.float32).abs().max()) == 448.0


def test_dwconv_validation(la):
    def call(**kw):
        a = dict(x=FAKE, y=FAKE, dt=la.LA_BF16, B=1, T=3, Hg=4, Wg=5, C=64, kt=1, kh=3, kw=3, w=FAKE, b=None)
        a.update(kw)
        return la.la_dwconv3d(a["x"], a["y"], a["dt"], a["B"], a["T"], a["Hg"], a["Wg"], a["C"], a["kt"], a["kh"],
                              a["kw"], a["w"], a["b"], None)
    assert call(x=None) == la.LA_EINVAL
    assert call(w=None) == la.LA_EINVAL
    assert call(y=FAKE + 2) == la.LA_EINVAL
    assert call(T=0) == la.LA_EINVAL
    assert call(dt=5) == la.LA_EINVAL
    assert call(C=12) == la.LA_EUNSUPPORTED
    assert call(kt=3, kh=3, kw=3) == la.LA_EUNSUPPORTED
    assert call(kt=1, kh=1, kw=1) == la.LA_EUNSUPPORTED


def test_token_split_validation(la):
    assert la.la_split_partial_bytes(1, 4, 32) == 4 * 1056 * 4
    assert la.la_split_partial_bytes(0, 4, 32) == 0
    # reduce: null / misaligned partial, bad sizes, small workspace
    assert la.la_block_reduce(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, None, None, FAKE, 1 << 30, None) == la.LA_EINVAL
    assert la.la_block_reduce(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, None, FAKE + 4, FAKE, 1 << 30, None) == la.LA_EINVAL
    assert la.la_block_reduce(FAKE, FAKE, la.LA_BF16, 1, 0, 4, 32, None, FAKE, FAKE, 1 << 30, None) == la.LA_EINVAL
    assert la.la_block_reduce(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, None, FAKE, FAKE, 8, None) == la.LA_EWORKSPACE
    # apply: rank count, unbound state, gathered pointer
    st = la.la_state()
    assert la.la_block_apply(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, FAKE, 2, st, 1, None, 1e-6, FAKE, 1 << 30,
                             None) == la.LA_EINVAL
    st.S, st.Z, st.B, st.H, st.d = FAKE, FAKE, 1, 4, 32
    for R in (0, 33):
        assert la.la_block_apply(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, FAKE, R, st, 1, None, 1e-6, FAKE, 1 << 30,
                                 None) == la.LA_EINVAL
    assert la.la_block_apply(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, None, 2, st, 1, None, 1e-6, FAKE, 1 << 30,
                             None) == la.LA_EINVAL
    assert la.la_block_apply(FAKE, FAKE, la.LA_BF16, 1, 64, 4, 32, FAKE, 2, st, 1, None, 1e-6, FAKE, 8,
                             None) == la.LA_EWORKSPACE
    assert st.blocks_committed == 0


def test_static_ws_validation(la):
    """The allocation-free variant rejects bad arguments, and shapes whose
    scratch exceeds its static array, before it looks up the array."""
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, dt=la.LA_BF16, B=1, N=256, H=4, d=32, tpb=0, rope=None,
                 eps=1e-6)
        a.update(kw)
        return la.la_full_forward_static_ws(a["q"], a["k"], a["v"], a["out"], a["dt"], a["B"], a["N"], a["H"],
                                            a["d"], a["tpb"], a["rope"], a["eps"], None)
    assert call(q=None) == la.LA_EINVAL
    assert call(v=FAKE + 4) == la.LA_EINVAL
    assert call(eps=-1.0) == la.LA_EINVAL
    assert call(eps=float("nan")) == la.LA_EINVAL
    assert call(tpb=-1) == la.LA_EINVAL
    assert call(d=16) == la.LA_EUNSUPPORTED
    assert call(rope=la.make_rope(Hg=2, Wg=2, t_offset=-1)) == la.LA_EINVAL
    # 64 x 2000 tokens x 64 heads in blocks of 100 needs far more than the array
    assert la.la_workspace_size(64, 2000, 64, 32, 100) > la.LA_STATIC_WS_BYTES
    assert call(B=64, N=2000, H=64, tpb=100) == la.LA_EWORKSPACE


def test_state_checkpoint_validation(la):
    st = la.la_state()
    c = la.la_state_counters()
    # an unbound state
    assert la.la_state_save(st, FAKE, FAKE, c, None) == la.LA_EINVAL
    assert la.la_state_restore(st, FAKE, FAKE, c, None) == la.LA_EINVAL
    st.S, st.Z, st.B, st.H, st.d = FAKE, FAKE, 1, 4, 32
    st.blocks_committed, st.t_next = 5, 15
    assert la.la_state_save(st, None, FAKE, c, None) == la.LA_EINVAL
    assert la.la_state_save(st, FAKE, None, c, None) == la.LA_EINVAL
    assert la.la_state_save(st, FAKE, FAKE, None, None) == la.LA_EINVAL
    assert la.la_state_restore(st, None, FAKE, c, None) == la.LA_EINVAL
    assert la.la_state_restore(st, FAKE, FAKE, None, None) == la.LA_EINVAL
    c.blocks_committed, c.t_next = -1, 0
    assert la.la_state_restore(st, FAKE, FAKE, c, None) == la.LA_EINVAL
    # nothing was enqueued, so the counters are untouched
    assert (st.blocks_committed, st.t_next) == (5, 15)


PAGE_TITLES = ("Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", "sd114.wiki")


def _decl_comment(text, name):
    """The comment block right before the LA_API declaration of `name`."""
    m = re.search(r"/\*((?:(?!\*/).)*)\*/\s*(?:typedef\s+struct\s*\{[^}]*\}\s*\w+;\s*)*(?:LA_API[^;]*;\s*)*LA_API[^;]*?\b" + name + r"\s*\(",
                  text, re.S)
    assert m, name
    # one line of prose: drop the comment's line breaks and leading stars
    return " ".join(re.sub(r"^\s*\*\s?", "", ln) for ln in m.group(1).splitlines()).replace("  ", " ")


def test_boundary_calls_cite_their_passages():
    """Each call of the boundary names the page and section that defines it,
    or says that the pages have none."""
    text = open(os.path.join(ROOT, "include", "la.h"), encoding="utf-8").read()
    for name in ("la_state_init", "la_block_forward", "la_full_forward", "la_workspace_size",
                 "la_state_save", "la_state_restore"):
        c = _decl_comment(text, name)
        assert any(t in c for t in PAGE_TITLES), name
        assert "section" in c, name
    assert "no counterpart" in _decl_comment(text, "la_status_string")
    assert "no counterpart" in _decl_comment(text, "la_workspace_size")
