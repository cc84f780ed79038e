"""Host-only checks of the C ABI: the library builds and loads, exports every
function include/flint_attn.h declares, and rejects bad arguments before it
touches the GPU (these calls pass fake, never-dereferenced addresses)."""
import ctypes
import os
import re

import pytest

import full_gqa_learned_b200 as fa
from full_gqa_learned_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flint_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flint_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("flint_attn_fwd", "flint_attn_workspace_bytes", "flint_attn_device_status",
              "flint_attn_last_error", "flint_attn_status_string", "flint_attn_abi_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_no_unexpected_exports(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r" T (flint_\w+)", out))
    assert exported == set(declared_functions())


def test_version_and_status_strings(lib):
    assert lib.flint_attn_abi_version() == 1
    assert lib.flint_attn_status_string(0) == b"FLINT_OK"
    assert lib.flint_attn_status_string(5) == b"FLINT_ERR_WORKSPACE"


def test_workspace_bytes(lib):
    assert fa.workspace_bytes(0, 1) > 0
    a = fa.workspace_bytes(4096, 1)
    # normalised FP16 keys dominate: 1 KiB per token
    assert 4096 * 1024 <= a < 4096 * 1024 + (1 << 20)
    assert fa.workspace_bytes(-1, 1) == 0
    assert fa.workspace_bytes(1 << 25, 1) == 0
    assert fa.workspace_bytes(4096, 8) >= a


A = 0x100000  # fake, 256-byte aligned, never dereferenced


def call(lib, **kw):
    args = dict(q=A, k=A, v=A, wq=A, wk=A, sinks=A, pos=None, cu=None, ndocs=0, mask=None,
                batch=0, seqlen=0, T=64, window=513, use_rope=1, theta=1e4, eps=1e-6,
                out=A, lse=A, ws=A, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return lib.flint_attn_fwd(args["q"], args["k"], args["v"], args["wq"], args["wk"],
                              args["sinks"], args["pos"], args["cu"], args["ndocs"],
                              args["mask"], args["batch"], args["seqlen"], args["T"],
                              args["window"], args["use_rope"], args["theta"], args["eps"],
                              args["out"], args["lse"], args["ws"], args["ws_bytes"],
                              args["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), 1),
    (dict(T=(1 << 24) + 1), 1),
    (dict(window=-5), 1),
    (dict(use_rope=2), 1),
    (dict(eps=0.0), 1),
    (dict(eps=float("nan")), 1),
    (dict(theta=1.0), 1),
    (dict(cu=A, mask=A), 1),
    (dict(cu=A, ndocs=-1), 1),
    (dict(mask=A, batch=3, seqlen=5, T=16), 1),
    (dict(mask=A, batch=0, seqlen=5, T=0), 1),
    (dict(q=None), 1),
    (dict(sinks=None), 1),
    (dict(out=None), 1),
    (dict(q=A + 8), 1),
    (dict(out=A + 2), 1),
    (dict(wq=A + 2), 1),
    (dict(ws=None), 5),
    (dict(ws=A + 64), 5),
    (dict(ws_bytes=1024), 5),
])
def test_invalid_arguments_rejected_on_host(lib, kw, status):
    assert call(lib, **kw) == status
    assert lib.flint_attn_last_error() != b""


def test_empty_input_is_a_noop(lib):
    assert call(lib, T=0) == 0
    assert call(lib, T=0, q=None, k=None, v=None, out=None, ws=None) == 0


def test_rope_theta_ignored_without_rope(lib):
    # theta is only validated on sliding layers; the call then fails on the
    # workspace size, before any device work
    assert call(lib, use_rope=0, theta=0.0, ws_bytes=16) == 5


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(fa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(fa, "_lib", None)
    with pytest.raises(ImportError):
        fa.load_library()
    importlib.reload(fa)


# ---------------------------------------------------------------- decode entry

def call_decode(lib, **kw):
    args = dict(q=A, k=A, v=A, wq=A, wk=A, sinks=A, kc=A, vc=A, lens=A, B=8, cap=513, window=513,
                use_rope=1, theta=1e4, eps=1e-6, out=A, lse=A, ws=A, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return lib.flint_attn_decode(args["q"], args["k"], args["v"], args["wq"], args["wk"], args["sinks"],
                                 args["kc"], args["vc"], args["lens"], args["B"], args["cap"],
                                 args["window"], args["use_rope"], args["theta"], args["eps"],
                                 args["out"], args["lse"], args["ws"], args["ws_bytes"], args["stream"])


def test_decode_workspace_bytes(lib):
    # header (status, item counter, per-(sequence, KV head) arrival counters:
    # 256 + 256 bytes for 8 sequences) + partials: 4 KV heads x splits x
    # (8 x 130) floats, for the larger of the two kernels' split counts
    # (CUDA cores: 256 positions of the window per split; tensor cores: 8
    # tiles of 128 cache slots)
    head = 256 + 256
    a = fa.decode_workspace_bytes(8, 513, 513)
    assert a == head + 8 * 4 * 3 * 8 * 130 * 4
    assert fa.decode_workspace_bytes(8, 4096, 0) == head + 8 * 4 * 16 * 8 * 130 * 4
    # a ring larger than the window: the tensor-core splits follow the slots
    assert fa.decode_workspace_bytes(8, 4096, 513) == head + 8 * 4 * 4 * 8 * 130 * 4
    assert fa.decode_workspace_bytes(-1, 513, 513) == 0
    assert fa.decode_workspace_bytes(8, 0, 513) == 0
    assert fa.decode_workspace_bytes(8, 513, -1) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1),
    (dict(B=70000), 1),
    (dict(cap=0), 1),
    (dict(window=-1), 1),
    (dict(use_rope=3), 1),
    (dict(eps=-1.0), 1),
    (dict(theta=0.5), 1),
    (dict(q=None), 1),
    (dict(kc=None), 1),
    (dict(lens=None), 1),
    (dict(kc=A + 8), 1),
    (dict(lens=A + 2), 1),
    (dict(ws=None), 5),
    (dict(ws=A + 16), 5),
    (dict(ws_bytes=512), 5),
])
def test_decode_invalid_arguments_rejected_on_host(lib, kw, status):
    assert call_decode(lib, **kw) == status
    assert lib.flint_attn_last_error() != b""


def test_decode_empty_batch_is_a_noop(lib):
    assert call_decode(lib, B=0) == 0
    assert call_decode(lib, B=0, q=None, kc=None, out=None, ws=None) == 0


# ---------------------------------------------------------------- backward entry

def call_bwd(lib, **kw):
    args = dict(q=A, k=A, v=A, wq=A, wk=A, sinks=A, pos=None, cu=None, ndocs=0, mask=None,
                batch=0, seqlen=0, T=64, window=513, use_rope=1, theta=1e4, eps=1e-6,
                out=A, lse=A, dout=A, dq=A, dk=A, dv=A, dwq=A, dwk=A, dsinks=A,
                ws=A, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return lib.flint_attn_bwd(args["q"], args["k"], args["v"], args["wq"], args["wk"], args["sinks"],
                              args["pos"], args["cu"], args["ndocs"], args["mask"], args["batch"],
                              args["seqlen"], args["T"], args["window"], args["use_rope"],
                              args["theta"], args["eps"], args["out"], args["lse"], args["dout"],
                              args["dq"], args["dk"], args["dv"], args["dwq"], args["dwk"],
                              args["dsinks"], args["ws"], args["ws_bytes"], args["stream"])


def test_bwd_workspace_bytes(lib):
    # the FP16 tensor-core operands q~, k~ dominate: 9 KiB per token, plus
    # bounds and D (136 bytes per token) and fixed per-CTA partials
    a = fa.bwd_workspace_bytes(4096)
    assert 4096 * (8192 + 1024) <= a < 4096 * (8192 + 1024 + 256) + (4 << 20)
    assert fa.bwd_workspace_bytes(0) > 0
    assert fa.bwd_workspace_bytes(-1) == 0
    assert fa.bwd_workspace_bytes((1 << 24) + 1) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), 1),
    (dict(T=(1 << 24) + 1), 1),
    (dict(window=-1), 1),
    (dict(use_rope=2), 1),
    (dict(eps=0.0), 1),
    (dict(theta=0.5), 1),
    (dict(cu=A, mask=A), 1),
    (dict(cu=A, ndocs=-2), 1),
    (dict(mask=A, batch=3, seqlen=5, T=16), 1),
    (dict(dsinks=None), 1),
    (dict(dwq=A + 2), 1),
    (dict(q=None), 1),
    (dict(lse=None), 1),
    (dict(dout=None), 1),
    (dict(dq=None), 1),
    (dict(dv=None), 1),
    (dict(dout=A + 8), 1),
    (dict(dk=A + 4), 1),
    (dict(lse=A + 2), 1),
    (dict(ws=None), 5),
    (dict(ws=A + 64), 5),
    (dict(ws_bytes=4096), 5),
])
def test_bwd_invalid_arguments_rejected_on_host(lib, kw, status):
    assert call_bwd(lib, **kw) == status
    assert lib.flint_attn_last_error() != b""


def test_bwd_empty_input_checks_the_small_gradients_first(lib):
    # T == 0 zeroes dq_norm_w, dk_norm_w and dsinks, so those must be given
    assert call_bwd(lib, T=0, dwk=None) == 1


def test_header_is_plain_c_and_links_against_the_library(lib, tmp_path):
    """A C11 program that includes the header and references every entry
    point compiles with -Wall -Werror and links against libflint_attn.so
    (nothing is run)."""
    import subprocess
    names = declared_functions()
    src = tmp_path / "use_abi.c"
    body = "\n".join("    p = (void (*)(void))&%s; (void)p;" % n for n in names)
    src.write_text('#include "flint_attn.h"\n#include <stdio.h>\n'
                   "int main(void) {\n    void (*p)(void);\n%s\n"
                   '    printf("%%d\\n", (int)FLINT_OK);\n    return 0;\n}\n' % body)
    exe = tmp_path / "use_abi"
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-Wno-pedantic",
                        "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                        "-L", os.path.dirname(fa.LIB_PATH), "-lflint_attn",
                        "-Wl,-rpath," + os.path.dirname(fa.LIB_PATH)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


# ---------------------------------------------------------------- projections and layer

def call_proj(lib, which, **kw):
    a = dict(x=A, w=A, T=64, hidden=2048, o0=A, o1=A, o2=A, stream=None)
    a.update(kw)
    if which == "qkv":
        return lib.flint_qkv_proj(a["x"], a["w"], a["T"], a["hidden"], a["o0"], a["o1"], a["o2"],
                                  a["stream"])
    return lib.flint_o_proj(a["x"], a["w"], a["T"], a["hidden"], a["o0"], a["stream"])


@pytest.mark.parametrize("which", ["qkv", "o"])
@pytest.mark.parametrize("kw", [dict(T=-1), dict(T=(1 << 24) + 1), dict(hidden=0), dict(hidden=100),
                                dict(hidden=1 << 20), dict(x=None), dict(w=None), dict(o0=None),
                                dict(x=A + 8), dict(w=A + 2), dict(o0=A + 4)])
def test_projection_arguments_rejected_on_host(lib, which, kw):
    assert call_proj(lib, which, **kw) == 1
    assert lib.flint_attn_last_error() != b""


@pytest.mark.parametrize("which", ["qkv", "o"])
def test_projection_empty_input_is_a_noop(lib, which):
    assert call_proj(lib, which, T=0, x=None, w=None, o0=None, o1=None, o2=None) == 0


def call_layer(lib, **kw):
    a = dict(x=A, wqkv=A, wo=A, wq=A, wk=A, sinks=A, pos=None, cu=None, ndocs=0, mask=None, batch=0,
             seqlen=0, T=64, hidden=2048, window=513, use_rope=1, theta=1e4, eps=1e-6, q=A, k=A, v=A,
             a=A, y=A, lse=A, ws=A, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.flint_attn_layer_fwd(a["x"], a["wqkv"], a["wo"], a["wq"], a["wk"], a["sinks"], a["pos"],
                                    a["cu"], a["ndocs"], a["mask"], a["batch"], a["seqlen"], a["T"],
                                    a["hidden"], a["window"], a["use_rope"], a["theta"], a["eps"],
                                    a["q"], a["k"], a["v"], a["a"], a["y"], a["lse"], a["ws"],
                                    a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(hidden=96), 1), (dict(x=None), 1), (dict(wo=None), 1), (dict(y=A + 2), 1),
    (dict(window=-1), 1), (dict(q=None), 1), (dict(a=None), 1), (dict(ws=None), 5),
    (dict(ws_bytes=1024), 5), (dict(cu=A, mask=A), 1),
])
def test_layer_arguments_rejected_on_host(lib, kw, status):
    assert call_layer(lib, **kw) == status
    assert lib.flint_attn_last_error() != b""


def test_fp16_policy_workspace_and_rejection(lib):
    a = fa.workspace_bytes(4096, 1)
    b = fa.fp16_workspace_bytes(4096, 1)
    # plus the FP16 queries and values: 9 KiB per token
    assert a + 4096 * 9216 <= b < a + 4096 * 9216 + 4096
    assert fa.fp16_workspace_bytes(-1, 1) == 0
    args = [A, A, A, A, A, A, None, None, 0, None, 0, 0, 64, 513, 1, 1e4, 1e-6, A, A, A, 0, None]
    args[20] = fa.workspace_bytes(64, 1)            # enough for the BF16 path, not for this one
    assert lib.flint_attn_fwd_fp16(*args) == 5
    args[20] = 1 << 40
    args[0] = A + 8                                 # misaligned q
    assert lib.flint_attn_fwd_fp16(*args) == 1
    args[0] = A
    args[12] = 0                                    # T = 0: no-op
    assert lib.flint_attn_fwd_fp16(*args) == 0
