"""Host-side checks of the C ABI (CPU only, no kernel launches).

* the in-tree library loads and exports every function include/gptoss.h declares;
* argument validation rejects bad calls before touching the GPU (each case
  returns before any CUDA runtime call, so it runs on a machine without one);
* the decode workspace size is consistent.
"""

import ctypes
import os
import re

import pytest

from attention_yarn_rope_b200 import _abi, build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return _abi.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "gptoss.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gptoss_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 8
    assert sorted(_abi.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in _abi.STATUS_NAMES.items():
        assert lib.gptoss_status_string(code).decode() == name
    assert lib.gptoss_status_string(99).decode() == "GPTOSS_ERR_UNKNOWN"


ROPE = _abi.RopeParams(150000.0, 32.0, 4096, 64, 1.0, 32.0)
S_BSHD_Q = _abi.Strides(4096 * 64 * 64, 64 * 64, 64)
S_BSHD_K = _abi.Strides(4096 * 8 * 64, 8 * 64, 64)
FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every case fails validation first


def _fwd(lib, **kw):
    a = dict(q=FAKE, sq=S_BSHD_Q, k=FAKE, sk=S_BSHD_K, v=FAKE, sv=S_BSHD_K, sinks=FAKE, pos=None, cu=None, B=1,
             S=4096, T=4096, Hq=64, Hkv=8, D=64, window=0, scale=0.125, rope=ctypes.byref(ROPE), out=FAKE,
             so=S_BSHD_Q, lse=None, ws=FAKE, ws_bytes=1 << 40)
    a.update(kw)
    return lib.gptoss_attn_fwd(a["q"], a["sq"], a["k"], a["sk"], a["v"], a["sv"], a["sinks"], a["pos"], a["cu"],
                               a["B"], a["S"], a["T"], a["Hq"], a["Hkv"], a["D"], a["window"], a["scale"],
                               a["rope"], a["out"], a["so"], a["lse"], a["ws"], a["ws_bytes"], None)


def test_attn_fwd_validation(lib):
    assert _fwd(lib, D=96) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert _fwd(lib, D=128) == _abi.GPTOSS_ERR_UNSUPPORTED          # D = 128 takes full rotary only (rope has 64)
    assert _fwd(lib, Hkv=7) == _abi.GPTOSS_ERR_INVALID_ARG          # Hq % Hkv != 0
    assert _fwd(lib, window=-1) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, T=4095) == _abi.GPTOSS_ERR_INVALID_ARG          # B*S != total for BSHD
    assert _fwd(lib, q=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, sinks=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, q=ctypes.c_void_p(0x10008)) == _abi.GPTOSS_ERR_INVALID_ARG  # not 16-byte aligned
    assert _fwd(lib, sq=_abi.Strides(0, 4097, 64)) == _abi.GPTOSS_ERR_INVALID_ARG  # stride not 16 B multiple
    # partial rotary: any multiple of 16 up to head_dim; others are unsupported
    bad_rope = _abi.RopeParams(150000.0, 32.0, 4096, 24, 1.0, 32.0)
    assert _fwd(lib, rope=ctypes.byref(bad_rope)) == _abi.GPTOSS_ERR_UNSUPPORTED
    bad_rope = _abi.RopeParams(150000.0, 32.0, 4096, 80, 1.0, 32.0)
    assert _fwd(lib, rope=ctypes.byref(bad_rope)) == _abi.GPTOSS_ERR_INVALID_ARG  # beyond head_dim
    bad_rope = _abi.RopeParams(150000.0, 32.0, 4096, 64, 32.0, 1.0)
    assert _fwd(lib, rope=ctypes.byref(bad_rope)) == _abi.GPTOSS_ERR_INVALID_ARG  # alpha >= beta
    # the workspace (fp16 rotated k and v, per-token angle table): required,
    # too small or misaligned is rejected
    need = lib.gptoss_attn_fwd_workspace_size(4096, 8, 64)
    assert need == 2 * 4096 * 8 * 64 * 2 + 4096 * 32 * 8
    assert _fwd(lib, ws=None, ws_bytes=0) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, ws=FAKE, ws_bytes=need - 16) == _abi.GPTOSS_ERR_INVALID_ARG
    assert _fwd(lib, ws=ctypes.c_void_p(0x10008), ws_bytes=need) == _abi.GPTOSS_ERR_INVALID_ARG
    # empty inputs are a successful no-op (nothing launched)
    assert _fwd(lib, B=0, T=0) == _abi.GPTOSS_OK
    assert _fwd(lib, S=0, T=0) == _abi.GPTOSS_OK


def test_attn_bwd_validation(lib):
    need = lib.gptoss_attn_bwd_workspace_size(4096, 64, 8, 64)
    # rotated q and k (fp16) + per-token angle table + <dout, out> and lse log2(e)
    # per row and head + fp32 dK and dV accumulators of split sweeps
    assert need == (4096 * 64 * 64 * 2 + 4096 * 8 * 64 * 2 + 4096 * 32 * 8 + 2 * 4096 * 64 * 4
                    + 2 * 4096 * 8 * 64 * 4)
    assert lib.gptoss_attn_bwd_workspace_size(4096, 64, 7, 64) == 0
    assert lib.gptoss_attn_bwd_workspace_size(4096, 64, 8, 128) == 0

    def call(**kw):
        a = dict(q=FAKE, dout=FAKE, lse=FAKE, dq=FAKE, dsinks=FAKE, B=1, S=4096, T=4096, Hq=64, Hkv=8, D=64,
                 window=0, scale=0.125, ws=FAKE, wsb=need, sq=S_BSHD_Q)
        a.update(kw)
        return lib.gptoss_attn_bwd(a["q"], a["sq"], FAKE, S_BSHD_K, FAKE, S_BSHD_K, FAKE, S_BSHD_Q, a["dout"],
                                   S_BSHD_Q, a["lse"], FAKE, None, None, a["B"], a["S"], a["T"], a["Hq"], a["Hkv"],
                                   a["D"], a["window"], a["scale"], ctypes.byref(a.get("rope", ROPE)), a["dq"], FAKE,
                                   FAKE, a["dsinks"], a["ws"], a["wsb"], None)

    assert call(D=128) == _abi.GPTOSS_ERR_UNSUPPORTED
    # partial rotary: a multiple of 16 features (whole 8-pair groups of the
    # RoPE transpose); others are unsupported
    assert call(rope=_abi.RopeParams(150000.0, 32.0, 4096, 40, 1.0, 32.0)) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert call(rope=_abi.RopeParams(150000.0, 32.0, 4096, 80, 1.0, 32.0)) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(Hq=2048, Hkv=8) == _abi.GPTOSS_ERR_UNSUPPORTED      # more heads than the sink reduction holds
    assert call(Hkv=7) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(window=-1) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(scale=float("inf")) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(T=4000) == _abi.GPTOSS_ERR_INVALID_ARG              # B*S != total for BSHD
    assert call(dsinks=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(lse=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(dout=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(dq=ctypes.c_void_p(0x10008)) == _abi.GPTOSS_ERR_INVALID_ARG  # not 16-byte aligned
    assert call(sq=_abi.Strides(0, 4097, 64)) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(wsb=need - 256) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(ws=None) == _abi.GPTOSS_ERR_INVALID_ARG


def test_rope_qk_validation(lib):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, qo=FAKE, ko=FAKE, B=1, S=16, Hq=64, Hkv=8, D=64, rope=ctypes.byref(ROPE))
        a.update(kw)
        return lib.gptoss_rope_qk(a["q"], S_BSHD_Q, a["k"], S_BSHD_K, a["qo"], S_BSHD_Q, a["ko"], S_BSHD_K, None,
                                  None, a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["rope"], None)

    assert call(rope=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(D=32) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert call(ko=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(B=-1) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(B=0) == _abi.GPTOSS_OK
    assert call(S=0) == _abi.GPTOSS_OK


def test_decode_validation_and_workspace(lib):
    ws = lib.gptoss_attn_decode_workspace_size(64, 32768, 64, 8, 64)
    assert ws > 0 and ws % 16 == 0
    assert lib.gptoss_attn_decode_workspace_size(64, 32768, 64, 8, 128) > ws  # D = 128: twice the partials
    assert lib.gptoss_attn_decode_workspace_size(64, 32768, 64, 8, 96) == 0
    assert lib.gptoss_attn_decode_workspace_size(1, 32768, 64, 7, 64) == 0

    def call(**kw):
        a = dict(B=64, L=32768, Hq=64, Hkv=8, D=64, window=0, ws=FAKE, wsb=ws, seq=FAKE)
        a.update(kw)
        return lib.gptoss_attn_decode(FAKE, FAKE, FAKE, a["seq"], FAKE, a["B"], a["L"], a["Hq"], a["Hkv"], a["D"],
                                      a["window"], 0.125, ctypes.byref(ROPE), FAKE, None, a["ws"], a["wsb"], None)

    assert call(wsb=ws - 16) == _abi.GPTOSS_ERR_INVALID_ARG   # workspace too small
    assert call(ws=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(seq=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(Hq=64, Hkv=2) == _abi.GPTOSS_ERR_UNSUPPORTED   # 32 query heads per group
    assert call(D=96) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert call(window=-5) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(B=0) == _abi.GPTOSS_OK


def test_paged_validation(lib):
    rp = ctypes.byref(ROPE)

    def dec(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, table=FAKE, maxb=4, bs=64, nb=16, lens=FAKE, sinks=FAKE, B=2, q_len=1,
                 Hq=64, Hkv=8, D=64, window=0, scale=0.125, out=FAKE, ws=FAKE, ws_bytes=1 << 30)
        a.update(kw)
        return lib.gptoss_attn_decode_paged(a["q"], a["k"], a["v"], a["table"], a["maxb"], a["bs"], a["nb"],
                                            a["lens"], a["sinks"], a["B"], a["q_len"], a["Hq"], a["Hkv"], a["D"],
                                            a["window"], a["scale"], rp, a["out"], None, a["ws"], a["ws_bytes"],
                                            None)

    assert dec(bs=48) == _abi.GPTOSS_ERR_UNSUPPORTED              # tiles would straddle blocks
    assert dec(nb=1 << 25, bs=128) == _abi.GPTOSS_ERR_UNSUPPORTED  # pool rows >= 2^31
    assert dec(maxb=0) == _abi.GPTOSS_ERR_INVALID_ARG
    assert dec(table=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert dec(ws_bytes=16) == _abi.GPTOSS_ERR_INVALID_ARG
    assert dec(q_len=0) == _abi.GPTOSS_ERR_INVALID_ARG
    assert dec(B=300, q_len=300) == _abi.GPTOSS_ERR_UNSUPPORTED   # 90000 query tokens > one grid dimension
    # the workspace holds every query token's partials: B x q_len sequences
    ws1 = lib.gptoss_attn_decode_workspace_size(2, 256, 64, 8, 64)
    ws4 = lib.gptoss_attn_decode_workspace_size(8, 256, 64, 8, 64)
    assert ws4 > ws1
    assert dec(q_len=4, ws_bytes=ws1) == _abi.GPTOSS_ERR_INVALID_ARG
    assert dec(B=0) == _abi.GPTOSS_OK

    def app(**kw):
        a = dict(kn=FAKE, vn=FAKE, lens=FAKE, table=FAKE, maxb=4, bs=64, kp=FAKE, vp=FAKE, nb=16, B=2, q_len=1,
                 Hkv=8, D=64)
        a.update(kw)
        return lib.gptoss_kv_append_paged(a["kn"], a["vn"], a["lens"], a["table"], a["maxb"], a["bs"], a["kp"],
                                          a["vp"], a["nb"], a["B"], a["q_len"], a["Hkv"], a["D"], rp, None)

    assert app(bs=100) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert app(Hkv=33) == _abi.GPTOSS_ERR_UNSUPPORTED  # one thread per (head, pair): 33 x 32 > 1024
    assert app(D=96) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert app(Hkv=17, D=128) == _abi.GPTOSS_ERR_UNSUPPORTED  # 17 x 64 threads > 1024
    assert app(kp=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert app(q_len=0) == _abi.GPTOSS_ERR_INVALID_ARG
    assert app(q_len=70000) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert app(B=0) == _abi.GPTOSS_OK


def test_wait_limit_setter(lib):
    assert lib.gptoss_set_wait_limit(1000) == _abi.GPTOSS_OK
    assert lib.gptoss_set_wait_limit(0) == _abi.GPTOSS_OK  # back to the default
    assert lib.gptoss_selftest_wait_timeout(0, FAKE, None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert lib.gptoss_selftest_wait_timeout(10, None, None) == _abi.GPTOSS_ERR_INVALID_ARG


def test_product_path_never_imports_oracle():
    pkg = os.path.join(ROOT, "attention_yarn_rope_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f


def test_oracle_is_independent_of_the_cuda_path():
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if f.endswith(".py"):
            txt = open(os.path.join(odir, f)).read()
            for line in txt.splitlines():
                if line.startswith(("import ", "from ")):
                    mod = line.split()[1]
                    assert mod.split(".")[0] in {"numpy", "math", "cmath", "__future__", ""} or mod.startswith("."), (f, line)


def test_qkv_rope_validation(lib):
    S_Q = _abi.Strides(4096 * 64 * 64, 64 * 64, 64)
    S_K = _abi.Strides(4096 * 8 * 64, 8 * 64, 64)
    need = lib.gptoss_qkv_rope_workspace_size(4096, 64)
    assert need >= 4096 * 32 * 8
    assert lib.gptoss_qkv_rope_workspace_size(4096, 96) == 0
    rp64 = _abi.RopeParams(150000.0, 32.0, 4096, 64, 1.0, 32.0)
    rp32 = _abi.RopeParams(150000.0, 32.0, 4096, 32, 1.0, 32.0)

    def call(**kw):
        a = dict(x=FAKE, xs=2880, w=FAKE, b=FAKE, B=1, S=4096, hid=2880, Hq=64, Hkv=8, D=64,
                 rope=ctypes.byref(rp64), q=FAKE, k=FAKE, v=FAKE, ws=FAKE, wsb=need)
        a.update(kw)
        return lib.gptoss_qkv_rope(a["x"], a["xs"], a["w"], a["b"], None, None, a["B"], a["S"], a["hid"], a["Hq"],
                                   a["Hkv"], a["D"], a["rope"], a["q"], S_Q, a["k"], S_K, a["v"], S_K, a["ws"],
                                   a["wsb"], None)

    assert call(D=96) == _abi.GPTOSS_ERR_UNSUPPORTED
    assert call(hid=2884, xs=2884) == _abi.GPTOSS_ERR_UNSUPPORTED       # rows of x not whole 16-byte units
    assert call(rope=ctypes.byref(rp32)) == _abi.GPTOSS_ERR_UNSUPPORTED  # partial rotary is not fused here
    assert call(Hkv=7) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(xs=2000) == _abi.GPTOSS_ERR_INVALID_ARG                  # row stride below hidden
    assert call(w=None) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(ws=None) == _abi.GPTOSS_ERR_INVALID_ARG                  # RoPE needs the angle table
    assert call(wsb=need - 16) == _abi.GPTOSS_ERR_INVALID_ARG
    assert call(S=0) == _abi.GPTOSS_OK
