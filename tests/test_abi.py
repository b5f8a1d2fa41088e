"""The C ABI library: it loads without a GPU, exports every entry point the
header declares, its params struct matches the binding's, and it rejects bad
arguments (and, on a machine without an sm_100 GPU, refuses to run) instead of
falling back to anything."""
import ctypes
import os
import re
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import diffusion_transformer_attention_bidirectional_b200 as K
from diffusion_transformer_attention_bidirectional_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "krea_attn.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"KREA_API\s+[\w\s\*]+?\b(krea_attn_\w+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert len(names) >= 10
    lib = _lib.lib()
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"
    out = subprocess.run(["nm", "-D", "--defined-only", str(_lib.LIB_PATH)], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (krea_attn_\w+)", out))
    assert exported == set(names), exported ^ set(names)


def test_params_layout_matches_header():
    fields = [f for f, _ in _lib.Params._fields_]
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"krea_attn.h\"\nint main(void){\n"
    prog += 'printf("%zu\\n", sizeof(krea_attn_params_t));\n'
    for f in fields:
        prog += f'printf("%zu\\n", offsetof(krea_attn_params_t, {f}));\n'
    prog += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(_lib.Params)
    for f, off in zip(fields, vals[1:]):
        assert getattr(_lib.Params, f).offset == off, f


def test_error_strings():
    for code in range(0, -9, -1):
        s = _lib.lib().krea_attn_error_string(code).decode()
        assert s and s != "unknown error"
    assert _lib.lib().krea_attn_abi_version() == 3


def _fwd(p, T=16, H=8, W=8, mode=0, ptr=1 << 20):
    return _lib.lib().krea_attn_fwd(ptr, ptr, ptr, None, ptr, T, H, W, mode, ctypes.byref(p), None)


def test_invalid_arguments_rejected_without_gpu():
    p = K.make_params(1, 4, 1, 64, 16, 8, 8, in_dtype="f16")
    bad = [
        dict(num_q_heads=6, num_kv_heads=4, code=-2),  # Hq % Hkv
        dict(head_dim=96, code=-2),
        dict(in_dtype=2, code=-2),                     # fp32 input
        dict(out_dtype=1, code=-1),                    # bf16 out for f16 in
        dict(q_start=64, code=-1),
        dict(abi_version=7, code=-1),
        dict(batch=0, code=-1),
    ]
    for b in bad:
        q = K.make_params(1, 4, 1, 64, 16, 8, 8, in_dtype="f16")
        code = b.pop("code")
        for f, v in b.items():
            setattr(q, f, v)
        assert _fwd(q) == code, b
    assert _fwd(p, ptr=(1 << 20) + 8) == -1             # misaligned pointer
    p.q_stride[2] = 60                                    # 120 bytes: not a 16-byte multiple
    assert _fwd(p) == -1
    w = K.make_params(1, 4, 1, 64, 16, 8, 8, window=4)
    assert _fwd(w, mode=2) == -1                          # even window


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_no_device_is_an_error_not_a_fallback():
    p = K.make_params(1, 4, 1, 64, 16, 8, 8, in_dtype="f16")
    assert _fwd(p) == _lib.ERR_NO_DEVICE
    with pytest.raises(ValueError):
        q = torch.zeros(1, 80, 4, 64, dtype=torch.float16)
        K.attention(q, q[:, :, :1], q[:, :, :1], text_len=16, grid_h=8, grid_w=8)


def test_workspace_sizes():
    p = K.make_params(1, 48, 12, 128, 512, 128, 128, in_dtype="f16")
    lay = K.workspace_layout(512, 128, 128, p)
    L = 512 + 128 * 128
    assert lay["q8"] >= L * 12 * 128 * 2          # centred keys first
    assert lay["k8"] - lay["q8"] >= L * 48 * 128
    assert lay["total"] == K.workspace_bytes("tilemix", 512, 128, 128, p)
    assert K.workspace_bytes("dense", 512, 128, 128, p) == 0
    for k in ("kc", "q8", "k8", "sq", "sk", "mu", "part"):
        assert lay[k] % 256 == 0


def test_prologue_arguments_rejected_without_gpu():
    L = _lib.lib()
    r = K.rope_params(128)
    assert tuple(r.axes_dim) == (32, 48, 48) and abs(r.theta - 1e4) < 1e-3 and abs(r.eps - 1e-6) < 1e-12
    s = (ctypes.c_int64 * 3)(1 << 20, 1024, 128)
    ptr = 1 << 20

    def call(rope, d=128, dtype=1, x=ptr):
        return L.krea_attn_qk_prologue(x, ptr, None, ptr, 1, 8, 8, d, dtype, s, s, ctypes.byref(rope), None, None,
                                       None)

    assert call(r, d=96) == _lib.ERR_UNSUPPORTED
    assert call(r, dtype=2) == _lib.ERR_UNSUPPORTED          # fp32
    assert call(r, x=ptr + 8) == _lib.ERR_INVALID_ARG         # misaligned rows
    bad = K.rope_params(128, axes_dim=(32, 47, 49))           # odd axis
    assert call(bad) == _lib.ERR_INVALID_ARG
    big = K.rope_params(128, axes_dim=(64, 48, 48))           # more rotary channels than head_dim
    assert call(big) == _lib.ERR_INVALID_ARG
    assert L.krea_attn_rope_table(ptr, 8, ctypes.byref(K.rope_params(128, theta=-1.0)), ptr, None) == -1


def test_rope_positions_layout():
    pos = K.rope_positions(2, 2, 3)
    assert pos.tolist() == [[0, 0, 0], [1, 0, 0], [0, 0, 0], [0, 0, 1], [0, 0, 2], [0, 1, 0], [0, 1, 1], [0, 1, 2]]
    buf = np.zeros((7, 3), dtype=np.int32)
    L = _lib.lib()
    assert L.krea_attn_rope_positions(2, 2, 3, buf.ctypes.data, 7) == _lib.ERR_INVALID_ARG  # capacity < L
    assert L.krea_attn_rope_positions(2, 2, 0, buf.ctypes.data, 7) == _lib.ERR_INVALID_ARG  # half a grid
    assert L.krea_attn_rope_positions(2, 2, 3, None, 8) == _lib.ERR_INVALID_ARG


def test_exchange_layout_matches_header():
    fields = [f for f, _ in _lib.Exchange._fields_]
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"krea_attn.h\"\nint main(void){\n"
    prog += 'printf("%zu\\n", sizeof(krea_exchange_t));\n'
    for f in fields:
        prog += f'printf("%zu\\n", offsetof(krea_exchange_t, {f}));\n'
    prog += 'printf("%d %d\\n", KREA_EXCHANGE_MAX_RANKS, KREA_IPC_HANDLE_BYTES);\nreturn 0;}\n'
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(_lib.Exchange)
    for f, off in zip(fields, vals[1:]):
        assert getattr(_lib.Exchange, f).offset == off, f
    assert vals[-2:] == [_lib.EXCHANGE_MAX_RANKS, _lib.IPC_HANDLE_BYTES]


def test_exchange_arguments_rejected_without_gpu():
    L = _lib.lib()
    ptr = 1 << 20
    s = (ctypes.c_int64 * 3)(1 << 20, 1024, 128)

    def ex(world=2, rank=0, tokens=64, reserved=0, dst_ok=True):
        e = _lib.Exchange()
        e.world, e.rank, e.tokens_per_rank, e.reserved = world, rank, tokens, reserved
        for j in range(max(0, min(world, 16))):
            e.dst[j] = ptr if dst_ok else None
        for i in range(3):
            e.dst_stride[i] = s[i]
        return e

    def s2h(e, heads=8, d=128, dtype=1, x=ptr):
        return L.krea_attn_seq_to_heads(x, 1, heads, d, dtype, s, ctypes.byref(e), None)

    assert s2h(ex()) == _lib.ERR_NO_DEVICE                    # well-formed: only the device is missing
    assert s2h(ex(), d=96) == _lib.ERR_UNSUPPORTED
    assert s2h(ex(), dtype=7) == _lib.ERR_INVALID_ARG
    assert s2h(ex(world=0)) == _lib.ERR_INVALID_ARG
    assert s2h(ex(world=17)) == _lib.ERR_INVALID_ARG
    assert s2h(ex(rank=2)) == _lib.ERR_INVALID_ARG
    assert s2h(ex(tokens=0)) == _lib.ERR_INVALID_ARG
    assert s2h(ex(reserved=1)) == _lib.ERR_INVALID_ARG
    assert s2h(ex(dst_ok=False)) == _lib.ERR_INVALID_ARG
    assert s2h(ex(world=3), heads=8) == _lib.ERR_INVALID_ARG  # 8 heads do not split over 3 ranks
    assert s2h(ex(), x=ptr + 8) == _lib.ERR_INVALID_ARG       # misaligned rows
    assert s2h(ex(tokens=1 << 24), heads=64) == _lib.ERR_TOO_LARGE
    # the inverse direction takes any head count (this rank's heads)
    assert L.krea_attn_heads_to_seq(ptr, 1, 3, 128, 1, s, ctypes.byref(ex(world=3)), None) == _lib.ERR_NO_DEVICE
    r = K.rope_params(128)
    pro = L.krea_attn_qk_prologue_to_heads
    assert pro(ptr, None, ptr, 1, 8, 128, 1, s, ctypes.byref(r), ctypes.byref(ex()), None) == _lib.ERR_NO_DEVICE
    assert pro(ptr, None, ptr, 1, 8, 128, 2, s, ctypes.byref(r), ctypes.byref(ex()), None) == _lib.ERR_UNSUPPORTED
    assert pro(ptr, None, ptr, 1, 6, 128, 1, s, ctypes.byref(r), ctypes.byref(ex(world=4)),
               None) == _lib.ERR_INVALID_ARG
    p = ctypes.c_void_p()
    h = (ctypes.c_ubyte * _lib.IPC_HANDLE_BYTES)()
    assert L.krea_attn_ipc_alloc(0, ctypes.byref(p), h) == _lib.ERR_INVALID_ARG
    assert L.krea_attn_ipc_alloc(256, ctypes.byref(p), h) == _lib.ERR_NO_DEVICE
    assert L.krea_attn_ipc_open(h, ctypes.byref(p)) == _lib.ERR_NO_DEVICE
    assert L.krea_attn_ipc_free(None) == _lib.ERR_INVALID_ARG
    assert L.krea_attn_ipc_close(None) == _lib.ERR_INVALID_ARG


def test_map_log_lines():
    # KREA_ATTN_LOG prints one line per map built (not for size queries) with the
    # map's tile counts; unset or "0", nothing
    import sys

    prog = ("import diffusion_transformer_attention_bidirectional_b200 as K\n"
            "K.get_map('scanline', 512, 64, 64, window=11)\n"
            "K.get_map('tilemix', 512, 128, 128, pattern='band', percentage=0.5)\n")

    def run(value):
        env = dict(os.environ)
        env.pop("KREA_ATTN_LOG", None)
        if value is not None:
            env["KREA_ATTN_LOG"] = value
        r = subprocess.run([sys.executable, "-c", prog], cwd=ROOT, env=env, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        return [ln for ln in r.stderr.splitlines() if ln.startswith("[krea_attn]")]

    lines = run("1")
    assert len(lines) == 2
    assert "map scanline T=512 grid=64x64" in lines[0] and "36x36 tiles, 484 active" in lines[0]
    assert "map tilemix" in lines[1] and "17424 active" in lines[1] and "7938 int8" in lines[1]
    assert run("0") == [] and run(None) == []
