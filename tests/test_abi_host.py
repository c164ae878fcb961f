"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before launching
anything (these calls return before any CUDA call is made)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wk():
    from linear_recurrent_lm_wkv7_b200 import build

    build.build()
    import linear_recurrent_lm_wkv7_b200 as wk

    return wk


def test_header_symbols_exported(wk):
    hdr = open(os.path.join(ROOT, "include", "wkv7.h")).read()
    declared = set(re.findall(r"^(?:int|size_t|const char\*)\s+(wkv7_\w+)\s*\(", hdr, flags=re.M))
    assert declared == set(wk.EXPORTS)
    lib = ctypes.CDLL(wk.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(wk):
    for code in wk.STATUS:
        assert wk.wkv7_status_string(code)
    assert wk.wkv7_version() >= 10000


# argument tuple for wkv7_forward: 9 pointers, B, T, H, D, offsets, io, w, stream
def _fwd(ptr=0x1000, B=1, T=8, H=1, D=64, offs=None, io=1, wd=0, **over):
    p = dict(r=ptr, w=ptr + 0x100000, k=ptr + 0x200000, v=ptr + 0x300000, a=ptr + 0x400000, b=ptr + 0x500000,
             s0=None, y=ptr + 0x600000, sT=None)
    p.update(over)
    return (p["r"], p["w"], p["k"], p["v"], p["a"], p["b"], p["s0"], p["y"], p["sT"], B, T, H, D, offs, io, wd, None)


def test_forward_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_forward
    assert call(*_fwd(D=32)) == -2  # head size
    assert call(*_fwd(B=0)) == -1
    assert call(*_fwd(T=-1)) == -1
    assert call(*_fwd(H=0)) == -1
    assert call(*_fwd(io=7)) == -1  # dtype code
    assert call(*_fwd(wd=3)) == -1
    assert call(*_fwd(r=None)) == -1  # null input
    assert call(*_fwd(y=None)) == -1  # null output
    assert call(*_fwd(k=0x1008 + 0x200000)) == -3  # misaligned
    assert call(*_fwd(sT=0x7000008)) == -3
    assert call(*_fwd(y=0x1000)) == -1  # y aliases r
    assert call(*_fwd(sT=0x1000 + 0x600000)) == -1  # sT overlaps y
    # sT overlapping s0 without being the same buffer
    assert call(*_fwd(s0=0x9000000, sT=0x9000000 + 4096)) == -1


def test_decode_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_decode
    base = [0x1000 + i * 0x100000 for i in range(9)]

    def args(**over):
        a = list(base)
        for k_, v_ in over.items():
            a[int(k_[1:])] = v_
        return tuple(a) + (2, 3, 64, 1, 1, None)

    assert call(*(args()[:-4] + (32, 1, 1, None))) == -2
    assert call(*args(p0=None)) == -1
    assert call(*args(p8=None)) == -1
    assert call(*args(p3=0x1004 + 0x300000)) == -3
    assert call(*args(p7=0x1000)) == -1  # y aliases r
    # partial overlap of s_in and s_out
    assert call(*args(p6=0x9000000, p8=0x9000000 + 256)) == -1


def test_oracle_and_library_share_no_code():
    """The oracle neither includes nor loads anything from the CUDA package, and
    the CUDA sources never mention the oracle."""
    osrc = open(os.path.join(ROOT, "oracle", "wkv7_oracle.c")).read()
    assert "#include \"" not in osrc
    opy = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    assert "linear_recurrent_lm_wkv7_b200" not in opy
    csrc = os.path.join(ROOT, "linear_recurrent_lm_wkv7_b200", "csrc")
    for f in os.listdir(csrc):
        assert "oracle" not in open(os.path.join(csrc, f)).read().lower(), f
    for f in ("__init__.py", "_binding.py", "build.py"):
        assert "oracle" not in open(os.path.join(ROOT, "linear_recurrent_lm_wkv7_b200", f)).read(), f


# argument tuple for wkv7_forward_gated: 11 pointers, B, T, H, D, offsets, io, w, stream
def _fwd_gated(ptr=0x1000, B=1, T=8, H=1, D=64, offs=None, io=1, wd=0, **over):
    p = dict(r=ptr, w=ptr + 0x100000, k=ptr + 0x200000, v=ptr + 0x300000, a=ptr + 0x400000, b=ptr + 0x500000,
             s0=None, rk=ptr + 0x700000, g=ptr + 0x800000, z=ptr + 0x600000, sT=None)
    p.update(over)
    return (p["r"], p["w"], p["k"], p["v"], p["a"], p["b"], p["s0"], p["rk"], p["g"], p["z"], p["sT"], B, T, H, D,
            offs, io, wd, None)


def test_forward_gated_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_forward_gated
    assert call(*_fwd_gated(rk=None)) == -1  # r_k is required
    assert call(*_fwd_gated(g=None)) == -1  # so is the gate
    assert call(*_fwd_gated(D=32)) == -2
    assert call(*_fwd_gated(g=0x1008 + 0x800000)) == -3  # misaligned gate
    assert call(*_fwd_gated(rk=0x1004 + 0x700000)) == -3  # misaligned r_k
    assert call(*_fwd_gated(z=0x1000 + 0x800000)) == -1  # z aliases g
    assert call(*_fwd_gated(z=0x1000 + 0x700000)) == -1  # z overlaps r_k
    assert call(*_fwd_gated(z=0x1000)) == -1  # z aliases r


# argument tuple for wkv7_forward_fused: 10 pointers, B, T, H, H_kv, D, offsets, io, w, stream
def _fwd_fused(ptr=0x1000, B=1, T=8, H=4, H_kv=2, D=64, offs=None, io=1, wd=0, **over):
    p = dict(r=ptr, w=ptr + 0x100000, k=ptr + 0x200000, v=ptr + 0x300000, alr=ptr + 0x400000, s0=None, rk=None,
             g=None, out=ptr + 0x600000, sT=None)
    p.update(over)
    return (p["r"], p["w"], p["k"], p["v"], p["alr"], p["s0"], p["rk"], p["g"], p["out"], p["sT"], B, T, H, H_kv,
            D, offs, io, wd, None)


def test_forward_fused_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_forward_fused
    assert call(*_fwd_fused(H_kv=3)) == -1  # H not a multiple of H_kv
    assert call(*_fwd_fused(H_kv=0)) == -1
    assert call(*_fwd_fused(H_kv=8)) == -1  # more kv heads than heads
    assert call(*_fwd_fused(rk=0x1000 + 0x700000)) == -1  # r_k without g
    assert call(*_fwd_fused(g=0x1000 + 0x800000)) == -1  # g without r_k
    assert call(*_fwd_fused(alr=None)) == -1
    assert call(*_fwd_fused(D=32)) == -2
    assert call(*_fwd_fused(k=0x1008 + 0x200000)) == -3  # misaligned
    assert call(*_fwd_fused(out=0x1000 + 0x200000)) == -1  # out aliases k
    # k holds T * H_kv * D bf16 = 2 KB; out starting 1 KB into it overlaps
    assert call(*_fwd_fused(out=0x1000 + 0x200000 + 1024)) == -1
    assert call(*_fwd_fused(sT=0x1000 + 0x300000)) == -1  # sT overlaps v


def test_decode_fused_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_decode_fused

    def args(B=2, H=4, H_kv=2, D=64, **over):
        p = dict(r=0x1000, w=0x101000, k=0x201000, v=0x301000, alr=0x401000, s_in=None, rk=None, g=None,
                 out=0x601000, s_out=0x701000)
        p.update(over)
        return (p["r"], p["w"], p["k"], p["v"], p["alr"], p["s_in"], p["rk"], p["g"], p["out"], p["s_out"], B, H,
                H_kv, D, 1, 1, None)

    assert call(*args(H_kv=3)) == -1
    assert call(*args(rk=0x801000)) == -1  # r_k without g
    assert call(*args(alr=None)) == -1
    assert call(*args(s_out=None)) == -1
    assert call(*args(D=32)) == -2
    assert call(*args(g=0x901008, rk=0x801000)) == -3  # misaligned gate
    assert call(*args(out=0x201000)) == -1  # out aliases k
    assert call(*args(s_out=0x401000)) == -1  # s_out overlaps a_lr



# argument tuple for wkv7_backward: 17 pointers, workspace bytes, B, T, H, D, offsets, io, w, stream
def _bwd(wk, B=1, T=8, H=1, D=64, offs=None, io=1, wd=0, wsb=None, **over):
    names = ("r", "w", "k", "v", "a", "b", "s0", "dy", "dsT", "dr", "dwl", "dk", "dv", "da", "db", "ds0", "ws")
    p = {n: 0x1000 + i * 0x100000 for i, n in enumerate(names)}
    p["s0"] = p["dsT"] = None
    p.update(over)
    if wsb is None:
        wsb = wk.wkv7_backward_workspace_bytes(B, T, H, 64, offs is not None)
    return tuple(p[n] for n in names) + (wsb, B, T, H, D, offs, io, wd, None)


def test_backward_workspace_size(wk):
    # a state is 64 x 64 fp32; C chunk slots per head (C = ceil(T / 64) per sequence
    # dense, ceil(T / 64) + B packed); 3 (C + B) states per head: M, Q and Qf, with
    # the boundary states over Qf, one spare slot of each per sequence
    assert wk.wkv7_backward_workspace_bytes(2, 130, 3, 64, False) == 3 * 3 * (6 + 2) * 16384
    assert wk.wkv7_backward_workspace_bytes(2, 130, 3, 64, True) == 3 * 3 * (5 + 2) * 16384
    assert wk.wkv7_backward_workspace_bytes(1, 21760, 1, 64, False) == 3 * (340 + 1) * 16384
    assert wk.wkv7_backward_workspace_bytes(2, 8192, 3, 64, True) == 3 * 3 * (128 + 2 + 2) * 16384
    assert wk.wkv7_backward_workspace_bytes(2, 130, 3, 32, False) == 0


def test_backward_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_backward
    assert call(*_bwd(wk, D=32)) == -2
    assert call(*_bwd(wk, B=0)) == -1
    assert call(*_bwd(wk, ds0=None)) == -1
    assert call(*_bwd(wk, ws=None)) == -1
    assert call(*_bwd(wk, dy=None)) == -1
    assert call(*_bwd(wk, wsb=1024)) == -1  # workspace too small
    assert call(*_bwd(wk, dk=0x1008 + 0xB00000)) == -3  # misaligned
    assert call(*_bwd(wk, dr=0x1000)) == -1  # dr aliases r
    assert call(*_bwd(wk, dk=0x1000 + 0x900000)) == -1  # dk aliases dr
    assert call(*_bwd(wk, ws=0x1000 + 0x700000)) == -1  # workspace overlaps dy


def test_backward_noalloc_rejects_before_any_cuda_call(wk):
    call = wk._binding.raw_call_backward_noalloc
    ptrs = tuple(0x1000 + i * 0x100000 for i in range(16))
    # B2 T8192 H32 needs (2 x 128 x 32 checkpoints + 2 x 32 x 64 chunk states) x 16 KB = 192 MiB
    assert call(*ptrs, 2, 8192, 32, 64, None, 1, 0, None) == -7
    assert wk.wkv7_status_string(-7)
    assert call(*ptrs, 0, 8, 1, 64, None, 1, 0, None) == -1
    assert call(*ptrs, 1, 8, 1, 32, None, 1, 0, None) == -2
    # a bad dtype code is an invalid argument even when the problem is also too large,
    # as wkv7_backward would report it (its checks come before the scratch limit)
    assert call(*ptrs, 2, 8192, 32, 64, None, 7, 0, None) == -1
    assert call(*ptrs, 2, 8192, 32, 64, None, 1, 5, None) == -1
    bwd_same = wk._binding.raw_call_backward
    assert bwd_same(*ptrs[:16], ptrs[0] + 0x8000000, 1 << 40, 2, 8192, 32, 64, None, 7, 0, None) == -1


# argument tuple for wkv7_forward_long: 10 pointers, workspace bytes, B, T, H, D, io, w, stream
def _fwd_long(wk, B=1, T=130, H=2, D=64, io=1, wd=0, wsb=None, **over):
    names = ("r", "w", "k", "v", "a", "b", "s0", "y", "sT", "ws")
    p = {n: 0x1000 + i * 0x1000000 for i, n in enumerate(names)}
    p["s0"] = p["sT"] = None
    p.update(over)
    if wsb is None:
        wsb = wk.wkv7_forward_long_workspace_bytes(B, T, H, 64)
    return tuple(p[n] for n in names) + (wsb, B, T, H, D, io, wd, None)


def test_forward_long_workspace_size(wk):
    # 16 KB tile + 32 KB fp32 block + 256 B of decay per 64-token chunk and head
    assert wk.wkv7_forward_long_workspace_bytes(2, 130, 3, 64) == 2 * 3 * 3 * 49408
    assert wk.wkv7_forward_long_workspace_bytes(1, 16384, 40, 64) == 256 * 40 * 49408
    assert wk.wkv7_forward_long_workspace_bytes(1, 0, 1, 64) == 0
    assert wk.wkv7_forward_long_workspace_bytes(0, 64, 1, 64) == 0
    assert wk.wkv7_forward_long_workspace_bytes(1, 64, 1, 32) == 0


def test_forward_long_rejects_bad_arguments(wk):
    call = wk._binding.raw_call_forward_long
    assert call(*_fwd_long(wk, io=0)) == -2  # fp32 inputs: use wkv7_forward
    assert call(*_fwd_long(wk, D=32)) == -2
    assert call(*_fwd_long(wk, B=0)) == -1
    assert call(*_fwd_long(wk, io=3)) == -1
    assert call(*_fwd_long(wk, ws=None)) == -1
    assert call(*_fwd_long(wk, y=None)) == -1
    assert call(*_fwd_long(wk, wsb=1024)) == -1  # workspace too small
    assert call(*_fwd_long(wk, ws=0x1008 + 0x9000000)) == -3  # misaligned
    assert call(*_fwd_long(wk, ws=0x1000 + 0x3000000)) == -1  # workspace overlaps v
    assert call(*_fwd_long(wk, y=0x1000 + 0x9000000)) == -1  # y aliases the workspace
    assert call(*_fwd_long(wk, sT=0x1000 + 0x4000000)) == -1  # sT overlaps a
    # token rows and (sequence, chunk, head) slots are numbered in 32 bits
    assert call(*_fwd_long(wk, B=2, T=1 << 30, H=1, wsb=0)) == -2
    assert call(*_fwd_long(wk, B=1 << 11, T=1 << 20, H=1, wsb=0)) == -2
    assert call(*_fwd_long(wk, B=1, T=1 << 24, H=1 << 13, wsb=0)) == -2
    # T + 63 must not wrap in the slot count: 2^25 chunks x 2^7 heads
    assert call(*_fwd_long(wk, B=1, T=(1 << 31) - 1, H=1 << 7, wsb=0)) == -2


def test_c_program_compiles_and_links(wk, tmp_path):
    """The C ABI is usable from plain C: a C99 program that includes the header and
    references every entry point compiles and links against the library (nothing
    is run, so no GPU is needed)."""
    import shutil
    import subprocess

    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_wkv7.c"
    calls = "\n".join(f"    (void)&{name};" for name in sorted(wk.EXPORTS))
    src.write_text('#include "wkv7.h"\n#include <stdio.h>\nint main(void) {\n' + calls +
                   '\n    printf("%s\\n", wkv7_status_string(WKV7_OK));\n    return 0;\n}\n')
    libdir = os.path.dirname(wk.LIB_PATH)
    cuda_lib = "/usr/local/cuda/lib64"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
           str(tmp_path / "use_wkv7"), wk.LIB_PATH, f"-Wl,-rpath-link,{cuda_lib}", f"-Wl,-rpath,{libdir}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_state_map_and_apply_reject_bad_arguments(wk):
    call = wk._binding.raw_call_state_map
    base = 0x10000000
    ins = [base + i * 0x1000000 for i in range(6)]  # r, w_log, k, v, a, b
    M, Q = base + 0x8000000, base + 0x9000000
    ok = lambda **o: [o.get("r", ins[0]), ins[1], ins[2], ins[3], ins[4], ins[5], o.get("M", M), o.get("Q", Q),
                      o.get("B", 2), o.get("T", 100), o.get("H", 3), o.get("D", 64), None, o.get("io", 1), 0, None]
    assert call(*ok(B=0)) == -1
    assert call(*ok(T=-1)) == -1
    assert call(*ok(D=32)) == -2
    assert call(*ok(io=9)) == -1
    assert call(*ok(M=None, Q=None)) == -1  # nothing to compute
    assert call(*ok(r=None)) == -1
    assert call(*ok(M=M + 8)) == -3
    assert call(*ok(Q=M + 4096)) == -1  # M and Q overlap
    assert call(*ok(M=ins[3] + 64)) == -1  # M overlaps v
    app = wk._binding.raw_call_state_apply
    S = base + 0xA000000
    assert app(S, M, Q, S, 0, 64, None) == -1
    assert app(S, M, Q, S, 4, 16, None) == -2
    assert app(S, None, Q, S, 4, 64, None) == -1
    assert app(S, M, Q, None, 4, 64, None) == -1
    assert app(S + 4, M, Q, S + 4, 4, 64, None) == -3
    assert app(S, M, Q, M + 64, 4, 64, None) == -1  # output overlaps M
    assert app(S, M, Q, S + 4096, 4, 64, None) == -1  # output overlaps S_in without being it
