"""The C ABI on a machine without a GPU: the library loads, exports every symbol that
include/*.h declares, sizes its workspace, and rejects bad arguments before it would
enqueue anything (so no CUDA call is reached in these tests)."""
import ctypes
import glob
import os
import re
import subprocess
import sys

import pytest

from mamba_ssd_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L = _lib.lib()
OK, INV, UNS, WS = _lib.SSD_OK, _lib.SSD_ERR_INVALID_ARG, _lib.SSD_ERR_UNSUPPORTED, _lib.SSD_ERR_WORKSPACE
F32, BF16 = _lib.SSD_DTYPE_F32, _lib.SSD_DTYPE_BF16
A = 0x10000        # a fake, 16-byte aligned device address (never dereferenced here)
MIS = 0x10002      # a misaligned one


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        names |= set(re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", open(h).read()))
    return names


def test_every_declared_symbol_is_exported_and_bound():
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert names == set(_lib.SIGNATURES), "Python signature table out of sync with the header"


def test_status_strings_and_version():
    for s in range(6):
        assert L.ssd_status_string(s)
    assert L.ssd_status_string(99) == b"unknown status"
    assert L.ssd_abi_version() == 5
    assert L.ssd_last_cuda_error() == 0


def _layout(B, Lx, H, P, N, block, transposed):
    up = lambda v: -(-v // 256) * 256
    nb = -(-Lx // block)
    per_tok = up(4 * B * H * nb * block)
    states = up(4 * B * nb * H * P * N)
    hT = up(2 * B * nb * H * P * N) if transposed else 0
    return 256 + 2 * per_tok + states + hT


def _fused_layout(B, Lx, H):
    """Status slot, then the run slots (one [N][P] fp32 state per head of a head pair) and the
    runs' decays: chains = B * H / 2, units = chains * ceil(L / 128), slots = chains + the
    largest grid (min(units, 160))."""
    up = lambda v: -(-v // 256) * 256
    nch = B * (H // 2)
    units = nch * -(-Lx // 128)
    slots = (nch + min(units, 160)) * 2
    return 256 + up(slots * 128 * 64 * 4) + up(slots * 4)


def ws_bytes(B, Lx, H, P, G, N, chunk, tensor_core_shape, fused=False):
    """With the fused kernels selected (SSD_PREFILL_KERNELS=fused), bf16 P=64 N=128 with an even
    number of heads per group and L > 0 needs only their run slots.  Otherwise: the larger of
    the CUDA-core layout (caller's chunk) and, for bf16 P=64 N=128, the block-state tensor-core
    layout (128-token blocks plus a bf16 copy of the carried states)."""
    if fused and tensor_core_shape and Lx > 0 and (H // G) % 2 == 0:
        return _fused_layout(B, Lx, H)
    need = _layout(B, Lx, H, P, N, chunk, False)
    if tensor_core_shape:
        need = max(need, _layout(B, Lx, H, P, N, 128, True))
    return need


@pytest.mark.parametrize("shape", [(1, 4096, 80, 64, 1, 128, 256), (8, 2048, 64, 64, 1, 128, 256),
                                   (2, 300, 4, 64, 2, 16, 64), (1, 1, 4, 64, 1, 32, 128),
                                   (1, 0, 4, 64, 1, 16, 256), (1, 300, 6, 64, 2, 128, 256),
                                   (1, 0, 8, 64, 1, 128, 256)])
def test_prefill_workspace_size(shape):
    B, Lx, H, P, G, N, chunk = shape
    got = L.ssd_chunk_scan_workspace_size(B, Lx, H, P, G, N, chunk, BF16)
    assert got == ws_bytes(B, Lx, H, P, G, N, chunk, P == 64 and N == 128) and got % 256 == 0
    got32 = L.ssd_chunk_scan_workspace_size(B, Lx, H, P, G, N, chunk, F32)
    assert got32 == ws_bytes(B, Lx, H, P, G, N, chunk, False)
    assert L.ssd_chunk_scan_workspace_size(0, Lx, H, P, G, N, chunk, BF16) == 0
    assert L.ssd_chunk_scan_workspace_size(B, Lx, H, 32, G, N, chunk, BF16) == 0   # unsupported P


@pytest.mark.parametrize("shape", [(1, 4096, 80, 64, 1, 128, 256), (8, 2048, 64, 64, 1, 128, 256),
                                   (1, 300, 6, 64, 2, 128, 256), (1, 0, 8, 64, 1, 128, 256)])
def test_prefill_workspace_size_fused(shape):
    # the environment switch is read once per process: query it in a child
    B, Lx, H, P, G, N, chunk = shape
    code = ("import sys; sys.path.insert(0, %r); from mamba_ssd_b200 import _lib; "
            "print(_lib.lib().ssd_chunk_scan_workspace_size(%d, %d, %d, %d, %d, %d, %d, 1))"
            % (ROOT, B, Lx, H, P, G, N, chunk))
    env = dict(os.environ, SSD_PREFILL_KERNELS="fused")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, check=True)
    assert int(out.stdout.strip()) == ws_bytes(B, Lx, H, P, G, N, chunk, True, fused=True)


def prefill(**kw):
    a = dict(x=A, dt=A, A_log=A, Bm=A, Cm=A, D=A, dt_bias=A, dt_min=1e-3, dt_max=0.1, h0=None,
             y=A, h_final=A, B=1, L=64, H=4, P=64, G=1, N=16, chunk=64, dtype=BF16, ws=A,
             ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.ssd_chunk_scan_fwd(a["x"], a["dt"], a["A_log"], a["Bm"], a["Cm"], a["D"],
                                a["dt_bias"], a["dt_min"], a["dt_max"], a["h0"], a["y"],
                                a["h_final"], a["B"], a["L"], a["H"], a["P"], a["G"], a["N"],
                                a["chunk"], a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), INV), (dict(Bm=None), INV), (dict(dt=None), INV), (dict(A_log=None), INV),
    (dict(y=MIS), INV), (dict(Cm=None), INV),  # C is needed whenever y is (y = NULL: state only)
    (dict(x=MIS), INV), (dict(Cm=MIS), INV), (dict(h0=MIS), INV), (dict(D=MIS), INV),
    (dict(B=-1), INV), (dict(L=-3), INV), (dict(H=0), INV), (dict(G=3), INV), (dict(dtype=7), INV),
    (dict(dt_min=0.5, dt_max=0.1), INV), (dict(dt_min=-1.0), INV), (dict(dt_max=float("nan")), INV),
    (dict(P=32), UNS), (dict(N=48), UNS), (dict(N=256), UNS), (dict(chunk=100), UNS),
    (dict(chunk=1024), UNS), (dict(chunk=32), UNS),
    (dict(ws=None), WS), (dict(ws_bytes=1024), WS), (dict(ws=A + 16), WS),
    (dict(B=0), OK),
])
def test_prefill_validation(kw, want):
    assert prefill(**kw) == want


def decode(**kw):
    a = dict(ssm=A, conv=A, xbc=A, dt=A, A_log=A, D=A, dt_bias=None, dt_min=1e-3, dt_max=0.1,
             w=A, b=A, y=A, B=1, H=80, P=64, G=1, N=128, K=4, dtype=BF16, ws=A, ws_bytes=256,
             stream=None)
    a.update(kw)
    return L.ssd_decode_step(a["ssm"], a["conv"], a["xbc"], a["dt"], a["A_log"], a["D"],
                             a["dt_bias"], a["dt_min"], a["dt_max"], a["w"], a["b"], a["y"], a["B"],
                             a["H"], a["P"], a["G"], a["N"], a["K"], a["dtype"], a["ws"],
                             a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(ssm=None), INV), (dict(conv=None), INV), (dict(w=None), INV), (dict(ssm=MIS), INV),
    (dict(H=81, G=2), INV), (dict(G=0), INV), (dict(dtype=2), INV), (dict(dt_min=0.2), INV),
    (dict(P=24), UNS), (dict(N=48), UNS), (dict(N=512), UNS), (dict(K=1), UNS), (dict(K=9), UNS),
    (dict(ws=None), WS), (dict(ws_bytes=0), WS), (dict(B=300), WS),
    (dict(ws_bytes=22527), WS), (dict(B=70000), UNS),
    (dict(B=0), OK),
])
def test_decode_validation(kw, want):
    assert decode(**kw) == want


def test_decode_workspace_size():
    # a 256-byte status slot, then B*(H*P + 2*G*N) floats and B*H float2, each part rounded
    # up to 256 bytes:  (B, H, P, G, N) -> 256 + u + (dt, a)
    assert L.ssd_decode_workspace_size(1, 80, 64, 1, 128) == 256 + 21504 + 768
    assert L.ssd_decode_workspace_size(16, 80, 64, 1, 128) == 256 + 344064 + 10240
    assert L.ssd_decode_workspace_size(3, 2, 16, 1, 16) == 256 + 768 + 256
    assert L.ssd_decode_workspace_size(0, 80, 64, 1, 128) == 0
    assert L.ssd_decode_workspace_size(1, 0, 64, 1, 128) == 0
    assert L.ssd_decode_workspace_size(1, 80, 64, 1, -1) == 0


@pytest.mark.parametrize("args,want", [
    ((A, A, A, A, A, 1, 16, 64, 1, BF16, None), UNS),
    ((A, A, A, A, A, 1, 16, 60, 4, BF16, None), UNS),
    ((A, None, A, A, A, 1, 16, 64, 4, BF16, None), INV),
    ((None, A, A, A, A, 1, 16, 64, 4, BF16, None), INV),
    ((A, A, A, A, A, 0, 16, 64, 4, BF16, None), OK),
    ((None, A, A, None, None, 2, 0, 64, 4, F32, None), OK),
    ((A, A, A, A, A, 1, 65535 * 32 + 1, 64, 4, BF16, None), UNS),
    ((A, A, A, A, A, 65536, 16, 64, 4, BF16, None), UNS),
])
def test_conv_validation(args, want):
    assert L.ssd_causal_conv1d_fwd(*args) == want


@pytest.mark.parametrize("status,limit_us", [(None, 1000), (A + 2, 1000), (A, 0), (A, 1000001)])
def test_selftest_validation(status, limit_us):
    # rejected before any launch, so it runs without a GPU
    assert L.ssd_selftest_wait_timeout(status, limit_us, None) == INV


def norm(**kw):
    a = dict(y=A, z=A, w=A, out=A, T=4096, C=5120, G=1, eps=1e-5, dtype=BF16, stream=None)
    a.update(kw)
    return L.ssd_gated_rmsnorm_fwd(a["y"], a["z"], a["w"], a["out"], a["T"], a["C"], a["G"], a["eps"],
                                   a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(y=None), INV), (dict(z=MIS), INV), (dict(w=None), INV), (dict(out=MIS), INV),
    (dict(T=-1), INV), (dict(C=0), INV), (dict(G=0), INV), (dict(C=5120, G=3), INV),
    (dict(dtype=5), INV), (dict(eps=-1e-3), INV), (dict(eps=float("nan")), INV),
    (dict(eps=float("inf")), INV),
    (dict(C=12), UNS), (dict(C=65536, G=1), UNS), (dict(C=640 * 70000, G=70000), UNS),
    (dict(T=0), OK), (dict(T=0, y=None, z=None, out=None), OK),
])
def test_norm_validation(kw, want):
    # every case is decided before a launch, so it runs without a GPU
    assert norm(**kw) == want


def varlen(cu, **kw):
    a = dict(x=A, dt=A, A_log=A, Bm=A, Cm=A, D=None, dt_bias=None, dt_min=1e-3, dt_max=0.1, h0=None, y=A,
             hf=None, n=len(cu) - 1 if cu is not None else 1, H=80, P=64, G=1, N=128, chunk=256, dtype=BF16,
             ws=A * 256, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    arr = (ctypes.c_int * len(cu))(*cu) if cu is not None else None
    return L.ssd_chunk_scan_varlen_fwd(a["x"], a["dt"], a["A_log"], a["Bm"], a["Cm"], a["D"], a["dt_bias"],
                                       a["dt_min"], a["dt_max"], a["h0"], a["y"], a["hf"],
                                       ctypes.cast(arr, ctypes.c_void_p) if arr is not None else None, a["n"],
                                       a["H"], a["P"], a["G"], a["N"], a["chunk"], a["dtype"], a["ws"],
                                       a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("cu,kw,want", [
    (None, {}, INV), ([0, 5], dict(n=-1), INV), ([1, 5], {}, INV), ([0, 5, 3], {}, INV),
    ([0, 5], dict(x=None), INV), ([0, 5], dict(dt=MIS), INV), ([0, 5], dict(A_log=None), INV),
    ([0, 5], dict(P=32), UNS), ([0, 5], dict(chunk=100), UNS),
    # the per-sequence (CUDA-core) path: f32 dt rows of sequence 1 would start 8 bytes in; the
    # one-pass tensor-core path reads the packed tensors from their bases and takes any start
    ([0, 1, 4], dict(H=2, N=16, dtype=F32), UNS),
    ([0, 5], dict(ws=None), WS), ([0, 5], dict(ws_bytes=256), WS), ([0, 5], dict(ws=A + 16), WS),
    ([0], {}, OK), ([0, 0, 0], dict(x=None, dt=None, Bm=None, Cm=None, y=None, n=0), OK),
])
def test_varlen_validation(cu, kw, want):
    # every case is decided before a launch, so it runs without a GPU
    assert varlen(cu, **kw) == want


def varlen_size(cu, H=80, P=64, G=1, N=128, chunk=256, dtype=BF16):
    arr = (ctypes.c_int * len(cu))(*cu)
    return L.ssd_chunk_scan_varlen_workspace_size(ctypes.cast(arr, ctypes.c_void_p), len(cu) - 1, H, P, G, N, chunk,
                                                  dtype)


def test_varlen_workspace_size():
    # one pass (bf16, P = 64, N = 128): the block-major prefill workspace of every block of the
    # batch, then the table (three int arrays of m + 1 entries, m non-empty sequences, each in
    # a 256-byte slot)
    cu = [0, 100, 100, 400, 4496]  # blocks 1 + 0 + 3 + 32 = 36, three non-empty sequences
    nb, H, P, N = 36, 80, 64, 128
    prefill = 256 + 2 * (4 * H * nb * 128) + 4 * nb * H * P * N + 2 * nb * H * P * N
    assert varlen_size(cu) == prefill + 3 * 256
    assert varlen_size(cu) == L.ssd_chunk_scan_workspace_size(1, nb * 128, H, P, 1, N, 256, BF16) + 3 * 256
    # the per-sequence path: the longest sequence's prefill workspace, shared
    assert varlen_size(cu, dtype=F32) == L.ssd_chunk_scan_workspace_size(1, 4096, H, P, 1, N, 256, F32)
    assert varlen_size([0]) == 0
    assert varlen_size([0, 5, 3]) == 0    # decreasing
    assert varlen_size([2, 5]) == 0       # not starting at 0
    assert varlen_size([0, 5], P=32) == 0
    assert varlen_size([0, 0, 0]) == 256 + 3 * 256  # no blocks: the status slot and the table


def test_header_is_plain_c_and_links(tmp_path):
    # the boundary is a C ABI: the header compiles as C99 and as C++17, and a C program links
    # against the library and calls it (host-only entry points: no GPU needed)
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "mamba_ssd.h"\n#include <stdio.h>\n'
                   "int main(void) {\n"
                   "  size_t ws = ssd_decode_workspace_size(16, 80, 64, 1, 128);\n"
                   "  printf(\"%d %zu %s\\n\", ssd_abi_version(), ws, ssd_status_string(SSD_OK));\n"
                   "  return ws == 256 + 344064 + 10240 ? 0 : 1;\n}\n")
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(_lib.LIB_PATH)
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", f"-I{inc}", str(src)],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", "c++", f"-I{inc}", str(src)]):
        subprocess.run(cmd, check=True)
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c99", f"-I{inc}", str(src), f"-L{libdir}", "-lmamba_ssd",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[0] == str(L.ssd_abi_version())


def conv_prefill(**kw):
    a = dict(xbc=A, w=A, b=None, dt=A, A_log=A, D=A, dt_bias=None, dt_min=1e-3, dt_max=0.1, h0=None,
             y=A, h_final=A, cs=A, B=1, L=64, H=4, P=64, G=1, N=16, K=4, chunk=64, dtype=BF16, ws=A,
             ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.ssd_conv_chunk_scan_fwd(a["xbc"], a["w"], a["b"], a["dt"], a["A_log"], a["D"], a["dt_bias"],
                                     a["dt_min"], a["dt_max"], a["h0"], a["y"], a["h_final"], a["cs"], a["B"],
                                     a["L"], a["H"], a["P"], a["G"], a["N"], a["K"], a["chunk"], a["dtype"],
                                     a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(xbc=None), INV), (dict(w=None), INV), (dict(dt=None), INV), (dict(y=None), INV),
    (dict(A_log=None), INV), (dict(xbc=MIS), INV), (dict(cs=MIS), INV), (dict(K=0), INV),
    (dict(K=1), UNS), (dict(K=9), UNS), (dict(N=12, P=64), UNS), (dict(P=32), UNS), (dict(B=70000), UNS),
    (dict(ws=None), WS), (dict(ws_bytes=4096), WS), (dict(G=3), INV), (dict(B=0), OK),
])
def test_conv_prefill_validation(kw, want):
    assert conv_prefill(**kw) == want


def test_conv_prefill_workspace_size():
    # the prefill's own workspace, then the conv output [B, L, Cc] (256-byte aligned)
    up = lambda v: -(-v // 256) * 256
    for (B, Lx, H, P, G, N, K, chunk, dt) in [(1, 4096, 80, 64, 1, 128, 4, 256, BF16), (2, 300, 4, 64, 2, 16, 4, 64, F32),
                                             (1, 0, 8, 64, 1, 128, 2, 256, BF16)]:
        Cc = H * P + 2 * G * N
        e = 2 if dt == BF16 else 4
        got = L.ssd_conv_chunk_scan_workspace_size(B, Lx, H, P, G, N, K, chunk, dt)
        assert got == L.ssd_chunk_scan_workspace_size(B, Lx, H, P, G, N, chunk, dt) + up(B * Lx * Cc * e)
    assert L.ssd_conv_chunk_scan_workspace_size(1, 64, 4, 64, 1, 16, 9, 64, BF16) == 0   # K out of range
    assert L.ssd_conv_chunk_scan_workspace_size(0, 64, 4, 64, 1, 16, 4, 64, BF16) == 0
