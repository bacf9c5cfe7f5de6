"""C-ABI checks that need no GPU: symbols, sizes and host-side argument validation.

Every call here is refused by a host check before any device work: calls
meant to pass the shape and layout checks give no workspace, and the workspace
check is the last one before the library touches a device.  So the library is
exercised on a machine without a device, and these calls stay on the host on a
machine with one (the addresses passed are never dereferenced).
"""
import ctypes
import os
import re
import subprocess

import pytest

import block_causal_linear_rope_b200 as blin

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "blin.h")

OK, INVALID, SHAPE, DTYPE, ALIGN, WORKSPACE, STATE = 0, -1, -2, -3, -4, -5, -6
FAKE = 1 << 20  # a 16-byte aligned non-NULL address that is never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(blin_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["blin_state_init", "blin_state_free", "blin_prefill", "blin_block_step",
                 "blin_prefill_workspace_size", "blin_last_error", "blin_state_copy_to_host",
                 "blin_state_copy_from_host", "blin_state_tensors", "blin_state_reset"]:
        assert want in names


def test_library_exports_every_declared_symbol():
    for name in declared_functions():
        assert hasattr(blin.lib, name), name


def test_library_exports_nothing_else():
    out = subprocess.run(["nm", "-D", "--defined-only", blin.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {s for s in exported if s.startswith("blin_")}
    assert ours == set(declared_functions())


def geom(T=21, Hg=30, Wg=52, F=3, split=(8, 12, 12), theta=1e4, eps=1e-6):
    return blin._geom(T, Hg, Wg, F, split, theta, eps)


def ws(B, H, d, g):
    return blin.lib.blin_prefill_workspace_size(B, H, d, ctypes.byref(g))


def tc_chunks(L, d):
    """State chunks per block on the tensor-core path: about 5 (d = 32) or 8 (d = 64) tiles of
    128 tokens each, a function of the block's length and d only."""
    nt = -(-L // 128)
    ct = 5 if d == 32 else 8
    return max(1, -(-nt // ct))


def test_workspace_size_formula():
    # 256 B of alignment slack, then, each padded to 256 B: the work counters,
    # the RoPE table, the chunk partials (chunks per block: the larger of the two
    # paths' counts) and the prefix states
    B, H, d = 1, 70, 32
    g = geom()
    E = d * d + d
    nblk = 21 // 3 + 1
    L = 3 * 30 * 52
    cpb = max(tc_chunks(L, d), -(-L // 1024))
    assert cpb == 8
    pad = lambda x: (x + 255) // 256 * 256
    want = (256 + 256 + pad(8 * (21 * 4 + 30 * 6 + 52 * 6 + 1))
            + pad(4 * B * H * nblk * cpb * E) + pad(4 * B * H * nblk * E))
    assert ws(B, H, d, g) == want


@pytest.mark.parametrize("L,d,want", [(4680, 32, 8), (10800, 32, 17), (1560, 64, 2), (48, 32, 1), (640, 32, 1),
                                      (641, 32, 2), (1024, 64, 1), (1025, 64, 2)])
def test_chunk_rule_examples(L, d, want):
    assert tc_chunks(L, d) == want


def test_workspace_size_rejects_bad_shapes():
    assert ws(1, 70, 48, geom()) == 0
    assert ws(1, 70, 32, geom(split=(8, 12, 10))) == 0
    assert ws(1, 70, 32, geom(split=(7, 13, 12))) == 0
    assert ws(0, 70, 32, geom()) == 0
    assert ws(1, 70, 32, geom(F=0)) == 0
    assert ws(1, 70, 32, geom(theta=0.0)) == 0
    assert ws(1, 70, 32, geom(eps=-1.0)) == 0


def prefill_raw(q=FAKE, k=FAKE, v=FAKE, o=FAKE, dt=1, B=1, H=2, d=32, g=None, st=None, w=FAKE, wb=1 << 30):
    g = g or geom(T=4, Hg=4, Wg=4)
    return blin.lib.blin_prefill(q, k, v, o, dt, B, H, d, ctypes.byref(g), st, w, wb, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(o=None), INVALID), (dict(dt=7), DTYPE), (dict(d=48), SHAPE),
    (dict(q=FAKE + 8), ALIGN), (dict(w=None), WORKSPACE), (dict(wb=16), WORKSPACE),
    (dict(w=FAKE + 4), ALIGN), (dict(B=0), INVALID),
    (dict(g=geom(T=4, Hg=4, Wg=4, split=(8, 8, 8))), SHAPE),
    (dict(g=geom(T=4, Hg=0, Wg=4)), INVALID), (dict(g=geom(T=4, Hg=4, Wg=4, F=0)), INVALID),
    (dict(g=geom(T=4, Hg=4, Wg=4, eps=float("nan"))), INVALID),
])
def test_prefill_rejects_bad_arguments_before_launch(kw, code):
    assert prefill_raw(**kw) == code
    assert blin.lib.blin_last_error().decode() != ""


def test_prefill_with_no_frames_is_a_no_op():
    assert prefill_raw(g=geom(T=0, Hg=4, Wg=4), w=None, wb=0) == OK


def test_geom_null_and_state_null():
    assert blin.lib.blin_prefill(FAKE, FAKE, FAKE, FAKE, 1, 1, 2, 32, None, None, FAKE, 1 << 20, None) == INVALID
    assert blin.lib.blin_block_step(FAKE, FAKE, FAKE, FAKE, 1, 1, 2, 32, None, None, 1, None) == INVALID
    g = geom(T=3, Hg=4, Wg=4)
    assert blin.lib.blin_block_step(FAKE, FAKE, FAKE, FAKE, 1, 1, 2, 32, ctypes.byref(g), None, 1, None) == INVALID


def test_block_step_argument_checks():
    def call(**kw):
        g = geom(T=kw.get("frames", 3), Hg=4, Wg=4, F=kw.get("F", 3), split=kw.get("split", (8, 12, 12)))
        return blin.lib.blin_block_step(kw.get("q", FAKE), FAKE, FAKE, FAKE, kw.get("dt", 1), 1, 2, kw.get("d", 32),
                                        ctypes.byref(g), FAKE, kw.get("commit", 1), None)
    assert call(frames=0) == INVALID
    assert call(F=0) == INVALID
    assert call(split=(8, 12, 14)) == SHAPE
    assert call(commit=2) == INVALID
    assert call(dt=5) == DTYPE
    assert call(q=FAKE + 2) == ALIGN


def test_last_path_starts_empty():
    import threading
    seen = []
    t = threading.Thread(target=lambda: seen.append(blin.lib.blin_last_path()))
    t.start()
    t.join()
    assert seen == [0]  # thread-local: a fresh thread has run nothing


def test_state_accessors_reject_null():
    assert blin.lib.blin_state_tensors(None, None, None, None) == INVALID
    assert blin.lib.blin_state_bytes(None) == 0
    assert blin.lib.blin_state_free(None) == OK
    out = ctypes.c_void_p()
    assert blin.lib.blin_state_init(1, 1, 40, None, ctypes.byref(out)) == SHAPE
    assert blin.lib.blin_state_init(0, 1, 32, None, ctypes.byref(out)) == INVALID
    assert blin.lib.blin_state_init(1, 1, 32, None, None) == INVALID


def test_version_string():
    assert b"sm_100a" in blin.lib.blin_version()


def strided_raw(lq=None, lo=None, dt=1, d=32, H=2, B=1):
    g = geom(T=4, Hg=4, Wg=4)
    mk = lambda t: None if t is None else ctypes.byref(blin.Layout(*t))
    # no workspace: a call whose layouts pass stops at the workspace check, the last
    # one before any device work, so these calls never touch a device
    return blin.lib.blin_prefill_strided(FAKE, FAKE, FAKE, FAKE, dt, B, H, d, ctypes.byref(g), mk(lq), mk(lo), None,
                                         None, 0, None)


@pytest.mark.parametrize("lq,lo,B,code", [
    ((96, 32, 64 * 96), None, 1, OK),                 # token-interleaved heads, valid
    ((16, 32 * 64, 2 * 32 * 64), None, 1, SHAPE),     # token stride below d
    ((36, 32, 64 * 36), None, 1, ALIGN),              # 72-byte rows: not a multiple of 16 bytes
    (None, (32, 64 * 32, 0), 2, SHAPE),               # batch stride 0 with B = 2
    (None, (32, 64 * 32, 0), 1, OK),                  # batch stride ignored for B = 1
])
def test_strided_layout_checks(lq, lo, B, code):
    rc = strided_raw(lq=lq, lo=lo, B=B)
    if code == OK:
        # valid layouts pass every shape and layout check
        assert rc == WORKSPACE, blin.lib.blin_last_error().decode()
    else:
        assert rc == code, blin.lib.blin_last_error().decode()


def fp4(data=FAKE, scale=FAKE, gs=1.0):
    return blin.Nvfp4(data, scale, gs)


def prefill_fp4_raw(q=None, k=None, v=None, split=(8, 12, 12)):
    g = geom(T=4, Hg=4, Wg=4, split=split)
    q, k, v = q or fp4(), k or fp4(), v or fp4()
    return blin.lib.blin_prefill_nvfp4(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), FAKE, 1, 2, 32,
                                       ctypes.byref(g), None, None, 0, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=fp4(data=None)), INVALID), (dict(k=fp4(scale=None)), INVALID),
    (dict(v=fp4(data=FAKE + 8)), ALIGN), (dict(q=fp4(scale=FAKE + 4)), ALIGN),
    (dict(k=fp4(gs=0.0)), INVALID), (dict(v=fp4(gs=-1.0)), INVALID),
    (dict(q=fp4(gs=float("inf"))), INVALID), (dict(k=fp4(gs=float("nan"))), INVALID),
    (dict(split=(16, 8, 8)), SHAPE),  # a valid split, but only (8, 12, 12) at d = 32 runs on the tensor cores
])
def test_nvfp4_operand_checks(kw, code):
    assert prefill_fp4_raw(**kw) == code, blin.lib.blin_last_error().decode()
    assert blin.lib.blin_last_error().decode() != ""


def test_nvfp4_null_operand_and_block_step_checks():
    g = geom(T=3, Hg=4, Wg=4)
    a = fp4()
    assert blin.lib.blin_prefill_nvfp4(None, ctypes.byref(a), ctypes.byref(a), FAKE, 1, 2, 32, ctypes.byref(g),
                                       None, None, 0, None) == INVALID
    # valid operands on the tensor-core split stop at the missing workspace
    assert blin.lib.blin_prefill_nvfp4(ctypes.byref(a), ctypes.byref(a), ctypes.byref(a), FAKE, 1, 2, 32,
                                       ctypes.byref(g), None, None, 0, None) == WORKSPACE
    bad = fp4(gs=0.0)
    assert blin.lib.blin_block_step_nvfp4(ctypes.byref(a), ctypes.byref(bad), ctypes.byref(a), FAKE, 1, 2, 32,
                                          ctypes.byref(g), FAKE, 1, None) == INVALID
    # operands pass, then the state is checked: NULL is refused before any launch
    assert blin.lib.blin_block_step_nvfp4(ctypes.byref(a), ctypes.byref(a), ctypes.byref(a), FAKE, 1, 2, 32,
                                          ctypes.byref(g), None, 1, None) == INVALID


@pytest.mark.parametrize("args,code", [
    ((0, 16, 4, 4, 1), INVALID), ((1, 12, 4, 4, 1), SHAPE), ((1, 16, 0, 4, 1), INVALID), ((1, 16, 4, 4, 7), DTYPE),
])
def test_tconv_state_init_checks(args, code):
    out = ctypes.c_void_p()
    assert blin.lib.blin_tconv_state_init(*args, None, ctypes.byref(out)) == code
    assert not out.value
    assert blin.lib.blin_tconv_state_init(1, 16, 4, 4, 1, None, None) == INVALID  # nowhere to put the handle


def test_tconv_state_accessors_reject_null():
    assert blin.lib.blin_tconv_state_free(None) == OK
    assert blin.lib.blin_tconv_state_bytes(None) == 0
    assert blin.lib.blin_tconv_state_frame(None, None, None) == INVALID


def tconv_raw(x=FAKE, taps=FAKE, bias=None, y=FAKE, dt=1, B=1, C=16, g=None, st=None, commit=0):
    g = g if g is not None else geom(T=4, Hg=4, Wg=4)
    return blin.lib.blin_tconv(x, taps, bias, y, dt, B, C, ctypes.byref(g), st, commit, None)


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), INVALID), (dict(taps=None), INVALID), (dict(y=None), INVALID), (dict(dt=9), DTYPE),
    (dict(B=0), INVALID), (dict(C=20), SHAPE), (dict(commit=2), INVALID), (dict(commit=1), INVALID),
    (dict(x=FAKE + 8), ALIGN), (dict(y=FAKE + 2), ALIGN), (dict(taps=FAKE + 2), ALIGN), (dict(bias=FAKE + 1), ALIGN),
    (dict(g=geom(T=-1, Hg=4, Wg=4)), INVALID), (dict(g=geom(T=4, Hg=0, Wg=4)), INVALID),
    (dict(g=geom(T=4, Hg=4, Wg=4, F=0)), INVALID),
])
def test_tconv_rejects_bad_arguments_before_launch(kw, code):
    assert tconv_raw(**kw) == code, blin.lib.blin_last_error().decode()
    assert blin.lib.blin_last_error().decode() != ""


def test_tconv_geom_null_and_empty_call():
    assert blin.lib.blin_tconv(FAKE, FAKE, None, FAKE, 1, 1, 16, None, None, 0, None) == INVALID
    # no frames and no state: nothing to do, nothing launched
    assert tconv_raw(g=geom(T=0, Hg=4, Wg=4)) == OK


@pytest.mark.parametrize("dt,H,T,F,msg", [
    (1, 1 << 22, 512, 1, "work units"),      # tensor-core path: 2^31 (head, chunk) units
    (0, 70000, 1, 1, "65535 heads"),         # CUDA-core path: heads on grid z
    (0, 2, 70000, 1, "65535 heads"),         # CUDA-core path: blocks on grid y (same message)
])
def test_launch_limits_are_refused_before_launch(dt, H, T, F, msg):
    g = geom(T=T, Hg=1, Wg=1, F=F)
    rc = blin.lib.blin_prefill(FAKE, FAKE, FAKE, FAKE, dt, 1, H, 32, ctypes.byref(g), None, None, 0, None)
    assert rc == SHAPE
    assert msg in blin.lib.blin_last_error().decode()


@pytest.mark.parametrize("dt,H,T", [(1, (1 << 22) - 4096, 512), (0, 65535, 1), (0, 2, 65535)])
def test_just_inside_the_launch_limits(dt, H, T):
    # passes the shape checks and stops at the (missing) workspace, before any device work
    g = geom(T=T, Hg=1, Wg=1, F=1)
    rc = blin.lib.blin_prefill(FAKE, FAKE, FAKE, FAKE, dt, 1, H, 32, ctypes.byref(g), None, None, 0, None)
    assert rc == WORKSPACE, blin.lib.blin_last_error().decode()


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "blin.h"

int main(void) {
    blin_geom g;
    memset(&g, 0, sizeof g);
    g.T = 21; g.Hgt = 45; g.Wid = 80; g.block_frames = 3;
    g.rope_split[0] = 8; g.rope_split[1] = 12; g.rope_split[2] = 12;
    g.theta = 10000.0f; g.eps = 1e-6f;
    size_t ws = blin_prefill_workspace_size(1, 70, 32, &g);
    blin_status rc = blin_prefill(NULL, NULL, NULL, NULL, BLIN_BF16, 1, 70, 32, &g, NULL, NULL, 0, NULL);
    printf("%s|%zu|%d|%s\n", blin_version(), ws, (int)rc, blin_last_error());
    return 0;
}
"""


def test_plain_c_client_builds_links_and_calls(tmp_path):
    """The boundary is usable from C99 alone: header, shared library, no Python or torch types."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = str(tmp_path / "client")
    pkg = os.path.dirname(blin.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", exe, "-L", pkg, "-lblin", "-Wl,-rpath," + pkg])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120, check=True).stdout.strip()
    version, ws_c, rc, msg = out.split("|", 3)
    assert version == blin.lib.blin_version().decode()
    assert int(ws_c) == ws(1, 70, 32, geom(T=21, Hg=45, Wg=80))
    assert int(rc) == INVALID and msg
    # and the header is valid C++ as well
    subprocess.check_call(["g++", "-std=c++11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-x",
                           "c++", HEADER])


# --------------------------------------------------------------------------- binding-side checks of caller buffers
def test_binding_checks_a_caller_given_output():
    import torch
    cpu = torch.device("cpu")
    ok = torch.empty(2, 3, 64, 32, dtype=torch.bfloat16)
    blin._check_out(ok, (2, 3, 64, 32), torch.bfloat16, cpu)
    blin._check_out(torch.empty(2, 64, 3, 32, dtype=torch.bfloat16).permute(0, 2, 1, 3), (2, 3, 64, 32),
                    torch.bfloat16, cpu)  # a strided view is fine where layouts are taken
    for bad in (torch.empty(2, 3, 63, 32, dtype=torch.bfloat16),   # too few rows: the kernels would write past it
                torch.empty(2, 3, 64, 32, dtype=torch.float32),    # wrong dtype
                torch.empty(2, 3, 32, 64, dtype=torch.bfloat16).transpose(2, 3),  # d not contiguous
                "not a tensor"):
        with pytest.raises(ValueError):
            blin._check_out(bad, (2, 3, 64, 32), torch.bfloat16, cpu)
    with pytest.raises(ValueError):  # entry points without layouts want a contiguous output
        blin._check_out(torch.empty(2, 64, 3, 32, dtype=torch.bfloat16).permute(0, 2, 1, 3), (2, 3, 64, 32),
                        torch.bfloat16, cpu, contiguous=True)
    with pytest.raises(ValueError):  # another device
        blin._check_out(torch.empty(2, 3, 64, 32, dtype=torch.bfloat16, device="meta"), (2, 3, 64, 32),
                        torch.bfloat16, cpu)


def test_binding_passes_workspace_bytes_not_elements():
    import torch
    cpu = torch.device("cpu")
    ws, ptr, nbytes = blin._workspace_arg(None, 1000, cpu)
    assert nbytes == 1000 and ptr.value == ws.data_ptr()
    ws, _, nbytes = blin._workspace_arg(torch.empty(300, dtype=torch.float32), 1000, cpu)
    assert nbytes == 1200
    with pytest.raises(ValueError):
        blin._workspace_arg(torch.empty(600, dtype=torch.uint8)[::2], 100, cpu)  # not contiguous
    with pytest.raises(ValueError):
        blin._workspace_arg(torch.empty(600, dtype=torch.uint8, device="meta"), 100, cpu)  # another device


def test_binding_refuses_an_output_over_an_input():
    import torch
    buf = torch.empty(2, 3, 64, 32)
    q = buf[:1]
    blin._check_no_overlap(buf[1:], q)                      # disjoint halves of one buffer
    for bad in (buf[:1], buf[0:2].reshape(2, 3, 64, 32)[:1]):
        with pytest.raises(ValueError):
            blin._check_no_overlap(bad, q)
    with pytest.raises(ValueError):
        blin._check_no_overlap(buf.view(-1)[16:].view(-1)[: 64 * 32].view(1, 1, 64, 32), q)  # shifted, overlapping
    fused = torch.empty(2, 64, 4, 3, 32)                    # [B, N, 4, H, d]: q, k, v and o interleaved
    views = [fused[:, :, i].permute(0, 2, 1, 3) for i in range(4)]
    blin._check_no_overlap(views[3], *views[:3])            # interleaved, no shared element: accepted
