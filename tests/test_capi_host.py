"""The C-ABI library on a machine without a GPU: it loads, exports every
function include/ssm.h declares, and rejects bad arguments before launching
anything (no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

import selective_state_space_24_b200 as ssm
from selective_state_space_24_b200 import build as ssm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE = 0x7F0000000000  # 16-byte aligned stand-in address; never dereferenced here


@pytest.fixture(scope="module")
def lib():
    ssm_build.build()
    return ssm.load()


def _declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        txt = open(os.path.join(ROOT, "include", h)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\([^;{]*\)\s*;", txt, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"ssm_scan_fwd", "bidir_scan_fwd", "ssd_chunk_fwd"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(names) == set(ssm.SIGNATURES), "binding and header disagree"


def test_version_and_status_strings(lib):
    assert lib.ssm_version() >= 100
    for code in range(8):
        assert lib.ssm_status_string(code).decode().startswith(ssm.STATUS[code])


def _dims(B=2, L=8, D=16, N=16, dt=ssm.SSM_F32):
    return ssm.ssm_dims(B, L, D, N, dt)


def _scan(lib, dims, x=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, out=FAKE, ws=None, wsb=0,
          z=None, last=None):
    return lib.ssm_scan_fwd(ctypes.byref(dims) if dims is not None else None, x, delta, None, 1,
                            A, B, C, None, z, 0, out, last, ws, wsb, None)


def test_null_dims_and_pointers(lib):
    assert _scan(lib, None) == 1
    assert _scan(lib, _dims(), x=None) == 1
    assert _scan(lib, _dims(), A=None) == 1
    assert _scan(lib, _dims(), out=None) == 1
    assert _scan(lib, _dims(B=-1)) == 1


def test_shape_dtype_alignment(lib):
    assert _scan(lib, _dims(N=17)) == 2
    assert _scan(lib, _dims(N=0)) == 2
    assert _scan(lib, _dims(dt=7)) == 4
    assert _scan(lib, _dims(D=6)) == 3                       # f32 needs dim % 4 == 0
    assert _scan(lib, _dims(D=12, dt=ssm.SSM_BF16)) == 3     # bf16 needs dim % 8 == 0
    assert _scan(lib, _dims(), x=FAKE + 4) == 3
    assert _scan(lib, _dims(), z=FAKE + 8) == 3


def test_workspace_too_small(lib):
    dims = _dims(B=1, L=4096, D=64, N=16)
    need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
    assert need > 0
    assert _scan(lib, dims, ws=None, wsb=0) == 5
    assert _scan(lib, dims, ws=FAKE, wsb=need - 1) == 5
    assert lib.ssm_scan_workspace_size(None) == 0


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024   # SSM_NOALLOC_SCRATCH_BYTES in include/ssm.h


def test_noalloc_scratch_covers_every_single_direction_plan(lib):
    """ssm_scan_fwd_noalloc refuses problems whose workspace exceeds its
    built-in array.  The segment plan sizes carries to one wave of CTAs, so
    no accepted single-direction shape should reach the limit: sweep batch,
    length, channels, states and dtype through ssm_scan_workspace_size."""
    txt = open(os.path.join(ROOT, "include", "ssm.h")).read()
    m = re.search(r"#define SSM_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", txt)
    assert m and int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == NOALLOC_SCRATCH_BYTES
    worst = 0
    for dt, dstep in ((ssm.SSM_F32, 4), (ssm.SSM_BF16, 8)):
        for B in (1, 2, 3, 7, 64, 1000, 100000):
            for L in (1, 15, 16, 17, 197, 4099, 16384, 1 << 20, 1 << 30):
                for D in (dstep, 3 * dstep, 64, 192, 200, 768, 2048, 8192, 1 << 16):
                    for N in (1, 7, 16):
                        dims = _dims(B=B, L=L, D=D, N=N, dt=dt)
                        need = lib.ssm_scan_workspace_size(ctypes.byref(dims))
                        worst = max(worst, need)
                        assert need <= NOALLOC_SCRATCH_BYTES, (B, L, D, N, dt, need)
    assert worst > 0


def test_bidir_validation(lib):
    dims = _dims()
    good = ssm.ssm_dir_params(None, FAKE, FAKE, FAKE, None, None, None)
    bad = ssm.ssm_dir_params(None, None, FAKE, FAKE, None, None, None)
    mis = ssm.ssm_dir_params(None, FAKE, FAKE + 2, FAKE, None, None, None)
    f = lambda fw, bw: lib.bidir_scan_fwd(ctypes.byref(dims), FAKE, FAKE, 1, fw, bw, FAKE, None,
                                          0, None)
    assert f(ctypes.byref(good), None) == 1
    assert f(ctypes.byref(good), ctypes.byref(bad)) == 1
    assert f(ctypes.byref(mis), ctypes.byref(good)) == 3
    gated = ssm.ssm_dir_params(None, FAKE, FAKE, FAKE, None, FAKE, None)
    assert f(ctypes.byref(gated), ctypes.byref(good)) == 1   # one direction gated only


def test_empty_problems_launch_nothing(lib):
    # zero batch / seqlen with no last_state: valid, nothing to do
    assert _scan(lib, _dims(B=0)) == 0
    assert _scan(lib, _dims(L=0)) == 0
    assert lib.ssm_scan_workspace_size(ctypes.byref(_dims(L=0))) == 0


def test_ssd_validation(lib):
    d = ssm.ssd_dims(1, 128, 2, 64, 128, 64, ssm.SSM_BF16)
    call = lambda dims, x=FAKE: lib.ssd_chunk_fwd(ctypes.byref(dims), x, FAKE, None, 1, FAKE, FAKE,
                                                  FAKE, None, None, FAKE, None, None, 0, None)
    assert call(ssm.ssd_dims(1, 128, 2, 64, 128, 64, ssm.SSM_F32)) == 4
    assert call(ssm.ssd_dims(1, 128, 2, 32, 128, 64, ssm.SSM_BF16)) == 2
    assert call(d, x=None) == 1
    assert call(d, x=FAKE + 2) == 3
    assert call(ssm.ssd_dims(0, 128, 2, 64, 128, 64, ssm.SSM_BF16)) == 0


def test_plan_is_deterministic(lib):
    for dims in (_dims(64, 197, 768, 16), _dims(8, 1024, 768, 16, ssm.SSM_BF16),
                 _dims(4, 16384, 192, 16, ssm.SSM_BF16)):
        a = lib.bidir_scan_workspace_size(ctypes.byref(dims))
        b = lib.bidir_scan_workspace_size(ctypes.byref(dims))
        assert a == b


def test_scan_plan(lib):
    """The launch-plan query: segment count and channels per lane for the
    workloads' sizes, the bounds the plan keeps, and its argument checks."""
    # Vim-Small bidirectional: two threads per channel, one pass
    assert ssm.scan_plan(64, 197, 768, 16, bidirectional=True) == (1, -2)
    # fewer channels on a short sequence: four or two threads per channel, one pass
    assert ssm.scan_plan(1, 196, 384, 16) == (1, -4)                       # Vim-Tiny
    assert ssm.scan_plan(16, 197, 768, 16, bidirectional=True) == (1, -2)
    assert ssm.scan_plan(8, 197, 768, 16, ssm.SSM_BF16) == (1, -4)
    assert ssm.scan_plan(256, 1024, 768, 16) == (1, -2)
    # ... never with N < 16, never for a long sequence with few channels
    assert ssm.scan_plan(1, 196, 384, 8)[1] in (1, 2)
    assert ssm.scan_plan(1, 4096, 384, 16)[1] in (1, 2)
    assert ssm.scan_plan(2, 1024, 768, 16, bidirectional=True)[1] in (1, 2)
    # the long-row bf16 workload has few channels and a long row: one per
    # lane, several segments; the hi-res one splits each channel over four
    # threads in one pass
    seg, cpl = ssm.scan_plan(4, 16384, 192, 16, ssm.SSM_BF16, bidirectional=True)
    assert cpl == 1 and 1 < seg <= (16384 + 15) // 16
    assert ssm.scan_plan(8, 1024, 768, 16, ssm.SSM_BF16, bidirectional=True) == (1, -4)
    # segments never shorter than 16 steps, never more than the steps
    for L in (1, 15, 16, 17, 100):
        seg, _ = ssm.scan_plan(1, L, 32, 16)
        assert 1 <= seg <= max(1, (L + 15) // 16)
    assert ssm.scan_plan(0, 10, 32, 16)[0] == 1      # empty problem
    assert ssm.scan_plan(2, 0, 32, 16)[0] == 1
    # the plan's segment count matches the workspace the scan asks for
    dims = _dims(2, 4096, 64, 16)
    seg, _ = ssm.scan_plan(2, 4096, 64, 16)
    assert seg > 1 and lib.ssm_scan_workspace_size(ctypes.byref(dims)) > 0
    with pytest.raises(ssm.SSMError):
        ssm.scan_plan(1, 10, 32, 17)                 # N > 16
    with pytest.raises(ssm.SSMError):
        ssm.scan_plan(1, 10, 30, 16)                 # D not a multiple of 4
    assert lib.ssm_scan_plan(None, 0, None, None) == 1


def test_s6_mapping_hook(lib):
    """ssm_debug_s6_mapping forces either thread layout (the plan reports
    it), refuses other modes, and mode 0 gives the cost model back."""
    try:
        with ssm.s6_mapping(ssm.MAPPING_SPLIT_STATES):
            assert ssm.scan_plan(64, 197, 768, 16, bidirectional=True) == (1, -4)
            assert ssm.scan_plan(1, 4096, 384, 16) == (1, -4)
            assert ssm.scan_plan(1, 196, 384, 8)[1] in (1, 2)     # N < 16: never
        with ssm.s6_mapping(ssm.MAPPING_WHOLE_CHANNELS):
            assert ssm.scan_plan(1, 196, 384, 16)[1] in (1, 2)
        assert ssm.scan_plan(1, 196, 384, 16) == (1, -4)
        with ssm.s6_mapping(ssm.MAPPING_SPLIT_STATES_2):
            assert ssm.scan_plan(64, 197, 768, 16, bidirectional=True) == (1, -2)
        assert lib.ssm_debug_s6_mapping(4) == 1
        assert lib.ssm_debug_s6_mapping(-1) == 1
    finally:
        lib.ssm_debug_s6_mapping(0)


def test_state_and_step_validation(lib):
    """ssm_scan_fwd_state and ssm_step reject bad arguments before launching."""
    dims = _dims(2, 8, 16, 16)
    # misaligned initial state
    st = lib.ssm_scan_fwd_state(ctypes.byref(dims), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None,
                                0, FAKE + 4, FAKE, None, None, 0, None)
    assert st == 3
    # a step is one time step
    st = lib.ssm_step(ctypes.byref(dims), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, FAKE,
                      FAKE, None)
    assert st == 2
    one = _dims(2, 1, 16, 16)
    assert lib.ssm_step(ctypes.byref(one), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, None,
                        FAKE, None) == 1          # no state
    assert lib.ssm_step(ctypes.byref(one), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, FAKE,
                        FAKE + 8, None) == 3      # misaligned out
    assert lib.ssm_step(None, FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, None) == 1
    empty = _dims(0, 1, 16, 16)
    assert lib.ssm_step(ctypes.byref(empty), None, None, None, 1, None, None, None, None, None, None,
                        None, None) == 0


def test_conv_validation(lib):
    dims = _dims(2, 8, 16, 16)
    bad = ssm.ssm_conv_params(FAKE, None, 5, 1)
    assert lib.ssm_scan_fwd_conv(ctypes.byref(dims), FAKE, ctypes.byref(bad), FAKE, None, 1, FAKE, FAKE,
                                 FAKE, None, None, 0, FAKE, None, None, 0, None) == 2
    nul = ssm.ssm_conv_params(None, None, 3, 1)
    assert lib.ssm_scan_fwd_conv(ctypes.byref(dims), FAKE, ctypes.byref(nul), FAKE, None, 1, FAKE, FAKE,
                                 FAKE, None, None, 0, FAKE, None, None, 0, None) == 1
    assert lib.ssm_scan_fwd_conv(ctypes.byref(dims), FAKE, None, FAKE, None, 1, FAKE, FAKE, FAKE, None,
                                 None, 0, FAKE, None, None, 0, None) == 1
    mis = ssm.ssm_conv_params(FAKE + 4, None, 3, 1)
    assert lib.ssm_scan_fwd_conv(ctypes.byref(dims), FAKE, ctypes.byref(mis), FAKE, None, 1, FAKE, FAKE,
                                 FAKE, None, None, 0, FAKE, None, None, 0, None) == 3


def test_bwd_workspace_and_validation(lib):
    """The backward's workspace holds the states entering every 4-step chunk,
    N padded to 4, 8 or 16 floats per channel; a short or misaligned
    workspace and missing gradient outputs are rejected before any launch."""
    for N in range(1, 17):
        ns = 4 if N <= 4 else 8 if N <= 8 else 16
        dims = _dims(2, 101, 96, N)
        assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims)) == 2 * 26 * 96 * ns * 4
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(_dims(N=17))) == 0
    assert lib.ssm_scan_bwd_workspace_size(None) == 0

    dims = _dims(2, 101, 96, 16)
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims))

    def bwd(ws=FAKE, wsb=need, dA=FAKE, dD=FAKE):
        # x, delta, bias, softplus, A, B, C, D, z, reverse, dout, dx, ddelta, dA, dB, dC, dD, dz, dbias
        return lib.ssm_scan_bwd(ctypes.byref(dims), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, FAKE, None, 0,
                                FAKE, FAKE, FAKE, dA, FAKE, FAKE, dD, None, None, ws, wsb, None)

    assert bwd(wsb=need - 1) == 5          # SSM_ERR_WORKSPACE_TOO_SMALL
    assert bwd(ws=None) == 5
    assert bwd(ws=FAKE + 4) == 3           # SSM_ERR_MISALIGNED
    assert bwd(dA=None) == 1               # SSM_ERR_INVALID_ARG
    assert bwd(dD=None) == 1               # D given without its gradient


def test_bidir_bwd_checks_both_directions_first(lib):
    """bidir_scan_bwd refuses a bad argument of either direction before it
    launches anything: on a machine without a GPU any launch attempt would
    end in SSM_ERR_CUDA (6), so a refusal code proves nothing was started."""
    dims = _dims(2, 33, 64, 16)
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims))
    p = ssm.ssm_dir_params(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None)   # bias, A, B, C, D, z
    good = ssm.ssm_dir_grads(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)

    def call(gf=good, gb=good, ws=FAKE, wsb=need, d=dims):
        return lib.bidir_scan_bwd(ctypes.byref(d), FAKE, FAKE, 1, ctypes.byref(p), ctypes.byref(p), FAKE,
                                  FAKE, FAKE, None if gf is None else ctypes.byref(gf),
                                  None if gb is None else ctypes.byref(gb), ws, wsb, None)

    no_dA = ssm.ssm_dir_grads(None, FAKE, FAKE, FAKE, FAKE, FAKE)
    no_dz = ssm.ssm_dir_grads(FAKE, FAKE, FAKE, FAKE, None, FAKE)
    misaligned = ssm.ssm_dir_grads(FAKE, FAKE + 8, FAKE, FAKE, FAKE, FAKE)
    assert call(gb=no_dA) == 1            # the reversed direction's dA missing
    assert call(gb=no_dz) == 1            # z given without its gradient
    assert call(gb=misaligned) == 3
    assert call(gf=no_dA) == 1
    assert call(gb=None) == 1
    assert call(wsb=need - 16) == 5
    assert call(d=_dims(2, 33, 64, 17)) == 2


def test_binding_signatures_match_the_header():
    """Every function include/ssm.h declares has a ctypes signature in the
    binding with the same number of parameters and, per parameter, the same
    kind: pointer, size_t or integer."""
    txt = open(os.path.join(ROOT, "include", "ssm.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    decls = re.findall(r"SSM_API\s+([\w\s\*]*?)\b(\w+)\s*\(([^;{]*)\)\s*;", txt)
    assert len(decls) == len(_declared_functions())
    ptr_types = (ctypes.c_void_p, ctypes.c_char_p)

    def kind_of_c(decl):
        if "*" in decl:
            return "ptr"
        if re.fullmatch(r"\s*void\s*", decl):
            return "void"
        if re.search(r"\bsize_t\b", decl):
            return "size"
        return "uint" if re.search(r"\bunsigned\b", decl) else "int"

    def kind_of_ctypes(t):
        if t is None:
            return "void"
        if t in ptr_types or isinstance(t, type) and issubclass(t, ctypes._Pointer):
            return "ptr"
        if t is ctypes.c_size_t:
            return "size"
        if t is ctypes.c_uint:
            return "uint"
        assert t in (ctypes.c_int, ctypes.c_int32), t
        return "int"

    for ret, name, args in decls:
        assert name in ssm.SIGNATURES, name
        restype, argtypes = ssm.SIGNATURES[name]
        params = [] if args.strip() in ("", "void") else [a.strip() for a in args.split(",")]
        assert len(params) == len(argtypes), f"{name}: {len(params)} vs {len(argtypes)}"
        for i, (c, t) in enumerate(zip(params, argtypes)):
            assert kind_of_c(c) == kind_of_ctypes(t), f"{name} argument {i}: {c!r} vs {t}"
        assert kind_of_c(ret) == kind_of_ctypes(restype), f"{name} returns {ret!r} vs {restype}"


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes structures have the C structures' field order, offsets and
    sizes (a plain C program compiled against include/ssm.h prints them)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    structs = ["ssm_dims", "ssd_dims", "ssm_dir_params", "ssm_dir_grads", "ssm_conv_params"]
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "ssm.h"', "int main(void) {"]
    for s in structs:
        lines.append(f'printf("{s} size %zu\\n", sizeof({s}));')
        for f, _ in getattr(ssm, s)._fields_:
            lines.append(f'printf("{s} {f} %zu\\n", offsetof({s}, {f}));')
    lines += ["return 0; }"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    c = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n"):
        if line:
            s, f, v = line.split()
            c[(s, f)] = int(v)
    for s in structs:
        cls = getattr(ssm, s)
        assert ctypes.sizeof(cls) == c[(s, "size")], s
        for f, _ in cls._fields_:
            assert getattr(cls, f).offset == c[(s, f)], f"{s}.{f}"


def test_checkpointing_pair_validation(lib):
    """The checkpointing forward / backward pair refuses missing or
    misaligned checkpoint arrays before launching anything (on this machine
    any launch would end in SSM_ERR_CUDA = 6); the checkpoint size is the
    recomputing backward's workspace size."""
    dims = _dims(2, 101, 96, 16)
    assert lib.ssm_scan_ckpt_size(ctypes.byref(dims)) == lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims))
    assert lib.ssm_scan_ckpt_size(ctypes.byref(_dims(L=0))) == 0
    assert lib.ssm_scan_ckpt_size(None) == 0

    def fwd(ck=FAKE):
        return lib.ssm_scan_fwd_ckpt(ctypes.byref(dims), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, 0,
                                     FAKE, None, ck, None, 0, None)

    assert fwd(ck=None) == 1
    assert fwd(ck=FAKE + 8) == 3
    p = ssm.ssm_dir_params(None, FAKE, FAKE, FAKE, None, None, None)
    bfw = lambda cf, cb: lib.bidir_scan_fwd_ckpt(ctypes.byref(dims), FAKE, FAKE, 1, ctypes.byref(p),
                                                 ctypes.byref(p), FAKE, cf, cb, None, 0, None)
    assert bfw(FAKE, None) == 1
    assert bfw(FAKE + 4, FAKE) == 3
    # an empty problem needs no checkpoint array
    e = _dims(2, 0, 96, 16)
    assert lib.ssm_scan_fwd_ckpt(ctypes.byref(e), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, 0, FAKE,
                                 None, None, None, 0, None) == 0

    def bwd(ck=FAKE, dA=FAKE):
        return lib.ssm_scan_bwd_ckpt(ctypes.byref(dims), FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, 0,
                                     FAKE, FAKE, FAKE, dA, FAKE, FAKE, None, None, None, ck, None)

    assert bwd(ck=None) == 1
    assert bwd(ck=FAKE + 4) == 3
    assert bwd(dA=None) == 1
    g = ssm.ssm_dir_grads(FAKE, FAKE, FAKE, None, None, None)
    bbw = lambda cf, cb: lib.bidir_scan_bwd_ckpt(ctypes.byref(dims), FAKE, FAKE, 1, ctypes.byref(p),
                                                 ctypes.byref(p), FAKE, FAKE, FAKE, ctypes.byref(g),
                                                 ctypes.byref(g), cf, cb, None)
    assert bbw(FAKE, None) == 1      # the reversed direction's array missing: refused before any launch
    assert bbw(None, FAKE) == 1


def test_zero_order_hold_validation(lib):
    """ssm_scan_fwd_zoh / bidir_scan_fwd_zoh: N must be 16 and the batch fit
    the grid, refused before anything runs (also for empty problems); other
    arguments as for the dt B scans; an empty problem with N = 16 is a
    no-op."""
    def single(dims, x=FAKE, init=None):
        return lib.ssm_scan_fwd_zoh(ctypes.byref(dims), x, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, 0,
                                    init, FAKE, None, None, 0, None)
    good = ssm.ssm_dir_params(None, FAKE, FAKE, FAKE, None, None, None)
    bidir = lambda dims: lib.bidir_scan_fwd_zoh(ctypes.byref(dims), FAKE, FAKE, 1, ctypes.byref(good),
                                                ctypes.byref(good), FAKE, None, 0, None)
    for d in (_dims(2, 8, 16, 8), _dims(2, 0, 16, 4), _dims(70000, 4, 16, 16)):
        assert single(d) == 2 and bidir(d) == 2
    assert single(_dims(2, 8, 16, 16), x=None) == 1
    assert single(_dims(2, 8, 16, 16), init=FAKE + 4) == 3
    assert lib.ssm_scan_fwd_zoh(None, FAKE, FAKE, None, 1, FAKE, FAKE, FAKE, None, None, 0, None, FAKE, None,
                                None, 0, None) == 1
    assert single(_dims(2, 0, 16, 16)) == 0 and bidir(_dims(0, 8, 16, 16)) == 0
