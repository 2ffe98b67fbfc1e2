"""CPU checks of the C ABI: the library loads, exports every symbol the header declares, and
host-side validation rejects bad arguments before anything reaches a GPU (every call here
fails validation, so no CUDA work is enqueued)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "omq.h")


@pytest.fixture(scope="module")
def omq():
    from post_quantization_lwc_b200 import build
    build.build()
    from post_quantization_lwc_b200 import omq as m
    return m


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:omq_status|const char\*|int|size_t|uint64_t)\s+(omq_\w+)\(",
                                 text, re.M)))


def test_header_declares_the_boundary():
    names = header_functions()
    for required in ("omq_lwc_quant", "omq_let_apply", "omq_fq_linear_fwd", "omq_fq_linear_bwd",
                     "omq_fold_pack"):
        assert required in names


def test_library_exports_every_declared_symbol(omq):
    lib = ctypes.CDLL(omq.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name
    assert sorted(omq.EXPORTS) == header_functions()


def test_status_strings_and_version(omq):
    lib = omq._lib
    for code in range(10):
        assert lib.omq_status_str(code)
    assert lib.omq_status_str(12345) == b"unknown status"
    assert omq.version() >= 10000


def test_workspace_queries(omq):
    M, N, K = 2048, 4096, 4096
    assert omq.fwd_workspace_bytes(M, N, K) >= 4 * (M // 128) * (N // 256)
    b = omq.bwd_workspace_bytes(M, N, K, 128)
    assert b >= 4 * N * K + 4 * M * K          # dW^ and dXq in fp32
    assert omq.step_workspace_bytes(M, N, K, 128) >= b
    assert omq.bwd_workspace_bytes(0, N, K, 128) == 0


FAKE = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


def test_lwc_validation(omq):
    lib = omq._lib
    P = FAKE
    ok = dict(W=P, wdt=1, N=16, K=256, group=128, bits=4, gl=P, bl=P, s=None, W_hat=P, hat=1,
              h=P, z=P, codes=None, rg=P)

    def call(**kw):
        a = {**ok, **kw}
        return lib.omq_lwc_quant(a["W"], a["wdt"], a["N"], a["K"], a["group"], a["bits"], a["gl"],
                                 a["bl"], a["s"], a["W_hat"], a["hat"], a["h"], a["z"], a["codes"],
                                 a["rg"], None)
    assert call(W=None) == 1
    assert call(h=None) == 1
    assert call(wdt=7) == 3
    assert call(bits=9) == 5
    assert call(bits=1) == 5
    assert call(K=250) == 2            # not a multiple of the group
    assert call(group=12) == 2         # group not a multiple of 8
    assert call(N=0) == 2
    assert call(group=32768, K=32768) == 2
    assert call(W=MISALIGNED) == 4
    assert call(s=MISALIGNED) == 4


def test_fold_pack_validation(omq):
    lib = omq._lib
    assert lib.omq_fold_pack(FAKE, 1, 16, 256, 128, 9, FAKE, FAKE, None, FAKE, FAKE, FAKE, None) == 5
    assert lib.omq_fold_pack(FAKE, 1, 16, 256, 128, 4, FAKE, FAKE, None, None, FAKE, FAKE, None) == 1


def test_let_validation(omq):
    lib = omq._lib
    f = lib.omq_let_apply
    assert f(None, 1, 8, 64, None, None, 16, FAKE, 1, None, None, None, None, 1, 0, None, None, None) == 1
    assert f(FAKE, 1, 8, 64, None, None, 5, FAKE, 1, None, None, None, None, 1, 0, None, None, None) == 5
    assert f(FAKE, 1, 8, 60, None, None, 16, FAKE, 1, None, None, None, None, 1, 0, None, None, None) == 2
    assert f(FAKE, 1, 8, 64, None, FAKE, 16, FAKE, 1, None, None, None, None, 1, 8, None, FAKE, None) == 1
    assert f(MISALIGNED, 1, 8, 64, None, None, 16, FAKE, 1, None, None, None, None, 1, 0, None, None, None) == 4


def test_fwd_validation(omq):
    lib = omq._lib
    f = lib.omq_fq_linear_fwd
    # no Y_ref: Y is required and loss / dY must be absent
    assert f(FAKE, FAKE, 1, 64, 64, 64, None, None, None, None, None, None, 0, None) == 1
    assert f(FAKE, FAKE, 1, 64, 64, 64, None, None, FAKE, FAKE, None, None, 0, None) == 1
    # with Y_ref: dY required, workspace required
    assert f(FAKE, FAKE, 1, 64, 64, 64, None, FAKE, None, None, None, None, 0, None) == 1
    assert f(FAKE, FAKE, 1, 64, 64, 64, None, FAKE, None, FAKE, FAKE, None, 0, None) == 6
    assert f(FAKE, FAKE, 1, 64, 60, 64, None, FAKE, None, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert f(FAKE, FAKE, 7, 64, 64, 64, None, FAKE, None, FAKE, FAKE, FAKE, 1 << 20, None) == 3


def test_bwd_validation(omq):
    lib = omq._lib
    a = omq.BwdArgs(M=64, N=64, K=128, group=64, bits=4, abits=16, dt=1, X=FAKE, W=FAKE,
                    gamma_logit=FAKE, beta_logit=FAKE, Xq=FAKE, W_hat=FAKE, h=FAKE, z=FAKE,
                    grp_range=FAKE, dY=FAKE, d_gamma_logit=FAKE, d_beta_logit=FAKE)
    assert lib.omq_fq_linear_bwd(None, FAKE, 1 << 30, None) == 1
    assert lib.omq_fq_linear_bwd(ctypes.byref(a), None, 0, None) == 6
    a.d_s = FAKE   # LET gradients need s and delta
    assert lib.omq_fq_linear_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == 1
    a.d_s = None
    a.bits = 9
    assert lib.omq_fq_linear_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == 5
    a.bits = 4
    a.K = 100
    assert lib.omq_fq_linear_bwd(ctypes.byref(a), FAKE, 1 << 30, None) == 2


def test_adamw_and_step_validation(omq):
    lib = omq._lib
    assert lib.omq_adamw_step(FAKE, FAKE, FAKE, FAKE, 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == 0
    assert lib.omq_adamw_step(FAKE, FAKE, FAKE, FAKE, -1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == 2
    assert lib.omq_adamw_step(FAKE, None, FAKE, FAKE, 8, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == 1
    assert lib.omq_adamw_step(FAKE, FAKE, FAKE, FAKE, 8, 1e-3, 0.9, 0.999, 1e-8, 0.0, 0, None) == 2
    s = omq.StepArgs(M=64, N=64, K=128, group=64, bits=4, abits=16, let=0, dt=1, step=1)
    assert lib.omq_calib_step(ctypes.byref(s), FAKE, 1 << 30, None) == 1


def test_struct_layouts_match_header(omq, tmp_path):
    """The ctypes mirrors have the offsets the C compiler gives the header's structs."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void){"]
    for cname, py in (("omq_bwd_args", omq.BwdArgs), ("omq_step_args", omq.StepArgs)):
        lines.append(f'printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append('printf("omq_range sizeof %zu\\n", sizeof(omq_range));')
    lines.append("return 0;}")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out.splitlines()}
    for cname, py in (("omq_bwd_args", omq.BwdArgs), ("omq_step_args", omq.StepArgs)):
        assert got[(cname, "sizeof")] == ctypes.sizeof(py)
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)
    assert got[("omq_range", "sizeof")] == 16     # the binding stores ranges as int32 [n, 4]


def test_qgemm_validation(omq):
    """omq_qgemm rejects bad arguments before any launch."""
    lib = omq._lib
    P = FAKE
    # float32 activations, 1 bit, K not a multiple of 64, N not a multiple of 8, NULL codes
    assert lib.omq_qgemm(P, 0, 16, 256, P, P, P, 64, 64, 4, None, P, None) == 3
    assert lib.omq_qgemm(P, 2, 16, 256, P, P, P, 64, 64, 1, None, P, None) == 5
    assert lib.omq_qgemm(P, 2, 16, 200, P, P, P, 64, 40, 4, None, P, None) == 2
    assert lib.omq_qgemm(P, 2, 16, 256, P, P, P, 60, 64, 4, None, P, None) == 2
    assert lib.omq_qgemm(P, 2, 16, 256, None, P, P, 64, 64, 4, None, P, None) == 1
    assert lib.omq_qgemm(MISALIGNED, 2, 16, 256, P, P, P, 64, 64, 4, None, P, None) == 4
    # 3-bit decode with float32 activations has no kernel
    assert lib.omq_qgemv(P, 0, 1, 256, P, P, P, 64, 64, 3, P, None) == 8
