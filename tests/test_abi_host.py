"""The C ABI on a host without a GPU: the library loads, exports every entry
point that include/ssd.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re
import subprocess

import pytest

import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import build as ssd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("ssd_scan_fwd", "ssd_scan_fwd_complex", "ssd_state_update", "ssd_scan_workspace_size",
              "ssd_last_error", "ssd_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\S+)", out))
    for n in declared_functions():
        assert n in exported, f"{n} declared in ssd.h but not exported"
        assert hasattr(lib, n)


def test_version(lib):
    assert "sm_100a" in ssd.ssd_version()


def test_workspace_size(lib):
    bad = ssd.SSD_WORKSPACE_INVALID
    # the tensor-core kernel (bf16, headdim 64, dstate 128) needs none
    assert ssd.ssd_scan_workspace_size(2, 2048, 64, 64, 1, 128, 256, False, ssd.SSD_BF16) == 0
    # the CUDA-core kernels keep per-chunk decays and states
    assert ssd.ssd_scan_workspace_size(2, 2048, 64, 64, 1, 128, 256, False, ssd.SSD_F32) > 0
    assert ssd.ssd_scan_workspace_size(1, 256, 16, 64, 16, 64, 256, True, ssd.SSD_F32) > 0
    assert ssd.ssd_scan_workspace_size(2, 2048, 64, 64, 3, 128, 256, False, ssd.SSD_BF16) == bad
    assert ssd.ssd_scan_workspace_size(2, 2048, 64, 64, 1, 128, 100, False, ssd.SSD_BF16) == bad
    assert ssd.ssd_scan_workspace_size(-1, 2048, 64, 64, 1, 128, 256, False, ssd.SSD_BF16) == bad


FAKE = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced: validation fails first


def scan_call(lib, **over):
    args = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, init=None, final=None, y=FAKE,
                io=ssd.SSD_BF16, b=1, T=16, H=2, P=64, G=1, N=128, Q=256, ws=FAKE, wsb=1 << 30,
                stream=None)
    args.update(over)
    a = args
    return lib.ssd_scan_fwd(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["init"], a["final"],
                            a["y"], a["io"], a["b"], a["T"], a["H"], a["P"], a["G"], a["N"], a["Q"],
                            a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,status,msg", [
    (dict(x=None), ssd.SSD_ERR_INVALID_ARG, "non-null"),
    (dict(y=None), ssd.SSD_ERR_INVALID_ARG, "non-null"),
    (dict(Q=100), ssd.SSD_ERR_INVALID_ARG, "chunk_size"),
    (dict(G=3), ssd.SSD_ERR_INVALID_ARG, "divide"),
    (dict(H=0), ssd.SSD_ERR_INVALID_ARG, "> 0"),
    (dict(T=-1), ssd.SSD_ERR_INVALID_ARG, ">= 0"),
    (dict(io=7), ssd.SSD_ERR_INVALID_ARG, "io_dtype"),
    (dict(B=ctypes.c_void_p((1 << 20) + 2)), ssd.SSD_ERR_INVALID_ARG, "aligned"),
    (dict(N=512), ssd.SSD_ERR_UNSUPPORTED, "dstate"),
    (dict(ws=None), ssd.SSD_ERR_WORKSPACE, "NULL"),
    (dict(wsb=16), ssd.SSD_ERR_WORKSPACE, "too small"),
])
def test_scan_validation(lib, over, status, msg):
    assert scan_call(lib, **over) == status
    assert msg in ssd.ssd_last_error()


def test_update_validation(lib):
    st = lib.ssd_state_update(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, ssd.SSD_BF16,
                              4, 2, 64, 1, 128, None)
    assert st == ssd.SSD_ERR_INVALID_ARG and "non-null" in ssd.ssd_last_error()
    st = lib.ssd_state_update(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, ssd.SSD_BF16,
                              4, 3, 64, 2, 128, None)
    assert st == ssd.SSD_ERR_INVALID_ARG and "divide" in ssd.ssd_last_error()
    st = lib.ssd_state_update_complex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                      4, 2, 0, 1, 64, None)
    assert st == ssd.SSD_ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ssd.ssd_scan_fwd(x, torch.zeros(1, 8, 2), torch.zeros(2), x.new_zeros(1, 8, 1, 128),
                         x.new_zeros(1, 8, 1, 128))


def test_bwd_workspace_size(lib):
    bad = ssd.SSD_WORKSPACE_INVALID
    assert ssd.ssd_scan_bwd_workspace_size(2, 2048, 64, 64, 1, 128) > 0
    assert lib.ssd_scan_bwd_workspace_size(2, 2048, 64, 65, 1, 128) == bad      # headdim > 64
    assert lib.ssd_scan_bwd_workspace_size(2, 2048, 64, 64, 3, 128) == bad      # groups must divide heads
    assert lib.ssd_scan_bwd_complex_workspace_size(4, 2048, 16, 64, 16, 64) > 0
    assert lib.ssd_scan_bwd_complex_workspace_size(4, 2048, 16, 64, 16, 128) == bad  # complex dstate > 64


def bwd_call(lib, fn="ssd_scan_bwd", **over):
    args = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, init=None, dy=FAKE, dfinal=None,
                dx=FAKE, ddt=FAKE, dA=FAKE, dB=FAKE, dC=FAKE, dD=None, dinit=None,
                b=1, T=16, H=2, P=64, G=1, N=64, ws=FAKE, wsb=1 << 30, stream=None)
    args.update(over)
    a = args
    return getattr(lib, fn)(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["init"], a["dy"], a["dfinal"],
                            a["dx"], a["ddt"], a["dA"], a["dB"], a["dC"], a["dD"], a["dinit"],
                            a["b"], a["T"], a["H"], a["P"], a["G"], a["N"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("fn", ["ssd_scan_bwd", "ssd_scan_bwd_complex"])
@pytest.mark.parametrize("over,status,msg", [
    (dict(x=None), ssd.SSD_ERR_INVALID_ARG, "required"),
    (dict(dy=None), ssd.SSD_ERR_INVALID_ARG, "required"),
    (dict(dA=None), ssd.SSD_ERR_INVALID_ARG, "required"),
    (dict(P=65), ssd.SSD_ERR_UNSUPPORTED, "headdim <= 64"),
    (dict(G=3), ssd.SSD_ERR_INVALID_ARG, "divide"),
    (dict(T=-1), ssd.SSD_ERR_INVALID_ARG, ">= 0"),
    (dict(dB=ctypes.c_void_p((1 << 20) + 4)), ssd.SSD_ERR_INVALID_ARG, "aligned"),
    (dict(ws=None), ssd.SSD_ERR_WORKSPACE, "needed"),
    (dict(wsb=16), ssd.SSD_ERR_WORKSPACE, "needed"),
])
def test_bwd_validation(lib, fn, over, status, msg):
    assert bwd_call(lib, fn, **over) == status
    assert msg in ssd.ssd_last_error()


def test_bwd_dstate_limits(lib):
    assert bwd_call(lib, "ssd_scan_bwd", N=129) == ssd.SSD_ERR_UNSUPPORTED
    assert "dstate <= 128" in ssd.ssd_last_error()
    assert bwd_call(lib, "ssd_scan_bwd_complex", N=65) == ssd.SSD_ERR_UNSUPPORTED
    assert "dstate <= 64" in ssd.ssd_last_error()


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++17")])
def test_header_compiles_as_c_and_cpp(tmp_path, lang, std):
    """include/ssd.h is a C ABI: it must compile, pedantically, as C and as C++,
    with no CUDA include."""
    import subprocess
    src = tmp_path / "use_header.c"
    src.write_text('#include "ssd.h"\n'
                   "int main(void) { return ssd_scan_bwd_workspace_size(1, 1, 1, 1, 1, 1) == 0 "
                   "&& ssd_scan_workspace_size(1, 1, 1, 1, 1, 1, 64, 0, SSD_F32) == 0; }\n")
    cc = "gcc" if lang == "c" else "g++"
    subprocess.check_call([cc, f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                           "-x", lang, "-I", os.path.join(ROOT, "include"), str(src)])


def test_final_state_and_fold_validation(lib):
    def fs_call(**over):
        a = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, init=None, final=FAKE, lam=None, io=ssd.SSD_BF16, b=1, T=256,
                 H=2, P=64, G=1, N=128, Q=256, ws=FAKE, wsb=1 << 30, stream=None)
        a.update(over)
        return lib.ssd_scan_final_state(a["x"], a["dt"], a["A"], a["B"], a["init"], a["final"], a["lam"],
                                        a["io"], a["b"], a["T"], a["H"], a["P"], a["G"], a["N"], a["Q"],
                                        a["ws"], a["wsb"], a["stream"])

    assert fs_call(final=None) == ssd.SSD_ERR_INVALID_ARG and "final_state" in ssd.ssd_last_error()
    assert fs_call(B=None) == ssd.SSD_ERR_INVALID_ARG and "non-null" in ssd.ssd_last_error()
    assert fs_call(lam=ctypes.c_void_p((1 << 20) + 4)) == ssd.SSD_ERR_INVALID_ARG
    assert fs_call(G=3) == ssd.SSD_ERR_INVALID_ARG
    assert fs_call(io=5) == ssd.SSD_ERR_INVALID_ARG
    # y NULL stays an error for the full scan (only the final-state entry point omits it)
    assert scan_call(lib, y=None, final=FAKE) == ssd.SSD_ERR_INVALID_ARG
    fold = lambda n, lam, out: lib.ssd_fold_states(FAKE, lam, n, out, 1, 2, 64, 128, None)
    assert fold(0, FAKE, FAKE) == ssd.SSD_ERR_INVALID_ARG
    assert fold(2, None, FAKE) == ssd.SSD_ERR_INVALID_ARG and "log_decay" in ssd.ssd_last_error()
    assert fold(2, FAKE, None) == ssd.SSD_ERR_INVALID_ARG
