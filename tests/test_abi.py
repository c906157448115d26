"""The C ABI loads, exports every declared symbol, and refuses bad arguments before any
launch (CPU only: every case here fails validation, so nothing reaches a GPU)."""
import ctypes
import glob
import os
import re

import pytest

from hybrid_mamba_ssm_causal_b200 import build as build_mod
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return sm.load_library()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"SSD_API\s+[\w\s\*]+?\b(\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("ssd_mixer_prefill", "ssd_mixer_decode_step", "ssd_mixer_prefill_workspace_size",
              "ssd_mixer_workspace_status", "ssd_status_string", "ssd_mixer_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), f"missing export {n}"


def test_status_strings(lib):
    for s in range(7):
        assert lib.ssd_status_string(s)
    assert lib.ssd_mixer_version() >= 100


def _dims(**kw):
    base = dict(batch=2, seqlen=64, nheads=4, headdim=16, ngroups=2, dstate=16, chunk=64, act="bf16")
    base.update(kw)
    return sm.Dims(**base)


FAKE = 1 << 40  # a 256-byte-aligned address that is never dereferenced


def call_prefill(lib, d, ptr=FAKE, ws_bytes=1 << 30, x_ld=None, chunk_ws=None):
    cd = d.c()
    HP, GN = d.d_inner, d.ngroups * d.dstate
    P = ctypes.c_void_p
    return lib.ssd_mixer_prefill(ctypes.byref(cd), ptr, x_ld or HP, FAKE, HP, FAKE, GN, FAKE, GN,
                                 FAKE, d.nheads, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                 FAKE, HP, FAKE, FAKE, FAKE, ws_bytes, None)


@pytest.mark.parametrize("bad,status", [
    (dict(dconv=3), sm.SSD_ERR_UNSUPPORTED),
    (dict(chunk=100), sm.SSD_ERR_UNSUPPORTED),
    (dict(chunk=8), sm.SSD_ERR_UNSUPPORTED),
    (dict(headdim=24), sm.SSD_ERR_UNSUPPORTED),
    (dict(dstate=256), sm.SSD_ERR_UNSUPPORTED),
    (dict(ngroups=3), sm.SSD_ERR_INVALID_ARG),
    (dict(eps=0.0), sm.SSD_ERR_INVALID_ARG),
    (dict(batch=-1), sm.SSD_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_dims(lib, bad, status):
    assert call_prefill(lib, _dims(**bad)) == status
    assert lib.ssd_mixer_prefill_workspace_size(ctypes.byref(_dims(**bad).c())) == 0


def test_prefill_rejects_misaligned_rows(lib):
    assert call_prefill(lib, _dims(), ptr=FAKE + 2) == sm.SSD_ERR_UNSUPPORTED
    assert call_prefill(lib, _dims(), x_ld=64 + 1) == sm.SSD_ERR_UNSUPPORTED


def test_prefill_rejects_small_workspace(lib):
    d = _dims()
    need = lib.ssd_mixer_prefill_workspace_size(ctypes.byref(d.c()))
    assert need > 0
    assert call_prefill(lib, d, ws_bytes=need - 1) == sm.SSD_ERR_INVALID_ARG


def test_decode_rejects_seqlen_not_one(lib):
    d = _dims(seqlen=2)
    cd = d.c()
    HP, GN = d.d_inner, d.ngroups * d.dstate
    st = lib.ssd_mixer_decode_step(ctypes.byref(cd), FAKE, HP, FAKE, HP, FAKE, GN, FAKE, GN, FAKE,
                                   d.nheads, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                   FAKE, HP, None)
    assert st == sm.SSD_ERR_INVALID_ARG


def test_workspace_size_grows_with_tokens(lib):
    a = lib.ssd_mixer_prefill_workspace_size(ctypes.byref(_dims(seqlen=64).c()))
    b = lib.ssd_mixer_prefill_workspace_size(ctypes.byref(_dims(seqlen=640).c()))
    assert b > 5 * a


def call_varlen(lib, d, cu=FAKE, ws_bytes=1 << 30, ssm=FAKE):
    cd = d.c()
    HP, GN = d.d_inner, d.ngroups * d.dstate
    return lib.ssd_mixer_prefill_varlen(ctypes.byref(cd), cu, None, None, FAKE, HP, FAKE, HP, FAKE, GN, FAKE, GN,
                                        FAKE, d.nheads, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ssm, FAKE,
                                        FAKE, HP, FAKE, ws_bytes, None)


def test_varlen_runs_the_tensor_core_shapes_only(lib):
    tc = _dims(batch=3, seqlen=500, nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128)
    assert lib.ssd_mixer_prefill_varlen_workspace_size(ctypes.byref(tc.c())) >= 256
    for bad in (dict(act="f32"), dict(headdim=32), dict(nheads=6, ngroups=2)):
        d = _dims(**{**dict(batch=3, seqlen=500, nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128), **bad})
        assert lib.ssd_mixer_prefill_varlen_workspace_size(ctypes.byref(d.c())) == 0
        assert call_varlen(lib, d) == sm.SSD_ERR_UNSUPPORTED


def test_varlen_rejects_missing_pointers_and_small_workspace(lib):
    d = _dims(batch=3, seqlen=500, nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128)
    assert call_varlen(lib, d, cu=None) == sm.SSD_ERR_INVALID_ARG
    assert call_varlen(lib, d, ssm=None) == sm.SSD_ERR_INVALID_ARG
    assert call_varlen(lib, d, ws_bytes=16) == sm.SSD_ERR_INVALID_ARG
    assert call_varlen(lib, d, cu=FAKE + 2) == sm.SSD_ERR_UNSUPPORTED   # cu_seqlens not 4-byte aligned


def call_backward(lib, d, ptr=FAKE, ws_bytes=1 << 34, dA=FAKE, dy_ld=None):
    cd = d.c()
    HP, GN, H = d.d_inner, d.ngroups * d.dstate, d.nheads
    rows = [ptr, HP, ptr, HP, ptr, GN, ptr, GN, ptr, H]
    grads = [FAKE, HP, FAKE, HP, FAKE, GN, FAKE, GN, FAKE, H]
    return lib.ssd_mixer_backward(ctypes.byref(cd), *rows, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                  FAKE, HP if dy_ld is None else dy_ld, None, None, *grads,
                                  dA, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, ws_bytes, None)


def test_backward_shapes_and_workspace_size(lib):
    ok = _dims(nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128, seqlen=300)
    need = lib.ssd_mixer_backward_workspace_size(ctypes.byref(ok.c()))
    # at least the gradient partial sums and the state entering every 64-token chunk
    assert need >= 4 * (2 * ok.batch * 300 * 8 * 4 * 128 + ok.batch * 5 * 8 * 64 * 128)
    for bad in (dict(headdim=128), dict(dconv=3), dict(nheads=3, ngroups=2)):
        d = _dims(**{**dict(nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128), **bad})
        assert lib.ssd_mixer_backward_workspace_size(ctypes.byref(d.c())) == 0
        assert call_backward(lib, d) in (sm.SSD_ERR_UNSUPPORTED, sm.SSD_ERR_INVALID_ARG)


def test_backward_rejects_bad_arguments(lib):
    d = _dims(nheads=8, headdim=64, ngroups=2, dstate=128, chunk=128, seqlen=300)
    need = lib.ssd_mixer_backward_workspace_size(ctypes.byref(d.c()))
    assert call_backward(lib, d, ws_bytes=need - 1) == sm.SSD_ERR_INVALID_ARG
    assert call_backward(lib, d, dA=None) == sm.SSD_ERR_INVALID_ARG
    assert call_backward(lib, d, ptr=None) == sm.SSD_ERR_INVALID_ARG
    assert call_backward(lib, d, ptr=FAKE + 2) == sm.SSD_ERR_UNSUPPORTED     # rows not 16-byte aligned
    assert call_backward(lib, d, dy_ld=d.d_inner - 1) == sm.SSD_ERR_UNSUPPORTED
    assert call_backward(lib, _dims(seqlen=65535 * 32 + 1)) == sm.SSD_ERR_UNSUPPORTED


def test_selftest_wait_rejects_bad_arguments(lib):
    assert lib.ssd_mixer_selftest_wait(None, 1000, 0, None) == sm.SSD_ERR_INVALID_ARG
    assert lib.ssd_mixer_selftest_wait(FAKE + 16, 1000, 0, None) == sm.SSD_ERR_INVALID_ARG
    assert lib.ssd_mixer_selftest_wait(FAKE, -1, 0, None) == sm.SSD_ERR_INVALID_ARG
    assert lib.ssd_mixer_selftest_wait(FAKE, 4000000001, 0, None) == sm.SSD_ERR_INVALID_ARG


def test_profile_accounting_without_launches(lib):
    import ctypes as C
    names, ms, cnt = (C.c_char_p * 8)(), (C.c_double * 8)(), (C.c_int * 8)()
    before = lib.ssd_mixer_launch_count()
    lib.ssd_mixer_profile_enable(1)
    assert lib.ssd_mixer_profile_read(names, ms, cnt, 8) == 0     # nothing recorded
    call_backward(lib, _dims(headdim=128))                         # refused before any launch
    assert lib.ssd_mixer_profile_read(names, ms, cnt, 8) == 0
    lib.ssd_mixer_profile_enable(0)
    assert lib.ssd_mixer_launch_count() == before


def test_header_is_plain_c_and_links(tmp_path):
    """A C99 translation unit that takes the address of every declared entry point compiles
    against include/ssd_mixer.h without warnings and links against the library."""
    import subprocess
    names = declared_symbols()
    src = tmp_path / "use_abi.c"
    body = "\n".join(f"    (void)&{n};" for n in names)
    src.write_text('#include "ssd_mixer.h"\nint main(void)\n{\n' + body + "\n    return 0;\n}\n")
    build_mod.build()
    lib_dir = os.path.dirname(build_mod.LIB)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(tmp_path / "use_abi"), "-L", lib_dir, "-lssd_mixer",
           "-Wl,--unresolved-symbols=ignore-in-shared-libs"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_prefill_path_query(lib):
    # bf16, P = 64, N = 128 and 2 or a multiple of 4 heads per group: the tensor-core kernel
    assert sm.ssd_mixer_prefill_path(_dims(headdim=64, dstate=128, nheads=8, ngroups=2)) == sm.SSD_PATH_TENSOR_CORES
    assert sm.ssd_mixer_prefill_path(_dims(headdim=64, dstate=128, nheads=4, ngroups=2)) == sm.SSD_PATH_TENSOR_CORES
    # fp32, other head dims, 3 heads per group: the CUDA-core kernels
    assert sm.ssd_mixer_prefill_path(_dims(act="f32", headdim=64, dstate=128)) == sm.SSD_PATH_CUDA_CORES
    assert sm.ssd_mixer_prefill_path(_dims(headdim=32, dstate=128)) == sm.SSD_PATH_CUDA_CORES
    assert sm.ssd_mixer_prefill_path(_dims(headdim=64, dstate=128, nheads=6, ngroups=2)) == sm.SSD_PATH_CUDA_CORES
    assert sm.ssd_mixer_prefill_path(_dims(dconv=3)) == sm.SSD_PATH_NONE


def test_stage_offsets_follow_the_workspace_layout(lib):
    d = _dims(act="f32", batch=2, seqlen=100, nheads=4, headdim=16, ngroups=2, dstate=16, chunk=64)
    off = sm.ssd_mixer_prefill_stage_offsets(d)
    b, L, H, HP, Cc = 2, 100, 4, 64, 64 + 2 * 32
    a256 = lambda v: (v + 255) // 256 * 256
    assert off["xbc_act"] % 256 == 0 and off["xbc_act"] >= 256
    assert off["delta"] >= a256(off["xbc_act"] + b * L * Cc * 4)
    assert off["y_pre"] + b * L * HP * 4 <= sm.ssd_mixer_prefill_workspace_size(d)
    with pytest.raises(sm.SsdError):
        sm.ssd_mixer_prefill_stage_offsets(_dims(headdim=64, dstate=128, nheads=8, ngroups=2))


def test_layer_and_projection_refuse_unsupported_arguments(lib):
    d = _dims(headdim=64, dstate=128, nheads=8, ngroups=2, seqlen=100)
    assert sm.ssd_mixer_layer_workspace_size(d, 256) > sm.ssd_mixer_prefill_workspace_size(d)
    assert sm.ssd_mixer_layer_workspace_size(d, 250) == 0                 # d_model not a multiple of 8
    assert sm.ssd_mixer_layer_workspace_size(_dims(act="f32", headdim=64, dstate=128), 256) == 0
    # K not a multiple of 8, misaligned workspace: refused before any launch
    assert lib.ssd_mixer_projection(4, 8, 12, FAKE, 16, FAKE, 16, FAKE, 8, FAKE, None) == sm.SSD_ERR_UNSUPPORTED
    assert lib.ssd_mixer_projection(4, 8, 16, FAKE, 16, FAKE, 16, FAKE, 8, FAKE + 8, None) == sm.SSD_ERR_INVALID_ARG
    assert lib.ssd_mixer_projection(0, 8, 16, None, 16, None, 16, None, 8, FAKE, None) == sm.SSD_OK


def _tc(b, L, H, G):
    return _dims(batch=b, seqlen=L, nheads=H, ngroups=G, headdim=64, dstate=128)


def test_prefill_plan_query(lib):
    """The main kernel's launch plan (host logic, nothing launched): whole rows in one launch
    unless rows of a group wider than a cluster outnumber the SMs; then pieces over a series of
    launches in which every piece's predecessor ran in an earlier launch."""
    if os.environ.get("SSD_MIXER_PREFILL_PIECES"):
        pytest.skip("piece count fixed by the environment")
    plan = lambda *a: sm.ssd_mixer_prefill_plan(_tc(*a), sms=148)
    # long_bf16 call: 256 rows of 128 blocks -> 4 pieces of 32, 7 launches (224 block-times, not 256)
    assert plan(1, 16384, 256, 8) == dict(launches=7, pieces=4, piece_blocks=32, ctas_per_launch=148)
    # mid_bf16: 512 rows of 32 blocks -> 2 pieces of 16, 7 launches (112, not 128)
    assert plan(8, 4096, 64, 8) == dict(launches=7, pieces=2, piece_blocks=16, ctas_per_launch=148)
    # small_bf16: groups of 4 heads held by clusters of 4 -> one launch of whole rows
    assert plan(2, 2048, 32, 8) == dict(launches=1, pieces=1, piece_blocks=16, ctas_per_launch=64)
    # fewer rows than SMs, and 256 short rows that pieces would not help: one launch
    assert plan(1, 16384, 64, 8) == dict(launches=1, pieces=1, piece_blocks=128, ctas_per_launch=64)
    assert plan(2, 300, 128, 16) == dict(launches=1, pieces=1, piece_blocks=3, ctas_per_launch=256)
    assert plan(0, 300, 128, 16)["launches"] == 0 and plan(2, 0, 128, 16)["launches"] == 0
    # invariants over a sweep, checked by replaying the queue of pieces launch by launch
    for b in (1, 2, 3, 5):
        for H, G in ((64, 8), (128, 16), (256, 8), (96, 12)):
            for L in (1, 129, 1000, 4096, 16384):
                p = plan(b, L, H, G)
                rows, nblk = b * H, -(-L // 128)
                if p["pieces"] == 1:
                    assert p["launches"] == 1 and p["ctas_per_launch"] == rows
                    continue
                per, pb, n = p["ctas_per_launch"], p["piece_blocks"], p["pieces"]
                assert rows >= 148 and per <= rows
                assert (n - 1) * pb < nblk <= n * pb
                assert p["launches"] == -(-rows * n // per)
                for pos in range(rows, rows * n):              # a piece after the first of its row
                    assert (pos - rows) // per < pos // per    # its predecessor ran in an earlier launch
    # other SM counts plan for their own waves
    assert sm.ssd_mixer_prefill_plan(_tc(1, 16384, 256, 8), sms=256)["pieces"] == 1
    # only the tensor-core path has a plan
    with pytest.raises(sm.SsdError):
        sm.ssd_mixer_prefill_plan(_dims(act="f32", headdim=64, dstate=128), sms=148)
    with pytest.raises(sm.SsdError):
        sm.ssd_mixer_prefill_plan(_tc(1, 16384, 256, 8), sms=-1)
