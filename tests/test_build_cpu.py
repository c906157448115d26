"""The in-tree build's staleness rule (CPU only): the library is rebuilt when any source,
header or the build script is newer than it, and only then."""
import glob
import os

from hybrid_mamba_ssm_causal_b200 import build as b


def test_library_is_stale_only_when_something_is_newer(tmp_path, monkeypatch):
    lib = tmp_path / "libssd_mixer.so"
    monkeypatch.setattr(b, "LIB", str(lib))
    assert b._stale()                                   # no library yet
    lib.write_bytes(b"\0")
    deps = b.sources() + glob.glob(os.path.join(b.CSRC, "*.cuh")) + glob.glob(os.path.join(b.CSRC, "*.h"))
    deps += glob.glob(os.path.join(b.INCLUDE, "*.h")) + [os.path.abspath(b.__file__)]
    newest = max(os.path.getmtime(p) for p in deps)
    os.utime(lib, (newest + 10, newest + 10))
    assert not b._stale()
    os.utime(lib, (newest - 10, newest - 10))
    assert b._stale()


def test_every_kernel_source_is_compiled():
    names = {os.path.basename(p) for p in b.sources()}
    for n in ("ssd_api.cu", "ssd_prefill_ws.cu", "ssd_prefill_simt.cu", "ssd_decode.cu", "ssd_backward.cu",
              "ssd_state_pass.cu", "ssd_prefill_static.cu", "ssd_profile.cu", "ssd_selftest.cu"):
        assert n in names
    assert b.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
