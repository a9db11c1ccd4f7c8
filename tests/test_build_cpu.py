"""How the native pieces are built, without a GPU: a library is rebuilt
whenever its sources, flags or compiler change (a content hash, not file
times, decides), and a build that would flush subnormal floats to zero
refuses to compile."""

import glob
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "loop_aware_quantized_b200", "csrc")
NVCC = "/usr/local/cuda/bin/nvcc"


def _nvcc(src, *flags):
    cmd = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), *flags, "-c", src,
           "-o", os.devnull]
    return subprocess.run(cmd, capture_output=True, text=True)


@pytest.mark.parametrize("flag", ["-ftz=true", "--use_fast_math"])
def test_flush_to_zero_build_is_refused(flag):
    src = os.path.join(CSRC, "append.cu")
    ok = _nvcc(src, "-ftz=false")
    assert ok.returncode == 0, ok.stderr[-2000:]
    bad = _nvcc(src, flag)
    assert bad.returncode != 0
    assert "loopkv_build_error_flush_to_zero_is_not_supported" in bad.stderr


def test_every_floating_point_kernel_carries_the_guard():
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        text = open(path).read()
        for name in ("decode_kernel", "append_kernel", "append_res2_kernel", "vq_decode_kernel",
                     "vq_encode_kernel"):
            i = text.find("\n" + name + "(")
            if i < 0:
                continue
            body = text[i: text.index("\n}", i)]
            assert "require_ieee_subnormals();" in body, (os.path.basename(path), name)


@pytest.mark.parametrize("mod", ["loop_aware_quantized_b200.build", "oracle.build", "synth.build"])
def test_stamp_decides_a_rebuild(mod, tmp_path, monkeypatch):
    import importlib
    b = importlib.import_module(mod)
    calls = []
    lib = str(tmp_path / "lib.so")

    def fake_compile(cmd, *a, **k):
        calls.append(cmd)
        out = cmd[cmd.index("-o") + 1]
        with open(out, "wb") as f:
            f.write(b"x")
        return 0

    monkeypatch.setattr(b, "LIB", lib)
    monkeypatch.setattr(b.subprocess, "check_call", fake_compile)
    b.build()
    assert len(calls) == 1 and os.path.exists(lib + ".stamp")
    b.build()
    assert len(calls) == 1                     # same sources, flags, compiler: reused
    os.utime(lib, (1, 1))                      # an old file time changes nothing
    b.build()
    assert len(calls) == 1
    with open(lib + ".stamp", "w") as f:       # a stamp of other sources: rebuilt
        f.write("0" * 64 + "\n")
    b.build()
    assert len(calls) == 2
    os.remove(lib + ".stamp")                  # no stamp: rebuilt
    b.build()
    assert len(calls) == 3
