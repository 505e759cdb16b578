"""Address and undefined-behaviour sanitizer lane for the host code (CPU only).

Two executables, built here with -fsanitize=address,undefined and run without a
GPU (the CPU lane of "perf(BACKEND-ROCM): cooperate across Q8_K activation
blocks", vllm.cpp PR #2472, CI classification comment):

* host_lane_oracle.c + oracle/oracle.c + synth/synth.c: the checker and the
  input generator on small paged problems in every mode;
* host_lane_abi.c + the library's own sources (pad_api.cpp by g++, the .cu files
  by nvcc with the same sm_100a flags as the product build, host side
  instrumented): plans over a grid of shapes, every decode entry point with one
  argument broken at a time, an empty batch.

A fourth executable links the library's host file with a fake of every CUDA
call it makes (host_lane_fake_cuda.cpp): what it hands the kernels and how
injected failures come back, with planted mistakes as its controls.
A third build of the library lane under -fsanitize=thread checks the host code
for data races while several threads plan at once (with a planted race as its
control).  The two never share a binary: the checker and the library stay apart.  The GPU
side has no sanitizer here; its bounds are covered by the kernels' own checks
(error word) and the parity tests.
"""
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import pytest

from paged_kv_attention_partition_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SAN = ["-fsanitize=address", "-fsanitize=undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]
ENV = dict(os.environ,
           ASAN_OPTIONS="detect_leaks=1:halt_on_error=1:abort_on_error=0",
           UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1")


def _cuda_home() -> str:
    return os.path.dirname(os.path.dirname(os.path.realpath(_build.nvcc())))


def _run(cmd, **kw):
    res = subprocess.run(cmd, capture_output=True, text=True, **kw)
    assert res.returncode == 0, " ".join(cmd) + "\n" + res.stdout + res.stderr
    return res


def _assert_clean(res):
    out = res.stdout + res.stderr
    assert res.returncode == 0, out
    for marker in ("runtime error", "AddressSanitizer", "LeakSanitizer", "FAIL "):
        assert marker not in out, out
    assert "clean" in res.stdout


def test_oracle_and_generator_under_sanitizers(tmp_path):
    exe = tmp_path / "lane_oracle"
    _run(["gcc", "-std=c11", "-O1", "-g", *SAN, "-Wall", "-Wextra", "-Werror",
          os.path.join(ROOT, "tests", "host_lane_oracle.c"), os.path.join(ROOT, "oracle", "oracle.c"),
          os.path.join(ROOT, "synth", "synth.c"), "-lm", "-lpthread", "-o", str(exe)])
    _assert_clean(subprocess.run([str(exe)], capture_output=True, text=True, env=ENV, timeout=300))


def test_c_abi_host_code_under_sanitizers(tmp_path):
    objs = _abi_objects(tmp_path, SAN)
    res = subprocess.run([_link(objs, SAN, str(tmp_path / "lane_abi"))], capture_output=True, text=True, env=ENV,
                         timeout=300)
    _assert_clean(res)


def _abi_objects(tmp_path, san, api_src=None):
    """Object files of the library (host side instrumented with `san`) and the
    ABI lane, compiled in parallel; `api_src` replaces pad_api.cpp."""
    cuda = _cuda_home()
    inc = ["-I", _build.INCLUDE, "-I", _build.CSRC]
    jobs, objs = [], []
    for src in _build.SOURCES:
        obj = str(tmp_path / (os.path.splitext(src)[0] + ".o"))
        objs.append(obj)
        path = os.path.join(_build.CSRC, src)
        if src.endswith(".cpp"):
            jobs.append(["g++", "-std=c++17", "-O1", "-g", *san, *inc, "-I", os.path.join(cuda, "include"),
                         "-c", api_src or path, "-o", obj])
        else:
            xc = [a for flag in san for a in ("-Xcompiler", flag)]
            jobs.append([_build.nvcc(), "-std=c++17", "-O1", "-g", *_build.ARCH_FLAGS, *xc, *inc, "-c", path,
                         "-o", obj])
    lane_obj = str(tmp_path / "lane_abi.o")
    objs.append(lane_obj)
    jobs.append(["gcc", "-std=c11", "-O1", "-g", *san, "-Wall", "-Wextra", "-Werror", "-I", _build.INCLUDE,
                 "-c", os.path.join(ROOT, "tests", "host_lane_abi.c"), "-o", lane_obj])
    with ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        for f in [ex.submit(_run, j) for j in jobs]:
            f.result()
    return objs


def _link(objs, san, exe):
    cuda = _cuda_home()
    _run(["g++", *san, *objs, "-L", os.path.join(cuda, "lib64"), "-lcudart_static", "-ldl", "-lrt", "-lpthread",
          "-o", exe])
    return exe


TSAN = ["-fsanitize=thread", "-fno-omit-frame-pointer"]
TSAN_ENV = dict(os.environ, TSAN_OPTIONS="halt_on_error=1")


def test_c_abi_host_code_under_thread_sanitizer(tmp_path):
    """The ABI lane's four threads plan at once, each the first to fill some
    slots of the library's per-device caches: no data race may be reported.
    Negative control: the same lane over a copy of pad_api.cpp whose SM-count
    cache is a plain int array must be reported."""
    objs = _abi_objects(tmp_path, TSAN)
    res = subprocess.run([_link(objs, TSAN, str(tmp_path / "lane_tsan"))], capture_output=True, text=True,
                         env=TSAN_ENV, timeout=300)
    out = res.stdout + res.stderr
    assert res.returncode == 0 and "ThreadSanitizer" not in out and "clean" in res.stdout, out[-3000:]

    src = open(os.path.join(_build.CSRC, "pad_api.cpp")).read()
    for a, b in (("static std::atomic<int> cache[64];", "static int cache[64];"),
                 ("cache[device].load(std::memory_order_relaxed)", "cache[device]"),
                 ("cache[device].store(n, std::memory_order_relaxed);", "cache[device] = n;")):
        assert src.count(a) == 1, a
        src = src.replace(a, b)
    racy = tmp_path / "racy" / "pad_api.cpp"
    racy.parent.mkdir()
    racy.write_text(src)
    obj = str(tmp_path / "pad_api.o")
    _run(["g++", "-std=c++17", "-O1", "-g", *TSAN, "-I", _build.INCLUDE, "-I", _build.CSRC, "-I",
          os.path.join(_cuda_home(), "include"), "-c", str(racy), "-o", obj])
    res = subprocess.run([_link(objs, TSAN, str(tmp_path / "lane_tsan_racy"))], capture_output=True, text=True,
                         env=TSAN_ENV, timeout=300)
    assert res.returncode != 0 and "data race" in res.stderr and "sm_count" in res.stderr, res.stderr[-3000:]


def _fake_lane(tmp_path, api_src, name):
    """The library's host file (or a copy of it) over the fake CUDA runtime of
    host_lane_fake_cuda.cpp, under ASan/UBSan; no CUDA library is linked."""
    exe = str(tmp_path / name)
    _run(["g++", "-std=c++17", "-O1", "-g", *SAN, "-I", _build.INCLUDE, "-I", _build.CSRC, "-I",
          os.path.join(_cuda_home(), "include"), os.path.join(ROOT, "tests", "host_lane_fake_cuda.cpp"), api_src,
          "-lpthread", "-o", exe])
    return exe


def test_c_abi_over_a_fake_runtime(tmp_path):
    """What pad_api.cpp hands the kernels (pointers, strides, plan, scratch, TMA
    maps) and how injected failures come back, with fakes of every CUDA call it
    makes; the missing-encoder case runs in a process of its own."""
    exe = _fake_lane(tmp_path, os.path.join(_build.CSRC, "pad_api.cpp"), "lane_fake")
    for args in ([], ["no-encoder"]):
        _assert_clean(subprocess.run([exe, *args], capture_output=True, text=True, env=ENV, timeout=300))


# Plausible mistakes in the host file, each of which the fake-runtime lane must catch.
PLANTED = {
    "partials swapped": ("pr.p.o_part = base != nullptr ? reinterpret_cast<float *>(base + pr.ws.o_part)",
                         "pr.p.o_part = base != nullptr ? reinterpret_cast<float *>(base + pr.ws.lse_part)"),
    "freed before the stream drained": ("    e = cudaStreamSynchronize(stream);\n"
                                        "    if (e != cudaSuccess) return cuda_fail(e, \"cudaStreamSynchronize\");\n"
                                        "    cudaFree(w.ptr);", "    cudaFree(w.ptr);"),
    "map strides swapped": ("{stride_bytes(2, rowb), (cuuint64_t)rw, stride_bytes(1, bs * rowb),",
                            "{stride_bytes(1, bs * rowb), (cuuint64_t)rw, stride_bytes(2, rowb),"),
    "scratch not cleared": ("  e = cudaMemsetAsync(w.ptr, 0, want, stream);\n"
                            "  if (e != cudaSuccess) return cuda_fail(e, \"cudaMemsetAsync(library scratch)\");\n",
                            ""),
}


def test_fake_runtime_lane_catches_planted_mistakes(tmp_path):
    src = open(os.path.join(_build.CSRC, "pad_api.cpp")).read()
    exes = {}
    for i, (name, (a, b)) in enumerate(PLANTED.items()):
        assert src.count(a) == 1, name
        d = tmp_path / f"m{i}"
        d.mkdir()
        (d / "pad_api.cpp").write_text(src.replace(a, b))
        exes[name] = str(d / "pad_api.cpp")
    with ThreadPoolExecutor(max_workers=len(exes)) as ex:
        built = {n: ex.submit(_fake_lane, tmp_path, p, f"lane_{i}") for i, (n, p) in enumerate(exes.items())}
        built = {n: f.result() for n, f in built.items()}
    for name, exe in built.items():
        res = subprocess.run([exe], capture_output=True, text=True, env=ENV, timeout=300)
        assert res.returncode != 0 and "FAIL" in res.stderr, f"{name}: not caught\n{res.stdout}{res.stderr[-1500:]}"


def test_lane_catches_a_planted_overrun(tmp_path):
    """Negative control: the same lane on a copy of the checker whose score loop
    runs one token past the sequence (a plausible off-by-one) must fail -- the
    last sequence fills its table row, so the extra token reads past the table."""
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    loop = "for (int64_t t = lo; t < L; ++t) {"
    i = src.index(loop)  # the first token loop: the scores
    assert src.index("s[t - lo] = p->scale * acc;", i) < src.index(loop, i + 1)
    bad = tmp_path / "oracle_overrun.c"
    bad.write_text(src[:i] + loop.replace("t < L", "t <= L") + src[i + len(loop):])
    exe = tmp_path / "lane_bad"
    _run(["gcc", "-std=c11", "-O1", "-g", *SAN, os.path.join(ROOT, "tests", "host_lane_oracle.c"), str(bad),
          os.path.join(ROOT, "synth", "synth.c"), "-lm", "-lpthread", "-o", str(exe)])
    res = subprocess.run([str(exe)], capture_output=True, text=True, env=ENV, timeout=300)
    assert res.returncode != 0 and "AddressSanitizer" in res.stderr, res.stdout + res.stderr[-2000:]


@pytest.mark.parametrize("lane", ["host_lane_oracle.c", "host_lane_abi.c"])
def test_lane_sources_do_not_mix_the_checker_and_the_library(lane):
    text = open(os.path.join(ROOT, "tests", lane)).read()
    if lane == "host_lane_abi.c":
        assert "oracle_" not in text and "synth_" not in text
    else:
        assert "pad.h" not in text and "pad_decode" not in text
