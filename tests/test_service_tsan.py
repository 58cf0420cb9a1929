"""The FFN service's host code under ThreadSanitizer, on the CPU.

- tests/mailbox_stress.cpp: two producer threads and one consumer through 1600 hand-offs of the
  mailbox.
- tests/service_loop_fake_device.cpp: the serving loop and its completer thread against a
  synchronous fake of the CUDA runtime calls they make (copies are memcpy, events complete
  ~50 us after they are recorded) and a stub layer: in-order service, a failing layer call,
  and stop with slots still posted.

The service source is compiled with -fsanitize=thread, so a missing acquire/release on any
hand-off shows up as a data race on the slot buffers."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
SERVICE = os.path.join(ROOT, "ffn_side_expert_b200", "csrc", "service.cu")


def _build_and_run(tmp_path, harness, link_cudart):
    gxx = shutil.which("g++")
    if not gxx or not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")):
        pytest.skip("needs g++ and the CUDA runtime headers")
    exe = tmp_path / os.path.splitext(harness)[0]
    cmd = [gxx, "-std=c++17", "-fsanitize=thread", "-O1", "-g", "-x", "c++", SERVICE,
           "-x", "none", os.path.join(ROOT, "tests", harness),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"), "-o", str(exe)]
    if link_cudart:
        lib = os.path.join(CUDA, "lib64")
        cmd += ["-L", lib, "-lcudart", f"-Wl,-rpath,{lib}"]
    b = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert b.returncode == 0, b.stderr[-2000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert "ThreadSanitizer" not in r.stderr, r.stderr[-4000:]
    assert r.returncode == 0, (r.stdout, r.stderr[-2000:])
    assert " 0 failures" in r.stdout


def test_mailbox_hand_offs_are_race_free(tmp_path):
    _build_and_run(tmp_path, "mailbox_stress.cpp", link_cudart=True)


def test_serving_loop_on_a_fake_device_is_race_free(tmp_path):
    _build_and_run(tmp_path, "service_loop_fake_device.cpp", link_cudart=False)
