"""The per-device record behind every kernel-attribute call of libzha.so
(cudaFuncSetAttribute acts on the current device only, so each device is set
on its own): a fake launch sequence over two devices, compiled with g++ and
run on the CPU."""
import os
import subprocess


def test_per_device_attribute_record(tmp_path):
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "host", "attr_once.cpp")
    exe = str(tmp_path / "attr_once")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", src, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
