"""Per-device caches of the host code (kernel attributes set once per device
and kernel, the SM count per device), compiled with the host C++ compiler and
run without a GPU (tests/native/device_cache_test.cpp)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_per_device_caches(tmp_path):
    cxx = shutil.which('g++') or shutil.which('c++')
    if not cxx:
        pytest.skip('no host C++ compiler')
    exe = tmp_path / 'device_cache_test'
    src = os.path.join(ROOT, 'tests', 'native', 'device_cache_test.cpp')
    inc = os.path.join(ROOT, 'llama_transformer_decoder_b200', 'csrc')
    subprocess.run([cxx, '-std=c++17', '-O1', '-pthread', '-I', inc, src, '-o', str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert 'device cache ok' in r.stdout
