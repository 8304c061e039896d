"""The CUDA-core decode kernels (selected by PA_DECODE_BF16_CUDA_CORES=1 and
PA_DECODE_E4M3_CUDA_CORES=1, read once per process), the mma.sync prefill kernel
(PA_PREFILL_MMA_SYNC=1) and the whole-block decode kernel for 8 KV heads
(PA_DECODE_AUTO_WHOLE_BLOCK=1) against the oracle: the parity tests run again in a child
process with the switches set."""
import os
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu
HERE = Path(__file__).resolve().parent


def test_cuda_core_kernels_every_variant():
    env = dict(os.environ, PA_DECODE_BF16_CUDA_CORES="1", PA_DECODE_E4M3_CUDA_CORES="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        str(HERE / "test_gpu_decode.py"), "-k", "every_kernel_variant or fp8_mha_reduced"],
                       env=env, cwd=HERE.parent, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_prefill_mma_sync_kernel():
    """The mma.sync prefill kernel (PA_PREFILL_MMA_SYNC=1) on the prefill parity tests."""
    env = dict(os.environ, PA_PREFILL_MMA_SYNC="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        str(HERE / "test_gpu_prefill.py")], env=env, cwd=HERE.parent, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_auto_schedule_whole_block_kernel():
    """PA_DECODE_AUTO_WHOLE_BLOCK=1 runs PA_PARTITION_AUTO at 8 KV heads on the whole-block
    kernel (and its merge kernel): the AUTO parity tests again in a child process."""
    env = dict(os.environ, PA_DECODE_AUTO_WHOLE_BLOCK="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        str(HERE / "test_gpu_decode.py"), "-k", "auto or split_vs_unsplit"],
                       env=env, cwd=HERE.parent, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
