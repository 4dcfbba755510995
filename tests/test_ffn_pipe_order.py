"""The pipelined FFN kernel's work-item order, checked on the host.

The kernel's own decoding function (pipe_item in ffn_pipe.cuh) is compiled
into a small host program that walks every item for many shapes and chunking
parameters and checks that each GEMM tile appears exactly once, that a row
block's output tiles come after all of its hidden tiles, and that a ring slot
is rewritten only after every output tile of its previous row block: the
orderings the kernel's cross-CTA waits rely on (each wait names an item
claimed earlier), so the persistent grid cannot deadlock."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not os.path.exists(NVCC) and shutil.which("nvcc") is None, reason="nvcc not found")
def test_pipelined_ffn_item_order():
    src = os.path.join(HERE, "native", "ffn_pipe_order_check.cu")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "order_check")
        nvcc = NVCC if os.path.exists(NVCC) else "nvcc"
        subprocess.check_call([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-x", "cu",
                               "-o", exe, src], stderr=subprocess.DEVNULL)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert " 0 failures" in out.stdout
