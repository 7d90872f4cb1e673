"""The NVTX recorder the GPU tests use to see the library's ranges
(tests/nvtx_recorder.c), checked on the host: built with gcc, loaded by the
NVTX v3 headers of a small C program through NVTX_INJECTION64_PATH, it
writes the program's domain, pushes and pops in order."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA_INC = "/usr/local/cuda/include"

DRIVER = r"""
#include <string.h>
#include <nvtx3/nvToolsExt.h>
static void push(nvtxDomainHandle_t d, const char* m) {
  nvtxEventAttributes_t a;
  memset(&a, 0, sizeof a);
  a.version = NVTX_VERSION;
  a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
  a.messageType = NVTX_MESSAGE_TYPE_ASCII;
  a.message.ascii = m;
  nvtxDomainRangePushEx(d, &a);
}
int main(void) {
  nvtxDomainHandle_t d = nvtxDomainCreateA("probe");
  push(d, "outer");
  push(d, "inner [0, 8)");
  nvtxDomainRangePop(d);
  nvtxDomainRangePop(d);
  return 0;
}
"""


def build_recorder(out_dir: str) -> str:
    """gcc the recorder into out_dir; returns the .so path."""
    lib = os.path.join(out_dir, "libnvtx_recorder.so")
    subprocess.run(["gcc", "-shared", "-fPIC", "-O1", "-I", CUDA_INC, os.path.join(HERE, "nvtx_recorder.c"),
                    "-o", lib], check=True, capture_output=True, text=True)
    return lib


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(os.path.join(CUDA_INC, "nvtx3")),
                    reason="needs gcc and the NVTX v3 headers")
def test_recorder_writes_domain_pushes_and_pops(tmp_path):
    lib = build_recorder(str(tmp_path))
    src = tmp_path / "drv.c"
    src.write_text(DRIVER)
    exe = str(tmp_path / "drv")
    subprocess.run(["gcc", "-I", CUDA_INC, str(src), "-o", exe, "-ldl"], check=True, capture_output=True)
    rec = tmp_path / "rec.txt"
    env = dict(os.environ, NVTX_INJECTION64_PATH=lib, NVTX_RECORD_FILE=str(rec))
    subprocess.run([exe], check=True, env=env, timeout=60)
    assert rec.read_text().splitlines() == ["domain probe", "push probe outer", "push probe inner [0, 8)",
                                            "pop probe", "pop probe"]
    # without the variable nothing is loaded and nothing written
    rec.unlink()
    env.pop("NVTX_INJECTION64_PATH")
    subprocess.run([exe], check=True, env=env, timeout=60)
    assert not rec.exists()
