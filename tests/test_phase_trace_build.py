"""The phase-trace tool still applies to the current GEMM source (no GPU).

diffusion_decoding_step_b200.phase_trace instruments a copy of gemm.cu by
matching anchors in it. This checks that every anchor matches once and that
the stamped copy compiles, so the tool breaks here first when the kernel
changes.
"""
import os
import shutil
import subprocess

from diffusion_decoding_step_b200 import build, phase_trace


def test_stamped_gemm_copy_compiles(tmp_path):
    csrc = tmp_path / "src" / "diffusion_decoding_step_b200" / "csrc"
    inc = tmp_path / "src" / "include"
    csrc.mkdir(parents=True)
    inc.mkdir(parents=True)
    for f in os.listdir(build.CSRC):
        shutil.copy(os.path.join(build.CSRC, f), csrc)
    shutil.copy(os.path.join(build.HERE, "..", "include", "dllm.h"), inc)
    phase_trace._patch(str(csrc / "kernels.cuh"), phase_trace._KERNELS)
    phase_trace._patch(str(csrc / "gemm.cu"), phase_trace._GEMM)
    text = (csrc / "gemm.cu").read_text()
    assert text.count("TS(") >= 14 and "dllm_gt_read" in text
    flags = [f for f in build.FLAGS if f != "-shared"]
    subprocess.run([build.nvcc(), *flags, "-c", str(csrc / "gemm.cu"), "-o",
                    str(tmp_path / "gemm.o")], check=True)
