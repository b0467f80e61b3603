"""The C ABI used from plain C: tests/c_abi/prefill.c includes only
include/xattn.h and the CUDA runtime, allocates with cudaMalloc and runs the
fused step. It is compiled with gcc on the CPU; on the GPU its output must
equal, bit for bit, what the Python binding returns for the same inputs."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from block_sparse_long_score_b200 import build as xbuild
from block_sparse_long_score_b200 import xattn as X

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


def _compile(tmp_path):
    xbuild.build()
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    exe = str(tmp_path / "prefill")
    libdir = os.path.dirname(X.library_path())
    cmd = [gcc, "-std=c11", "-O1", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c_abi", "prefill.c"), "-o", exe,
           "-L", libdir, "-lxattn", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_program_compiles_against_the_header_alone(tmp_path):
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
def test_c_program_matches_the_binding(tmp_path):
    from block_sparse_long_score_b200 import xattn_score_select, xattn_sparse_attn
    from block_sparse_long_score_b200.synth import make_problem
    exe = _compile(tmp_path)
    prob = make_problem("c1", L=1088, hq=4, hkv=2)         # a short last block too
    raw = b"".join(t.contiguous().view(torch.int16).numpy().tobytes()
                   for t in (prob.Q, prob.K, prob.V))
    inp, out = tmp_path / "in.bin", tmp_path / "out.bin"
    inp.write_bytes(raw)
    tau = float(prob.tau[0])
    args = [exe, str(inp), str(out), "1", str(prob.hq), str(prob.hkv), str(prob.L),
            str(prob.d), str(prob.B), str(prob.S), "1" if prob.causal else "0", repr(tau)]
    r = subprocess.run(args, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    got = torch.from_numpy(np.frombuffer(out.read_bytes(), dtype=np.int16).copy())
    got = got.view(torch.bfloat16).reshape(prob.Q.shape)
    Q, K, V = prob.Q.cuda(), prob.K.cuda(), prob.V.cuda()
    _, counts, idx = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, [tau] * prob.hq)
    ref = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal)
    torch.cuda.synchronize()
    assert torch.equal(got, ref.cpu())
