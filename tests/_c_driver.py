"""Build and drive tests/c_abi/flce_c_driver.c, a plain C99 caller of the C ABI."""
import os
import shutil
import struct
import subprocess

import numpy as np

from lm_head_linear_tmem_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "flce_c_driver.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
IN_HEADER = struct.Struct("<8s4q2f2i")
OUT_HEADER = struct.Struct("<8sfIq")


def build_driver(out_dir: str) -> str:
    """Compile with -std=c99 -Wall -Wextra -Werror against include/flce.h and link
    the in-tree library and the CUDA runtime; returns the executable's path."""
    so = build.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    exe = os.path.join(out_dir, "flce_c_driver")
    pkg = os.path.dirname(so)
    cmd = [cc, "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           SRC, "-o", exe, "-L", pkg, "-l:_flce.so", f"-Wl,-rpath,{pkg}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{CUDA}/lib64"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"C driver build failed:\n{res.stderr}")
    return exe


def write_input(path, hidden_bits, weight_bits, labels, ignore_index, softcap, grad_scale,
                reduction):
    N, H = hidden_bits.shape
    V = weight_bits.shape[0]
    with open(path, "wb") as f:
        f.write(IN_HEADER.pack(b"FLCEIN1\0", N, H, V, ignore_index, softcap, grad_scale,
                               reduction, 0))
        f.write(np.ascontiguousarray(hidden_bits, dtype=np.uint16).tobytes())
        f.write(np.ascontiguousarray(weight_bits, dtype=np.uint16).tobytes())
        f.write(np.ascontiguousarray(labels, dtype=np.int64).tobytes())


def read_output(path, N, H, V):
    with open(path, "rb") as f:
        magic, loss, status, ntok = OUT_HEADER.unpack(f.read(OUT_HEADER.size))
        assert magic == b"FLCEOUT\0"
        lse = np.frombuffer(f.read(4 * N), dtype=np.float32)
        dh = np.frombuffer(f.read(4 * N * H), dtype=np.float32).reshape(N, H)
        dw = np.frombuffer(f.read(4 * V * H), dtype=np.float32).reshape(V, H)
    return dict(loss=loss, status=status, ntok=ntok, lse=lse, dh=dh, dw=dw)
