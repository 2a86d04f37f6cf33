"""Build the plain-C demo of the C ABI (tests/c/abi_demo.c) against
include/sfn.h and libsfn.so with gcc."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "predictor_gated_channel_b200")
CUDA = "/usr/local/cuda"


def build_demo(out_path: str) -> str:
    cmd = ["gcc", "-std=c99", "-O1", "-Wall", "-Werror", os.path.join(ROOT, "tests", "c", "abi_demo.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", PKG, "-lsfn", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + PKG, "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", out_path]
    subprocess.run(cmd, check=True)
    return out_path
