"""The C ABI from a plain C99 host program on the GPU, without Python in the
call path: the program allocates device memory with the CUDA runtime, copies
seeded inputs in, asks the planner for the split count (lengths included) and
the workspace size, calls fd_decode on the default stream, checks the device
error word and writes the outputs back.  The test compares them with the fp64
oracle and checks that the program's split count is the Python binding's."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import assert_close, reference

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

C_SOURCE = r"""
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <math.h>
#include <cuda_runtime_api.h>
#include "fd.h"

static void* read_file(const char* dir, const char* name, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  void* buf = malloc(bytes);
  if (!f || !buf || fread(buf, 1, bytes, f) != bytes) exit(10);
  fclose(f);
  return buf;
}

static void write_file(const char* dir, const char* name, const void* buf, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(buf, 1, bytes, f) != bytes) exit(11);
  fclose(f);
}

static void* to_device(const void* host, size_t bytes) {
  void* dev = NULL;
  if (cudaMalloc(&dev, bytes) != cudaSuccess) exit(12);
  if (cudaMemcpy(dev, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) exit(13);
  return dev;
}

int main(int argc, char** argv) {
  if (argc != 7) return 1;
  const char* dir = argv[1];
  fd_problem p = {0};
  p.B = atoi(argv[2]);
  p.Hq = atoi(argv[3]);
  p.Hkv = atoi(argv[4]);
  p.D = atoi(argv[5]);
  p.max_len = atoi(argv[6]);
  const size_t q_bytes = (size_t)p.B * p.Hq * p.D * 2;
  const size_t kv_bytes = (size_t)p.B * p.Hkv * p.max_len * p.D * 2;
  int32_t* lens = (int32_t*)read_file(dir, "lens.bin", (size_t)p.B * 4);
  void* q = to_device(read_file(dir, "q.bin", q_bytes), q_bytes);
  void* k = to_device(read_file(dir, "k.bin", kv_bytes), kv_bytes);
  void* v = to_device(read_file(dir, "v.bin", kv_bytes), kv_bytes);
  void* d_lens = to_device(lens, (size_t)p.B * 4);
  const int S = fd_plan_problem(0, &p, lens);
  if (S < 1) return 3;
  const size_t ws_bytes = fd_workspace_bytes(p.B, p.Hq, p.D, S);
  void* ws = NULL;
  if (ws_bytes && cudaMalloc(&ws, ws_bytes) != cudaSuccess) return 14;
  void* out = NULL;
  float* lse = NULL;
  if (cudaMalloc(&out, q_bytes) != cudaSuccess) return 15;
  if (cudaMalloc((void**)&lse, (size_t)p.B * p.Hq * 4) != cudaSuccess) return 16;
  const float scale = 1.0f / sqrtf((float)p.D);
  fd_status st = fd_decode(&p, q, k, v, (const int32_t*)d_lens, NULL, scale, S, out, lse, ws,
                           ws_bytes, NULL);
  if (st != FD_OK) {
    fprintf(stderr, "fd_decode: %s\n", fd_status_string(st));
    return 4;
  }
  st = fd_check_device_error(NULL);
  if (st != FD_OK) {
    fprintf(stderr, "device: %s\n", fd_status_string(st));
    return 5;
  }
  void* h_out = malloc(q_bytes);
  void* h_lse = malloc((size_t)p.B * p.Hq * 4);
  if (!h_out || !h_lse) return 17;
  if (cudaMemcpy(h_out, out, q_bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return 18;
  if (cudaMemcpy(h_lse, lse, (size_t)p.B * p.Hq * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return 19;
  write_file(dir, "out.bin", h_out, q_bytes);
  write_file(dir, "lse.bin", h_lse, (size_t)p.B * p.Hq * 4);
  printf("%d\n", S);
  return 0;
}
"""


def test_c_host_program_decodes_through_the_abi(cuda_device, tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    B, Hq, Hkv, D, L = 3, 32, 8, 128, 5000
    w = wl.make_problem(B, Hq, Hkv, D, L, seed=470, seqlens=[5000, 1200, 0], nan_pad=True)
    for name, arr in (("q.bin", w.q), ("k.bin", w.k), ("v.bin", w.v),
                      ("lens.bin", np.asarray(w.seqlens, dtype=np.int32))):
        np.ascontiguousarray(arr).tofile(tmp_path / name)
    src = tmp_path / "decode.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "decode"
    libdir = os.path.dirname(fd.LIB_PATH)
    cudalib = os.path.join(CUDA, "lib64")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-O2",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lfd", "-L", cudalib, "-lcudart",
                    "-lm", f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{cudalib}"], check=True)
    r = subprocess.run([str(exe), str(tmp_path), str(B), str(Hq), str(Hkv), str(D), str(L)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stderr)
    S = int(r.stdout.strip())
    prob = fd.make_problem(B, Hq, Hkv, D, L)
    assert S == fd.fd_plan_problem(0, prob, w.seqlens)
    got = wl.bf16_bits_to_f64(np.fromfile(tmp_path / "out.bin", dtype=np.uint16)
                              .reshape(B, Hq, D))
    got_lse = np.fromfile(tmp_path / "lse.bin", dtype=np.float32).reshape(B, Hq).astype(np.float64)
    ref, ref_lse = reference(w)
    assert_close(got, got_lse, ref, ref_lse, f"C host program, S={S}")
