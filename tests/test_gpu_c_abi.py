"""The C ABI doing GPU work from C: a C99 program (include/gdn.h and the CUDA runtime, no
torch) allocates device buffers with cudaMalloc, copies seeded inputs in, and calls
gdn_chunk_fwd (tensor-core path: bf16 q/k/v, d = 128, chunk 64; workspace sized by
gdn_chunk_fwd_workspace_bytes), gdn_gate_norm on its y, and gdn_decode_step on its final
state, then gdn_device_error. Its outputs are compared here with the fp64 oracle at the
bf16-input bar (max|d| / rms <= 2e-2)."""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import TOL, oracle_prefill, rel_err

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "gated_deltanet_05_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

PROGRAM = r'''
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime.h>
#include "gdn.h"

static void *read_file(const char *dir, const char *name, size_t bytes)
{
    char path[1024];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) { fprintf(stderr, "missing %s\n", path); exit(10); }
    void *p = malloc(bytes);
    if (fread(p, 1, bytes, f) != bytes) { fprintf(stderr, "short %s\n", path); exit(11); }
    fclose(f);
    return p;
}

static void write_file(const char *dir, const char *name, const void *p, size_t bytes)
{
    char path[1024];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(p, 1, bytes, f) != bytes) exit(12);
    fclose(f);
}

static void *to_device(const void *h, size_t bytes)
{
    void *d = NULL;
    if (cudaMalloc(&d, bytes) != cudaSuccess) exit(13);
    if (cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) exit(14);
    return d;
}

#define CHECK(call) do { gdn_status s_ = (call); if (s_ != GDN_OK) { \
    fprintf(stderr, "%s -> %s\n", #call, gdn_status_string(s_)); return 20; } } while (0)

int main(int argc, char **argv)
{
    const char *dir = argv[1];
    int *dims = (int *)read_file(dir, "dims.bin", 4 * sizeof(int));
    const int n_seq = dims[0], n_tok = dims[1], H = dims[2], d = dims[3];
    const size_t tok = (size_t)n_tok * H, vec = tok * d, st = (size_t)n_seq * H * d * d;
    int32_t *cu = (int32_t *)read_file(dir, "cu.bin", (n_seq + 1) * sizeof(int32_t));
    void *q = to_device(read_file(dir, "q.bin", vec * 2), vec * 2);
    void *k = to_device(read_file(dir, "k.bin", vec * 2), vec * 2);
    void *v = to_device(read_file(dir, "v.bin", vec * 2), vec * 2);
    void *z = to_device(read_file(dir, "z.bin", vec * 2), vec * 2);
    float *la = (float *)to_device(read_file(dir, "la.bin", tok * 4), tok * 4);
    float *be = (float *)to_device(read_file(dir, "beta.bin", tok * 4), tok * 4);
    float *w = (float *)to_device(read_file(dir, "w.bin", d * 4), d * 4);
    int32_t *cu_d = (int32_t *)to_device(cu, (n_seq + 1) * sizeof(int32_t));
    const size_t dtok = (size_t)n_seq * H;
    void *dq = to_device(read_file(dir, "dq.bin", dtok * d * 4), dtok * d * 4);
    void *dk = to_device(read_file(dir, "dk.bin", dtok * d * 4), dtok * d * 4);
    void *dv = to_device(read_file(dir, "dv.bin", dtok * d * 4), dtok * d * 4);
    float *da = (float *)to_device(read_file(dir, "dalpha.bin", dtok * 4), dtok * 4);
    float *db = (float *)to_device(read_file(dir, "dbeta.bin", dtok * 4), dtok * 4);

    float *y, *S_T, *o, *yd;
    void *ws = NULL;
    if (cudaMalloc((void **)&y, vec * 4) || cudaMalloc((void **)&S_T, st * 4) ||
        cudaMalloc((void **)&o, vec * 4) || cudaMalloc((void **)&yd, dtok * d * 4)) return 15;
    const size_t ws_bytes = gdn_chunk_fwd_workspace_bytes(n_seq, n_tok, H, d, d, 64);
    if (ws_bytes == 0) return 16;
    if (cudaMalloc(&ws, ws_bytes) != cudaSuccess) return 17;

    CHECK(gdn_chunk_fwd(q, k, v, GDN_BF16, la, be, NULL, cu_d, cu, n_seq, H, d, d, 64, 1.0f, y, GDN_F32,
                        S_T, ws, ws_bytes, NULL));
    CHECK(gdn_gate_norm(y, GDN_F32, z, GDN_BF16, w, (int64_t)tok, d, 1e-6f, o, GDN_F32, NULL));
    float *S_h = (float *)malloc(st * 4);
    if (cudaMemcpy(S_h, S_T, st * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return 18;
    CHECK(gdn_decode_step(dq, dk, dv, GDN_F32, da, db, S_T, n_seq, H, d, d, 1.0f, yd, GDN_F32, NULL));
    CHECK(gdn_device_error(NULL));

    float *y_h = (float *)malloc(vec * 4), *o_h = (float *)malloc(vec * 4);
    float *S2_h = (float *)malloc(st * 4), *yd_h = (float *)malloc(dtok * d * 4);
    if (cudaMemcpy(y_h, y, vec * 4, cudaMemcpyDeviceToHost) || cudaMemcpy(o_h, o, vec * 4, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(S2_h, S_T, st * 4, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(yd_h, yd, dtok * d * 4, cudaMemcpyDeviceToHost)) return 19;
    write_file(dir, "y_out.bin", y_h, vec * 4);
    write_file(dir, "o_out.bin", o_h, vec * 4);
    write_file(dir, "S_out.bin", S_h, st * 4);
    write_file(dir, "S2_out.bin", S2_h, st * 4);
    write_file(dir, "yd_out.bin", yd_h, dtok * d * 4);
    printf("ok\n");
    return 0;
}
'''


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    lib = os.path.join(LIBDIR, "libgdn_b200.so")
    if not os.path.exists(lib):
        pytest.skip("libgdn_b200.so not built")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = tmp_path_factory.mktemp("cabi")
    src, exe = d / "gpu_abi.c", d / "gpu_abi"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(CUDA, "include"), str(src), "-o", str(exe), "-L", LIBDIR,
                    "-lgdn_b200", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    "-Wl,-rpath," + LIBDIR, "-Wl,-rpath," + os.path.join(CUDA, "lib64")], check=True)
    return str(exe)


def test_c_program_runs_the_hot_path(program, tmp_path):
    w = W.Workload("cabi", "bf16", (200, 37, 64), 2, 128, 128, 64, seed=77)
    inp = W.make_prefill_inputs(w)
    n_seq, n_tok, H, d = 3, int(inp["cu_seqlens"][-1]), 2, 128
    x = W.make_decode_inputs(W.WORKLOADS["decode"], 5, n_seq=n_seq, H=H, d=d)
    raw = lambda t: t.contiguous().view(torch.int16).numpy().tobytes() if t.dtype == torch.bfloat16 \
        else t.contiguous().numpy().tobytes()
    files = {"dims.bin": np.array([n_seq, n_tok, H, d], dtype=np.int32).tobytes(),
             "cu.bin": inp["cu_seqlens"].numpy().astype(np.int32).tobytes(),
             "q.bin": raw(inp["q"]), "k.bin": raw(inp["k"]), "v.bin": raw(inp["v"]), "z.bin": raw(inp["z"]),
             "la.bin": raw(inp["log_alpha"]), "beta.bin": raw(inp["beta"]), "w.bin": raw(inp["w_norm"]),
             "dq.bin": raw(x["q"]), "dk.bin": raw(x["k"]), "dv.bin": raw(x["v"]),
             "dalpha.bin": raw(x["alpha"]), "dbeta.bin": raw(x["beta"])}
    for name, b in files.items():
        (tmp_path / name).write_bytes(b)
    r = subprocess.run([program, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    load = lambda name, shape: np.fromfile(tmp_path / name, dtype=np.float32).reshape(shape).astype(np.float64)
    y = load("y_out.bin", (n_tok, H, d))
    o = load("o_out.bin", (n_tok, H, d))
    S = load("S_out.bin", (n_seq, H, d, d))
    S2 = load("S2_out.bin", (n_seq, H, d, d))
    yd = load("yd_out.bin", (n_seq, H, d))
    y_ref, S_ref = oracle_prefill(inp)
    assert rel_err(y, y_ref) <= TOL["bf16"]
    assert rel_err(S, S_ref) <= TOL["bf16"]
    o_ref = oracle.gate_norm(y_ref, inp["z"], inp["w_norm"])
    assert rel_err(o, o_ref) <= TOL["bf16"]
    # the decode step continues from the prefill's final state (as the C program left it)
    yd_ref, S2_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                                        oracle.state_from_lib(S))
    assert rel_err(yd, yd_ref) <= TOL["f32"]
    assert rel_err(S2, oracle.state_to_lib(S2_ref)) <= TOL["f32"]
