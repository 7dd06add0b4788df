"""The C ABI from a plain C program on the GPU: device buffers from
cudaMalloc, no Python or torch on the path.  The program runs a verify
attention whose answer is known in closed form (all scores equal, so every
output is the mean of the visible V rows, all 1.0) and a penalty/accept
call with planted maxima, and checks the statuses and the results."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

PROG = r"""
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include "ts_verify.h"

#define CHECK(x) do { if (!(x)) { fprintf(stderr, "failed: %s (line %d)\n", #x, __LINE__); return 1; } } while (0)

int main(void) {
    const int T = 40, HQ = 32, HKV = 8, D = 128, NCTX = 4096, V = 1000;
    const long cap = NCTX + T;
    int32_t parent[40];
    parent[0] = -1;
    for (int i = 1; i < T; ++i) parent[i] = (i - 1) / 3;

    /* q = 0 makes every score 0: each output row is the mean of the V rows
       it sees, and every V element is 1.0 (bf16 0x3F80) */
    const size_t nq = (size_t)T * HQ * D, nkv = (size_t)HKV * cap * D;
    uint16_t *hv = (uint16_t *)malloc(nkv * 2);
    for (size_t i = 0; i < nkv; ++i) hv[i] = 0x3F80;
    void *q, *k, *v, *ws;
    float *out;
    CHECK(cudaMalloc(&q, nq * 2) == cudaSuccess);
    CHECK(cudaMalloc(&k, nkv * 2) == cudaSuccess);
    CHECK(cudaMalloc(&v, nkv * 2) == cudaSuccess);
    CHECK(cudaMalloc((void **)&out, nq * 4) == cudaSuccess);
    CHECK(cudaMemset(q, 0, nq * 2) == cudaSuccess);
    CHECK(cudaMemset(k, 0, nkv * 2) == cudaSuccess);
    CHECK(cudaMemcpy(v, hv, nkv * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    const size_t wsb = ts_tree_verify_attn_workspace_size(HQ, HKV, D, NCTX, T);
    CHECK(wsb > 0);
    CHECK(cudaMalloc(&ws, wsb) == cudaSuccess);
    CHECK(cudaMemset(ws, 0, wsb) == cudaSuccess);
    CHECK(ts_tree_verify_attn(q, k, v, cap, HQ, HKV, D, NCTX, T, parent, 0.08838835f, out, ws,
                              wsb, NULL) == TS_OK);
    CHECK(cudaDeviceSynchronize() == cudaSuccess);
    CHECK(ts_workspace_status(ws, NULL, 1) == TS_OK);
    float *ho = (float *)malloc(nq * 4);
    CHECK(cudaMemcpy(ho, out, nq * 4, cudaMemcpyDeviceToHost) == cudaSuccess);
    double err = 0.0;
    for (size_t i = 0; i < nq; ++i) err = fmax(err, fabs(ho[i] - 1.0));
    CHECK(err <= 2e-3);

    /* penalty/accept: node i's largest logit is 5.0 at id (7 i + 3) % V; the
       window holds none of them; tree tokens repeat the parent's argmax on
       the first child only, so the accepted path is 0 -> 1 -> 4 -> 13 */
    float *hl = (float *)malloc((size_t)T * V * 4);
    for (int i = 0; i < T; ++i)
        for (int j = 0; j < V; ++j) hl[(size_t)i * V + j] = (j == (7 * i + 3) % V) ? 5.0f : -1.0f;
    int32_t htok[40], hwin[4] = {999, 998, 997, 996};
    htok[0] = 0;
    for (int i = 1; i < T; ++i)
        htok[i] = (i == 3 * parent[i] + 1) ? (7 * parent[i] + 3) % V : 500 + i;
    float *lg;
    int32_t *win, *tok, *acc, *am;
    CHECK(cudaMalloc((void **)&lg, (size_t)T * V * 4) == cudaSuccess);
    CHECK(cudaMalloc((void **)&win, sizeof hwin) == cudaSuccess);
    CHECK(cudaMalloc((void **)&tok, sizeof htok) == cudaSuccess);
    CHECK(cudaMalloc((void **)&acc, (2 + T) * 4) == cudaSuccess);
    CHECK(cudaMalloc((void **)&am, T * 4) == cudaSuccess);
    CHECK(cudaMemcpy(lg, hl, (size_t)T * V * 4, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(win, hwin, sizeof hwin, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(tok, htok, sizeof htok, cudaMemcpyHostToDevice) == cudaSuccess);
    const size_t pwb = ts_penalize_accept_workspace_size(T, V);
    void *pws;
    CHECK(cudaMalloc(&pws, pwb) == cudaSuccess);
    CHECK(cudaMemset(pws, 0, pwb) == cudaSuccess);
    CHECK(ts_penalize_accept(lg, T, V, win, 4, 1.2f, parent, tok, am, acc, pws, pwb, NULL) == TS_OK);
    CHECK(cudaDeviceSynchronize() == cudaSuccess);
    int32_t hacc[42], ham[40];
    CHECK(cudaMemcpy(hacc, acc, sizeof hacc, cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(ham, am, sizeof ham, cudaMemcpyDeviceToHost) == cudaSuccess);
    for (int i = 0; i < T; ++i) CHECK(ham[i] == (7 * i + 3) % V);
    CHECK(hacc[0] == 3 && hacc[2] == 0 && hacc[3] == 1 && hacc[4] == 4 && hacc[5] == 13);
    CHECK(hacc[1] == (7 * 13 + 3) % V);
    puts("ok");
    return 0;
}
"""


@pytest.mark.gpu
def test_c_program_runs_the_path_through_the_abi(tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_ultra_long_b200 import LIB_PATH, build
    build.build()
    src = tmp_path / "consumer.c"
    src.write_text(PROG)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(CUDA, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-l:libtsverify.so", "-Wl,-rpath," + libdir,
                    "-L", os.path.join(CUDA, "lib64"), "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
                    "-lcudart", "-lm"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stderr)
