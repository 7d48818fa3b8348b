"""A plain C program drives the whole ZeRO-2 step through the C ABI.

No Python and no torch on the data path: the program allocates every buffer
with the CUDA runtime, reads seeded inputs from a file, runs three steps
through the native runner (zero_runner_create / _launch / _commit, one of
them with an injected inf so that it is skipped), then the staged route
(zero_reduce_scatter_grads + zero_adam_step_reduced) for one more step,
writes the committed state back to a file, and rebuilds the parameters from 4
rank shards with zero_allgather_params (an odd partition: ranks 1-3 sit off
their destination's 16-byte phase).  The test compares every array
with the oracle bit for bit, and the runner's t and loss scale with the
oracle's rule.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

C_PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <stdint.h>
#include <cuda_runtime_api.h>
#include "zero.h"

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
    fprintf(stderr, "CUDA: %s at line %d\n", cudaGetErrorString(e_), __LINE__); return 2; } } while (0)
#define ZK(x) do { int r_ = (x); if (r_ != ZERO_OK) { \
    fprintf(stderr, "zero: %s (%s) at line %d\n", zero_strerror(r_), zero_last_error(), __LINE__); return 3; } } while (0)

static void* dalloc(size_t bytes) { void* p = NULL; return cudaMalloc(&p, bytes) == cudaSuccess ? p : NULL; }

int main(int argc, char** argv) {
    if (argc != 6) return 1;
    const int world = atoi(argv[3]), steps = atoi(argv[5]);
    const int64_t n = atoll(argv[4]);
    FILE* in = fopen(argv[1], "rb");
    if (!in) return 1;
    uint16_t* g_host = malloc((size_t)(steps + 1) * world * n * 2);
    float* master_host = malloc((size_t)n * 4);
    uint16_t* params_host = malloc((size_t)n * 2);
    if (fread(g_host, 2, (size_t)(steps + 1) * world * n, in) != (size_t)(steps + 1) * world * n) return 1;
    if (fread(master_host, 4, (size_t)n, in) != (size_t)n) return 1;
    if (fread(params_host, 2, (size_t)n, in) != (size_t)n) return 1;
    fclose(in);

    void* grads[ZERO_MAX_WORLD];
    for (int k = 0; k < world; ++k) if (!(grads[k] = dalloc((size_t)n * 2))) return 2;
    zero_bucket_banks_t bk;
    bk.padded_numel = n;
    bk.grad_bufs = (const void* const*)grads;
    for (int b = 0; b < 2; ++b) {
        bk.master[b] = dalloc((size_t)n * 4); bk.m[b] = dalloc((size_t)n * 4); bk.v[b] = dalloc((size_t)n * 4);
        bk.params[b] = dalloc((size_t)n * 2);
        if (!bk.master[b] || !bk.m[b] || !bk.v[b] || !bk.params[b]) return 2;
        CK(cudaMemcpy(bk.master[b], master_host, (size_t)n * 4, cudaMemcpyHostToDevice));
        CK(cudaMemcpy(bk.params[b], params_host, (size_t)n * 2, cudaMemcpyHostToDevice));
        CK(cudaMemset(bk.m[b], 0, (size_t)n * 4));
        CK(cudaMemset(bk.v[b], 0, (size_t)n * 4));
    }
    int32_t* flag_dev = dalloc(8);
    int32_t* flag_host = NULL;
    CK(cudaHostAlloc((void**)&flag_host, 4, cudaHostAllocDefault));
    zero_adam_hparams_t hp = {1e-3f, 0.9f, 0.999f, 1e-8f, 0.01f, 1, 0.0f};
    zero_runner_t* r = NULL;
    ZK(zero_runner_create(&bk, 1, world, ZERO_F16, ZERO_F16, &hp, 65536.0f, 1000, 1.0f, flag_dev, flag_host,
                          NULL, NULL, &r));
    for (int s = 0; s < steps; ++s) {
        for (int k = 0; k < world; ++k)
            CK(cudaMemcpy(grads[k], g_host + ((size_t)s * world + k) * n, (size_t)n * 2, cudaMemcpyHostToDevice));
        int32_t applied = -1;
        ZK(zero_runner_launch(r, NULL));
        ZK(zero_runner_commit(r, NULL, &applied));
        printf("applied %d\n", applied);
    }
    int64_t t; float scale; int32_t good, bank;
    ZK(zero_runner_state(r, &t, &scale, &good, &bank));
    printf("state %lld %g %d\n", (long long)t, scale, good);
    zero_runner_destroy(r);

    /* one more step by the staged route, in place on the committed bank */
    for (int k = 0; k < world; ++k)
        CK(cudaMemcpy(grads[k], g_host + ((size_t)steps * world + k) * n, (size_t)n * 2, cudaMemcpyHostToDevice));
    float* reduced = dalloc((size_t)n * 4);
    if (!reduced) return 2;
    CK(cudaMemset(flag_dev, 0, 8));
    ZK(zero_reduce_scatter_grads((const void* const*)grads, world, n, ZERO_ALL_PARTITIONS, ZERO_F16, scale, 0.0f,
                                 reduced, flag_dev, NULL, NULL, NULL));
    hp.step = t + 1;
    ZK(zero_adam_step_reduced(reduced, n, bk.master[bank], bk.m[bank], bk.v[bank], bk.master[bank], bk.m[bank],
                              bk.v[bank], bk.params[bank], ZERO_F16, &hp, flag_dev + 1, flag_dev, NULL, 0.0f, NULL));
    int32_t flags[2];
    CK(cudaMemcpy(flags, flag_dev, 8, cudaMemcpyDeviceToHost));
    printf("staged %d %d\n", flags[0], flags[1]);

    FILE* out = fopen(argv[2], "wb");
    float* f = malloc((size_t)n * 4);
    float* arrs[3] = {bk.master[bank], bk.m[bank], bk.v[bank]};
    for (int i = 0; i < 3; ++i) {
        CK(cudaMemcpy(f, arrs[i], (size_t)n * 4, cudaMemcpyDeviceToHost));
        fwrite(f, 4, (size_t)n, out);
    }
    CK(cudaMemcpy(params_host, bk.params[bank], (size_t)n * 2, cudaMemcpyDeviceToHost));
    fwrite(params_host, 2, (size_t)n, out);

    /* the all-gather: the parameters split into `world` rank shards of their
       own, rebuilt into one buffer (P odd: ranks 1.. are realigned) */
    const int64_t P = n / world;
    void* shards[ZERO_MAX_WORLD];
    for (int k = 0; k < world; ++k) {
        if (!(shards[k] = dalloc((size_t)P * 2))) return 2;
        CK(cudaMemcpy(shards[k], (const uint16_t*)bk.params[bank] + (size_t)k * P, (size_t)P * 2,
                      cudaMemcpyDeviceToDevice));
    }
    uint16_t* full = dalloc((size_t)n * 2);
    int32_t* status = dalloc(4);
    if (!full || !status) return 2;
    CK(cudaMemset(full, 0xEE, (size_t)n * 2));
    CK(cudaMemset(status, 0, 4));
    ZK(zero_allgather_params((const void* const*)shards, world, 0, P, ZERO_F16, full, status, NULL));
    int32_t st = -1;
    CK(cudaMemcpy(&st, status, 4, cudaMemcpyDeviceToHost));
    printf("gather %d\n", st);
    CK(cudaMemcpy(params_host, full, (size_t)n * 2, cudaMemcpyDeviceToHost));
    fwrite(params_host, 2, (size_t)n, out);
    fclose(out);
    return 0;
}
"""


def test_c_program_runs_the_step_through_the_abi(tmp_path):
    world, n, steps = 4, 4 * 250_003, 3
    inject_step = 2                      # the second runner step overflows and is skipped
    adam = workloads.AdamConfig(weight_decay=0.01)
    master = workloads.master(n, 61)
    ref = oracle.initial_state(master)
    scaler = oracle.Scaler(65536.0)
    G_all = []
    for s in range(1, steps + 2):
        G = [workloads.grads(n, workloads.seed_for(62, s, k), 1e-3, scaler.scale) for k in range(world)]
        if s == inject_step:
            workloads.inject(G[1], np.array([17]), np.array([True]))
        G_all.append(G)
        if s <= steps:
            ovf, _ = oracle.flat_step(G, ref, adam, scaler.t + 1, scaler.scale, float(world))   # skips on overflow
            if not ovf:
                scaler.t += 1
            scaler.scale, scaler.good_steps = oracle.loss_scale_update(scaler.scale, scaler.good_steps, bool(ovf))
    # the staged step uses the scale after the runner's steps
    G_last = [workloads.grads(n, workloads.seed_for(62, steps + 1, k), 1e-3, scaler.scale) for k in range(world)]
    G_all[-1] = G_last
    oracle.flat_step(G_last, ref, adam, scaler.t + 1, scaler.scale, float(world))

    inp = tmp_path / "in.bin"
    with open(inp, "wb") as f:
        for G in G_all:
            for g in G:
                f.write(g.tobytes())
        f.write(master.astype(np.float32).tobytes())
        f.write(oracle.initial_state(master).params.tobytes())
    src = tmp_path / "driver.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "driver"
    libdir = os.path.dirname(Z.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(CUDA, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-lzero", f"-Wl,-rpath,{libdir}",
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"])
    outp = tmp_path / "out.bin"
    r = subprocess.run([str(exe), str(inp), str(outp), str(world), str(n), str(steps)], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.splitlines()
    assert lines[:3] == ["applied 1", "applied 0", "applied 1"]
    t, scale, good = lines[3].split()[1:]
    assert int(t) == scaler.t == 2 and float(scale) == scaler.scale == 32768.0 and int(good) == scaler.good_steps
    assert lines[4] == "staged 0 0"
    data = outp.read_bytes()
    got = [np.frombuffer(data, np.float32, n, i * 4 * n) for i in range(3)]
    params = np.frombuffer(data, np.uint16, n, 12 * n)
    for arr, name in zip(got, ("master", "m", "v")):
        assert np.array_equal(arr.view(np.uint32), getattr(ref, name).view(np.uint32)), name
    assert np.array_equal(params, ref.params)
    # the all-gather of the 4 rank shards through the C ABI
    assert lines[5] == "gather 0"
    P = n // world
    gathered = np.frombuffer(data, np.uint16, n, 14 * n)
    assert np.array_equal(gathered, oracle.allgather([ref.params[r * P:(r + 1) * P] for r in range(world)], 0, P))
