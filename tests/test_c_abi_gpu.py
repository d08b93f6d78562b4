"""The boundary end to end from C: a plain C program (gcc, C11, the CUDA
runtime's C API for memory only) copies host buffers to the device, calls
fa_compress_kv, fa_attention_fwd (bf16 and int8 K/V, with the epilogue
chain) and fa_attention_decode through include/fa.h, and copies the results
back to files.  The codes and scales must equal the oracle's bit for bit and
the outputs must pass the bf16 gate against the fp64 oracle (fkl_python
PR #6, Summary: flash_attention, compress_kv and the decode step;
Verification: codes exact, outputs within max abs 2e-2 / relative L2 5e-3)."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from conftest import assert_close_bf16
from flashattention_attention_b200 import inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
B, HQ, HKV, D, SQ, SK = 2, 8, 2, 128, 100, 256
LENS = (256, 133)

C_SOURCE = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime.h>
#include "fa.h"

#define B %(B)d
#define HQ %(HQ)d
#define HKV %(HKV)d
#define D %(D)d
#define SQ %(SQ)d
#define SK %(SK)d

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
    fprintf(stderr, "%%s: %%s\n", #x, cudaGetErrorString(e_)); return 1; } } while (0)
#define FK(x) do { fa_status s_ = (x); if (s_ != FA_OK) { \
    fprintf(stderr, "%%s: %%s\n", #x, fa_status_string(s_)); return 1; } } while (0)

static char path[4096];
static const char *at(const char *dir, const char *name) {
    snprintf(path, sizeof path, "%%s/%%s", dir, name);
    return path;
}
static void *load(const char *dir, const char *name, size_t bytes) {
    FILE *f = fopen(at(dir, name), "rb");
    void *p = malloc(bytes);
    if (!f || !p || fread(p, 1, bytes, f) != bytes) { fprintf(stderr, "read %%s\n", name); exit(1); }
    fclose(f);
    return p;
}
static void save(const char *dir, const char *name, const void *p, size_t bytes) {
    FILE *f = fopen(at(dir, name), "wb");
    if (!f || fwrite(p, 1, bytes, f) != bytes) { fprintf(stderr, "write %%s\n", name); exit(1); }
    fclose(f);
}
/* device copy of a host buffer */
static int upload(void **dst, const void *src, size_t bytes) {
    if (cudaMalloc(dst, bytes) != cudaSuccess) return 1;
    return cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice) != cudaSuccess;
}
/* host file of a device buffer */
static int download(const char *dir, const char *name, const void *src, size_t bytes) {
    void *h = malloc(bytes);
    if (!h || cudaMemcpy(h, src, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
    save(dir, name, h, bytes);
    free(h);
    return 0;
}

int main(int argc, char **argv) {
    if (argc != 2) return 2;
    const char *dir = argv[1];
    const size_t nq = (size_t)B * HQ * SQ * D, nk = (size_t)B * HKV * SK * D, nd = (size_t)B * HQ * D;
    const size_t rows = (size_t)B * HKV * SK;
    void *q, *k, *v, *qd, *out, *dec, *ws;
    int8_t *kc, *vc;
    float *ks, *vs;
    int32_t *lens;
    const int32_t host_lens[B] = {%(L0)d, %(L1)d};
    if (upload(&q, load(dir, "q.bin", nq * 2), nq * 2) || upload(&k, load(dir, "k.bin", nk * 2), nk * 2) ||
        upload(&v, load(dir, "v.bin", nk * 2), nk * 2) || upload(&qd, load(dir, "qdec.bin", nd * 2), nd * 2) ||
        upload((void **)&lens, host_lens, sizeof host_lens)) {
        fprintf(stderr, "upload\n");
        return 1;
    }
    CK(cudaMalloc(&out, nq * 2));
    CK(cudaMalloc(&dec, nd * 2));
    CK(cudaMalloc((void **)&kc, nk));
    CK(cudaMalloc((void **)&vc, nk));
    CK(cudaMalloc((void **)&ks, rows * 4));
    CK(cudaMalloc((void **)&vs, rows * 4));

    /* bf16 prefill, causal, epilogue [Mul(2), Add(0.5)] */
    fa_fwd_params p;
    memset(&p, 0, sizeof p);
    p.q = q; p.k = k; p.v = v; p.out = out;
    p.q_dtype = FA_BF16; p.kv_dtype = FA_BF16;
    p.batch = B; p.hq = HQ; p.hkv = HKV; p.head_dim = D;
    p.seqlen_q = SQ; p.seqlen_k = SK;
    p.causal = 1;
    p.softmax_scale = 1.0f / sqrtf((float)D);
    p.n_epilogue = 2;
    p.epilogue[0].op = FA_EPI_MUL; p.epilogue[0].value = 2.0f;
    p.epilogue[1].op = FA_EPI_ADD; p.epilogue[1].value = 0.5f;
    FK(fa_attention_fwd(&p, 0));
    CK(cudaDeviceSynchronize());
    if (download(dir, "out_bf16.bin", out, nq * 2)) return 1;

    /* the int8 cache: codes and one scale per (token, KV head) */
    FK(fa_compress_kv(k, FA_BF16, (int64_t)rows, D, kc, ks, 0));
    FK(fa_compress_kv(v, FA_BF16, (int64_t)rows, D, vc, vs, 0));

    /* the same prefill over the int8 cache */
    p.k = kc; p.v = vc; p.kv_dtype = FA_I8; p.k_scales = ks; p.v_scales = vs;
    FK(fa_attention_fwd(&p, 0));
    CK(cudaDeviceSynchronize());
    if (download(dir, "out_i8.bin", out, nq * 2)) return 1;

    /* one decode step per sequence over the int8 cache */
    fa_decode_params dp;
    memset(&dp, 0, sizeof dp);
    dp.q = qd; dp.k_cache = kc; dp.v_cache = vc; dp.k_scales = ks; dp.v_scales = vs;
    dp.cache_seqlens = lens; dp.out = dec; dp.kv_dtype = FA_I8;
    dp.batch = B; dp.hq = HQ; dp.hkv = HKV; dp.head_dim = D; dp.capacity = SK;
    dp.softmax_scale = 1.0f / sqrtf((float)D);
    dp.workspace_bytes = fa_decode_workspace_size(B, HQ, SK, D);
    CK(cudaMalloc(&ws, dp.workspace_bytes));
    dp.workspace = ws;
    FK(fa_attention_decode(&dp, 0));
    CK(cudaDeviceSynchronize());
    FK(fa_check_device_error(0));
    if (download(dir, "out_dec.bin", dec, nd * 2) || download(dir, "kc.bin", kc, nk) ||
        download(dir, "vc.bin", vc, nk) || download(dir, "ks.bin", ks, rows * 4) ||
        download(dir, "vs.bin", vs, rows * 4))
        return 1;
    cudaFree(q); cudaFree(k); cudaFree(v); cudaFree(qd); cudaFree(out); cudaFree(dec);
    cudaFree(kc); cudaFree(vc); cudaFree(ks); cudaFree(vs); cudaFree(lens); cudaFree(ws);
    printf("c gpu abi ok\n");
    return 0;
}
""" % dict(B=B, HQ=HQ, HKV=HKV, D=D, SQ=SQ, SK=SK, L0=LENS[0], L1=LENS[1])


def _bf16_bytes(t: torch.Tensor) -> bytes:
    return t.contiguous().view(torch.int16).numpy().tobytes()


def _bf16_from(path, shape) -> np.ndarray:
    raw = np.fromfile(path, dtype=np.int16).reshape(shape)
    return torch.from_numpy(raw).view(torch.bfloat16).float().numpy()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_runs_prefill_and_decode_on_host_buffers(tmp_path):
    from flashattention_attention_b200 import build
    lib = build.build()
    w = inputs.dense_prefill("c-abi", batch=B, hq=HQ, hkv=HKV, s_q=SQ, s_k=SK, d=D, dtype=torch.bfloat16,
                             causal=True, seed=71)
    q_dec = inputs.normal(np.random.default_rng(72), (B * HQ, D), torch.bfloat16)
    for name, t in (("q.bin", w.q), ("k.bin", w.k), ("v.bin", w.v), ("qdec.bin", q_dec)):
        (tmp_path / name).write_bytes(_bf16_bytes(t))
    src = tmp_path / "abi_gpu.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi_gpu"
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), str(src), "-o", str(exe),
           "-L", os.path.dirname(lib), "-lfa", "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + os.path.dirname(lib), "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe), str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "c gpu abi ok" in r.stdout, r.stdout + r.stderr

    epi = [("mul", 2.0), ("add", 0.5)]
    got = _bf16_from(tmp_path / "out_bf16.bin", (B * HQ, SQ, D))
    ref = oracle.attention(w.q, w.k, w.v, hq=HQ, hkv=HKV, causal=True, epilogue=epi)
    assert_close_bf16(got, ref, what="C program: bf16 prefill")

    rk, rks = oracle.compress_kv(w.k)
    rv, rvs = oracle.compress_kv(w.v)
    kc = np.fromfile(tmp_path / "kc.bin", dtype=np.int8).reshape(rk.shape)
    vc = np.fromfile(tmp_path / "vc.bin", dtype=np.int8).reshape(rv.shape)
    ks = np.fromfile(tmp_path / "ks.bin", dtype=np.uint32).reshape(rks.shape)
    vs = np.fromfile(tmp_path / "vs.bin", dtype=np.uint32).reshape(rvs.shape)
    assert np.array_equal(kc, rk) and np.array_equal(vc, rv)
    assert np.array_equal(ks, rks.view(np.uint32)) and np.array_equal(vs, rvs.view(np.uint32))

    kd, vd = oracle.dequantize(rk, rks), oracle.dequantize(rv, rvs)
    got = _bf16_from(tmp_path / "out_i8.bin", (B * HQ, SQ, D))
    ref = oracle.attention(w.q, kd, vd, hq=HQ, hkv=HKV, causal=True, epilogue=epi)
    assert_close_bf16(got, ref, what="C program: int8 prefill")

    got = _bf16_from(tmp_path / "out_dec.bin", (B * HQ, D))
    ref = oracle.decode(q_dec.reshape(B * HQ, 1, D), kd, vd, np.array(LENS), hq=HQ, hkv=HKV)
    assert_close_bf16(got, ref.reshape(B * HQ, D), what="C program: int8 decode")
