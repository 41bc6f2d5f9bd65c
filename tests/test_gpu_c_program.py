"""A plain C99 program drives a whole prefill through the C ABI: it reads
Q, K, V from files into page-locked buffers (cudaMallocHost), sizes and
allocates the device workspace itself, calls crisp_prefill_host and writes O,
the log-sum-exp and the routes back to files. Its output must match the
device-resident path (crisp_route + crisp_select + crisp_sparse_prefill)
within the attention tolerance of the parity tests."""
import os
import subprocess

import numpy as np
import pytest
import torch

from synthetic import Workload, make_qkv

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"

PROGRAM = r'''
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime_api.h>
#include "crisp.h"

static int load(const char* dir, const char* name, void* dst, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) return -1;
  size_t got = fread(dst, 1, bytes, f);
  fclose(f);
  return got == bytes ? 0 : -1;
}

static int save(const char* dir, const char* name, const void* src, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f) return -1;
  size_t put = fwrite(src, 1, bytes, f);
  fclose(f);
  return put == bytes ? 0 : -1;
}

int main(int argc, char** argv) {
  if (argc != 8) return 2;
  const char* dir = argv[1];
  crisp_params p = {.batch = atoi(argv[2]), .h_q = atoi(argv[3]), .h_kv = atoi(argv[4]),
                    .seqlen = atoi(argv[5]), .head_dim = atoi(argv[6]), .block = atoi(argv[7]),
                    .alpha = 1.0f, .gamma = 0.95f, .tau_proxy = 0.2f, .tau_jsd = 0.1f,
                    .k_min_blocks = 8, .router = CRISP_ROUTER_CSTRUCT, .vs_rule = CRISP_VS_ALPHA,
                    .sm_scale = 0.0f, .vs_granularity = CRISP_GRAN_TILE, .seq_lens = NULL};
  const size_t rows_q = (size_t)p.batch * p.h_q * p.seqlen, rows_kv = (size_t)p.batch * p.h_kv * p.seqlen;
  const size_t row = (size_t)p.head_dim * 2;
  void *q, *k, *v, *o;
  float* lse;
  int32_t* pattern = (int32_t*)malloc((size_t)p.batch * p.h_q * 4);
  if (cudaMallocHost(&q, rows_q * row) || cudaMallocHost(&k, rows_kv * row) || cudaMallocHost(&v, rows_kv * row) ||
      cudaMallocHost(&o, rows_q * row) || cudaMallocHost((void**)&lse, rows_q * 4))
    return 3;
  if (load(dir, "q.bin", q, rows_q * row) || load(dir, "k.bin", k, rows_kv * row) || load(dir, "v.bin", v, rows_kv * row))
    return 4;
  const int kv_per_chunk = 1;
  size_t dws = crisp_prefill_host_workspace_size(&p, kv_per_chunk);
  void* ws = NULL;
  if (dws == 0 || cudaMalloc(&ws, dws)) return 5;
  int rc = crisp_prefill_host(&p, q, k, v, o, lse, NULL, pattern, kv_per_chunk, ws, dws, NULL);
  printf("%d %s\n", rc, crisp_status_string(rc));
  if (rc == CRISP_OK &&
      (save(dir, "o.bin", o, rows_q * row) || save(dir, "lse.bin", lse, rows_q * 4) ||
       save(dir, "pattern.bin", pattern, (size_t)p.batch * p.h_q * 4)))
    return 6;
  cudaFree(ws);
  cudaFreeHost(q); cudaFreeHost(k); cudaFreeHost(v); cudaFreeHost(o); cudaFreeHost(lse);
  free(pattern);
  return rc == CRISP_OK ? 0 : 7;
}
'''


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_block_sparse_qk_b200 import build
    build.build()


def test_c_program_runs_a_prefill_from_host_buffers(tmp_path):
    import dynamic_block_sparse_qk_b200 as C
    w = Workload("cprog", 2, 8, 2, 128, 4096, 128, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    q, k, v, _ = make_qkv(w)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        t.contiguous().view(torch.int16).numpy().tofile(str(tmp_path / f"{nm}.bin"))
    src = tmp_path / "prefill.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "prefill"
    pkg = os.path.join(ROOT, "dynamic_block_sparse_qk_b200")
    subprocess.run(["gcc", "-std=c99", "-O2", "-I", os.path.join(ROOT, "include"), "-I", CUDA + "/include",
                    str(src), "-o", str(exe), "-L", pkg, "-lcrisp", "-Wl,-rpath," + pkg,
                    "-L", CUDA + "/lib64", "-lcudart", "-Wl,-rpath," + CUDA + "/lib64"], check=True)
    proc = subprocess.run([str(exe), str(tmp_path), str(w.batch), str(w.h_q), str(w.h_kv), str(w.seqlen),
                           str(w.head_dim), str(w.block)], capture_output=True, text=True, timeout=300)
    assert proc.returncode == 0, (proc.returncode, proc.stdout, proc.stderr)
    assert proc.stdout.split()[0] == "0"
    o = torch.from_numpy(np.fromfile(str(tmp_path / "o.bin"), dtype=np.int16)).view(torch.bfloat16).view(q.shape)
    lse = torch.from_numpy(np.fromfile(str(tmp_path / "lse.bin"), dtype=np.float32)).view(q.shape[:3])
    pattern = torch.from_numpy(np.fromfile(str(tmp_path / "pattern.bin"), dtype=np.int32))
    ref = C.crisp_prefill(q.cuda(), k.cuda(), v.cuda(), block=w.block)
    assert torch.equal(pattern, ref["pattern"].cpu())
    err = (o.float() - ref["o"].cpu().float()).abs()
    assert float(err.max()) <= 2e-2 and float(err.mean()) <= 2e-3
    assert torch.allclose(lse, ref["lse"].cpu(), atol=2e-3, rtol=0)
