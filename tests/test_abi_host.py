"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/crisp.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from dynamic_block_sparse_qk_b200 import binding as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "crisp.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(crisp_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from dynamic_block_sparse_qk_b200 import build
    build.build()
    return B.load_library()


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert set(names) == set(B.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.crisp_version() == 10200
    assert lib.crisp_status_string(0) == b"ok"
    assert lib.crisp_status_string(-3) == b"workspace too small"


def _p(**kw):
    base = dict(batch=1, h_q=32, h_kv=8, seqlen=32768, head_dim=128, block=128)
    base.update(kw)
    return B.make_params(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(h_q=30), -2), (dict(head_dim=96), -2), (dict(block=32), -2), (dict(seqlen=0), -2),
    (dict(seqlen=256), -2), (dict(block=64, seqlen=128), -2), (dict(seqlen=2 ** 21), -2), (dict(block=64, seqlen=2 ** 19), -2),
    (dict(alpha=0.0), -1), (dict(gamma=1.5), -1), (dict(gamma=0.0), -1), (dict(k_min_blocks=0), -1),
    (dict(router=7), -1), (dict(vs_rule=3), -1), (dict(sm_scale=-1.0), -1), (dict(batch=0), -2),
    (dict(h_q=32, h_kv=0), -2),
    # batch * h_q * seqlen = 2^31 query rows: beyond 32-bit tile coordinates
    (dict(batch=64, h_q=64, h_kv=8, seqlen=2 ** 19), -2),
    (dict(granularity=2), -1), (dict(granularity="token", block=64, seqlen=4096), -2),
])
def test_check_params_rejects(lib, kw, code):
    p = _p(**kw)
    assert lib.crisp_check_params(ctypes.byref(p)) == code
    assert lib.crisp_workspace_size(ctypes.byref(p)) == 0


def test_valid_configs_have_workspace(lib):
    for kw in (dict(), dict(batch=1, h_q=2, h_kv=1, seqlen=2048, head_dim=64, block=64),
               dict(h_q=28, h_kv=4, seqlen=131072), dict(seqlen=524288),
               dict(batch=63, h_q=64, h_kv=8, seqlen=2 ** 19),
               dict(seqlen=257), dict(seqlen=1000), dict(block=64, seqlen=129), dict(seqlen=32768 + 37),
               dict(granularity="token")):
        p = _p(**kw)
        assert lib.crisp_check_params(ctypes.byref(p)) == 0
        assert lib.crisp_workspace_size(ctypes.byref(p)) > 0


def test_entry_points_validate_before_launch(lib):
    p = _p()
    fake = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
    need = lib.crisp_workspace_size(ctypes.byref(p))
    # null / misaligned workspace, too-small workspace, null tensors
    assert lib.crisp_route(ctypes.byref(p), fake, fake, None, need, fake, fake, fake, fake, None) == -1
    assert lib.crisp_route(ctypes.byref(p), fake, fake, ctypes.c_void_p((1 << 20) + 8), need,
                           fake, fake, fake, fake, None) == -1
    assert lib.crisp_route(ctypes.byref(p), fake, fake, fake, need - 1, fake, fake, fake, fake, None) == -3
    assert lib.crisp_route(ctypes.byref(p), None, fake, fake, need, fake, fake, fake, fake, None) == -1
    assert lib.crisp_route(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 2), fake, fake, need, fake,
                           fake, fake, fake, None) == -1
    assert lib.crisp_select(ctypes.byref(p), fake, fake, fake, fake, fake, fake, need, None, None,
                            None, fake, None) == -1
    assert lib.crisp_sparse_prefill(ctypes.byref(p), fake, fake, fake, fake, fake, None, None,
                                    fake, need, None) == -1
    assert lib.crisp_dense_prefill(ctypes.byref(p), fake, fake, None, fake, None, fake, need, None) == -1
    bad = _p(block=96)
    assert lib.crisp_dense_prefill(ctypes.byref(bad), fake, fake, fake, fake, None, fake, need, None) == -2
    st = ctypes.c_int32(0)
    assert lib.crisp_get_device_status(fake, None, None) == -1
    assert lib.crisp_get_device_status(ctypes.c_void_p((1 << 20) + 8), ctypes.byref(st), None) == -1
    assert lib.crisp_selftest_pipeline_timeout(ctypes.byref(p), fake, fake, fake, fake, fake, need, 0, None) == -1
    assert lib.crisp_selftest_pipeline_timeout(ctypes.byref(p), fake, fake, fake, fake, fake, need, 1 << 20,
                                               None) == -1
    assert lib.crisp_selftest_pipeline_timeout(ctypes.byref(p), fake, fake, fake, None, fake, need, 64, None) == -1
    assert lib.crisp_selftest_pipeline_timeout(ctypes.byref(p), fake, fake, fake, fake, fake, need - 1, 64,
                                               None) == -3


def test_host_prefill_validates_before_any_copy(lib):
    p = _p(seqlen=4096)
    fake = ctypes.c_void_p(1 << 20)
    need = lib.crisp_prefill_host_workspace_size(ctypes.byref(p), 1)
    assert need > 0
    assert lib.crisp_prefill_host_workspace_size(ctypes.byref(p), 3) == 0        # 3 does not divide h_kv = 8
    assert lib.crisp_prefill_host_workspace_size(ctypes.byref(p), 0) == 0
    assert lib.crisp_prefill_host_workspace_size(ctypes.byref(p), 2) > need     # bigger chunks, bigger slots
    assert lib.crisp_prefill_host(ctypes.byref(p), None, fake, fake, fake, None, None, None, 1, fake, need,
                                  None) == -1
    assert lib.crisp_prefill_host(ctypes.byref(p), fake, fake, fake, fake, None, None, None, 1, fake, need - 1,
                                  None) == -3
    assert lib.crisp_prefill_host(ctypes.byref(p), fake, fake, fake, fake, None, None, None, 1,
                                  ctypes.c_void_p((1 << 20) + 8), need, None) == -1
    withlens = _p(seqlen=4096)
    withlens.seq_lens = ctypes.c_void_p(1 << 20)                # device lengths are not taken here
    assert lib.crisp_prefill_host(ctypes.byref(withlens), fake, fake, fake, fake, None, None, None, 1, fake,
                                  need, None) == -1


def test_selftest_validates_before_launch(lib):
    fake = ctypes.c_void_p(1 << 20)                       # aligned, never dereferenced on failure
    assert lib.crisp_selftest_wait_timeout(None, 1000, None) == -1
    assert lib.crisp_selftest_wait_timeout(ctypes.c_void_p((1 << 20) + 8), 1000, None) == -1
    assert lib.crisp_selftest_wait_timeout(fake, 0, None) == -1
    assert lib.crisp_selftest_wait_timeout(fake, (1 << 31) + 1, None) == -1


def test_params_struct_layout_matches_header(lib, tmp_path):
    # 10 int32 + 4 float fields, then the 8-byte seq_lens pointer; the C
    # compiler's view of include/crisp.h must agree with the ctypes mirror
    assert ctypes.sizeof(B.CrispParams) == 15 * 4 + 4 + 8        # 4 bytes of padding before the pointer
    assert B.CrispParams.seq_lens.offset == 64
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "crisp.h"\n'
        'int main(void) { printf("%zu %zu %zu %zu\\n", sizeof(crisp_params),'
        ' offsetof(crisp_params, seq_lens), offsetof(crisp_params, sm_scale),'
        ' offsetof(crisp_params, vs_granularity)); return 0; }\n')
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c99", "-I", inc, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert [int(x) for x in out] == [ctypes.sizeof(B.CrispParams), B.CrispParams.seq_lens.offset,
                                     B.CrispParams.sm_scale.offset, B.CrispParams.vs_granularity.offset]


def test_binding_rejects_host_lengths_and_bad_enums():
    import torch
    with pytest.raises(ValueError):
        B.make_params(2, 4, 2, 4096, 128, seq_lens=torch.tensor([4096, 100], dtype=torch.int32))
    with pytest.raises(KeyError):
        B.make_params(1, 4, 2, 4096, 128, vs_rule="median")
    p = B.make_params(1, 4, 2, 4096, 128, granularity="token", vs_rule="alpha_median", router="jsd")
    assert (p.vs_granularity, p.vs_rule, p.router) == (1, 2, 1)


def test_c_program_links_and_calls_the_library(lib, tmp_path):
    # a plain C99 program, linked against libcrisp.so, makes the host-side
    # calls of the C example (no device work): version, validation, workspace
    # size, status strings, and an entry point refusing NULL pointers
    src = tmp_path / "use.c"
    src.write_text(r'''
#include <stdio.h>
#include "crisp.h"
int main(void) {
  crisp_params p = {.batch = 1, .h_q = 32, .h_kv = 8, .seqlen = 524288, .head_dim = 128,
                    .block = 128, .alpha = 1.0f, .gamma = 0.95f, .tau_proxy = 0.2f,
                    .tau_jsd = 0.1f, .k_min_blocks = 8, .router = CRISP_ROUTER_CSTRUCT,
                    .vs_rule = CRISP_VS_ALPHA, .sm_scale = 0.0f,
                    .vs_granularity = CRISP_GRAN_TILE, .seq_lens = NULL};
  int ok = crisp_check_params(&p);
  size_t ws = crisp_workspace_size(&p);
  int route = crisp_route(&p, NULL, NULL, NULL, ws, NULL, NULL, NULL, NULL, NULL);
  p.seqlen = 2 * 128;                      /* N_b = 2: below the minimum of 3 blocks */
  printf("%d %d %zu %d %d %zu|%s|%s\n", crisp_version(), ok, ws, route, crisp_check_params(&p),
         crisp_workspace_size(&p), crisp_status_string(CRISP_OK), crisp_status_string(CRISP_ERR_SHAPE));
  return 0;
}
''')
    exe = tmp_path / "use"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "dynamic_block_sparse_qk_b200")
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                    "-L", pkg, "-lcrisp", "-Wl,-rpath," + pkg], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    nums, ok_name, shape_name = out.split("|")
    version, ok, ws, route, bad, ws_bad = (int(x) for x in nums.split())
    p = B.make_params(1, 32, 8, 524288, 128)
    assert version == lib.crisp_version()
    assert ok == 0 and ws == B.crisp_workspace_size(p) > 0
    assert route == -1                                     # CRISP_ERR_ARG, nothing launched
    assert bad == -2 and ws_bad == 0                       # CRISP_ERR_SHAPE
    lib.crisp_status_string.restype = ctypes.c_char_p
    assert ok_name == lib.crisp_status_string(0).decode()
    assert shape_name == lib.crisp_status_string(-2).decode()


def test_host_input_prefill_rejects_unpinned_tensors():
    # prefill_from_host copies from page-locked memory only; a pageable (or
    # device) tensor is refused before any stream, workspace or copy exists
    import torch
    from dynamic_block_sparse_qk_b200 import prefill_from_host
    q = torch.zeros(1, 4, 1024, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 1024, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="pinned host memory"):
        prefill_from_host(q, k, k.clone(), torch.empty_like(q), block=64)
